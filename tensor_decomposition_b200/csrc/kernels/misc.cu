// Small helper kernels: storage rounding, float64 norms (the relative Frobenius error the
// JoLT abstract reports, arXiv 2607.12550v2), the factor column sign rule and the
// non-finite input check. Reductions use a fixed grid and a fixed tree so results are
// bit-reproducible from run to run.
#include "../jolt_internal.h"

namespace jolt {
namespace {

template <typename T>
__device__ __forceinline__ double ld_as_double(const T* p, int64_t i);
template <>
__device__ __forceinline__ double ld_as_double<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return (double)__bfloat162float(p[i]);
}
template <>
__device__ __forceinline__ double ld_as_double<float>(const float* p, int64_t i) {
  return (double)p[i];
}

__device__ __forceinline__ double block_sum(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
  __syncthreads();
  return t;
}

__global__ void k_round_bf16(int64_t n, const float* in, __nv_bfloat16* ob, float* of) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const __nv_bfloat16 b = __float2bfloat16_rn(in[i]);
    if (ob) ob[i] = b;
    if (of) of[i] = __bfloat162float(b);
  }
}

constexpr int kSumBlocks = 64;

// 16-byte vector of 8 bf16 or 4 float values, widened to double.
template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, int64_t i, double* out) {
    const uint4 u = *reinterpret_cast<const uint4*>(p + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      out[2 * k] = (double)__uint_as_float(w[k] << 16);
      out[2 * k + 1] = (double)__uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, int64_t i, double* out) {
    const float4 f = *reinterpret_cast<const float4*>(p + i);
    out[0] = f.x; out[1] = f.y; out[2] = f.z; out[3] = f.w;
  }
};

// Squared norms, vectorised when the array and its length allow 16-byte loads.
template <typename T>
__global__ void k_sumsq_part(int64_t n, const T* x, int64_t stride, double* part) {
  __shared__ double red[32];
  const T* p = x + (int64_t)blockIdx.y * stride;
  constexpr int V = Vec16<T>::N;
  double acc = 0.0;
  const bool vec = (reinterpret_cast<uintptr_t>(p) % 16 == 0);
  const int64_t nv = vec ? n / V : 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nv; i += (int64_t)gridDim.x * blockDim.x) {
    double v[V];
    Vec16<T>::load(p, i * V, v);
#pragma unroll
    for (int k = 0; k < V; ++k) acc = fma(v[k], v[k], acc);
  }
  for (int64_t i = nv * V + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const double v = ld_as_double(p, i);
    acc = fma(v, v, acc);
  }
  const double t = block_sum(acc, red);
  if (threadIdx.x == 0) part[blockIdx.y * gridDim.x + blockIdx.x] = t;
}

// A non-finite input makes its squared norm non-finite (bf16 / float32 squares cannot
// overflow float64), so the norm pass doubles as the NaN / Inf check.
__global__ void k_sum_rows(int rows, int cols, const double* part, double* out, int32_t* status) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  double t = 0.0;
  for (int c = 0; c < cols; ++c) t += part[(int64_t)r * cols + c];
  out[r] = t;
  if (status && !isfinite(t)) atomicOr(status, ST_NONFINITE);
}

template <typename T>
__global__ void k_relfrob_part(uint64_t n, const T* a, const T* b, double* part) {
  __shared__ double red[32];
  constexpr int V = Vec16<T>::N;
  double sd = 0.0, sr = 0.0;
  const bool vec = (reinterpret_cast<uintptr_t>(a) % 16 == 0) && (reinterpret_cast<uintptr_t>(b) % 16 == 0);
  const int64_t nv = vec ? (int64_t)(n / V) : 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nv; i += (int64_t)gridDim.x * blockDim.x) {
    double x[V], y[V];
    Vec16<T>::load(a, i * V, x);
    Vec16<T>::load(b, i * V, y);
#pragma unroll
    for (int k = 0; k < V; ++k) {
      const double d = x[k] - y[k];
      sd = fma(d, d, sd);
      sr = fma(x[k], x[k], sr);
    }
  }
  for (int64_t i = nv * V + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const double x = ld_as_double(a, i), y = ld_as_double(b, i);
    sd = fma(x - y, x - y, sd);
    sr = fma(x, x, sr);
  }
  const double td = block_sum(sd, red);
  const double tr = block_sum(sr, red);
  if (threadIdx.x == 0) {
    part[2 * blockIdx.x] = td;
    part[2 * blockIdx.x + 1] = tr;
  }
}

// Sum of the per-block partials: one block, each thread a fixed strided subset, then the
// fixed block tree (deterministic).
__global__ void k_relfrob_final(int nb, const double* part, double* out2) {
  __shared__ double red[32];
  double d = 0.0, r = 0.0;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    d += part[2 * i];
    r += part[2 * i + 1];
  }
  const double td = block_sum(d, red);
  const double tr = block_sum(r, red);
  if (threadIdx.x == 0) {
    out2[0] = td;
    out2[1] = tr;
  }
}

// Sign rule per column: the entry of largest magnitude (first on ties) becomes positive.
// Block = 32 columns x kSignLanes row lanes (a warp reads 128 contiguous bytes of a row); the
// same block then flips U's and W's columns.
constexpr int kSignLanes = 32;
__global__ void __launch_bounds__(32 * kSignLanes) k_sign_fix(int rows, int cols, float* U, int64_t ldu, int64_t sU,
                                                             float* W, int w_rows, int64_t ldw, int64_t sW) {
  constexpr int RL = kSignLanes;
  __shared__ float bv[RL][32];
  __shared__ int bi[RL][32];
  __shared__ float sgn[32];
  const int cx = threadIdx.x & 31, ry = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + cx;
  float* u = U + (int64_t)blockIdx.y * sU;
  float best = -1.0f;
  int bidx = 0x7fffffff;
  if (c < cols) {
    // rows visited in increasing order (first wins ties), four loads in flight per thread
    int r = ry;
    for (; r + 3 * RL < rows; r += 4 * RL) {
      float a[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) a[k] = fabsf(u[(int64_t)(r + RL * k) * ldu + c]);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (a[k] > best) { best = a[k]; bidx = r + RL * k; }
    }
    for (; r < rows; r += RL) {
      const float a = fabsf(u[(int64_t)r * ldu + c]);
      if (a > best) { best = a; bidx = r; }
    }
  }
  bv[ry][cx] = best;
  bi[ry][cx] = bidx;
  __syncthreads();
  if (ry == 0) {
    for (int k = 1; k < RL; ++k) {
      const float v = bv[k][cx];
      const int i = bi[k][cx];
      if (v > best || (v == best && i < bidx)) { best = v; bidx = i; }
    }
    float sg = 1.0f;
    if (c < cols && bidx < rows && u[(int64_t)bidx * ldu + c] < 0.0f) sg = -1.0f;
    sgn[cx] = sg;
  }
  __syncthreads();
  if (c >= cols) return;
  const float sg = sgn[cx];
  if (sg > 0.0f) return;
#pragma unroll 4
  for (int r = ry; r < rows; r += RL) u[(int64_t)r * ldu + c] = -u[(int64_t)r * ldu + c];
  if (W) {
    float* w = W + (int64_t)blockIdx.y * sW;
#pragma unroll 4
    for (int r = ry; r < w_rows; r += RL) w[(int64_t)r * ldw + c] = -w[(int64_t)r * ldw + c];
  }
}

__global__ void k_check_finite_bf16(int64_t n, const __nv_bfloat16* x, int32_t* status) {
  bool bad = false;
  const uint16_t* u = reinterpret_cast<const uint16_t*>(x);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    bad |= ((u[i] & 0x7F80u) == 0x7F80u);
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, ST_NONFINITE);
}

__global__ void k_check_finite_f32(int64_t n, const float* x, int32_t* status) {
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    bad |= !isfinite(x[i]);
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, ST_NONFINITE);
}

}  // namespace

cudaError_t round_bf16(int64_t n, const float* in, __nv_bfloat16* ob, float* of, cudaStream_t s) {
  int b = (int)((n + 255) / 256);
  if (b > 1184) b = 1184;
  if (b < 1) b = 1;
  k_round_bf16<<<b, 256, 0, s>>>(n, in, ob, of);
  note_launch();
  return cudaGetLastError();
}

cudaError_t sumsq_batched(int batch, int64_t n, const void* x, ElemType t, int64_t stride,
                          double* out, double* part, int32_t* status, cudaStream_t s) {
  dim3 g(kSumBlocks, batch);
  if (t == EL_BF16)
    k_sumsq_part<__nv_bfloat16><<<g, 256, 0, s>>>(n, (const __nv_bfloat16*)x, stride, part);
  else
    k_sumsq_part<float><<<g, 256, 0, s>>>(n, (const float*)x, stride, part);
  note_launch();
  k_sum_rows<<<(batch + 127) / 128, 128, 0, s>>>(batch, kSumBlocks, part, out, status);
  note_launch();
  return cudaGetLastError();
}

// Fixed device scratch of the allocation-free relative-error entry point: the per-block
// partial sums (2 per block, up to kRelfrobStaticBlocks blocks) followed by the two totals.
// One array per device, shared by every caller of that entry point: concurrent calls race.
static __device__ __align__(256) double g_relfrob_scratch[2 * kRelfrobStaticBlocks + 2];

cudaError_t relfrob_static_scratch(double** p) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(p), g_relfrob_scratch);
}

int relfrob_blocks(uint64_t n) {
  uint64_t b = (n + 2047) / 2048;
  if (b > 1184) b = 1184;
  if (b < 1) b = 1;
  return (int)b;
}

cudaError_t relfrob_partial(const void* ref, const void* approx, uint64_t n, ElemType t,
                            double* partials, int nblocks, double* out2, cudaStream_t s) {
  if (t == EL_BF16)
    k_relfrob_part<__nv_bfloat16><<<nblocks, 256, 0, s>>>(n, (const __nv_bfloat16*)ref,
                                                          (const __nv_bfloat16*)approx, partials);
  else
    k_relfrob_part<float><<<nblocks, 256, 0, s>>>(n, (const float*)ref, (const float*)approx,
                                                  partials);
  note_launch();
  k_relfrob_final<<<1, 256, 0, s>>>(nblocks, partials, out2);
  note_launch();
  return cudaGetLastError();
}

cudaError_t sign_fix(int batch, int rows, int cols, float* U, int64_t ldu, int64_t sU, float* W,
                     int w_rows, int64_t ldw, int64_t sW, cudaStream_t s) {
  dim3 g((cols + 31) / 32, batch);
  k_sign_fix<<<g, 32 * kSignLanes, 0, s>>>(rows, cols, U, ldu, sU, W, w_rows, ldw, sW);
  note_launch();
  return cudaGetLastError();
}

cudaError_t check_finite(int64_t n, const void* x, ElemType t, int32_t* status, cudaStream_t s) {
  int b = (int)((n + 255) / 256);
  if (b > 2368) b = 2368;
  if (b < 1) b = 1;
  if (t == EL_BF16)
    k_check_finite_bf16<<<b, 256, 0, s>>>(n, (const __nv_bfloat16*)x, status);
  else
    k_check_finite_f32<<<b, 256, 0, s>>>(n, (const float*)x, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
