// Layout helpers for the tensor-core path of the factor analysis:
//  * the token-contiguous copy X^T[lt][h][d][t] of every layer-tensor, so that contractions
//    over tokens read K-major tiles (the JoLT token unfolding, "A JoLT for the KV Cache",
//    arXiv 2607.12550v2, Abstract, is contracted over tokens for the sketch passes A^T Q and
//    Q^T A and for the feature Gram);
//  * splitting a float32 array into up to three bf16 parts (x = p0 + p1 + p2 to ~2^-24);
//  * summing per-head float32 Gram partials in float64.
#include "../jolt_internal.h"

namespace jolt {
namespace {

// One 64 x 64 tile of X[l][h] (T x D) -> X^T[base + l][h] (D x T): 16-byte loads of 8
// features, a shared tile, 16-byte stores of 8 tokens. T and D are multiples of 8.
constexpr int kTT = 64, kTS = kTT + 8;   // tile edge, shared row stride (bf16)
__global__ void __launch_bounds__(256) k_transpose_x(const __nv_bfloat16* X, __nv_bfloat16* XT, int H, int T, int D,
                                                     int lt_base) {
  __shared__ __align__(16) __nv_bfloat16 tile[kTT * kTS];
  const int lh = blockIdx.z;                   // l * H + h within this kind
  const int t0 = blockIdx.x * kTT, d0 = blockIdx.y * kTT;
  const __nv_bfloat16* src = X + (int64_t)lh * T * D;
  const int l = lh / H, h = lh % H;
  __nv_bfloat16* dst = XT + ((int64_t)(lt_base + l) * H + h) * D * T;
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    const int q = threadIdx.x + 256 * v, r = q >> 3, c = q & 7;   // token row r, 8-feature chunk c
    const int t = t0 + r, d = d0 + 8 * c;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (t < T && d < D) w = *reinterpret_cast<const uint4*>(src + (int64_t)t * D + d);
    *reinterpret_cast<uint4*>(tile + r * kTS + 8 * c) = w;
  }
  __syncthreads();
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    const int q = threadIdx.x + 256 * v, r = q >> 3, c = q & 7;   // feature row r, 8-token chunk c
    const int d = d0 + r, t = t0 + 8 * c;
    if (d >= D || t >= T) continue;
    __align__(16) __nv_bfloat16 o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = tile[(8 * c + j) * kTS + r];
    *reinterpret_cast<uint4*>(dst + (int64_t)d * T + t) = *reinterpret_cast<const uint4*>(o);
  }
}

__global__ void k_split_bf16(int64_t n, const float* x, __nv_bfloat16* p0, __nv_bfloat16* p1,
                             __nv_bfloat16* p2) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    const __nv_bfloat16 a = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(a);
    const __nv_bfloat16 b = __float2bfloat16_rn(r1);
    p0[i] = a;
    if (p1) p1[i] = b;
    if (p2) p2[i] = __float2bfloat16_rn(r1 - __bfloat162float(b));
  }
}

// Split in[b] (R x C, float32 or float64) into bf16 parts, written in the same layout
// (same[0..2], [b][R][C]) and/or transposed (tr[0..2], [b][C][R]); null outputs are skipped.
template <typename TI>
__global__ void k_split_dual(int R, int C, const TI* in, __nv_bfloat16* s0, __nv_bfloat16* s1, __nv_bfloat16* s2,
                             __nv_bfloat16* t0, __nv_bfloat16* t1, __nv_bfloat16* t2) {
  __shared__ float tile[3][32][33];
  const int b = blockIdx.z;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
  const TI* src = in + (int64_t)b * R * C;
  const int64_t base = (int64_t)b * R * C;
  for (int rr = ty; rr < 32; rr += 8) {
    const int r = r0 + rr, c = c0 + tx;
    float p0 = 0.0f, p1 = 0.0f, p2 = 0.0f;
    if (r < R && c < C) {
      const double v = (double)src[(int64_t)r * C + c];
      const __nv_bfloat16 h0 = __double2bfloat16(v);
      const double r1 = v - (double)__bfloat162float(h0);
      const __nv_bfloat16 h1 = __double2bfloat16(r1);
      const __nv_bfloat16 h2 = __double2bfloat16(r1 - (double)__bfloat162float(h1));
      p0 = __bfloat162float(h0); p1 = __bfloat162float(h1); p2 = __bfloat162float(h2);
      const int64_t o = base + (int64_t)r * C + c;
      if (s0) s0[o] = h0;
      if (s1) s1[o] = h1;
      if (s2) s2[o] = h2;
    }
    tile[0][rr][tx] = p0; tile[1][rr][tx] = p1; tile[2][rr][tx] = p2;
  }
  if (!t0) return;
  __syncthreads();
  for (int cc = ty; cc < 32; cc += 8) {
    const int c = c0 + cc, r = r0 + tx;
    if (r < R && c < C) {
      const int64_t o = base + (int64_t)c * R + r;
      t0[o] = __float2bfloat16_rn(tile[0][tx][cc]);
      if (t1) t1[o] = __float2bfloat16_rn(tile[1][tx][cc]);
      if (t2) t2[o] = __float2bfloat16_rn(tile[2][tx][cc]);
    }
  }
}

// out[i][e] = sum_h part[i][h][e] in float64 (fixed order), stored as float32 and float64.
__global__ void k_sum_heads(int n, int H, int64_t per, const float* part, float* out32, double* out64) {
  const int64_t total = (int64_t)n * per;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / per, r = e % per;
    double s = 0.0;
    for (int h = 0; h < H; ++h) s += (double)part[(i * H + h) * per + r];
    if (out32) out32[e] = (float)s;
    if (out64) out64[e] = s;
  }
}

int grid_for(int64_t n) {
  int64_t b = (n + 255) / 256;
  if (b > 4096) b = 4096;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t transpose_x(const __nv_bfloat16* X, __nv_bfloat16* XT, int L, int H, int T, int D, int lt_base,
                        cudaStream_t s) {
  if (T % 8 || D % 8) return cudaErrorInvalidValue;
  const dim3 g((T + kTT - 1) / kTT, (D + kTT - 1) / kTT, L * H);
  k_transpose_x<<<g, 256, 0, s>>>(X, XT, H, T, D, lt_base);
  note_launch();
  return cudaGetLastError();
}

cudaError_t split_bf16(int64_t n, const float* x, __nv_bfloat16* p0, __nv_bfloat16* p1, __nv_bfloat16* p2,
                       cudaStream_t s) {
  k_split_bf16<<<grid_for(n), 256, 0, s>>>(n, x, p0, p1, p2);
  note_launch();
  return cudaGetLastError();
}

cudaError_t split_dual(int batch, int R, int C, const void* in, bool in_f64, __nv_bfloat16* const* same,
                       __nv_bfloat16* const* tr, cudaStream_t s) {
  const dim3 g((C + 31) / 32, (R + 31) / 32, batch);
  __nv_bfloat16* s0 = same ? same[0] : nullptr;
  __nv_bfloat16* s1 = same ? same[1] : nullptr;
  __nv_bfloat16* s2 = same ? same[2] : nullptr;
  __nv_bfloat16* t0 = tr ? tr[0] : nullptr;
  __nv_bfloat16* t1 = tr ? tr[1] : nullptr;
  __nv_bfloat16* t2 = tr ? tr[2] : nullptr;
  if (in_f64)
    k_split_dual<double><<<g, 256, 0, s>>>(R, C, (const double*)in, s0, s1, s2, t0, t1, t2);
  else
    k_split_dual<float><<<g, 256, 0, s>>>(R, C, (const float*)in, s0, s1, s2, t0, t1, t2);
  note_launch();
  return cudaGetLastError();
}

cudaError_t sum_heads(int n, int H, int64_t per, const float* part, float* out32, double* out64, cudaStream_t s) {
  k_sum_heads<<<grid_for((int64_t)n * per), 256, 0, s>>>(n, H, per, part, out32, out64);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
