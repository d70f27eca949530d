// Layout helpers for the tensor-core path of the factor analysis:
//  * splitting a float32 array into up to three bf16 parts (x = p0 + p1 + p2 to ~2^-24);
//  * summing per-head float32 Gram partials in float64.
#include "../jolt_internal.h"

namespace jolt {
namespace {

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
