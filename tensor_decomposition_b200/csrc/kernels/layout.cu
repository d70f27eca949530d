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
// Batch i = blockIdx.y; with vec (per a multiple of 4, 16-byte aligned arrays) four entries per
// thread (16-byte loads, four partials in flight), one otherwise.
__global__ void k_sum_heads(int H, int64_t per, bool vec, const float* part, float* out32, double* out64) {
  const int64_t i = blockIdx.y;
  const float* src = part + i * H * per;
  if (vec) {
    const int64_t per4 = per / 4;
    const float4* s4 = reinterpret_cast<const float4*>(src);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < per4; e += (int64_t)gridDim.x * blockDim.x) {
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      int h = 0;
      for (; h + 4 <= H; h += 4) {
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = s4[(int64_t)(h + k) * per4 + e];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          a0 += (double)v[k].x;
          a1 += (double)v[k].y;
          a2 += (double)v[k].z;
          a3 += (double)v[k].w;
        }
      }
      for (; h < H; ++h) {
        const float4 v = s4[(int64_t)h * per4 + e];
        a0 += (double)v.x;
        a1 += (double)v.y;
        a2 += (double)v.z;
        a3 += (double)v.w;
      }
      const int64_t o = i * per + 4 * e;
      if (out32) *reinterpret_cast<float4*>(out32 + o) = make_float4((float)a0, (float)a1, (float)a2, (float)a3);
      if (out64) {
        *reinterpret_cast<double2*>(out64 + o) = make_double2(a0, a1);
        *reinterpret_cast<double2*>(out64 + o + 2) = make_double2(a2, a3);
      }
    }
  } else {
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < per; e += (int64_t)gridDim.x * blockDim.x) {
      double a = 0.0;
      for (int h = 0; h < H; ++h) a += (double)src[(int64_t)h * per + e];
      if (out32) out32[i * per + e] = (float)a;
      if (out64) out64[i * per + e] = a;
    }
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
  if (n <= 0 || per <= 0) return cudaSuccess;
  if (n > 65535) return cudaErrorInvalidValue;
  // 16-byte vectors need a multiple of 4 entries and aligned arrays; otherwise the scalar path
  const bool vec = per % 4 == 0 && (reinterpret_cast<uintptr_t>(part) | reinterpret_cast<uintptr_t>(out32) |
                                    reinterpret_cast<uintptr_t>(out64)) % 16 == 0;
  int64_t bx = ((vec ? per / 4 : per) + 255) / 256;
  if (bx > 1024) bx = 1024;
  k_sum_heads<<<dim3((unsigned)bx, (unsigned)n), 256, 0, s>>>(H, per, vec, part, out32, out64);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
