// Fused decode of the JoLT codec: unpack, dequantise, inverse-rotate, add the Tucker part
// and store, one pass per row.
//
// "A JoLT for the KV Cache" (arXiv 2607.12550v2, Abstract) reconstructs the cache from the
// partial Tucker factors plus the rotated low-bit residual. For row t of head h:
//     x_hat = u_t M_h + y_hat Pi^T,   M_h = G_h U_D^T (r_t x D),
//     y_hat_i = s (2 c_i + 1 - 2^b) / 2^b      (mid-rise cell centres),
// with u_t = U_T[t, :r_t] and the row's fp16 scale s and b-bit codes c. Arithmetic is
// float32 (the stored parts are bf16 / fp16 / small integers, so every product is exact);
// the output is rounded to nearest even into bf16, or stored as float32.
#include "../jolt_internal.h"

namespace jolt {
namespace {

constexpr int kRowsPerWarp = 4;
constexpr int kWarps = 8;
constexpr int kChunk = 1024;   // tokens per CTA (M_h is built once per CTA)

__global__ void __launch_bounds__(256) k_decode(DecodeArgs a) {
  extern __shared__ unsigned char smraw[];
  const int chunk = blockIdx.x, h = blockIdx.y, i = blockIdx.z;
  const int lt = a.lt_ids[i];
  const StreamMeta* m = a.meta;
  const int rt = m->lt_rank[lt][0], rd = m->lt_rank[lt][1], b = m->lt_rank[lt][2];
  const int D = a.D;
  float* M_s = reinterpret_cast<float*>(smraw);        // rt x D
  float* PT = M_s + kMaxN * D;                          // PT[i][d] = Pi[d][i]
  float* work = PT + D * D;                             // G_h (rt x rd) + U_D^T (rd x D), later row staging
  __nv_bfloat16* G_s = reinterpret_cast<__nv_bfloat16*>(work);
  __nv_bfloat16* UDt = G_s + kMaxN * kMaxN;
  const __nv_bfloat16* UT = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UT]);
  const __nv_bfloat16* UD = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UD]);
  const __nv_bfloat16* G = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_G]) +
                           (int64_t)h * rt * rd;
  const __half* scales = reinterpret_cast<const __half*>(a.body + m->off[lt][JOLT_PART_SCALES]);
  const unsigned char* codes = a.body + m->off[lt][JOLT_PART_CODES];
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    PT[c * D + r] = a.Pi[e];
  }
  for (int e = threadIdx.x; e < rt * rd; e += blockDim.x) G_s[e] = G[e];
  for (int e = threadIdx.x; e < D * rd; e += blockDim.x) {
    const int d = e / rd, j = e % rd;
    UDt[j * D + d] = UD[e];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < rt * D; e += blockDim.x) {
    const int k = e / D, d = e % D;
    float acc = 0.0f;
    for (int j = 0; j < rd; ++j)
      acc = fmaf(__bfloat162float(G_s[k * rd + j]), __bfloat162float(UDt[j * D + d]), acc);
    M_s[e] = acc;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* us = work + warp * kRowsPerWarp * 2 * kMaxN;   // [4][128] u rows, then [4][128] y_hat rows
  float* ys = us + kRowsPerWarp * kMaxN;
  const int rowbytes = D * b / 8;
  const float inv2b = 1.0f / (float)(1 << b);
  const float off2b = 1.0f - (float)(1 << b);
  const int t_begin = chunk * kChunk, t_end = min(a.T, t_begin + kChunk);
  const int layer = lt >> 1, kind = lt & 1;
  const int64_t obase = (((int64_t)layer * a.H + h) * a.T) * D;
  for (int t0 = t_begin + warp * kRowsPerWarp; t0 < t_end; t0 += kWarps * kRowsPerWarp) {
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int t = t0 + r;
      const int64_t row = (int64_t)h * a.T + t;
      float sc = 0.0f;
      if (b > 0 && t < t_end) sc = __half2float(scales[row]);
      for (int q = 0; q < 4; ++q) {
        const int d = lane + 32 * q;
        float uv = 0.0f, yv = 0.0f;
        if (t < t_end) {
          if (d < rt) uv = __bfloat162float(UT[(int64_t)t * rt + d]);
          if (b > 0) {
            const int bitpos = d * b;
            const unsigned char* rp = codes + row * rowbytes;
            unsigned int w = rp[bitpos >> 3];
            if ((bitpos >> 3) + 1 < rowbytes) w |= (unsigned int)rp[(bitpos >> 3) + 1] << 8;
            const int c = (int)((w >> (bitpos & 7)) & ((1u << b) - 1u));
            yv = sc * (((float)(2 * c) + off2b) * inv2b);
          }
        }
        us[r * kMaxN + d] = uv;
        ys[r * kMaxN + d] = yv;
      }
    }
    __syncwarp();
    float acc[kRowsPerWarp][4];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[r][q] = 0.0f;
    for (int k = 0; k < rt; ++k) {
      float mv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) mv[q] = M_s[k * D + lane + 32 * q];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        const float uv = us[r * kMaxN + k];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][q] = fmaf(uv, mv[q], acc[r][q]);
      }
    }
    if (b > 0) {
      for (int ii = 0; ii < D; ++ii) {
        float pv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) pv[q] = PT[ii * D + lane + 32 * q];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const float yv = ys[r * kMaxN + ii];
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[r][q] = fmaf(yv, pv[q], acc[r][q]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int t = t0 + r;
      if (t >= t_end) continue;
      const int64_t o = obase + (int64_t)t * D;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int d = lane + 32 * q;
        if (a.ot == EL_BF16)
          reinterpret_cast<__nv_bfloat16*>(a.out[kind])[o + d] = __float2bfloat16_rn(acc[r][q]);
        else
          reinterpret_cast<float*>(a.out[kind])[o + d] = acc[r][q];
      }
    }
    __syncwarp();
  }
}

}  // namespace

cudaError_t decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.D != kD) return cudaErrorInvalidValue;
  const size_t sm = ((size_t)kMaxN * kD + (size_t)kD * kD) * sizeof(float) +
                    2 * (size_t)kMaxN * kMaxN * sizeof(__nv_bfloat16);
  cudaError_t e = cudaFuncSetAttribute(k_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const dim3 g((a.T + kChunk - 1) / kChunk, a.H, a.n_lt);
  k_decode<<<g, kWarps * 32, sm, s>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
