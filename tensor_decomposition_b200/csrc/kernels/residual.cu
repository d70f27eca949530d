// Fused residual coding of the JoLT codec: reconstruct, subtract, rotate, row absmax,
// b-bit quantisation and bit packing, in one pass over X.
//
// "A JoLT for the KV Cache" (arXiv 2607.12550v2, Abstract) restores the energy the
// truncation discards "with a rotated low-bit residual: a random orthogonal rotation
// followed by low-bit quantization". For a row x = X[h, t, :] (D features), with the stored
// (bf16) factors and core, the rotated residual is
//     y = (x - u_t G_h U_D^T) Pi = x Pi - u_t N_h,   N_h = (G_h U_D^T) Pi   (r_t x D),
// u_t = U_T[t, :r_t]. Quantiser (a reading; the pages fix none): s = fp16(max_i |y_i|)
// (round to nearest even, saturating at 65504), c_i = clamp(floor(y_i 2^(b-1) / s + 2^(b-1)),
// 0, 2^b - 1), codes packed LSB first, code i at bits [i b, i b + b) of the row, written as
// whole 32-bit words.
//
// Arithmetic is float64 end to end (IEEE float64 products and sums on the FP64 tensor-core
// MMA; the inputs are bf16 / fp32 values), which keeps every code equal to the one a float64
// restatement computes from the same stored factors, except for values within ~1e-13 s of a
// cell boundary.
#include "../jolt_internal.h"

namespace jolt {
namespace {

constexpr int kChunk = 256;          // tokens per CTA

__device__ __forceinline__ const void* x_row_ptr(const ResidualArgs& a, int lt, int h, int t) {
  const int layer = lt >> 1, kind = lt & 1;
  const int64_t off = (((int64_t)layer * a.H + h) * a.T + t) * a.D;
  const void* x = kind ? a.X[1] : a.X[0];   // constant indices: the argument stays in parameter space
  return a.xt == EL_BF16 ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(x) + off)
                         : (const void*)(reinterpret_cast<const float*>(x) + off);
}

// P = U_D[:, :r_d]^T Pi (r_d x D, float64) once per layer-tensor (with the Hadamard rotation,
// which the residual coder applies itself, P = U_D^T). Thread = 8 rows j0 .. x 4 columns e0 ..
// (a warp spans the 128 columns of its 8 rows): per d one 16-byte load of Pi's row, one of
// U_D's, 32 fused multiply-adds, each entry a chain in d order. Every product of stored values
// (bf16 x fp32) is exact in float64; only the sums round.
constexpr int kPRows = 8;
__global__ void __launch_bounds__(128) k_resid_p(ResidualArgs a, double* Pbuf) {
  const int i = blockIdx.y;
  const int lt = a.lt_ids[i];
  const StreamMeta* m = a.meta;
  const int rt = m->lt_rank[lt][0], rd = m->lt_rank[lt][1], b = m->lt_rank[lt][2];
  if ((b == 0 && !a.measure) || rt == 0) return;
  constexpr int D = kD;
  const int j0 = kPRows * (4 * blockIdx.x + (threadIdx.x >> 5)), e0 = 4 * (threadIdx.x & 31);
  if (j0 >= rd) return;   // rd is a multiple of 16
  const __nv_bfloat16* UD = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UD]);
  double* P = Pbuf + (int64_t)i * D * D;
  double acc[kPRows][4];
  if (a.hadamard) {
#pragma unroll
    for (int r = 0; r < kPRows; ++r)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[r][q] = (double)__bfloat162float(UD[(e0 + q) * rd + j0 + r]);
  } else {
#pragma unroll
    for (int r = 0; r < kPRows; ++r)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[r][q] = 0.0;
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
      const float4 pv = *reinterpret_cast<const float4*>(a.Pi + d * D + e0);
      const uint4 uw = *reinterpret_cast<const uint4*>(UD + d * rd + j0);   // U_D[d][j0 .. j0 + 7]
      const uint32_t w[4] = {uw.x, uw.y, uw.z, uw.w};
      const double p4[4] = {(double)pv.x, (double)pv.y, (double)pv.z, (double)pv.w};
#pragma unroll
      for (int r = 0; r < kPRows; ++r) {
        const double u = (double)__uint_as_float((r & 1) ? (w[r >> 1] & 0xffff0000u) : (w[r >> 1] << 16));
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][q] = fma(u, p4[q], acc[r][q]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kPRows; ++r) {
    *reinterpret_cast<double2*>(P + (j0 + r) * D + e0) = make_double2(acc[r][0], acc[r][1]);
    *reinterpret_cast<double2*>(P + (j0 + r) * D + e0 + 2) = make_double2(acc[r][2], acc[r][3]);
  }
}

// Pi^T (float32) in the coder's shared-memory layout: row n at stride kPSRow, PiT[n][k] = Pi[k][n].
constexpr int kPSRow = 132;
__global__ void __launch_bounds__(256) k_pi_t(const float* Pi, float* PiT) {
  const int n = blockIdx.x;
  for (int k = threadIdx.x; k < kPSRow; k += blockDim.x) PiT[n * kPSRow + k] = k < kD ? Pi[k * kD + n] : 0.0f;
}

// N_h = G_h P in float64 for one (layer-tensor, head): P and G_h in shared memory, thread =
// 4 x 4 block of N_h (rows k0 .., columns e0 ..), each entry a chain of r_d fused multiply-adds
// in j order.
__global__ void __launch_bounds__(256) k_resid_prep(ResidualArgs a, const double* Pbuf, double* Nbuf, int R) {
  extern __shared__ double P_s[];                 // [r_d][D], then G_h [r_t][r_d] as float
  const int h = blockIdx.x, i = blockIdx.y;
  const int lt = a.lt_ids[i];
  const StreamMeta* m = a.meta;
  const int rt = m->lt_rank[lt][0], rd = m->lt_rank[lt][1], b = m->lt_rank[lt][2];
  if ((b == 0 && !a.measure) || rt == 0) return;
  constexpr int D = kD, Q = kD / 4;
  const __nv_bfloat16* G = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_G]) +
                           (int64_t)h * rt * rd;
  float* G_s = reinterpret_cast<float*>(P_s + rd * D);
  const double2* P = reinterpret_cast<const double2*>(Pbuf + (int64_t)i * D * D);
  for (int u = threadIdx.x; u < rd * D / 2; u += blockDim.x) reinterpret_cast<double2*>(P_s)[u] = P[u];
  for (int u = threadIdx.x; u < rt * rd; u += blockDim.x) G_s[u] = __bfloat162float(G[u]);
  __syncthreads();
  // -N_h^T in the coder's layout: row n (feature) of r_t entries at stride r_t + 4
  double* NT = Nbuf + ((int64_t)i * a.H + h) * D * (R + 4);
  const int SN = rt + 4;
  for (int task = threadIdx.x; task < (rt / 4) * Q; task += blockDim.x) {
    const int k0 = 4 * (task / Q), e0 = 4 * (task % Q);
    double acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[r][q] = 0.0;
    for (int j = 0; j < rd; ++j) {
      const double2 p01 = *reinterpret_cast<const double2*>(P_s + j * D + e0);
      const double2 p23 = *reinterpret_cast<const double2*>(P_s + j * D + e0 + 2);
      const double pv[4] = {p01.x, p01.y, p23.x, p23.y};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const double g = (double)G_s[(k0 + r) * rd + j];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][q] = fma(g, pv[q], acc[r][q]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      *reinterpret_cast<double2*>(NT + (int64_t)(e0 + q) * SN + k0) = make_double2(-acc[0][q], -acc[1][q]);
      *reinterpret_cast<double2*>(NT + (int64_t)(e0 + q) * SN + k0 + 2) = make_double2(-acc[2][q], -acc[3][q]);
    }
  }
}

// y = [x | u] [Pi ; -N]: one float64 GEMM with K = D + r_t on the FP64 tensor-core MMA
// (m8n8k4: a warp multiplies an 8 x 4 by a 4 x 8 block; fragments per the PTX ISA). A CTA
// works on 256 tokens of one (layer-tensor, head) in tiles of 16 rows, with two groups of
// eight warps taking alternate tiles: while one group multiplies, the other quantises and
// packs, so the MMA pipe does not wait for the row-wise steps. Within a group, warp w computes
// rows 8 (w / 4) .. +7 and columns 32 (w % 4) .. +31 of its tile; y stays in the
// accumulators (the row absmax is combined through a 16 x 4 table in shared memory).
__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
}

constexpr int kRows = 16;          // rows per tile
constexpr int kPS = kPSRow;        // row stride (floats) of Pi^T: conflict-free fragment loads
constexpr int kGroups = 2;

template <bool kMeasure, bool kHad>
__global__ void __launch_bounds__(512, 1) k_residual(ResidualArgs a, const double* Nbuf, int R) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int chunk = blockIdx.x, h = blockIdx.y, i = blockIdx.z;
  const int lt = a.lt_ids[i];
  const StreamMeta* m = a.meta;
  const int rt = m->lt_rank[lt][0], b = m->lt_rank[lt][2];
  if (!kMeasure && b == 0) return;
  const int D = a.D;                       // 128
  const int K = D + rt;                    // GEMM depth
  const int SN = rt + 4;                   // row stride (doubles) of N^T
  const int SA = K + 4;                    // row stride (floats) of an A tile
  float* PT = reinterpret_cast<float*>(smraw);                                    // [D][kPS]
  double* NT = reinterpret_cast<double*>(PT + D * kPS);                           // [D][SN] = -N^T
  double* PM = NT + (size_t)D * SN;                                               // [2][kRows][4] row maxima
  float* AT = reinterpret_cast<float*>(PM + kGroups * kRows * 4);                 // [2][kRows][SA]
  unsigned char* CS = reinterpret_cast<unsigned char*>(AT + (size_t)kGroups * kRows * SA);   // [2][kRows][D]
  const int tid = threadIdx.x;
  // Pi^T and -N^T arrive in their shared-memory images: straight 16-byte copies
  if (!kHad)
    for (int e = tid; e < D * kPS / 4; e += 512)
      reinterpret_cast<float4*>(PT)[e] = reinterpret_cast<const float4*>(a.PiT)[e];
  {
    const double2* Ng = reinterpret_cast<const double2*>(Nbuf + ((int64_t)i * a.H + h) * D * (R + 4));
    for (int e = tid; e < D * SN / 2; e += 512) reinterpret_cast<double2*>(NT)[e] = Ng[e];
  }
  const __nv_bfloat16* UT = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UT]);
  __half* scales = reinterpret_cast<__half*>(a.body + m->off[lt][JOLT_PART_SCALES]);
  unsigned char* codes = a.body + m->off[lt][JOLT_PART_CODES];
  const int rowbytes = D * b / 8;
  const double half = b > 0 ? (double)(1 << (b - 1)) : 0.0;
  const int cmax = (1 << b) - 1;
  double errs[9] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};   // measure mode: sum of (y - y_hat_b)^2
  const int t_begin = chunk * kChunk, t_end = min(a.T, t_begin + kChunk);
  // group g takes the tiles t_begin + (2 k + g) kRows
  const int g = tid >> 8, gt = tid & 255, warp = gt >> 5, lane = tid & 31;
  float* At = AT + (size_t)g * kRows * SA;
  double* pm = PM + g * kRows * 4;
  unsigned char* cs = CS + g * kRows * D;
  const int rg = warp >> 2, cg = warp & 3;
  const int ar = 8 * rg + (lane >> 2), ak = lane & 3;
  // Hadamard mode: signs s_c of this thread's eight columns c = 32 cg + 8 j + 2 ak + e (bit
  // 2 j + e set: negative; Pi[c][0] = s_c / sqrt(D)) and the group's exchange rows (padded)
  constexpr int kXS = 132;
  double* xg = reinterpret_cast<double*>(smraw) + (size_t)g * kRows * kXS;
  uint32_t sneg = 0;
  if (kHad)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (a.Pi[(32 * cg + 8 * j + 2 * ak + e) * D] < 0.0f) sneg |= 1u << (2 * j + e);
  const int wpr = rowbytes / 4;                         // 32-bit words per packed row (4 b)
  const int c_first = (32 * lane) / b;                  // codes overlapping word `lane`
  const int c_last = min(D - 1, (32 * lane + 31) / b);
  __syncthreads();
  // A tile: x rows followed by u rows, as float (bf16 and float32 inputs are exact), from
  // 16-byte vector loads; thread (r = gt / 16, j = gt % 16) takes chunk j of row r (x) and
  // chunk j of u (if any). The group's next tile is loaded into registers during the MMAs.
  const int fr = gt >> 4, fj = gt & 15;
  uint4 px0 = make_uint4(0, 0, 0, 0), px1 = make_uint4(0, 0, 0, 0), pu = make_uint4(0, 0, 0, 0);
  auto fetch = [&](int t0) {
    const int t = t0 + fr;
    const bool live = t < t_end;
    px0 = px1 = pu = make_uint4(0, 0, 0, 0);
    if (live) {
      const uint4* xr = reinterpret_cast<const uint4*>(x_row_ptr(a, lt, h, t));
      if (a.xt == EL_BF16) {
        px0 = xr[fj];
      } else {
        px0 = xr[2 * fj];
        px1 = xr[2 * fj + 1];
      }
      if (8 * fj < rt) pu = *reinterpret_cast<const uint4*>(UT + (int64_t)t * rt + 8 * fj);   // rt: multiple of 16
    }
  };
  auto stage = [&]() {
    float* dst = At + fr * SA;
    if (a.xt == EL_BF16) {
      const uint32_t wv[4] = {px0.x, px0.y, px0.z, px0.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        dst[8 * fj + 2 * q] = __uint_as_float(wv[q] << 16);
        dst[8 * fj + 2 * q + 1] = __uint_as_float(wv[q] & 0xFFFF0000u);
      }
    } else {
      const uint32_t wv[8] = {px0.x, px0.y, px0.z, px0.w, px1.x, px1.y, px1.z, px1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[8 * fj + e] = __uint_as_float(wv[e]);
    }
    if (8 * fj < rt) {
      const uint32_t wv[4] = {pu.x, pu.y, pu.z, pu.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        dst[D + 8 * fj + 2 * q] = __uint_as_float(wv[q] << 16);
        dst[D + 8 * fj + 2 * q + 1] = __uint_as_float(wv[q] & 0xFFFF0000u);
      }
    }
  };
  // fp16 scale of a row from its absmax (round to nearest even, saturating at 65504)
  auto row_scale = [&](int r) -> __half {
    const double mx = fmax(fmax(pm[r * 4], pm[r * 4 + 1]), fmax(pm[r * 4 + 2], pm[r * 4 + 3]));
    return mx >= 65504.0 ? __float2half_rn(65504.0f) : __double2half(mx);
  };
  const int t_first = t_begin + g * kRows;
  if (t_first < t_end) fetch(t_first);
  for (int t0 = t_first; t0 < t_end; t0 += kGroups * kRows) {
    stage();
    group_sync(g);
    if (t0 + kGroups * kRows < t_end) fetch(t0 + kGroups * kRows);
    double acc[4][2];
    const float* arow = At + ar * SA + ak;
    const double* qb = NT + (32 * cg + (lane >> 2)) * SN + ak;
    if constexpr (kHad) {
      // accumulators start at x (this thread's entries of row ar); only -u M_h is multiplied
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) acc[j][e] = (double)At[ar * SA + 32 * cg + 8 * j + 2 * ak + e];
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = 0.0;
      const float* pb = PT + (32 * cg + (lane >> 2)) * kPS + ak;    // fragment j at + 8 j kPS
      // K = D part (x Pi), fully unrolled so the fragment loads of later steps can be issued early
#pragma unroll
      for (int k0 = 0; k0 < kD; k0 += 4) {
        const double av = (double)arow[k0];
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma_8x8x4(acc[j][0], acc[j][1], av, (double)pb[8 * j * kPS + k0]);
      }
    }
    // K = r_t part (-u N), four steps per unrolled block (r_t is a multiple of 16)
    for (int k0 = 0; k0 < rt; k0 += 16) {
#pragma unroll
      for (int kk = 0; kk < 16; kk += 4) {
        const double av = (double)arow[kD + k0 + kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma_8x8x4(acc[j][0], acc[j][1], av, qb[8 * j * SN + k0 + kk]);
      }
    }
    if constexpr (kHad) {
      // y = FWHT(r * s) / sqrt(D) over the 128 columns of row ar: column bit 0 (e) and bits 3-4
      // (j) inside the thread, bits 1-2 (ak) across lanes, bits 5-6 (cg) across the row's four
      // warps through shared memory (a 4-point transform per entry)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if ((sneg >> (2 * j + e)) & 1u) acc[j][e] = -acc[j][e];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const double a0 = acc[j][0], a1 = acc[j][1];
        acc[j][0] = a0 + a1;
        acc[j][1] = a0 - a1;
      }
#pragma unroll
      for (int jb = 1; jb <= 2; jb <<= 1)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (!(j & jb))
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const double lo = acc[j][e], hi = acc[j | jb][e];
              acc[j][e] = lo + hi;
              acc[j | jb][e] = lo - hi;
            }
#pragma unroll
      for (int m = 1; m <= 2; m <<= 1)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const double p = __shfl_xor_sync(0xffffffffu, acc[j][e], m);
            acc[j][e] = (ak & m) ? p - acc[j][e] : acc[j][e] + p;
          }
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) xg[ar * kXS + 32 * cg + 8 * j + 2 * ak + e] = acc[j][e];
      group_sync(g);
      const double inv = 1.0 / sqrt((double)kD);
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          double o = 0.0;
#pragma unroll
          for (int c2 = 0; c2 < 4; ++c2) {
            const double v = xg[ar * kXS + 32 * c2 + 8 * j + 2 * ak + e];
            o = (__popc(cg & c2) & 1) ? o - v : o + v;
          }
          acc[j][e] = o * inv;
        }
    }
    // row absmax: this thread's 8 entries of row ar, the 4 lanes of the row, then the 4 warps
    // of the row (columns 32 cg .. +31) through the table
    double mx = 0.0;
#pragma unroll
    for (int j = 0; j < 4; ++j) mx = fmax(mx, fmax(fabs(acc[j][0]), fabs(acc[j][1])));
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if ((lane & 3) == 0) pm[ar * 4 + cg] = mx;
    group_sync(g);
    if constexpr (kMeasure) {
      // exact squared error of every allowed width at this row's fp16 scale s: b = 0 stores no
      // residual (error y^2); otherwise c = clamp(floor(y 2^(b-1) / s + 2^(b-1))) and
      // y_hat = (2 c + 1 - 2^b) (s / 2^b), both products exact in float64 (s = 0: every code 0)
      const double sd = (double)__half2float(row_scale(ar));
#pragma unroll
      for (int bb = 0; bb <= 8; ++bb) {
        if (!((a.bits_mask >> bb) & 1u)) continue;
        double e = 0.0;
        if (bb == 0) {
#pragma unroll
          for (int j = 0; j < 4; ++j) e = fma(acc[j][1], acc[j][1], fma(acc[j][0], acc[j][0], e));
        } else {
          const double hb = (double)(1 << (bb - 1)), inv = sd > 0.0 ? hb / sd : 0.0;
          const double cell = sd * (1.0 / (double)(1 << bb));
          const double top = (double)((1 << bb) - 1);
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int ee = 0; ee < 2; ++ee) {
              double c = 0.0;
              if (sd > 0.0) c = fmin(fmax(floor(fma(acc[j][ee], inv, hb)), 0.0), top);
              const double d = acc[j][ee] - (2.0 * c + 1.0 - 2.0 * hb) * cell;
              e = fma(d, d, e);
            }
        }
        errs[bb] += e;
      }
      continue;
    }
    // codes: c = floor(y * (2^(b-1) / s) + 2^(b-1)), clamped, with one reciprocal per row
    // (it can differ from a divide-per-entry only for values within ~1e-16 s of a cell boundary)
    {
      const double sd = (double)__half2float(row_scale(ar));
      const double inv = sd > 0.0 ? half / sd : 0.0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int cc[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          int c = 0;
          if (sd > 0.0) {
            const double f = floor(fma(acc[j][e], inv, half));
            c = f < 0.0 ? 0 : (f > (double)cmax ? cmax : (int)f);
          }
          cc[e] = c;
        }
        const int col = 32 * cg + 8 * j + 2 * (lane & 3);
        *reinterpret_cast<uint16_t*>(cs + ar * D + col) = (uint16_t)(cc[0] | (cc[1] << 8));
      }
    }
    group_sync(g);
    // pack: warp w of the group handles rows 2 w and 2 w + 1; lane owns 32-bit word `lane`
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = 2 * warp + rr;
      const int t = t0 + r;
      if (t < t_end) {
        const int64_t row = (int64_t)h * a.T + t;
        if (lane < wpr) {
          uint32_t word = 0;
          for (int q = c_first; q <= c_last; ++q) {
            const int sh2 = q * b - 32 * lane;
            const uint32_t cv = cs[r * D + q];
            word |= sh2 >= 0 ? (cv << sh2) : (cv >> (-sh2));
          }
          reinterpret_cast<uint32_t*>(codes + row * rowbytes)[lane] = word;
        }
        if (lane == 0) scales[row] = row_scale(r);
      }
    }
  }
  if constexpr (kMeasure) {
    // fixed-order reduction of the 512 threads' sums: warp butterflies, then warps in order
#pragma unroll
    for (int bb = 0; bb <= 8; ++bb)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) errs[bb] += __shfl_xor_sync(0xffffffffu, errs[bb], o);
    __syncthreads();                                   // every group is past its last tile
    double* red = reinterpret_cast<double*>(AT);       // [16][9]
    if (lane == 0)
#pragma unroll
      for (int bb = 0; bb <= 8; ++bb) red[(tid >> 5) * 9 + bb] = errs[bb];
    __syncthreads();
    if (tid < 9) {
      double sum = 0.0;
      for (int w = 0; w < 16; ++w) sum += red[w * 9 + tid];
      const int nchunk = (a.T + kChunk - 1) / kChunk;
      a.meas_part[(((int64_t)i * a.H + h) * nchunk + chunk) * 9 + tid] = sum;
    }
  }
}

}  // namespace

// P [r_d][D] float64 and G_h [r_t][r_d] float32 at the largest ranks
static size_t residual_prep_smem() { return (size_t)kD * kD * sizeof(double) + (size_t)kD * kD * sizeof(float); }

cudaError_t residual_encode(const ResidualArgs& a, double* Pbuf, double* Nbuf, int R, cudaStream_t s) {
  if (a.D != kD) return cudaErrorInvalidValue;
  if (!a.hadamard) {
    if (!a.PiT) return cudaErrorInvalidValue;
    k_pi_t<<<kD, 128, 0, s>>>(a.Pi, a.PiT);
    note_launch();
  }
  k_resid_p<<<dim3(kD / (4 * kPRows), a.n_lt), 128, 0, s>>>(a, Pbuf);
  note_launch();
  const size_t sp = residual_prep_smem();
  cudaError_t e = cudaFuncSetAttribute(k_resid_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp);
  if (e != cudaSuccess) return e;
  k_resid_prep<<<dim3(a.H, a.n_lt), 256, sp, s>>>(a, Pbuf, Nbuf, R);
  note_launch();
  // Pi^T (float), -N^T (float64), the row-max tables, the two groups' A tiles (float) and codes
  const size_t sm = (size_t)kD * kPS * sizeof(float) + (size_t)kD * (R + 4) * sizeof(double) +
                    (size_t)kGroups * kRows * 4 * sizeof(double) +
                    (size_t)kGroups * kRows * (kD + R + 4) * sizeof(float) + (size_t)kGroups * kRows * kD;
  const dim3 g((a.T + kChunk - 1) / kChunk, a.H, a.n_lt);
  if (a.measure && !a.meas_part) return cudaErrorInvalidValue;
  auto launch = [&](auto kern) {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e2 != cudaSuccess) return e2;
    kern<<<g, 512, sm, s>>>(a, Nbuf, R);
    return cudaSuccess;
  };
  if (a.measure) e = a.hadamard ? launch(k_residual<true, true>) : launch(k_residual<true, false>);
  else e = a.hadamard ? launch(k_residual<false, true>) : launch(k_residual<false, false>);
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
