// Fused decode of the JoLT codec on the 5th-generation tensor cores: unpack, dequantise,
// inverse-rotate, add the Tucker part and store.
//
// "A JoLT for the KV Cache" (arXiv 2607.12550v2, Abstract) reconstructs the cache from the
// partial Tucker factors plus the rotated low-bit residual. For the rows t of head h:
//     X_hat = U_T M_h + diag(s) Y_hat Pi^T,   M_h = G_h U_D^T (r_t x D),
//     Y_hat[t][i] = (2 c + 1 - 2^b) / 2^b     (mid-rise cell centres at unit scale),
// with U_T[:, :r_t], the row's fp16 scale s and b-bit codes c.
//
// One CTA per (layer-tensor, head) walks the T rows in tiles of 128:
//  * prologue: M_h^T = U_D G_h^T on the tensor core (both operands are the stored bf16
//    factors, so the products are exact and only the float32 sum rounds); M_h^T is kept in
//    shared memory as two bf16 parts (hi + lo, ~2^-17 relative), Pi (float32) scaled by 2^10 as
//    two fp16 parts (~2^-22 relative; the scale keeps the low parts out of the subnormals);
//  * producers (warps 4-11) copy the tile's U_T rows and unpack its codes into the fp16
//    integers m = 2 c + 1 - 2^b (exact: |m| < 2^8), both in the 128-byte-swizzled K-major
//    layout. Two codes become one 32-bit word by an integer multiply-add onto the bit pattern of
//    fp16 1024 and one packed fp16 subtraction (no integer-to-float conversion). The codes and
//    U_T rows of the tile three ahead are prefetched into L2, those of the next tile loaded into
//    registers while the current tile is unpacked;
//    the code tiles go to two alternating buffers, so a tile is unpacked while the previous one
//    is multiplied;
//  * warp 12 issues tcgen05.mma: acc1 = U_T (M_h^T)_p^T (bf16), then acc2 = m (2^10 Pi)_p^T over
//    the parts p (fp16), double-buffered in Tensor Memory (4 x 128 columns). The U_T buffer is
//    single: it is released as soon as the Tucker products of a tile complete, ahead of the
//    residual ones;
//  * the epilogue (warps 0-3, one row per thread) forms acc1 + (s 2^-(b+10)) acc2 and stores
//    bf16 (round to nearest even) or float32; the row's next scale is loaded a tile ahead.
// Every wait is bounded: a timeout sets ST_TIMEOUT in the stream status and the CTA runs on
// to its end without hanging.
#include "../jolt_internal.h"
#include "gemm_tc.h"
#include "sm100.cuh"
#include <type_traits>

namespace jolt {
namespace {

using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kEpiWarps = 4;                  // warps 0-3: TMEM lane quadrant = warp
constexpr int kProducers = 256;               // warps 4-11
constexpr int kProdWarp0 = kEpiWarps;
constexpr int kMmaWarp = kProdWarp0 + kProducers / 32;
constexpr int kThreads = 32 * (kMmaWarp + 1);  // 13 warps
constexpr int kOpBytes = 128 * 128 * 2;       // one 128 x 128 bf16 operand (two swizzle atoms)
constexpr uint32_t kMaxPoll = 1u << 22;
// dynamic shared memory: B1 parts (M_h^T), B2 parts (Pi), A1 (U_T tile), two A2 (cell centres)
constexpr int kOffB1 = 0;
constexpr int kOffB2 = 2 * kOpBytes;
constexpr int kOffA1 = 4 * kOpBytes;
constexpr int kOffA2 = 5 * kOpBytes;
constexpr int kSmemBytes = 7 * kOpBytes + 1024;
constexpr int kUtVec = 8;      // 16-byte U_T vectors per producer thread and tile (128 rows x r_t <= 128)

// Byte offset of the 16-byte chunk `c16` (8 bf16, k = 8 c16 ..) of row `row` in a K-major
// 128-row operand with 128-byte swizzling: 64-element atoms of 16 KB, rows of 128 bytes, the
// chunk index XOR-ed with the row's position in its 8-row group.
__device__ __forceinline__ uint32_t sw128(int row, int c16) {
  return (uint32_t)((c16 >> 3) * 16384 + row * 128 + (((c16 & 7) ^ (row & 7)) << 4));
}

// Descriptor of the 16-wide K slice `kk` of a 128-row operand at shared address `base`.
__device__ __forceinline__ uint64_t slice_desc(uint32_t base, int kk) {
  return desc_kmajor_sw128(base + (uint32_t)((kk >> 2) * 16384 + (kk & 3) * 32));
}

// Tile store: the box at (c0, c1, c2) of `map` from shared memory (128-byte swizzled image), then
// a commit of the bulk group; wait_group_read(0) before the shared memory is written again.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Split 8 floats into bf16 hi and lo parts (16 bytes each).
__device__ __forceinline__ void split8(const float (&v)[8], uint4& hi, uint4& lo) {
  float h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    l[i] = v[i] - h[i];
  }
  hi = make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
  lo = make_uint4(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]), pack_bf16x2(l[4], l[5]), pack_bf16x2(l[6], l[7]));
}

// Split 8 floats, scaled by 2^10, into fp16 hi and lo parts (16 bytes each).
constexpr float kPiScale = 1024.0f;
__device__ __forceinline__ void split8_f16(const float (&v)[8], uint4& hi, uint4& lo) {
  uint32_t h2[4], l2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a0 = v[2 * i] * kPiScale, a1 = v[2 * i + 1] * kPiScale;
    const __half x0 = __float2half_rn(a0), x1 = __float2half_rn(a1);
    const __half y0 = __float2half_rn(a0 - __half2float(x0)), y1 = __float2half_rn(a1 - __half2float(x1));
    const __half2 hx = __halves2half2(x0, x1), hy = __halves2half2(y0, y1);
    h2[i] = *reinterpret_cast<const uint32_t*>(&hx);
    l2[i] = *reinterpret_cast<const uint32_t*>(&hy);
  }
  hi = make_uint4(h2[0], h2[1], h2[2], h2[3]);
  lo = make_uint4(l2[0], l2[1], l2[2], l2[3]);
}

// Two b-bit codes c0 (low half) and c1 (high half), packed as 16-bit fields in `cc`, to the fp16
// pair (2 c0 + 1 - 2^b, 2 c1 + 1 - 2^b): 2 cc + (0x6400 + 513 - 2^b) per half is the bit pattern
// of fp16 1536 + m (0x6400 is 1024.0; 257 <= 512 + m <= 767 stays in its binade, no carry between
// the halves), and subtracting 1536 leaves m exactly.
__device__ __forceinline__ uint32_t codes_to_f16x2(uint32_t cc, uint32_t bias2) {
  const uint32_t biased = cc * 2u + bias2;
  const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&biased), __floats2half2_rn(1536.0f, 1536.0f));
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* status) {
  if (mbar_wait(bar, parity, kMaxPoll)) return true;
  atomicOr(status, ST_TIMEOUT);
  return false;
}

// Output tensor maps: [L][H][T][128] bf16 as (128, T, L * H) with a 64 x 32 box (one epilogue
// warp's rows, half of the features), 128-byte swizzle; used when the output is bf16.
struct OutMaps {
  CUtensorMap m[2];
};

__global__ void __launch_bounds__(kThreads, 1) k_decode_tc(DecodeArgs a, const __grid_constant__ OutMaps om) {
  extern __shared__ uint8_t smraw[];
  __shared__ __align__(8) uint64_t bar_pro, bar_afull[2], bar_a1free, bar_a2free[2];
  __shared__ __align__(8) uint64_t bar_accfull[2], bar_accempty[2];
  __shared__ uint32_t tmem_base;
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, li = blockIdx.y;
  const int lt = a.lt_ids[li];
  const StreamMeta* m = a.meta;
  int32_t* status = const_cast<int32_t*>(&m->status);
  const int rt = m->lt_rank[lt][0], rd = m->lt_rank[lt][1], b = m->lt_rank[lt][2];
  const bool tucker = rt > 0 && rd > 0, resid = b > 0;
  const int T = a.T, H = a.H;
  const __nv_bfloat16* UT = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UT]);
  const __nv_bfloat16* UD = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UD]);
  const __nv_bfloat16* G = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_G]) +
                           (int64_t)h * rt * rd;
  const __half* scales = reinterpret_cast<const __half*>(a.body + m->off[lt][JOLT_PART_SCALES]);
  const uint8_t* codes = a.body + m->off[lt][JOLT_PART_CODES];
  const int rowbytes = 16 * b;             // D * b / 8 bytes per row, D = 128
  const int ntiles = (T + kTileRows - 1) / kTileRows;
  const uint32_t sB1 = smem_u32(sm + kOffB1), sB2 = smem_u32(sm + kOffB2);
  const uint32_t sA1 = smem_u32(sm + kOffA1), sA2 = smem_u32(sm + kOffA2);

  if (tid == 0) {
    mbar_init(&bar_pro, 1);
    mbar_init(&bar_a1free, 1);
    for (int j = 0; j < 2; ++j) {
      mbar_init(&bar_afull[j], kProducers);
      mbar_init(&bar_a2free[j], 1);
      mbar_init(&bar_accfull[j], 1);
      mbar_init(&bar_accempty[j], 32 * kEpiWarps);
    }
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  // ---------------------------------------------------------------- prologue
  // Pi (float32, row n = output feature, k = rotated coordinate) -> 2^10 Pi as two fp16 parts (B2)
  for (int u = tid; u < 128 * 16; u += kThreads) {
    const int n = u >> 4, c = u & 15;
    const float4 p0 = *reinterpret_cast<const float4*>(a.Pi + n * 128 + 8 * c);
    const float4 p1 = *reinterpret_cast<const float4*>(a.Pi + n * 128 + 8 * c + 4);
    const float v[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    uint4 hi, lo;
    split8_f16(v, hi, lo);
    *reinterpret_cast<uint4*>(sm + kOffB2 + sw128(n, c)) = hi;
    *reinterpret_cast<uint4*>(sm + kOffB2 + kOpBytes + sw128(n, c)) = lo;
  }
  // U_D (rows n, K = r_d) into A1 and G_h (rows k, K = r_d) into A2 for M_h^T = U_D G_h^T
  if (tucker) {
    const int cpr = rd / 8;
    for (int u = tid; u < 128 * cpr; u += kThreads) {
      const int n = u / cpr, c = u - n * cpr;
      *reinterpret_cast<uint4*>(sm + kOffA1 + sw128(n, c)) =
          *reinterpret_cast<const uint4*>(UD + (int64_t)n * rd + 8 * c);
    }
    for (int u = tid; u < rt * cpr; u += kThreads) {
      const int k = u / cpr, c = u - k * cpr;
      *reinterpret_cast<uint4*>(sm + kOffA2 + sw128(k, c)) =
          *reinterpret_cast<const uint4*>(G + (int64_t)k * rd + 8 * c);
    }
  }
  fence_async_shared();
  __syncthreads();
  if (tucker) {
    if (warp == kMmaWarp) {
      if (elect_one()) {
        tc_fence_after();
        const uint32_t id = idesc_bf16_f32(128, rt);
        for (int kk = 0; kk < rd / 16; ++kk)
          umma_bf16(tmem, slice_desc(sA1, kk), slice_desc(sA2, kk), id, kk > 0 ? 1u : 0u);
        umma_commit(&bar_pro);
      }
      __syncwarp();
    } else if (warp < 4) {
      wait_or_flag(&bar_pro, 0, status);
      tc_fence_after();
      const int n = 32 * warp + lane;   // feature row of M_h^T
      for (int c = 0; c < (rt + 31) / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(32 * c), r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c16 = 4 * c + q;
          if (8 * c16 < rt) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[8 * q + j]);
            uint4 hi, lo;
            split8(v, hi, lo);
            *reinterpret_cast<uint4*>(sm + kOffB1 + sw128(n, c16)) = hi;
            *reinterpret_cast<uint4*>(sm + kOffB1 + kOpBytes + sw128(n, c16)) = lo;
          }
        }
      }
      fence_async_shared();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---------------------------------------------------------------- tiles of 128 rows
  if (warp >= kProdWarp0 && warp < kMmaWarp) {
    // producers: U_T rows -> A1, unpacked codes -> A2[tile parity]. Thread pt takes half a row of
    // codes (row pt / 2, codes 64 (pt % 2) ..): 64 codes of b bits are 8 b contiguous bytes at byte
    // 8 b pt of the tile's code block, loaded as b aligned 8-byte words one tile ahead. The loop
    // is instantiated per code width, so every bit position is a constant: a pair of codes is one
    // shift of 2b bits and one spread of the second code to bit 16. U_T rows go through registers
    // one tile ahead as well; the tile three ahead is prefetched into L2.
    const int pt = tid - 32 * kProdWarp0;
    const int cpr = tucker ? rt / 8 : 0;   // 16-byte vectors per U_T row
    // u / cpr for u < 2048 as (u * cmul) >> 20, cmul = ceil(2^20 / cpr): exact, since the
    // fraction u / cpr is at most 1 - 1 / cpr and the error u (cmul - 2^20 / cpr) / 2^20 is below
    // 2^-9 for cpr <= 16
    const uint32_t cmul = tucker ? ((1u << 20) + (uint32_t)cpr - 1u) / (uint32_t)cpr : 0u;
    auto udiv = [&](int u) { return (int)(((uint32_t)u * cmul) >> 20); };
    uint4 ut[kUtVec];
    auto load_ut = [&](int it2) {
      const int t2 = it2 * kTileRows, rows2 = min(kTileRows, T - t2);
      const __nv_bfloat16* src = UT + (int64_t)t2 * rt;
#pragma unroll
      for (int q = 0; q < kUtVec; ++q) {
        const int u = pt + kProducers * q;
        ut[q] = (it2 < ntiles && u < rows2 * cpr)
                    ? *reinterpret_cast<const uint4*>(src + (int64_t)udiv(u) * rt + 8 * (u - udiv(u) * cpr))
                    : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    // the codes and U_T rows of tile it2 into L2 (one thread): the register loads of a tile,
    // issued one tile ahead, then find them there instead of waiting on DRAM
    auto prefetch_tile = [&](int it2) {
      if (pt != 0 || it2 >= ntiles) return;
      const int t2 = it2 * kTileRows, rows2 = min(kTileRows, T - t2);
      if (resid) prefetch_l2(codes + ((int64_t)h * T + t2) * rowbytes, (uint32_t)(rows2 * rowbytes));
      if (tucker) prefetch_l2(UT + (int64_t)t2 * rt, (uint32_t)(rows2 * rt * 2));
    };
    const int r_own = pt >> 1, hf = pt & 1;
    auto run = [&](auto Bc) {
      constexpr int B = decltype(Bc)::value;    // code width; 0: no residual
      constexpr int NW = B > 0 ? B : 1;         // 8-byte words per half row
      uint64_t cw[NW];
      auto load_codes = [&](int it2) {
        if constexpr (B > 0) {
          const int t2 = it2 * kTileRows, rows2 = min(kTileRows, T - t2);
          const uint64_t* w = reinterpret_cast<const uint64_t*>(codes + ((int64_t)h * T + t2) * rowbytes) + NW * pt;
          const bool ok = it2 < ntiles && r_own < rows2;
#pragma unroll
          for (int q = 0; q < NW; ++q) cw[q] = ok ? __ldg(w + q) : 0ull;
        }
      };
      const uint32_t bias = B > 0 ? 0x6400u + 513u - (1u << B) : 0u;
      const uint32_t bias2 = bias | (bias << 16);
      prefetch_tile(1);
      prefetch_tile(2);
      load_codes(0);
      if (tucker) load_ut(0);
      for (int it = 0; it < ntiles; ++it) {
        prefetch_tile(it + 3);
        const int buf = it & 1, use = it >> 1;
        const int rows = min(kTileRows, T - it * kTileRows);
        if constexpr (B > 0) {
          // A2[buf] was last read by the residual products of tile it - 2
          wait_or_flag(&bar_a2free[buf], (uint32_t)((use & 1) ^ 1), status);
          uint8_t* a2 = sm + kOffA2 + buf * kOpBytes;
          constexpr uint32_t m1 = (1u << B) - 1u;
#pragma unroll
          for (int j = 0; j < 8; ++j) {          // 16-byte chunk j: codes 8 j .. 8 j + 7 of the half row
            uint32_t y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              constexpr int kPair = 2 * B;
              const int bit = (8 * j + 2 * e) * B, wi = bit >> 6, sh = bit & 63;
              uint64_t v = cw[wi] >> sh;
              if (sh + kPair > 64) v |= cw[wi + 1] << (64 - sh);
              const uint32_t x = (uint32_t)v;
              y[e] = codes_to_f16x2((x & m1) | ((x << (16 - B)) & (m1 << 16)), bias2);
            }
            if (r_own < rows)
              *reinterpret_cast<uint4*>(a2 + sw128(r_own, 8 * hf + j)) = make_uint4(y[0], y[1], y[2], y[3]);
          }
          load_codes(it + 1);
        }
        if (tucker) {
          // A1 was last read by the Tucker products of tile it - 1
          wait_or_flag(&bar_a1free, (uint32_t)((it & 1) ^ 1), status);
#pragma unroll
          for (int q = 0; q < kUtVec; ++q) {
            const int u = pt + kProducers * q;
            if (u < rows * cpr) {
              const int ur = udiv(u);
              *reinterpret_cast<uint4*>(sm + kOffA1 + sw128(ur, u - ur * cpr)) = ut[q];
            }
          }
          load_ut(it + 1);
        }
        fence_async_shared();
        mbar_arrive(&bar_afull[buf]);
      }
    };
    switch (resid ? b : 0) {
      case 1: run(std::integral_constant<int, 1>{}); break;
      case 2: run(std::integral_constant<int, 2>{}); break;
      case 3: run(std::integral_constant<int, 3>{}); break;
      case 4: run(std::integral_constant<int, 4>{}); break;
      case 5: run(std::integral_constant<int, 5>{}); break;
      case 6: run(std::integral_constant<int, 6>{}); break;
      case 7: run(std::integral_constant<int, 7>{}); break;
      case 8: run(std::integral_constant<int, 8>{}); break;
      default: run(std::integral_constant<int, 0>{}); break;
    }
  } else if (warp == kMmaWarp) {
    if (elect_one()) {
      const uint32_t id = idesc_bf16_f32(128, 128);
      const uint32_t id16 = idesc_f16_f32(128, 128);
      for (int it = 0; it < ntiles; ++it) {
        const int buf = it & 1, use = it >> 1;
        wait_or_flag(&bar_afull[buf], (uint32_t)(use & 1), status);
        wait_or_flag(&bar_accempty[buf], (uint32_t)((use & 1) ^ 1), status);
        tc_fence_after();
        const uint32_t d1 = tmem + (uint32_t)(buf * 256), d2 = d1 + 128;
        if (tucker)
          for (int kk = 0; kk < rt / 16; ++kk)
#pragma unroll
            for (int p = 0; p < 2; ++p)
              umma_bf16(d1, slice_desc(sA1, kk), slice_desc(sB1 + p * kOpBytes, kk), id, (kk | p) ? 1u : 0u);
        umma_commit(&bar_a1free);         // the U_T tile may be overwritten once these complete
        if (resid) {
          const uint32_t a2 = sA2 + (uint32_t)(buf * kOpBytes);
          for (int kk = 0; kk < 8; ++kk)
#pragma unroll
            for (int p = 0; p < 2; ++p)
              umma_bf16(d2, slice_desc(a2, kk), slice_desc(sB2 + p * kOpBytes, kk), id16, (kk | p) ? 1u : 0u);
        }
        umma_commit(&bar_a2free[buf]);
        umma_commit(&bar_accfull[buf]);
      }
    }
    __syncwarp();
  } else if (warp < kEpiWarps) {
    // epilogue: TMEM lanes 32 warp .. 32 warp + 31 are rows of the tile
    const int q4 = warp;
    const int layer = lt >> 1, kind = lt & 1;
    const int64_t obase = ((int64_t)layer * H + h) * T * 128;
    void* const outk = kind ? a.out[1] : a.out[0];   // constant indices: the argument stays in parameter space
    // With r_t <= 64 the second halves of the two M_h^T parts are unused: each warp stages its
    // 32 rows there as two boxes of 64 features (4 KB each, the 128-byte swizzled image of a box;
    // features 0-63 in part 0's half, 64-127 in part 1's) and stores them with two tensor copies;
    // otherwise every thread stores its row directly.
    const bool staged = a.ot == EL_BF16 && rt <= 64;
    uint8_t* stage0 = sm + kOffB1 + kOpBytes / 2 + warp * 4096;
    // the row's scale for tile it + 1 is loaded while tile it is waited for and stored
    // s 2^-(b+10): the cell centre is m / 2^b and Pi entered scaled by 2^10 (exact powers of two)
    const float unscale = resid ? 1.0f / ((float)(1 << b) * kPiScale) : 0.0f;
    auto load_scale = [&](int it2) {
      const int t2 = it2 * kTileRows + 32 * q4 + lane;
      return (resid && t2 < T) ? __half2float(scales[(int64_t)h * T + t2]) * unscale : 0.0f;
    };
    float s_next = load_scale(0);
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1, use = it >> 1;
      const float s = s_next;
      if (it + 1 < ntiles) s_next = load_scale(it + 1);
      wait_or_flag(&bar_accfull[buf], (uint32_t)(use & 1), status);
      tc_fence_after();
      const int t = it * kTileRows + 32 * q4 + lane;
      const bool valid = t < T;
      const uint32_t tb = tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)(buf * 256);
      if (staged) {
        // the previous tile's tensor copy has read the staging buffer
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r1[32], r2[32];
        if (tucker) tmem_ld32(tb + (uint32_t)(32 * c), r1);
        if (resid) tmem_ld32(tb + 128u + (uint32_t)(32 * c), r2);
        tmem_ld_wait();
        float o[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float v = tucker ? __uint_as_float(r1[j]) : 0.0f;
          if (resid) v = fmaf(s, __uint_as_float(r2[j]), v);
          o[j] = v;
        }
        if (staged) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int g = 4 * (c & 1) + q;     // 16-byte granule of the 128-byte box row
            *reinterpret_cast<uint4*>(stage0 + (c >> 1) * kOpBytes + lane * 128 + ((g ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16x2(o[8 * q], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                           pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
          }
        } else if (valid) {
          if (a.ot == EL_BF16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(outk) + obase +
                                                  (int64_t)t * 128 + 32 * c);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_bf16x2(o[8 * q], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                                  pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(outk) + obase +
                                                    (int64_t)t * 128 + 32 * c);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar_accempty[buf]);
      if (staged) {
        fence_async_shared();
        __syncwarp();
        // rows beyond T fall outside the map and are not written
        if (lane == 0) {
          tma_store_3d(&om.m[kind], stage0, 0, it * kTileRows + 32 * q4, layer * H + h);
          tma_store_3d(&om.m[kind], stage0 + kOpBytes, 64, it * kTileRows + 32 * q4, layer * H + h);
        }
      }
    }
    if (staged && lane == 0) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.D != kD) return cudaErrorInvalidValue;
  if (a.n_lt <= 0 || a.T <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_decode_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  OutMaps om;
  memset(&om, 0, sizeof(om));
  if (a.ot == EL_BF16) {
    const uint64_t dims[3] = {128, (uint64_t)a.T, (uint64_t)a.L * a.H};
    const uint64_t str[2] = {256, (uint64_t)a.T * 256};
    for (int k = 0; k < 2; ++k)
      if (a.out[k] && !tc_map_bf16_rows32(&om.m[k], a.out[k], 3, dims, str)) return cudaErrorInvalidValue;
  }
  const dim3 g(a.H, a.n_lt);
  k_decode_tc<<<g, kThreads, kSmemBytes, s>>>(a, om);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
