// Batched bf16 GEMM on the 5th-generation tensor cores: C[b] = sum_p A_p[b] B_p[b]^T.
//
// It carries the dense contractions of the JoLT factor analysis ("A JoLT for the KV Cache",
// arXiv 2607.12550v2, Abstract: the partial Tucker factors of the token and feature axes and
// the randomized-SVD "FlashJoLT" sketch): the feature Gram C_D = sum_h X_h^T X_h and the
// four sketch passes A Omega, A^T Q, A Q', Q^T A over the token unfolding A = X_(2).
// float32 operands enter as a sum of up to three bf16 parts (hi + lo + lo2), each part one
// more pass of the tensor core over the same accumulator.
//
// Structure: persistent, one CTA per SM looping over 128 x 128 output tiles. Warp 0 issues
// TMA tile loads (128 rows x 64 bf16, 128-byte swizzle, no multicast) into a ring of stages
// that runs on across tiles; warp 1 owns two Tensor Memory accumulators and issues
// tcgen05.mma (M = 128, N = 128, K = 16) from one thread, alternating between them tile by
// tile; warps 4-11 read a finished accumulator back with tcgen05.ld and store float32 (and/or
// bf16 parts) while the next tile is being loaded and multiplied (two warps per TMEM lane
// quadrant, one per half of the columns, so that each SM sub-partition has two epilogue warps
// to interleave). Every wait is bounded and
// reports ST_TIMEOUT instead of hanging.
#include "../jolt_internal.h"
#include "sm100.cuh"
#include "gemm_tc.h"

namespace jolt {
namespace {

using namespace sm100;

constexpr int kTile = 128;
constexpr int kBK = 64;
constexpr int kTileBytes = kTile * kBK * 2;   // 16 KB per operand part and stage
constexpr uint32_t kMaxPoll = 1u << 22;
constexpr uint32_t kMnHalf = 64 * kBK * 2;    // one 64-row half of an MN-major tile (8 KB)

__host__ __device__ __forceinline__ bool is_mn(int mode) {
  return mode == VIEW_MN || mode == VIEW_MN_XFEAT || mode == VIEW_MN_XHEAD;
}

__device__ __forceinline__ void view_coords(const TcView& v, int row0, int kb, int b, int& c0, int& c1, int& c2,
                                            int& c3) {
  if (v.nch > 1) {
    kb += (b % v.nch) * v.ckb;
    b /= v.nch;
  }
  if (v.ksplit > 0 && b >= v.ksplit) b -= v.ksplit;
  switch (v.mode) {
    case VIEW_X_TOKENROWS: {           // map (D, T, H, L): rows t, K = (h, d)
      const int kpd = v.D / kBK;
      c0 = (kb % kpd) * kBK; c1 = row0; c2 = kb / kpd; c3 = b;
      break;
    }
    case VIEW_ROWS_K_HEAD:             // map (K, rows, H, n), batch b = i * H + h
      c0 = kb * kBK; c1 = row0; c2 = b % v.H; c3 = b / v.H;
      break;
    case VIEW_MN:                      // map (rows, K, batch), rows contiguous
      c0 = row0 + (b % v.H) * v.D; c1 = kb * kBK; c2 = b / v.H; c3 = 0;
      break;
    case VIEW_MN_XFEAT:                // map (D, T, H, L): rows (h, d), K = t
      c0 = row0 % v.D; c1 = kb * kBK; c2 = row0 / v.D; c3 = b;
      break;
    case VIEW_MN_XHEAD:                // same map, batch b = layer * H + h: rows d, K = t
      c0 = row0; c1 = kb * kBK; c2 = b % v.H; c3 = b / v.H;
      break;
    default:                           // VIEW_ROWS_K: map (K, rows, batch), batch index b / H
      c0 = kb * kBK; c1 = row0; c2 = b / v.H; c3 = 0;
      break;
  }
}

__device__ __forceinline__ void view_load(const TcView& v, const CUtensorMap* map, void* dst, uint64_t* bar,
                                          int row0, int kb, int b) {
  if (v.ksplit > 0 && (v.nch > 1 ? b / v.nch : b) >= v.ksplit) ++map;   // the second source
  int c0, c1, c2, c3;
  view_coords(v, row0, kb, b, c0, c1, c2, c3);
  if (v.mode == VIEW_ROWS_K) {
    tma_load_3d(dst, map, bar, c0, c1, c2);
  } else if (v.mode == VIEW_MN) {
    // two boxes of 64 rows x 64 k: the tile's MN-major halves, kMnHalf bytes apart
    tma_load_3d(dst, map, bar, c0, c1, c2);
    tma_load_3d(static_cast<uint8_t*>(dst) + kMnHalf, map, bar, c0 + 64, c1, c2);
  } else if (v.mode == VIEW_MN_XFEAT || v.mode == VIEW_MN_XHEAD) {
    tma_load_4d(dst, map, bar, c0, c1, c2, c3);
    tma_load_4d(static_cast<uint8_t*>(dst) + kMnHalf, map, bar, c0 + 64, c1, c2, c3);
  } else {
    tma_load_4d(dst, map, bar, c0, c1, c2, c3);
  }
}

// bf16 parts of v at offset off: v = p0 + p1 + p2 (each remainder is exact in float32).
__device__ __forceinline__ void put_parts(__nv_bfloat16* const (&P)[3], int64_t off, float v) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h0);
  const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
  P[0][off] = h0;
  if (P[1]) P[1][off] = h1;
  if (P[2]) P[2][off] = __float2bfloat16_rn(r1 - __bfloat162float(h1));
}

// Three bf16 parts of 8 floats (16 bytes per part).
__device__ __forceinline__ void parts8(const float (&v)[8], uint4& h0, uint4& h1, uint4& h2) {
  uint32_t w0[4], w1[4], w2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float a[2], b[2], c[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float x = v[2 * i + k];
      a[k] = __bfloat162float(__float2bfloat16_rn(x));
      const float r1 = x - a[k];
      b[k] = __bfloat162float(__float2bfloat16_rn(r1));
      c[k] = r1 - b[k];
    }
    const __nv_bfloat162 pa = __floats2bfloat162_rn(a[0], a[1]), pb = __floats2bfloat162_rn(b[0], b[1]),
                         pc = __floats2bfloat162_rn(c[0], c[1]);
    w0[i] = *reinterpret_cast<const uint32_t*>(&pa);
    w1[i] = *reinterpret_cast<const uint32_t*>(&pb);
    w2[i] = *reinterpret_cast<const uint32_t*>(&pc);
  }
  h0 = make_uint4(w0[0], w0[1], w0[2], w0[3]);
  h1 = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  h2 = make_uint4(w2[0], w2[1], w2[2], w2[3]);
}

// Parts of one warp's 32 x 32 chunk (staged as stg[m][n], row stride 33) into a layout with
// unit stride along m (sm == 1) or along n (sn == 1): each lane stores 8 consecutive values
// per part as one 16-byte vector (4 vectors per lane); other cases and ragged edges store
// element by element.
__device__ __forceinline__ void store_parts_chunk(__nv_bfloat16* const (&P)[3], int64_t off, int64_t sm, int64_t sn,
                                                  const float* stg, int lane, int mrow0, int ncol0, int M, int N) {
  const bool mcont = sm == 1, ncont = sn == 1 && !mcont;
  const int64_t other = mcont ? sn : sm;
  bool vec = (mcont || ncont) && (off % 8 == 0) && (other % 8 == 0);
#pragma unroll
  for (int i = 0; i < 3; ++i) vec = vec && (!P[i] || (reinterpret_cast<uintptr_t>(P[i]) & 15) == 0);
  const int q = lane & 3;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    // m-contiguous: column j = 8 pass + lane / 4, rows 8 q .. 8 q + 7
    // n-contiguous: row r = 8 pass + lane / 4, columns 8 q .. 8 q + 7
    const int a = 8 * pass + (lane >> 2);
    const int mm0 = mcont ? mrow0 + 8 * q : mrow0 + a;
    const int nn0 = mcont ? ncol0 + a : ncol0 + 8 * q;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = mcont ? stg[(8 * q + i) * 33 + a] : stg[a * 33 + 8 * q + i];
    const bool full = mcont ? (nn0 < N && mm0 + 7 < M) : (mm0 < M && nn0 + 7 < N);
    if (vec && full) {
      uint4 h0, h1, h2;
      parts8(v, h0, h1, h2);
      const int64_t o = off + (int64_t)mm0 * sm + (int64_t)nn0 * sn;
      *reinterpret_cast<uint4*>(P[0] + o) = h0;
      if (P[1]) *reinterpret_cast<uint4*>(P[1] + o) = h1;
      if (P[2]) *reinterpret_cast<uint4*>(P[2] + o) = h2;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int mm = mcont ? mm0 + i : mm0, nn = mcont ? nn0 : nn0 + i;
        if (mm < M && nn < N) put_parts(P, off + (int64_t)mm * sm + (int64_t)nn * sn, v[i]);
      }
    }
  }
}

constexpr int kEpiWarps = 8;                         // warps 4 .. 11
constexpr int kStgBytes = kEpiWarps * 32 * 33 * 4;   // epilogue staging: one 32 x 33 float chunk per warp

// Tile t of the launch: n tiles fastest (consecutive tiles of a CTA share A rows through L2),
// then m tiles, then the batch.
__device__ __forceinline__ void tile_coords(int t, int ntn, int ntm, int& n0, int& m0, int& b) {
  const int per_b = ntn * ntm;
  b = t / per_b;
  const int r = t - b * per_b;
  m0 = (r / ntn) * kTile;
  n0 = (r % ntn) * kTile;
}

// Persistent: CTA c takes the tiles c, c + gridDim.x, ... Warp 0 streams the operand tiles of
// all of them through the stage ring; warp 1 accumulates tile i in TMEM buffer i & 1 (two
// 128-column buffers), so that warps 4-11 read tile i back and store it while tile i + 1 is
// loaded and multiplied. Barriers: full / empty per stage (TMA bytes / MMA completion),
// acc_full per buffer (MMA completion), acc_empty per buffer (the eight epilogue warps).
template <int STAGES>
__global__ void __launch_bounds__(128 + 32 * kEpiWarps, 1) k_gemm_tc(const __grid_constant__ TcGemmParams p, int ntiles, int ntn,
                                                     int ntm) {
  extern __shared__ uint8_t smraw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_s;   // a wait ran out: every role stops at its next tile or k-block
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbl = p.b_same ? 0 : p.nb;   // B parts loaded per stage
  const int stage_bytes = (p.na + nbl) * kTileBytes;
  int npairs = p.npairs;
  int8_t pa[9], pb[9];
  if (npairs == 0) {
    npairs = p.na > p.nb ? p.na : p.nb;
    for (int t = 0; t < npairs; ++t) {
      pa[t] = (int8_t)(t < p.na ? t : p.na - 1);
      pb[t] = (int8_t)(t < p.nb ? t : p.nb - 1);
    }
  } else {
    for (int t = 0; t < npairs; ++t) {
      pa[t] = p.pair_a[t];
      pb[t] = p.pair_b[t];
    }
  }
  volatile int* abort_v = &abort_s;
  auto fail = [&]() {
    *abort_v = 1;
    atomicOr(p.status, ST_TIMEOUT);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&acc_full[j], 1);
      mbar_init(&acc_empty[j], kEpiWarps);
    }
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.na; ++i) prefetch_tensormap(&p.amap[i]);
    for (int i = 0; i < p.nb; ++i) prefetch_tensormap(&p.bmap[i]);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 2 * kTile);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (elect_one()) {
      uint32_t g = 0;   // k-blocks issued by this CTA (stage ring position)
      for (int t = blockIdx.x; t < ntiles && !*abort_v; t += gridDim.x) {
        int n0, m0, b;
        tile_coords(t, ntn, ntm, n0, m0, b);
        for (int kb = 0; kb < p.KB; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          if (!mbar_wait(&empty_bar[s], ((g / STAGES) & 1) ^ 1, kMaxPoll) || *abort_v) {
            fail();
            break;
          }
          uint8_t* st = smem + s * stage_bytes;
          mbar_arrive_expect_tx(&full_bar[s], (uint32_t)stage_bytes);
          for (int i = 0; i < p.na; ++i) view_load(p.av, &p.amap[i], st + i * kTileBytes, &full_bar[s], m0, kb, b);
          for (int i = 0; i < nbl; ++i)
            view_load(p.bv, &p.bmap[i], st + (p.na + i) * kTileBytes, &full_bar[s], n0, kb, b);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const bool a_mn = is_mn(p.av.mode), b_mn = p.b_same ? a_mn : is_mn(p.bv.mode);
      const uint32_t idesc = idesc_bf16_f32(kTile, kTile) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u);
      uint32_t g = 0;
      int i = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort_v; t += gridDim.x, ++i) {
        const int ab = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (!mbar_wait(&acc_empty[ab], (use & 1) ^ 1, kMaxPoll)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * kTile);
        bool ok = true;
        for (int kb = 0; kb < p.KB; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          if (!mbar_wait(&full_bar[s], (g / STAGES) & 1, kMaxPoll) || *abort_v) {
            fail();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * stage_bytes);
          for (int q = 0; q < npairs; ++q) {
            const int ia = pa[q], ib = pb[q];
            const uint32_t abase = st + ia * kTileBytes;
            const uint32_t bbase = p.b_same ? st + ib * kTileBytes : st + (p.na + ib) * kTileBytes;
            // K = 16 per MMA: 32 bytes along a K-major line, or 16 lines (two 8-line groups)
            // of an MN-major tile
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint64_t ad = a_mn ? desc_mnmajor_sw128(abase + k * 2048, kMnHalf, 1024)
                                       : desc_kmajor_sw128(abase + k * 32);
              const uint64_t bd = b_mn ? desc_mnmajor_sw128(bbase + k * 2048, kMnHalf, 1024)
                                       : desc_kmajor_sw128(bbase + k * 32);
              umma_bf16(d, ad, bd, idesc, (kb | q | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty_bar[s]);   // frees the stage once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
    }
  } else if (warp >= 4) {
    // a warp reaches TMEM lanes 32 (warp % 4) .. + 31 only: warps 4 + e and 8 + e share lane
    // quadrant e and take the first and the second half of the columns
    const int e = warp & 3, half = (warp - 4) >> 2;
    constexpr int kChunks = kTile / 32 / 2;       // 32-column chunks per warp and tile
    // Outputs contiguous along n (row-major C: c_sn = 1, or a part layout with unit n stride)
    // go through shared memory in 32 x 32 chunks, so that a store instruction covers
    // consecutive n of one row; outputs contiguous along m are stored from the registers
    // (consecutive lanes, consecutive m).
    float* stg = reinterpret_cast<float*>(smem + STAGES * stage_bytes) + (warp - 4) * (32 * 33);
    const bool has_c = p.C != nullptr;
    const bool c_n = has_c && p.c_sn == 1;
    const bool parts = p.ps[0] || p.pt[0];
    // float32 C goes out as 16-byte vectors, 8 lanes on 32 consecutive entries of one row (n
    // contiguous) or of one column (m contiguous), when the strides and the base allow it
    const int64_t c_other = c_n ? p.c_sm : p.c_sn;
    const bool c_vec = has_c && (p.c_sn == 1 || p.c_sm == 1) && (c_other % 4 == 0) && (p.c_sb % 4 == 0) &&
                       (p.c_batch_in <= 0 || p.c_sb_out % 4 == 0) && (reinterpret_cast<uintptr_t>(p.C) & 15) == 0;
    const int q8 = lane & 7, r4 = lane >> 3;
    int i = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
      const int ab = i & 1;
      const uint32_t use = (uint32_t)(i >> 1);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[ab], use & 1, kMaxPoll));   // warp-uniform
      if (!ok || *abort_v) {
        if (lane == 0 && !ok) fail();
        break;
      }
      tc_fence_after();
      int n0, m0, b;
      tile_coords(t, ntn, ntm, n0, m0, b);
      int64_t boff;
      if (p.c_batch_in > 0) boff = (int64_t)(b / p.c_batch_in) * p.c_sb_out + (int64_t)(b % p.c_batch_in) * p.c_sb;
      else boff = (int64_t)b * p.c_sb;
      float* C = has_c ? p.C + boff : nullptr;
      const int64_t poff = (int64_t)b * p.c_sb, toff = (int64_t)b * p.t_sb;
      const uint32_t tbase = tmem + (uint32_t)(ab * kTile) + ((uint32_t)(32 * e) << 16);
      const int mr0 = m0 + 32 * e;   // first row of this warp's chunks
#pragma unroll 1
      for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
        uint32_t r[32];
        tmem_ld32(tbase + (uint32_t)(c * 32), r);
        tmem_ld_wait();
        if (c == (half + 1) * kChunks - 1) {
          // the whole accumulator is in registers or staged: hand the buffer back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
        // staged as stg[m][n] (row stride 33: conflict-free by rows and by columns)
#pragma unroll
        for (int j = 0; j < 32; ++j) stg[lane * 33 + j] = __uint_as_float(r[j]);
        __syncwarp();
        const int nc0 = n0 + c * 32;
        if (has_c) {
          if (c_vec) {
            // lane = (vector q8 of 4 entries, line r4 + 4 k): n-contiguous lines are rows,
            // m-contiguous lines are columns
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int ln = r4 + 4 * k;
              const int mm = c_n ? mr0 + ln : mr0 + 4 * q8, nn = c_n ? nc0 + 4 * q8 : nc0 + ln;
              float4 v4;
              if (c_n) v4 = make_float4(stg[ln * 33 + 4 * q8], stg[ln * 33 + 4 * q8 + 1], stg[ln * 33 + 4 * q8 + 2],
                                        stg[ln * 33 + 4 * q8 + 3]);
              else v4 = make_float4(stg[(4 * q8) * 33 + ln], stg[(4 * q8 + 1) * 33 + ln], stg[(4 * q8 + 2) * 33 + ln],
                                    stg[(4 * q8 + 3) * 33 + ln]);
              float* dst = C + (int64_t)mm * p.c_sm + (int64_t)nn * p.c_sn;
              const bool full = c_n ? (mm < p.M && nn + 3 < p.N) : (nn < p.N && mm + 3 < p.M);
              if (full) {
                *reinterpret_cast<float4*>(dst) = v4;
              } else {
                const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int m2 = c_n ? mm : mm + u, n2 = c_n ? nn + u : nn;
                  if (m2 < p.M && n2 < p.N) C[(int64_t)m2 * p.c_sm + (int64_t)n2 * p.c_sn] = vv[u];
                }
              }
            }
          } else {
            const int m = mr0 + lane;
            if (m < p.M) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int n = nc0 + j;
                if (n < p.N) C[(int64_t)m * p.c_sm + (int64_t)n * p.c_sn] = stg[lane * 33 + j];
              }
            }
          }
        }
        if (parts) {
          if (p.ps[0]) store_parts_chunk(p.ps, poff, p.c_sm, p.c_sn, stg, lane, mr0, nc0, p.M, p.N);
          if (p.pt[0]) store_parts_chunk(p.pt, toff, p.t_sm, p.t_sn, stg, lane, mr0, nc0, p.M, p.N);
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 2 * kTile);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

}  // namespace

static bool map_box(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                    uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 2 || rank > 5) return false;
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t box[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    estr[i] = 1;
    box[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) {
    gstr[i] = strides[i];
    if (strides[i] % 16) return false;
  }
  if (reinterpret_cast<uintptr_t>(base) % 16) return false;
  box[0] = kBK;     // 64 bf16 = 128 bytes, the swizzle span
  box[1] = box1;
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), gdim, gstr,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tc_map_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides) {
  return map_box(map, base, rank, dims, strides, kTile);   // 64 K x 128 rows
}

bool tc_map_bf16_rows32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides) {
  return map_box(map, base, rank, dims, strides, 32);      // 64 entries x 32 rows
}

bool tc_map_bf16_x_mn(CUtensorMap* map, const void* X, int64_t L, int64_t H, int64_t T, int64_t D) {
  if (L <= 0 || H <= 0 || T <= 0 || D <= 0 || D % 8) return false;
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)T, (uint64_t)H, (uint64_t)L};
  const uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)(T * D * 2), (uint64_t)(H * T * D * 2)};
  return map_box(map, X, 4, dims, str, kBK);   // 64 features x 64 tokens
}

bool tc_map_bf16_mn(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int64_t batch) {
  if (rows <= 0 || K <= 0 || batch <= 0 || rows % 8) return false;
  const uint64_t dims[3] = {(uint64_t)rows, (uint64_t)K, (uint64_t)batch};
  const uint64_t str[2] = {(uint64_t)rows * 2, (uint64_t)(rows * K * 2)};
  return map_box(map, base, 3, dims, str, kBK);   // 64 rows x 64 K
}

cudaError_t gemm_tc(int batch, const TcGemmParams& p, cudaStream_t s) {
  if (batch <= 0 || p.M <= 0 || p.N <= 0) return cudaSuccess;
  if (p.na < 1 || p.na > 3 || p.nb < 1 || p.nb > 3 || batch > 65535 || p.npairs < 0 || p.npairs > 9)
    return cudaErrorInvalidValue;
  for (int t = 0; t < p.npairs; ++t)
    if (p.pair_a[t] < 0 || p.pair_a[t] >= p.na || p.pair_b[t] < 0 || p.pair_b[t] >= p.nb) return cudaErrorInvalidValue;
  if (p.b_same && (p.M > kTile || p.N > kTile || p.nb > p.na)) return cudaErrorInvalidValue;
  if ((p.av.ksplit > 0 && p.na != 1) || (p.bv.ksplit > 0 && p.nb != 1) || p.av.ksplit < 0 || p.bv.ksplit < 0)
    return cudaErrorInvalidValue;
  if ((p.av.mode == VIEW_MN && (p.av.D % 8 || p.av.H < 1)) || (p.bv.mode == VIEW_MN && (p.bv.D % 8 || p.bv.H < 1)))
    return cudaErrorInvalidValue;
  // X views: a tile's 128 rows lie within one head
  if (((p.av.mode == VIEW_MN_XFEAT || p.av.mode == VIEW_MN_XHEAD) && (p.av.D % kTile || p.av.H < 1)) ||
      ((p.bv.mode == VIEW_MN_XFEAT || p.bv.mode == VIEW_MN_XHEAD) && (p.bv.D % kTile || p.bv.H < 1)))
    return cudaErrorInvalidValue;
  if ((p.ps[0] || p.pt[0]) && p.c_batch_in > 0) return cudaErrorInvalidValue;
  const int stage_bytes = (p.na + (p.b_same ? 0 : p.nb)) * kTileBytes;
  const int ntn = (p.N + kTile - 1) / kTile, ntm = (p.M + kTile - 1) / kTile;
  const int64_t nt64 = (int64_t)ntn * ntm * batch;
  if (nt64 > INT32_MAX) return cudaErrorInvalidValue;
  const int ntiles = (int)nt64;
  static int nsm[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (nsm[dev] == 0) {
    e = cudaDeviceGetAttribute(&nsm[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int grid = ntiles < nsm[dev] ? ntiles : nsm[dev];
  // One persistent CTA per SM with the deepest ring (at most 6 stages) that fits next to the
  // epilogue staging buffer.
  constexpr int kAvail = 226 * 1024 - kStgBytes - 1024;
  int stages = kAvail / stage_bytes;
  if (stages > 6) stages = 6;
  if (stages == 5) stages = 4;
  if (stages < 2) return cudaErrorInvalidValue;
  const int smem = stages * stage_bytes + kStgBytes + 1024;
  switch (stages) {
    case 2:
      e = cudaFuncSetAttribute(k_gemm_tc<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_gemm_tc<2><<<grid, 128 + 32 * kEpiWarps, smem, s>>>(p, ntiles, ntn, ntm);
      break;
    case 3:
      e = cudaFuncSetAttribute(k_gemm_tc<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_gemm_tc<3><<<grid, 128 + 32 * kEpiWarps, smem, s>>>(p, ntiles, ntn, ntm);
      break;
    case 4:
      e = cudaFuncSetAttribute(k_gemm_tc<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_gemm_tc<4><<<grid, 128 + 32 * kEpiWarps, smem, s>>>(p, ntiles, ntn, ntm);
      break;
    default:
      e = cudaFuncSetAttribute(k_gemm_tc<6>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess) k_gemm_tc<6><<<grid, 128 + 32 * kEpiWarps, smem, s>>>(p, ntiles, ntn, ntm);
      break;
  }
  if (e != cudaSuccess) return e;
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
