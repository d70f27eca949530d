// Host-visible description of the tensor-core GEMM (gemm_tc.cu). Separate from
// jolt_internal.h because it needs the driver API's CUtensorMap type.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace jolt {

// How an operand's 128-row x 64-column tiles are addressed in its tensor map.
enum TcViewMode : int32_t {
  VIEW_ROWS_K = 0,        // 3-D map (K, rows, batch)
  VIEW_X_TOKENROWS = 1,   // 4-D map of X [L][H][T][D] as (D, T, H, L): rows = tokens, K = (head, feature)
  VIEW_ROWS_K_HEAD = 3,   // 4-D map (K, rows, H, n), batch index = i * H + h (e.g. K-chunked Grams:
                          // (chunk entries, rows, chunk, i))
  VIEW_MN = 4,            // 3-D map (rows, K, batch) from tc_map_bf16_mn, rows contiguous: the operand
                          // enters the MMA MN-major (two 64-row halves per tile); batch index b / H,
                          // row offset (b % H) * D (D a multiple of 8)
  VIEW_MN_XFEAT = 5,      // 4-D map of X [L][H][T][D] as (D, T, H, L) from tc_map_bf16_x_mn, MN-major:
                          // rows = (head, feature) (a tile within one head: D a multiple of 128),
                          // K = tokens, batch = layer
  VIEW_MN_XHEAD = 6       // same map, batch index = layer * H + head: rows = features, K = tokens
};

struct TcView {
  int32_t mode = VIEW_ROWS_K;
  int32_t D = 128;
  int32_t H = 1;   // VIEW_ROWS_K: batch index divisor (operands shared by H consecutive batches)
  // K split: with nch > 1 the batch index is (b / nch, chunk = b % nch) and chunk covers the
  // 64-entry K blocks [chunk * ckb, chunk * ckb + ckb) of the view
  int32_t nch = 1;
  int32_t ckb = 0;
  // Two sources: batch indices (after the K split) >= ksplit read the operand's next map
  // (maps[i + 1]; single-part operands only) at index b - ksplit. 0: one source.
  int32_t ksplit = 0;
};

struct TcGemmParams {
  CUtensorMap amap[3];
  CUtensorMap bmap[3];
  TcView av, bv;
  int32_t na = 1, nb = 1;   // bf16 parts of A and B
  // Products summed into the accumulator: A part pair_a[i] times B part pair_b[i]. With
  // npairs = 0 the products are (t, t) for t < max(na, nb), each index clamped to its count.
  int32_t npairs = 0;
  int8_t pair_a[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  int8_t pair_b[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  int32_t b_same = 0;       // 1: B is A (same maps, same tile: M = N <= 128); B tiles are not loaded
  int32_t M = 0, N = 0, KB = 0;
  float* C = nullptr;       // C[b] + m * c_sm + n * c_sn
  int64_t c_sm = 0, c_sn = 0, c_sb = 0, c_sb_out = 0;
  int32_t c_batch_in = 0;   // > 0: batch offset = (b / c_batch_in) * c_sb_out + (b % c_batch_in) * c_sb
  // Optional bf16 parts of the float32 result (v = p0 + p1 + p2, ~2^-24 relative), written in
  // C's layout (ps[i] + b * c_sb + m * c_sm + n * c_sn) and/or a second layout (pt[i] + b * t_sb
  // + m * t_sm + n * t_sn); null parts are skipped, C may be null. Not with c_batch_in.
  __nv_bfloat16* ps[3] = {nullptr, nullptr, nullptr};
  __nv_bfloat16* pt[3] = {nullptr, nullptr, nullptr};
  int64_t t_sm = 0, t_sn = 0, t_sb = 0;
  int32_t* status = nullptr;
};

// 2-D..5-D bf16 tensor map with a 64 x 128 box and 128-byte swizzle. dims[0] is the
// contiguous dimension; strides[i] is the byte stride of dims[i + 1]. False if the driver
// entry point is missing or an alignment rule fails.
bool tc_map_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides);

// The same with a 64 x 32 box (tiles of 32 rows, e.g. one warp's rows of a stored tile).
bool tc_map_bf16_rows32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides);

// [batch][K][rows] bf16 (rows contiguous, rows a multiple of 8) as the 3-D map (rows, K, batch)
// with a 64 x 64 box, for VIEW_MN operands.
bool tc_map_bf16_mn(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int64_t batch);

// X [L][H][T][D] bf16 as the 4-D map (D, T, H, L) with a 64 x 64 box, for VIEW_MN_XFEAT and
// VIEW_MN_XHEAD operands.
bool tc_map_bf16_x_mn(CUtensorMap* map, const void* X, int64_t L, int64_t H, int64_t T, int64_t D);

cudaError_t gemm_tc(int batch, const TcGemmParams& p, cudaStream_t s);

}  // namespace jolt
