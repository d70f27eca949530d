// Internal declarations shared by the host runtime (jolt_api.cpp) and the kernel files.
// Nothing here is part of the public C ABI (include/jolt.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/jolt.h"

namespace jolt {

constexpr int kD = 128;            // the supported head_dim
constexpr int kMaxL = 128;         // layers per stream
constexpr int kMaxLT = 2 * kMaxL;  // layer-tensors per stream
constexpr int kMaxGroups = 64;
constexpr int kMaxN = 128;         // largest in-shared-memory eigenproblem / sketch width
constexpr int kSketchRankCap = 256;   // token-rank cap of the randomized-SVD encoder's grid
constexpr int kMaxRank = 112;      // largest token rank implemented (sketch width rank + 16 <= kMaxN)
constexpr int kAlign = 256;        // byte alignment of every stream part

// Device status word bits (OR-ed by kernels, read by the host after a sync).
enum : int32_t { ST_NOT_CONVERGED = 1, ST_NONFINITE = 2, ST_INFEASIBLE = 4, ST_TIMEOUT = 8 };

// Per-stream metadata written on the device by the allocator and read by the
// residual-coding and decode kernels, so no host round trip sits inside encode.
struct StreamMeta {
  int32_t status;
  int32_t num_lt;
  int64_t body_bytes;
  double lambda[2];
  int32_t alloc[kMaxGroups][2][3];      // (r_t, r_d, b) per group and kind
  int32_t lt_rank[kMaxLT][3];           // (r_t, r_d, b) per layer-tensor
  int64_t off[kMaxLT][JOLT_NUM_PARTS];  // byte offset of each part in the body
  int64_t bytes_by_part[JOLT_NUM_PARTS];
};

// Counts kernel launches made by this library (read through jolt_launch_count).
void note_launch();

// ------------------------------------------------------------------ generic SIMT GEMM
// Index map with an optional second level: i -> (i / in) * s_out + (i % in) * s_in when
// in > 0, else i * s_in. It expresses the token unfolding X_(2)[t, h*D + d] = X[h][t][d]
// without copying X.
struct Idx2 {
  int64_t s_in = 0, s_out = 0;
  int32_t in = 0;
};
enum ElemType : int32_t { EL_BF16 = 0, EL_F32 = 1, EL_F64 = 2 };
struct Operand {
  const void* p = nullptr;
  ElemType t = EL_F32;
  Idx2 batch, row, k;  // row = m for the A operand, n for the B operand
};
struct OutDesc {
  void* p = nullptr;
  ElemType t = EL_F32;  // EL_F32 or EL_F64
  Idx2 batch, m, n;
};
// C[b](m, n) = alpha * sum_k A[b](m, k) * B[b](n, k) + beta * C[b](m, n), fp64 accumulation.
cudaError_t gemm_simt(int batch, int M, int N, int K, const Operand& A, const Operand& B,
                      const OutDesc& C, double alpha, double beta, cudaStream_t s);

// ------------------------------------------------------------------ kernels (launchers)
// Counter-based normals (SplitMix64 + Box-Muller), see rotation.cu.
cudaError_t gauss_f64(uint64_t seed, uint64_t stream_id, int64_t n, double* out, cudaStream_t s);
// Sketch matrices Omega_lt = bf16(N(0,1)) of shape [HD][l], lt in [0, n_lt) uses stream 2 + lt_id[lt].
// transposed = true stores element (i, j) at [j][i] (layout [l][HD]).
cudaError_t sketch_omega(uint64_t seed, const int32_t* lt_ids_host, int n_lt, int64_t HD, int l,
                         __nv_bfloat16* out, bool transposed, cudaStream_t s);
// Haar rotation from a D x D float64 Gaussian (Householder QR, signs of diag(R) moved into Q).
// Randomized Hadamard rotation diag(s) H / sqrt(D) of the seed's rotation stream (D a power of 2).
cudaError_t hadamard_pi(uint64_t seed, int D, float* Pi_f32, __nv_bfloat16* Pi_bf16, cudaStream_t s);
cudaError_t haar_from_gauss(const double* G, int D, float* Pi_f32, __nv_bfloat16* Pi_bf16,
                            cudaStream_t s);
// Batched two-sided cyclic Jacobi, n even, n <= 128; V columns = eigenvectors, eigenvalues
// descending. Sets ST_NOT_CONVERGED in *status when max_sweeps is reached.
cudaError_t jacobi_eig(int batch, int n, const float* A, int64_t sA, float* V, int64_t sV,
                       float* lam, int64_t sL, int max_sweeps, int32_t* status, cudaStream_t s);
// Eigenpairs of PSD matrices (n <= 128, float64 input) by one-sided Jacobi on a Cholesky
// factor; same output convention as jacobi_eig.
cudaError_t eig_psd(int batch, int n, const double* C, int64_t sC, float* V, int64_t sV, float* lam, int64_t sL,
                    int max_sweeps, int32_t* status, cudaStream_t s);
// Two independent batches in one launch (e.g. the feature and the token eigenproblems).
cudaError_t eig_psd2(int batch0, int n0, const double* C0, int64_t sC0, float* V0, int64_t sV0, float* lam0,
                     int64_t sL0, int batch1, int n1, const double* C1, int64_t sC1, float* V1, int64_t sV1,
                     float* lam1, int64_t sL1, int max_sweeps, int32_t* status, cudaStream_t s);
// The same two-batch eigenproblems by Householder tridiagonalisation, bisection, twisted
// factorisations and back-transformation (eig_small.cu); any n <= 128, status flags
// ST_NONFINITE for a non-finite input or result.
cudaError_t eig_small2(int batch0, int n0, const double* C0, int64_t sC0, float* V0, int64_t sV0, float* lam0,
                       int64_t sL0, int batch1, int n1, const double* C1, int64_t sC1, float* V1, int64_t sV1,
                       float* lam1, int64_t sL1, int32_t* status, cudaStream_t s);
// Leading eigenpairs of batch dense symmetric n x n float64 matrices (A, batch stride sA; A is
// overwritten) by Householder tridiagonalisation, bisection and inverse iteration (tridiag.cu):
// on return *Z points at the R eigenvectors, [batch][n][tridiag_rpad(R)] float64 (column r,
// eigenvalues descending; orthonormal to about eps ||A|| / gap), *lam at the R eigenvalues,
// [batch][tridiag_rpad(R)]. Both live in `scratch` (tridiag_scratch_doubles doubles).
int tridiag_rpad(int R);
size_t tridiag_scratch_doubles(int batch, int n, int R);
cudaError_t eig_top_dense(int batch, int n, int R, double* A, int64_t sA, double* scratch, double** Z,
                         double** lam, cudaStream_t s);
// Shifted-CholeskyQR helper: Rinv = inverse of chol(W + shift * trace(W)/n * I), W n x n.
cudaError_t chol_inv(int batch, int n, const double* W, int64_t sW, double* Rinv, int64_t sR,
                     double shift, int32_t* status, cudaStream_t s);
cudaError_t chol_inv_f32(int batch, int n, const float* W, int64_t sW, double* Rinv, int64_t sR,
                         double shift, int32_t* status, cudaStream_t s);
// Column sign rule: largest |entry| of each column positive (lowest index on ties).
// Signs are computed on U (rows x cols, row stride ldu) and applied to U and to the
// optional companion W (w_rows x cols, row stride ldw).
cudaError_t sign_fix(int batch, int rows, int cols, float* U, int64_t ldu, int64_t sU, float* W,
                     int w_rows, int64_t ldw, int64_t sW, cudaStream_t s);
// Round float -> bf16 (RNE) into two copies: bf16 and float-of-bf16.
cudaError_t round_bf16(int64_t n, const float* in, __nv_bfloat16* out_b, float* out_f, cudaStream_t s);
// Squared Frobenius norm (float64, fixed reduction order) of each of `batch` arrays of n elements.
// `scratch` holds batch * 64 doubles.
// A non-finite norm sets ST_NONFINITE in *status (when status is not null).
cudaError_t sumsq_batched(int batch, int64_t n, const void* x, ElemType t, int64_t stride,
                          double* out, double* scratch, int32_t* status, cudaStream_t s);
// Sum of squared differences and squared reference (float64), deterministic.
cudaError_t relfrob_partial(const void* ref, const void* approx, uint64_t n, ElemType t,
                            double* partials, int nblocks, double* out2, cudaStream_t s);
int relfrob_blocks(uint64_t n);
// Block cap of relfrob_blocks and capacity of the fixed scratch of the allocation-free
// variant; relfrob_static_scratch returns that scratch's device address for the current device
// (2 * kRelfrobStaticBlocks partial sums, then the two totals).
constexpr int kRelfrobStaticBlocks = 1184;
cudaError_t relfrob_static_scratch(double** p);

struct TableArgs {
  int n_lt, H, R, D, step;
  const int32_t* lt_ids;  // device [n_lt]: row of E written for buffer index i
  const float* Gmax;   // [n_lt][H][R][D]
  const double* xx;    // [n_lt]
  double* E;           // [2L][ngrid], row lt = 2*layer + kind
  int ngrid;           // 1 + (R/step)*(D/step)
};
cudaError_t energy_table(const TableArgs& a, cudaStream_t s);

struct DualArgs {
  int L, H, T, D, G, has_v, step, R, split;
  int nbits;
  int32_t bits[9];
  double phi[9];
  int64_t budget_pool[2];
  int ngrid;
  const double* E;    // [2L][ngrid] (lt = 2*layer + kind)
  double* unit_err;   // [G*2][nbits*ngrid] debug copy of the tables
  const int32_t* cand_order;   // [nbits*ngrid] candidates (bi * ngrid + grid) by (bytes, b, r_t, r_d)
  StreamMeta* meta;
  int tables_ready = 0;        // 1: unit_err is already filled (second dual of the measured-b refinement)
};
cudaError_t dual_allocate(const DualArgs& a, cudaStream_t s);
// Measured-b refinement: per-layer-tensor sums of the residual coder's partial errors
// meas_part [n_lt][H][nchunk][9] (fixed order) into meas_lt [n_lt][9], and the units' tables
// for the second dual: the measured error of each allowed b at the unit's chosen ranks (from
// meta->alloc), +inf at every other rank.
cudaError_t measured_tables(const DualArgs& a, const double* meas_part, int nchunk, double* meas_lt,
                            cudaStream_t s);

struct PackArgs {
  int n_lt, H, T, D, R;
  const int32_t* lt_ids;     // device [n_lt] -> lt index (2*layer + kind)
  const __nv_bfloat16* UT;   // [n_lt][T][R]
  const __nv_bfloat16* UD;   // [n_lt][D][D]
  const float* Gmax;         // [n_lt][H][R][D]
  const StreamMeta* meta;
  uint8_t* body;
};
cudaError_t pack_factors(const PackArgs& a, cudaStream_t s);

struct ResidualArgs {
  int n_lt, H, T, D;
  const int32_t* lt_ids;     // device [n_lt]
  const void* X[2];          // K, V base pointers [L][H][T][D]
  ElemType xt;
  const float* Pi;           // [D][D] float32
  const StreamMeta* meta;
  uint8_t* body;
  // measured-b refinement: measure = 1 writes no codes; every layer-tensor (whatever its b) adds
  // its exact squared quantisation error for each width in bits_mask (b = 0: ||y||^2) into
  // meas_part [n_lt][H][ceil(T / 256)][9], one fixed-order sum per CTA
  int measure = 0;
  uint32_t bits_mask = 0;
  double* meas_part = nullptr;
  // randomized Hadamard rotation (Pi = diag(s) H / sqrt(D), s = sign of Pi's first column):
  // y = FWHT((x - u M_h) * s) / sqrt(D) with M_h = G_h U_D^T, the rotation as log2(D) butterfly
  // stages instead of a D x D product
  int hadamard = 0;
  // scratch [D][132] float32 for Pi^T in the coder's shared-memory layout (written by
  // residual_encode)
  float* PiT = nullptr;
};
// Pbuf: float64 scratch [n_lt][D][D] for P = U_D^T Pi; Nbuf: float64 scratch [n_lt][H][D][R + 4]
// for -N_h^T (N_h = G_h P) in the coder's shared-memory layout (row stride r_t + 4).
cudaError_t residual_encode(const ResidualArgs& a, double* Pbuf, double* Nbuf, int R, cudaStream_t s);

struct DecodeArgs {
  int n_lt, L, H, T, D;
  const int32_t* lt_ids;     // device [n_lt]
  void* out[2];              // K_out, V_out
  ElemType ot;
  const float* Pi;           // [D][D] float32
  const StreamMeta* meta;
  const uint8_t* body;
};
cudaError_t decode(const DecodeArgs& a, cudaStream_t s);

// Attention over the compressed cache (attention.cu): out = softmax(scale Q K_hat^T) V_hat per
// query, K_hat / V_hat never formed. Q, out: [L][Hq][n][D]; query head j reads KV head j / (Hq/H).
struct AttnArgs {
  int L, H, T, D, Hq, n, R;      // R: the stream's largest token rank (>= 1)
  float scale;
  const StreamMeta* meta;
  const uint8_t* body;
  const float* Pi;               // [D][D]
  const __nv_bfloat16* Q;
  float* out;
  float* qpi;                    // scratch [L][Hq][n][D]
  float* qhat;                   // scratch [L][Hq][n][R]
  float* part;                   // scratch [L][H][nchunk][ngroups][attn_part_floats(R)]
  int nchunk, ngroups;
};
int attn_groups(int Hq, int H, int n);
int attn_chunks(int T);
int attn_part_floats(int R);
cudaError_t attention(const AttnArgs& a, cudaStream_t s);

// Layout helpers of the tensor-core path (layout.cu).
cudaError_t split_bf16(int64_t n, const float* x, __nv_bfloat16* p0, __nv_bfloat16* p1, __nv_bfloat16* p2,
                       cudaStream_t s);
cudaError_t sum_heads(int n, int H, int64_t per, const float* part, float* out32, double* out64, cudaStream_t s);
// bf16 parts (3) of batch R x C float32 / float64 matrices, in the same and/or transposed layout.
cudaError_t split_dual(int batch, int R, int C, const void* in, bool in_f64, __nv_bfloat16* const* same,
                       __nv_bfloat16* const* tr, cudaStream_t s);

// Check for NaN/Inf in an input tensor (sets ST_NONFINITE).
cudaError_t check_finite(int64_t n, const void* x, ElemType t, int32_t* status, cudaStream_t s);

}  // namespace jolt
