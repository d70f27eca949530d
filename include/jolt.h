/*
 * jolt.h - C ABI of the JoLT KV-cache codec for NVIDIA B200 (sm_100a).
 *
 * The method is the one of "A JoLT for the KV Cache: Near-Lossless KV Cache Compression
 * via Joint Tucker and JL-Residual Allocation for LLMs" (arXiv 2607.12550v2, Abstract):
 * each layer's key (or value) cache X in R^{H x T x D} (heads x tokens x features) gets a
 * partial Tucker decomposition over the token and feature axes only,
 *     X[h] ~ U_T G[h] U_D^T,   U_T: T x r_t,  U_D: D x r_d,  G: H x r_t x r_d,
 * the truncation residual is rotated by a seeded random orthogonal D x D matrix and
 * quantised to b bits per entry with one fp16 scale per row, and a single Lagrangian dual
 * picks (r_t, r_d, b) per layer group, separately for K and V, under one byte budget.
 * The randomized-SVD token factor is the Abstract's "FlashJoLT" variant. Decode rebuilds
 * G x2 U_T x3 U_D plus the inverse-rotated, dequantised residual.
 *
 * Conventions for every entry point:
 *  - Tensors are row-major [layers][heads][tokens][head_dim] on the CUDA device that is
 *    current when the call is made. Pointers marked "device" must be device pointers
 *    (cudaMalloc / PyTorch CUDA storage), pointers marked "host" must be host memory.
 *  - `cuda_stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Encode and decode enqueue work on it and return without waiting for the device.
 *  - Every function returns a jolt_status. On failure, jolt_last_error() returns a
 *    message for the calling thread. Nothing aborts the process.
 *  - Errors found on the device (Jacobi not converged, non-finite input, spin timeout)
 *    are recorded in a status word of the stream object; they surface at the next call
 *    that synchronises (jolt_stream_status, jolt_stream_info, jolt_stream_to_host).
 *  - The caller owns input and output tensors. The library owns plans and streams and
 *    their device memory; release them with jolt_plan_destroy / jolt_stream_destroy.
 *  - A plan holds one workspace: encodes that share a plan must be issued on one CUDA
 *    stream (or otherwise serialised).
 *
 * The library supports head_dim == 128 and a batch of one sequence per stream. The candidate
 * token ranks run to R = min(T, H*D, byte_budget / (layer-tensors * 2T)), at most 256 for the
 * randomized-SVD encoder and at most jolt_config.rt_max when that is set; the kernels implement
 * R <= 112 (sketch width R + oversample <= 128), and jolt_plan refuses a larger R with
 * JOLT_ERR_UNSUPPORTED (set rt_max <= 112).
 */
#ifndef JOLT_H
#define JOLT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define JOLT_API __declspec(dllexport)
#else
#define JOLT_API __attribute__((visibility("default")))
#endif

typedef enum {
  JOLT_OK = 0,
  JOLT_ERR_INVALID_ARG = 1,       /* bad shape, pointer, size or option */
  JOLT_ERR_BUDGET_INFEASIBLE = 2, /* the smallest allowed choices exceed the byte budget */
  JOLT_ERR_OOM = 3,               /* device allocation failed */
  JOLT_ERR_CUDA = 4,              /* a CUDA runtime call failed (message names it) */
  JOLT_ERR_NOT_CONVERGED = 5,     /* an eigensolver hit its sweep limit (result still usable) */
  JOLT_ERR_NONFINITE = 6,         /* NaN or Inf met in the input */
  JOLT_ERR_TIMEOUT = 7,           /* a bounded device wait gave up */
  JOLT_ERR_CORRUPT_STREAM = 8,    /* bad magic, version, size or CRC in a serialized stream */
  JOLT_ERR_UNSUPPORTED = 9        /* valid request outside what the library implements */
} jolt_status;

typedef enum { JOLT_BF16 = 0, JOLT_F32 = 1 } jolt_dtype;

typedef enum { JOLT_ENC_AUTO = 0, JOLT_ENC_EXACT = 1, JOLT_ENC_SKETCH = 2 } jolt_encoder;

typedef enum { JOLT_EIG_TRIDIAG = 0, JOLT_EIG_JACOBI = 1 } jolt_eig_solver;

/* Shape of one sequence's cache. `dtype` is both the input and the decoded output type. */
typedef struct {
  int32_t layers, heads, tokens, head_dim;
  int32_t has_v;      /* 0: keys only (V pointers are ignored), 1: keys and values */
  jolt_dtype dtype;
} jolt_shape;

/* Codec options; jolt_config_default() fills the defaults shown. */
typedef struct {
  jolt_encoder encoder;      /* AUTO (default): exact if tokens <= 1024, else sketch */
  int32_t oversample;        /* sketch oversampling p (16) */
  int32_t power_iters;       /* sketch power iterations q (1) */
  int32_t rank_step;         /* candidate ranks are multiples of this (16) */
  int32_t rt_max;            /* cap on the candidate token ranks; 0 = none beyond the grid's own
                                (see the preamble); plans need R <= 112 */
  uint32_t bits_mask;        /* bit b set => residual bit-width b allowed (0x1FF = 0..8) */
  int32_t split_kv_budget;   /* 0: one budget pool for K and V; 1: half the budget each */
  int32_t max_jacobi_sweeps; /* sweep limit of the Jacobi eigensolver (30; eig_solver = JACOBI) */
  int32_t factors;           /* 1 (default): Tucker factors on the candidate grid; 0: residual
                                only, r_t = r_d = 0 for every layer-tensor (with bits_mask = 1 << b
                                this is per-row b-bit quantisation of the rotated cache, the
                                quantisation-only in-codec baseline; the factor analysis is
                                skipped). The Tucker-only baseline is bits_mask = 1 (b = 0). */
  int32_t measured_b;        /* 0 (default): the dual's errors use the phi(b) quantiser model.
                                1: measured-b refinement: after the dual, one extra pass of the
                                residual coder measures the exact squared error of every allowed
                                b at each unit's chosen ranks, and a second dual re-chooses b per
                                unit with those errors (ranks unchanged). */
  int32_t rotation;          /* 0 (default): Haar rotation Pi (Q factor of a Gaussian matrix);
                                1: randomized Hadamard Pi = diag(s) H / sqrt(D), s random signs of
                                the seed's rotation stream, H the Sylvester Hadamard matrix (D a
                                power of two); recorded in the stream header */
  jolt_eig_solver eig_solver; /* solver of the feature and sketch eigenproblems (n <= 128):
                                TRIDIAG (default): Householder tridiagonalisation, bisection,
                                twisted-factorisation vectors, back-transformation; JACOBI:
                                one-sided Jacobi on a Cholesky factor, to convergence */
} jolt_config;

typedef struct jolt_plan_s* jolt_plan_t;
typedef struct jolt_stream_s* jolt_stream_t;

/* Parts of a stream, in the order they are laid out and counted. */
enum { JOLT_PART_UT = 0, JOLT_PART_UD = 1, JOLT_PART_G = 2, JOLT_PART_SCALES = 3,
       JOLT_PART_CODES = 4, JOLT_NUM_PARTS = 5 };

/* Debug exports (parity tests): see jolt_export_debug. */
enum { JOLT_DBG_PI = 0,        /* float32 [D][D] rotation Pi used by encode */
       JOLT_DBG_UT_F32 = 1,    /* float32 [T][R] token factor before bf16 rounding, layer-tensor lt */
       JOLT_DBG_UD_F32 = 2,    /* float32 [D][D] feature factor before bf16 rounding, lt */
       JOLT_DBG_TABLE = 3,     /* float64 per-unit error table, unit = lt (group*2 + kind) */
       JOLT_DBG_XX = 4,        /* float64 [2*L] squared Frobenius norm of every layer-tensor */
       JOLT_DBG_LAMBDA = 5,    /* float64 [2] dual variable of each budget pool */
       JOLT_DBG_OMEGA = 6,     /* bf16 bits [HD][l] sketch matrix of layer-tensor lt */
       JOLT_DBG_MEAS = 7 };    /* float64 [9] measured squared error of residual width b (index b,
                                  zero for widths not allowed) at the chosen ranks, layer-tensor
                                  lt; plans with measured_b = 1 only */

JOLT_API void jolt_config_default(jolt_config* cfg);

/*
 * jolt_plan - validate a shape and budget and reserve the encode workspace.
 *
 * byte_budget: bytes the whole stream may spend on stored factors, cores, packed codes and
 *   scales (the "one byte budget" of the Abstract); the header and alignment padding are
 *   not counted. A compression ratio N means byte_budget = bf16 bytes of the cache / N.
 * num_groups: layers are split into contiguous groups, group g holding layers
 *   [g*L/G, (g+1)*L/G); each group picks its own (r_t, r_d, b) for K and for V.
 * cfg: NULL for defaults.
 * Errors: INVALID_ARG (non-positive sizes, head_dim != 128, groups > layers, bad options),
 *   BUDGET_INFEASIBLE (the cheapest allowed choice of every group exceeds the budget),
 *   UNSUPPORTED (the candidate grid's largest token rank exceeds 112, see the preamble),
 *   OOM, CUDA. On success *out owns device workspace until jolt_plan_destroy.
 */
JOLT_API jolt_status jolt_plan(const jolt_shape* shape, uint64_t byte_budget, int32_t num_groups,
                               const jolt_config* cfg, jolt_plan_t* out);

/* Plan facts: largest token rank R, sketch width l (0 for exact), encoder used, workspace
 * bytes. Any output pointer may be NULL. */
JOLT_API jolt_status jolt_plan_info(jolt_plan_t plan, int32_t* rt_max, int32_t* sketch_l,
                                    int32_t* encoder, uint64_t* workspace_bytes);

/*
 * jolt_encode - compress one sequence's cache (device K, and V when the shape has V).
 *
 * K, V: device tensors [L][H][T][D] of the plan's dtype. They are only read.
 * seed: selects the rotation Pi (the Abstract's random orthogonal rotation) and the sketch
 *   matrices; it is stored in the stream so decode can rebuild Pi.
 * Phases, all on `cuda_stream`: factor analysis of every layer-tensor (Gram / sketch GEMMs,
 *   Jacobi eigensolver, CholeskyQR, core projection, error table), the Lagrangian dual over
 *   all groups, then residual coding. The host does not wait for the device.
 * *out: a device-resident stream owned by the caller until jolt_stream_destroy.
 */
JOLT_API jolt_status jolt_encode(jolt_plan_t plan, const void* K, const void* V, uint64_t seed,
                                 void* cuda_stream, jolt_stream_t* out);

/*
 * jolt_decode - rebuild the cache: X_hat[h] = U_T G[h] U_D^T + dequant(codes) Pi^T.
 *
 * K_out, V_out: device tensors [L][H][T][D] of the stream's dtype (bf16 output is rounded to
 *   nearest even). V_out is ignored for a keys-only stream. Enqueued on `cuda_stream`.
 */
JOLT_API jolt_status jolt_decode(jolt_stream_t stream, void* K_out, void* V_out, void* cuda_stream);

/*
 * jolt_attention - attention of a few queries per head over the compressed cache of a stream,
 *   for every layer, without rebuilding the cache:
 *       out[l][j][i] = sum_t softmax_t(scale * Q[l][j][i] . K_hat[l][h][t]) V_hat[l][h][t],
 *   h = j / (q_heads / heads) (grouped-query attention; q_heads = heads is multi-head). K_hat and
 *   V_hat are the stream's reconstructions G x2 U_T x3 U_D + dequant(codes) Pi^T, used in factored
 *   form: scores from U_T, G_h U_D^T q, the codes, the scales and Pi^T q; the value sum from the
 *   softmax-weighted sums of U_T rows and of scaled cell centres, mapped back through G_h, U_D, Pi.
 *   The method's pages compress the cache that attention reads (Abstract); this consumer of the
 *   stream is this library's own, with the same linear algebra as the decode.
 * Q: device bf16 [layers][q_heads][n_queries][head_dim]; out: device float32, same shape. The
 *   stream must hold K and V (bf16). Enqueued on `cuda_stream`; takes scratch from the library's
 *   memory pool. Errors: INVALID_ARG (null pointers, q_heads not a multiple of the KV heads, no V),
 *   UNSUPPORTED (float32 streams).
 */
JOLT_API jolt_status jolt_attention(jolt_stream_t stream, const void* Q, int32_t q_heads, int32_t n_queries,
                                    float scale, float* out, void* cuda_stream);

/*
 * jolt_rel_frob_error - ||ref - approx||_F / ||ref||_F over n elements (the error measure the
 *   Abstract reports), accumulated in float64. ref, approx: device arrays of `dtype`.
 *   Synchronises `cuda_stream`; *out is host memory. Returns 0 when ||ref|| = 0.
 */
JOLT_API jolt_status jolt_rel_frob_error(const void* ref, const void* approx, uint64_t n,
                                         jolt_dtype dtype, void* cuda_stream, double* out);

/*
 * jolt_rel_frob_error_noalloc - the value jolt_rel_frob_error returns, computed with the same
 *   kernels, grid and reduction order, but without allocating anything: the per-block partial
 *   sums and the two totals live in one fixed device array inside the library, of
 *   2 * 1184 + 2 float64 (18,960 bytes) per device. The method has no counterpart of this
 *   entry point (the paper only defines the error measure); it exists for callers that must
 *   not allocate device memory.
 *
 *   Arguments, layout and the result are those of jolt_rel_frob_error; ref and approx must be
 *   on the current device. n above JOLT_REL_FROB_NOALLOC_MAX_N returns JOLT_ERR_INVALID_ARG
 *   (any smaller n fits the fixed scratch: the grid is capped at 1184 blocks).
 *   Every call looks up the array's device address in the current context (a symbol lookup,
 *   no allocation), so calls after cudaDeviceReset or a new primary context stay valid. The
 *   call synchronises `cuda_stream` (it cannot be captured in a CUDA graph). The array is shared
 *   by every caller on a device: overlapping calls (other threads, or other streams) race on it
 *   and may return wrong values.
 */
#define JOLT_REL_FROB_NOALLOC_MAX_N (1ULL << 62)
JOLT_API jolt_status jolt_rel_frob_error_noalloc(const void* ref, const void* approx, uint64_t n,
                                                 jolt_dtype dtype, void* cuda_stream, double* out);

/* Synchronise on the stream's CUDA stream and report device-side errors of its encode. */
JOLT_API jolt_status jolt_stream_status(jolt_stream_t stream);

/*
 * jolt_stream_info - synchronise and report the allocation and the stored bytes.
 * bytes_by_part: host [5] bytes of U_T, U_D, G, scales, codes over all layer-tensors (or NULL).
 * alloc: host [num_groups][2][3] (r_t, r_d, b) per group and kind (or NULL).
 * lambdas: host [2] dual variable of each pool (or NULL).
 */
JOLT_API jolt_status jolt_stream_info(jolt_stream_t stream, uint64_t* bytes_by_part,
                                      int32_t* alloc, double* lambdas);

/*
 * jolt_stream_to_host - serialize: header (magic "JOLT", version 1, flags (bit 0 has V, bit 1
 *   float32 output, bit 2 separate K/V budgets, bit 3 randomized Hadamard rotation, bits 8..15
 *   encoder), shape, seed, allocation table), body (per layer-tensor lt = 2*layer + kind: U_T [T][r_t] bf16, U_D [D][r_d] bf16,
 *   G [H][r_t][r_d] bf16, scales [H][T] fp16, codes [H][T][D*b/8] bytes with code i at bits
 *   [i*b, i*b+b) LSB first; each part starts at a multiple of 256 bytes), then CRC-32.
 * buf: host buffer of *len bytes, or NULL to query the size into *len.
 */
JOLT_API jolt_status jolt_stream_to_host(jolt_stream_t stream, void* buf, uint64_t* len);

/* jolt_stream_from_host - parse a serialized stream (checks magic, version, sizes, CRC)
 * into a new device stream; Pi is rebuilt from the stored seed (and rotation kind) on `cuda_stream`. */
JOLT_API jolt_status jolt_stream_from_host(const void* buf, uint64_t len, void* cuda_stream,
                                           jolt_stream_t* out);

/* jolt_export_debug - copy an internal array (JOLT_DBG_*) of the last encode to host memory.
 * lt selects the layer-tensor (or unit for JOLT_DBG_TABLE). buf NULL queries *len. Syncs. */
JOLT_API jolt_status jolt_export_debug(jolt_stream_t stream, int32_t what, int32_t lt, void* buf,
                                       uint64_t* len);

/* Tracing. jolt_profile_enable(1) brackets every encode / decode / error phase with CUDA
 * events recorded on the stream the phase runs on, and counts the kernel launches inside it.
 * jolt_profile_report synchronises the device, writes a JSON object
 * {"phase": {"calls": n, "launches": k, "total_ms": t}, ...} (NUL-terminated; buf NULL queries
 * *len) and clears the records. jolt_launch_count returns the number of kernels this library
 * has launched since it was loaded; jolt_alloc_count the number of device allocations it has
 * requested (plan workspaces, stream bodies, scratch), whether served by the driver or by the
 * library's memory pool. */
JOLT_API jolt_status jolt_profile_enable(int32_t on);
JOLT_API jolt_status jolt_profile_report(char* buf, uint64_t* len);
JOLT_API uint64_t jolt_launch_count(void);
JOLT_API uint64_t jolt_alloc_count(void);

/* jolt_selftest_gemm_bf16 - C = A B^T on the tensor cores (tcgen05.mma with TMA tile loads),
 * the building block of the factor analysis, exposed so its numerics can be tested alone.
 * A: device bf16 [M][K], B: device bf16 [N][K] (row-major, K contiguous, K a multiple of 8),
 * C: device float32 [M][N]. Products are exact, sums are float32. Synchronises `cuda_stream`;
 * returns JOLT_ERR_TIMEOUT if a bounded wait inside the kernel gave up. */
JOLT_API jolt_status jolt_selftest_gemm_bf16(int32_t M, int32_t N, int32_t K, const void* A, const void* B,
                                             float* C, void* cuda_stream);

/* jolt_selftest_gemm_bf16_layout - the same product with either operand stored transposed, as
 * the analysis keeps its bf16 bases (the operand then enters the MMA MN-major): A is [M][K]
 * (a_mn = 0) or [K][M] (a_mn = 1), B is [N][K] (b_mn = 0) or [K][N] (b_mn = 1); a transposed
 * operand needs M (N) a multiple of 8. Otherwise as jolt_selftest_gemm_bf16. */
JOLT_API jolt_status jolt_selftest_gemm_bf16_layout(int32_t M, int32_t N, int32_t K, const void* A, int32_t a_mn,
                                                    const void* B, int32_t b_mn, float* C, void* cuda_stream);

/* jolt_selftest_eig_dense - the R largest eigenvalues (descending) and their eigenvectors of
 * `batch` dense symmetric n x n float64 matrices, by the solver of the exact token factor above 128
 * tokens (Householder tridiagonalisation, bisection, inverse iteration, back-transformation, then
 * two CholeskyQR passes), exposed so its numerics can be tested alone.
 * A: device float64 [batch][n][n] (only read), V: device float64 [batch][n][R] (eigenvector r in
 * column r), lam: device float64 [batch][R]. 2 <= n <= 4096, 1 <= R <= min(n, 128). Allocates its
 * own scratch; synchronises `cuda_stream`; NOT_CONVERGED when the vectors were too close to
 * dependent for the re-orthonormalisation. */
JOLT_API jolt_status jolt_selftest_eig_dense(int32_t batch, int32_t n, int32_t R, const double* A, double* V,
                                             double* lam, void* cuda_stream);

/* jolt_selftest_eig_small - all n eigenpairs of `batch` dense symmetric n x n float64 matrices by
 * the solver of the feature and sketch eigenproblems (`solver`: JOLT_EIG_TRIDIAG or
 * JOLT_EIG_JACOBI), exposed so its numerics can be tested alone.
 * A: device float64 [batch][n][n] (the lower triangle is read), V: device float32 [batch][n][n]
 * (eigenvector r in column r), lam: device float32 [batch][n], eigenvalues descending.
 * 1 <= n <= 128. Synchronises
 * `cuda_stream`; NOT_CONVERGED when Jacobi reached its sweep limit, NONFINITE for a non-finite
 * input or result. */
JOLT_API jolt_status jolt_selftest_eig_small(int32_t batch, int32_t n, const double* A, float* V, float* lam,
                                             int32_t solver, void* cuda_stream);

/* Release a stream. Its device memory is freed in order on the CUDA stream the stream was
 * created on (encode or jolt_stream_from_host); synchronise any other CUDA stream that still
 * reads it (e.g. a decode issued elsewhere) before destroying it. */
JOLT_API void jolt_stream_destroy(jolt_stream_t stream);
JOLT_API void jolt_plan_destroy(jolt_plan_t plan);

/* Message of the last failed call on this thread ("" if none). */
JOLT_API const char* jolt_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* JOLT_H */
