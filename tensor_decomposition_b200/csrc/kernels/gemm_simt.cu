// Generic batched strided GEMM on the CUDA cores with float64 accumulation.
//
// It serves the small and oddly-strided contractions of the factor analysis (CholeskyQR
// Grams and triangular updates, Rayleigh-Ritz rotation U_T = Q W, the core projection
// G[h] = U_T^T X_h U_D of "A JoLT for the KV Cache" (arXiv 2607.12550v2, Abstract: "partial
// Tucker decomposition that compresses only the token and feature axes")). Operands are
// bf16 / fp32 / fp64 values, so every product is exact in float64 and only the sum rounds.
// Two-level index maps let the token unfolding X_(2)[t, h*D + d] = X[h][t][d] be read in place.
#include "../jolt_internal.h"

namespace jolt {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

__device__ __forceinline__ int64_t imap(const Idx2& x, int64_t i) {
  return x.in > 0 ? (i / x.in) * x.s_out + (i % x.in) * x.s_in : i * x.s_in;
}

template <typename T>
__device__ __forceinline__ double ldv(const void* p, int64_t off) {
  return (double)reinterpret_cast<const T*>(p)[off];
}
template <>
__device__ __forceinline__ double ldv<__nv_bfloat16>(const void* p, int64_t off) {
  return (double)__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[off]);
}

template <typename T>
__device__ __forceinline__ void load_tile(const Operand& op, int64_t boff, int rows, int K, int r0,
                                          int k0, double (*tile)[BM + 1]) {
  // tile[k][r], BK x BM; coalesce along whichever index is contiguous in memory.
  const bool row_fast = (op.row.in == 0 ? op.row.s_in == 1 : op.row.s_in == 1);
  for (int e = threadIdx.x; e < BM * BK; e += blockDim.x) {
    int r, k;
    if (row_fast) { r = e % BM; k = e / BM; }
    else { k = e % BK; r = e / BK; }
    const int gr = r0 + r, gk = k0 + k;
    double v = 0.0;
    if (gr < rows && gk < K) v = ldv<T>(op.p, boff + imap(op.row, gr) + imap(op.k, gk));
    tile[k][r] = v;
  }
}

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) k_gemm(int M, int N, int K, Operand A, Operand B,
                                              OutDesc C, double alpha, double beta) {
  __shared__ double As[BK][BM + 1];
  __shared__ double Bs[BK][BN + 1];
  const int b = blockIdx.z;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int64_t aoff = imap(A.batch, b), boff = imap(B.batch, b), coff = imap(C.batch, b);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  for (int k0 = 0; k0 < K; k0 += BK) {
    load_tile<TA>(A, aoff, M, K, m0, k0, As);
    load_tile<TB>(B, boff, N, K, n0, k0, Bs);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      double a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      TC* cp = reinterpret_cast<TC*>(C.p) + coff + imap(C.m, m) + imap(C.n, n);
      double v = alpha * acc[i][j];
      if (beta != 0.0) v += beta * (double)(*cp);
      *cp = (TC)v;
    }
  }
}

template <typename TA, typename TB>
cudaError_t launch_c(int batch, int M, int N, int K, const Operand& A, const Operand& B,
                     const OutDesc& C, double alpha, double beta, cudaStream_t s) {
  dim3 g((N + BN - 1) / BN, (M + BM - 1) / BM, batch);
  if (C.t == EL_F64)
    k_gemm<TA, TB, double><<<g, 256, 0, s>>>(M, N, K, A, B, C, alpha, beta);
  else
    k_gemm<TA, TB, float><<<g, 256, 0, s>>>(M, N, K, A, B, C, alpha, beta);
  note_launch();
  return cudaGetLastError();
}

template <typename TA>
cudaError_t launch_b(int batch, int M, int N, int K, const Operand& A, const Operand& B,
                     const OutDesc& C, double alpha, double beta, cudaStream_t s) {
  switch (B.t) {
    case EL_BF16: return launch_c<TA, __nv_bfloat16>(batch, M, N, K, A, B, C, alpha, beta, s);
    case EL_F32: return launch_c<TA, float>(batch, M, N, K, A, B, C, alpha, beta, s);
    default: return launch_c<TA, double>(batch, M, N, K, A, B, C, alpha, beta, s);
  }
}

}  // namespace

cudaError_t gemm_simt(int batch, int M, int N, int K, const Operand& A, const Operand& B,
                      const OutDesc& C, double alpha, double beta, cudaStream_t s) {
  if (batch <= 0 || M <= 0 || N <= 0) return cudaSuccess;
  if (batch > 65535) return cudaErrorInvalidValue;
  switch (A.t) {
    case EL_BF16: return launch_b<__nv_bfloat16>(batch, M, N, K, A, B, C, alpha, beta, s);
    case EL_F32: return launch_b<float>(batch, M, N, K, A, B, C, alpha, beta, s);
    default: return launch_b<double>(batch, M, N, K, A, B, C, alpha, beta, s);
  }
}

}  // namespace jolt
