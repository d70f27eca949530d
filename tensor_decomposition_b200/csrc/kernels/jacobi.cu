// Batched symmetric eigensolver (two-sided cyclic Jacobi) and the Cholesky-inverse step of
// shifted CholeskyQR, both held in shared memory, one CTA per matrix.
//
// They solve the small factor problems of the JoLT codec ("A JoLT for the KV Cache",
// arXiv 2607.12550v2, Abstract): the feature factor U_D from the eigenvectors of
// C_D = sum_h X_h^T X_h (D x D), and, for the randomized-SVD ("FlashJoLT") token factor,
// the Rayleigh-Ritz rotation W from B B^T (l x l) and the orthonormalisation of sketches.
//
// Jacobi: n even, n <= 128. Each sweep runs n - 1 rounds of the circle-method tournament,
// so a round rotates n/2 disjoint (p, q) pairs at once. The rotation is the symmetric Schur
// 2x2 step (Golub & Van Loan, Matrix Computations, sec. 8.5): tau = (a_qq - a_pp) / (2 a_pq),
// t = sign(tau) / (|tau| + sqrt(1 + tau^2)), c = 1 / sqrt(1 + t^2), s = t c, and
// A <- J^T A J with J_pp = c, J_pq = s, J_qp = -s, J_qq = c. A is held in float32; the
// rotations and the accumulated eigenvectors V are float64, so V stays orthonormal to
// ~1e-15 however many rounds run (float32 V drifts off unit norm). A pair is skipped when
// |a_pq| <= 1e-7 sqrt(|a_pp a_qq|) or |a_pq| <= 1e-10 max_i |a_ii|; a sweep without any
// rotation ends the solve. Eigenvalues are returned in descending order with their
// eigenvector columns (no sign normalisation here).
#include "../jolt_internal.h"

namespace jolt {
namespace {

constexpr int kLd = kMaxN + 1;   // padded row stride of the shared matrices

__device__ __forceinline__ int tour_player(int pos, int r, int n) {
  return pos == 0 ? 0 : ((pos - 1 + r) % (n - 1)) + 1;
}

__global__ void __launch_bounds__(512) k_jacobi(int n, const float* Ain, int64_t sA, float* Vout,
                                                int64_t sV, float* lam, int64_t sL, int max_sweeps,
                                                int32_t* status) {
  extern __shared__ double smd[];
  double* V = smd;                      // n x kLd, float64: stays orthogonal over many rounds
  double* csd = V + kMaxN * kLd;        // c[64], s[64] in float64
  float* A = reinterpret_cast<float*>(csd + kMaxN);   // n x kLd
  float* cs = A + kMaxN * kLd;          // c[64], s[64] in float32 for the A update
  int* pq = reinterpret_cast<int*>(cs + kMaxN);  // p[64], q[64]
  int* rank = pq + kMaxN;               // n
  __shared__ int rotated;
  __shared__ float dmax_s;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int h = n / 2;
  const float* a_in = Ain + (int64_t)blockIdx.x * sA;
  for (int i = tid; i < n * n; i += nt) {
    const int r = i / n, c = i % n;
    A[r * kLd + c] = a_in[i];
    V[r * kLd + c] = (r == c) ? 1.0 : 0.0;
  }
  __syncthreads();
  if (tid == 0) {
    float m = 0.0f;
    for (int i = 0; i < n; ++i) m = fmaxf(m, fabsf(A[i * kLd + i]));
    dmax_s = m;
  }
  __syncthreads();
  const float atol = 1e-10f * dmax_s;
  int sweep = 0;
  for (; sweep < max_sweeps; ++sweep) {
    if (tid == 0) rotated = 0;
    __syncthreads();
    for (int r = 0; r < n - 1; ++r) {
      if (tid < h) {
        int p = tour_player(tid, r, n), q = tour_player(n - 1 - tid, r, n);
        if (p > q) { const int t = p; p = q; q = t; }
        const float app = A[p * kLd + p], aqq = A[q * kLd + q], apq = A[p * kLd + q];
        double c = 1.0, s = 0.0;
        if (fabsf(apq) > atol && fabsf(apq) > 1e-7f * sqrtf(fabsf(app * aqq))) {
          const double tau = ((double)aqq - (double)app) / (2.0 * (double)apq);
          const double t = fabs(tau) > 1e150 ? 0.5 / tau
                                             : (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
          rotated = 1;
        }
        csd[tid] = c;
        csd[kMaxN / 2 + tid] = s;
        cs[tid] = (float)c;
        cs[kMaxN / 2 + tid] = (float)s;
        pq[tid] = p;
        pq[kMaxN / 2 + tid] = q;
      }
      __syncthreads();
      // A <- J^T A J over all 2x2 blocks of pairs (disjoint, so in place).
      for (int blk = tid; blk < h * h; blk += nt) {
        const int a = blk / h, b = blk % h;
        const int pa = pq[a], qa = pq[kMaxN / 2 + a], pb = pq[b], qb = pq[kMaxN / 2 + b];
        const float ca = cs[a], sa = cs[kMaxN / 2 + a], cb = cs[b], sb = cs[kMaxN / 2 + b];
        const float a00 = A[pa * kLd + pb], a01 = A[pa * kLd + qb];
        const float a10 = A[qa * kLd + pb], a11 = A[qa * kLd + qb];
        const float t00 = cb * a00 - sb * a01, t01 = sb * a00 + cb * a01;
        const float t10 = cb * a10 - sb * a11, t11 = sb * a10 + cb * a11;
        float n00 = ca * t00 - sa * t10, n10 = sa * t00 + ca * t10;
        float n01 = ca * t01 - sa * t11, n11 = sa * t01 + ca * t11;
        if (a == b && sa != 0.0f) { n01 = 0.0f; n10 = 0.0f; }
        A[pa * kLd + pb] = n00;
        A[pa * kLd + qb] = n01;
        A[qa * kLd + pb] = n10;
        A[qa * kLd + qb] = n11;
      }
      // V <- V J
      for (int idx = tid; idx < n * h; idx += nt) {
        const int i = idx / h, k = idx % h;
        const int p = pq[k], q = pq[kMaxN / 2 + k];
        const double c = csd[k], s = csd[kMaxN / 2 + k];
        const double vp = V[i * kLd + p], vq = V[i * kLd + q];
        V[i * kLd + p] = c * vp - s * vq;
        V[i * kLd + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
    if (!rotated) break;
    __syncthreads();
  }
  if (sweep == max_sweeps && tid == 0 && status) atomicOr(status, ST_NOT_CONVERGED);
  // Descending order; equal eigenvalues keep index order.
  for (int i = tid; i < n; i += nt) {
    const float li = A[i * kLd + i];
    int rk = 0;
    for (int j = 0; j < n; ++j) {
      const float lj = A[j * kLd + j];
      rk += (lj > li) || (lj == li && j < i);
    }
    rank[i] = rk;
  }
  __syncthreads();
  float* vo = Vout + (int64_t)blockIdx.x * sV;
  for (int e = tid; e < n * n; e += nt) {
    const int r = e / n, c = e % n;     // eigenvector c, component r
    vo[r * n + rank[c]] = (float)V[r * kLd + c];
  }
  if (lam)
    for (int i = tid; i < n; i += nt) lam[(int64_t)blockIdx.x * sL + rank[i]] = A[i * kLd + i];
}

// Rinv = R^{-1} with R^T R = W + shift * (trace(W) / n) I (upper triangular R), float64 in
// shared memory (one n x (n+1) array, the inverse overwrites the factor in place). A
// non-positive pivot is raised to a tiny floor and flags ST_NOT_CONVERGED.
__global__ void __launch_bounds__(256) k_chol_inv(int n, const double* W, int64_t sW, double* Rinv,
                                                  int64_t sR, double shift, int32_t* status) {
  extern __shared__ double dm[];
  const int ld = n + 1;
  double* R = dm;              // n x ld
  double* x = R + n * ld;      // n
  __shared__ double tr_s;
  const int tid = threadIdx.x, nt = blockDim.x;
  const double* w = W + (int64_t)blockIdx.x * sW;
  for (int i = tid; i < n * n; i += nt) R[(i / n) * ld + (i % n)] = w[i];
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int i = 0; i < n; ++i) t += R[i * ld + i];
    tr_s = t;
  }
  __syncthreads();
  const double add = shift * tr_s / n;
  for (int i = tid; i < n; i += nt) R[i * ld + i] += add;
  __syncthreads();
  // Right-looking Cholesky, W = R^T R, R upper triangular (kept in the upper triangle).
  for (int k = 0; k < n; ++k) {
    if (tid == 0) {
      double d = R[k * ld + k];
      const double floor_v = 1e-30 + 1e-14 * (tr_s > 0 ? tr_s / n : 1.0);
      if (!(d > floor_v)) {
        d = floor_v;
        if (status) atomicOr(status, ST_NOT_CONVERGED);
      }
      R[k * ld + k] = sqrt(d);
    }
    __syncthreads();
    const double rkk = R[k * ld + k];
    for (int j = k + 1 + tid; j < n; j += nt) R[k * ld + j] /= rkk;
    __syncthreads();
    for (int idx = tid; idx < (n - k - 1) * (n - k - 1); idx += nt) {
      const int i = k + 1 + idx / (n - k - 1), j = k + 1 + idx % (n - k - 1);
      if (j >= i) R[i * ld + j] -= R[k * ld + i] * R[k * ld + j];
    }
    __syncthreads();
  }
  // In-place inverse of the upper triangle, column by column: with the leading j x j block
  // already inverted, column j above the diagonal is -R^{-1}_jj * (R^{-1}_{0:j,0:j} R_{0:j,j}).
  for (int j = 0; j < n; ++j) {
    const double inv_jj = 1.0 / R[j * ld + j];
    for (int i = tid; i < j; i += nt) {
      double v = 0.0;
      for (int k = i; k < j; ++k) v += R[i * ld + k] * R[k * ld + j];
      x[i] = v;
    }
    __syncthreads();
    for (int i = tid; i < j; i += nt) R[i * ld + j] = -inv_jj * x[i];
    if (tid == 0) R[j * ld + j] = inv_jj;
    __syncthreads();
  }
  double* o = Rinv + (int64_t)blockIdx.x * sR;
  for (int i = tid; i < n * n; i += nt) {
    const int r = i / n, c = i % n;
    o[i] = (c >= r) ? R[r * ld + c] : 0.0;
  }
}

}  // namespace

cudaError_t jacobi_eig(int batch, int n, const float* A, int64_t sA, float* V, int64_t sV,
                       float* lam, int64_t sL, int max_sweeps, int32_t* status, cudaStream_t s) {
  if (n <= 0 || n > kMaxN || (n & 1)) return cudaErrorInvalidValue;
  if (batch <= 0) return cudaSuccess;
  const size_t smem = ((size_t)kMaxN * kLd + kMaxN) * sizeof(double) +
                      ((size_t)kMaxN * kLd + kMaxN) * sizeof(float) + 2 * kMaxN * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(k_jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_jacobi<<<batch, 512, smem, s>>>(n, A, sA, V, sV, lam, sL, max_sweeps, status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t chol_inv(int batch, int n, const double* W, int64_t sW, double* Rinv, int64_t sR,
                     double shift, int32_t* status, cudaStream_t s) {
  if (n <= 0 || n > kMaxN) return cudaErrorInvalidValue;
  if (batch <= 0) return cudaSuccess;
  const size_t smem = ((size_t)n * (n + 1) + n) * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(k_chol_inv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_chol_inv<<<batch, 256, smem, s>>>(n, W, sW, Rinv, sR, shift, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
