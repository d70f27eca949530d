// Batched symmetric eigensolver (two-sided cyclic Jacobi) and the Cholesky-inverse step of
// shifted CholeskyQR, both held in shared memory, one CTA per matrix.
//
// They solve the small factor problems of the JoLT codec ("A JoLT for the KV Cache",
// arXiv 2607.12550v2, Abstract): the feature factor U_D from the eigenvectors of
// C_D = sum_h X_h^T X_h (D x D), and, for the randomized-SVD ("FlashJoLT") token factor,
// the Rayleigh-Ritz rotation W from B B^T (l x l) and the orthonormalisation of sketches.
//
// Jacobi: n <= 128, padded to 128. Each sweep runs 127 rounds of the circle-method tournament,
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

__device__ __forceinline__ int tour_player(int pos, int r) {
  return pos == 0 ? 0 : ((pos - 1 + r) % (kMaxN - 1)) + 1;
}

// Every problem is embedded in a 128 x 128 one (indices >= n get the diagonal value
// -(1 + trace), zero coupling, so they never rotate against the real block and sort last);
// the fixed size turns all index arithmetic into shifts and masks.
__global__ void __launch_bounds__(512) k_jacobi(int n, const float* Ain, int64_t sA, float* Vout,
                                                int64_t sV, float* lam, int64_t sL, int max_sweeps,
                                                int32_t* status) {
  constexpr int NP = kMaxN, HP = kMaxN / 2;
  extern __shared__ double smd[];
  double* V = smd;                      // NP x kLd, float64: stays orthogonal over many rounds
  double* csd = V + NP * kLd;           // c[64], s[64] in float64
  float* A = reinterpret_cast<float*>(csd + NP);   // NP x kLd
  float* cs = A + NP * kLd;             // c[64], s[64] in float32 for the A update
  int* pq = reinterpret_cast<int*>(cs + NP);       // p[64], q[64]
  int* rank = pq + NP;                  // NP
  __shared__ int rotated;
  __shared__ float dmax_s, pad_s;
  const int tid = threadIdx.x;
  const float* a_in = Ain + (int64_t)blockIdx.x * sA;
  if (tid == 0) {
    float tr = 0.0f;
    for (int i = 0; i < n; ++i) tr += fabsf(a_in[(int64_t)i * n + i]);
    pad_s = -(1.0f + tr);
  }
  __syncthreads();
  for (int e = tid; e < NP * NP; e += 512) {
    const int r = e >> 7, c = e & (NP - 1);
    float v = 0.0f;
    if (r < n && c < n) v = a_in[(int64_t)r * n + c];
    else if (r == c) v = pad_s;
    A[r * kLd + c] = v;
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
    for (int r = 0; r < NP - 1; ++r) {
      if (tid < HP) {
        int p = tour_player(tid, r), q = tour_player(NP - 1 - tid, r);
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
        csd[HP + tid] = s;
        cs[tid] = (float)c;
        cs[HP + tid] = (float)s;
        pq[tid] = p;
        pq[HP + tid] = q;
      }
      __syncthreads();
      // A <- J^T A J over the 2x2 blocks (a, b), a <= b, of pairs (disjoint, so in place);
      // block (b, a) is the transpose and is written by the same thread.
#pragma unroll 2
      for (int j = 0; j < HP * HP / 512; ++j) {
        const int blk = tid + 512 * j;
        const int a = blk >> 6, b = blk & (HP - 1);
        if (a > b) continue;
        const int pa = pq[a], qa = pq[HP + a], pb = pq[b], qb = pq[HP + b];
        const float ca = cs[a], sa = cs[HP + a], cb = cs[b], sb = cs[HP + b];
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
        if (a != b) {
          A[pb * kLd + pa] = n00;
          A[qb * kLd + pa] = n01;
          A[pb * kLd + qa] = n10;
          A[qb * kLd + qa] = n11;
        }
      }
      // V <- V J; a warp walks one column pair down 32 consecutive rows
#pragma unroll 4
      for (int j = 0; j < NP * HP / 512; ++j) {
        const int idx = tid + 512 * j;
        const int k = idx >> 7, i = idx & (NP - 1);
        const int p = pq[k], q = pq[HP + k];
        const double c = csd[k], s = csd[HP + k];
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
  // Descending order; equal eigenvalues keep index order (padding sorts last).
  for (int i = tid; i < NP; i += 512) {
    const float li = A[i * kLd + i];
    int rk = 0;
    for (int j = 0; j < NP; ++j) {
      const float lj = A[j * kLd + j];
      rk += (lj > li) || (lj == li && j < i);
    }
    rank[i] = rk;
  }
  __syncthreads();
  float* vo = Vout + (int64_t)blockIdx.x * sV;
  for (int e = tid; e < n * n; e += 512) {
    const int r = e / n, c = e % n;     // eigenvector c, component r
    vo[r * n + rank[c]] = (float)V[r * kLd + c];
  }
  if (lam)
    for (int i = tid; i < n; i += 512) lam[(int64_t)blockIdx.x * sL + rank[i]] = A[i * kLd + i];
}

// Rinv = R^{-1} with R^T R = W + shift * (trace(W) / n) I (R upper triangular), float64.
// R and its inverse are kept as packed upper triangles in shared memory (n (n + 1) / 2 each).
// Cholesky: right-looking, 3 barriers per pivot. Inverse: thread c back-substitutes column c
// (R x = e_c), reading its own earlier entries of X. A non-positive pivot is raised to a tiny
// floor and flags ST_NOT_CONVERGED.
__device__ __forceinline__ int pk(int i, int k, int n) { return i * n - (i * (i - 1)) / 2 + (k - i); }

__global__ void __launch_bounds__(512) k_chol_inv(int n, const double* W, int64_t sW, double* Rinv,
                                                  int64_t sR, double shift, int32_t* status) {
  extern __shared__ double dm[];
  const int np = n * (n + 1) / 2;
  double* R = dm;              // packed upper triangle of the factor
  double* X = R + np;          // packed upper triangle of the inverse
  __shared__ double tr_s;
  const int tid = threadIdx.x, nt = blockDim.x;
  const double* w = W + (int64_t)blockIdx.x * sW;
  for (int e = tid; e < n * n; e += nt) {
    const int i = e / n, k = e % n;
    if (k >= i) R[pk(i, k, n)] = w[e];
  }
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int i = 0; i < n; ++i) t += R[pk(i, i, n)];
    tr_s = t;
  }
  __syncthreads();
  const double add = shift * tr_s / n;
  for (int i = tid; i < n; i += nt) R[pk(i, i, n)] += add;
  __syncthreads();
  for (int k = 0; k < n; ++k) {
    if (tid == 0) {
      double d = R[pk(k, k, n)];
      const double floor_v = 1e-30 + 1e-14 * (tr_s > 0 ? tr_s / n : 1.0);
      if (!(d > floor_v)) {
        d = floor_v;
        if (status) atomicOr(status, ST_NOT_CONVERGED);
      }
      R[pk(k, k, n)] = sqrt(d);
    }
    __syncthreads();
    const double rkk = R[pk(k, k, n)];
    for (int j = k + 1 + tid; j < n; j += nt) R[pk(k, j, n)] /= rkk;
    __syncthreads();
    const int m = n - k - 1;
    for (int e = tid; e < m * m; e += nt) {
      const int i = k + 1 + e / m, j = k + 1 + e % m;
      if (j >= i) R[pk(i, j, n)] -= R[pk(k, i, n)] * R[pk(k, j, n)];
    }
    __syncthreads();
  }
  for (int c = tid; c < n; c += nt) {
    for (int i = c; i >= 0; --i) {
      double v0 = (i == c) ? 1.0 : 0.0, v1 = 0.0;
      int k = i + 1;
      for (; k + 1 <= c; k += 2) {
        v0 -= R[pk(i, k, n)] * X[pk(k, c, n)];
        v1 -= R[pk(i, k + 1, n)] * X[pk(k + 1, c, n)];
      }
      if (k <= c) v0 -= R[pk(i, k, n)] * X[pk(k, c, n)];
      X[pk(i, c, n)] = (v0 + v1) / R[pk(i, i, n)];
    }
  }
  __syncthreads();
  double* o = Rinv + (int64_t)blockIdx.x * sR;
  for (int e = tid; e < n * n; e += nt) {
    const int r = e / n, c = e % n;
    o[e] = (c >= r) ? X[pk(r, c, n)] : 0.0;
  }
}

}  // namespace

cudaError_t jacobi_eig(int batch, int n, const float* A, int64_t sA, float* V, int64_t sV,
                       float* lam, int64_t sL, int max_sweeps, int32_t* status, cudaStream_t s) {
  if (n <= 0 || n > kMaxN) return cudaErrorInvalidValue;
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
  const size_t smem = (size_t)n * (n + 1) * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(k_chol_inv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_chol_inv<<<batch, 512, smem, s>>>(n, W, sW, Rinv, sR, shift, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
