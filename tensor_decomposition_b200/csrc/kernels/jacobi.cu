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
#include <type_traits>

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

// Right-looking Cholesky by 16-column blocks of the 128 x 128 array A (row stride LD): on
// entry the lower triangle holds the matrix (identity on the padding, upper triangle zero),
// on exit the blocks below the diagonal hold L (A = L L^T) and Dv the inverses of the
// diagonal blocks of L (zero above their diagonal). kKeepL = true: the diagonal blocks hold
// L_kk in their lower half. kKeepL = false: the upper triangle holds X^T with X = L^{-1},
// formed alongside the factorisation (right-looking block forward substitution of L X = I with
// B = I kept transposed in the upper triangle: at step k, X_k = L_kk^{-1} B_k, then
// B_i -= L_ik X_k below), through the scratch Xs [16][128].
//  * Diagonal block: warp 0, lane i holding row i in registers. The next pivot is broadcast
//    as soon as its lane has it, so that its reciprocal square root (CUDA's float64 rsqrt)
//    overlaps the broadcast of column k (through Ls) and the row updates; then L_kk^{-1}.
//  * Panel phase: L21 = A21 L_kk^{-T} (into Pt) and X_k (into Xs), one pass of 512 items.
//  * Trailing phase: L21 back into A, the rank-16 update of the trailing lower triangle and
//    the update of B below block k, in 4 x 4 register tiles; X_k back into the upper triangle.
// A pivot not above floor_v is raised to it and sets *floored (pivots of the n x n problem
// only). Called by all NT threads of the block.
constexpr int kCholLD = kMaxN + 1;
constexpr int kPanelLD = kMaxN + 8;   // row stride of the panel and X scratch: conflict-free MMA fragments

// D += A B on the FP64 tensor-core MMA (m8n8k4, row.col): lane l holds A[l / 4][l % 4],
// B[l % 4][l / 4] and D[l / 4][2 (l % 4) .. + 1] (fragments per the PTX ISA).
__device__ __forceinline__ void dmma_f64(double& d0, double& d1, double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
      : "+d"(d0), "+d"(d1)
      : "d"(a), "d"(b));
}

template <bool kKeepL, int NT = 512>
__device__ __forceinline__ void chol_blocks(double* A, double* Dv, double* Pt, double* Ls, double* Is, double* Xs,
                                            int n, double floor_v, int* floored) {
  constexpr int NP = kMaxN, LD = kCholLD, BS = 16, NBLK = NP / BS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int kb = 0; kb < NBLK; ++kb) {
    const int k0 = kb * BS;
    double* D = Dv + kb * BS * BS;
    if (warp == 0) {
      // lane i (and its mirror i + 16) holds row i of the diagonal block
      const int i = lane & (BS - 1);
      double a[BS];
#pragma unroll
      for (int j = 0; j < BS; ++j) a[j] = A[(k0 + i) * LD + k0 + j];
      bool fl = false;
      double isv = 0.0;   // lane i: 1 / l_ii
      double d = __shfl_sync(0xffffffffu, a[0], 0);
      {
        const bool low = !(d > floor_v);
        fl = fl | (low & (k0 < n));
        d = low ? floor_v : d;
      }
      double inv = rsqrt(d);
#pragma unroll
      for (int k = 0; k < BS; ++k) {
        const double lk = (i == k) ? d * inv : (i > k ? a[k] * inv : 0.0);
        a[k] = lk;
        isv = (i == k) ? inv : isv;
        // lane k + 1's updated diagonal goes out first: the next pivot's square root does
        // not wait for column k's broadcast
        double dnext = 0.0;
        if (k + 1 < BS) dnext = __shfl_sync(0xffffffffu, fma(-lk, lk, a[k + 1]), k + 1);
        double lj[BS];
        if (lane < BS) Ls[k * BS + i] = lk;
        __syncwarp();
#pragma unroll
        for (int j = 1; j < BS; ++j)
          if (j > k) lj[j] = Ls[k * BS + j];
#pragma unroll
        for (int j = 1; j < BS; ++j)
          if (j > k && i >= j) a[j] = fma(-lk, lj[j], a[j]);
        if (k + 1 < BS) {
          const bool low = !(dnext > floor_v);
          fl = fl | (low & (k0 + k + 1 < n));
          d = low ? floor_v : dnext;
          inv = rsqrt(d);
        }
      }
      __syncwarp();   // the column broadcasts are read; Ls takes the factor
      if (lane < BS) {
        Is[i] = isv;
#pragma unroll
        for (int j = 0; j < BS; ++j) Ls[i * (BS + 1) + j] = a[j];
      }
      __syncwarp();
      // column i of L_kk^{-1}, right-looking substitution (entries above the diagonal stay 0)
      double acc[BS], x[BS];
#pragma unroll
      for (int r = 0; r < BS; ++r) acc[r] = (r == i) ? 1.0 : 0.0;
#pragma unroll
      for (int m = 0; m < BS; ++m) {
        x[m] = acc[m] * Is[m];
#pragma unroll
        for (int r = 1; r < BS; ++r)
          if (r > m) acc[r] = fma(-Ls[r * (BS + 1) + m], x[m], acc[r]);
      }
      if (lane < BS) {
#pragma unroll
        for (int r = 0; r < BS; ++r) {
          D[r * BS + i] = x[r];
          if (!kKeepL && r >= i) A[(k0 + i) * LD + k0 + r] = x[r];   // T = X^T, upper half of the block
          if (kKeepL && r <= i) A[(k0 + i) * LD + k0 + r] = a[r];    // L_kk, lower half of the block
        }
        if (fl && lane == 0) *floored = 1;
      }
    }
    __syncthreads();
    const int rows = NP - k0 - BS;
    // panel L21 = A21 L11^{-T} into Pt only; thread = (group g of 4 columns, row), consecutive
    // lanes on consecutive rows. L11^{-1} is stored with zeros above its diagonal, so every
    // output is a full 16-term sum. A keeps A21 until the trailing phase copies L21 back.
    // With the inverse: X_k[:, c] = L_kk^{-1} B_k[:, c] for c < k0 (thread = (group g of 4
    // rows, column c)) and X_kk = L_kk^{-1} into Xs [m][c]; 4 rows + 4 k0 + 64 = 512 items.
    const int nx = kKeepL ? 0 : 4 * k0 + 64;
    for (int u = tid; u < 4 * rows + nx; u += NT) {
      if (u < 4 * rows) {
        const int g = u / rows, i = k0 + BS + (u - g * rows);
        double v[BS];
#pragma unroll
        for (int m = 0; m < BS; ++m) v[m] = A[i * LD + k0 + m];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = 4 * g + jj;
          double o = 0.0;
#pragma unroll
          for (int m = 0; m < BS; ++m) o = fma(v[m], D[j * BS + m], o);
          Pt[j * kPanelLD + i] = o;
        }
      } else if (u < 4 * rows + 4 * k0) {
        const int w = u - 4 * rows, g = w / k0, c = w - g * k0;
        double bv[BS];
#pragma unroll
        for (int m = 0; m < BS; ++m) bv[m] = A[c * LD + k0 + m];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          double o = 0.0;
#pragma unroll
          for (int m = 0; m < BS; ++m) o = fma(D[(4 * g + rr) * BS + m], bv[m], o);
          Xs[(4 * g + rr) * kPanelLD + c] = o;
        }
      } else {
        const int w = u - 4 * rows - 4 * k0;   // 64 items: row w / 4, columns 4 (w % 4) ..
        const int r = w >> 2, c4 = 4 * (w & 3);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) Xs[r * kPanelLD + k0 + c4 + cc] = D[r * BS + c4 + cc];
      }
    }
    __syncthreads();
    // L21 back into A (the trailing tiles below read Pt and write only columns >= k0 + BS);
    // X_k back into the upper triangle (block row k of X^T's columns c < k0)
    for (int u = tid; u < BS * rows; u += NT) {
      const int j = u / rows, i = k0 + BS + (u - j * rows);
      A[i * LD + k0 + j] = Pt[j * kPanelLD + i];
    }
    if (!kKeepL)
      for (int u = tid; u < BS * k0; u += NT) {
        const int m = u / k0, c = u - m * k0;
        A[c * LD + k0 + m] = Xs[m * kPanelLD + c];
      }
    // trailing update of the lower triangle, A22 -= L21 L21^T, and (inverse) of B below block
    // k, B_i[:, c] -= L_ik X_k[:, c] for c < k0 + 16 (kept transposed: T[c][i] -= sum_m
    // X_k[m][c] L21[i][m]), on the FP64 MMA: warp w takes the 16 x 16 blocks w, w + NT / 32, ...
    // as 2 x 2 tiles of 8 x 8 (four k = 4 steps over the panel width, two A and two B fragments
    // per step). Diagonal blocks of A22 skip their upper tile and store the lower half of their
    // diagonal tiles only: the upper triangle belongs to T.
    const int t16 = rows / 16, cnt = t16 * (t16 + 1) / 2, cntb = kKeepL ? 0 : t16 * (kb + 1);
    const int fr = lane >> 2, fq = lane & 3;
    for (int t = warp; t < cnt + cntb; t += NT / 32) {
      const double* pa;
      const double* pb;
      double* cp;
      bool diag = false;
      if (t < cnt) {
        int bi = (int)((sqrtf(8.0f * (float)t + 1.0f) - 1.0f) * 0.5f);
        while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
        while (bi * (bi + 1) / 2 > t) --bi;
        const int bj = t - bi * (bi + 1) / 2;
        const int i0 = k0 + BS + 16 * bi, j0 = k0 + BS + 16 * bj;
        pa = Pt + fq * kPanelLD + i0 + fr;         // A[r][q] = L21[i0 + r][q]
        pb = Pt + fq * kPanelLD + j0 + fr;         // B[q][c] = L21[j0 + c][q]
        cp = A + (i0 + fr) * LD + j0 + 2 * fq;
        diag = bi == bj;
      } else {
        const int tb = t - cnt, cb = tb / t16, bi = tb - cb * t16;
        const int c0 = 16 * cb, r0 = k0 + BS + 16 * bi;
        pa = Xs + fq * kPanelLD + c0 + fr;         // A[c][q] = X_k[q][c0 + c]
        pb = Pt + fq * kPanelLD + r0 + fr;         // B[q][i] = L21[r0 + i][q]
        cp = A + (c0 + fr) * LD + r0 + 2 * fq;
      }
      // tile (u, v): rows 8 u .., columns 8 v ..; d[u][v][0..1]
      double d[2][2][2];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const bool skip = diag && u < v;
          d[u][v][0] = skip ? 0.0 : cp[8 * u * LD + 8 * v];
          d[u][v][1] = skip ? 0.0 : cp[8 * u * LD + 8 * v + 1];
        }
#pragma unroll
      for (int m0 = 0; m0 < BS; m0 += 4) {
        const double a0 = -pa[m0 * kPanelLD], a1 = -pa[m0 * kPanelLD + 8];
        const double b0 = pb[m0 * kPanelLD], b1 = pb[m0 * kPanelLD + 8];
        dmma_f64(d[0][0][0], d[0][0][1], a0, b0);
        dmma_f64(d[1][0][0], d[1][0][1], a1, b0);
        dmma_f64(d[1][1][0], d[1][1][1], a1, b1);
        if (!diag) dmma_f64(d[0][1][0], d[0][1][1], a0, b1);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          if (diag && u < v) continue;
          const bool dt = diag && u == v;
          if (!dt || 2 * fq <= fr) cp[8 * u * LD + 8 * v] = d[u][v][0];
          if (!dt || 2 * fq + 1 <= fr) cp[8 * u * LD + 8 * v + 1] = d[u][v][1];
        }
    }
    __syncthreads();
  }
}

// Eigenpairs of a batch of symmetric positive semi-definite n x n matrices C (n <= 128),
// float64 input, by one-sided (Hestenes) Jacobi on a Cholesky factor:
//   C + sigma I = M M^T (M = R^T, R the upper Cholesky factor, sigma = 1e-13 trace / n keeps
//   the factorisation defined; it shifts every eigenvalue by sigma and leaves the vectors);
//   column pairs (p, q) of M are rotated, M <- M J, until all columns are mutually orthogonal;
//   then M = U Sigma, so the normalised columns are the eigenvectors of C and the squared
//   column norms (minus sigma) its eigenvalues. No eigenvector matrix is accumulated.
// M lives in shared memory in float64, column-major, padded with zero rows/columns to 128.
// Each round of the circle-method tournament rotates 64 disjoint pairs:
// the three dot products are warp-shuffle reductions; the rotation (Golub & Van Loan sec.
// 8.6, one-sided Jacobi) uses zeta = (beta - alpha) / (2 gamma), t = sign(zeta) /
// (|zeta| + sqrt(1 + zeta^2)), c = 1 / sqrt(1 + t^2), s = t c, computed in float32 and
// renormalised in float64 by one Newton step so that c^2 + s^2 = 1 to ~1e-15. A pair rotates
// when gamma^2 > 1e-14 alpha beta; a sweep with no rotation ends the solve. Each warp works on
// four pairs of a round at once, eight lanes per pair (16 rows each), so the dot products need
// only three shuffle steps.
struct EigBatch {
  const double* C;
  int64_t sC;
  float* V;
  int64_t sV;
  float* lam;
  int64_t sL;
  int n, count;
};

// f(integral_constant<int, K>) for K = K0 .. N - 1, unrolled at compile time
constexpr int kEigWarps = 16;  // warps per eigenproblem (4 slots, 8 columns each; 8 warps of 8 slots ran 1.5x slower)

template <int K0, int N, class F>
__device__ __forceinline__ void unroll_phases(F& f) {
  if constexpr (K0 < N) {
    f(std::integral_constant<int, K0>{});
    unroll_phases<K0 + 1, N>(f);
  }
}

// A sweep in which no pair was further than sqrt(kCheckCos2) from orthogonal (cosine of the
// two columns) is followed by the Gram test below instead of a verifying sweep. Convergence is
// quadratic at the end: after a sweep whose largest cosine is 1e-4 the next one rarely finds a
// pair above the 1e-7 rotation threshold; a test that fails costs about a tenth of a sweep.
constexpr double kCheckCos2 = 1e-8;
// shared memory of k_eig_psd: the Cholesky's arrays (A, diagonal inverses, panel, diagonal
// factor and its reciprocals), which the column array, the Gram test's padded copy and the
// norms and ranks overlay
constexpr size_t kEigSmemDoubles = (size_t)kMaxN * kCholLD + 8 * 256 + 16 * kPanelLD + 16 * 17 + 16;
static_assert((size_t)kMaxN * (kMaxN + 4) + kMaxN <= kEigSmemDoubles, "Gram test array (stride kMaxN + 4)");
static_assert((size_t)kMaxN * kMaxN + kMaxN + kMaxN / 2 <= kEigSmemDoubles, "columns, norms, ranks");

// The sweep's rotation criterion for a pair with dot product g and squared norms a, b: the
// same power-of-two scale and float conversion as the angle computation.
__device__ __forceinline__ bool pair_rotates(double g, double a, double b) {
  const int ex = (__double2hiint(a + b) >> 20) & 0x7ff;
  const double sc2 = __hiloint2double((2046 - ex) << 20, 0);
  return g * g > 1e-14 * (a * b) && (float)(g * (2.0 * sc2)) != 0.0f;
}

// Whether every pair of the 128 columns, copied column-major at stride kGramLD with their
// squared norms after them, passes the rotation criterion without rotating, i.e. whether a
// sweep would leave them as they are. The upper triangle of M^T M is formed in 8 x 8 tiles on
// the FP64 MMA (m8n8k4, fragments per the PTX ISA; warp w takes tiles w, w + W, ..., two
// accumulator chains per tile; the stride makes the fragment loads conflict-free). Kept out of
// line so that its registers do not add to those of the sweep. Ends with a barrier after its
// last read of the copy (the next round's column exchange overwrites it) and returns the same
// value in every thread.
constexpr int kGramLD = kMaxN + 4;

template <int W>
__device__ __noinline__ bool gram_all_converged(const double* Mc, int* violated) {
  constexpr int NP = kMaxN, NB = NP / 8;
  const double* cn = Mc + NP * kGramLD;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, kk = lane & 3;
  bool bad = false;
  for (int t = warp; t < NB * (NB + 1) / 2; t += W) {
    int bi = 0, rem = t;          // t-th tile of the upper triangle, row by row
    while (rem >= NB - bi) {
      rem -= NB - bi;
      ++bi;
    }
    const int bj = bi + rem;
    const double* pa = Mc + (8 * bi + r) * kGramLD + kk;
    const double* pb = Mc + (8 * bj + r) * kGramLD + kk;
    double c0 = 0.0, c1 = 0.0, e0 = 0.0, e1 = 0.0;
#pragma unroll 4
    for (int k0 = 0; k0 < NP; k0 += 8) {
      dmma_f64(c0, c1, pa[k0], pb[k0]);
      dmma_f64(e0, e1, pa[k0 + 4], pb[k0 + 4]);
    }
    const int i = 8 * bi + r, j = 8 * bj + 2 * kk;
    bad |= i < j && pair_rotates(c0 + e0, cn[i], cn[j]);
    bad |= i < j + 1 && pair_rotates(c1 + e1, cn[i], cn[j + 1]);
  }
  if (bad) *violated = 1;
  __syncthreads();
  return *violated == 0;
}

// Two independent batches share one launch (blocks [0, b0.count) take the first). W warps of
// S = 64 / W tournament slots each (W = 8: 16 columns of 4 rows per lane in registers).
template <int W>
__global__ void __launch_bounds__(32 * W) k_eig_psd(EigBatch b0, EigBatch b1, int max_sweeps, int32_t* status) {
  constexpr int NP = kMaxN, NT = 32 * W, S = 64 / W, GL = 32 / S;   // GL lanes per slot group
  static_assert(W * S == 64 && (S & (S - 1)) == 0 && S >= 2, "slots per warp");
  const bool first = (int)blockIdx.x < b0.count;
  const EigBatch& eb = first ? b0 : b1;
  const int bi = first ? (int)blockIdx.x : (int)blockIdx.x - b0.count;
  const int n = eb.n;
  const double* Cin = eb.C;
  const int64_t sC = eb.sC, sV = eb.sV, sL = eb.sL;
  float* Vout = eb.V;
  float* lam = eb.lam;
  extern __shared__ double ms[];
  double* M = ms;                 // column-major: column j at M + j * NP (during Cholesky: row-major R)
  double* nrm = M + NP * NP;      // NP squared column norms
  int* rank = reinterpret_cast<int*>(nrm + NP);
  __shared__ int rotated[2], large[2], violated;
  __shared__ double sigma_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double* c_in = Cin + (int64_t)bi * sC;
  // C + sigma I = L L^T by the blocked Cholesky (sigma = 1e-13 trace / n; pivots floored at
  // 1e-3 sigma), in the padded row-major array A that overlays M
  double* A = ms;                                  // NP x kCholLD
  double* Dv = A + NP * kCholLD;
  double* Pt = Dv + NP * 16;
  double* Ls = Pt + 16 * kPanelLD;
  double* Is = Ls + 16 * 17;
  __shared__ int floored;
  constexpr int PER = NP * NP / NT;
  double cv[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int e = tid + NT * q, r = e >> 7, c = e & (NP - 1);
    cv[q] = (c <= r && r < n) ? c_in[(int64_t)r * n + c] : 0.0;
  }
  if (tid < 32) {
    double t = 0.0;
    for (int i = tid; i < n; i += 32) t += fabs(c_in[(int64_t)i * n + i]);
    for (int o = 16; o > 0; o >>= 1) t += __shfl_down_sync(0xffffffffu, t, o);
    if (tid == 0) {
      sigma_s = 1e-13 * (t > 0.0 ? t / n : 1.0);
      floored = 0;
    }
  }
  __syncthreads();
  const double sigma = sigma_s;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int e = tid + NT * q, r = e >> 7, c = e & (NP - 1);
    double v = (c <= r && r < n) ? cv[q] + (r == c ? sigma : 0.0) : 0.0;
    if (r >= n && r == c) v = 1.0;
    A[r * kCholLD + c] = v;
  }
  __syncthreads();
  chol_blocks<true, NT>(A, Dv, Pt, Ls, Is, nullptr, n, sigma * 1e-3, &floored);
  // M = L column-major (column j of M is column j of L), padding columns zero
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int e = tid + NT * q, c = e >> 7, r = e & (NP - 1);
    cv[q] = (r >= c && r < n && c < n) ? A[r * kCholLD + c] : 0.0;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < PER; ++q) M[tid + NT * q] = cv[q];
  __syncthreads();
  // ---- sweeps with the columns in registers. Warp w holds the tournament slots S w .. S w + S - 1;
  // slot k pairs position k (top) with position 127 - k (bottom), and position j starts with
  // column j. Lane l holds rows l, l + 32, l + 64, l + 96 of its 2 S columns.
  constexpr int RPL = NP / 32;
  double top[S][RPL], bot[S][RPL];
#pragma unroll
  for (int s = 0; s < S; ++s)
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
      top[s][i] = M[(S * warp + s) * NP + lane + 32 * i];
      bot[s][i] = M[(NP - 1 - S * warp - s) * NP + lane + 32 * i];
    }
  __syncthreads();
  // column exchange at the warp boundaries, double-buffered by round parity (reuses M)
  double* XT = M;                    // [2][W][NP]: top of slot S w + S - 1 handed to warp w + 1
  double* XB = M + 2 * W * NP;       // [2][W][NP]: bottom of slot S w handed to warp w - 1
  double* XN = M + 4 * W * NP;       // [2][W][2]: the squared norms of those two columns
  const int grp = lane / GL;         // the slot whose pair parameters this lane computes
  // rotated[sweep & 1] collects this sweep's flag; the other entry is reset for the next
  // sweep while nobody reads it
  if (tid == 0) rotated[0] = rotated[1] = large[0] = large[1] = 0;
  __syncthreads();
  int sweep = 0;
  for (; sweep < max_sweeps; ++sweep) {
    int any = 0;
    // squared column norms of slot `grp` (top: na, bottom: nb), exact at the start of the
    // sweep: per-lane partial sums, then butterflies over the 32 lanes
    double na = 0.0, nb = 0.0;
#pragma unroll
    for (int s = 0; s < S; ++s) {
      double a = 0.0, b = 0.0;
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        a = fma(top[s][i], top[s][i], a);
        b = fma(bot[s][i], bot[s][i], b);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
      }
      if (grp == s) {
        na = a;
        nb = b;
      }
    }
    // One round at tournament phase K (rounds done in this sweep, mod S). The slots' columns
    // are not moved between registers from round to round: logical top slot s lives in
    // top[(s - K) mod S] and logical bottom slot s in bot[(s + K) mod S], so the column leaving
    // a warp and the one arriving share a register and nothing else is copied.
    // Partial sums (this lane's rows) of gamma for the local slots 1 .. S - 2 at phase K: their
    // columns never wait for another warp.
    double vpre[S > 2 ? S - 2 : 1];
    auto partials_local = [&](auto kc) {
      constexpr int K = decltype(kc)::value;
#pragma unroll
      for (int s = 1; s <= S - 2; ++s) {
        double g = 0.0;
#pragma unroll
        for (int i = 0; i < RPL; ++i) g = fma(top[(s - K + S) % S][i], bot[(s + K) % S][i], g);
        vpre[s - 1] = g;
      }
    };
    partials_local(std::integral_constant<int, 0>{});
    auto round = [&](auto kc) {
      constexpr int K = decltype(kc)::value;
      // a power of two within a factor 2 of 1 / (a + b) for this group's pair
      const int ex = (__double2hiint(na + nb) >> 20) & 0x7ff;
      const double sc2 = __hiloint2double((2046 - ex) << 20, 0);
      // gamma of the S slots: per-lane partial sums, then a transposed butterfly that leaves
      // slot grp's sum in the GL lanes of group grp (identical in all of them): log2 S steps
      // halve the values a lane carries, then plain steps finish the sum
      double v[S];
#pragma unroll
      for (int s = 1; s <= S - 2; ++s) v[s] = vpre[s - 1];
#pragma unroll
      for (int s = 0; s < S; s += S - 1) {
        double g = 0.0;
#pragma unroll
        for (int i = 0; i < RPL; ++i) g = fma(top[(s - K + S) % S][i], bot[(s + K) % S][i], g);
        v[s] = g;
      }
#pragma unroll
      for (int half = S / 2, m = 16; half >= 1; half >>= 1, m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const double keep = up ? v[i + half] : v[i], send = up ? v[i] : v[i + half];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      double g = v[0];
#pragma unroll
      for (int m = GL / 2; m >= 1; m >>= 1) g += __shfl_xor_sync(0xffffffffu, g, m);
      const double a = na, b = nb;
      // rotation angle in float on (b - a, 2 gamma) scaled by the power of two of a + b (both
      // are at most a + b, so the squares below stay in range): with d = b - a,
      // r = sqrt(d^2 + 4 gamma^2) and w = |d| + r, the rotation that zeroes gamma is
      // c = w / sqrt(w^2 + 4 gamma^2), s = sign(d) 2 gamma / sqrt(w^2 + 4 gamma^2), i.e.
      // t = s / c = sign(zeta) / (|zeta| + sqrt(1 + zeta^2)) with zeta = d / (2 gamma)
      // (Golub & Van Loan sec. 8.5.2) using two reciprocal square roots and no division
      const float df = (float)((b - a) * sc2), gf = (float)(g * (2.0 * sc2));
      const bool rot = g * g > 1e-14 * (a * b) && gf != 0.0f;
      // the angle is computed whether or not the pair rotates (no divergent branch); a pair that
      // does not rotate takes (c, s) = (1, 0) and keeps its norms
      double c, sn;
      {
        const float q = fmaf(df, df, gf * gf);
        const float w = fabsf(df) + q * rsqrtf(q);
        const float z = rsqrtf(fmaf(w, w, gf * gf));
        const double c0 = (double)(w * z), s0 = (double)((df < 0.0f ? -gf : gf) * z);
        const double fix = 1.5 - 0.5 * (c0 * c0 + s0 * s0);   // one Newton step: c^2 + s^2 = 1
        c = rot ? c0 * fix : 1.0;
        sn = rot ? s0 * fix : 0.0;
        // squared norms after p' = c p - s q, q' = s p + c q
        const double cc = c * c, ss = sn * sn, cs2 = 2.0 * c * sn * g;
        const double na_r = fma(cc, a, fma(ss, b, -cs2)), nb_r = fma(ss, a, fma(cc, b, cs2));
        na = rot ? na_r : a;
        nb = rot ? nb_r : b;
      }
      // bit 0: a pair rotated; bit 1: a pair was further from orthogonal than the Gram test's bound
      any |= (int)rot | ((int)(g * g > kCheckCos2 * (a * b)) << 1);
      // rotate every slot with its group's (c, s); (1, 0) leaves a pair unchanged exactly, so a
      // warp none of whose pairs rotates skips the arithmetic
      if (__any_sync(0xffffffffu, rot)) {
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const double cs = __shfl_sync(0xffffffffu, c, GL * s);
          const double ss = __shfl_sync(0xffffffffu, sn, GL * s);
          // a slot whose pair does not rotate has (c, s) = (1, 0) exactly: skipping it leaves the
          // same bits (the branch is uniform over the warp)
          if (ss == 0.0) continue;
          double* tp = top[(s - K + S) % S];
          double* bp = bot[(s + K) % S];
#pragma unroll
          for (int i = 0; i < RPL; ++i) {
            // both s products first, so that each result overwrites its own input
            const double sq = ss * bp[i], sp = ss * tp[i];
            tp[i] = fma(cs, tp[i], -sq);
            bp[i] = fma(cs, bp[i], sp);
          }
        }
      }
      // next round of the circle tournament: position 0 stays, positions 1 .. 127 advance by
      // one. Tops move to the next slot, bottoms to the previous; slot 0's bottom becomes
      // slot 1's top and slot 63's top becomes its own bottom. The squared norms move with
      // their columns. Leaving: top slot S - 1 (to warp + 1) and bottom slot 0 (to warp - 1).
      constexpr int kOutT = (S - 1 - K + S) % S, kOutB = K % S, kFixed = (S - K) % S;
      constexpr int par = K & 1;
      double* xt = XT + (par * W + warp) * NP;
      double* xb = XB + (par * W + warp) * NP;
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        if (warp < W - 1) xt[lane + 32 * i] = top[kOutT][i];
        if (warp > 0) xb[lane + 32 * i] = bot[kOutB][i];
      }
      if (warp < W - 1 && lane == GL * (S - 1)) XN[(par * W + warp) * 2] = na;   // top of slot S w + S - 1
      if (warp > 0 && lane == 0) XN[(par * W + warp) * 2 + 1] = nb;              // bottom of slot S w
      const double up_a = __shfl_up_sync(0xffffffffu, (warp == 0 && grp == 0) ? nb : na, GL);
      const double dn_b = __shfl_down_sync(0xffffffffu, nb, GL);
      // moves that stay inside the edge warps, then the next round's partial sums of the local
      // slots (their columns are all here), then the barrier and the two arriving columns
      if (warp == 0) {
        // position 0 stays in slot 0's top; the leaving bottom becomes slot 1's top
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
          top[kOutT][i] = top[kFixed][i];
          top[kFixed][i] = bot[kOutB][i];
        }
      } else if (warp == W - 1) {
        // slot 63's top turns into its own bottom
#pragma unroll
        for (int i = 0; i < RPL; ++i) bot[kOutB][i] = top[kOutT][i];
      }
      partials_local(std::integral_constant<int, (K + 1) % S>{});
      __syncthreads();
      const double* xin_t = XT + (par * W + (warp > 0 ? warp - 1 : 0)) * NP;
      const double* xin_b = XB + (par * W + (warp < W - 1 ? warp + 1 : W - 1)) * NP;
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        if (warp > 0) top[kOutT][i] = xin_t[lane + 32 * i];
        if (warp < W - 1) bot[kOutB][i] = xin_b[lane + 32 * i];
      }
      const double na_new = grp >= 1 ? up_a : (warp == 0 ? na : XN[(par * W + warp - 1) * 2]);
      const double nb_new = grp <= S - 2 ? dn_b : (warp < W - 1 ? XN[(par * W + warp + 1) * 2 + 1] : na);
      na = na_new;
      nb = nb_new;
    };
    // 128 rounds: the 127 of the tournament and the first one again, so that every sweep starts
    // at phase 0 (the columns end one position further on per sweep; only their set matters)
    for (int r = 0; r < NP; r += S) unroll_phases<0, S>(round);
    if (any & 1) rotated[sweep & 1] = 1;
    if (any & 2) large[sweep & 1] = 1;
    if (tid == 0) rotated[(sweep + 1) & 1] = large[(sweep + 1) & 1] = 0;
    __syncthreads();
    if (!rotated[sweep & 1]) break;
    // A sweep whose pairs were all within kCheckCos2 of orthogonal is usually followed by one
    // that rotates nothing. That sweep only tests every pair once against the rotation
    // criterion with M unchanged, so the same test on the Gram matrix M^T M of the columns
    // as they stand decides it at a tenth of the cost; the sweep runs only if a pair fails.
    if (!large[sweep & 1]) {
      double* Mc = ms;
      double* cn = ms + NP * kGramLD;
      if (tid == 0) violated = 0;
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const int pt = S * warp + s, pb = NP - 1 - S * warp - s;
        double a = 0.0, b = 0.0;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
          Mc[pt * kGramLD + lane + 32 * i] = top[s][i];
          Mc[pb * kGramLD + lane + 32 * i] = bot[s][i];
          a = fma(top[s][i], top[s][i], a);
          b = fma(bot[s][i], bot[s][i], b);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          a += __shfl_xor_sync(0xffffffffu, a, o);
          b += __shfl_xor_sync(0xffffffffu, b, o);
        }
        if (lane == 0) {
          cn[pt] = a;
          cn[pb] = b;
        }
      }
      __syncthreads();
      if (gram_all_converged<W>(Mc, &violated)) break;
    }
  }
  if (sweep == max_sweeps && tid == 0 && status) atomicOr(status, ST_NOT_CONVERGED);
  // the columns, in the positions the last sweep left them in (their order does not matter:
  // they are ranked by norm below)
#pragma unroll
  for (int s = 0; s < S; ++s)
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
      M[(S * warp + s) * NP + lane + 32 * i] = top[s][i];
      M[(NP - 1 - S * warp - s) * NP + lane + 32 * i] = bot[s][i];
    }
  __syncthreads();
  // column norms, descending order (zero padding sorts last)
  for (int j = warp; j < NP; j += W) {
    const double* mj = M + j * NP + 4 * lane;
    double a = mj[0] * mj[0] + mj[1] * mj[1] + mj[2] * mj[2] + mj[3] * mj[3];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) nrm[j] = a;
  }
  __syncthreads();
  for (int i = tid; i < NP; i += NT) {
    const double li = nrm[i];
    int rk = 0;
    for (int j = 0; j < NP; ++j) {
      const double lj = nrm[j];
      rk += (lj > li) || (lj == li && j < i);
    }
    rank[i] = rk;
  }
  __syncthreads();
  float* vo = Vout + (int64_t)bi * sV;
  for (int e = tid; e < n * NP; e += NT) {
    const int c = e >> 7, r = e & (NP - 1);   // column c of M, row r
    if (r >= n || rank[c] >= n) continue;
    const double inv = nrm[c] > 0.0 ? 1.0 / sqrt(nrm[c]) : 0.0;
    vo[(int64_t)r * n + rank[c]] = (float)(M[c * NP + r] * inv);
  }
  if (lam)
    for (int c = tid; c < NP; c += NT)
      if (rank[c] < n) lam[(int64_t)bi * sL + rank[c]] = (float)(nrm[c] - sigma);
}

// Rinv = R^{-1} with R^T R = W + shift * (trace(W) / n) I (R upper triangular), float64.
// The n x n problem is embedded in a 128 x 128 one (identity on the padding) and blocked by 16.
// With L = R^T (W = L L^T) and X = L^{-1}, R^{-1} = X^T. One shared 128 x 129 array holds L
// in its lower triangle and T = X^T in its upper triangle; the diagonal blocks of L are not
// needed once their inverses are formed, so T takes over their upper half.
// The blocked Cholesky (chol_blocks) forms X alongside L: at block step k, X_k = L_kk^{-1} B_k
// in the panel phase and B_i -= L_ik X_k for the block rows below in the trailing phase
// (right-looking block forward substitution of L X = I, B = I initially, kept transposed in
// T), so the inverse takes no barriers of its own. A pivot below a tiny floor is raised to it
// and flags ST_NOT_CONVERGED.
template <typename TW>
__global__ void __launch_bounds__(512) k_chol_inv(int n, const TW* W, int64_t sW, double* Rinv,
                                                  int64_t sR, double shift, int32_t* status) {
  constexpr int NP = kMaxN, LD = kMaxN + 1, BS = 16, NBLK = NP / BS;
  extern __shared__ double dm[];
  double* A = dm;                          // NP x LD
  double* Dv = A + NP * LD;                // NBLK x BS x BS: L_kk^{-1} (lower, zero above)
  double* Pt = Dv + NBLK * BS * BS;        // BS x kPanelLD: the current panel, transposed
  double* Ls = Pt + BS * kPanelLD;         // BS x (BS + 1): the current diagonal factor
  double* Is = Ls + BS * (BS + 1);         // BS: 1 / L_kk diagonal
  double* Xs = Is + BS;                    // BS x kPanelLD: the current block row of X
  __shared__ double tr_s;
  __shared__ int floored;
  const int tid = threadIdx.x, lane = tid & 31;
  const TW* w = W + (int64_t)blockIdx.x * sW;
  if (tid == 0) floored = 0;
  // every load of W in flight before the first barrier (32 elements per thread)
  TW wv[NP * NP / 512];
#pragma unroll
  for (int q = 0; q < NP * NP / 512; ++q) {
    const int e = tid + 512 * q, r = e >> 7, c = e & (NP - 1);
    wv[q] = (c <= r && r < n) ? w[(int64_t)r * n + c] : (TW)0;
  }
  if (tid < 32) {
    double t = 0.0;
    for (int i = tid; i < n; i += 32) t += (double)w[(int64_t)i * n + i];
    for (int o = 16; o > 0; o >>= 1) t += __shfl_down_sync(0xffffffffu, t, o);
    if (tid == 0) tr_s = t;
  }
  __syncthreads();
  const double tr = tr_s;
  const double add = shift * tr / n;
  const double floor_v = 1e-30 + 1e-14 * (tr > 0 ? tr / n : 1.0);
  // lower triangle from W plus the shift, identity on the padding; upper triangle zero
#pragma unroll
  for (int q = 0; q < NP * NP / 512; ++q) {
    const int e = tid + 512 * q, r = e >> 7, c = e & (NP - 1);
    double v = (c <= r && r < n) ? (double)wv[q] + (r == c ? add : 0.0) : 0.0;
    if (r >= n && r == c) v = 1.0;
    A[r * LD + c] = v;
  }
  __syncthreads();
  chol_blocks<false>(A, Dv, Pt, Ls, Is, Xs, n, floor_v, &floored);
  if (floored && tid == 0 && status) atomicOr(status, ST_NOT_CONVERGED);
  double* o = Rinv + (int64_t)blockIdx.x * sR;
  for (int e = tid; e < n * n; e += 512) {
    const int r = e / n, c = e - r * n;
    o[e] = (c >= r) ? A[r * LD + c] : 0.0;
  }
  (void)lane;
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

cudaError_t eig_psd2(int batch0, int n0, const double* C0, int64_t sC0, float* V0, int64_t sV0, float* lam0,
                     int64_t sL0, int batch1, int n1, const double* C1, int64_t sC1, float* V1, int64_t sV1,
                     float* lam1, int64_t sL1, int max_sweeps, int32_t* status, cudaStream_t s) {
  if (n0 <= 0 || n0 > kMaxN || (batch1 > 0 && (n1 <= 0 || n1 > kMaxN))) return cudaErrorInvalidValue;
  if (batch0 + batch1 <= 0) return cudaSuccess;
  // the blocked Cholesky's arrays (A, diagonal inverses, panel, diagonal factor) overlay M,
  // the column norms and the ranks
  const size_t smem = kEigSmemDoubles * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(k_eig_psd<kEigWarps>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  EigBatch b0{C0, sC0, V0, sV0, lam0, sL0, n0, batch0};
  EigBatch b1{C1, sC1, V1, sV1, lam1, sL1, batch1 > 0 ? n1 : n0, batch1 > 0 ? batch1 : 0};
  k_eig_psd<kEigWarps><<<batch0 + b1.count, 32 * kEigWarps, smem, s>>>(b0, b1, max_sweeps, status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t eig_psd(int batch, int n, const double* C, int64_t sC, float* V, int64_t sV, float* lam, int64_t sL,
                    int max_sweeps, int32_t* status, cudaStream_t s) {
  return eig_psd2(batch, n, C, sC, V, sV, lam, sL, 0, 0, nullptr, 0, nullptr, 0, nullptr, 0, max_sweeps, status, s);
}

template <typename TW>
static cudaError_t chol_inv_t(int batch, int n, const TW* W, int64_t sW, double* Rinv, int64_t sR, double shift,
                              int32_t* status, cudaStream_t s) {
  if (n <= 0 || n > kMaxN) return cudaErrorInvalidValue;
  if (batch <= 0) return cudaSuccess;
  // A (128 x 129), diagonal-block inverses (8 x 16 x 16), panel (16 x 128), diagonal factor
  // (16 x 17), its reciprocal diagonal (16) and the current block row of X (16 x 128), float64
  const size_t smem = ((size_t)kMaxN * (kMaxN + 1) + 8 * 256 + 16 * kPanelLD + 16 * 17 + 16 + 16 * kPanelLD) * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(k_chol_inv<TW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_chol_inv<TW><<<batch, 512, smem, s>>>(n, W, sW, Rinv, sR, shift, status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t chol_inv(int batch, int n, const double* W, int64_t sW, double* Rinv, int64_t sR,
                     double shift, int32_t* status, cudaStream_t s) {
  return chol_inv_t<double>(batch, n, W, sW, Rinv, sR, shift, status, s);
}

cudaError_t chol_inv_f32(int batch, int n, const float* W, int64_t sW, double* Rinv, int64_t sR,
                         double shift, int32_t* status, cudaStream_t s) {
  return chol_inv_t<float>(batch, n, W, sW, Rinv, sR, shift, status, s);
}

}  // namespace jolt
