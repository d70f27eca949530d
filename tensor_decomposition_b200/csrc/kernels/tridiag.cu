// Leading eigenpairs of dense symmetric matrices too large for one SM's Jacobi eigensolver: the
// exact token factor of the JoLT codec ("A JoLT for the KV Cache", arXiv 2607.12550v2, Abstract:
// a partial Tucker decomposition over the token and feature axes), whose exact variant takes the
// token factor U_T from the leading eigenvectors of the token Gram C_T = sum_h X_h X_h^T (T x T).
//
// A direct method in float64 (Golub & Van Loan, Matrix Computations, 4th ed.: sec. 8.3.1
// Householder tridiagonalisation, sec. 8.4.1 bisection on Sturm sequences, sec. 7.6.1 inverse
// iteration):
//  1. k_sytrd: A = Q T Q^T, T tridiagonal, Q = H_0 H_1 ... H_{n-3}, H_k = I - tau_k v_k v_k^T with
//     v_k zero above row k + 1 and v_k[k + 1] = 1. Reflections are formed column by column in
//     panels of kNB; inside a panel the two-sided update A <- A - v w^T - w v^T is kept pending
//     (the current column and the matrix-vector product of each step subtract the panel's
//     pending terms) and applied to the trailing matrix once at the end of the panel.
//  2. k_stebz: the R largest eigenvalues of T by bisection on the Sturm count (the number of
//     negative pivots of the LDL^T factorisation of T - x I), from the Gershgorin interval.
//  3. k_stein: each eigenvector of T by inverse iteration: three solves with T - lambda I by
//     Gaussian elimination with partial pivoting, from a fixed pseudo-random start vector;
//     k_stein_cluster: the members of a cluster of eigenvalues closer than 1e-10 ||T|| one after
//     another, each solve followed by Gram-Schmidt against the members already computed;
//  4. k_ormtr: back-transformation Z <- H_0 ... H_{n-3} Z of the R vectors.
// The caller re-orthonormalises the R vectors (CholeskyQR in float64): inverse iteration gives
// vectors orthogonal to ~eps ||T|| / gap only, and coincident eigenvalues need it.
// Step 1 runs on a cluster of two CTAs per matrix: each CTA forms the matrix-vector product of a
// column step for one half of the columns (its threads also split the rows when the trailing
// block has fewer column pairs than threads) and reads the other half from its peer's shared
// memory; the rest of a column step is computed by both CTAs alike, and the panel's trailing
// update is split by columns. One CTA per matrix in step 2, one thread per eigenvector (one warp
// per tight cluster) in step 3, one warp per vector in step 4.
#include "../jolt_internal.h"

namespace jolt {
namespace {

constexpr int kNB = 32;           // panel width of the tridiagonalisation
constexpr int kSyThreads = 512;   // threads of k_sytrd
constexpr int kRowChunk = 32;     // rows per register block of the trailing update
constexpr int kSyCluster = 2;     // CTAs per matrix in k_sytrd

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Barrier over both CTAs of the cluster; memory written before it (shared memory of either CTA,
// and global memory after a __threadfence) is visible to both after it.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The double at the same shared-memory offset as `p`, in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ double peer_f64(const double* p, uint32_t rank) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  double v;
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(ra) : "memory");
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over the block (kSyThreads threads); every thread receives the total. `red` holds
// kSyThreads / 32 doubles; the call starts and ends with a barrier.
__device__ __forceinline__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kSyThreads / 32; ++w) t += red[w];
  return t;
}

// Householder tridiagonalisation of one n x n symmetric matrix (full storage, row-major) per
// cluster of kSyCluster CTAs. On exit d, e hold the diagonal and subdiagonal of T, tau and row k of
// A (entries k + 1 .. n - 1) the reflector H_k (written by the cluster's first CTA). Vp / Wp:
// [kNB][n] scratch per CTA (the panel's v and w; both CTAs of a matrix hold the same values).
// Every barrier of the loop is reached by both CTAs the same number of times: the trip counts
// depend on n alone. A is read at L2 (ld.global.cg), since the peer's SM writes parts of it.
__global__ void __cluster_dims__(kSyCluster, 1, 1) __launch_bounds__(kSyThreads)
    k_sytrd(int n, double* A_all, int64_t sA, double* d_all, double* e_all, double* tau_all, double* Vp_all,
            double* Wp_all) {
  extern __shared__ double sm[];
  double* cs = sm;                  // [n] current column k, then the Householder vector v
  double* ys = cs + n;              // [n] y = A v, then w
  double* xb = ys + n;              // [2][n] this CTA's half of y = A v, by column-step parity (read by the peer)
  double* red = xb + 2 * n;         // [kSyThreads / 32] block reduction
  double* t1 = red + kSyThreads / 32;   // [kNB] W^T v
  double* t2 = t1 + kNB;                // [kNB] V^T v
  double* bc = t2 + kNB;                // [4] broadcast: tau, scale, beta, flag
  double* stg = bc + 4;                 // [2][kNB][kRowChunk] trailing-update row factors
  double* part = stg + 2 * kNB * kRowChunk;   // [2 kSyThreads] partial sums of the row slices
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const bool lead = rank == 0;
  const int b = blockIdx.x / kSyCluster;
  double* A = A_all + (int64_t)b * sA;
  double* d = d_all + (int64_t)b * n;
  double* e = e_all + (int64_t)b * n;
  double* tau = tau_all + (int64_t)b * n;
  double* Vp = Vp_all + (int64_t)blockIdx.x * kNB * n;
  double* Wp = Wp_all + (int64_t)blockIdx.x * kNB * n;
  for (int k0 = 0; k0 < n - 2; k0 += kNB) {
    const int kb = min(kNB, n - 2 - k0);
    for (int j = 0; j < kb; ++j) {
      const int k = k0 + j;
      // 1. column k of the current matrix (row k by symmetry: coalesced) with the panel's pending
      // corrections, rows k .. n - 1
      double ss = 0.0;
      for (int i = k + tid; i < n; i += kSyThreads) {
        double c = __ldcg(A + (int64_t)k * n + i);
        for (int l = 0; l < j; ++l)
          c -= Vp[(int64_t)l * n + i] * Wp[(int64_t)l * n + k] + Wp[(int64_t)l * n + i] * Vp[(int64_t)l * n + k];
        cs[i] = c;
        if (i >= k + 2) ss = fma(c, c, ss);
      }
      const double xn2 = block_sum(ss, red);   // barriers inside: cs is complete after it
      // 2. reflector H_k with H_k x = beta e_1 for x = column k below the diagonal (LAPACK's
      // dlarfg convention: v[0] = 1, beta = -sign(alpha) ||x||, tau = (beta - alpha) / beta)
      if (tid == 0) {
        const double alpha = cs[k + 1];
        double t = 0.0, scal = 0.0, beta = alpha;
        if (xn2 > 0.0) {
          beta = -copysign(sqrt(alpha * alpha + xn2), alpha);
          t = (beta - alpha) / beta;
          scal = 1.0 / (alpha - beta);
        }
        bc[0] = t;
        bc[1] = scal;
        if (lead) {
          d[k] = cs[k];
          e[k] = beta;
          tau[k] = t;
        }
      }
      __syncthreads();
      const double tk = bc[0], scal = bc[1];
      for (int i = tid; i < n; i += kSyThreads) {
        double v = 0.0;
        if (i == k + 1) v = 1.0;
        else if (i > k + 1) v = cs[i] * scal;
        if (i >= k + 1) cs[i] = v;
        Vp[(int64_t)j * n + i] = v;
      }
      __syncthreads();
      // 3. y = (A - V W^T - W V^T) v over rows and columns k + 1 .. n - 1; A is the matrix as at
      // the start of the panel. This CTA takes one half of the columns, the peer the other. A
      // thread takes two adjacent columns (one 16-byte load per row; the pairs start at an even
      // column, the one below k + 1 is computed and dropped) over a slice of the rows, keeping
      // sixteen rows' loads in flight; when the CTA has fewer column pairs than threads the rows
      // are cut into S slices whose sums are added in slice order. The CTA's results go to ys
      // and to xb[k % 2], from which the peer copies them after the cluster barrier.
      double* xk = xb + (k & 1) * n;
      int pa, pb;   // the peer's columns [pa, pb)
      if (n & 1) {
        // odd order: rows are not 16-byte aligned pairs; one column per thread over all rows
        const int nc = n - k - 1, h = (nc + 1) >> 1;
        const int ca = lead ? k + 1 : k + 1 + h, cb = lead ? k + 1 + h : n;
        pa = lead ? k + 1 + h : k + 1;
        pb = lead ? n : k + 1 + h;
        for (int col = ca + tid; col < cb; col += kSyThreads) {
          double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
          const double* Ac = A + col;
          int i = k + 1;
          for (; i + 3 < n; i += 4) {
            a0 = fma(__ldcg(Ac + (int64_t)i * n), cs[i], a0);
            a1 = fma(__ldcg(Ac + (int64_t)(i + 1) * n), cs[i + 1], a1);
            a2 = fma(__ldcg(Ac + (int64_t)(i + 2) * n), cs[i + 2], a2);
            a3 = fma(__ldcg(Ac + (int64_t)(i + 3) * n), cs[i + 3], a3);
          }
          for (; i < n; ++i) a0 = fma(__ldcg(Ac + (int64_t)i * n), cs[i], a0);
          const double y = (a0 + a1) + (a2 + a3);
          ys[col] = y;
          xk[col] = y;
        }
      } else {
        const int c0 = (k + 1) & ~1;
        const int np = (n - c0) >> 1, h = (np + 1) >> 1;
        const int qa = lead ? 0 : h, nq = lead ? h : np - h;   // this CTA's pairs [qa, qa + nq)
        pa = c0 + 2 * (lead ? h : 0);
        pb = lead ? n : c0 + 2 * h;
        const int m = n - (k + 1);
        int S = 1;
        while (2 * S * nq <= kSyThreads && 2 * S * 16 <= m) S *= 2;
        const int rs = (m + S - 1) / S;   // rows per slice
        for (int u = tid; u < S * nq; u += kSyThreads) {
          const int sl = u / nq, q = u - sl * nq;
          const int col = c0 + 2 * (qa + q);
          double ax[8], ay[8];
#pragma unroll
          for (int v = 0; v < 8; ++v) ax[v] = ay[v] = 0.0;
          const double* Ac = A + col;
          int i = k + 1 + sl * rs;
          const int iend = min(n, i + rs);
          for (; i + 15 < iend; i += 16) {
            double2 t[16];
#pragma unroll
            for (int v = 0; v < 16; ++v) t[v] = __ldcg(reinterpret_cast<const double2*>(Ac + (int64_t)(i + v) * n));
#pragma unroll
            for (int v = 0; v < 16; ++v) {
              ax[v & 7] = fma(t[v].x, cs[i + v], ax[v & 7]);
              ay[v & 7] = fma(t[v].y, cs[i + v], ay[v & 7]);
            }
          }
          for (; i < iend; ++i) {
            const double2 t = __ldcg(reinterpret_cast<const double2*>(Ac + (int64_t)i * n));
            ax[0] = fma(t.x, cs[i], ax[0]);
            ay[0] = fma(t.y, cs[i], ay[0]);
          }
          const double sx = ((ax[0] + ax[1]) + (ax[2] + ax[3])) + ((ax[4] + ax[5]) + (ax[6] + ax[7]));
          const double sy = ((ay[0] + ay[1]) + (ay[2] + ay[3])) + ((ay[4] + ay[5]) + (ay[6] + ay[7]));
          if (S == 1) {
            if (col >= k + 1) ys[col] = xk[col] = sx;
            ys[col + 1] = xk[col + 1] = sy;
          } else {
            part[2 * u] = sx;
            part[2 * u + 1] = sy;
          }
        }
        if (S > 1) {
          __syncthreads();
          for (int q = tid; q < nq; q += kSyThreads) {
            const int col = c0 + 2 * (qa + q);
            double sx = part[2 * q], sy = part[2 * q + 1];
            for (int sl = 1; sl < S; ++sl) {
              sx += part[2 * (sl * nq + q)];
              sy += part[2 * (sl * nq + q) + 1];
            }
            if (col >= k + 1) ys[col] = xk[col] = sx;
            ys[col + 1] = xk[col + 1] = sy;
          }
        }
      }
      // the peer's half of y (it is not overwritten before the next column step's barrier: xb
      // alternates with the step's parity)
      cluster_barrier();
      for (int col = max(pa, k + 1) + tid; col < pb; col += kSyThreads) ys[col] = peer_f64(xk + col, peer);
      // reflector storage in row k (dead from here on), written once both CTAs have read the
      // column from that row (step 1 of this column step precedes the barrier in each)
      if (lead)
        for (int i = k + 1 + tid; i < n; i += kSyThreads) A[(int64_t)k * n + i] = cs[i];
      // W^T v and V^T v for the panel's earlier columns (warp l takes column l)
      for (int l = warp; l < j; l += kSyThreads / 32) {
        double s1 = 0.0, s2 = 0.0;
        for (int i = k + 1 + lane; i < n; i += 32) {
          s1 = fma(Wp[(int64_t)l * n + i], cs[i], s1);
          s2 = fma(Vp[(int64_t)l * n + i], cs[i], s2);
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        if (lane == 0) {
          t1[l] = s1;
          t2[l] = s2;
        }
      }
      __syncthreads();
      double sp = 0.0;
      for (int col = k + 1 + tid; col < n; col += kSyThreads) {
        double y = ys[col];
        for (int l = 0; l < j; ++l) y -= Vp[(int64_t)l * n + col] * t1[l] + Wp[(int64_t)l * n + col] * t2[l];
        const double w = tk * y;
        ys[col] = w;
        sp = fma(w, cs[col], sp);
      }
      const double wv = block_sum(sp, red);
      // 4. w = tau y - (tau / 2) (tau y . v) v
      const double a2 = -0.5 * tk * wv;
      for (int i = tid; i < n; i += kSyThreads) Wp[(int64_t)j * n + i] = i > k ? ys[i] + a2 * cs[i] : 0.0;
      __syncthreads();
    }
    // trailing update of rows and columns k1 .. n - 1: A -= V W^T + W V^T over the panel. A thread
    // takes a column and a block of kRowChunk rows (accumulators in registers); the rows' factors
    // are staged in shared memory.
    const int k1 = k0 + kb;
    const int hc = (n - k1 + 1) >> 1;
    const int ca = lead ? k1 : k1 + hc, cb = lead ? k1 + hc : n;   // this CTA's columns
    double* sV = stg;
    double* sW = stg + kNB * kRowChunk;
    for (int i0 = k1; i0 < n; i0 += kRowChunk) {
      const int nr = min(kRowChunk, n - i0);
      __syncthreads();
      for (int u = tid; u < kb * kRowChunk; u += kSyThreads) {
        const int l = u / kRowChunk, rr = u - l * kRowChunk;
        const bool ok = rr < nr;
        sV[u] = ok ? Vp[(int64_t)l * n + i0 + rr] : 0.0;
        sW[u] = ok ? Wp[(int64_t)l * n + i0 + rr] : 0.0;
      }
      __syncthreads();
      for (int c = ca + tid; c < cb; c += kSyThreads) {
        double acc[kRowChunk];
#pragma unroll
        for (int rr = 0; rr < kRowChunk; ++rr) acc[rr] = 0.0;
        for (int l = 0; l < kb; ++l) {
          const double vc = Vp[(int64_t)l * n + c], wc = Wp[(int64_t)l * n + c];
#pragma unroll
          for (int rr = 0; rr < kRowChunk; ++rr)
            acc[rr] = fma(sV[l * kRowChunk + rr], wc, fma(sW[l * kRowChunk + rr], vc, acc[rr]));
        }
#pragma unroll
        for (int rr = 0; rr < kRowChunk; ++rr)
          if (rr < nr) A[(int64_t)(i0 + rr) * n + c] = __ldcg(A + (int64_t)(i0 + rr) * n + c) - acc[rr];
      }
    }
    // the next panel reads rows of the columns the peer updated
    __threadfence();
    cluster_barrier();
  }
  if (lead && tid == 0) {
    if (n >= 2) {
      d[n - 2] = __ldcg(A + (int64_t)(n - 2) * n + n - 2);
      e[n - 2] = __ldcg(A + (int64_t)(n - 1) * n + n - 2);
      tau[n - 2] = 0.0;
    }
    d[n - 1] = __ldcg(A + (int64_t)(n - 1) * n + n - 1);
    e[n - 1] = 0.0;
    tau[n - 1] = 0.0;
  }
}

// Number of eigenvalues of the tridiagonal (d, e2 = e^2) below x: the negative pivots of the
// LDL^T factorisation of T - x I, a pivot of magnitude below pivmin being taken as -pivmin.
__device__ __forceinline__ int sturm_count(int n, const double* d, const double* e2, double x, double pivmin) {
  double q = d[0] - x;
  if (fabs(q) <= pivmin) q = -pivmin;
  int c = q < 0.0;
  for (int i = 1; i < n; ++i) {
    q = (d[i] - x) - e2[i - 1] / q;
    if (fabs(q) <= pivmin) q = -pivmin;
    c += q < 0.0;
  }
  return c;
}

// R largest eigenvalues (descending) of each tridiagonal by bisection; one thread per eigenvalue.
__global__ void __launch_bounds__(128) k_stebz(int n, int R, const double* d_all, const double* e_all,
                                               double* lam_all, int64_t sL) {
  extern __shared__ double smb[];
  double* d = smb;
  double* e2 = d + n;
  __shared__ double glo, ghi, pmin;
  const int b = blockIdx.x, tid = threadIdx.x;
  const double* dg = d_all + (int64_t)b * n;
  const double* eg = e_all + (int64_t)b * n;
  for (int i = tid; i < n; i += blockDim.x) {
    d[i] = dg[i];
    e2[i] = i < n - 1 ? eg[i] * eg[i] : 0.0;
  }
  __syncthreads();
  if (tid == 0) {
    double lo = d[0], hi = d[0], emax = 0.0;
    for (int i = 0; i < n; ++i) {
      const double r = (i > 0 ? fabs(eg[i - 1]) : 0.0) + (i < n - 1 ? fabs(eg[i]) : 0.0);
      lo = fmin(lo, d[i] - r);
      hi = fmax(hi, d[i] + r);
      emax = fmax(emax, e2[i]);
    }
    const double w = fmax(fabs(lo), fabs(hi));
    glo = lo - 2.0 * 2.2e-16 * w * n - 1e-300;
    ghi = hi + 2.0 * 2.2e-16 * w * n + 1e-300;
    pmin = 2.2250738585072014e-308 * fmax(1.0, emax);
  }
  __syncthreads();
  for (int r = tid; r < R; r += blockDim.x) {
    const int idx = n - 1 - r;          // ascending index of the r-th largest eigenvalue
    double lo = glo, hi = ghi;
    for (int it = 0; it < 256; ++it) {
      const double mid = 0.5 * (lo + hi);
      if (!(hi - lo > 2.0 * 2.2e-16 * fmax(fabs(lo), fabs(hi))) || mid == lo || mid == hi) break;
      if (sturm_count(n, d, e2, mid, pmin) <= idx) lo = mid;
      else hi = mid;
    }
    lam_all[(int64_t)b * sL + r] = 0.5 * (lo + hi);
  }
}

// SplitMix64 finaliser (Steele, Lea & Flood 2014), for the fixed start vectors.
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Inverse iteration on one tridiagonal (d, e), column-interleaved work arrays: element i of
// column c lives at [i * Rp + c], so that the 32 threads of a warp working on 32 consecutive
// columns touch contiguous memory at every step.
struct TriWork {
  const double *d, *e;
  double *u0, *u1, *u2, *ll, *pv;   // LU of T - lambda I: U's three diagonals, multipliers, swaps
  int n, Rp;
};

__device__ __forceinline__ double tri_norm(const double* d, const double* e, int n) {
  double t = 0.0;
  for (int i = 0; i < n; ++i) t = fmax(t, fabs(d[i]) + (i > 0 ? fabs(e[i - 1]) : 0.0) + (i < n - 1 ? fabs(e[i]) : 0.0));
  return t;
}

// Gaussian elimination with partial pivoting of T - lam I into work column c (one thread); the
// working row i holds (a, bb) at columns (i, i + 1). A zero pivot is replaced by `tiny`.
__device__ void tri_factor(const TriWork& w, int c, double lam, double tiny) {
  const int n = w.n, Rp = w.Rp;
  double a = w.d[0] - lam, bb = n > 1 ? w.e[0] : 0.0;
  for (int i = 0; i < n - 1; ++i) {
    const double cc = w.e[i], an = w.d[i + 1] - lam, bn = i + 2 < n ? w.e[i + 1] : 0.0;
    const int64_t o = (int64_t)i * Rp + c;
    if (fabs(a) >= fabs(cc)) {
      const double p = a != 0.0 ? a : tiny;
      const double l = cc / p;
      w.u0[o] = p; w.u1[o] = bb; w.u2[o] = 0.0; w.ll[o] = l; w.pv[o] = 0.0;
      a = an - l * bb;
      bb = bn;
    } else {
      const double l = a / cc;
      w.u0[o] = cc; w.u1[o] = an; w.u2[o] = bn; w.ll[o] = l; w.pv[o] = 1.0;
      a = bb - l * an;
      bb = -l * bn;
    }
  }
  w.u0[(int64_t)(n - 1) * Rp + c] = a != 0.0 ? a : tiny;
}

// x <- (T - lam I)^{-1} x with the factorisation of work column c; x is column xc of X (same
// interleaving). Returns max |x|. One thread.
__device__ double tri_solve(const TriWork& w, int c, double* X, int xc) {
  const int n = w.n, Rp = w.Rp;
  for (int i = 0; i < n - 1; ++i) {
    const int64_t o = (int64_t)i * Rp + c, xo = (int64_t)i * Rp + xc;
    double xi = X[xo], xj = X[xo + Rp];
    if (w.pv[o] != 0.0) {
      const double t = xi;
      xi = xj;
      xj = t;
    }
    X[xo] = xi;
    X[xo + Rp] = xj - w.ll[o] * xi;
  }
  double xp1 = 0.0, xp2 = 0.0, mx = 0.0;
  for (int i = n - 1; i >= 0; --i) {
    const int64_t o = (int64_t)i * Rp + c, xo = (int64_t)i * Rp + xc;
    const double v = (X[xo] - w.u1[o] * xp1 - w.u2[o] * xp2) / w.u0[o];
    X[xo] = v;
    xp2 = xp1;
    xp1 = v;
    mx = fmax(mx, fabs(v));
  }
  return mx;
}

// Start vector of eigenvector r: uniform in (-1, 1) from the counter (r, i).
__device__ __forceinline__ double start_entry(int r, int i) {
  const uint64_t w = mix64(((uint64_t)(r + 1) << 32) + (uint64_t)i + 0x9E3779B97F4A7C15ull);
  return (double)(w >> 11) * (2.0 / 9007199254740992.0) - 1.0;
}

// Eigenvalues closer than kTight * ||T|| are treated as one cluster: independently computed
// inverse-iteration vectors are orthogonal only to ~eps ||T|| / gap, so the members of such a
// cluster are computed one after another and orthogonalised against each other (below).
constexpr double kTight = 1e-10;

__device__ __forceinline__ TriWork tri_work(int b, int n, int Rp, const double* d_all, const double* e_all,
                                            double* work) {
  const int64_t plane = (int64_t)n * Rp, base = (int64_t)b * 5 * plane;
  TriWork w;
  w.d = d_all + (int64_t)b * n;
  w.e = e_all + (int64_t)b * n;
  w.u0 = work + base;
  w.u1 = w.u0 + plane;
  w.u2 = w.u1 + plane;
  w.ll = w.u2 + plane;
  w.pv = w.ll + plane;
  w.n = n;
  w.Rp = Rp;
  return w;
}

// Eigenvector r of tridiagonal b by inverse iteration (one thread; 32 consecutive r per warp):
// three solves from the start vector, scaled to unit max norm after each, then unit 2-norm.
// Members of a tight cluster are left to k_stein_cluster; T = 0 gives the unit vectors.
__global__ void __launch_bounds__(32) k_stein(int n, int R, int Rp, const double* d_all, const double* e_all,
                                              const double* lam_all, int64_t sL, double* work, double* Z) {
  const int b = blockIdx.x, r = blockIdx.y * 32 + threadIdx.x;
  if (r >= R) return;
  const TriWork w = tri_work(b, n, Rp, d_all, e_all, work);
  double* X = Z + (int64_t)b * n * Rp;
  const double* lam = lam_all + (int64_t)b * sL;
  const double tnorm = tri_norm(w.d, w.e, n);
  if (tnorm == 0.0) {
    for (int i = 0; i < n; ++i) X[(int64_t)i * Rp + r] = i == r ? 1.0 : 0.0;
    return;
  }
  const double tau = kTight * tnorm;
  if ((r > 0 && lam[r - 1] - lam[r] <= tau) || (r + 1 < R && lam[r] - lam[r + 1] <= tau)) return;
  tri_factor(w, r, lam[r], fmax(tnorm * 2.2e-16, 1e-280));
  for (int i = 0; i < n; ++i) X[(int64_t)i * Rp + r] = start_entry(r, i);
  for (int it = 0; it < 3; ++it) {
    const double mx = tri_solve(w, r, X, r);
    const double s = (mx > 0.0 && isfinite(mx)) ? 1.0 / mx : 1.0;
    for (int i = 0; i < n; ++i) X[(int64_t)i * Rp + r] *= s;
  }
  double nn = 0.0;
  for (int i = 0; i < n; ++i) nn = fma(X[(int64_t)i * Rp + r], X[(int64_t)i * Rp + r], nn);
  const double s = nn > 0.0 ? 1.0 / sqrt(nn) : 0.0;
  for (int i = 0; i < n; ++i) X[(int64_t)i * Rp + r] *= s;
}

__device__ __forceinline__ double warp_dot_col(const double* X, int n, int Rp, int c1, int c2) {
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += 32) s = fma(X[(int64_t)i * Rp + c1], X[(int64_t)i * Rp + c2], s);
  return warp_sum(s);
}

// The members r0 .. r1 of a tight cluster (one warp per cluster, launched for every r; only the
// warp of a cluster's first member works): member after member, inverse iteration with its own
// shift, each solve followed by Gram-Schmidt against the members already computed and a
// normalisation, so that the members span the cluster's invariant subspace instead of collapsing
// onto the direction the solves amplify most.
__global__ void __launch_bounds__(32) k_stein_cluster(int n, int R, int Rp, const double* d_all, const double* e_all,
                                                      const double* lam_all, int64_t sL, double* work, double* Z) {
  const int b = blockIdx.x, r0 = blockIdx.y, lane = threadIdx.x;
  const TriWork w = tri_work(b, n, Rp, d_all, e_all, work);
  double* X = Z + (int64_t)b * n * Rp;
  const double* lam = lam_all + (int64_t)b * sL;
  const double tnorm = tri_norm(w.d, w.e, n);
  if (tnorm == 0.0) return;
  const double tau = kTight * tnorm;
  if (r0 > 0 && lam[r0 - 1] - lam[r0] <= tau) return;           // not the first member
  int r1 = r0;
  while (r1 + 1 < R && lam[r1] - lam[r1 + 1] <= tau) ++r1;
  if (r1 == r0) return;                                          // a singleton: done by k_stein
  for (int rr = r0; rr <= r1; ++rr) {
    if (lane == 0) tri_factor(w, r0, lam[rr], fmax(tnorm * 2.2e-16, 1e-280));
    for (int i = lane; i < n; i += 32) X[(int64_t)i * Rp + rr] = start_entry(rr, i);
    __syncwarp();
    for (int it = 0; it < 3; ++it) {
      if (lane == 0) tri_solve(w, r0, X, rr);
      __syncwarp();
      for (int j = r0; j < rr; ++j) {
        const double dj = warp_dot_col(X, n, Rp, j, rr);
        for (int i = lane; i < n; i += 32) X[(int64_t)i * Rp + rr] = fma(-dj, X[(int64_t)i * Rp + j], X[(int64_t)i * Rp + rr]);
        __syncwarp();
      }
      const double nn = warp_dot_col(X, n, Rp, rr, rr);
      const double s = nn > 0.0 && isfinite(nn) ? 1.0 / sqrt(nn) : 0.0;
      for (int i = lane; i < n; i += 32) X[(int64_t)i * Rp + rr] *= s;
      __syncwarp();
    }
  }
}

// Z <- H_0 H_1 ... H_{n-3} Z for the vectors r of one CTA (one warp per vector, the vector in
// shared memory); reflector k is row k of A from column k + 1 on, with its tau.
__global__ void __launch_bounds__(512) k_ormtr(int n, int R, int Rp, int cw, const double* A_all, int64_t sA,
                                               const double* tau_all, double* Z) {
  extern __shared__ double zs[];          // [cw][n]
  const int b = blockIdx.x, c = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * cw + c;
  const double* A = A_all + (int64_t)b * sA;
  const double* tau = tau_all + (int64_t)b * n;
  double* zg = Z + (int64_t)b * n * Rp;
  double* z = zs + (int64_t)c * n;
  if (r >= R) return;
  for (int i = lane; i < n; i += 32) z[i] = zg[(int64_t)i * Rp + r];
  __syncwarp();
  for (int k = n - 3; k >= 0; --k) {
    const double t = tau[k];
    if (t == 0.0) continue;
    const double* v = A + (int64_t)k * n;     // v[k + 1] = 1
    double s = 0.0;
    for (int i = k + 1 + lane; i < n; i += 32) s = fma(v[i], z[i], s);
    s = warp_sum(s) * t;
    __syncwarp();
    for (int i = k + 1 + lane; i < n; i += 32) z[i] = fma(-s, v[i], z[i]);
    __syncwarp();
  }
  for (int i = lane; i < n; i += 32) zg[(int64_t)i * Rp + r] = z[i];
}

}  // namespace

int tridiag_rpad(int R) { return (R + 31) / 32 * 32; }

size_t tridiag_scratch_doubles(int batch, int n, int R) {
  const size_t Rp = (size_t)tridiag_rpad(R);
  return (size_t)batch * (3 * (size_t)n          // d, e, tau
                          + 2 * (size_t)kSyCluster * kNB * n   // panel v, w of each CTA
                          + Rp                   // eigenvalues
                          + 5 * (size_t)n * Rp   // LU of T - lambda I per vector
                          + (size_t)n * Rp);     // eigenvectors [n][Rp]
}

cudaError_t eig_top_dense(int batch, int n, int R, double* A, int64_t sA, double* scratch, double** Zout,
                          double** lam_out, cudaStream_t s) {
  if (batch <= 0) return cudaSuccess;
  if (n < 2 || R < 1 || R > n) return cudaErrorInvalidValue;
  const int Rp = tridiag_rpad(R);
  double* d = scratch;
  double* e = d + (size_t)batch * n;
  double* tau = e + (size_t)batch * n;
  double* Vp = tau + (size_t)batch * n;
  double* Wp = Vp + (size_t)batch * kSyCluster * kNB * n;
  double* lam = Wp + (size_t)batch * kSyCluster * kNB * n;
  double* work = lam + (size_t)batch * Rp;
  double* Z = work + (size_t)batch * 5 * n * Rp;
  const size_t sm1 =
      (4 * (size_t)n + kSyThreads / 32 + 2 * kNB + 4 + 2 * kNB * kRowChunk + 2 * kSyThreads) * sizeof(double);
  if (sm1 > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e1 = cudaFuncSetAttribute(k_sytrd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
  if (e1 != cudaSuccess) return e1;
  k_sytrd<<<batch * kSyCluster, kSyThreads, sm1, s>>>(n, A, sA, d, e, tau, Vp, Wp);
  note_launch();
  const size_t sm2 = 2 * (size_t)n * sizeof(double);
  e1 = cudaFuncSetAttribute(k_stebz, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (e1 != cudaSuccess) return e1;
  k_stebz<<<batch, 128, sm2, s>>>(n, R, d, e, lam, Rp);
  note_launch();
  k_stein<<<dim3(batch, Rp / 32), 32, 0, s>>>(n, R, Rp, d, e, lam, Rp, work, Z);
  note_launch();
  k_stein_cluster<<<dim3(batch, R), 32, 0, s>>>(n, R, Rp, d, e, lam, Rp, work, Z);
  note_launch();
  int cw = 16;
  while (cw > 1 && (size_t)cw * n * sizeof(double) > 200 * 1024) cw /= 2;
  const size_t sm4 = (size_t)cw * n * sizeof(double);
  e1 = cudaFuncSetAttribute(k_ormtr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm4);
  if (e1 != cudaSuccess) return e1;
  k_ormtr<<<dim3(batch, (R + cw - 1) / cw), 32 * cw, sm4, s>>>(n, R, Rp, cw, A, sA, tau, Z);
  note_launch();
  *Zout = Z;
  *lam_out = lam;
  return cudaGetLastError();
}

}  // namespace jolt
