// Eigenpairs of small dense symmetric matrices (order n <= 128, float64 input) by a direct
// method: the JoLT codec's feature Gram C_D (D x D) and the FlashJoLT Rayleigh-Ritz matrix
// B B^T (l x l) ("A JoLT for the KV Cache", arXiv 2607.12550v2, Abstract: the partial Tucker
// factors are the leading eigenvectors of these Grams).
//
// One CTA of 512 threads per matrix; the matrix lives in registers, the rest in shared memory.
// Steps (Golub & Van Loan, Matrix Computations, 4th ed.):
//  1. A is scaled by 2^-e so that its largest absolute row sum lies in [1/2, 1) (exact).
//  2. Householder tridiagonalisation A = Q T Q^T (sec. 8.3.1) with A in registers: thread
//     (i, q) holds row i, columns 32 q .. 32 q + 31. Step k takes x = A[k+1 : n, k],
//     beta = -sign(x_0) ||x||, u = x - beta e_1 (rows k + 1 .. n - 1), tau = 2 / u^T u =
//     1 / (beta (beta - x_0)), p = tau A u, w = p - (tau / 2)(p^T u) u and A <- A - u w^T - w u^T;
//     T's diagonal entry is A[k][k], its subdiagonal entry beta. A warp whose rows or columns
//     all lie in the reduced part skips the step's products. The reflectors are kept for step 5
//     from the 32-row group of row k + 1 on, zeros below, so that step needs no masks.
//  3. All n eigenvalues of T by bisection (sec. 8.4.1) on the Sturm count, the number of sign
//     changes along the leading principal minors p_i(x) of T - x I, which follow
//     p_i = (d_i - x) p_{i-1} - e_{i-1}^2 p_{i-2}: no division, the pair rescaled by a power of
//     two every eight terms. A first round counts at 511 points of the Gershgorin interval (one
//     per thread) and gives each eigenvalue its bracket; then one thread per eigenvalue bisects
//     down to an interval of 2 eps max(|lo|, |hi|) + 4 eps ||T||.
//  4. The eigenvector of T for each eigenvalue from the twisted factorisation of T - lambda I
//     (Parlett & Dhillon, "Fernando's solution to Wilkinson's problem: an application of double
//     factorization", Linear Algebra Appl. 267 (1997)): forward pivots D+_i, backward pivots
//     D-_i, the twist index r where |gamma_r| = |D+_r + D-_r - (d_r - lambda)| is smallest,
//     then z_r = 1, z_i = -(e_i / D+_i) z_{i+1} above r and z_i = -(e_{i-1} / D-_i) z_{i-1}
//     below. One thread per vector. Eigenvalues within 1e-8 ||T|| of a neighbour form a
//     cluster, whose vectors are not determined one by one: its members are computed by
//     inverse iteration one after another (three solves with T - lambda I, Gaussian
//     elimination with partial pivoting), each solve followed by Gram-Schmidt against the
//     members already done (one warp).
//  5. Back-transformation Z <- H_0 H_1 ... H_{n-3} Z (sec. 5.1.6) with Z in registers: thread
//     (c, g) holds rows 32 g .. 32 g + 31 of vector c. Four reflectors per barrier, in the
//     compact form of their product: the four dot products u^T z from the same z, corrected by
//     the u^T u of the pairs (formed by the idle warps during step 4).
// Output as the one-sided Jacobi solver's: eigenvalues descending, the vectors as columns of a
// row-major n x n array, float32. Vectors are orthonormal to ~eps ||A|| / gap, eigenvalues
// accurate to a few eps ||A||.
#include "../jolt_internal.h"
#include <type_traits>

namespace jolt {
namespace {

constexpr int kN = kMaxN;                  // padded order
constexpr int kT = 512;                    // threads per matrix
constexpr int kStage = kN + 1;             // row stride of the staged input
constexpr double kEps = 2.220446049250313e-16;
constexpr double kSturmFloor = 0x1p-60;    // added to |d_i - x| in the Sturm count (||T|| < 1)
constexpr double kTwistPiv = 0x1p-400;     // smallest magnitude of a twisted-factorisation pivot
constexpr double kClusterTol = 1e-8;       // relative to ||T||: orthogonality ~eps / 1e-8 outside clusters

// Reflector k is kept from the first row of the 32-row group holding row k + 1 to row kN - 1,
// zeros up to row k and beyond row n - 1, at Up[ub[k] + row]: a thread reading its group's 32
// rows of a reflector needs no mask. Every reflector takes a multiple of 32 entries, so the
// pairs of rows are 16-byte aligned.
constexpr int kUp = 10080;   // sum over k < kN - 2 of kN - 32 floor((k + 1) / 32)

// shared memory, in doubles
constexpr int kOffUp = 0;
constexpr int kOffZ = kOffUp + kUp;             // Z: [kN][kN], vector c in column c
constexpr int kOffD = kOffZ + kN * kN;          // d, e, e2, tau, lam, znrm
constexpr int kOffX = kOffD + 6 * kN;           // the current column x, two buffers
constexpr int kOffW = kOffX + 2 * kN;           // row k + 1 of A, two buffers
constexpr int kOffP = kOffW + 2 * kN;           // partial sums [2][4][kN]; LU scratch of a cluster
constexpr int kOffMisc = kOffP + 8 * kN;        // 64 scalars, then the reflector bases (kN ints)
constexpr int kSmemDoubles = kOffMisc + 64 + kN / 2;
static_assert(kOffZ + kN * kStage <= kOffX, "the staged input overlays Z and the vectors after it");
static_assert(kSmemDoubles * 8 <= 227 * 1024, "shared memory of one CTA");

struct SmallBatch {
  const double* C;
  int64_t sC;
  float* V;
  int64_t sV;
  float* lam;
  int64_t sL;
  int n, count;
};

template <int K0, int N, class F>
__device__ __forceinline__ void unroll_steps(F& f) {
  if constexpr (K0 < N) {
    f(std::integral_constant<int, K0>{});
    unroll_steps<K0 + 1, N>(f);
  }
}

// Butterfly reductions: every lane ends with the same value.
__device__ __forceinline__ double wsum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double wmax(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double wmin(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Rescale the pair (p, pp) by the power of two that brings the larger into [1, 2) (exact).
__device__ __forceinline__ void rescale_pair(double& p, double& pp) {
  const double m = fmax(fabs(p), fabs(pp));
  const int ex = ((__double2hiint(m) >> 20) & 0x7ff) - 1023;
  const double sc = __hiloint2double((1023 - ex) << 20, 0);   // 2^-ex
  p *= sc;
  pp *= sc;
}

// Number of eigenvalues of T below x: sign changes along p_{-1} = 1, p_0, ..., p_{n-1}, p_i the
// leading (i + 1) x (i + 1) minor of T - x I, p_i = (d_i - x) p_{i-1} - f_i p_{i-2} with f_i =
// e_{i-1}^2 (f_0 = 0). A zero minor inside the sequence adds exactly one change whichever sign it
// is given. |d_i - x| is raised by kSturmFloor, keeping the sign bit (a change of T far below
// eps ||T||): across a split (e_i = 0) the minors are products of the d_i - x, and a
// repeated diagonal value hit exactly by x would otherwise underflow them to zero between two
// rescalings, after which no sign change counts. d and f are padded to n8 (a multiple of 8) with
// d_i = 4 > x and f_i = 0, which change no sign; eight terms per chunk, the next chunk's
// coefficients loaded while the current one runs.
__device__ __forceinline__ double sturm_term(double v) {
  return v + copysign(kSturmFloor, v);   // (|v| + 2^-60) with the sign bit of v
}

__device__ __forceinline__ int sturm_below(int n8, const double* d, const double* f, double x) {
  const double2* d2 = reinterpret_cast<const double2*>(d);
  const double2* f2 = reinterpret_cast<const double2*>(f);
  double p = 1.0, pp = 0.0;
  int c = 0;
  double2 dv[4], fv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    dv[u] = d2[u];
    fv[u] = f2[u];
  }
  for (int i0 = 0; i0 < n8; i0 += 8) {
    const int nx = (i0 + 8 < n8 ? i0 + 8 : i0) >> 1;
    double2 dn[4], fn[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dn[u] = d2[nx + u];
      fn[u] = f2[nx + u];
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const double dd = (u & 1) ? dv[u >> 1].y : dv[u >> 1].x;
      const double ff = (u & 1) ? fv[u >> 1].y : fv[u >> 1].x;
      const double pn = fma(sturm_term(dd - x), p, -(ff * pp));
      c += (int)((unsigned)(__double2hiint(pn) ^ __double2hiint(p)) >> 31);
      pp = p;
      p = pn;
    }
    rescale_pair(p, pp);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dv[u] = dn[u];
      fv[u] = fn[u];
    }
  }
  return c;
}

__device__ __forceinline__ double twist_pivot(double v) {
  return fabs(v) >= kTwistPiv ? v : (v < 0.0 ? -kTwistPiv : kTwistPiv);
}

// Eigenvector of T for the eigenvalue lmb by the twisted factorisation; z is column j of Z
// (stride kN), used for the pivots on the way. Returns 1 / ||z||. The forward pivots are
// D+_i = p_i / p_{i-1} with p the leading minors of T - lmb I, the backward ones D-_i =
// s_i / s_{i+1} with s the trailing minors (s_i = (d_i - lmb) s_{i+1} - f_{i+1} s_{i+2}): the
// recurrences run on the minors (rescaled by powers of two every eight terms), so the divisions
// stay off their dependency chains. A minor that comes out exactly zero is replaced by kTwistPiv
// times the previous one (pivot +-kTwistPiv, as for the quotient form).
__device__ double twisted_vector(int n, const double* d, const double* e, const double* f, double lmb,
                                 double* z) {
  double p = 1.0, pp = 0.0;
  for (int i = 0; i < n; ++i) {
    double pn = fma(d[i] - lmb, p, -(f[i] * pp));
    if (pn == 0.0) pn = kTwistPiv * p;
    z[i * kN] = twist_pivot(pn / p);
    pp = p;
    p = pn;
    if ((i & 7) == 7) rescale_pair(p, pp);
  }
  double s = 1.0, ss = 0.0, best = 0.0;
  int r = n - 1;
  for (int i = n - 1; i >= 0; --i) {
    const double ti = d[i] - lmb;
    double sn = fma(ti, s, -((i + 1 < n ? f[i + 1] : 0.0) * ss));
    if (sn == 0.0) sn = kTwistPiv * s;
    const double g = fabs(z[i * kN] + twist_pivot(sn / s) - ti);
    if (i == n - 1 || g < best) {
      best = g;
      r = i;
    }
    ss = s;
    s = sn;
    if ((i & 7) == 0) rescale_pair(s, ss);
  }
  s = 1.0;
  ss = 0.0;
  for (int i = n - 1; i > r; --i) {
    double sn = fma(d[i] - lmb, s, -((i + 1 < n ? f[i + 1] : 0.0) * ss));
    if (sn == 0.0) sn = kTwistPiv * s;
    z[i * kN] = twist_pivot(sn / s);
    ss = s;
    s = sn;
    if ((i & 7) == 0) rescale_pair(s, ss);
  }
  double v = 1.0, nn = 1.0;
  z[r * kN] = 1.0;
  for (int i = r - 1; i >= 0; --i) {
    v = -(e[i] / z[i * kN]) * v;
    z[i * kN] = v;
    nn = fma(v, v, nn);
  }
  v = 1.0;
  for (int i = r + 1; i < n; ++i) {
    v = -(e[i - 1] / z[i * kN]) * v;
    z[i * kN] = v;
    nn = fma(v, v, nn);
  }
  return 1.0 / sqrt(nn);
}

// Gaussian elimination with partial pivoting of T - lmb I (one thread). Row i of the working
// matrix is (a, bb) at columns (i, i + 1); the factors go to wk = [u0 | u1 | u2 | l | swap] (kN
// each): U's three diagonals, the multipliers and the row interchanges. A zero pivot is
// replaced by tiny.
__device__ void tri_lu(int n, const double* d, const double* e, double lmb, double tiny, double* wk) {
  double* u0 = wk;
  double* u1 = u0 + kN;
  double* u2 = u1 + kN;
  double* ll = u2 + kN;
  double* sw = ll + kN;
  double a = d[0] - lmb, bb = n > 1 ? e[0] : 0.0;
  for (int i = 0; i < n - 1; ++i) {
    const double cc = e[i], an = d[i + 1] - lmb, bn = i + 2 < n ? e[i + 1] : 0.0;
    if (fabs(a) >= fabs(cc)) {
      const double p = a != 0.0 ? a : tiny;
      const double l = cc / p;
      u0[i] = p;
      u1[i] = bb;
      u2[i] = 0.0;
      ll[i] = l;
      sw[i] = 0.0;
      a = an - l * bb;
      bb = bn;
    } else {
      const double l = a / cc;
      u0[i] = cc;
      u1[i] = an;
      u2[i] = bn;
      ll[i] = l;
      sw[i] = 1.0;
      a = bb - l * an;
      bb = -l * bn;
    }
  }
  u0[n - 1] = a != 0.0 ? a : tiny;
}

// z <- (T - lmb I)^{-1} z with the factors of tri_lu (one thread), then z scaled to unit max
// norm; z is a column of Z (stride kN).
__device__ void tri_lu_solve(int n, const double* wk, double* z) {
  const double* u0 = wk;
  const double* u1 = u0 + kN;
  const double* u2 = u1 + kN;
  const double* ll = u2 + kN;
  const double* sw = ll + kN;
  for (int i = 0; i < n - 1; ++i) {
    double xi = z[i * kN], xj = z[(i + 1) * kN];
    if (sw[i] != 0.0) {
      const double tmp = xi;
      xi = xj;
      xj = tmp;
    }
    z[i * kN] = xi;
    z[(i + 1) * kN] = xj - ll[i] * xi;
  }
  double x1 = 0.0, x2 = 0.0, mx = 0.0;
  for (int i = n - 1; i >= 0; --i) {
    const double v = (z[i * kN] - u1[i] * x1 - u2[i] * x2) / u0[i];
    z[i * kN] = v;
    x2 = x1;
    x1 = v;
    mx = fmax(mx, fabs(v));
  }
  const double s = (mx > 0.0 && isfinite(mx)) ? 1.0 / mx : 1.0;
  for (int i = 0; i < n; ++i) z[i * kN] *= s;
}

// SplitMix64 finaliser (Steele, Lea & Flood 2014), for the start vectors of cluster members.
__device__ __forceinline__ double start_entry(int m, int i) {
  uint64_t z = ((uint64_t)(m + 1) << 32) + (uint64_t)i + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (double)(z >> 11) * (2.0 / 9007199254740992.0) - 1.0;
}

// Vectors of the clusters of eigenvalues closer than ctol (one warp, the whole matrix).
__device__ void cluster_vectors(int n, const double* d, const double* e, const double* lam, double ctol,
                                double tiny, double* Z, double* znrm, double* wk) {
  const int lane = threadIdx.x & 31;
  int j0 = 0;
  while (j0 < n) {
    int j1 = j0;
    while (j1 + 1 < n && lam[j1 + 1] - lam[j1] <= ctol) ++j1;
    for (int m = j0; j1 > j0 && m <= j1; ++m) {
      double* z = Z + m;
      if (lane == 0) tri_lu(n, d, e, lam[m], tiny, wk);
      for (int i = lane; i < n; i += 32) z[i * kN] = start_entry(m, i);
      __syncwarp();
      for (int it = 0; it < 3; ++it) {
        if (lane == 0) tri_lu_solve(n, wk, z);
        __syncwarp();
        for (int c = j0; c < m; ++c) {
          double s = 0.0;
          for (int i = lane; i < n; i += 32) s = fma(Z[i * kN + c], z[i * kN], s);
          s = wsum(s);
          for (int i = lane; i < n; i += 32) z[i * kN] = fma(-s, Z[i * kN + c], z[i * kN]);
          __syncwarp();
        }
        double s = 0.0;
        for (int i = lane; i < n; i += 32) s = fma(z[i * kN], z[i * kN], s);
        s = wsum(s);
        const double inv = (s > 0.0 && isfinite(s)) ? 1.0 / sqrt(s) : 0.0;
        for (int i = lane; i < n; i += 32) z[i * kN] *= inv;
        __syncwarp();
      }
      if (lane == 0) znrm[m] = 1.0;
    }
    j0 = j1 + 1;
  }
}

__global__ void __launch_bounds__(kT, 1) k_eig_small(SmallBatch b0, SmallBatch b1, int32_t* status) {
  const bool first = (int)blockIdx.x < b0.count;
  const SmallBatch& sb = first ? b0 : b1;
  const int bi = first ? (int)blockIdx.x : (int)blockIdx.x - b0.count;
  const int n = sb.n;
  extern __shared__ __align__(16) double sm[];
  double* Up = sm + kOffUp;
  double* Zs = sm + kOffZ;
  double* d = sm + kOffD;
  double* e = d + kN;
  double* e2 = e + kN;
  double* tau = e2 + kN;
  double* lam = tau + kN;
  double* znrm = lam + kN;
  double* xs = sm + kOffX;
  double* ws = sm + kOffW;
  double* p4 = sm + kOffP;
  double* misc = sm + kOffMisc;
  int* ub = reinterpret_cast<int*>(misc + 64);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int i = t & (kN - 1), q = t >> 7, rb = warp & 3;

  // ---- 1. the lower triangle staged in shared memory (coalesced), mirrored into registers
  const double* Cb = sb.C + (int64_t)bi * sb.sC;
  for (int r = warp; r < n; r += kT / 32)
    for (int c = lane; c <= r; c += 32) Zs[r * kStage + c] = Cb[(int64_t)r * n + c];
  for (int x = t; x < kUp; x += kT) Up[x] = 0.0;
  if (t == 0) {
    int base = 0;
    for (int k = 0; k <= kN - 3; ++k) {
      const int g0 = 32 * ((k + 1) >> 5);
      ub[k] = base - g0;
      base += kN - g0;
    }
  }
  __syncthreads();
  double a[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int c = 32 * q + j;
    a[j] = (i < n && c < n) ? (c <= i ? Zs[i * kStage + c] : Zs[c * kStage + i]) : 0.0;
  }
  double rs = 0.0;
#pragma unroll
  for (int j = 0; j < 32; ++j) rs += fabs(a[j]);
  p4[q * kN + i] = rs;
  const bool bad = __syncthreads_or(!isfinite(rs));
  if (warp < 4) {
    const double v = wmax(p4[i] + p4[kN + i] + p4[2 * kN + i] + p4[3 * kN + i]);
    if (lane == 0) misc[warp] = v;
  }
  __syncthreads();
  const double anorm = fmax(fmax(misc[0], misc[1]), fmax(misc[2], misc[3]));
  if (bad || anorm == 0.0) {
    float* vo = sb.V + (int64_t)bi * sb.sV;
    float* lo_out = sb.lam ? sb.lam + (int64_t)bi * sb.sL : nullptr;
    // a non-finite input gives NaN output and the status flag; the zero matrix has the unit
    // vectors and zero eigenvalues
    const float fill = bad ? __int_as_float(0x7fc00000) : 0.0f;
    for (int x = t; x < n * n; x += kT) vo[x] = bad ? fill : (x / n == x % n ? 1.0f : 0.0f);
    if (lo_out)
      for (int x = t; x < n; x += kT) lo_out[x] = fill;
    if (bad && t == 0 && status) atomicOr(status, ST_NONFINITE);
    return;
  }
  int ex;   // the scale 2^-ex (kept in shared memory until the output)
  frexp(anorm, &ex);
  int* ex_s = reinterpret_cast<int*>(misc + 12);
  if (t == 0) *ex_s = ex;
  {
    const double sc = ldexp(1.0, -ex);
#pragma unroll
    for (int j = 0; j < 32; ++j) a[j] *= sc;
  }

  // ---- 2. Householder tridiagonalisation. Two barriers per step: after the column x is
  // published, and after the partial products A u (p4, one per row and column quarter) and the
  // per-warp partial sums of u^T A u (red) are; each warp then forms the w entries it needs
  // (its rows' and its 32 columns') itself. The steps of each column quarter are unrolled, so
  // that column k + 1 (the one u = x - beta e_{k+1} changes) is a fixed register.
  double* red = misc + 16;
  auto step = [&](auto JJ, int Q) {
    constexpr int jj = decltype(JJ)::value;
    const int k = 32 * Q + jj;
    double* x = xs + (k & 1) * kN;
    if (q == Q) {
      x[i] = i > k ? a[jj] : 0.0;
      if (i == k) d[k] = a[jj];
    }
    __syncthreads();
    const int qmin = (k + 1) >> 5;
    const bool active = (32 * rb + 31 > k) && q >= qmin;
    // sum_j A_ij x_j over this thread's columns (corrected for u below)
    double s = 0.0;
    if (active) {
      const double2* xq = reinterpret_cast<const double2*>(x + 32 * q);
      double s0 = 0.0, s1 = 0.0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const double2 v = xq[j];
        s0 = fma(a[2 * j], v.x, s0);
        s1 = fma(a[2 * j + 1], v.y, s1);
      }
      s = s0 + s1;
    }
    double sg = 0.0;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const double xv = x[lane + 32 * m];
      sg += lane + 32 * m == k + 1 ? 0.0 : xv * xv;
    }
    sg = wsum(sg);
    const double alpha = x[k + 1];
    if (sg == 0.0) {   // already reduced: H_k = I (same decision in every warp)
      if (t == 0) {
        e[k] = alpha;
        tau[k] = 0.0;
      }
      return;
    }
    const double beta = -copysign(sqrt(fma(alpha, alpha, sg)), alpha);
    const double tk = 1.0 / (beta * (beta - alpha));
    double su = 0.0;
    if (active) {
      if constexpr (jj < 31) {
        if (q == Q) s = fma(-beta, a[jj + 1], s);
      } else {
        if (q == Q + 1) s = fma(-beta, a[0], s);
      }
      p4[q * kN + i] = s;
      su = s * (i == k + 1 ? alpha - beta : x[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) su += __shfl_down_sync(0xffffffffu, su, o);
    if (lane == 0) red[warp] = su;
    if (warp == 0) {   // the reflector, for the back-transformation
      double* ur = Up + ub[k];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int row = lane + 32 * m;
        if (row > k && row < n) ur[row] = row == k + 1 ? alpha - beta : x[row];
      }
      if (lane == 0) {
        e[k] = beta;
        tau[k] = tk;
      }
    }
    __syncthreads();
    if (active) {
      // p = tau A u, K = (tau / 2) p^T u, w = p - K u: this thread's row i and column c of
      // the warp's quarter (each warp keeps its own copy of its 32 columns' w)
      const double2* r2 = reinterpret_cast<const double2*>(red);
      double rv[8];
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) {
        const double2 v = r2[w8];
        rv[w8] = v.x + v.y;
      }
      const double uau = ((rv[0] + rv[1]) + (rv[2] + rv[3])) + ((rv[4] + rv[5]) + (rv[6] + rv[7]));
      const double K = 0.5 * tk * tk * uau;
      const int c = 32 * q + lane;
      double pi = 0.0, pc = 0.0;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        if (qq >= qmin) {
          pi += p4[qq * kN + i];
          pc += p4[qq * kN + c];
        }
      }
      const double ui = i == k + 1 ? alpha - beta : x[i];
      const double uc = c == k + 1 ? alpha - beta : x[c];
      const double wi = i > k ? fma(-K, ui, tk * pi) : 0.0;
      double* wq = p4 + 4 * kN + 32 * warp;
      wq[lane] = c > k ? fma(-K, uc, tk * pc) : 0.0;
      __syncwarp();
      // A <- A - u w^T - w u^T on this thread's entries (u_j = x_j but at column k + 1)
      const double2* xq = reinterpret_cast<const double2*>(x + 32 * q);
      const double2* wq2 = reinterpret_cast<const double2*>(wq);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const double2 xv = xq[j], wv = wq2[j];
        a[2 * j] = fma(-ui, wv.x, fma(-wi, xv.x, a[2 * j]));
        a[2 * j + 1] = fma(-ui, wv.y, fma(-wi, xv.y, a[2 * j + 1]));
      }
      if constexpr (jj < 31) {
        if (q == Q) a[jj + 1] = fma(wi, beta, a[jj + 1]);
      } else {
        if (q == Q + 1) a[0] = fma(wi, beta, a[0]);
      }
      __syncwarp();
    }
  };
  for (int Q = 0; Q < 4 && 32 * Q <= n - 3; ++Q) {
    auto body = [&](auto JJ) {
      if (32 * Q + decltype(JJ)::value <= n - 3) step(JJ, Q);
    };
    unroll_steps<0, 32>(body);
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int c = 32 * q + j;
    if (c == n - 2 && i == n - 2) d[n - 2] = a[j];
    if (c == n - 2 && i == n - 1) e[n - 2] = a[j];
    if (c == n - 1 && i == n - 1) d[n - 1] = a[j];
  }
  __syncthreads();

  // ---- 3. eigenvalues: one round of multisection over the Gershgorin interval at 511 points
  // (one per thread), then bisection from the bracket each eigenvalue falls in
  const int n8 = (n + 7) & ~7;
  if (warp == 0) {
    double glo = 1e300, ghi = -1e300;
    for (int r = lane; r < kN; r += 32) {
      if (r < n) {
        const double rad = (r > 0 ? fabs(e[r - 1]) : 0.0) + (r < n - 1 ? fabs(e[r]) : 0.0);
        glo = fmin(glo, d[r] - rad);
        ghi = fmax(ghi, d[r] + rad);
      } else {
        d[r] = 4.0;   // Sturm-count padding (no sign change)
      }
      e2[r] = (r >= 1 && r < n) ? e[r - 1] * e[r - 1] : 0.0;
    }
    glo = wmin(glo);
    ghi = wmax(ghi);
    if (lane == 0) {
      const double tn = fmax(fabs(glo), fabs(ghi));
      const double pad = 2.0 * kEps * n * tn + 1e-300;
      misc[8] = glo - pad;
      misc[9] = ghi + pad;
      misc[10] = tn;
    }
  }
  __syncthreads();
  const double tn = misc[10], g0 = misc[8], g1 = misc[9];
  auto grid_pt = [&](int m) { return m <= 0 ? g0 : (m >= kT ? g1 : fma((double)m, (g1 - g0) * (1.0 / kT), g0)); };
  int* cnt = reinterpret_cast<int*>(p4);   // counts at the kT + 1 grid points
  if (t < kT - 1) cnt[t + 1] = sturm_below(n8, d, e2, grid_pt(t + 1));
  if (t == 0) {
    cnt[0] = 0;
    cnt[kT] = n;
  }
  __syncthreads();
  if (t < n) {
    int mlo = 0, mhi = kT;
    while (mhi - mlo > 1) {
      const int mid = (mlo + mhi) >> 1;
      if (cnt[mid] <= t) mlo = mid;
      else mhi = mid;
    }
    double lo = grid_pt(mlo), hi = grid_pt(mhi);
    const double atol = 4.0 * kEps * tn;
    for (int it = 0; it < 128; ++it) {
      if (hi - lo <= fmax(2.0 * kEps * fmax(fabs(lo), fabs(hi)), atol)) break;
      const double mid = 0.5 * (lo + hi);
      if (!(mid > lo && mid < hi)) break;
      if (sturm_below(n8, d, e2, mid) <= t) lo = mid;
      else hi = mid;
    }
    lam[t] = 0.5 * (lo + hi);
  }
  __syncthreads();

  // ---- 4. eigenvectors of T, one thread per eigenvalue (warps 0-3); meanwhile warps 4-15 form
  // the products cc[delta - 1][k] = u_k^T u_{k+delta}, delta = 1..3, of the blocked
  // back-transformation (in the x and y buffers, free after step 2)
  double* cc = xs;
  const double ctol = kClusterTol * tn;
  if (t < n) {
    const bool clustered = (t > 0 && lam[t] - lam[t - 1] <= ctol) || (t < n - 1 && lam[t + 1] - lam[t] <= ctol);
    if (!clustered) znrm[t] = twisted_vector(n, d, e, e2, lam[t], Zs + t);
  } else if (warp >= 4) {
    for (int idx = warp - 4; idx < 3 * kN; idx += kT / 32 - 4) {
      const int k = idx / 3, dl = idx - 3 * k + 1;
      double v = 0.0;
      if (k + dl <= n - 3) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int row = lane + 32 * m;
          if (row > k + dl && row < n) v = fma(Up[ub[k] + row], Up[ub[k + dl] + row], v);
        }
        v = wsum(v);
      }
      if (lane == 0) cc[(dl - 1) * kN + k] = v;
    }
  }
  __syncthreads();
  if (warp == 0) cluster_vectors(n, d, e, lam, ctol, fmax(tn * kEps, 1e-280), Zs, znrm, p4);
  __syncthreads();

  // ---- 5. back-transformation, thread (c, g) = (i, q), four reflectors per barrier: for
  // H_{k-3} H_{k-2} H_{k-1} H_k z, with a_m = u_{k-m}^T z from the z on entry,
  // w_m = tau_{k-m} (a_m - sum_{m' < m} (u_{k-m}^T u_{k-m'}) w_{m'}) and z <- z - sum_m u_{k-m} w_m
  double z[32];
  {
    const double zn = i < n ? znrm[i] : 0.0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int row = 32 * q + j;
      z[j] = (row < n && i < n) ? Zs[row * kN + i] * zn : 0.0;
    }
  }
  __syncthreads();   // Z becomes the partial-sum buffer [2][4 reflectors][4 row groups][kN]
  int par = 0;
  const int row0 = 32 * q;
  for (int kb = n - 3; kb >= 0; kb -= 4) {
    const int gmin = (max(kb - 3, 0) + 1) >> 5;
    const bool act = q >= gmin;
    double* pb = Zs + par * 16 * kN;
    par ^= 1;
    if (act) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k = kb - m;
        double s0 = 0.0, s1 = 0.0;
        if (k >= 0 && q >= ((k + 1) >> 5)) {   // reflector k is stored from group (k + 1) / 32 on
          const double2* u2 = reinterpret_cast<const double2*>(Up + ub[k] + row0);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const double2 uv = u2[j];
            s0 = fma(uv.x, z[2 * j], s0);
            s1 = fma(uv.y, z[2 * j + 1], s1);
          }
        }
        pb[(4 * m + q) * kN + i] = s0 + s1;
      }
    }
    __syncthreads();
    if (act) {
      double w[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k = kb - m;
        double v = 0.0;
        for (int gg = gmin; gg < 4; ++gg) v += pb[(4 * m + gg) * kN + i];
#pragma unroll
        for (int mp = 0; mp < m; ++mp) v = fma(-cc[(m - mp - 1) * kN + (k >= 0 ? k : 0)], w[mp], v);
        w[m] = k >= 0 ? tau[k] * v : 0.0;
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k = kb - m;
        if (k >= 0 && q >= ((k + 1) >> 5)) {
          const double2* u2 = reinterpret_cast<const double2*>(Up + ub[k] + row0);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const double2 uv = u2[j];
            z[2 * j] = fma(-uv.x, w[m], z[2 * j]);
            z[2 * j + 1] = fma(-uv.y, w[m], z[2 * j + 1]);
          }
        }
      }
    }
  }

  // ---- 6. output: eigenvalues descending, vector of ascending index c in column n - 1 - c
  float* vo = sb.V + (int64_t)bi * sb.sV;
  float* lo_out = sb.lam ? sb.lam + (int64_t)bi * sb.sL : nullptr;
  bool nonfinite = false;
  if (i < n) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int row = 32 * q + j;
      if (row < n) {
        vo[(int64_t)row * n + (n - 1 - i)] = (float)z[j];
        nonfinite |= !isfinite(z[j]);
      }
    }
  }
  if (t < n) {
    const double l = ldexp(lam[t], *ex_s);
    nonfinite |= !isfinite(l);
    if (lo_out) lo_out[n - 1 - t] = (float)l;
  }
  if (nonfinite && status) atomicOr(status, ST_NONFINITE);
}

}  // namespace

cudaError_t eig_small2(int batch0, int n0, const double* C0, int64_t sC0, float* V0, int64_t sV0, float* lam0,
                       int64_t sL0, int batch1, int n1, const double* C1, int64_t sC1, float* V1, int64_t sV1,
                       float* lam1, int64_t sL1, int32_t* status, cudaStream_t s) {
  if (n0 <= 0 || n0 > kN || (batch1 > 0 && (n1 <= 0 || n1 > kN))) return cudaErrorInvalidValue;
  if (batch0 + batch1 <= 0) return cudaSuccess;
  const size_t smem = (size_t)kSmemDoubles * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(k_eig_small, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  SmallBatch b0{C0, sC0, V0, sV0, lam0, sL0, n0, batch0};
  SmallBatch b1{C1, sC1, V1, sV1, lam1, sL1, batch1 > 0 ? n1 : n0, batch1 > 0 ? batch1 : 0};
  k_eig_small<<<batch0 + b1.count, kT, smem, s>>>(b0, b1, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
