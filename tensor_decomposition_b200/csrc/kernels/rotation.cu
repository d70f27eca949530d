// Seeded randomness of the codec: the counter-based normal generator, the Gaussian sketch
// matrices of the FlashJoLT token factor, and the rotation Pi (Haar, or randomized Hadamard).
//
// "A JoLT for the KV Cache" (arXiv 2607.12550v2, Abstract) rotates the truncation residual
// by a random orthogonal matrix before the low-bit quantisation; the news summary of the
// paper (aimodeling.com, English summary) calls it a Johnson-Lindenstrauss rotation that
// whitens the residual. The library draws it as a Haar matrix: the Q factor of a D x D
// standard-normal matrix with the signs of R's diagonal moved into Q (Mezzadri 2007).
//
// Generator (stated here because the CPU oracle implements it independently):
// SplitMix64 (Steele, Lea & Flood 2014). key(seed, stream) = mix64(seed + mix64(stream + 1));
// word i = mix64(key + (i + 1) * 0x9E3779B97F4A7C15); uniform = (word >> 11) * 2^-53;
// normal n = Box-Muller pair n / 2, cos branch for even n, sin branch for odd n:
// r = sqrt(-2 ln(1 - u1)), theta = 6.283185307179586 * u2.
#include "../jolt_internal.h"

namespace jolt {
namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr double kTwoPi = 6.283185307179586;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double uniform53(uint64_t key, uint64_t i) {
  return (double)(mix64(key + (i + 1ull) * kGamma) >> 11) * 0x1.0p-53;
}

__device__ __forceinline__ double normal_at(uint64_t key, uint64_t n) {
  const uint64_t j = n >> 1;
  const double u1 = uniform53(key, 2 * j);
  const double u2 = uniform53(key, 2 * j + 1);
  const double r = sqrt(-2.0 * log(1.0 - u1));
  const double th = kTwoPi * u2;
  return (n & 1) ? r * sin(th) : r * cos(th);
}

__global__ void k_gauss_f64(uint64_t key, int64_t n, double* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = normal_at(key, (uint64_t)i);
}

struct OmegaKeys {
  uint64_t key[kMaxLT];
};

// Omega element (i, j) is normal number i * l + j of the layer-tensor's stream.
__global__ void k_sketch_omega(OmegaKeys keys, int64_t HD, int l, int transposed, __nv_bfloat16* out) {
  const int lt = blockIdx.y;
  const uint64_t key = keys.key[lt];
  const int64_t per = HD * l;
  __nv_bfloat16* o = out + (int64_t)lt * per;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < per;
       e += (int64_t)gridDim.x * blockDim.x) {
    // transposed: output index e = j * HD + i holds element (i, j); writes stay contiguous
    const uint64_t n = transposed ? (uint64_t)((e % HD) * l + e / HD) : (uint64_t)e;
    o[e] = __double2bfloat16(normal_at(key, n));
  }
}

// One CTA: Householder QR of G (D x D, float64, in shared memory), Q formed in place by
// backward accumulation of the reflectors, then Pi = Q diag(sign(R_kk)).
// Reflector k: beta = -sign(alpha) ||x||, tau = (beta - alpha) / beta, v = x / (alpha - beta),
// v_0 = 1, so that (I - tau v v^T) x = beta e_1.
__global__ void k_haar_qr(const double* G, int n, float* Pi32, __nv_bfloat16* Pib) {
  extern __shared__ double sm[];
  const int ld = n + 1;
  double* A = sm;                 // n x ld
  double* tau = A + n * ld;       // n
  double* beta = tau + n;         // n
  double* w = beta + n;           // n
  __shared__ double red[32];
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int i = tid; i < n * n; i += nt) A[(i / n) * ld + (i % n)] = G[i];
  __syncthreads();
  for (int k = 0; k < n; ++k) {
    // sigma^2 = sum_{i>k} A[i][k]^2 (fixed-order: thread i partials, then warp tree)
    double part = 0.0;
    for (int i = k + 1 + tid; i < n; i += nt) part += A[i * ld + k] * A[i * ld + k];
    for (int o = 16; o > 0; o >>= 1) part += __shfl_down_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) red[tid >> 5] = part;
    __syncthreads();
    if (tid == 0) {
      double sig = 0.0;
      for (int wq = 0; wq < (nt + 31) / 32; ++wq) sig += red[wq];
      const double alpha = A[k * ld + k];
      double t = 0.0, b = alpha, scal = 0.0;
      if (sig != 0.0) {
        const double nrm = sqrt(alpha * alpha + sig);
        b = alpha >= 0.0 ? -nrm : nrm;
        t = (b - alpha) / b;
        scal = 1.0 / (alpha - b);
      }
      tau[k] = t;
      beta[k] = b;
      w[0] = scal;
    }
    __syncthreads();
    const double scal = w[0];
    __syncthreads();
    for (int i = k + 1 + tid; i < n; i += nt) A[i * ld + k] *= scal;
    if (tid == 0) A[k * ld + k] = 1.0;   // v_0 = 1 during the update
    __syncthreads();
    const double tk = tau[k];
    // w_j = sum_{i>=k} v_i A[i][j], j > k
    for (int j = k + 1 + tid; j < n; j += nt) {
      double s = 0.0;
      for (int i = k; i < n; ++i) s += A[i * ld + k] * A[i * ld + j];
      w[j] = s;
    }
    __syncthreads();
    for (int idx = tid; idx < (n - k) * (n - k - 1); idx += nt) {
      const int i = k + idx / (n - k - 1);
      const int j = k + 1 + idx % (n - k - 1);
      A[i * ld + j] -= tk * A[i * ld + k] * w[j];
    }
    __syncthreads();
  }
  // Q = H_0 ... H_{n-1} I, overwriting the reflectors (columns from last to first).
  for (int k = n - 1; k >= 0; --k) {
    const double tk = tau[k];
    if (k < n - 1) {
      if (tid == 0) A[k * ld + k] = 1.0;
      __syncthreads();
      for (int j = k + 1 + tid; j < n; j += nt) {
        double s = 0.0;
        for (int i = k; i < n; ++i) s += A[i * ld + k] * A[i * ld + j];
        w[j] = s;
      }
      __syncthreads();
      for (int idx = tid; idx < (n - k) * (n - k - 1); idx += nt) {
        const int i = k + idx / (n - k - 1);
        const int j = k + 1 + idx % (n - k - 1);
        A[i * ld + j] -= tk * A[i * ld + k] * w[j];
      }
      __syncthreads();
    }
    for (int i = k + 1 + tid; i < n; i += nt) A[i * ld + k] *= -tk;
    if (tid == 0) A[k * ld + k] = 1.0 - tk;
    for (int i = tid; i < k; i += nt) A[i * ld + k] = 0.0;
    __syncthreads();
  }
  for (int i = tid; i < n * n; i += nt) {
    const int r = i / n, c = i % n;
    const double v = beta[c] < 0.0 ? -A[r * ld + c] : A[r * ld + c];
    Pi32[i] = (float)v;
    if (Pib) Pib[i] = __float2bfloat16_rn((float)v);
  }
}

// Randomized Hadamard rotation Pi = diag(s) H / sqrt(D) (the structured Johnson-Lindenstrauss
// transform of Ailon & Chazelle 2006), D a power of two: H is the Sylvester Hadamard matrix,
// H[i][j] = (-1)^popcount(i & j), and s_i = -1 when the top bit of word i of the rotation stream
// is set, +1 otherwise. Entry (i, j) is formed in float64 and rounded like the Haar matrix.
__global__ void k_hadamard_pi(uint64_t key, int D, float* Pi32, __nv_bfloat16* Pib) {
  const double inv = 1.0 / sqrt((double)D);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < D * D; e += gridDim.x * blockDim.x) {
    const int i = e / D, j = e - i * D;
    const bool neg_s = (mix64(key + ((uint64_t)i + 1ull) * kGamma) >> 63) != 0;
    const bool neg_h = (__popc(i & j) & 1) != 0;
    const double v = (neg_s != neg_h) ? -inv : inv;
    Pi32[e] = (float)v;
    if (Pib) Pib[e] = __float2bfloat16_rn((float)v);
  }
}

}  // namespace

static uint64_t host_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

cudaError_t gauss_f64(uint64_t seed, uint64_t stream_id, int64_t n, double* out, cudaStream_t s) {
  const uint64_t key = host_mix64(seed + host_mix64(stream_id + 1ull));
  const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
  k_gauss_f64<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(key, n, out);
  note_launch();
  return cudaGetLastError();
}

cudaError_t sketch_omega(uint64_t seed, const int32_t* lt_ids, int n_lt, int64_t HD, int l,
                         __nv_bfloat16* out, bool transposed, cudaStream_t s) {
  if (n_lt > kMaxLT) return cudaErrorInvalidValue;
  OmegaKeys keys;
  for (int i = 0; i < n_lt; ++i)
    keys.key[i] = host_mix64(seed + host_mix64((uint64_t)(2 + lt_ids[i]) + 1ull));
  const int64_t per = HD * l;
  int bx = (int)((per + 255) / 256);
  if (bx > 64) bx = 64;
  k_sketch_omega<<<dim3(bx, n_lt), 256, 0, s>>>(keys, HD, l, transposed ? 1 : 0, out);
  note_launch();
  return cudaGetLastError();
}

cudaError_t hadamard_pi(uint64_t seed, int D, float* Pi_f32, __nv_bfloat16* Pi_bf16, cudaStream_t s) {
  if (D <= 0 || (D & (D - 1))) return cudaErrorInvalidValue;
  const uint64_t key = host_mix64(seed + host_mix64(1ull + 1ull));   // the rotation stream (1)
  k_hadamard_pi<<<(D * D + 255) / 256, 256, 0, s>>>(key, D, Pi_f32, Pi_bf16);
  note_launch();
  return cudaGetLastError();
}

cudaError_t haar_from_gauss(const double* G, int D, float* Pi_f32, __nv_bfloat16* Pi_bf16,
                            cudaStream_t s) {
  const size_t smem = ((size_t)D * (D + 1) + 3 * (size_t)D) * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(k_haar_qr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_haar_qr<<<1, 512, smem, s>>>(G, D, Pi_f32, Pi_bf16);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
