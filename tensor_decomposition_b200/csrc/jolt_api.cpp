// Host runtime of the JoLT codec behind the C ABI declared in include/jolt.h: plan
// validation and workspace, encode / decode orchestration on one CUDA stream, stream
// serialization with CRC-32, and error reporting.
//
// Method: "A JoLT for the KV Cache: Near-Lossless KV Cache Compression via Joint Tucker and
// JL-Residual Allocation for LLMs" (arXiv 2607.12550v2, Abstract). Encode runs the three
// stages of the Abstract in order: partial Tucker analysis of every layer-tensor (token and
// feature factors, core at the largest ranks, truncation-energy table), the single
// Lagrangian dual over all layer groups and both kinds, and the rotated low-bit residual.
#include <algorithm>
#include <array>
#include <atomic>
#include <mutex>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <type_traits>
#include <string>
#include <vector>

#include "jolt_internal.h"
#include "kernels/gemm_tc.h"

using namespace jolt;

namespace {

// Largest token count of the exact encoder: its token Gram is a dense T x T float64 matrix per
// layer-tensor, reduced to tridiagonal form on one SM each.
constexpr int kExactMaxTokens = 4096;

thread_local std::string g_err;

jolt_status fail(jolt_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

#define CK(call)                                                                          \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return fail(e_ == cudaErrorMemoryAllocation ? JOLT_ERR_OOM : JOLT_ERR_CUDA,        \
                  "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
  } while (0)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// kappa_D = E[max_{i<D} z_i^2], z ~ N(0, I_D) = int_0^inf 2y (1 - erf(y/sqrt 2)^D) dy, by
// composite Simpson's rule on [0, 40] with step 1/1024; 1 - erf^D = -expm1(D log1p(-erfc)).
double kappa_of(int D) {
  const int n = 40 * 1024;
  const double h = 40.0 / n;
  auto f = [D](double y) {
    const double e = std::erfc(y / std::sqrt(2.0));
    return 2.0 * y * (-std::expm1((double)D * std::log1p(-e)));
  };
  double s = f(0.0) + f(40.0);
  for (int i = 1; i < n; ++i) s += (i & 1 ? 4.0 : 2.0) * f(i * h);
  return s * h / 3.0;
}

int64_t lt_bytes_h(int H, int T, int D, int rt, int rd, int b) {
  const int64_t tucker = 2 * ((int64_t)T * rt + (int64_t)D * rd + (int64_t)H * rt * rd);
  const int64_t resid = b > 0 ? (int64_t)H * T * (D * b / 8 + 2) : 0;
  return tucker + resid;
}

int group_of_layer(int l, int L, int G) {
  int g = 0;
  while (g + 1 < G && ((int64_t)(g + 1) * L) / G <= l) ++g;
  return g;
}

// CRC-32 (IEEE 802.3, reflected polynomial 0xEDB88320), table driven.
uint32_t crc32_ieee(const uint8_t* p, size_t n, uint32_t crc = 0) {
  static uint32_t table[256];
  static bool init = false;
  if (!init) {
    for (uint32_t i = 0; i < 256; ++i) {
      uint32_t c = i;
      for (int k = 0; k < 8; ++k) c = (c & 1) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
      table[i] = c;
    }
    init = true;
  }
  crc = ~crc;
  for (size_t i = 0; i < n; ++i) crc = table[(crc ^ p[i]) & 0xFFu] ^ (crc >> 8);
  return ~crc;
}

template <typename T>
T* carve(char*& cur, size_t count) {
  cur = reinterpret_cast<char*>(align_up(reinterpret_cast<size_t>(cur), 256));
  T* p = reinterpret_cast<T*>(cur);
  cur += count * sizeof(T);
  return p;
}

// ---------------------------------------------------------------- tracing
// When enabled, each phase of encode / decode is bracketed by CUDA events recorded on the
// stream it runs on, and the kernel launches inside it are counted.
std::atomic<uint64_t> g_launches{0};
std::mutex g_prof_mu;
bool g_prof_on = false;
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
  uint64_t launches;
};
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

class Prof {
 public:
  Prof(const char* name, cudaStream_t s) : name_(name), s_(s) {
    std::lock_guard<std::mutex> g(g_prof_mu);
    if (!g_prof_on) return;
    a_ = take_event();
    l0_ = g_launches.load();
    cudaEventRecord(a_, s_);
  }
  ~Prof() {
    if (!a_) return;
    std::lock_guard<std::mutex> g(g_prof_mu);
    cudaEvent_t b = take_event();
    cudaEventRecord(b, s_);
    g_prof.push_back({name_, a_, b, g_launches.load() - l0_});
  }

 private:
  const char* name_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr;
  uint64_t l0_ = 0;
};
#define PROF_CAT2(a, b) a##b
#define PROF_CAT(a, b) PROF_CAT2(a, b)
#define PROF(name, s) Prof PROF_CAT(prof_, __LINE__)(name, s)

}  // namespace

namespace jolt {
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace jolt

namespace {
// Stream-ordered allocations (stream bodies, small scratch) come from one memory pool per
// device owned by the library. Its release threshold is unbounded, so memory freed with
// cudaFreeAsync stays mapped for the next encode instead of being returned to the driver at
// every synchronisation (the default pool's behaviour, which re-maps tens of MB per call).
constexpr int kPoolDevices = 64;
std::mutex g_pool_mu;
cudaMemPool_t g_pools[kPoolDevices] = {};

// Device allocations requested by the library (read through jolt_alloc_count).
std::atomic<uint64_t> g_allocs{0};

cudaError_t dev_malloc(void** ptr, size_t bytes) {
  g_allocs.fetch_add(1, std::memory_order_relaxed);
  return cudaMalloc(ptr, bytes);
}
template <typename T>
cudaError_t dev_malloc(T** ptr, size_t bytes) {
  return dev_malloc(reinterpret_cast<void**>(ptr), bytes);
}

cudaError_t pool_malloc(void** ptr, size_t bytes, cudaStream_t s) {
  g_allocs.fetch_add(1, std::memory_order_relaxed);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kPoolDevices) return cudaMallocAsync(ptr, bytes, s);
  cudaMemPool_t pool;
  {
    std::lock_guard<std::mutex> g(g_pool_mu);
    if (!g_pools[dev]) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      cudaMemPool_t np;
      e = cudaMemPoolCreate(&np, &props);
      if (e != cudaSuccess) return e;
      uint64_t keep = UINT64_MAX;
      e = cudaMemPoolSetAttribute(np, cudaMemPoolAttrReleaseThreshold, &keep);
      if (e != cudaSuccess) {
        cudaMemPoolDestroy(np);
        return e;
      }
      g_pools[dev] = np;
    }
    pool = g_pools[dev];
  }
  return cudaMallocFromPoolAsync(ptr, bytes, pool, s);
}
template <typename T>
cudaError_t pool_malloc(T** ptr, size_t bytes, cudaStream_t s) {
  return pool_malloc(reinterpret_cast<void**>(ptr), bytes, s);
}
}  // namespace

// ============================================================================ objects
struct jolt_plan_s {
  jolt_shape shape{};
  jolt_config cfg{};
  uint64_t budget = 0;
  int G = 1, encoder = JOLT_ENC_SKETCH, R = 0, l = 0, step = 16, nbits = 0, ngrid = 1, n_lt = 0;
  int bits[9] = {0};
  double phi[9] = {0};
  double kappa = 0;
  int64_t pool_budget[2] = {0, 0};
  std::vector<int32_t> lt_ids;   // buffer index i -> lt = 2*layer + kind (kind-major order)
  int32_t* d_lt_ids = nullptr;
  int32_t* d_cand_order = nullptr;   // dual candidates in tie-break order (bytes, b, r_t, r_d)
  std::vector<int32_t> cand_order;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  // workspace views
  double *xx = nullptr, *xx_part = nullptr;
  double* CD = nullptr;      // feature Grams, float64
  float *UD32 = nullptr, *UDf = nullptr, *lamD = nullptr;
  __nv_bfloat16 *UDb = nullptr, *Om = nullptr, *UTb = nullptr;
  float *Y = nullptr, *Y2 = nullptr, *Z = nullptr, *Z2 = nullptr, *Bm = nullptr,
        *Wv = nullptr, *lamB = nullptr, *UT32 = nullptr, *UTf = nullptr, *P = nullptr, *Gmax = nullptr,
        *VT = nullptr, *lamT = nullptr;
  double *BB = nullptr, *CT = nullptr;   // sketch and token Grams, float64
  double *Wg = nullptr, *Rinv = nullptr, *E = nullptr, *unit_err = nullptr, *Nbuf = nullptr, *Pbuf = nullptr;
  float* PiT = nullptr;   // Pi^T in the residual coder's shared-memory layout
  double *meas_part = nullptr, *meas_lt = nullptr;   // measured-b refinement
  float* Qfinal = nullptr;   // final sketch basis (one of Y / Y2)
  bool q_t = false;          // Qfinal stored as Q^T [l][T] (tensor-core path) instead of Q [T][l]
  bool use_tc = false;       // bf16 inputs with T % 8 == 0: contractions over X on tcgen05
  float* Cpart = nullptr;            // [n][H][D][D] per-head Gram partials
  __nv_bfloat16* QTp[3] = {nullptr, nullptr, nullptr};   // bf16 parts of a float32 basis [n][l][rows]
  __nv_bfloat16* QTp2[3] = {nullptr, nullptr, nullptr};  // second part set (CholeskyQR ping-pong)
  __nv_bfloat16* RTp[3] = {nullptr, nullptr, nullptr};   // parts of R^{-T} (CholeskyQR)
  float* Wpart = nullptr;                                // K-chunk partial Grams (CholeskyQR)
  int qset = 0;                                          // part set holding the final sketch basis
  int q_iters = 1;                                       // power iterations of the subspace iteration
  bool exact_dense = false;                              // exact token factor by the dense eigensolver (T > 128)
  double* tri = nullptr;                                 // its scratch (tridiag_scratch_doubles)
  float* CTpart = nullptr;                               // per-head token Gram partials [n][H][T][T] (tensor cores)
  double *Qx = nullptr, *Gx = nullptr, *Rx = nullptr;    // its CholeskyQR: [n][T][R], [n][R][R] x 2
  float* Wf = nullptr;                                   // float32 CholeskyQR Grams
  __nv_bfloat16* UDt = nullptr;                          // U_D^T (rounded factor, exact in bf16)
  __nv_bfloat16* Pp[3] = {nullptr, nullptr, nullptr};    // bf16 parts of the core intermediate P
  double* Gpi = nullptr;
  float* Pi32 = nullptr;
  __nv_bfloat16* Pib = nullptr;
  bool pi_valid = false;
  uint64_t pi_seed = 0;
  bool om_valid = false;     // the sketch matrices in Om belong to om_seed (a function of the seed only)
  uint64_t om_seed = 0;
  jolt_stream_s* last = nullptr;
  int device = 0;
};

struct jolt_stream_s {
  int L = 0, H = 0, T = 0, D = 0, has_v = 0, G = 1, encoder = 0, step = 16, R = 0, split = 0;
  int rotation = 0;   // 0 Haar, 1 randomized Hadamard
  jolt_dtype dtype = JOLT_BF16;
  uint64_t seed = 0;
  StreamMeta* d_meta = nullptr;
  uint8_t* d_body = nullptr;
  size_t body_cap = 0;
  float* d_Pi = nullptr;
  double* d_Gpi = nullptr;
  int32_t* d_lt_ids = nullptr;
  int n_lt = 0;
  cudaStream_t cs = nullptr;
  jolt_plan_s* plan = nullptr;
};

// ============================================================================ helpers
namespace {

Operand opnd(const void* p, ElemType t, Idx2 batch, Idx2 row, Idx2 k) {
  Operand o;
  o.p = p;
  o.t = t;
  o.batch = batch;
  o.row = row;
  o.k = k;
  return o;
}
OutDesc outd(void* p, ElemType t, Idx2 batch, Idx2 m, Idx2 n) {
  OutDesc o;
  o.p = p;
  o.t = t;
  o.batch = batch;
  o.m = m;
  o.n = n;
  return o;
}
Idx2 I1(int64_t s) {
  Idx2 x;
  x.s_in = s;
  return x;
}
Idx2 I2(int32_t in, int64_t s_in, int64_t s_out) {
  Idx2 x;
  x.in = in;
  x.s_in = s_in;
  x.s_out = s_out;
  return x;
}

// Shifted CholeskyQR of n_lt tall matrices Y (rows x l, row-major, batch stride rows*l):
// pass 1 with shift s = 11 (rows l + l (l + 1)) 2^-53 ||Y||^2 (Fukaya, Kannan, Nakatsukasa,
// Yamamoto & Yanagisawa 2020), later passes unshifted. Intermediate bases of the power
// iteration only need their column space, so they take one pass; the final basis takes two.
// The passes ping-pong between bufA (holding Y) and bufB; the result pointer is returned.
float* cholqr(jolt_plan_s* p, int rows, float* bufA, float* bufB, int passes, int32_t* status,
              cudaStream_t s, jolt_status* st) {
  const int l = p->l, n = p->n_lt;
  float* src = bufA;
  float* dst = bufB;
  *st = JOLT_OK;
  auto ck = [&](cudaError_t e) {
    if (e != cudaSuccess && *st == JOLT_OK) *st = fail(JOLT_ERR_CUDA, "cholqr: %s", cudaGetErrorString(e));
  };
  for (int pass = 0; pass < passes; ++pass) {
    // Wg = src^T src (l x l, float64)
    ck(gemm_simt(n, l, l, rows, opnd(src, EL_F32, I1((int64_t)rows * l), I1(1), I1(l)),
                 opnd(src, EL_F32, I1((int64_t)rows * l), I1(1), I1(l)),
                 outd(p->Wg, EL_F64, I1((int64_t)l * l), I1(l), I1(1)), 1.0, 0.0, s));
    const double shift =
        pass == 0 ? 11.0 * ((double)rows * l + (double)l * (l + 1)) * std::ldexp(1.0, -53) * l : 0.0;
    ck(chol_inv(n, l, p->Wg, (int64_t)l * l, p->Rinv, (int64_t)l * l, shift, status, s));
    // dst = src * Rinv
    ck(gemm_simt(n, rows, l, l, opnd(src, EL_F32, I1((int64_t)rows * l), I1(l), I1(1)),
                 opnd(p->Rinv, EL_F64, I1((int64_t)l * l), I1(1), I1(l)),
                 outd(dst, EL_F32, I1((int64_t)rows * l), I1(l), I1(1)), 1.0, 0.0, s));
    std::swap(src, dst);
  }
  return src;
}

// Tensor maps of the operand views (see kernels/gemm_tc.h).
bool map_x(CUtensorMap* m, const void* X, int L, int H, int T, int D) {
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)T, (uint64_t)H, (uint64_t)L};
  const uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)T * D * 2, (uint64_t)H * T * D * 2};
  return tc_map_bf16(m, X, 4, dims, str);
}
bool map_rows(CUtensorMap* m, const void* P, int64_t K, int64_t rows, int64_t batch) {
  const uint64_t dims[3] = {(uint64_t)K, (uint64_t)rows, (uint64_t)batch};
  const uint64_t str[2] = {(uint64_t)K * 2, (uint64_t)(rows * K * 2)};
  return tc_map_bf16(m, P, 3, dims, str);
}

// [n][rows][K] bf16 with K = chunks * chunk, seen as (chunk, rows, chunks, n): one batch per
// (i, chunk), the tile box spanning 64 entries of a chunk and 128 rows.
bool map_kchunk(CUtensorMap* m, const void* P, int64_t rows, int64_t K, int64_t chunk, int64_t batch) {
  const uint64_t dims[4] = {(uint64_t)chunk, (uint64_t)rows, (uint64_t)(K / chunk), (uint64_t)batch};
  const uint64_t str[3] = {(uint64_t)K * 2, (uint64_t)chunk * 2, (uint64_t)(rows * K * 2)};
  return tc_map_bf16(m, P, 4, dims, str);
}
// [n][H][D][K] bf16 seen as (K, D, H, n): per-head row blocks.
bool map_perhead(CUtensorMap* m, const void* P, int64_t K, int64_t D, int64_t H, int64_t batch) {
  const uint64_t dims[4] = {(uint64_t)K, (uint64_t)D, (uint64_t)H, (uint64_t)batch};
  const uint64_t str[3] = {(uint64_t)K * 2, (uint64_t)(D * K * 2), (uint64_t)(H * D * K * 2)};
  return tc_map_bf16(m, P, 4, dims, str);
}
// Three bf16 parts of a float32 basis [n][l][rows] (rows contiguous). GEMMs that contract over
// the rows read it K-major; those that contract over l read it MN-major (VIEW_MN).
struct PartSet {
  __nv_bfloat16* s[3];
};

// Products of two three-part operands kept for float32 accuracy: (0,0) (0,1) (1,0) (1,1) (0,2) (2,0).
void six_products(TcGemmParams& g) {
  static const int8_t pa[6] = {0, 0, 1, 1, 0, 2}, pb[6] = {0, 1, 0, 1, 2, 0};
  g.npairs = 6;
  for (int i = 0; i < 6; ++i) { g.pair_a[i] = pa[i]; g.pair_b[i] = pb[i]; }
}

// K chunks of a long contraction over K entries: the fewest chunks of at most 2048 entries that
// split K into whole 64-entry blocks; the tensor cores accumulate along one chunk in float32 and
// the chunks are summed in float64 (a float32 accumulator chained over tens of thousands of
// entries lost ~1e-3 rad of the leading token factors at T = 32768). 1 when K <= 2048 or when K
// does not split that way.
int k_chunks(int64_t K) {
  if (K <= 2048) return 1;
  for (int c = 2; c <= 64; ++c)
    if (K % c == 0 && (K / c) % 64 == 0 && K / c <= 2048) return c;
  return 1;
}

// Number of K chunks of a K-split Gram over `rows` entries: up to 16, each a whole number of
// 8-element groups (TMA row-stride rule) and at least 512 long (a chunk's float32 partial Gram
// should not outweigh the operand tiles it reads); 1 when rows does not split.
int gram_chunks(int rows) {
  for (int c = 16; c > 1; c /= 2)
    if (rows % c == 0 && (rows / c) % 8 == 0 && rows / c >= 512) return c;
  return 1;
}

// CholeskyQR on the tensor cores over bf16 parts. A basis Y^T [n][l][rows] is held as three
// bf16 parts (set.s). Each pass forms the Gram W = Y^T Y from the six part products of order
// <= 2 as float32 partial sums over up to 16 chunks of the rows (one CTA each), sums the chunks
// in float64, inverts its Cholesky factor in float64, and forms Q^T = R^{-T} Y^T from the six
// part products of R^{-T} and Y (read MN-major from the same parts), whose epilogue writes Q's
// parts into the other set. Pass 1 adds 1e-6 trace(W)
// to the diagonal (a shifted CholeskyQR step; the accumulation error of the Gram is ~1e-7), so
// the factorisation exists for any sketch; the column space is unchanged by the shift.
// Returns the index of the set that holds the result.
int cholqr_tc(jolt_plan_s* p, int rows, PartSet* sets, int cur, int passes, int32_t* status, cudaStream_t s,
              jolt_status* st) {
  const int l = p->l, n = p->n_lt;
  *st = JOLT_OK;
  auto ck = [&](cudaError_t e) {
    if (e != cudaSuccess && *st == JOLT_OK) *st = fail(JOLT_ERR_CUDA, "cholqr: %s", cudaGetErrorString(e));
  };
  const int nch = gram_chunks(rows);
  for (int pass = 0; pass < passes && *st == JOLT_OK; ++pass) {
    const PartSet& in = sets[cur];
    const PartSet& out = sets[cur ^ 1];
    TcGemmParams g;
    g.status = status;
    for (int i = 0; i < 3; ++i)
      if (!map_kchunk(&g.amap[i], in.s[i], l, rows, rows / nch, n)) {
        *st = fail(JOLT_ERR_CUDA, "tensor map rejected");
        return cur;
      }
    g.av.mode = VIEW_ROWS_K_HEAD;      // (K chunk, rows, chunk, i)
    g.av.H = nch;
    g.na = g.nb = 3;
    g.b_same = 1;
    six_products(g);
    g.M = l; g.N = l; g.KB = (rows / nch + 63) / 64;
    g.C = p->Wpart; g.c_sm = l; g.c_sn = 1; g.c_sb = (int64_t)l * l;
    ck(gemm_tc(n * nch, g, s));
    ck(sum_heads(n, nch, (int64_t)l * l, p->Wpart, nullptr, p->Wg, s));
    ck(chol_inv(n, l, p->Wg, (int64_t)l * l, p->Rinv, (int64_t)l * l, pass == 0 ? 1e-6 * l : 0.0, status, s));
    ck(split_dual(n, l, l, p->Rinv, true, nullptr, p->RTp, s));
    TcGemmParams m;
    m.status = status;
    for (int i = 0; i < 3; ++i)
      if (!map_rows(&m.amap[i], p->RTp[i], l, l, n) || !tc_map_bf16_mn(&m.bmap[i], in.s[i], rows, l, n)) {
        *st = fail(JOLT_ERR_CUDA, "tensor map rejected");
        return cur;
      }
    m.bv.mode = VIEW_MN;             // Y from its [l][rows] parts, rows contiguous
    m.na = m.nb = 3;
    six_products(m);
    m.M = l; m.N = rows; m.KB = (l + 63) / 64;
    m.C = nullptr;
    m.c_sm = rows; m.c_sn = 1; m.c_sb = (int64_t)l * rows;       // Q^T parts [l][rows]
    for (int i = 0; i < 3; ++i) m.ps[i] = out.s[i];
    ck(gemm_tc(n, m, s));
    cur ^= 1;
  }
  return cur;
}

// CholeskyQR on the transposed layout: Y^T [n][l][rows] -> Q^T (same layout), passes as above.
float* cholqr_t(jolt_plan_s* p, int rows, float* bufA, float* bufB, int passes, int32_t* status, cudaStream_t s,
                jolt_status* st) {
  const int l = p->l, n = p->n_lt;
  float* src = bufA;
  float* dst = bufB;
  *st = JOLT_OK;
  auto ck = [&](cudaError_t e) {
    if (e != cudaSuccess && *st == JOLT_OK) *st = fail(JOLT_ERR_CUDA, "cholqr: %s", cudaGetErrorString(e));
  };
  for (int pass = 0; pass < passes; ++pass) {
    // W[i][j] = sum_t Y^T[i][t] Y^T[j][t]
    ck(gemm_simt(n, l, l, rows, opnd(src, EL_F32, I1((int64_t)rows * l), I1(rows), I1(1)),
                 opnd(src, EL_F32, I1((int64_t)rows * l), I1(rows), I1(1)),
                 outd(p->Wg, EL_F64, I1((int64_t)l * l), I1(l), I1(1)), 1.0, 0.0, s));
    const double shift =
        pass == 0 ? 11.0 * ((double)rows * l + (double)l * (l + 1)) * std::ldexp(1.0, -53) * l : 0.0;
    ck(chol_inv(n, l, p->Wg, (int64_t)l * l, p->Rinv, (int64_t)l * l, shift, status, s));
    // Q^T[j][t] = sum_i Rinv[i][j] Y^T[i][t]
    ck(gemm_simt(n, l, rows, l, opnd(p->Rinv, EL_F64, I1((int64_t)l * l), I1(1), I1(l)),
                 opnd(src, EL_F32, I1((int64_t)rows * l), I1(1), I1(rows)),
                 outd(dst, EL_F32, I1((int64_t)rows * l), I1(rows), I1(1)), 1.0, 0.0, s));
    std::swap(src, dst);
  }
  return src;
}

// Leading R eigenvectors of `batch` symmetric T x T float64 matrices A (overwritten) by the dense
// eigensolver, then two CholeskyQR passes in float64 (Q = Z R^-1 with R^T R = Z^T Z) so that the R
// columns are orthonormal to rounding. `out` receives [batch][T][R] (float32 or float64), `lam`
// (optional, float64 [batch][R]) the eigenvalues, descending. tri: tridiag_scratch_doubles(batch,
// T, R); Qx: batch T R, Gx and Rx: batch R^2 float64.
cudaError_t dense_top_eig(int batch, int T, int R, double* A, int64_t sA, double* tri, double* Qx, double* Gx,
                          double* Rx, void* out, ElemType out_t, double* lam, int32_t* status, cudaStream_t s) {
  double *Z = nullptr, *lz = nullptr;
  cudaError_t e = eig_top_dense(batch, T, R, A, sA, tri, &Z, &lz, s);
  if (e != cudaSuccess) return e;
  const int Rp = tridiag_rpad(R);
  const double* src = Z;
  int64_t ld = Rp;
  for (int pass = 0; pass < 2 && e == cudaSuccess; ++pass) {
    e = gemm_simt(batch, R, R, T, opnd(src, EL_F64, I1((int64_t)T * ld), I1(1), I1(ld)),
                  opnd(src, EL_F64, I1((int64_t)T * ld), I1(1), I1(ld)),
                  outd(Gx, EL_F64, I1((int64_t)R * R), I1(R), I1(1)), 1.0, 0.0, s);
    if (e == cudaSuccess) e = chol_inv(batch, R, Gx, (int64_t)R * R, Rx, (int64_t)R * R, 0.0, status, s);
    if (e == cudaSuccess)
      e = gemm_simt(batch, T, R, R, opnd(src, EL_F64, I1((int64_t)T * ld), I1(ld), I1(1)),
                    opnd(Rx, EL_F64, I1((int64_t)R * R), I1(1), I1(R)),
                    outd(pass == 0 ? (void*)Qx : out, pass == 0 ? EL_F64 : out_t, I1((int64_t)T * R), I1(R), I1(1)),
                    1.0, 0.0, s);
    src = Qx;
    ld = R;
  }
  if (e == cudaSuccess && lam)
    e = cudaMemcpy2DAsync(lam, sizeof(double) * R, lz, sizeof(double) * Rp, sizeof(double) * R, (size_t)batch,
                          cudaMemcpyDeviceToDevice, s);
  return e;
}

}  // namespace

// ============================================================================ API
extern "C" {

JOLT_API void jolt_config_default(jolt_config* c) {
  if (!c) return;
  c->encoder = JOLT_ENC_AUTO;
  c->oversample = 16;
  c->power_iters = 1;
  c->rank_step = 16;
  c->rt_max = 0;
  c->bits_mask = 0x1FFu;
  c->factors = 1;
  c->measured_b = 0;
  c->rotation = 0;
  c->split_kv_budget = 0;
  c->max_jacobi_sweeps = 30;
  c->eig_solver = JOLT_EIG_TRIDIAG;
}

JOLT_API const char* jolt_last_error(void) { return g_err.c_str(); }

JOLT_API jolt_status jolt_plan(const jolt_shape* shape, uint64_t byte_budget, int32_t num_groups,
                               const jolt_config* cfg_in, jolt_plan_t* out) {
  g_err.clear();
  if (!shape || !out) return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: null shape or out");
  *out = nullptr;
  jolt_config cfg;
  jolt_config_default(&cfg);
  if (cfg_in) cfg = *cfg_in;
  const jolt_shape& sh = *shape;
  if (sh.layers <= 0 || sh.heads <= 0 || sh.tokens <= 0 || sh.head_dim <= 0)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: non-positive dimension");
  if (sh.head_dim != kD)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: head_dim %d unsupported (supported: 128)", sh.head_dim);
  if (sh.layers > kMaxL) return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: at most %d layers", kMaxL);
  if (sh.dtype != JOLT_BF16 && sh.dtype != JOLT_F32) return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: dtype");
  if (num_groups <= 0 || num_groups > sh.layers || num_groups > kMaxGroups)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: num_groups must be in [1, min(layers, %d)]", kMaxGroups);
  if (cfg.rank_step <= 0 || kD % cfg.rank_step != 0)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: rank_step must divide %d", kD);
  if (cfg.oversample < 0 || cfg.power_iters < 0 || cfg.power_iters > 8 || cfg.max_jacobi_sweeps <= 0)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: bad sketch or solver option");
  if ((cfg.bits_mask & 0x1FFu) == 0 || (cfg.bits_mask & ~0x1FFu))
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: bits_mask must select widths in 0..8");
  if (cfg.rt_max < 0) return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: rt_max < 0");
  if (cfg.eig_solver != JOLT_EIG_TRIDIAG && cfg.eig_solver != JOLT_EIG_JACOBI)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: eig_solver must be TRIDIAG (0) or JACOBI (1)");
  if (cfg.factors != 0 && cfg.factors != 1) return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: factors must be 0 or 1");
  if (cfg.measured_b != 0 && cfg.measured_b != 1)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: measured_b must be 0 or 1");
  if (cfg.rotation != 0 && cfg.rotation != 1)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: rotation must be 0 (Haar) or 1 (randomized Hadamard)");
  if (byte_budget == 0) return fail(JOLT_ERR_INVALID_ARG, "jolt_plan: zero byte budget");

  jolt_plan_s* p = new (std::nothrow) jolt_plan_s();
  if (!p) return fail(JOLT_ERR_OOM, "jolt_plan: host allocation");
  p->shape = sh;
  p->cfg = cfg;
  p->budget = byte_budget;
  p->G = num_groups;
  p->step = cfg.rank_step;
  const int L = sh.layers, H = sh.heads, T = sh.tokens, D = sh.head_dim;
  const int kinds = sh.has_v ? 2 : 1;
  p->n_lt = L * kinds;
  for (int k = 0; k < kinds; ++k)
    for (int l = 0; l < L; ++l) p->lt_ids.push_back(2 * l + k);
  const int64_t per_lt = (int64_t)(byte_budget / (uint64_t)p->n_lt);
  int enc = cfg.encoder;
  if (enc == JOLT_ENC_AUTO) enc = T <= 1024 ? JOLT_ENC_EXACT : JOLT_ENC_SKETCH;
  // Largest token rank of the candidate grid: min(T, HD, budget per layer-tensor / (2T)) (a
  // larger token factor alone would exceed the layer-tensor's share of the budget), at most
  // kSketchRankCap for the randomized-SVD encoder, and at most rt_max when the caller sets it.
  int64_t cap = enc == JOLT_ENC_SKETCH ? kSketchRankCap : INT32_MAX;
  if (cfg.rt_max > 0) cap = std::min<int64_t>(cap, cfg.rt_max);
  if (cfg.factors == 0) cap = 0;   // residual only: the grid is the single point r_t = r_d = 0
  int64_t R = std::min<int64_t>({(int64_t)T, (int64_t)H * D, per_lt / (2 * (int64_t)T), cap});
  R -= R % p->step;
  p->R = (int)std::max<int64_t>(0, R);
  if (p->R > kMaxRank) {
    const int R0 = p->R;
    delete p;
    return fail(JOLT_ERR_UNSUPPORTED,
                "jolt_plan: the candidate grid reaches token rank %d; this library implements token ranks up to "
                "%d (set jolt_config.rt_max <= %d)",
                R0, kMaxRank, kMaxRank);
  }
  p->q_iters = cfg.power_iters;
  if (enc == JOLT_ENC_EXACT && T > kMaxN) {
    // The token Gram is too large for one CTA's Jacobi eigensolver: its leading eigenvectors
    // come from the dense float64 eigensolver (tridiagonalisation, bisection, inverse iteration)
    if (T > kExactMaxTokens) {
      delete p;
      return fail(JOLT_ERR_UNSUPPORTED,
                  "jolt_plan: the exact encoder forms the %d x %d token Gram; above %d tokens use the sketch encoder",
                  T, T, kExactMaxTokens);
    }
    p->exact_dense = p->R > 0;
  }
  p->encoder = enc;
  if (enc == JOLT_ENC_SKETCH) {
    int l = (int)std::min<int64_t>({(int64_t)p->R + cfg.oversample, (int64_t)T, (int64_t)H * D});
    if (l > kMaxN || (l & 1) || l < p->R || l <= 0) {
      delete p;
      return fail(JOLT_ERR_UNSUPPORTED, "jolt_plan: sketch width %d must be even, >= r_t max and <= %d", l, kMaxN);
    }
    p->l = l;
  } else {
    if (T & 1) {
      delete p;
      return fail(JOLT_ERR_UNSUPPORTED, "jolt_plan: exact path needs an even token count");
    }
  }
  p->nbits = 0;
  for (int b = 0; b <= 8; ++b)
    if (cfg.bits_mask & (1u << b)) p->bits[p->nbits++] = b;
  p->kappa = kappa_of(D);
  for (int i = 0; i < p->nbits; ++i)
    p->phi[i] = p->bits[i] == 0 ? 1.0 : p->kappa / (3.0 * std::pow(4.0, p->bits[i]));
  p->ngrid = 1 + (p->R / p->step) * (D / p->step);
  {
    // dual candidates c = bit index * ngrid + grid index, ordered by the tie-break key
    const int ncand = p->nbits * p->ngrid, nJ = D / p->step;
    std::vector<std::array<int64_t, 4>> key(ncand);
    for (int c = 0; c < ncand; ++c) {
      const int gi = c % p->ngrid, b = p->bits[c / p->ngrid];
      const int rt = gi == 0 ? 0 : ((gi - 1) / nJ + 1) * p->step, rd = gi == 0 ? 0 : ((gi - 1) % nJ + 1) * p->step;
      key[c] = {lt_bytes_h(H, T, D, rt, rd, b), b, rt, rd};
    }
    p->cand_order.resize(ncand);
    for (int c = 0; c < ncand; ++c) p->cand_order[c] = c;
    std::sort(p->cand_order.begin(), p->cand_order.end(), [&](int x, int y) { return key[x] < key[y]; });
  }
  if (sh.has_v && cfg.split_kv_budget) {
    p->pool_budget[0] = (int64_t)(byte_budget / 2);
    p->pool_budget[1] = (int64_t)byte_budget - p->pool_budget[0];
  } else {
    p->pool_budget[0] = (int64_t)byte_budget;
  }
  // feasibility: the cheapest candidate of every unit must fit its pool
  {
    int64_t minb_lt = INT64_MAX;
    for (int bi = 0; bi < p->nbits; ++bi) {
      const int b = p->bits[bi];
      minb_lt = std::min(minb_lt, lt_bytes_h(H, T, D, 0, 0, b));
      if (p->R >= p->step) minb_lt = std::min(minb_lt, lt_bytes_h(H, T, D, p->step, p->step, b));
    }
    const int npools = (sh.has_v && cfg.split_kv_budget) ? 2 : 1;
    const int64_t per_pool_lts = npools == 2 ? L : (int64_t)p->n_lt;
    if (minb_lt * per_pool_lts > p->pool_budget[0]) {
      delete p;
      return fail(JOLT_ERR_BUDGET_INFEASIBLE, "jolt_plan: minimum %lld bytes exceed the budget",
                  (long long)(minb_lt * per_pool_lts));
    }
  }
  // tensor-core path: bf16 inputs whose token stride is a multiple of 16 bytes (TMA rule), and
  // whose contractions over the tokens split into float32 chunks of at most 2048 tokens (whole
  // 64-token blocks); other token counts take the SIMT kernels, which accumulate in float64
  p->use_tc = sh.dtype == JOLT_BF16 && (T % 8) == 0 && (T <= 2048 || k_chunks(T) > 1) &&
              T / gram_chunks(T) <= 2048;
  // workspace
  const int64_t n = p->n_lt, HD = (int64_t)H * D, Rm = std::max(p->R, 1), l = std::max(p->l, 2);
  auto layout = [&](char* base, bool assign) -> size_t {
    char* cur = base;
    auto take = [&](auto*& ptr, size_t count) {
      using T_ = std::remove_reference_t<decltype(*ptr)>;
      T_* v = carve<T_>(cur, count);
      if (assign) ptr = v;
    };
    take(p->xx, n);
    take(p->xx_part, n * 64);
    take(p->CD, n * D * D);
    take(p->UD32, n * D * D);
    take(p->UDf, n * D * D);
    take(p->lamD, n * D);
    take(p->UDb, n * D * D);
    take(p->UT32, n * T * Rm);
    take(p->UTf, n * T * Rm);
    take(p->UTb, n * T * Rm);
    take(p->P, n * H * Rm * D);
    take(p->Gmax, n * H * Rm * D);
    take(p->E, 2 * (int64_t)L * p->ngrid);
    take(p->unit_err, 2 * (int64_t)p->G * p->nbits * p->ngrid);
    take(p->Nbuf, n * H * D * (Rm + 4));
    take(p->PiT, (int64_t)D * 132);
    take(p->Pbuf, n * D * D);
    if (cfg.measured_b) {
      take(p->meas_part, n * H * ((T + 255) / 256) * 9);
      take(p->meas_lt, n * 9);
    }
    take(p->Gpi, (int64_t)D * D);
    take(p->Pi32, (int64_t)D * D);
    take(p->Pib, (int64_t)D * D);
    if (p->use_tc) {
      take(p->Cpart, n * H * D * D * k_chunks(T));   // per-head (and per K chunk) partials
      if (p->encoder == JOLT_ENC_SKETCH) {
        for (int i = 0; i < 3; ++i) take(p->QTp[i], n * l * std::max<int64_t>(T, HD));
        for (int i = 0; i < 3; ++i) take(p->QTp2[i], n * l * std::max<int64_t>(T, HD));
        for (int i = 0; i < 3; ++i) take(p->RTp[i], n * l * l);
        take(p->Wf, n * l * l);
        take(p->Wpart, n * 16 * l * l);
      }
      take(p->UDt, n * D * D);
      for (int i = 0; i < 3; ++i) take(p->Pp[i], n * H * Rm * D);
    }
    if (p->encoder == JOLT_ENC_SKETCH) {
      take(p->Om, n * HD * l);
      take(p->Y, n * T * l);
      take(p->Y2, n * T * l);
      take(p->Z, n * HD * l);
      take(p->Z2, n * HD * l);
      take(p->Wg, n * l * l);
      take(p->Rinv, n * l * l);
      take(p->Bm, n * l * HD);
      take(p->BB, n * l * l);
      take(p->Wv, n * l * l);
      take(p->lamB, n * l);
    } else {
      take(p->CT, n * T * T);
      if (p->exact_dense && p->use_tc) take(p->CTpart, n * H * T * T);
      if (p->exact_dense) {
        take(p->tri, tridiag_scratch_doubles((int)n, T, (int)Rm));
        take(p->Qx, n * T * Rm);
        take(p->Gx, n * Rm * Rm);
        take(p->Rx, n * Rm * Rm);
      } else {
        take(p->VT, n * T * T);
        take(p->lamT, n * T);
      }
    }
    return (size_t)(cur - base) + 256;
  };
  p->ws_bytes = layout(nullptr, false);
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = dev_malloc(&p->ws, p->ws_bytes);
  if (e == cudaSuccess) e = dev_malloc(&p->d_lt_ids, sizeof(int32_t) * p->lt_ids.size());
  if (e == cudaSuccess) e = dev_malloc(&p->d_cand_order, sizeof(int32_t) * p->cand_order.size());
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_cand_order, p->cand_order.data(), sizeof(int32_t) * p->cand_order.size(),
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_lt_ids, p->lt_ids.data(), sizeof(int32_t) * p->lt_ids.size(), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    jolt_status st = fail(e == cudaErrorMemoryAllocation ? JOLT_ERR_OOM : JOLT_ERR_CUDA,
                          "jolt_plan: workspace of %zu bytes: %s", p->ws_bytes, cudaGetErrorString(e));
    if (p->ws) cudaFree(p->ws);
    if (p->d_lt_ids) cudaFree(p->d_lt_ids);
    if (p->d_cand_order) cudaFree(p->d_cand_order);
    delete p;
    return st;
  }
  layout(reinterpret_cast<char*>(align_up(reinterpret_cast<size_t>(p->ws), 256)), true);
  *out = p;
  return JOLT_OK;
}

JOLT_API jolt_status jolt_plan_info(jolt_plan_t p, int32_t* rt_max, int32_t* sketch_l, int32_t* encoder,
                                    uint64_t* workspace_bytes) {
  if (!p) return fail(JOLT_ERR_INVALID_ARG, "jolt_plan_info: null plan");
  if (rt_max) *rt_max = p->R;
  if (sketch_l) *sketch_l = p->encoder == JOLT_ENC_SKETCH ? p->l : 0;
  if (encoder) *encoder = p->encoder;
  if (workspace_bytes) *workspace_bytes = p->ws_bytes;
  return JOLT_OK;
}

static jolt_status make_stream(jolt_plan_s* p, uint64_t seed, cudaStream_t cs, jolt_stream_s** out) {
  jolt_stream_s* st = new (std::nothrow) jolt_stream_s();
  if (!st) return fail(JOLT_ERR_OOM, "stream: host allocation");
  const jolt_shape& sh = p->shape;
  st->L = sh.layers; st->H = sh.heads; st->T = sh.tokens; st->D = sh.head_dim;
  st->has_v = sh.has_v ? 1 : 0; st->G = p->G; st->encoder = p->encoder; st->step = p->step;
  st->rotation = p->cfg.rotation;
  st->R = p->R; st->split = (sh.has_v && p->cfg.split_kv_budget) ? 1 : 0; st->dtype = sh.dtype;
  st->seed = seed; st->cs = cs; st->plan = p; st->n_lt = p->n_lt;
  st->body_cap = align_up((size_t)p->budget + (size_t)JOLT_NUM_PARTS * kAlign * p->n_lt + kAlign, kAlign);
  cudaError_t e = pool_malloc(&st->d_body, st->body_cap, cs);
  if (e == cudaSuccess) e = pool_malloc(&st->d_meta, sizeof(StreamMeta), cs);
  if (e == cudaSuccess) e = pool_malloc(&st->d_Pi, sizeof(float) * kD * kD, cs);
  if (e == cudaSuccess) e = pool_malloc(&st->d_lt_ids, sizeof(int32_t) * p->n_lt, cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->d_meta, 0, sizeof(StreamMeta), cs);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->d_lt_ids, p->d_lt_ids, sizeof(int32_t) * p->n_lt, cudaMemcpyDeviceToDevice, cs);
  if (e != cudaSuccess) {
    jolt_stream_destroy(st);
    return fail(e == cudaErrorMemoryAllocation ? JOLT_ERR_OOM : JOLT_ERR_CUDA, "stream allocation: %s",
                cudaGetErrorString(e));
  }
  *out = st;
  return JOLT_OK;
}

static jolt_status analyse(jolt_plan_s* p, jolt_stream_s* st, const void* X[2], uint64_t seed, cudaStream_t s) {
  const jolt_shape& sh = p->shape;
  const int L = sh.layers, H = sh.heads, T = sh.tokens, D = sh.head_dim, R = p->R;
  const int kinds = sh.has_v ? 2 : 1;
  const int n = p->n_lt;
  const int64_t HD = (int64_t)H * D, HTD = (int64_t)H * T * D;
  const ElemType xt = sh.dtype == JOLT_BF16 ? EL_BF16 : EL_F32;
  int32_t* status = &st->d_meta->status;
  {
    PROF("check_norms", s);
    for (int k = 0; k < kinds; ++k) {
      CK(sumsq_batched(L, HTD, X[k], xt, HTD, p->xx + (int64_t)k * L, p->xx_part + (int64_t)k * L * 64,
                       status, s));
    }
  }
  // residual only (factors = 0): the grid is the single point r_t = r_d = 0, whose energy is
  // ||X||^2; no factor, core or sketch is needed
  if (p->cfg.factors == 0) {
    PROF("energy_table", s);
    TableArgs ta;
    ta.n_lt = n; ta.H = H; ta.R = 0; ta.D = D; ta.step = p->step; ta.lt_ids = p->d_lt_ids;
    ta.Gmax = p->Gmax; ta.xx = p->xx; ta.E = p->E; ta.ngrid = p->ngrid;
    CK(energy_table(ta, s));
    return JOLT_OK;
  }
  // Tensor maps of X [L][H][T][D] per kind: K-major tiles (rows = tokens, K = features) for
  // the contractions over the features, MN-major tiles (rows = features, K = tokens) for those
  // over the tokens, so X is read in place by both.
  CUtensorMap mx[2], mxm[2];
  if (p->use_tc) {
    for (int k = 0; k < kinds; ++k)
      if (!map_x(&mx[k], X[k], L, H, T, D) || !tc_map_bf16_x_mn(&mxm[k], X[k], L, H, T, D))
        return fail(JOLT_ERR_CUDA, "tensor map of X rejected");
    PROF("feature_gram", s);
    // per-head partials C_D[lt][h] = X_h^T X_h on the tensor cores (one operand tile serves A
    // and B), then a float64 sum over heads
    const int kc = k_chunks(T);
    TcGemmParams g;
    g.amap[0] = mxm[0];
    g.amap[1] = mxm[kinds - 1];
    g.av.mode = VIEW_MN_XHEAD;
    g.av.H = H;
    g.av.D = D;
    g.av.ksplit = kinds > 1 ? L * H : 0;   // (layer, head) batches of V after those of K
    g.b_same = 1;
    g.av.nch = kc;
    g.av.ckb = T / kc / 64;
    g.M = D; g.N = D; g.KB = kc > 1 ? T / kc / 64 : (T + 63) / 64;
    g.C = p->Cpart; g.c_sm = D; g.c_sn = 1; g.c_sb = (int64_t)D * D;
    g.status = status;
    CK(gemm_tc(n * H * kc, g, s));
    CK(sum_heads(n, H * kc, (int64_t)D * D, p->Cpart, nullptr, p->CD, s));
  } else {
    PROF("feature_gram", s);
    // C_D = sum over rows r = (h, t) of X[r, :]^T X[r, :]
    for (int k = 0; k < kinds; ++k)
      CK(gemm_simt(L, D, D, H * T, opnd(X[k], xt, I1(HTD), I1(1), I1(D)), opnd(X[k], xt, I1(HTD), I1(1), I1(D)),
                   outd(p->CD + (int64_t)k * L * D * D, EL_F64, I1((int64_t)D * D), I1(D), I1(1)), 1.0, 0.0, s));
  }
  // The feature eigenproblems are solved together with the token ones (one launch, both batches
  // side by side on the SMs); U_D is first needed by the core projection.
  auto feature_sign_round = [&]() -> jolt_status {
    PROF("sign_round", s);
    CK(sign_fix(n, D, D, p->UD32, D, (int64_t)D * D, nullptr, 0, 0, 0, s));
    CK(round_bf16((int64_t)n * D * D, p->UD32, p->UDb, p->UDf, s));
    return JOLT_OK;
  };
  auto eig_feature_and = [&](int n1, const double* C1, float* V1, float* lam1) -> jolt_status {
    PROF("small_eig", s);
    if (p->cfg.eig_solver == JOLT_EIG_JACOBI)
      CK(eig_psd2(n, D, p->CD, (int64_t)D * D, p->UD32, (int64_t)D * D, p->lamD, D, n1 > 0 ? n : 0, n1, C1,
                  (int64_t)n1 * n1, V1, (int64_t)n1 * n1, lam1, n1, p->cfg.max_jacobi_sweeps, status, s));
    else
      CK(eig_small2(n, D, p->CD, (int64_t)D * D, p->UD32, (int64_t)D * D, p->lamD, D, n1 > 0 ? n : 0, n1, C1,
                    (int64_t)n1 * n1, V1, (int64_t)n1 * n1, lam1, n1, status, s));
    return JOLT_OK;
  };
  if (R == 0) {
    jolt_status r = eig_feature_and(0, nullptr, nullptr, nullptr);
    if (r != JOLT_OK) return r;
    r = feature_sign_round();
    if (r != JOLT_OK) return r;
  }
  if (R > 0) {
    if (p->encoder == JOLT_ENC_SKETCH && p->use_tc) {
      const int l = p->l;
      p->q_t = true;
      {
        PROF("sketch_omega", s);
        if (!(p->om_valid && p->om_seed == seed)) {
          std::vector<int32_t> ids = p->lt_ids;
          CK(sketch_omega(seed, ids.data(), n, HD, l, p->Om, true, s));   // Omega^T [l][HD]
          p->om_valid = true;
          p->om_seed = seed;
        }
      }
      jolt_status r = JOLT_OK;
      // two part sets: every basis lives as bf16 parts, written by the epilogue that makes it
      PartSet sets[2];
      for (int i = 0; i < 3; ++i) {
        sets[0].s[i] = p->QTp[i];
        sets[1].s[i] = p->QTp2[i];
      }
      auto tc_params = [&]() {
        TcGemmParams g;
        g.status = status;
        return g;
      };
      // Y^T = (A Omega)^T or (A Q')^T: rows t, K = (h, d); parts of Y^T [l][T] and Y [T][l]
      auto y_pass = [&](const __nv_bfloat16* const* bparts, int nparts, const PartSet& out) -> jolt_status {
        for (int k = 0; k < kinds; ++k) {
          TcGemmParams g = tc_params();
          g.amap[0] = mx[k];
          g.av.mode = VIEW_X_TOKENROWS;
          g.av.D = D;
          for (int i = 0; i < nparts; ++i)
            if (!map_rows(&g.bmap[i], bparts[i] + (int64_t)k * L * l * HD, HD, l, L))
              return fail(JOLT_ERR_CUDA, "tensor map rejected");
          g.na = 1; g.nb = nparts;
          g.M = T; g.N = l; g.KB = (int)(HD / 64);
          g.C = nullptr;
          g.c_sm = 1; g.c_sn = T; g.c_sb = (int64_t)l * T;
          for (int i = 0; i < 3; ++i) g.ps[i] = out.s[i] + (int64_t)k * L * l * T;
          CK(gemm_tc(L, g, s));
        }
        return JOLT_OK;
      };
      int cur = 0;
      {
        PROF("sketch_gemm", s);
        const __nv_bfloat16* om[1] = {p->Om};
        r = y_pass(om, 1, sets[cur]);
        if (r != JOLT_OK) return r;
      }
      const int q = p->q_iters;
      {
        PROF("cholqr", s);
        cur = cholqr_tc(p, T, sets, cur, q > 0 ? 1 : 3, status, s, &r);
        if (r != JOLT_OK) return r;
      }
      for (int it = 0; it < q; ++it) {
        {
          PROF("sketch_gemm", s);
          // Z^T = (A^T Q)^T: rows (h, d), K = t (X read MN-major); parts of Z^T [l][HD]
          const int kc = k_chunks(T);
          TcGemmParams g = tc_params();
          g.amap[0] = mxm[0];
          g.amap[1] = mxm[kinds - 1];
          g.av.mode = VIEW_MN_XFEAT;
          g.av.D = D;
          g.av.ksplit = kinds > 1 ? L : 0;
          for (int i = 0; i < 2; ++i)
            if (!map_rows(&g.bmap[i], sets[cur].s[i], T, l, n)) return fail(JOLT_ERR_CUDA, "tensor map rejected");
          g.na = 1; g.nb = 2;
          g.M = (int)HD; g.N = l; g.KB = (T + 63) / 64;
          g.c_sm = 1; g.c_sn = HD; g.c_sb = (int64_t)l * HD;
          if (kc == 1) {
            g.C = nullptr;
            for (int i = 0; i < 3; ++i) g.ps[i] = sets[cur ^ 1].s[i];
            CK(gemm_tc(n, g, s));
          } else {
            // long K: float32 partials per chunk of tokens, float64 sum, then the parts
            g.av.nch = g.bv.nch = kc;
            g.av.ckb = g.bv.ckb = T / kc / 64;
            g.KB = T / kc / 64;
            g.C = p->Cpart;
            CK(gemm_tc(n * kc, g, s));
            CK(sum_heads(n, kc, (int64_t)l * HD, p->Cpart, p->Z, nullptr, s));
            CK(split_dual(n, l, (int)HD, p->Z, false, sets[cur ^ 1].s, nullptr, s));
          }
          cur ^= 1;
        }
        {
          PROF("cholqr", s);
          cur = cholqr_tc(p, (int)HD, sets, cur, 1, status, s, &r);
          if (r != JOLT_OK) return r;
        }
        {
          PROF("sketch_gemm", s);
          const __nv_bfloat16* qp[2] = {sets[cur].s[0], sets[cur].s[1]};
          r = y_pass(qp, 2, sets[cur ^ 1]);
          if (r != JOLT_OK) return r;
          cur ^= 1;
        }
        {
          PROF("cholqr", s);
          cur = cholqr_tc(p, T, sets, cur, it + 1 == q ? 3 : 1, status, s, &r);
          if (r != JOLT_OK) return r;
        }
      }
      {
        PROF("sketch_gemm", s);
        // B = Q^T A (l x HD): rows j, K = t; Q^T in three bf16 parts for float32 accuracy, X
        // read MN-major. B's bf16 parts [l][HD] (for B B^T, and MN-major for the per-head core)
        // go to the part set that does not hold Q.
        const PartSet& bs = sets[cur ^ 1];
        const int kc = k_chunks(T);
        TcGemmParams g = tc_params();
        for (int i = 0; i < 3; ++i)
          if (!map_rows(&g.amap[i], sets[cur].s[i], T, l, n)) return fail(JOLT_ERR_CUDA, "tensor map rejected");
        g.bmap[0] = mxm[0];
        g.bmap[1] = mxm[kinds - 1];
        g.bv.mode = VIEW_MN_XFEAT;
        g.bv.D = D;
        g.bv.ksplit = kinds > 1 ? L : 0;
        g.na = 3; g.nb = 1;
        g.M = l; g.N = (int)HD; g.KB = (T + 63) / 64;
        g.c_sm = HD; g.c_sn = 1; g.c_sb = (int64_t)l * HD;
        if (kc == 1) {
          g.C = p->Bm;
          for (int i = 0; i < 3; ++i) g.ps[i] = bs.s[i];
          CK(gemm_tc(n, g, s));
        } else {
          // long K: float32 partials per chunk of tokens, summed in float64, then the parts
          g.av.nch = g.bv.nch = kc;
          g.av.ckb = g.bv.ckb = T / kc / 64;
          g.KB = T / kc / 64;
          g.C = p->Cpart;
          CK(gemm_tc(n * kc, g, s));
          CK(sum_heads(n, kc, (int64_t)l * HD, p->Cpart, p->Bm, nullptr, s));
          CK(split_dual(n, l, (int)HD, p->Bm, false, bs.s, nullptr, s));
        }
      }
      p->Qfinal = nullptr;
      p->qset = cur;
    }
    if (p->encoder == JOLT_ENC_SKETCH && !p->use_tc) {
      const int l = p->l;
      p->q_t = false;
      {
        PROF("sketch_omega", s);
        if (!(p->om_valid && p->om_seed == seed)) {
          std::vector<int32_t> ids = p->lt_ids;
          CK(sketch_omega(seed, ids.data(), n, HD, l, p->Om, false, s));
          p->om_valid = true;
          p->om_seed = seed;
        }
      }
      jolt_status r = JOLT_OK;
      {
        PROF("sketch_gemm", s);
        // Y0 = A Omega, A[t, h*D + d] = X[h][t][d]
        for (int k = 0; k < kinds; ++k)
          CK(gemm_simt(L, T, l, (int)HD, opnd(X[k], xt, I1(HTD), I1(D), I2(D, 1, (int64_t)T * D)),
                       opnd(p->Om + (int64_t)k * L * HD * l, EL_BF16, I1(HD * l), I1(1), I1(l)),
                       outd(p->Y + (int64_t)k * L * T * l, EL_F32, I1((int64_t)T * l), I1(l), I1(1)), 1.0, 0.0, s));
      }
      const int q = p->q_iters;
      float* Q;
      {
        PROF("cholqr", s);
        Q = cholqr(p, T, p->Y, p->Y2, q > 0 ? 1 : 2, status, s, &r);
        if (r != JOLT_OK) return r;
      }
      for (int it = 0; it < q; ++it) {
        {
          PROF("sketch_gemm", s);
          // Z = A^T Q  (HD x l)
          for (int k = 0; k < kinds; ++k)
            CK(gemm_simt(L, (int)HD, l, T, opnd(X[k], xt, I1(HTD), I2(D, 1, (int64_t)T * D), I1(D)),
                         opnd(Q + (int64_t)k * L * T * l, EL_F32, I1((int64_t)T * l), I1(1), I1(l)),
                         outd(p->Z + (int64_t)k * L * HD * l, EL_F32, I1(HD * l), I1(l), I1(1)), 1.0, 0.0, s));
        }
        float* Qz;
        {
          PROF("cholqr", s);
          Qz = cholqr(p, (int)HD, p->Z, p->Z2, 1, status, s, &r);
          if (r != JOLT_OK) return r;
        }
        float* Ydst = (Q == p->Y) ? p->Y2 : p->Y;
        float* Yalt = (Q == p->Y) ? p->Y : p->Y2;
        {
          PROF("sketch_gemm", s);
          // Y = A Q'
          for (int k = 0; k < kinds; ++k)
            CK(gemm_simt(L, T, l, (int)HD, opnd(X[k], xt, I1(HTD), I1(D), I2(D, 1, (int64_t)T * D)),
                         opnd(Qz + (int64_t)k * L * HD * l, EL_F32, I1(HD * l), I1(1), I1(l)),
                         outd(Ydst + (int64_t)k * L * T * l, EL_F32, I1((int64_t)T * l), I1(l), I1(1)), 1.0, 0.0, s));
        }
        {
          PROF("cholqr", s);
          Q = cholqr(p, T, Ydst, Yalt, it + 1 == q ? 2 : 1, status, s, &r);
          if (r != JOLT_OK) return r;
        }
      }
      {
        PROF("sketch_gemm", s);
        // B = Q^T A (l x HD)
        for (int k = 0; k < kinds; ++k)
          CK(gemm_simt(L, l, (int)HD, T, opnd(Q + (int64_t)k * L * T * l, EL_F32, I1((int64_t)T * l), I1(1), I1(l)),
                       opnd(X[k], xt, I1(HTD), I2(D, 1, (int64_t)T * D), I1(D)),
                       outd(p->Bm + (int64_t)k * L * l * HD, EL_F32, I1(l * HD), I1(HD), I1(1)), 1.0, 0.0, s));
      }
      p->Qfinal = Q;
    }
    if (p->encoder == JOLT_ENC_SKETCH && p->use_tc) {
      const int l = p->l;
      const int nch = (int)(HD / 128);
      {
        PROF("small_gemm", s);
        // B B^T: float32 partial Grams over 128-wide chunks of the (head, feature) axis on the
        // tensor cores (B in three bf16 parts), summed over the chunks in float64
        __nv_bfloat16* const* bsame = p->qset ? p->QTp : p->QTp2;     // B parts [l][HD] (set qset ^ 1)
        TcGemmParams g;
        g.status = status;
        for (int i = 0; i < 3; ++i)
          if (!map_kchunk(&g.amap[i], bsame[i], l, HD, 128, n)) return fail(JOLT_ERR_CUDA, "tensor map rejected");
        g.av.mode = VIEW_ROWS_K_HEAD;      // (K, rows, chunk, i)
        g.av.H = nch;
        g.na = g.nb = 3;
        g.b_same = 1;
        six_products(g);
        g.M = l; g.N = l; g.KB = 2;
        g.C = p->Cpart; g.c_sm = l; g.c_sn = 1; g.c_sb = (int64_t)l * l;
        CK(gemm_tc(n * nch, g, s));
        CK(sum_heads(n, nch, (int64_t)l * l, p->Cpart, nullptr, p->BB, s));
      }
      {
        jolt_status r = eig_feature_and(l, p->BB, p->Wv, p->lamB);
        if (r != JOLT_OK) return r;
        r = feature_sign_round();
        if (r != JOLT_OK) return r;
      }
      {
        PROF("small_gemm", s);
        // U_T = Q W[:, :R]: rows t, K = the sketch index; Q from its parts [l][T] (MN-major),
        // W^T parts
        CK(split_dual(n, l, l, p->Wv, false, nullptr, p->RTp, s));
        __nv_bfloat16* const* qs = p->qset ? p->QTp2 : p->QTp;
        TcGemmParams g;
        g.status = status;
        for (int i = 0; i < 3; ++i)
          if (!tc_map_bf16_mn(&g.amap[i], qs[i], T, l, n) || !map_rows(&g.bmap[i], p->RTp[i], l, l, n))
            return fail(JOLT_ERR_CUDA, "tensor map rejected");
        g.av.mode = VIEW_MN;
        g.na = g.nb = 3;
        six_products(g);
        g.M = T; g.N = R; g.KB = (l + 63) / 64;
        g.C = p->UT32; g.c_sm = R; g.c_sn = 1; g.c_sb = (int64_t)T * R;
        CK(gemm_tc(n, g, s));
      }
      {
        PROF("sign_round", s);
        CK(sign_fix(n, T, R, p->UT32, R, (int64_t)T * R, p->Wv, l, l, (int64_t)l * l, s));
        CK(round_bf16((int64_t)n * T * R, p->UT32, p->UTb, p->UTf, s));
      }
      {
        PROF("core", s);
        // P[h] = W_R^T B_h (R x D): W^T parts (signs fixed), head h's columns of the B parts
        // [l][HD] (set qset ^ 1), MN-major
        CK(split_dual(n, l, l, p->Wv, false, nullptr, p->RTp, s));
        __nv_bfloat16* const* bsp = p->qset ? p->QTp : p->QTp2;
        TcGemmParams g;
        g.status = status;
        for (int i = 0; i < 3; ++i)
          if (!map_rows(&g.amap[i], p->RTp[i], l, l, n) || !tc_map_bf16_mn(&g.bmap[i], bsp[i], HD, l, n))
            return fail(JOLT_ERR_CUDA, "tensor map rejected");
        g.av.H = H;                       // W^T shared by the heads of a layer-tensor
        g.bv.mode = VIEW_MN;
        g.bv.H = H;
        g.bv.D = D;
        g.na = g.nb = 3;
        six_products(g);
        g.M = R; g.N = D; g.KB = (l + 63) / 64;
        g.C = p->P; g.c_sm = D; g.c_sn = 1; g.c_sb = (int64_t)R * D;
        CK(gemm_tc(n * H, g, s));
      }
    } else if (p->encoder == JOLT_ENC_SKETCH) {
      const int l = p->l;
      {
        PROF("small_gemm", s);
        // B B^T
        CK(gemm_simt(n, l, l, (int)HD, opnd(p->Bm, EL_F32, I1(l * HD), I1(HD), I1(1)),
                     opnd(p->Bm, EL_F32, I1(l * HD), I1(HD), I1(1)),
                     outd(p->BB, EL_F64, I1((int64_t)l * l), I1(l), I1(1)), 1.0, 0.0, s));
      }
      {
        jolt_status r = eig_feature_and(l, p->BB, p->Wv, p->lamB);
        if (r != JOLT_OK) return r;
        r = feature_sign_round();
        if (r != JOLT_OK) return r;
      }
      {
        PROF("small_gemm", s);
        // U_T = Q W[:, :R]
        CK(gemm_simt(n, T, R, l, opnd(p->Qfinal, EL_F32, I1((int64_t)T * l), p->q_t ? I1(1) : I1(l),
                                      p->q_t ? I1(T) : I1(1)),
                     opnd(p->Wv, EL_F32, I1((int64_t)l * l), I1(1), I1(l)),
                     outd(p->UT32, EL_F32, I1((int64_t)T * R), I1(R), I1(1)), 1.0, 0.0, s));
      }
      {
        PROF("sign_round", s);
        CK(sign_fix(n, T, R, p->UT32, R, (int64_t)T * R, p->Wv, l, l, (int64_t)l * l, s));
        CK(round_bf16((int64_t)n * T * R, p->UT32, p->UTb, p->UTf, s));
      }
      {
        PROF("core", s);
        // core: P[h] = W_R^T B_h (R x D); G_max[h] = P[h] U_D(rounded) below
        CK(gemm_simt(n * H, R, D, l, opnd(p->Wv, EL_F32, I2(H, 0, (int64_t)l * l), I1(1), I1(l)),
                     opnd(p->Bm, EL_F32, I2(H, D, l * HD), I1(1), I1(HD)),
                     outd(p->P, EL_F32, I1((int64_t)R * D), I1(D), I1(1)), 1.0, 0.0, s));
      }
    } else {
      if (p->use_tc && p->CTpart) {
        PROF("token_gram", s);
        // exact: C_T = sum_h X_h X_h^T. Per-head partials on the tensor cores (rows t, K = the
        // head's 128 features, one K chunk per head: the bf16 products are exact, the float32 sum
        // runs over 128 terms), summed over the heads in float64.
        for (int k = 0; k < kinds; ++k) {
          TcGemmParams g;
          g.status = status;
          g.amap[0] = mx[k];
          g.bmap[0] = mx[k];
          g.av.mode = g.bv.mode = VIEW_X_TOKENROWS;
          g.av.D = g.bv.D = D;
          g.av.nch = g.bv.nch = H;
          g.av.ckb = g.bv.ckb = D / 64;
          g.M = T; g.N = T; g.KB = D / 64;
          g.C = p->CTpart + (int64_t)k * L * H * T * T;
          g.c_sm = T; g.c_sn = 1; g.c_sb = (int64_t)T * T;
          CK(gemm_tc(L * H, g, s));
        }
        CK(sum_heads(n, H, (int64_t)T * T, p->CTpart, nullptr, p->CT, s));
      } else {
        PROF("token_gram", s);
        // exact: C_T = A A^T (T x T), all eigenvectors, keep the leading R
        for (int k = 0; k < kinds; ++k)
          CK(gemm_simt(L, T, T, (int)HD, opnd(X[k], xt, I1(HTD), I1(D), I2(D, 1, (int64_t)T * D)),
                       opnd(X[k], xt, I1(HTD), I1(D), I2(D, 1, (int64_t)T * D)),
                       outd(p->CT + (int64_t)k * L * T * T, EL_F64, I1((int64_t)T * T), I1(T), I1(1)), 1.0, 0.0, s));
      }
      if (!p->exact_dense) {
        jolt_status r = eig_feature_and(T, p->CT, p->VT, p->lamT);
        if (r != JOLT_OK) return r;
        r = feature_sign_round();
        if (r != JOLT_OK) return r;
        PROF("sign_round", s);
        CK(cudaMemcpy2DAsync(p->UT32, sizeof(float) * R, p->VT, sizeof(float) * T, sizeof(float) * R,
                             (size_t)n * T, cudaMemcpyDeviceToDevice, s));
      } else {
        jolt_status r = eig_feature_and(0, nullptr, nullptr, nullptr);
        if (r != JOLT_OK) return r;
        r = feature_sign_round();
        if (r != JOLT_OK) return r;
        PROF("token_eig", s);
        CK(dense_top_eig(n, T, R, p->CT, (int64_t)T * T, p->tri, p->Qx, p->Gx, p->Rx, p->UT32, EL_F32, nullptr,
                         status, s));
      }
      {
        PROF("sign_round", s);
        CK(sign_fix(n, T, R, p->UT32, R, (int64_t)T * R, nullptr, 0, 0, 0, s));
        CK(round_bf16((int64_t)n * T * R, p->UT32, p->UTb, p->UTf, s));
      }
      if (p->use_tc && p->CTpart && T <= 2048) {
        PROF("core", s);
        // P[h] = U_T(rounded)^T X_h (R x D) on the tensor cores: U_T is exact in bf16 (one part,
        // MN-major from its [T][R] layout, shared by the heads), X_h MN-major in place
        for (int k = 0; k < kinds; ++k) {
          TcGemmParams g;
          g.status = status;
          if (!tc_map_bf16_mn(&g.amap[0], p->UTb + (int64_t)k * L * T * R, R, T, L))
            return fail(JOLT_ERR_CUDA, "tensor map rejected");
          g.bmap[0] = mxm[k];
          g.av.mode = VIEW_MN;
          g.av.H = H;
          g.av.D = 0;
          g.bv.mode = VIEW_MN_XHEAD;
          g.bv.H = H;
          g.bv.D = D;
          g.M = R; g.N = D; g.KB = (T + 63) / 64;
          g.C = p->P + (int64_t)k * L * H * R * D;
          g.c_sm = D; g.c_sn = 1; g.c_sb = (int64_t)R * D;
          CK(gemm_tc(L * H, g, s));
        }
      } else {
        PROF("core", s);
        // P[h] = U_T(rounded)^T X_h  (R x D)
        for (int k = 0; k < kinds; ++k)
          CK(gemm_simt(L * H, R, D, T, opnd(p->UTf + (int64_t)k * L * T * R, EL_F32, I2(H, 0, (int64_t)T * R), I1(1), I1(R)),
                       opnd(X[k], xt, I1((int64_t)T * D), I1(1), I1(D)),
                       outd(p->P + (int64_t)k * L * H * R * D, EL_F32, I1((int64_t)R * D), I1(D), I1(1)), 1.0, 0.0, s));
      }
    }
    if (p->use_tc) {
      PROF("core", s);
      // G_max[h] = P[h] U_D: P in three bf16 parts, U_D (rounded, exact in bf16) transposed
      __nv_bfloat16* udt[3] = {p->UDt, nullptr, nullptr};
      __nv_bfloat16* const* pp = p->Pp;
      CK(split_dual(n, D, D, p->UDf, false, nullptr, udt, s));
      CK(split_bf16((int64_t)n * H * R * D, p->P, pp[0], pp[1], pp[2], s));
      TcGemmParams g;
      g.status = status;
      for (int i = 0; i < 3; ++i)
        if (!map_rows(&g.amap[i], pp[i], D, R, (int64_t)n * H)) return fail(JOLT_ERR_CUDA, "tensor map rejected");
      if (!map_rows(&g.bmap[0], p->UDt, D, D, n)) return fail(JOLT_ERR_CUDA, "tensor map rejected");
      g.bv.H = H;                         // U_D shared by the heads of a layer-tensor
      g.na = 3; g.nb = 1;
      g.M = R; g.N = D; g.KB = (D + 63) / 64;
      g.C = p->Gmax; g.c_sm = D; g.c_sn = 1; g.c_sb = (int64_t)R * D;
      CK(gemm_tc(n * H, g, s));
    } else {
      PROF("core", s);
      CK(gemm_simt(n * H, R, D, D, opnd(p->P, EL_F32, I1((int64_t)R * D), I1(D), I1(1)),
                   opnd(p->UDf, EL_F32, I2(H, 0, (int64_t)D * D), I1(1), I1(D)),
                   outd(p->Gmax, EL_F32, I1((int64_t)R * D), I1(D), I1(1)), 1.0, 0.0, s));
    }
  }
  {
    PROF("energy_table", s);
    TableArgs ta;
    ta.n_lt = n; ta.H = H; ta.R = R; ta.D = D; ta.step = p->step; ta.lt_ids = p->d_lt_ids;
    ta.Gmax = p->Gmax; ta.xx = p->xx; ta.E = p->E; ta.ngrid = p->ngrid;
    CK(energy_table(ta, s));
  }
  return JOLT_OK;
}

JOLT_API jolt_status jolt_encode(jolt_plan_t p, const void* K, const void* V, uint64_t seed, void* cuda_stream,
                                 jolt_stream_t* out) {
  g_err.clear();
  if (!p || !K || !out) return fail(JOLT_ERR_INVALID_ARG, "jolt_encode: null plan, K or out");
  if (p->shape.has_v && !V) return fail(JOLT_ERR_INVALID_ARG, "jolt_encode: the plan has V but V is null");
  *out = nullptr;
  cudaStream_t s = (cudaStream_t)cuda_stream;
  CK(cudaSetDevice(p->device));
  jolt_stream_s* st = nullptr;
  jolt_status r = make_stream(p, seed, s, &st);
  if (r != JOLT_OK) return r;
  const jolt_shape& sh = p->shape;
  const int D = sh.head_dim;
  auto bail = [&](jolt_status x) { jolt_stream_destroy(st); return x; };
  // rotation Pi for this seed (cached in the plan), copied into the stream for decode
  if (!(p->pi_valid && p->pi_seed == seed)) {
    PROF("rotation", s);
    cudaError_t e;
    if (p->cfg.rotation == 1) {
      e = hadamard_pi(seed, D, p->Pi32, p->Pib, s);
    } else {
      e = gauss_f64(seed, 1, (int64_t)D * D, p->Gpi, s);
      if (e == cudaSuccess) e = haar_from_gauss(p->Gpi, D, p->Pi32, p->Pib, s);
    }
    if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "rotation: %s", cudaGetErrorString(e)));
    p->pi_valid = true;
    p->pi_seed = seed;
  }
  cudaError_t e = cudaMemcpyAsync(st->d_Pi, p->Pi32, sizeof(float) * D * D, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "copy Pi: %s", cudaGetErrorString(e)));
  const void* X[2] = {K, V};
  r = analyse(p, st, X, seed, s);
  if (r != JOLT_OK) return bail(r);
  DualArgs da;
  da.L = sh.layers; da.H = sh.heads; da.T = sh.tokens; da.D = D; da.G = p->G; da.has_v = sh.has_v ? 1 : 0;
  da.step = p->step; da.R = p->R; da.split = st->split; da.nbits = p->nbits;
  for (int i = 0; i < 9; ++i) { da.bits[i] = p->bits[i]; da.phi[i] = p->phi[i]; }
  da.budget_pool[0] = p->pool_budget[0]; da.budget_pool[1] = p->pool_budget[1];
  da.ngrid = p->ngrid; da.E = p->E; da.unit_err = p->unit_err; da.meta = st->d_meta;
  da.cand_order = p->d_cand_order;
  {
    PROF("dual", s);
    e = dual_allocate(da, s);
  }
  if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "dual: %s", cudaGetErrorString(e)));
  PackArgs pa;
  pa.n_lt = p->n_lt; pa.H = sh.heads; pa.T = sh.tokens; pa.D = D; pa.R = std::max(p->R, 1);
  pa.lt_ids = p->d_lt_ids; pa.UT = p->UTb; pa.UD = p->UDb; pa.Gmax = p->Gmax; pa.meta = st->d_meta;
  pa.body = st->d_body;
  {
    PROF("pack", s);
    e = pack_factors(pa, s);
  }
  if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "pack: %s", cudaGetErrorString(e)));
  ResidualArgs ra;
  ra.n_lt = p->n_lt; ra.H = sh.heads; ra.T = sh.tokens; ra.D = D; ra.lt_ids = p->d_lt_ids;
  ra.X[0] = K; ra.X[1] = V; ra.xt = sh.dtype == JOLT_BF16 ? EL_BF16 : EL_F32; ra.Pi = st->d_Pi;
  ra.meta = st->d_meta; ra.body = st->d_body; ra.PiT = p->PiT;
  ra.hadamard = p->cfg.rotation == 1 ? 1 : 0;
  if (p->cfg.measured_b) {
    // measured-b refinement: exact errors of every allowed width at the chosen ranks (one pass of
    // the residual coder that writes no codes), then a second dual over b with those errors; the
    // layout and the packed factors follow the new widths
    ResidualArgs rm = ra;
    rm.measure = 1;
    rm.bits_mask = p->cfg.bits_mask;
    rm.meas_part = p->meas_part;
    {
      PROF("measure_b", s);
      e = residual_encode(rm, p->Pbuf, p->Nbuf, std::max(p->R, 1), s);
      if (e == cudaSuccess) e = measured_tables(da, p->meas_part, (sh.tokens + 255) / 256, p->meas_lt, s);
    }
    if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "measure_b: %s", cudaGetErrorString(e)));
    DualArgs d2 = da;
    d2.tables_ready = 1;
    {
      PROF("dual", s);
      e = dual_allocate(d2, s);
    }
    if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "dual: %s", cudaGetErrorString(e)));
    {
      PROF("pack", s);
      e = pack_factors(pa, s);
    }
    if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "pack: %s", cudaGetErrorString(e)));
  }
  {
    PROF("residual", s);
    e = residual_encode(ra, p->Pbuf, p->Nbuf, std::max(p->R, 1), s);
  }
  if (e != cudaSuccess) return bail(fail(JOLT_ERR_CUDA, "residual: %s", cudaGetErrorString(e)));
  p->last = st;
  *out = st;
  return JOLT_OK;
}

JOLT_API jolt_status jolt_decode(jolt_stream_t st, void* K_out, void* V_out, void* cuda_stream) {
  g_err.clear();
  if (!st || !K_out) return fail(JOLT_ERR_INVALID_ARG, "jolt_decode: null stream or K_out");
  if (st->has_v && !V_out) return fail(JOLT_ERR_INVALID_ARG, "jolt_decode: stream has V but V_out is null");
  DecodeArgs a;
  a.n_lt = st->n_lt; a.L = st->L; a.H = st->H; a.T = st->T; a.D = st->D; a.lt_ids = st->d_lt_ids;
  a.out[0] = K_out; a.out[1] = V_out; a.ot = st->dtype == JOLT_BF16 ? EL_BF16 : EL_F32;
  a.Pi = st->d_Pi; a.meta = st->d_meta; a.body = st->d_body;
  PROF("decode", (cudaStream_t)cuda_stream);
  CK(decode(a, (cudaStream_t)cuda_stream));
  return JOLT_OK;
}

JOLT_API jolt_status jolt_attention(jolt_stream_t st, const void* Q, int32_t q_heads, int32_t n_queries,
                                    float scale, float* out, void* cuda_stream) {
  g_err.clear();
  if (!st || !Q || !out) return fail(JOLT_ERR_INVALID_ARG, "jolt_attention: null stream, Q or out");
  if (!st->has_v) return fail(JOLT_ERR_INVALID_ARG, "jolt_attention: the stream holds keys only");
  if (st->dtype != JOLT_BF16) return fail(JOLT_ERR_UNSUPPORTED, "jolt_attention: bf16 streams only");
  if (q_heads <= 0 || n_queries <= 0 || q_heads % st->H != 0)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_attention: q_heads must be a positive multiple of the %d KV heads", st->H);
  cudaStream_t s = (cudaStream_t)cuda_stream;
  AttnArgs a;
  a.L = st->L; a.H = st->H; a.T = st->T; a.D = st->D; a.Hq = q_heads; a.n = n_queries; a.R = std::max(st->R, 1);
  a.scale = scale; a.meta = st->d_meta; a.body = st->d_body; a.Pi = st->d_Pi;
  a.Q = reinterpret_cast<const __nv_bfloat16*>(Q); a.out = out;
  a.nchunk = attn_chunks(st->T); a.ngroups = attn_groups(q_heads, st->H, n_queries);
  const size_t nqv = (size_t)a.L * q_heads * n_queries;
  const size_t floats = nqv * (kD + a.R) + (size_t)a.L * a.H * a.nchunk * a.ngroups * attn_part_floats(a.R);
  float* scratch = nullptr;
  PROF("attention", s);
  CK(pool_malloc(&scratch, floats * sizeof(float), s));
  a.qpi = scratch;
  a.qhat = scratch + nqv * kD;
  a.part = a.qhat + nqv * a.R;
  cudaError_t e = attention(a, s);
  cudaError_t e2 = cudaFreeAsync(scratch, s);
  if (e == cudaSuccess) e = e2;
  if (e != cudaSuccess) return fail(JOLT_ERR_CUDA, "jolt_attention: %s", cudaGetErrorString(e));
  return JOLT_OK;
}

JOLT_API jolt_status jolt_rel_frob_error(const void* ref, const void* approx, uint64_t n, jolt_dtype dtype,
                                         void* cuda_stream, double* out) {
  g_err.clear();
  if (!ref || !approx || !out) return fail(JOLT_ERR_INVALID_ARG, "jolt_rel_frob_error: null pointer");
  if (dtype != JOLT_BF16 && dtype != JOLT_F32) return fail(JOLT_ERR_INVALID_ARG, "jolt_rel_frob_error: dtype");
  cudaStream_t s = (cudaStream_t)cuda_stream;
  const int nb = relfrob_blocks(n);
  Prof prof_rf("rel_frob", s);
  double* scratch = nullptr;
  CK(pool_malloc(&scratch, sizeof(double) * (2 * (size_t)nb + 2), s));
  cudaError_t e = relfrob_partial(ref, approx, n, dtype == JOLT_BF16 ? EL_BF16 : EL_F32, scratch + 2, nb, scratch, s);
  double h[2] = {0.0, 0.0};
  if (e == cudaSuccess) e = cudaMemcpyAsync(h, scratch, sizeof(h), cudaMemcpyDeviceToHost, s);
  cudaError_t e2 = cudaFreeAsync(scratch, s);
  if (e == cudaSuccess) e = e2;
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(JOLT_ERR_CUDA, "jolt_rel_frob_error: %s", cudaGetErrorString(e));
  *out = h[1] > 0.0 ? std::sqrt(h[0]) / std::sqrt(h[1]) : 0.0;
  return JOLT_OK;
}

JOLT_API jolt_status jolt_rel_frob_error_noalloc(const void* ref, const void* approx, uint64_t n,
                                                 jolt_dtype dtype, void* cuda_stream, double* out) {
  g_err.clear();
  if (!ref || !approx || !out) return fail(JOLT_ERR_INVALID_ARG, "jolt_rel_frob_error_noalloc: null pointer");
  if (dtype != JOLT_BF16 && dtype != JOLT_F32)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_rel_frob_error_noalloc: dtype");
  if (n > JOLT_REL_FROB_NOALLOC_MAX_N)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_rel_frob_error_noalloc: n = %llu exceeds the limit %llu",
                (unsigned long long)n, (unsigned long long)JOLT_REL_FROB_NOALLOC_MAX_N);
  const int nb = relfrob_blocks(n);
  if (nb > kRelfrobStaticBlocks)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_rel_frob_error_noalloc: %d partial sums exceed the fixed scratch of %d",
                nb, kRelfrobStaticBlocks);
  // The fixed scratch's device address in the current context, looked up on every call (a
  // symbol lookup allocates nothing), so a context torn down and created again is followed.
  double* scratch = nullptr;
  {
    const cudaError_t e = relfrob_static_scratch(&scratch);
    if (e != cudaSuccess || !scratch)
      return fail(JOLT_ERR_CUDA, "jolt_rel_frob_error_noalloc: scratch address: %s", cudaGetErrorString(e));
  }
  cudaStream_t s = (cudaStream_t)cuda_stream;
  Prof prof_rf("rel_frob", s);
  // The two totals are cleared before the kernels run (every partial slot is written).
  cudaError_t e = cudaMemsetAsync(scratch, 0, 2 * sizeof(double), s);
  if (e == cudaSuccess)
    e = relfrob_partial(ref, approx, n, dtype == JOLT_BF16 ? EL_BF16 : EL_F32, scratch + 2, nb, scratch, s);
  double h[2] = {0.0, 0.0};
  if (e == cudaSuccess) e = cudaMemcpyAsync(h, scratch, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(JOLT_ERR_CUDA, "jolt_rel_frob_error_noalloc: %s", cudaGetErrorString(e));
  *out = h[1] > 0.0 ? std::sqrt(h[0]) / std::sqrt(h[1]) : 0.0;
  return JOLT_OK;
}

static jolt_status read_meta(jolt_stream_s* st, StreamMeta* m) {
  CK(cudaStreamSynchronize(st->cs));
  CK(cudaMemcpy(m, st->d_meta, sizeof(StreamMeta), cudaMemcpyDeviceToHost));
  return JOLT_OK;
}

static jolt_status status_of(int32_t bits) {
  if (bits & ST_NONFINITE) return fail(JOLT_ERR_NONFINITE, "non-finite value in the input");
  if (bits & ST_INFEASIBLE) return fail(JOLT_ERR_BUDGET_INFEASIBLE, "budget infeasible");
  if (bits & ST_TIMEOUT) return fail(JOLT_ERR_TIMEOUT, "a bounded device wait gave up");
  if (bits & ST_NOT_CONVERGED) return fail(JOLT_ERR_NOT_CONVERGED, "an eigensolver or Cholesky step hit its limit");
  return JOLT_OK;
}

JOLT_API jolt_status jolt_stream_status(jolt_stream_t st) {
  g_err.clear();
  if (!st) return fail(JOLT_ERR_INVALID_ARG, "jolt_stream_status: null stream");
  StreamMeta m;
  jolt_status r = read_meta(st, &m);
  if (r != JOLT_OK) return r;
  return status_of(m.status);
}

JOLT_API jolt_status jolt_stream_info(jolt_stream_t st, uint64_t* bytes_by_part, int32_t* alloc, double* lambdas) {
  g_err.clear();
  if (!st) return fail(JOLT_ERR_INVALID_ARG, "jolt_stream_info: null stream");
  StreamMeta m;
  jolt_status r = read_meta(st, &m);
  if (r != JOLT_OK) return r;
  if (bytes_by_part)
    for (int i = 0; i < JOLT_NUM_PARTS; ++i) bytes_by_part[i] = (uint64_t)m.bytes_by_part[i];
  if (alloc)
    for (int g = 0; g < st->G; ++g)
      for (int k = 0; k < 2; ++k)
        for (int j = 0; j < 3; ++j) alloc[(g * 2 + k) * 3 + j] = m.alloc[g][k][j];
  if (lambdas) { lambdas[0] = m.lambda[0]; lambdas[1] = m.lambda[1]; }
  return status_of(m.status);
}

// ---------------------------------------------------------------- serialization
static size_t header_bytes(int G) { return align_up(64 + 24 * (size_t)G, 16); }

static void put32(std::vector<uint8_t>& b, size_t off, uint32_t v) { memcpy(&b[off], &v, 4); }
static void put64(std::vector<uint8_t>& b, size_t off, uint64_t v) { memcpy(&b[off], &v, 8); }

JOLT_API jolt_status jolt_stream_to_host(jolt_stream_t st, void* buf, uint64_t* len) {
  g_err.clear();
  if (!st || !len) return fail(JOLT_ERR_INVALID_ARG, "jolt_stream_to_host: null stream or len");
  StreamMeta m;
  jolt_status r = read_meta(st, &m);
  if (r != JOLT_OK) return r;
  if (m.status & (ST_NONFINITE | ST_INFEASIBLE)) return status_of(m.status);
  const size_t hb = header_bytes(st->G);
  const size_t total = hb + (size_t)m.body_bytes + 4;
  if (!buf) { *len = total; return JOLT_OK; }
  if (*len < total) return fail(JOLT_ERR_INVALID_ARG, "jolt_stream_to_host: buffer of %llu < %zu bytes",
                                (unsigned long long)*len, total);
  std::vector<uint8_t> head(hb, 0);
  memcpy(&head[0], "JOLT", 4);
  put32(head, 4, 1);
  put32(head, 8, (uint32_t)hb);
  const uint32_t flags = (uint32_t)st->has_v | ((st->dtype == JOLT_F32 ? 1u : 0u) << 1) |
                         ((uint32_t)st->split << 2) | ((uint32_t)(st->rotation & 1) << 3) |
                         ((uint32_t)st->encoder << 8);
  put32(head, 12, flags);
  const int32_t ints[8] = {st->L, st->H, st->T, st->D, st->G, st->step, st->R, 0};
  memcpy(&head[16], ints, sizeof(ints));
  put64(head, 48, st->seed);
  put64(head, 56, (uint64_t)m.body_bytes);
  for (int g = 0; g < st->G; ++g)
    for (int k = 0; k < 2; ++k) {
      int32_t a3[3] = {0, 0, 0};
      if (k == 0 || st->has_v)
        for (int j = 0; j < 3; ++j) a3[j] = m.alloc[g][k][j];
      memcpy(&head[64 + 24 * g + 12 * k], a3, 12);
    }
  uint8_t* o = reinterpret_cast<uint8_t*>(buf);
  memcpy(o, head.data(), hb);
  CK(cudaMemcpy(o + hb, st->d_body, (size_t)m.body_bytes, cudaMemcpyDeviceToHost));
  // padding between parts is not guaranteed zero on the device: clear it on the host
  {
    size_t cur = 0;
    for (int l = 0; l < st->L; ++l)
      for (int k = 0; k < (st->has_v ? 2 : 1); ++k) {
        const int lt = 2 * l + k;
        const int rt = m.lt_rank[lt][0], rd = m.lt_rank[lt][1], b = m.lt_rank[lt][2];
        const size_t sz[5] = {(size_t)st->T * rt * 2, (size_t)st->D * rd * 2, (size_t)st->H * rt * rd * 2,
                              b > 0 ? (size_t)st->H * st->T * 2 : 0,
                              b > 0 ? (size_t)st->H * st->T * (st->D * b / 8) : 0};
        for (int pp = 0; pp < 5; ++pp) {
          const size_t off = (size_t)m.off[lt][pp];
          if (off > cur) memset(o + hb + cur, 0, off - cur);
          cur = off + sz[pp];
        }
      }
  }
  const uint32_t crc = crc32_ieee(o, hb + (size_t)m.body_bytes);
  memcpy(o + hb + (size_t)m.body_bytes, &crc, 4);
  *len = total;
  return JOLT_OK;
}

JOLT_API jolt_status jolt_stream_from_host(const void* buf, uint64_t len, void* cuda_stream, jolt_stream_t* out) {
  g_err.clear();
  if (!buf || !out) return fail(JOLT_ERR_INVALID_ARG, "jolt_stream_from_host: null pointer");
  *out = nullptr;
  const uint8_t* b = reinterpret_cast<const uint8_t*>(buf);
  if (len < 68 || memcmp(b, "JOLT", 4) != 0) return fail(JOLT_ERR_CORRUPT_STREAM, "bad magic or short buffer");
  uint32_t ver, hb, flags;
  memcpy(&ver, b + 4, 4);
  memcpy(&hb, b + 8, 4);
  memcpy(&flags, b + 12, 4);
  if (ver != 1) return fail(JOLT_ERR_CORRUPT_STREAM, "unsupported version %u", ver);
  int32_t ints[8];
  memcpy(ints, b + 16, sizeof(ints));
  uint64_t seed, body;
  memcpy(&seed, b + 48, 8);
  memcpy(&body, b + 56, 8);
  const int L = ints[0], H = ints[1], T = ints[2], D = ints[3], G = ints[4];
  if (L <= 0 || L > kMaxL || H <= 0 || T <= 0 || D != kD || G <= 0 || G > L || G > kMaxGroups)
    return fail(JOLT_ERR_CORRUPT_STREAM, "header shape out of range");
  if (hb != header_bytes(G) || len != (uint64_t)hb + body + 4) return fail(JOLT_ERR_CORRUPT_STREAM, "size mismatch");
  uint32_t crc;
  memcpy(&crc, b + hb + body, 4);
  if (crc != crc32_ieee(b, hb + body)) return fail(JOLT_ERR_CORRUPT_STREAM, "CRC mismatch");
  const int has_v = flags & 1;
  StreamMeta m;
  memset(&m, 0, sizeof(m));
  for (int g = 0; g < G; ++g)
    for (int k = 0; k < 2; ++k) memcpy(m.alloc[g][k], b + 64 + 24 * g + 12 * k, 12);
  int64_t cur = 0;
  for (int l = 0; l < L; ++l) {
    const int g = group_of_layer(l, L, G);
    for (int k = 0; k < (has_v ? 2 : 1); ++k) {
      const int lt = 2 * l + k;
      const int rt = m.alloc[g][k][0], rd = m.alloc[g][k][1], bb = m.alloc[g][k][2];
      if (rt < 0 || rt > kMaxN || rd < 0 || rd > D || bb < 0 || bb > 8 || (rt == 0) != (rd == 0))
        return fail(JOLT_ERR_CORRUPT_STREAM, "allocation table out of range");
      m.lt_rank[lt][0] = rt; m.lt_rank[lt][1] = rd; m.lt_rank[lt][2] = bb;
      const int64_t sz[5] = {(int64_t)T * rt * 2, (int64_t)D * rd * 2, (int64_t)H * rt * rd * 2,
                             bb > 0 ? (int64_t)H * T * 2 : 0, bb > 0 ? (int64_t)H * T * (D * bb / 8) : 0};
      for (int pp = 0; pp < 5; ++pp) {
        const int64_t off = (cur + kAlign - 1) / kAlign * kAlign;
        m.off[lt][pp] = off;
        cur = off + sz[pp];
        m.bytes_by_part[pp] += sz[pp];
      }
    }
  }
  if ((uint64_t)cur != body) return fail(JOLT_ERR_CORRUPT_STREAM, "body size does not match the allocation table");
  m.body_bytes = cur;
  m.num_lt = L * (has_v ? 2 : 1);
  cudaStream_t s = (cudaStream_t)cuda_stream;
  jolt_stream_s* st = new (std::nothrow) jolt_stream_s();
  if (!st) return fail(JOLT_ERR_OOM, "host allocation");
  st->L = L; st->H = H; st->T = T; st->D = D; st->has_v = has_v; st->G = G;
  st->encoder = (flags >> 8) & 0xFF; st->step = ints[5]; st->R = ints[6]; st->split = (flags >> 2) & 1;
  st->dtype = (flags & 2) ? JOLT_F32 : JOLT_BF16; st->seed = seed; st->cs = s; st->n_lt = m.num_lt;
  st->body_cap = std::max<size_t>((size_t)body, 256);
  std::vector<int32_t> ids;
  for (int k = 0; k < (has_v ? 2 : 1); ++k)
    for (int l = 0; l < L; ++l) ids.push_back(2 * l + k);
  cudaError_t e = pool_malloc(&st->d_body, st->body_cap, s);
  if (e == cudaSuccess) e = pool_malloc(&st->d_meta, sizeof(StreamMeta), s);
  if (e == cudaSuccess) e = pool_malloc(&st->d_Pi, sizeof(float) * D * D, s);
  if (e == cudaSuccess) e = pool_malloc(&st->d_Gpi, sizeof(double) * D * D, s);
  if (e == cudaSuccess) e = pool_malloc(&st->d_lt_ids, sizeof(int32_t) * ids.size(), s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->d_body, b + hb, (size_t)body, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->d_meta, &m, sizeof(m), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->d_lt_ids, ids.data(), sizeof(int32_t) * ids.size(), cudaMemcpyHostToDevice, s);
  st->rotation = (int)((flags >> 3) & 1u);
  if (st->rotation == 1) {
    if (e == cudaSuccess) e = hadamard_pi(seed, D, st->d_Pi, nullptr, s);
  } else {
    if (e == cudaSuccess) e = gauss_f64(seed, 1, (int64_t)D * D, st->d_Gpi, s);
    if (e == cudaSuccess) e = haar_from_gauss(st->d_Gpi, D, st->d_Pi, nullptr, s);
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);   // host buffers above are stack / vector
  if (e != cudaSuccess) {
    jolt_stream_destroy(st);
    return fail(JOLT_ERR_CUDA, "jolt_stream_from_host: %s", cudaGetErrorString(e));
  }
  *out = st;
  return JOLT_OK;
}

JOLT_API jolt_status jolt_export_debug(jolt_stream_t st, int32_t what, int32_t lt, void* buf, uint64_t* len) {
  g_err.clear();
  if (!st || !len) return fail(JOLT_ERR_INVALID_ARG, "jolt_export_debug: null stream or len");
  CK(cudaStreamSynchronize(st->cs));
  jolt_plan_s* p = st->plan;
  const void* src = nullptr;
  size_t n = 0;
  bool host_src = false;
  StreamMeta m;
  std::vector<double> tmp;
  auto index_of = [&](int lt_) -> int {
    if (!p) return -1;
    for (size_t i = 0; i < p->lt_ids.size(); ++i)
      if (p->lt_ids[i] == lt_) return (int)i;
    return -1;
  };
  if (what == JOLT_DBG_PI) {
    src = st->d_Pi;
    n = sizeof(float) * st->D * st->D;
  } else if (what == JOLT_DBG_LAMBDA) {
    CK(cudaMemcpy(&m, st->d_meta, sizeof(m), cudaMemcpyDeviceToHost));
    tmp.assign(m.lambda, m.lambda + 2);
    src = tmp.data();
    n = sizeof(double) * 2;
    host_src = true;
  } else {
    if (!p || p->last != st) return fail(JOLT_ERR_INVALID_ARG, "jolt_export_debug: plan no longer holds this stream's encode");
    const int i = index_of(lt);
    switch (what) {
      case JOLT_DBG_UT_F32:
        if (i < 0) return fail(JOLT_ERR_INVALID_ARG, "bad lt");
        src = p->UT32 + (int64_t)i * st->T * p->R;
        n = sizeof(float) * st->T * p->R;
        break;
      case JOLT_DBG_UD_F32:
        if (i < 0) return fail(JOLT_ERR_INVALID_ARG, "bad lt");
        src = p->UD32 + (int64_t)i * st->D * st->D;
        n = sizeof(float) * st->D * st->D;
        break;
      case JOLT_DBG_TABLE:
        if (lt < 0 || lt >= 2 * st->G) return fail(JOLT_ERR_INVALID_ARG, "bad unit");
        src = p->unit_err + (int64_t)lt * p->nbits * p->ngrid;
        n = sizeof(double) * p->nbits * p->ngrid;
        break;
      case JOLT_DBG_MEAS: {
        if (!p->meas_lt) return fail(JOLT_ERR_INVALID_ARG, "the plan has no measured-b refinement");
        int i = -1;
        for (size_t j = 0; j < p->lt_ids.size(); ++j)
          if (p->lt_ids[j] == lt) i = (int)j;
        if (i < 0) return fail(JOLT_ERR_INVALID_ARG, "bad layer-tensor");
        src = p->meas_lt + (int64_t)i * 9;
        n = sizeof(double) * 9;
        break;
      }
      case JOLT_DBG_XX:
        tmp.assign(2 * (size_t)st->L, 0.0);
        for (size_t j = 0; j < p->lt_ids.size(); ++j)
          CK(cudaMemcpy(&tmp[p->lt_ids[j]], p->xx + j, sizeof(double), cudaMemcpyDeviceToHost));
        src = tmp.data();
        n = sizeof(double) * tmp.size();
        host_src = true;
        break;
      case JOLT_DBG_OMEGA: {
        if (i < 0 || p->encoder != JOLT_ENC_SKETCH) return fail(JOLT_ERR_INVALID_ARG, "no sketch for this lt");
        const int64_t HD = (int64_t)st->H * st->D, l = p->l;
        n = sizeof(__nv_bfloat16) * HD * l;
        std::vector<uint16_t> raw((size_t)(HD * l));
        CK(cudaMemcpy(raw.data(), p->Om + (int64_t)i * HD * l, n, cudaMemcpyDeviceToHost));
        tmp.assign((n + 7) / 8, 0.0);
        uint16_t* o = reinterpret_cast<uint16_t*>(tmp.data());
        for (int64_t r = 0; r < HD; ++r)          // always exported as [HD][l]
          for (int64_t c = 0; c < l; ++c) o[r * l + c] = p->use_tc ? raw[(size_t)(c * HD + r)] : raw[(size_t)(r * l + c)];
        src = tmp.data();
        host_src = true;
        break;
      }
      default:
        return fail(JOLT_ERR_INVALID_ARG, "jolt_export_debug: unknown item %d", what);
    }
  }
  if (!buf) { *len = n; return JOLT_OK; }
  if (*len < n) return fail(JOLT_ERR_INVALID_ARG, "jolt_export_debug: buffer too small");
  if (host_src) memcpy(buf, src, n);
  else CK(cudaMemcpy(buf, src, n, cudaMemcpyDeviceToHost));
  *len = n;
  return JOLT_OK;
}

namespace {
jolt_status selftest_gemm(const char* who, int32_t M, int32_t N, int32_t K, const void* A, int32_t a_mn, const void* B,
                          int32_t b_mn, float* C, void* cuda_stream) {
  g_err.clear();
  if (M <= 0 || N <= 0 || K <= 0 || (K % 8) || !A || !B || !C || (a_mn && M % 8) || (b_mn && N % 8))
    return fail(JOLT_ERR_INVALID_ARG, "%s: bad sizes or pointers", who);
  cudaStream_t s = (cudaStream_t)cuda_stream;
  TcGemmParams p;
  const uint64_t adims[3] = {(uint64_t)K, (uint64_t)M, 1}, astr[2] = {(uint64_t)K * 2, (uint64_t)K * M * 2};
  const uint64_t bdims[3] = {(uint64_t)K, (uint64_t)N, 1}, bstr[2] = {(uint64_t)K * 2, (uint64_t)K * N * 2};
  const bool aok = a_mn ? tc_map_bf16_mn(&p.amap[0], A, M, K, 1) : tc_map_bf16(&p.amap[0], A, 3, adims, astr);
  const bool bok = b_mn ? tc_map_bf16_mn(&p.bmap[0], B, N, K, 1) : tc_map_bf16(&p.bmap[0], B, 3, bdims, bstr);
  if (!aok || !bok) return fail(JOLT_ERR_INVALID_ARG, "%s: tensor map rejected", who);
  if (a_mn) p.av.mode = VIEW_MN;
  if (b_mn) p.bv.mode = VIEW_MN;
  p.na = p.nb = 1;
  p.M = M; p.N = N; p.KB = (K + 63) / 64;
  p.C = C; p.c_sm = N; p.c_sn = 1; p.c_sb = (int64_t)M * N;
  int32_t* st = nullptr;
  CK(pool_malloc(&st, sizeof(int32_t), s));
  CK(cudaMemsetAsync(st, 0, sizeof(int32_t), s));
  p.status = st;
  cudaError_t e = gemm_tc(1, p, s);
  int32_t h = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, st, sizeof(h), cudaMemcpyDeviceToHost, s);
  cudaFreeAsync(st, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(JOLT_ERR_CUDA, "%s: %s", who, cudaGetErrorString(e));
  return status_of(h);
}
}  // namespace

JOLT_API jolt_status jolt_selftest_gemm_bf16(int32_t M, int32_t N, int32_t K, const void* A, const void* B,
                                             float* C, void* cuda_stream) {
  return selftest_gemm("jolt_selftest_gemm_bf16", M, N, K, A, 0, B, 0, C, cuda_stream);
}

JOLT_API jolt_status jolt_selftest_gemm_bf16_layout(int32_t M, int32_t N, int32_t K, const void* A, int32_t a_mn,
                                                    const void* B, int32_t b_mn, float* C, void* cuda_stream) {
  return selftest_gemm("jolt_selftest_gemm_bf16_layout", M, N, K, A, a_mn, B, b_mn, C, cuda_stream);
}

JOLT_API jolt_status jolt_selftest_eig_dense(int32_t batch, int32_t n, int32_t R, const double* A, double* V,
                                             double* lam, void* cuda_stream) {
  g_err.clear();
  if (batch <= 0 || n < 2 || n > kExactMaxTokens || R < 1 || R > n || R > kMaxN || !A || !V || !lam)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_selftest_eig_dense: need batch >= 1, 2 <= n <= %d, 1 <= R <= min(n, %d)",
                kExactMaxTokens, kMaxN);
  cudaStream_t s = (cudaStream_t)cuda_stream;
  double *a = nullptr, *tri = nullptr, *qx = nullptr, *gx = nullptr, *rx = nullptr;
  int32_t* st = nullptr;
  const size_t nn = (size_t)batch * n * n;
  cudaError_t e = dev_malloc(&a, nn * sizeof(double));
  if (e == cudaSuccess) e = dev_malloc(&tri, tridiag_scratch_doubles(batch, n, R) * sizeof(double));
  if (e == cudaSuccess) e = dev_malloc(&qx, (size_t)batch * n * R * sizeof(double));
  if (e == cudaSuccess) e = dev_malloc(&gx, (size_t)batch * R * R * sizeof(double));
  if (e == cudaSuccess) e = dev_malloc(&rx, (size_t)batch * R * R * sizeof(double));
  if (e == cudaSuccess) e = dev_malloc(&st, sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMemsetAsync(st, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(a, A, nn * sizeof(double), cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = dense_top_eig(batch, n, R, a, (int64_t)n * n, tri, qx, gx, rx, V, EL_F64, lam, st, s);
  int32_t hs = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&hs, st, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  for (void* q : {(void*)a, (void*)tri, (void*)qx, (void*)gx, (void*)rx, (void*)st})
    if (q) cudaFree(q);
  if (e != cudaSuccess) return fail(JOLT_ERR_CUDA, "jolt_selftest_eig_dense: %s", cudaGetErrorString(e));
  if (hs & ST_NOT_CONVERGED) return fail(JOLT_ERR_NOT_CONVERGED, "jolt_selftest_eig_dense: a Cholesky pivot was floored");
  return JOLT_OK;
}

JOLT_API jolt_status jolt_selftest_eig_small(int32_t batch, int32_t n, const double* A, float* V, float* lam,
                                             int32_t solver, void* cuda_stream) {
  g_err.clear();
  if (batch <= 0 || n < 1 || n > kMaxN || !A || !V || !lam ||
      (solver != JOLT_EIG_TRIDIAG && solver != JOLT_EIG_JACOBI))
    return fail(JOLT_ERR_INVALID_ARG, "jolt_selftest_eig_small: need batch >= 1, 1 <= n <= %d, solver 0 or 1", kMaxN);
  cudaStream_t s = (cudaStream_t)cuda_stream;
  int32_t* st = nullptr;
  cudaError_t e = dev_malloc(&st, sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMemsetAsync(st, 0, sizeof(int32_t), s);
  const int64_t nn = (int64_t)n * n;
  if (e == cudaSuccess)
    e = solver == JOLT_EIG_JACOBI
            ? eig_psd2(batch, n, A, nn, V, nn, lam, n, 0, 0, nullptr, 0, nullptr, 0, nullptr, 0, 30, st, s)
            : eig_small2(batch, n, A, nn, V, nn, lam, n, 0, 0, nullptr, 0, nullptr, 0, nullptr, 0, st, s);
  int32_t hs = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&hs, st, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (st) cudaFree(st);
  if (e != cudaSuccess) return fail(JOLT_ERR_CUDA, "jolt_selftest_eig_small: %s", cudaGetErrorString(e));
  if (hs & ST_NONFINITE) return fail(JOLT_ERR_NONFINITE, "jolt_selftest_eig_small: non-finite input or result");
  if (hs & ST_NOT_CONVERGED) return fail(JOLT_ERR_NOT_CONVERGED, "jolt_selftest_eig_small: Jacobi sweep limit");
  return JOLT_OK;
}

JOLT_API uint64_t jolt_launch_count(void) { return g_launches.load(); }

JOLT_API uint64_t jolt_alloc_count(void) { return g_allocs.load(); }

JOLT_API jolt_status jolt_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = on != 0;
  return JOLT_OK;
}

JOLT_API jolt_status jolt_profile_report(char* buf, uint64_t* len) {
  g_err.clear();
  if (!len) return fail(JOLT_ERR_INVALID_ARG, "jolt_profile_report: null len");
  CK(cudaDeviceSynchronize());
  std::lock_guard<std::mutex> g(g_prof_mu);
  struct Agg { std::string name; uint64_t calls = 0, launches = 0; double ms = 0.0; };
  std::vector<Agg> agg;
  for (const ProfRec& r : g_prof) {
    float ms = 0.0f;
    cudaEventElapsedTime(&ms, r.a, r.b);
    size_t i = 0;
    while (i < agg.size() && agg[i].name != r.name) ++i;
    if (i == agg.size()) { agg.push_back(Agg()); agg.back().name = r.name; }
    agg[i].calls += 1;
    agg[i].launches += r.launches;
    agg[i].ms += ms;
  }
  std::string out = "{";
  for (size_t i = 0; i < agg.size(); ++i) {
    char tmp[256];
    snprintf(tmp, sizeof(tmp), "%s\"%s\": {\"calls\": %llu, \"launches\": %llu, \"total_ms\": %.6f}",
             i ? ", " : "", agg[i].name.c_str(), (unsigned long long)agg[i].calls,
             (unsigned long long)agg[i].launches, agg[i].ms);
    out += tmp;
  }
  out += "}";
  if (!buf) { *len = out.size() + 1; return JOLT_OK; }
  if (*len < out.size() + 1) return fail(JOLT_ERR_INVALID_ARG, "jolt_profile_report: buffer too small");
  memcpy(buf, out.c_str(), out.size() + 1);
  *len = out.size() + 1;
  for (const ProfRec& r : g_prof) { g_pool.push_back(r.a); g_pool.push_back(r.b); }
  g_prof.clear();
  return JOLT_OK;
}

JOLT_API void jolt_stream_destroy(jolt_stream_t st) {
  if (!st) return;
  if (st->plan && st->plan->last == st) st->plan->last = nullptr;
  // stream-ordered release after the work already enqueued on the encode stream
  if (st->d_body) cudaFreeAsync(st->d_body, st->cs);
  if (st->d_meta) cudaFreeAsync(st->d_meta, st->cs);
  if (st->d_Pi) cudaFreeAsync(st->d_Pi, st->cs);
  if (st->d_Gpi) cudaFreeAsync(st->d_Gpi, st->cs);
  if (st->d_lt_ids) cudaFreeAsync(st->d_lt_ids, st->cs);
  delete st;
}

JOLT_API void jolt_plan_destroy(jolt_plan_t p) {
  if (!p) return;
  cudaDeviceSynchronize();
  if (p->ws) cudaFree(p->ws);
  if (p->d_lt_ids) cudaFree(p->d_lt_ids);
  if (p->d_cand_order) cudaFree(p->d_cand_order);
  delete p;
}

}  // extern "C"
