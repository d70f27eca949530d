// Attention over the compressed cache: softmax(scale q K_hat^T) V_hat for a few queries per head,
// read from a JoLT stream without rebuilding K_hat or V_hat.
//
// The JoLT pages compress the KV cache that attention reads ("A JoLT for the KV Cache", arXiv
// 2607.12550v2, Abstract: partial Tucker factors plus a rotated low-bit residual); by linearity of
// that reconstruction, with s_t the row scale and Y_hat the unit-scale cell centres,
//     q . K_hat[h, t] = U_T[t] (G_h (U_D^T q)) + s_t Y_hat[h, t] . (Pi^T q),
//     sum_t p_t V_hat[h, t] = ((p^T U_T) G_h) U_D^T + ((p * s)^T Y_hat[h]) Pi^T,
// so a query needs the stored factors, the codes and the scales only (about half the bytes of a
// bf16 cache at 2x). Grouped-query attention: query head j reads KV head j / (Hq / H).
//  * k_attn_prep: per query, Pi^T q and G_h (U_D^T q) for the keys of its layer (float32);
//  * k_attn_partial: one CTA per (chunk of kChunk tokens, KV head, layer and group of at most kQ
//    queries); a half-warp takes a token at a time (lane i: features 8i .. 8i + 7 and every 16th
//    entry of the U_T row), forms the score, and keeps an online softmax (running max m, sum l)
//    with the two weighted sums of the value side (Y_hat weighted by p s, U_T by p);
//  * k_attn_combine: merges the chunks (rescaled by e^(m_c - m)) and applies G_h, U_D and Pi of
//    the values.
#include "../jolt_internal.h"

namespace jolt {
namespace {

constexpr int kQ = 4;          // queries per CTA
constexpr int kChunk = 256;    // tokens per CTA
constexpr int kHalfWarps = 8;  // 4 warps

__device__ __forceinline__ float bf(const __nv_bfloat16 v) { return __bfloat162float(v); }

struct LtView {
  int rt, rd, b;
  const __nv_bfloat16 *UT, *UD, *G;
  const __half* sc;
  const uint8_t* codes;
};

__device__ __forceinline__ LtView lt_view(const AttnArgs& a, int lt) {
  const StreamMeta* m = a.meta;
  LtView v;
  v.rt = m->lt_rank[lt][0];
  v.rd = m->lt_rank[lt][1];
  v.b = m->lt_rank[lt][2];
  if (v.rt == 0 || v.rd == 0) v.rt = v.rd = 0;
  v.UT = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UT]);
  v.UD = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UD]);
  v.G = reinterpret_cast<const __nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_G]);
  v.sc = reinterpret_cast<const __half*>(a.body + m->off[lt][JOLT_PART_SCALES]);
  v.codes = a.body + m->off[lt][JOLT_PART_CODES];
  return v;
}

// qpi = Pi^T q and qhat = G_h (U_D^T q) (keys of the query's layer); one CTA per query vector.
__global__ void __launch_bounds__(128) k_attn_prep(AttnArgs a) {
  __shared__ float q[kD], qt[kD];
  const int idx = blockIdx.x;                       // ((layer * Hq) + j) * n + i
  const int layer = idx / (a.Hq * a.n), j = (idx / a.n) % a.Hq;
  const int h = j / (a.Hq / a.H);
  const int tid = threadIdx.x;
  q[tid] = bf(a.Q[(int64_t)idx * kD + tid]);
  __syncthreads();
  float s = 0.0f;
  for (int e = 0; e < kD; ++e) s = fmaf(a.Pi[e * kD + tid], q[e], s);
  a.qpi[(int64_t)idx * kD + tid] = s;
  const LtView k = lt_view(a, 2 * layer);
  if (tid < k.rd) {
    float t = 0.0f;
    for (int e = 0; e < kD; ++e) t = fmaf(bf(k.UD[e * k.rd + tid]), q[e], t);
    qt[tid] = t;
  }
  __syncthreads();
  for (int r = tid; r < a.R; r += 128) {
    float t = 0.0f;
    if (r < k.rt) {
      const __nv_bfloat16* g = k.G + ((int64_t)h * k.rt + r) * k.rd;
      for (int c = 0; c < k.rd; ++c) t = fmaf(bf(g[c]), qt[c], t);
    }
    a.qhat[(int64_t)idx * a.R + r] = t;
  }
}

// Eight codes of a row: the b bytes at byte offset byte0 of a 16-byte aligned row block, from the
// two aligned 8-byte words around them.
__device__ __forceinline__ uint64_t codes8(const uint8_t* blk, int byte0) {
  const uint64_t* w = reinterpret_cast<const uint64_t*>(blk + (byte0 & ~7));
  const int sh = (byte0 & 7) * 8;
  const uint64_t lo = __ldg(w);
  return sh ? (lo >> sh) | (__ldg(w + 1) << (64 - sh)) : lo;
}

__global__ void __launch_bounds__(128) k_attn_partial(AttnArgs a) {
  const int chunk = blockIdx.x, h = blockIdx.y, layer = blockIdx.z / a.ngroups, grp = blockIdx.z % a.ngroups;
  const int tid = threadIdx.x, hw = tid >> 4, l16 = tid & 15;
  const int g = a.Hq / a.H, nqv = g * a.n;
  const int q0 = grp * kQ, nq = min(kQ, nqv - q0);
  const LtView K = lt_view(a, 2 * layer), V = lt_view(a, 2 * layer + 1);
  const int t0 = chunk * kChunk, t1 = min(a.T, t0 + kChunk);
  // this lane's slice of each query's Pi^T q (features 8 l16 ..) and of G_h U_D^T q (every 16th)
  float qp[kQ][8], qsum[kQ], qh[kQ][8];
#pragma unroll
  for (int q = 0; q < kQ; ++q) {
    const int qv = q0 + min(q, nq - 1);
    const int64_t idx = ((int64_t)layer * a.Hq + h * g + qv / a.n) * a.n + qv % a.n;
    float s = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      qp[q][e] = a.qpi[idx * kD + 8 * l16 + e];
      s += qp[q][e];
    }
    qsum[q] = s;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = l16 + 16 * k;
      qh[q][k] = r < K.rt ? a.qhat[idx * a.R + r] : 0.0f;
    }
  }
  const int rowK = 16 * K.b, rowV = 16 * V.b;
  const float ck = K.b ? 2.0f / (float)(1 << K.b) : 0.0f, ok = K.b ? (1.0f - (float)(1 << K.b)) / (float)(1 << K.b) : 0.0f;
  const float cv = V.b ? 2.0f / (float)(1 << V.b) : 0.0f, ov = V.b ? (1.0f - (float)(1 << V.b)) / (float)(1 << V.b) : 0.0f;
  const uint64_t mk = K.b ? (1ull << K.b) - 1ull : 0ull, mv = V.b ? (1ull << V.b) - 1ull : 0ull;
  float m[kQ], l[kQ], ay[kQ][8], au[kQ][8];
#pragma unroll
  for (int q = 0; q < kQ; ++q) {
    m[q] = -INFINITY;
    l[q] = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ay[q][e] = au[q][e] = 0.0f;
  }
  for (int t = t0 + hw; t < t1; t += kHalfWarps) {
    // score: residual part s_t (Y_hat . Pi^T q) and Tucker part U_T[t] . qhat
    float part[kQ];
#pragma unroll
    for (int q = 0; q < kQ; ++q) part[q] = 0.0f;
    if (K.b) {
      const uint64_t v = codes8(K.codes + ((int64_t)h * a.T + t) * rowK, l16 * K.b);
      float dq[kQ];
#pragma unroll
      for (int q = 0; q < kQ; ++q) dq[q] = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float c = (float)(uint32_t)((v >> (e * K.b)) & mk);
#pragma unroll
        for (int q = 0; q < kQ; ++q) dq[q] = fmaf(c, qp[q][e], dq[q]);
      }
      const float sk = __half2float(K.sc[(int64_t)h * a.T + t]);
#pragma unroll
      for (int q = 0; q < kQ; ++q) part[q] = sk * fmaf(ck, dq[q], ok * qsum[q]);
    }
    if (K.rt) {
      const __nv_bfloat16* ut = K.UT + (int64_t)t * K.rt;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = l16 + 16 * k;
        if (r < K.rt) {
          const float u = bf(ut[r]);
#pragma unroll
          for (int q = 0; q < kQ; ++q) part[q] = fmaf(u, qh[q][k], part[q]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kQ; ++q)
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) part[q] += __shfl_xor_sync(0xffffffffu, part[q], o);
    // online softmax and the value side
    float p[kQ];
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      const float sc = a.scale * part[q];
      const float mn = fmaxf(m[q], sc);
      const float corr = expf(m[q] - mn);
      p[q] = expf(sc - mn);
      l[q] = fmaf(l[q], corr, p[q]);
      m[q] = mn;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ay[q][e] *= corr;
        au[q][e] *= corr;
      }
    }
    if (V.b) {
      const uint64_t v = codes8(V.codes + ((int64_t)h * a.T + t) * rowV, l16 * V.b);
      const float sv = __half2float(V.sc[(int64_t)h * a.T + t]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float y = fmaf(cv, (float)(uint32_t)((v >> (e * V.b)) & mv), ov) * sv;
#pragma unroll
        for (int q = 0; q < kQ; ++q) ay[q][e] = fmaf(p[q], y, ay[q][e]);
      }
    }
    if (V.rt) {
      const __nv_bfloat16* ut = V.UT + (int64_t)t * V.rt;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = l16 + 16 * k;
        if (r < V.rt) {
          const float u = bf(ut[r]);
#pragma unroll
          for (int q = 0; q < kQ; ++q) au[q][k] = fmaf(p[q], u, au[q][k]);
        }
      }
    }
  }
  // merge the eight half-warps' states, then write this chunk's (m, l, Y sum, U_T sum) per query
  const int PW = 2 + kD + a.R;
  extern __shared__ float st[];                 // [kHalfWarps][kQ][PW]
#pragma unroll
  for (int q = 0; q < kQ; ++q) {
    float* o = st + ((int64_t)hw * kQ + q) * PW;
    if (l16 == 0) {
      o[0] = m[q];
      o[1] = l[q];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) o[2 + 8 * l16 + e] = ay[q][e];
    for (int k = 0; k < 8; ++k)
      if (l16 + 16 * k < a.R) o[2 + kD + l16 + 16 * k] = au[q][k];
  }
  __syncthreads();
  float* out = a.part + ((((int64_t)layer * a.H + h) * a.nchunk + chunk) * a.ngroups + grp) * kQ * PW;
  for (int u = tid; u < kQ * PW; u += 128) {
    const int q = u / PW, c = u - q * PW;
    float mx = -INFINITY;
    for (int w = 0; w < kHalfWarps; ++w) mx = fmaxf(mx, st[(w * kQ + q) * PW]);
    float acc = 0.0f;
    if (c == 0) {
      acc = mx;
    } else {
      for (int w = 0; w < kHalfWarps; ++w) {
        const float mw = st[(w * kQ + q) * PW];
        const float f = mw == -INFINITY ? 0.0f : expf(mw - mx);
        acc = fmaf(f, st[(w * kQ + q) * PW + c], acc);
      }
    }
    out[u] = acc;
  }
}

// Merge the chunks of one (layer, KV head, query group) and apply the value factors:
// O = (a_U G_h) U_D^T + a_Y Pi^T with a_U, a_Y the softmax-weighted sums.
__global__ void __launch_bounds__(128) k_attn_combine(AttnArgs a) {
  const int h = blockIdx.x, layer = blockIdx.y / a.ngroups, grp = blockIdx.y % a.ngroups;
  const int g = a.Hq / a.H, nqv = g * a.n, q0 = grp * kQ, nq = min(kQ, nqv - q0);
  const int tid = threadIdx.x, PW = 2 + kD + a.R;
  const LtView V = lt_view(a, 2 * layer + 1);
  __shared__ float ay[kD], au[kD], w[kD];
  __shared__ float mstar, lstar;
  for (int q = 0; q < nq; ++q) {
    const float* base = a.part + (((int64_t)layer * a.H + h) * a.nchunk * a.ngroups + grp) * kQ * PW + (int64_t)q * PW;
    const int64_t cs = (int64_t)a.ngroups * kQ * PW;     // stride between chunks
    if (tid == 0) {
      float mx = -INFINITY;
      for (int c = 0; c < a.nchunk; ++c) mx = fmaxf(mx, base[c * cs]);
      float ls = 0.0f;
      for (int c = 0; c < a.nchunk; ++c) ls += base[c * cs + 1] * expf(base[c * cs] - mx);
      mstar = mx;
      lstar = ls;
    }
    __syncthreads();
    const float mx = mstar, inv = 1.0f / lstar;
    {
      float y = 0.0f, u = 0.0f;
      for (int c = 0; c < a.nchunk; ++c) {
        const float f = expf(base[c * cs] - mx);
        y = fmaf(f, base[c * cs + 2 + tid], y);
        if (tid < a.R) u = fmaf(f, base[c * cs + 2 + kD + tid], u);
      }
      ay[tid] = y * inv;
      au[tid] = u * inv;
    }
    __syncthreads();
    if (tid < V.rd) {
      float s = 0.0f;
      for (int k = 0; k < V.rt; ++k) s = fmaf(au[k], bf(V.G[((int64_t)h * V.rt + k) * V.rd + tid]), s);
      w[tid] = s;
    }
    __syncthreads();
    float o = 0.0f;
    for (int c = 0; c < V.rd; ++c) o = fmaf(bf(V.UD[tid * V.rd + c]), w[c], o);
    if (V.b)
      for (int d = 0; d < kD; ++d) o = fmaf(a.Pi[tid * kD + d], ay[d], o);
    const int qv = q0 + q;
    const int64_t idx = ((int64_t)layer * a.Hq + h * g + qv / a.n) * a.n + qv % a.n;
    a.out[idx * kD + tid] = o;
    __syncthreads();
  }
}

}  // namespace

int attn_groups(int Hq, int H, int n) { return (Hq / H * n + kQ - 1) / kQ; }
int attn_chunks(int T) { return (T + kChunk - 1) / kChunk; }
int attn_part_floats(int R) { return kQ * (2 + kD + R); }

cudaError_t attention(const AttnArgs& a, cudaStream_t s) {
  if (a.D != kD || a.Hq % a.H != 0 || a.n <= 0) return cudaErrorInvalidValue;
  k_attn_prep<<<a.L * a.Hq * a.n, 128, 0, s>>>(a);
  note_launch();
  const size_t sm = (size_t)kHalfWarps * kQ * (2 + kD + a.R) * sizeof(float);
  k_attn_partial<<<dim3(a.nchunk, a.H, a.L * a.ngroups), 128, sm, s>>>(a);
  note_launch();
  k_attn_combine<<<dim3(a.H, a.L * a.ngroups), 128, 0, s>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
