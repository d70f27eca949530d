// Error table, Lagrangian dual allocator and factor packing of the JoLT codec.
//
// "A JoLT for the KV Cache" (arXiv 2607.12550v2, Abstract): "A single Lagrangian dual
// allocates the Tucker ranks and the residual bit-widths together, per layer group and
// separately for keys and values, under one byte budget." The pages give no formula, so:
//  * candidate (r_t, r_d) are (0, 0) and every multiple of the rank step up to (R, D);
//  * table entry E(r_t, r_d) = max(0, ||X||^2 - sum_{h, i < r_t, j < r_d} G_max[h, i, j]^2),
//    the exact truncation energy of orthonormal nested factors, summed over a group's layers;
//  * err(r_t, r_d, b) = E * phi(b), phi(0) = 1, phi(b) = kappa_D / (3 * 4^b) (uniform
//    quantisation error over a cell of the whitened residual, kappa_D = E[max_i z_i^2]);
//  * bytes = layers * (2 (T r_t + D r_d + H r_t r_d) + [b > 0] H T (D b / 8 + 2));
//  * per budget pool, lambda is bisected geometrically on [1e-30, 1e30] * (energy / budget)
//    until hi / lo <= 1 + 1e-15; each unit takes argmin err + lambda * bytes with ties broken
//    by fewer bytes, then smaller (b, r_t, r_d); the feasible choice at `hi` is kept.
// The arithmetic uses explicit round-to-nearest double operations (no fused multiply-add),
// so the same table gives the same allocation as a plain float64 restatement.
#include "../jolt_internal.h"

namespace jolt {
namespace {

// One CTA per layer-tensor; thread (I, J) sums the squared core over block rows
// [I*step, (I+1)*step) and columns [J*step, (J+1)*step) in a fixed order.
__global__ void k_energy_table(int H, int R, int D, int step, const float* Gmax, const double* xx,
                               double* E, int ngrid, const int32_t* lt_ids) {
  extern __shared__ double sb[];  // [R/step][D/step] block sums, then prefix sums
  const int lt = blockIdx.x;
  const int nI = R / step, nJ = D / step;
  const float* g = Gmax + (int64_t)lt * H * R * D;
  for (int blk = threadIdx.x; blk < nI * nJ; blk += blockDim.x) {
    const int I = blk / nJ, J = blk % nJ;
    double acc = 0.0;
    for (int h = 0; h < H; ++h)
      for (int i = I * step; i < (I + 1) * step; ++i)
        for (int j = J * step; j < (J + 1) * step; ++j) {
          const double v = (double)g[((int64_t)h * R + i) * D + j];
          acc += v * v;
        }
    sb[blk] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const double x2 = xx[lt];
    double* e = E + (int64_t)lt_ids[lt] * ngrid;
    e[0] = x2;
    // prefix over J within each row block, then over I
    for (int I = 0; I < nI; ++I)
      for (int J = 1; J < nJ; ++J) sb[I * nJ + J] += sb[I * nJ + J - 1];
    for (int I = 1; I < nI; ++I)
      for (int J = 0; J < nJ; ++J) sb[I * nJ + J] += sb[(I - 1) * nJ + J];
    for (int I = 0; I < nI; ++I)
      for (int J = 0; J < nJ; ++J) {
        const double r = x2 - sb[I * nJ + J];
        e[1 + I * nJ + J] = r > 0.0 ? r : 0.0;
      }
  }
}

// The same table for the default grid (step 16, D = 128): warp w sums row block I = w % 8 over
// the heads h = w / 8, w / 8 + 4, .. (four head groups, 32 warps: four times the loads in
// flight) and its 16 rows with coalesced float4 loads (lane l holds columns 4l .. 4l + 3, so the
// 4 lanes 4J .. 4J + 3 cover column block J), in float64; the four head groups are then added in
// a fixed order.
constexpr int kEtGroups = 4;
__global__ void __launch_bounds__(256 * kEtGroups) k_energy_table16(int H, int R, const float* Gmax, const double* xx,
                                                                    double* E, int ngrid, const int32_t* lt_ids) {
  constexpr int D = kD, step = 16, nJ = D / step;
  __shared__ double sp[kEtGroups][(kMaxN / step) * nJ];
  __shared__ double sb[(kMaxN / step) * nJ];
  const int lt = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nI = R / step, I = warp & 7, hg = warp >> 3;
  const float* g = Gmax + (int64_t)lt * H * R * D;
  if (I < nI) {
    double acc = 0.0;
    for (int h = hg; h < H; h += kEtGroups) {
      const float4* row = reinterpret_cast<const float4*>(g + ((int64_t)h * R + I * step) * D) + lane;
#pragma unroll 4
      for (int i = 0; i < step; ++i) {
        const float4 v = row[i * (D / 4)];
        acc += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if ((lane & 3) == 0) sp[hg][I * nJ + (lane >> 2)] = acc;
  }
  __syncthreads();
  if (threadIdx.x < nI * nJ) {
    double t = 0.0;
#pragma unroll
    for (int q = 0; q < kEtGroups; ++q) t += sp[q][threadIdx.x];
    sb[threadIdx.x] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const double x2 = xx[lt];
    double* e = E + (int64_t)lt_ids[lt] * ngrid;
    e[0] = x2;
    for (int I = 0; I < nI; ++I)
      for (int J = 1; J < nJ; ++J) sb[I * nJ + J] += sb[I * nJ + J - 1];
    for (int I = 1; I < nI; ++I)
      for (int J = 0; J < nJ; ++J) sb[I * nJ + J] += sb[(I - 1) * nJ + J];
    for (int I = 0; I < nI; ++I)
      for (int J = 0; J < nJ; ++J) {
        const double r = x2 - sb[I * nJ + J];
        e[1 + I * nJ + J] = r > 0.0 ? r : 0.0;
      }
  }
}

__device__ __forceinline__ int64_t lt_bytes(int H, int T, int D, int rt, int rd, int b) {
  const int64_t tucker = 2 * ((int64_t)T * rt + (int64_t)D * rd + (int64_t)H * rt * rd);
  const int64_t resid = b > 0 ? (int64_t)H * T * (D * b / 8 + 2) : 0;
  return tucker + resid;
}

__device__ __forceinline__ void grid_rank(int gi, int step, int D, int& rt, int& rd) {
  if (gi == 0) { rt = 0; rd = 0; return; }
  const int nJ = D / step;
  rt = ((gi - 1) / nJ + 1) * step;
  rd = ((gi - 1) % nJ + 1) * step;
}

constexpr int kMaxUnits = 2 * kMaxGroups;

// Unit tables: err[u][b][grid] = (sum over the group's layers, in increasing layer order, of
// E_lt[grid]) * phi(b), for u = 2 g + kind.
__global__ void k_unit_tables(DualArgs a) {
  const int ncand = a.nbits * a.ngrid;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < a.G * 2 * a.ngrid; e += gridDim.x * blockDim.x) {
    const int u = e / a.ngrid, gi = e % a.ngrid;
    const int g = u / 2, k = u % 2;
    if (k == 1 && !a.has_v) continue;
    const int l0 = (int)(((int64_t)g * a.L) / a.G), l1 = (int)(((int64_t)(g + 1) * a.L) / a.G);
    double s = 0.0;
    for (int l = l0; l < l1; ++l) s = __dadd_rn(s, a.E[(int64_t)(2 * l + k) * a.ngrid + gi]);
    for (int bi = 0; bi < a.nbits; ++bi)
      a.unit_err[(int64_t)u * ncand + bi * a.ngrid + gi] = __dmul_rn(s, a.phi[bi]);
  }
}

// Measured-b refinement. meas_lt[i][b] = sum over (head, chunk), in order, of the residual
// coder's per-CTA sums; then one thread per (unit, allowed width): the unit's error for that
// width is the sum over its layers (increasing layer order) of meas_lt, entered at the grid
// point of the unit's chosen ranks (meta->alloc); every other grid point takes +inf, so the
// second dual re-chooses b only.
__global__ void k_meas_lt(int n_lt, int H, int nchunk, const double* meas_part, double* meas_lt) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_lt * 9; e += gridDim.x * blockDim.x) {
    const int i = e / 9, b = e % 9;
    double s = 0.0;
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < nchunk; ++c) s += meas_part[(((int64_t)i * H + h) * nchunk + c) * 9 + b];
    meas_lt[e] = s;
  }
}

__global__ void k_meas_units(DualArgs a, const double* meas_lt) {
  const int ncand = a.nbits * a.ngrid;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < a.G * 2 * a.nbits; e += gridDim.x * blockDim.x) {
    const int u = e / a.nbits, bi = e % a.nbits;
    const int g = u / 2, k = u % 2;
    if (k == 1 && !a.has_v) continue;
    const int l0 = (int)(((int64_t)g * a.L) / a.G), l1 = (int)(((int64_t)(g + 1) * a.L) / a.G);
    double s = 0.0;
    for (int l = l0; l < l1; ++l) s += meas_lt[(int64_t)(k * a.L + l) * 9 + a.bits[bi]];   // position of lt = 2 l + k
    const int rt = a.meta->alloc[g][k][0], rd = a.meta->alloc[g][k][1];
    for (int gi = 0; gi < a.ngrid; ++gi) {
      int r1, r2;
      grid_rank(gi, a.step, a.D, r1, r2);
      a.unit_err[(int64_t)u * ncand + bi * a.ngrid + gi] = (r1 == rt && r2 == rd) ? s : __longlong_as_double(0x7ff0000000000000LL);
    }
  }
}

constexpr size_t kDualSmem = 160 * 1024;

// One CTA per budget pool. The candidates come ranked by the tie-break key (bytes, b, r_t,
// r_d), so a unit's choice at lambda is the smallest (cost, rank): each warp scans one unit's
// candidates. The geometric bisection of lambda is evaluated three steps at a time: the seven
// midpoints the next three steps can visit (a binary tree of intervals) are computed exactly as
// the sequential search computes them and evaluated in parallel, then every thread walks the
// tree with the sequential rule (termination test and step cap included). The result is
// bit-identical to one bisection step per barrier, with a third of the barriers.
constexpr int kTreeNodes = 7;      // three bisection levels

__global__ void __launch_bounds__(1024) k_dual_pool(DualArgs a) {
  extern __shared__ unsigned char dsm[];
  __shared__ int slot_unit[kMaxUnits];
  __shared__ int slot_nlay[kMaxUnits];
  __shared__ int schoice[2][kTreeNodes][kMaxUnits];
  __shared__ int nslot_s;
  __shared__ double esum_s;
  const int pool = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = (int)(blockDim.x >> 5);
  const int nu = a.G * 2;
  const int ncand = a.nbits * a.ngrid;
  const int npools = (a.has_v && a.split) ? 2 : 1;
  StreamMeta* meta = a.meta;
  // shared: rank -> bytes per layer (int64 and float64) and attributes, then the cached errors
  int64_t* cb = reinterpret_cast<int64_t*>(dsm);                     // [ncand] by rank
  double* cbd = reinterpret_cast<double*>(cb + ncand);               // [ncand] by rank
  int* cattr = reinterpret_cast<int*>(cbd + ncand);                  // [ncand] b | rt << 8 | rd << 20
  int* rank_of = cattr + ncand;                                      // [ncand] candidate -> rank
  int* cand_of = rank_of + ncand;                                    // [ncand] rank -> candidate
  double* err_s = reinterpret_cast<double*>(cand_of + ncand + (ncand & 1));   // [nslot][ncand] by rank
  if (tid == 0) {
    int ns = 0;
    for (int u = 0; u < nu; ++u) {
      const int k = u % 2;
      if (k == 1 && !a.has_v) continue;
      if (npools == 2 && k != pool) continue;
      slot_unit[ns] = u;
      const int g = u / 2;
      slot_nlay[ns] = (int)(((int64_t)(g + 1) * a.L) / a.G - ((int64_t)g * a.L) / a.G);
      ++ns;
    }
    nslot_s = ns;
    // sum of the pool's unit energies E(0, 0), each summed over its layers in order
    double esum = 0.0;
    for (int i = 0; i < ns; ++i) {
      const int u = slot_unit[i], g = u / 2, k = u % 2;
      const int l0 = (int)(((int64_t)g * a.L) / a.G), l1 = (int)(((int64_t)(g + 1) * a.L) / a.G);
      double s = 0.0;
      for (int l = l0; l < l1; ++l) s = __dadd_rn(s, a.E[(int64_t)(2 * l + k) * a.ngrid]);
      esum = __dadd_rn(esum, s);
    }
    esum_s = esum;
  }
  // candidates in tie-break order (ranked on the host when the plan was made)
  for (int r = tid; r < ncand; r += blockDim.x) {
    const int c = a.cand_order[r];
    int rt, rd;
    grid_rank(c % a.ngrid, a.step, a.D, rt, rd);
    const int b = a.bits[c / a.ngrid];
    const int64_t by = lt_bytes(a.H, a.T, a.D, rt, rd, b);
    rank_of[c] = r;
    cand_of[r] = c;
    cb[r] = by;
    cbd[r] = (double)by;
    cattr[r] = b | (rt << 8) | (rd << 20);
  }
  __syncthreads();
  const int nslot = nslot_s;
  const size_t err_cap = (kDualSmem - (size_t)ncand * 32 - 16) / 8;
  const bool cached = (size_t)nslot * ncand <= err_cap;
  if (cached)
    for (int e = tid; e < nslot * ncand; e += blockDim.x) {
      const int us = e / ncand, c = e % ncand;
      err_s[(size_t)us * ncand + rank_of[c]] = a.unit_err[(int64_t)slot_unit[us] * ncand + c];
    }
  __syncthreads();
  const int64_t budget = a.budget_pool[pool];
  // rank of the smallest (cost, rank) of slot us at lam; warp-collective, every lane returns it
  auto choose_rank = [&](double lam, int us) -> int {
    const double nl = (double)slot_nlay[us];
    const double* ep = err_s + (size_t)us * ncand;
    const double* eg = a.unit_err + (int64_t)slot_unit[us] * ncand;
    double best = 0.0;
    int bi = -1;
    for (int r = lane; r < ncand; r += 32) {
      const double e = cached ? ep[r] : eg[cand_of[r]];
      const double cost = __dadd_rn(e, __dmul_rn(lam, __dmul_rn(nl, cbd[r])));
      if (bi < 0 || cost < best) {
        best = cost;
        bi = r;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const double oc = __shfl_xor_sync(0xffffffffu, best, o);
      const int ob = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob >= 0 && (bi < 0 || oc < best || (oc == best && ob < bi))) {
        best = oc;
        bi = ob;
      }
    }
    return bi;
  };
  // choices of every slot at lams[0 .. nn) into buffer buf; the caller synchronises
  auto evaluate = [&](const double* lams, int nn, int buf) {
    for (int item = warp; item < nn * nslot; item += nwarps) {
      const int node = item / nslot, us = item - node * nslot;
      const int r = choose_rank(lams[node], us);
      if (lane == 0) schoice[buf][node][us] = r;
    }
  };
  auto total = [&](int buf, int node) {
    int64_t tb = 0;
    for (int us = 0; us < nslot; ++us) tb += (int64_t)slot_nlay[us] * cb[schoice[buf][node][us]];
    return tb;
  };
  int buf = 0;
  double lam = 0.0;
  bool use_min = false;
  int64_t minb = 0;
  for (int us = 0; us < nslot; ++us) minb += (int64_t)slot_nlay[us] * cb[0];
  if (minb > budget) {
    if (tid == 0) atomicOr(&meta->status, ST_INFEASIBLE);
    use_min = true;                       // keep the minimum-bytes choice
  } else {
    const double zero[1] = {0.0};
    evaluate(zero, 1, buf);
    __syncthreads();
    if (total(buf, 0) > budget) {
      const double scale = __ddiv_rn(esum_s, (double)budget);
      double lo = __dmul_rn(1e-30, scale), hi = __dmul_rn(1e30, scale);
      int it = 0;
      bool done = false;
      while (!done) {
        // the midpoints of the next three steps: node i has interval [nlo, nhi]; its left
        // child follows a feasible midpoint ([nlo, mid]), its right child an infeasible one
        double nlo[kTreeNodes], nhi[kTreeNodes], mid[kTreeNodes];
        nlo[0] = lo;
        nhi[0] = hi;
#pragma unroll
        for (int i = 0; i < kTreeNodes; ++i) {
          mid[i] = __dsqrt_rn(__dmul_rn(nlo[i], nhi[i]));
          if (2 * i + 2 < kTreeNodes) {
            nlo[2 * i + 1] = nlo[i];
            nhi[2 * i + 1] = mid[i];
            nlo[2 * i + 2] = mid[i];
            nhi[2 * i + 2] = nhi[i];
          }
        }
        buf ^= 1;
        evaluate(mid, kTreeNodes, buf);
        __syncthreads();
        int node = 0;
        for (int lvl = 0; lvl < 3; ++lvl) {
          if (it >= 200 || !(__ddiv_rn(hi, lo) > 1.0 + 1e-15)) {
            done = true;
            break;
          }
          const bool feas = total(buf, node) <= budget;
          if (feas) hi = mid[node];
          else lo = mid[node];
          ++it;
          node = feas ? 2 * node + 1 : 2 * node + 2;
        }
      }
      lam = hi;
      buf ^= 1;
      const double at_hi[1] = {hi};
      evaluate(at_hi, 1, buf);
      __syncthreads();
    }
  }
  if (tid == 0) {
    meta->lambda[pool] = lam;
    for (int us = 0; us < nslot; ++us) {
      const int u = slot_unit[us];
      const int at = cattr[use_min ? 0 : schoice[buf][0][us]];
      meta->alloc[u / 2][u % 2][0] = (at >> 8) & 0xFFF;
      meta->alloc[u / 2][u % 2][1] = at >> 20;
      meta->alloc[u / 2][u % 2][2] = at & 0xFF;
    }
  }
}

// Layout of the body: lt-major (layer, then kind), parts U_T, U_D, G, scales, codes, each
// starting at a 256-byte boundary. A layer-tensor's parts occupy the sum of their sizes rounded
// up to 256 bytes, so the offsets follow from one exclusive prefix sum over the layer-tensors
// (one thread per layer-tensor, launched with kMaxLT threads).
__global__ void __launch_bounds__(kMaxLT) k_layout(DualArgs a) {
  __shared__ int64_t foot[kMaxLT];
  __shared__ unsigned long long bp[JOLT_NUM_PARTS];
  StreamMeta* meta = a.meta;
  const int kinds = a.has_v ? 2 : 1, nlt = a.L * kinds, t = threadIdx.x;
  if (t < JOLT_NUM_PARTS) bp[t] = 0;
  int64_t sz[JOLT_NUM_PARTS] = {0, 0, 0, 0, 0};
  int64_t f = 0;
  int lt = 0;
  if (t < nlt) {
    const int l = t / kinds, k = t % kinds;
    lt = 2 * l + k;
    int g = 0;
    while (g + 1 < a.G && ((int64_t)(g + 1) * a.L) / a.G <= l) ++g;
    const int rt = meta->alloc[g][k][0], rd = meta->alloc[g][k][1], b = meta->alloc[g][k][2];
    meta->lt_rank[lt][0] = rt;
    meta->lt_rank[lt][1] = rd;
    meta->lt_rank[lt][2] = b;
    sz[0] = (int64_t)a.T * rt * 2;
    sz[1] = (int64_t)a.D * rd * 2;
    sz[2] = (int64_t)a.H * rt * rd * 2;
    sz[3] = b > 0 ? (int64_t)a.H * a.T * 2 : 0;
    sz[4] = b > 0 ? (int64_t)a.H * a.T * (a.D * b / 8) : 0;
    for (int p = 0; p < JOLT_NUM_PARTS; ++p) f += (sz[p] + kAlign - 1) / kAlign * kAlign;
  }
  foot[t] = f;
  __syncthreads();
  // inclusive scan of the footprints (Hillis-Steele, fixed order of additions)
  for (int o = 1; o < kMaxLT; o <<= 1) {
    const int64_t v = t >= o ? foot[t - o] : 0;
    __syncthreads();
    foot[t] += v;
    __syncthreads();
  }
  if (t < nlt) {
    int64_t cur = t > 0 ? foot[t - 1] : 0;          // 256-aligned start of this layer-tensor
    for (int p = 0; p < JOLT_NUM_PARTS; ++p) {
      meta->off[lt][p] = cur;
      atomicAdd(&bp[p], (unsigned long long)sz[p]);
      cur += (sz[p] + kAlign - 1) / kAlign * kAlign;
    }
    if (t == nlt - 1) meta->body_bytes = cur - (sz[4] + kAlign - 1) / kAlign * kAlign + sz[4];
  }
  __syncthreads();
  if (t < JOLT_NUM_PARTS) meta->bytes_by_part[t] = (int64_t)bp[t];
}

// Copy the chosen leading blocks of the factors and the bf16-rounded core into the body.
__global__ void k_pack_factors(PackArgs a) {
  const int i = blockIdx.y;            // index into lt_ids
  const int lt = a.lt_ids[i];
  const StreamMeta* m = a.meta;
  const int rt = m->lt_rank[lt][0], rd = m->lt_rank[lt][1];
  __nv_bfloat16* ut = reinterpret_cast<__nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UT]);
  __nv_bfloat16* ud = reinterpret_cast<__nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_UD]);
  __nv_bfloat16* gg = reinterpret_cast<__nv_bfloat16*>(a.body + m->off[lt][JOLT_PART_G]);
  const __nv_bfloat16* UT = a.UT + (int64_t)i * a.T * a.R;
  const __nv_bfloat16* UD = a.UD + (int64_t)i * a.D * a.D;
  const float* Gm = a.Gmax + (int64_t)i * a.H * a.R * a.D;
  const int64_t n_ut = (int64_t)a.T * rt, n_ud = (int64_t)a.D * rd, n_g = (int64_t)a.H * rt * rd;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n_ut + n_ud + n_g; e += stride) {
    if (e < n_ut) {
      const int64_t t = e / rt, c = e % rt;
      ut[e] = UT[t * a.R + c];
    } else if (e < n_ut + n_ud) {
      const int64_t f = e - n_ut;
      const int64_t d = f / rd, c = f % rd;
      ud[f] = UD[d * a.D + c];
    } else {
      const int64_t f = e - n_ut - n_ud;
      const int64_t h = f / ((int64_t)rt * rd), r = f % ((int64_t)rt * rd);
      const int64_t ii = r / rd, j = r % rd;
      gg[f] = __float2bfloat16_rn(Gm[(h * a.R + ii) * a.D + j]);
    }
  }
}

}  // namespace

cudaError_t energy_table(const TableArgs& a, cudaStream_t s) {
  if (a.step == 16 && a.D == kD && a.R <= kMaxN) {
    k_energy_table16<<<a.n_lt, 256 * kEtGroups, 0, s>>>(a.H, a.R, a.Gmax, a.xx, a.E, a.ngrid, a.lt_ids);
    note_launch();
    return cudaGetLastError();
  }
  const size_t smem = (size_t)(a.R / a.step) * (a.D / a.step) * sizeof(double) + sizeof(double);
  k_energy_table<<<a.n_lt, 128, smem, s>>>(a.H, a.R, a.D, a.step, a.Gmax, a.xx, a.E, a.ngrid,
                                           a.lt_ids);
  note_launch();
  return cudaGetLastError();
}

cudaError_t dual_allocate(const DualArgs& a, cudaStream_t s) {
  if (a.G > kMaxGroups || a.L > kMaxL) return cudaErrorInvalidValue;
  const int units = a.G * 2 * a.ngrid;
  if (!a.tables_ready) {
    k_unit_tables<<<(units + 255) / 256, 256, 0, s>>>(a);
    note_launch();
  }
  cudaError_t e = cudaFuncSetAttribute(k_dual_pool, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDualSmem);
  if (e != cudaSuccess) return e;
  const int npools = (a.has_v && a.split) ? 2 : 1;
  const int slots = a.has_v && !a.split ? 2 * a.G : a.G;
  const int items = slots * kTreeNodes;
  const int threads = 32 * (items < 32 ? items : 32);
  k_dual_pool<<<npools, threads, kDualSmem, s>>>(a);
  note_launch();
  k_layout<<<1, kMaxLT, 0, s>>>(a);
  note_launch();
  return cudaGetLastError();
}

cudaError_t measured_tables(const DualArgs& a, const double* meas_part, int nchunk, double* meas_lt,
                            cudaStream_t s) {
  const int n_lt = a.L * (a.has_v ? 2 : 1);
  k_meas_lt<<<(n_lt * 9 + 255) / 256, 256, 0, s>>>(n_lt, a.H, nchunk, meas_part, meas_lt);
  note_launch();
  k_meas_units<<<1, 256, 0, s>>>(a, meas_lt);
  note_launch();
  return cudaGetLastError();
}

cudaError_t pack_factors(const PackArgs& a, cudaStream_t s) {
  k_pack_factors<<<dim3(64, a.n_lt), 256, 0, s>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace jolt
