"""JoLT encode / decode, restated step by step in float64 (oracle).

Test infrastructure only; see oracle/__init__.py for the sources. Step numbers below
follow the method's stage order on the pages: partial Tucker over (tokens, features)
-> rotated low-bit residual -> one Lagrangian dual over ranks and bit-widths.

Notation: one layer-tensor X in R^{H x T x D} (heads x tokens x features). The token
unfolding A = X_(2) in R^{T x HD} has A[t, h*D + d] = X[h, t, d]. U_T (T x r_t) and
U_D (D x r_d) are shared by all heads; the core is G[h] = U_T^T X_h U_D (H x r_t x r_d).

Readings taken where the pages are silent:
* truncated HOSVD: each factor comes from the Gram of the original tensor, no HOOI sweeps;
  factors are computed once at the largest candidate rank and truncated to leading
  columns, so every candidate core is a leading block of one core G_max;
* FlashJoLT = randomized subspace iteration (Halko, Martinsson & Tropp 2011, Alg. 4.4)
  on A with a bf16 Gaussian sketch of l = R + p columns and q power iterations, then the
  small eigenproblem of B B^T with B = Q^T A;
* each factor column is signed so that its entry of largest magnitude (lowest index on
  a tie) is positive;
* residual quantiser: per row y in R^D, s = fp16(max |y_i|); code
  c_i = clamp(floor(y_i 2^(b-1) / s + 2^(b-1)), 0, 2^b - 1); value s (2 c_i + 1 - 2^b) / 2^b
  (mid-rise, 2^b cells over [-s, s]); codes packed LSB-first into a little-endian bit
  stream of D*b/8 bytes per row;
* error model for the dual: exact truncation energy E(r_t, r_d) = ||X||^2 - ||G_lead||^2
  times phi(b), with phi(0) = 1 and phi(b) = kappa_D / (3 * 4^b), kappa_D = E[max_i z_i^2]
  for z ~ N(0, I_D): the whitened residual's quantisation error is treated as uniform
  over a cell (the news summary describes the rotated residual as nearly independent and
  uniformly distributed within a cell);
* bytes per layer-tensor = 2 (T r_t + D r_d + H r_t r_d) + [b > 0] H T (D b / 8 + 2).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from .numerics import (round_bf16, round_fp16_sat, round_f32, haar_rotation, rotation_matrix,
                       sketch_matrix)

RANK_STEP = 16
# Largest token rank on the grid of the randomized-SVD encoder. The pages fix no grid; the reading
# taken: ranks run to min(T, HD, budget per layer-tensor / (2T)) (a larger token factor alone
# would exceed the layer-tensor's share of the budget), and the FlashJoLT sketch, which exists for
# long contexts, stops at 256 columns before oversampling. The exact encoder has no extra cap.
SKETCH_RT_CAP = 256
OVERSAMPLE = 16
POWER_ITERS = 1
KINDS = 2          # layer-tensor index lt = layer * 2 + kind (kind 0 = K, 1 = V)


# ============================================================================ shapes / grid
def group_ranges(L: int, G: int):
    """Contiguous layer groups: group g holds layers [g L / G, (g + 1) L / G) (integer division)."""
    return [range(g * L // G, (g + 1) * L // G) for g in range(G)]


def layer_bytes(H: int, T: int, D: int, rt: int, rd: int, b: int) -> int:
    """Bytes one layer-tensor stores: bf16 U_T, U_D, core; b-bit codes + fp16 scale per row."""
    tucker = 2 * (T * rt + D * rd + H * rt * rd)
    resid = H * T * (D * b // 8 + 2) if b > 0 else 0
    return tucker + resid


def rt_max(H: int, T: int, D: int, budget_per_lt: int, step: int, cap: int | None) -> int:
    """Largest token rank on the grid: min(T, HD, budget / (2T), cap), rounded down to `step`
    (`cap` None: no cap beyond the first three)."""
    r = min(T, H * D, budget_per_lt // (2 * T))
    if cap is not None:
        r = min(r, cap)
    return max(0, r - r % step)


def rank_grid(R: int, D: int, step: int):
    """Candidate (r_t, r_d): (0, 0) plus every multiple of `step` up to (R, D); r_t = 0 iff r_d = 0."""
    g = [(0, 0)]
    for rt in range(step, R + 1, step):
        for rd in range(step, D + 1, step):
            g.append((rt, rd))
    return g


def kappa(D: int) -> float:
    """kappa_D = E[max_{i<D} z_i^2], z ~ N(0, I_D) = int_0^inf 2y (1 - erf(y/sqrt 2)^D) dy.

    Composite Gauss-Legendre quadrature on [0, 40]; 1 - erf^D is evaluated as
    -expm1(D log1p(-erfc(y / sqrt 2))) to keep the tail accurate.
    """
    xg, wg = np.polynomial.legendre.leggauss(20)
    edges = np.linspace(0.0, 40.0, 801)
    total = 0.0
    erfc = np.vectorize(math.erfc)
    for a, bnd in zip(edges[:-1], edges[1:]):
        y = 0.5 * (bnd - a) * xg + 0.5 * (bnd + a)
        e = erfc(y / math.sqrt(2.0))
        f = 2.0 * y * (-np.expm1(D * np.log1p(-e)))
        total += 0.5 * (bnd - a) * float(np.dot(wg, f))
    return total


def phi(b: int, kap: float) -> float:
    """Fraction of residual energy left after b-bit quantisation (1 when b = 0)."""
    return 1.0 if b == 0 else kap / (3.0 * 4.0 ** b)


# ============================================================================ factors
def token_unfolding(X):
    H, T, D = X.shape
    return X.transpose(1, 0, 2).reshape(T, H * D)


def feature_gram(X):
    """C_D = sum_h X_h^T X_h (D x D)."""
    H, T, D = X.shape
    Xf = X.reshape(H * T, D)
    return Xf.T @ Xf


def token_gram(X):
    """C_T = sum_h X_h X_h^T (T x T) = A A^T."""
    A = token_unfolding(X)
    return A @ A.T


def eig_desc(C):
    """Eigenpairs of a symmetric matrix, eigenvalues descending."""
    w, V = np.linalg.eigh(C)
    return w[::-1].copy(), V[:, ::-1].copy()


def column_signs(U):
    """+1 / -1 per column so that the column's largest-magnitude entry becomes positive."""
    idx = np.argmax(np.abs(U), axis=0)               # first index on ties
    v = U[idx, np.arange(U.shape[1])]
    return np.where(v < 0, -1.0, 1.0)


def qr_q(Y):
    """Orthonormal basis (reduced Householder QR) of the columns of Y."""
    Q, _ = np.linalg.qr(Y)
    return Q


def exact_token_factor(X, R: int):
    """Leading R eigenvectors of the token Gram (exact HOSVD), unsigned."""
    w, V = eig_desc(token_gram(X))
    return V[:, :R], w


def feature_factor(X):
    """All D eigenvectors of the feature Gram, unsigned."""
    w, V = eig_desc(feature_gram(X))
    return V, w


def sketch_size(R: int, p: int, T: int, HD: int) -> int:
    return min(R + p, T, HD)


def sketch_token_factor(X, R: int, p: int, q: int, seed: int, lt: int):
    """FlashJoLT token factor by randomized subspace iteration.

    Q0 = orth(A Omega); q times: Q = orth(A orth(A^T Q)); B = Q^T A; B B^T = W Lambda W^T;
    U_T = Q W[:, :R]. Returns (U_T, W_R, B, Q, eigenvalues of B B^T).
    """
    A = token_unfolding(X)
    T, HD = A.shape
    l = sketch_size(R, p, T, HD)
    Om = sketch_matrix(seed, lt, HD, l)
    Q = qr_q(A @ Om)
    for _ in range(q):
        Q = qr_q(A.T @ Q)
        Q = qr_q(A @ Q)
    B = Q.T @ A
    w, W = eig_desc(B @ B.T)
    WR = W[:, :R]
    return Q @ WR, WR, B, Q, w


def core_exact(X, U_T, U_D):
    """G[h] = U_T^T X_h U_D."""
    return np.einsum("tr,htd,de->hre", U_T, X, U_D, optimize=True)


def core_sketch(B, WR, U_D, H: int, D: int):
    """G[h] = W_R^T B_h U_D with B_h = B[:, hD:(h+1)D]; equals U_T^T X_h U_D when U_T = Q W_R."""
    l = B.shape[0]
    Bh = B.reshape(l, H, D)
    return np.einsum("lr,lhd,de->hre", WR, Bh, U_D, optimize=True)


# ============================================================================ residual codec
def quantize_rows(Y, b: int, spec: bool = True):
    """Per-row absmax scale and b-bit codes of rows Y[..., D]. Returns (s, codes, dist).

    `dist` is each entry's distance to the nearest cell boundary, in units of the row
    scale (|y - boundary| / s), for the boundary-case accounting of parity tests.
    """
    m = np.abs(Y).max(axis=-1)
    s = round_fp16_sat(m) if spec else m.copy()
    half = 2.0 ** (b - 1)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = (Y * half) / s[..., None] + half
    c = np.floor(u)
    nearest = np.clip(np.round(u), 1, 2 ** b - 1)       # interior cell boundaries 1 .. 2^b - 1
    dist = np.abs(u - nearest) / half
    c = np.clip(c, 0, 2 ** b - 1)
    zero = ~(s > 0)
    c[zero] = 0
    dist[zero] = np.inf
    return s, c.astype(np.int64), dist


def dequantize_rows(s, codes, b: int):
    """Row values s (2 c + 1 - 2^b) / 2^b."""
    return s[..., None] * (2.0 * codes + 1.0 - 2.0 ** b) / (2.0 ** b)


def pack_codes(codes, b: int):
    """b-bit codes [..., D] -> bytes [..., D*b/8]; code i occupies bits [i b, i b + b), LSB first."""
    c = np.asarray(codes, dtype=np.int64)
    bits = ((c[..., :, None] >> np.arange(b)) & 1).astype(np.uint8)       # [..., D, b]
    bits = bits.reshape(*c.shape[:-1], c.shape[-1] * b)
    return np.packbits(bits, axis=-1, bitorder="little")


def unpack_codes(packed, b: int, D: int):
    bits = np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=-1, bitorder="little")
    bits = bits[..., : D * b].reshape(*packed.shape[:-1], D, b).astype(np.int64)
    return (bits << np.arange(b)).sum(-1)


def residual_rotated(X, U_T, G, U_D, Pi):
    """Y_h = (X_h - U_T G_h U_D^T) Pi, rows of every head (H x T x D)."""
    rec = np.einsum("tr,hre,de->htd", U_T, G, U_D, optimize=True) if U_T.shape[1] else 0.0
    return np.einsum("htd,de->hte", X - rec, Pi, optimize=True)


def tucker_part(U_T, G, U_D, H, T, D):
    if U_T.shape[1] == 0:
        return np.zeros((H, T, D))
    return np.einsum("tr,hre,de->htd", U_T, G, U_D, optimize=True)


# ============================================================================ dual
@dataclass
class Unit:
    """One (group, kind) allocation unit with its candidate table."""
    group: int
    kind: int
    err: np.ndarray        # float64 [n]
    nbytes: np.ndarray     # int64 [n]
    b: np.ndarray
    rt: np.ndarray
    rd: np.ndarray
    energy: float          # E(0, 0): the unit's total energy


def choose(unit: Unit, lam: float) -> int:
    """argmin err + lam * bytes; ties -> fewer bytes, then smaller (b, r_t, r_d)."""
    cost = unit.err + lam * unit.nbytes.astype(np.float64)
    order = np.lexsort((unit.rd, unit.rt, unit.b, unit.nbytes, cost))
    return int(order[0])


class BudgetInfeasible(ValueError):
    pass


def dual_allocate(units, budget: int, max_iter: int = 200):
    """Lagrangian dual over one budget pool: bisect lambda, each unit picks its argmin.

    If the smallest choices exceed the budget the pool is infeasible. If lambda = 0 fits,
    it is the answer. Otherwise lambda is bisected geometrically on
    [1e-30, 1e30] * (sum of unit energies / budget) until hi / lo <= 1 + 1e-15 (or
    `max_iter` steps) and the (feasible) choice at `hi` is returned with lambda = hi.
    Returns (list of candidate indices, lambda).
    """
    minb = sum(int(u.nbytes.min()) for u in units)
    if minb > budget:
        raise BudgetInfeasible(f"minimum bytes {minb} exceed budget {budget}")

    def total(lam):
        idx = [choose(u, lam) for u in units]
        return idx, sum(int(u.nbytes[i]) for u, i in zip(units, idx))

    idx, tb = total(0.0)
    if tb <= budget:
        return idx, 0.0
    esum = 0.0
    for u in units:
        esum = esum + u.energy
    scale = esum / float(budget)
    lo, hi = 1e-30 * scale, 1e30 * scale
    for _ in range(max_iter):
        if not (hi / lo > 1.0 + 1e-15):
            break
        mid = math.sqrt(lo * hi)
        _, tb = total(mid)
        if tb <= budget:
            hi = mid
        else:
            lo = mid
    idx, tb = total(hi)
    assert tb <= budget
    return idx, hi


# ============================================================================ encode / decode
@dataclass
class LTCode:
    """What the stream stores for one layer-tensor (float64 arrays on their storage grids)."""
    rt: int
    rd: int
    b: int
    U_T: np.ndarray        # T x rt
    U_D: np.ndarray        # D x rd
    G: np.ndarray          # H x rt x rd
    scales: np.ndarray     # H x T   (empty when b == 0)
    codes: np.ndarray      # H x T x D ints (empty when b == 0)


@dataclass
class OracleStream:
    L: int
    H: int
    T: int
    D: int
    has_v: bool
    num_groups: int
    seed: int
    encoder: str
    rank_step: int
    rt_max: int
    split_kv: bool
    out_f32: bool
    alloc: np.ndarray                  # [G][2][3] (r_t, r_d, b)
    lts: dict = field(default_factory=dict)
    rotation: str = "haar"             # "haar" or "hadamard"

    def kinds(self):
        return (0, 1) if self.has_v else (0,)


@dataclass
class Plan:
    L: int
    H: int
    T: int
    D: int
    has_v: bool
    budget: int
    num_groups: int
    encoder: str = "exact"
    rank_step: int = RANK_STEP
    rt_cap: int | None = None  # None: the reading (SKETCH_RT_CAP for the sketch, none for exact)
    oversample: int = OVERSAMPLE
    power_iters: int = POWER_ITERS
    bits: tuple = tuple(range(9))
    split_kv: bool = False
    out_f32: bool = False
    measured_b: bool = False   # re-choose b per unit with measured quantisation errors
    rotation: str = "haar"     # "haar" or "hadamard" (randomized Hadamard, §8f-3 of the reading)

    def kinds(self):
        return (0, 1) if self.has_v else (0,)

    def n_lt(self):
        return self.L * len(self.kinds())

    def pools(self):
        """[(kinds in pool, pool budget)]."""
        if self.has_v and self.split_kv:
            bk = self.budget // 2
            return [((0,), bk), ((1,), self.budget - bk)]
        return [(self.kinds(), self.budget)]

    def cap(self):
        """Token-rank cap: an explicit `rt_cap`, else the reading's (256 for the sketch)."""
        if self.rt_cap is not None:
            return self.rt_cap
        return SKETCH_RT_CAP if self.encoder == "sketch" else None

    def R(self):
        return rt_max(self.H, self.T, self.D, self.budget // self.n_lt(), self.rank_step, self.cap())

    def grid(self):
        return rank_grid(self.R(), self.D, self.rank_step)


def analyse_layer_tensor(plan: Plan, X, seed: int, lt: int, spec: bool = True, factors=None):
    """Phase A for one layer-tensor: factors at the largest ranks, G_max, energy table.

    `factors` = (U_T, U_D) overrides the computed (already signed, rounded) factors; the
    core is then the exact projection U_T^T X_h U_D.
    """
    H, T, D = X.shape
    R = plan.R()
    info = {}
    if factors is not None:
        U_T, U_D = factors
        Gmax = core_exact(X, U_T, U_D)
    else:
        U_D, wD = feature_factor(X)
        sd = column_signs(U_D)
        U_D = U_D * sd
        if spec:
            U_D = round_bf16(U_D)
        info["wD"] = wD
        if R == 0:
            U_T = np.zeros((T, 0))
            Gmax = np.zeros((H, 0, D))
        elif plan.encoder == "exact":
            U_T, wT = exact_token_factor(X, R)
            st = column_signs(U_T)
            U_T = U_T * st
            info["U_T_unrounded"] = U_T.copy()
            if spec:
                U_T = round_bf16(U_T)
            Gmax = core_exact(X, U_T, U_D)
            info["wT"] = wT
        else:
            U_T, WR, B, Q, wB = sketch_token_factor(X, R, plan.oversample, plan.power_iters, seed, lt)
            st = column_signs(U_T)
            U_T = U_T * st
            WR = WR * st
            info["U_T_unrounded"] = U_T.copy()
            if spec:
                U_T = round_bf16(U_T)
            Gmax = core_sketch(B, WR, U_D, H, D)
            info["wT"] = wB
        info["U_D_unrounded_signs"] = sd
    xx = float((X * X).sum())
    S = (Gmax * Gmax).sum(axis=0)                     # R x D
    P = S.cumsum(axis=0).cumsum(axis=1) if S.size else S
    grid = plan.grid()
    E = np.empty(len(grid))
    for i, (rt, rd) in enumerate(grid):
        E[i] = xx if rt == 0 else max(0.0, xx - float(P[rt - 1, rd - 1]))
    return dict(U_T=U_T, U_D=U_D, Gmax=Gmax, E=E, xx=xx, **info)


def build_units(plan: Plan, E_lt: dict, kap: float):
    """Per (group, kind) candidate tables: err = sum over the group's layers of E * phi(b)."""
    grid = plan.grid()
    units = []
    for g, lay in enumerate(group_ranges(plan.L, plan.num_groups)):
        for k in plan.kinds():
            Eg = np.zeros(len(grid))
            for l in lay:
                Eg = Eg + E_lt[l * KINDS + k]
            err, nb, bb, rts, rds = [], [], [], [], []
            for b in plan.bits:
                ph = phi(b, kap)
                for i, (rt, rd) in enumerate(grid):
                    err.append(Eg[i] * ph)
                    nb.append(len(lay) * layer_bytes(plan.H, plan.T, plan.D, rt, rd, b))
                    bb.append(b)
                    rts.append(rt)
                    rds.append(rd)
            units.append(Unit(g, k, np.array(err), np.array(nb, dtype=np.int64), np.array(bb),
                              np.array(rts), np.array(rds), float(Eg[0])))
    return units


def allocate(plan: Plan, units):
    """Run the dual per pool; returns alloc [G][2][3] and the lambdas."""
    alloc = np.zeros((plan.num_groups, 2, 3), dtype=np.int64)
    lams = []
    for kinds, bud in plan.pools():
        us = [u for u in units if u.kind in kinds]
        idx, lam = dual_allocate(us, bud)
        lams.append(lam)
        for u, i in zip(us, idx):
            alloc[u.group, u.kind] = (u.rt[i], u.rd[i], u.b[i])
    return alloc, lams


def measure_b_errors(plan: Plan, tens: dict, A: dict, alloc, Pi, spec: bool = True):
    """Exact squared error of every allowed b at each unit's chosen ranks (the refinement of the
    phi(b) model, §8f-1 of the reading): with Y the rotated residual of the stored factors,
    ||Y||^2 for b = 0 and ||Y - dequant(quant_b(Y))||^2 for b > 0, summed over the unit's
    layers. Returns {(group, kind): {b: error}}."""
    meas = {}
    for g, lay in enumerate(group_ranges(plan.L, plan.num_groups)):
        for k in plan.kinds():
            rt, rd = int(alloc[g, k][0]), int(alloc[g, k][1])
            acc = {int(b): 0.0 for b in plan.bits}
            for l in lay:
                lt = l * KINDS + k
                a = A[lt]
                G = a["Gmax"][:, :rt, :rd]
                if spec:
                    G = round_bf16(G)
                Y = residual_rotated(tens[k][l], a["U_T"][:, :rt], G, a["U_D"][:, :rd], Pi)
                for b in plan.bits:
                    b = int(b)
                    if b == 0:
                        acc[b] += float(np.sum(Y * Y))
                    else:
                        s, c, _ = quantize_rows(Y, b, spec)
                        d = Y - dequantize_rows(s, c, b)
                        acc[b] += float(np.sum(d * d))
            meas[(g, k)] = acc
    return meas


def refine_b(plan: Plan, units, alloc, meas):
    """Second dual: every unit keeps the ranks of `alloc` and re-chooses b with the measured
    errors (candidates at other ranks take an infinite error, so they are never chosen; the
    bytes, tie-break and lambda search are those of the first dual). Returns (alloc, lambdas)."""
    units2 = []
    for u in units:
        rt, rd = int(alloc[u.group, u.kind][0]), int(alloc[u.group, u.kind][1])
        m = meas[(u.group, u.kind)]
        err = np.array([m[int(b)] if (int(r1) == rt and int(r2) == rd) else np.inf
                        for b, r1, r2 in zip(u.b, u.rt, u.rd)])
        units2.append(Unit(u.group, u.kind, err, u.nbytes, u.b, u.rt, u.rd, u.energy))
    return allocate(plan, units2)


def encode(plan: Plan, K, V, seed: int, spec: bool = True, alloc=None, factors=None,
           Pi=None, keep=False):
    """Full encode. K, V: [L][H][T][D] arrays (V may be None). Returns (OracleStream, debug).

    `alloc` forces the allocation ([G][2][3]); `factors` maps lt -> (U_T, U_D) at the
    largest ranks; `Pi` replaces the rotation (e.g. the GPU's float32 one).
    """
    tens = {0: np.asarray(K, dtype=np.float64)}
    if plan.has_v:
        tens[1] = np.asarray(V, dtype=np.float64)
    kap = kappa(plan.D)
    if Pi is None:
        Pi = rotation_matrix(seed, plan.D, plan.rotation)
    A = {}
    for l in range(plan.L):
        for k in plan.kinds():
            lt = l * KINDS + k
            f = factors.get(lt) if factors is not None else None
            A[lt] = analyse_layer_tensor(plan, tens[k][l], seed, lt, spec, f)
    units = build_units(plan, {lt: a["E"] for lt, a in A.items()}, kap)
    lams = None
    meas = None
    if alloc is None:
        alloc, lams = allocate(plan, units)
        if plan.measured_b:
            meas = measure_b_errors(plan, tens, A, alloc, Pi, spec)
            alloc, lams = refine_b(plan, units, alloc, meas)
    st = OracleStream(plan.L, plan.H, plan.T, plan.D, plan.has_v, plan.num_groups, seed,
                      plan.encoder, plan.rank_step, plan.R(), plan.split_kv, plan.out_f32,
                      np.asarray(alloc, dtype=np.int64), rotation=plan.rotation)
    for g, lay in enumerate(group_ranges(plan.L, plan.num_groups)):
        for l in lay:
            for k in plan.kinds():
                lt = l * KINDS + k
                rt, rd, b = (int(v) for v in alloc[g, k])
                a = A[lt]
                U_T = a["U_T"][:, :rt]
                U_D = a["U_D"][:, :rd]
                G = a["Gmax"][:, :rt, :rd]
                if spec:
                    G = round_bf16(G)
                X = tens[k][l]
                if b > 0:
                    Y = residual_rotated(X, U_T, G, U_D, Pi)
                    s, c, _ = quantize_rows(Y, b, spec)
                else:
                    s = np.zeros((plan.H, 0))
                    c = np.zeros((plan.H, plan.T, 0), dtype=np.int64)
                st.lts[lt] = LTCode(rt, rd, b, U_T, U_D, G, s, c)
    dbg = dict(analysis=A, units=units, lambdas=lams, kappa=kap, Pi=Pi, measured=meas)
    return st, dbg


def decode_lt(st: OracleStream, lt: int, Pi=None):
    """float64 reconstruction of one layer-tensor: G x2 U_T x3 U_D + dequant(codes) Pi^T."""
    c = st.lts[lt]
    if Pi is None:
        Pi = rotation_matrix(st.seed, st.D, st.rotation)
    Xh = tucker_part(c.U_T, c.G, c.U_D, st.H, st.T, st.D)
    if c.b > 0:
        Yh = dequantize_rows(c.scales, c.codes, c.b)
        Xh = Xh + np.einsum("hte,de->htd", Yh, Pi, optimize=True)
    return Xh


def round_output(Xh, out_f32: bool):
    return round_f32(Xh) if out_f32 else round_bf16(Xh)


def decode(st: OracleStream, Pi=None, rounded=True):
    """Whole cache: returns (K_hat, V_hat) as float64 [L][H][T][D] on the output grid."""
    if Pi is None:
        Pi = rotation_matrix(st.seed, st.D, st.rotation)
    outs = []
    for k in st.kinds():
        arr = np.stack([decode_lt(st, l * KINDS + k, Pi) for l in range(st.L)])
        outs.append(round_output(arr, st.out_f32) if rounded else arr)
    return outs[0], (outs[1] if st.has_v else None)


def rel_frob(X, Xh) -> float:
    """||X - X_hat||_F / ||X||_F in float64."""
    X = np.asarray(X, dtype=np.float64)
    Xh = np.asarray(Xh, dtype=np.float64)
    den = math.sqrt(float((X * X).sum()))
    return math.sqrt(float(((X - Xh) ** 2).sum())) / den if den > 0 else 0.0


def principal_angles(U1, U2):
    """Principal angles (radians) between the column spaces of U1 and U2."""
    Q1 = qr_q(U1)
    Q2 = qr_q(U2)
    s = np.linalg.svd(Q1.T @ Q2, compute_uv=False)
    return np.arccos(np.clip(s, -1.0, 1.0))
