"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, then
compare with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import copy
import numpy as np

import synth
from oracle import jolt as oj
from oracle import numerics as onum
from oracle import stream as ostream

ANGLE_TOL = 1e-3           # rad, leading subspace of the exact HOSVD factors
GAP_REL = 1e-4             # eigengap (relative to the top eigenvalue) that makes a column "leading"
# Token-rank cap given to both sides of every test plan: the library implements ranks up to 112,
# while the method's default grid reaches 256 (sketch) or the budget bound (exact) on these
# workloads; both the GPU plan (jolt_config.rt_max) and the oracle plan (rt_cap) get it explicitly.
RT_MAX = 112
REL_ERR_TOL = 0.01         # GPU relative Frobenius error within 1% (relative) of the oracle's
BOUNDARY_BAND = 1e-6       # codes may differ only within this distance (units of the row scale)


def to_torch(a: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda()


def decode_tol(ref: np.ndarray, out_f32: bool) -> np.ndarray:
    """max(1e-3, one output ulp at the oracle's value): bf16 output rounding alone reaches
    half an ulp, which exceeds 1e-3 once |x| >= 0.5."""
    if out_f32:
        return np.full(ref.shape, 1e-3)
    a = np.abs(ref)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    ulp = np.ldexp(1.0, (e - 7).astype(np.int64))
    return np.maximum(1e-3, ulp)


def oracle_plan(cfg, budget, encoder, groups=None, split=None, bits=None, **kw):
    kw.setdefault("rt_cap", RT_MAX)
    return oj.Plan(L=cfg.layers, H=cfg.heads, T=cfg.tokens, D=cfg.head_dim, has_v=cfg.has_v,
                   budget=budget, num_groups=groups or cfg.groups, encoder=encoder,
                   split_kv=cfg.split_kv if split is None else split,
                   bits=tuple(bits or cfg.bits), out_f32=(cfg.dtype == "f32"), **kw)


def gpu_encode(cfg, K, V, budget, encoder, seed=42, groups=None, split=None, bits=None):
    """Encode on the GPU through the C ABI. Returns (plan, stream, K_dev, V_dev)."""
    from tensor_decomposition_b200 import jolt as J
    c = J.jolt_config_default()
    c.encoder = J.JOLT_ENC_EXACT if encoder == "exact" else J.JOLT_ENC_SKETCH
    c.rt_max = RT_MAX
    c.split_kv_budget = int(cfg.split_kv if split is None else split)
    mask = 0
    for b in (bits or cfg.bits):
        mask |= 1 << b
    c.bits_mask = mask
    dt = J.JOLT_BF16 if cfg.dtype == "bf16" else J.JOLT_F32
    plan = J.jolt_plan(cfg.layers, cfg.heads, cfg.tokens, cfg.head_dim, cfg.has_v, dt, budget,
                       groups or cfg.groups, c)
    Kd = to_torch(K, cfg.dtype)
    Vd = to_torch(V, cfg.dtype) if cfg.has_v else None
    st = J.jolt_encode(plan, Kd, Vd, seed)
    J.jolt_stream_status(st)
    return plan, st, Kd, Vd


def gpu_decode(cfg, st, Kd, Vd):
    import torch
    from tensor_decomposition_b200 import jolt as J
    Ko = torch.empty_like(Kd)
    Vo = torch.empty_like(Vd) if Vd is not None else None
    J.jolt_decode(st, Ko, Vo)
    torch.cuda.synchronize()
    return Ko, Vo


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def leading_count(w, kmax):
    """Number of leading eigenvectors whose next relative eigengap is at least GAP_REL."""
    w = np.asarray(w, dtype=np.float64)
    k = 0
    for i in range(min(kmax, len(w) - 1)):
        if (w[i] - w[i + 1]) / w[0] < GAP_REL:
            break
        k = i + 1
    return k


def codes_parity(ost, Xs: dict, Pi_gpu: np.ndarray):
    """Re-code the GPU's stored factors with the oracle; return (mismatches outside the band,
    mismatches inside it, scale mismatches, compared codes)."""
    out_band = in_band = scale_bad = total = 0
    for lt, c in ost.lts.items():
        if c.b == 0:
            continue
        X = Xs[lt]
        Y = oj.residual_rotated(X, c.U_T, c.G, c.U_D, Pi_gpu)
        s, codes, dist = oj.quantize_rows(Y, c.b)
        same_scale = s == c.scales
        scale_bad += int((~same_scale).sum())
        diff = (codes != c.codes) & same_scale[..., None]
        out_band += int((diff & (dist > BOUNDARY_BAND)).sum())
        in_band += int((diff & (dist <= BOUNDARY_BAND)).sum())
        total += codes.size
    return out_band, in_band, scale_bad, total


def oracle_lt_reconstruction(plan, X, seed, lt, rt, rd, b, Pi=None):
    """Oracle float64 reconstruction of one layer-tensor at forced (r_t, r_d, b), with the
    oracle's own factors (spec mode) and the same sketch stream as layer-tensor `lt`."""
    a = oj.analyse_layer_tensor(plan, X, seed, lt, spec=True)
    if Pi is None:
        Pi = onum.rotation_matrix(seed, plan.D, plan.rotation)
    U_T, U_D = a["U_T"][:, :rt], a["U_D"][:, :rd]
    G = onum.round_bf16(a["Gmax"][:, :rt, :rd])
    rec = oj.tucker_part(U_T, G, U_D, plan.H, plan.T, plan.D)
    if b > 0:
        Y = oj.residual_rotated(X, U_T, G, U_D, Pi)
        s, c, _ = oj.quantize_rows(Y, b)
        rec = rec + np.einsum("hte,de->htd", oj.dequantize_rows(s, c, b), Pi)
    return oj.round_output(rec, plan.out_f32), a


def check_allocation(J, st, ost, op, cfg):
    """Budget and allocation checks that need only the GPU's exported tables: every pool within
    its budget, the accounting formula equal to the stored array sizes, and the oracle's dual fed
    the GPU's tables (and squared norms) reproducing the GPU's allocation exactly. Returns the
    oracle units (one per group and kind)."""
    kinds = (0, 1) if cfg.has_v else (0,)
    info = J.jolt_stream_info(st, op.num_groups)
    assert np.array_equal(info["alloc"], ost.alloc)
    ranges = oj.group_ranges(cfg.layers, op.num_groups)
    for kinds_p, bud in op.pools():
        used = sum(oj.layer_bytes(cfg.heads, cfg.tokens, 128, *ost.alloc[g, k]) * len(lay)
                   for g, lay in enumerate(ranges) for k in kinds_p)
        assert used <= bud
    total = 0
    for g, lay in enumerate(ranges):
        for k in kinds:
            total += len(lay) * oj.layer_bytes(cfg.heads, cfg.tokens, 128, *(int(v) for v in ost.alloc[g, k]))
    assert sum(info["bytes_by_part"].values()) == total
    units = []
    grid = op.grid()
    for g, lay in enumerate(ranges):
        for k in kinds:
            tab = J.jolt_export_debug(st, J.JOLT_DBG_TABLE, 2 * g + k)
            bb, rts, rds, nb = [], [], [], []
            for b in op.bits:
                for rt, rd in grid:
                    bb.append(b), rts.append(rt), rds.append(rd)
                    nb.append(len(lay) * oj.layer_bytes(cfg.heads, cfg.tokens, 128, rt, rd, b))
            units.append(oj.Unit(g, k, tab, np.array(nb, dtype=np.int64), np.array(bb), np.array(rts),
                                 np.array(rds), 0.0))
    xx = J.jolt_export_debug(st, J.JOLT_DBG_XX)
    for u in units:
        e = 0.0
        for l in ranges[u.group]:
            e = e + xx[2 * l + u.kind]
        u.energy = e
    alloc_o, _ = oj.allocate(op, units)
    assert np.array_equal(alloc_o, ost.alloc)
    return units


def fullsize_check(J, cfg, ratio, sample, seq=0, encoder="sketch", seed=42, bits=None, factors=1, measured_b=0,
                   rotation=0, keep=False):
    """Encode and decode a whole workload on the GPU in the launch configuration bench.py
    times and check it on sampled layer-tensors against the oracle: the allocation (whole
    cache), principal angles of the factors (when the plan has them), residual codes, the decode
    and the relative error at the GPU's allocation. `bits` restricts the residual widths and
    `factors = 0` forces r_t = r_d = 0 (the in-codec baselines). With `measured_b = 1` the GPU's
    measured error of every allowed width is also compared, per sampled layer-tensor, with the
    oracle's measurement from the GPU's stored factors (float64, relative 1e-9)."""
    import torch
    dev = torch.device("cuda", 0)
    K, V = synth.gen_cache_torch(cfg, dev, seq=seq)
    budget = synth.kv.budget_bytes(cfg, ratio)
    c = J.jolt_config_default()
    c.encoder = J.JOLT_ENC_SKETCH if encoder == "sketch" else J.JOLT_ENC_EXACT
    c.rt_max = RT_MAX
    c.split_kv_budget = int(cfg.split_kv)
    mask = 0
    for b in (bits or cfg.bits):
        mask |= 1 << b
    c.bits_mask = mask
    c.factors = factors
    c.measured_b = measured_b
    c.rotation = rotation
    plan = J.jolt_plan(cfg.layers, cfg.heads, cfg.tokens, cfg.head_dim, cfg.has_v, J.JOLT_BF16, budget,
                       cfg.groups, c)
    st = J.jolt_encode(plan, K, V, seed)
    J.jolt_stream_status(st)
    Ko, Vo = torch.empty_like(K), torch.empty_like(V)
    J.jolt_decode(st, Ko, Vo)
    torch.cuda.synchronize()
    ost = ostream.parse(J.jolt_stream_to_host(st), lts=set(sample))
    op = oracle_plan(cfg, budget, encoder, bits=bits, measured_b=bool(measured_b),
                     rotation="hadamard" if rotation else "haar", rt_cap=RT_MAX if factors else 0)
    assert ost.rt_max == op.R()
    check_allocation(J, st, ost, op, cfg)
    Pi = J.jolt_export_debug(st, J.JOLT_DBG_PI).reshape(128, 128).astype(np.float64)
    if rotation:
        Pi = onum.hadamard_rotation(seed, 128)   # the residual coder applies it exactly (float64 FWHT)
    assert ost.rotation == ("hadamard" if rotation else "haar")
    report = {"alloc": ost.alloc.tolist()}
    if keep:
        report["_keep"] = (Ko, Vo, st)
    for lt in sample:
        l, k = lt // 2, lt % 2
        X = host((K if k == 0 else V)[l])
        worst, where = 0.0, None
        a = oj.analyse_layer_tensor(op, X, seed, lt, spec=False) if factors else None
        UD = J.jolt_export_debug(st, J.JOLT_DBG_UD_F32, lt).reshape(128, 128).astype(np.float64) if factors else None
        kd = leading_count(a["wD"], 128) if factors else 0
        if kd:
            ang = oj.principal_angles(UD[:, :kd], a["U_D"][:, :kd]).max()
            if ang > worst:
                worst, where = ang, ("U_D", kd)
        if op.R() and factors:
            UT = J.jolt_export_debug(st, J.JOLT_DBG_UT_F32, lt).reshape(cfg.tokens, op.R()).astype(np.float64)
            kt = leading_count(a["wT"], op.R())
            if kt:
                ang = oj.principal_angles(UT[:, :kt], a["U_T_unrounded"][:, :kt]).max()
                if ang > worst:
                    w = np.asarray(a["wT"], dtype=np.float64)
                    worst, where = ang, ("U_T", kt, float((w[kt - 1] - w[kt]) / w[0]),
                                         [float(np.arccos(np.clip(abs(UT[:, j] @ a["U_T_unrounded"][:, j]) /
                                                                  np.linalg.norm(UT[:, j]), 0, 1))) for j in range(kt)])
        assert worst < ANGLE_TOL, (lt, worst, where)
        if measured_b:
            c_lt = ost.lts[lt]
            Y = oj.residual_rotated(X, c_lt.U_T, c_lt.G, c_lt.U_D, Pi)
            got_m = J.jolt_export_debug(st, J.JOLT_DBG_MEAS, lt)
            for bb in op.bits:
                if bb == 0:
                    ref_m = float(np.sum(Y * Y))
                else:
                    s_, q_, _ = oj.quantize_rows(Y, bb)
                    ref_m = float(np.sum((Y - oj.dequantize_rows(s_, q_, bb)) ** 2))
                assert abs(got_m[bb] - ref_m) <= 1e-9 * max(ref_m, 1e-300), (lt, bb, got_m[bb], ref_m)
        # codes of this layer-tensor
        out_band, in_band, scale_bad, total = codes_parity(only_lt(ost, lt), {lt: X}, Pi)
        assert scale_bad == 0 and out_band == 0, (lt, scale_bad, out_band, in_band, total)
        # decode of this layer-tensor
        ref = oj.round_output(oj.decode_lt(ost, lt, Pi=None), ost.out_f32)
        got = host((Ko if k == 0 else Vo)[l])
        assert (np.abs(got - ref) <= decode_tol(ref, ost.out_f32)).all(), (lt, np.abs(got - ref).max())
        # error at the GPU's allocation
        g = [gg for gg, lay in enumerate(oj.group_ranges(cfg.layers, op.num_groups)) if l in lay][0]
        rt, rd, b = (int(v) for v in ost.alloc[g, k])
        rec, _ = oracle_lt_reconstruction(op, X, seed, lt, rt, rd, b)
        e_gpu, e_orc = oj.rel_frob(X, got), oj.rel_frob(X, rec)
        assert abs(e_gpu / e_orc - 1.0) <= REL_ERR_TOL, (lt, e_gpu, e_orc)
        report[lt] = dict(max_angle=worst, codes=total, boundary_mismatches=in_band, err=(e_gpu, e_orc))
    J.jolt_stream_status(st)
    return report


def only_lt(ost, lt):
    """A shallow copy of the parsed stream that holds one layer-tensor (codes_parity walks all)."""
    one = copy.copy(ost)
    one.lts = {lt: ost.lts[lt]}
    return one
