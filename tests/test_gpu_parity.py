"""GPU parity: the CUDA path (through the C ABI) against the float64 CPU oracle.

Tolerances (each stated where it is asserted, with the arithmetic behind it):
* factors: principal angles < 1e-3 rad on the leading columns whose relative eigengap is
  at least 1e-4 (float64 eigensolvers fed float64-summed Grams);
* relative Frobenius error within 1% (relative) of the oracle's at the GPU's allocation;
* decode: |gpu - cpu decode of the GPU stream| <= max(1e-3, one bf16 ulp of the value);
* residual codes bit-exact when the oracle re-codes the GPU's stored factors, except within
  1e-6 (row-scale units) of a cell boundary; scales bit-exact.
"""
import math

import numpy as np
import pytest

import synth
from gpu_common import (ANGLE_TOL, REL_ERR_TOL, codes_parity, decode_tol, gpu_decode,
                        gpu_encode, host, leading_count, oracle_lt_reconstruction, oracle_plan,
                        to_torch)
from oracle import jolt as oj
from oracle import numerics as onum
from oracle import stream as ostream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_decomposition_b200 import build
    build.build()
    from tensor_decomposition_b200 import jolt
    return jolt


def small_cfg(tokens=200, layers=4, heads=8, seed=1101):
    return synth.config(1, layers=layers, tokens=tokens, heads=heads, seed=seed, groups=2)


# ------------------------------------------------------------------ elementary kernels
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rel_frob_matches_float64(J, dtype):
    rng = np.random.default_rng(0)
    n = 1_000_003                                     # ragged against every block size
    a = rng.standard_normal(n).astype(np.float32)
    b = (a + 0.01 * rng.standard_normal(n)).astype(np.float32)
    ta, tb = to_torch(a, dtype), to_torch(b, dtype)
    ha, hb = host(ta), host(tb)
    ref = math.sqrt(((ha - hb) ** 2).sum()) / math.sqrt((ha ** 2).sum())
    got = J.jolt_rel_frob_error(ta, tb)
    assert abs(got / ref - 1.0) < 1e-12
    z = to_torch(np.zeros(10, np.float32), dtype)
    assert J.jolt_rel_frob_error(z, z) == 0.0


def test_rotation_and_sketch_are_the_oracles(J):
    cfg = small_cfg()
    K, V = synth.gen_cache_numpy(cfg)
    budget = synth.bf16_bytes(cfg) // 2
    plan, st, _, _ = gpu_encode(cfg, K, V, budget, "sketch", seed=42)
    Pi = J.jolt_export_debug(st, J.JOLT_DBG_PI).reshape(128, 128).astype(np.float64)
    Po = onum.haar_rotation(42, 128)
    assert np.abs(Pi - Po).max() <= 1.2e-7                     # float32 rounding of Pi
    assert np.abs(Pi.T @ Pi - np.eye(128)).max() < 2e-6
    info = J.jolt_plan_info(plan)
    l = info["sketch_l"]
    for lt in (0, 3, 6):
        om = J.jolt_export_debug(st, J.JOLT_DBG_OMEGA, lt)
        ref = onum.bf16_bits(onum.sketch_matrix(42, lt, cfg.heads * 128, l)).reshape(-1)
        assert np.array_equal(om, ref)


# ------------------------------------------------------------------ minimal slice: decode an oracle stream
@pytest.mark.parametrize("encoder", ["sketch", "exact"])
def test_gpu_decodes_an_oracle_stream(J, encoder):
    cfg = small_cfg(tokens=120, layers=2, heads=4)
    K, V = synth.gen_cache_numpy(cfg)
    op = oracle_plan(cfg, synth.bf16_bytes(cfg) // 2, encoder)
    ost, _ = oj.encode(op, K, V, seed=7)
    buf = ostream.serialize(ost)
    st = J.jolt_stream_from_host(buf)
    import torch
    Ko = torch.empty(K.shape, dtype=torch.bfloat16, device="cuda")
    Vo = torch.empty(V.shape, dtype=torch.bfloat16, device="cuda")
    J.jolt_decode(st, Ko, Vo)
    torch.cuda.synchronize()
    Kr, Vr = oj.decode(ost)
    for got, ref in ((host(Ko), Kr), (host(Vo), Vr)):
        assert (np.abs(got - ref) <= decode_tol(ref, False)).all()
    assert J.jolt_stream_to_host(st) == buf


# ------------------------------------------------------------------ full encode parity
def _parity(J, cfg, encoder, budget, seed=42):
    K, V = synth.gen_cache_numpy(cfg)
    plan, st, Kd, Vd = gpu_encode(cfg, K, V, budget, encoder, seed=seed)
    buf = J.jolt_stream_to_host(st)
    ost = ostream.parse(buf)
    op = oracle_plan(cfg, budget, encoder)
    assert ost.rt_max == op.R()
    kinds = (0, 1) if cfg.has_v else (0,)
    Xs = {2 * l + k: (K if k == 0 else V)[l].astype(np.float64) for l in range(cfg.layers) for k in kinds}
    report = {}

    # budget: every pool within its budget, accounting formula = stored array sizes
    info = J.jolt_stream_info(st, op.num_groups)
    assert np.array_equal(info["alloc"], ost.alloc)
    for kinds_p, bud in op.pools():
        used = sum(oj.layer_bytes(cfg.heads, cfg.tokens, 128, *ost.alloc[g, k]) * len(lay)
                   for g, lay in enumerate(oj.group_ranges(cfg.layers, op.num_groups)) for k in kinds_p)
        assert used <= bud
    assert sum(info["bytes_by_part"].values()) == sum(
        oj.layer_bytes(cfg.heads, cfg.tokens, 128, c.rt, c.rd, c.b) for c in ost.lts.values())

    # allocation: the oracle's dual fed the GPU's tables reproduces the GPU's choice
    units = []
    grid = op.grid()
    for g, lay in enumerate(oj.group_ranges(cfg.layers, op.num_groups)):
        for k in kinds:
            tab = J.jolt_export_debug(st, J.JOLT_DBG_TABLE, 2 * g + k)
            bb, rts, rds, nb = [], [], [], []
            for b in op.bits:
                for rt, rd in grid:
                    bb.append(b), rts.append(rt), rds.append(rd)
                    nb.append(len(lay) * oj.layer_bytes(cfg.heads, cfg.tokens, 128, rt, rd, b))
            units.append(oj.Unit(g, k, tab, np.array(nb, dtype=np.int64), np.array(bb), np.array(rts),
                                 np.array(rds), 0.0))
    # energy E(0,0) per unit: the exported squared norms summed over the group in layer order
    xx = J.jolt_export_debug(st, J.JOLT_DBG_XX)
    for u in units:
        e = 0.0
        for l in oj.group_ranges(cfg.layers, op.num_groups)[u.group]:
            e = e + xx[2 * l + u.kind]
        u.energy = e
    alloc_o, _ = oj.allocate(op, units)
    assert np.array_equal(alloc_o, ost.alloc)
    # the tables themselves: oracle tables from its own factors, close to the GPU's
    for u in units:
        lay = oj.group_ranges(cfg.layers, op.num_groups)[u.group]
        E_o = sum(oj.analyse_layer_tensor(op, Xs[2 * l + u.kind], seed, 2 * l + u.kind)["E"] for l in lay)
        E_g = u.err[op.bits.index(0) * len(grid):][:len(grid)] if 0 in op.bits else None
        if E_g is not None:
            assert np.allclose(E_g, E_o, rtol=1e-2, atol=1e-5 * E_o[0])

    # factors: leading subspaces
    worst = 0.0
    for lt, X in Xs.items():
        a = oj.analyse_layer_tensor(op, X, seed, lt, spec=False)
        UD = J.jolt_export_debug(st, J.JOLT_DBG_UD_F32, lt).reshape(128, 128).astype(np.float64)
        k = leading_count(a["wD"], 128)
        if k:
            worst = max(worst, oj.principal_angles(UD[:, :k], a["U_D"][:, :k]).max())
        if op.R():
            UT = J.jolt_export_debug(st, J.JOLT_DBG_UT_F32, lt).reshape(cfg.tokens, op.R()).astype(np.float64)
            k = leading_count(a["wT"], op.R())
            if k:
                worst = max(worst, oj.principal_angles(UT[:, :k], a["U_T_unrounded"][:, :k]).max())
    report["max_angle"] = worst
    assert worst < ANGLE_TOL

    # residual codes: bit-exact except at cell boundaries
    Pi = J.jolt_export_debug(st, J.JOLT_DBG_PI).reshape(128, 128).astype(np.float64)
    out_band, in_band, scale_bad, total = codes_parity(ost, Xs, Pi)
    report.update(codes=total, boundary_mismatches=in_band)
    assert scale_bad == 0 and out_band == 0, (scale_bad, out_band, in_band, total)

    # decode: GPU vs CPU decode of the GPU's own stream
    Ko, Vo = gpu_decode(cfg, st, Kd, Vd)
    Kr, Vr = oj.decode(ost)
    for got, ref in ((Ko, Kr), (Vo, Vr)):
        if got is None:
            continue
        g = host(got)
        assert (np.abs(g - ref) <= decode_tol(ref, ost.out_f32)).all(), np.abs(g - ref).max()

    # error: GPU vs the oracle at the GPU's allocation, per kind
    for k in kinds:
        ref_t, out_t = (Kd, Ko) if k == 0 else (Vd, Vo)
        e_gpu = J.jolt_rel_frob_error(ref_t, out_t)
        num = den = 0.0
        for l in range(cfg.layers):
            g = [gg for gg, lay in enumerate(oj.group_ranges(cfg.layers, op.num_groups)) if l in lay][0]
            rt, rd, b = (int(v) for v in ost.alloc[g, k])
            X = Xs[2 * l + k]
            rec, _ = oracle_lt_reconstruction(op, X, seed, 2 * l + k, rt, rd, b)
            num += ((X - rec) ** 2).sum()
            den += (X ** 2).sum()
        e_orc = math.sqrt(num / den)
        report[f"err_{k}"] = (e_gpu, e_orc)
        assert abs(e_gpu / e_orc - 1.0) <= REL_ERR_TOL, (e_gpu, e_orc)
    J.jolt_stream_status(st)
    return report


def test_sketch_encode_parity_ragged(J):
    cfg = small_cfg(tokens=200)                     # T = 200: ragged against 64-row tiles and 256-token chunks
    r = _parity(J, cfg, "sketch", synth.bf16_bytes(cfg) // 2)
    print(r)


def test_sketch_encode_parity_three_x(J):
    cfg = small_cfg(tokens=256, seed=1202)
    r = _parity(J, cfg, "sketch", synth.bf16_bytes(cfg) // 3)
    print(r)


def test_exact_encode_parity_single_layer(J):
    cfg = synth.config(0, tokens=128)              # exact token Gram 128 x 128, float32 output
    r = _parity(J, cfg, "exact", synth.bf16_bytes(cfg) // 2)
    print(r)


def test_exact_encode_parity_config0_full(J):
    cfg = synth.config(0)                          # 1 x 8 x 256 x 128, float32: token Gram 256 x 256
    r = _parity(J, cfg, "exact", synth.bf16_bytes(cfg) // 2)
    print(r)


def test_exact_encode_parity_t1024(J):
    cfg = synth.config(1, layers=2, seed=1404, groups=2)   # Mistral shape at T = 1024, exact token factor
    r = _parity(J, cfg, "exact", synth.bf16_bytes(cfg) // 2)
    print(r)


def test_sketch_encode_parity_long_unsplit_tokens(J):
    """T = 2056 = 8 x 257: the contractions over the tokens cannot split into whole 64-token
    chunks of at most 2048, so the plan takes the float64-accumulating SIMT contractions."""
    cfg = small_cfg(tokens=2056, layers=2, heads=2, seed=1505)
    r = _parity(J, cfg, "sketch", synth.bf16_bytes(cfg) // 2)
    print(r)


def test_zero_rows_give_zero_scales(J):
    """A token whose feature rows are zero in every head of a layer-tensor has a zero token-factor
    row (it lies outside the range of the token Gram and of the sketch), hence a zero residual
    row: scale 0 and all codes 0 on both sides (the s = 0 branch of the quantiser)."""
    cfg = small_cfg(tokens=200, layers=2, heads=4, seed=1606)
    K, V = synth.gen_cache_numpy(cfg)
    K[0, :, 5, :] = 0.0
    V[1, :, 17, :] = 0.0
    budget = synth.bf16_bytes(cfg) // 2
    for encoder in ("sketch", "exact"):
        plan, st, Kd, Vd = gpu_encode(cfg, K, V, budget, encoder)
        ost = ostream.parse(J.jolt_stream_to_host(st))
        for lt, t in ((0, 5), (3, 17)):
            c = ost.lts[lt]
            if c.b:
                assert (c.scales[:, t] == 0).all() and (c.codes[:, t, :] == 0).all()
        r = _parity_of_stream(J, cfg, K, V, st, Kd, Vd, encoder, budget)
        print(encoder, r)


def _parity_of_stream(J, cfg, K, V, st, Kd, Vd, encoder, budget, seed=42):
    """Codes and decode of an encoded stream against the oracle (the checks of _parity that need
    no re-encode)."""
    ost = ostream.parse(J.jolt_stream_to_host(st))
    kinds = (0, 1) if cfg.has_v else (0,)
    Xs = {2 * l + k: (K if k == 0 else V)[l].astype(np.float64) for l in range(cfg.layers) for k in kinds}
    Pi = J.jolt_export_debug(st, J.JOLT_DBG_PI).reshape(128, 128).astype(np.float64)
    out_band, in_band, scale_bad, total = codes_parity(ost, Xs, Pi)
    assert scale_bad == 0 and out_band == 0, (scale_bad, out_band, in_band, total)
    Ko, Vo = gpu_decode(cfg, st, Kd, Vd)
    Kr, Vr = oj.decode(ost)
    for got, ref in ((Ko, Kr), (Vo, Vr)):
        g = host(got)
        assert (np.abs(g - ref) <= decode_tol(ref, ost.out_f32)).all(), np.abs(g - ref).max()
    return dict(codes=total, boundary_mismatches=in_band)


def test_restricted_bits_and_joint_pool(J):
    cfg = synth.config(1, layers=3, tokens=136, seed=1303, groups=3, split_kv=False, bits=(1, 2, 3, 4))
    r = _parity(J, cfg, "sketch", synth.bf16_bytes(cfg) // 3)
    print(r)


# ------------------------------------------------------------------ error reporting on the device
def test_nonfinite_input_is_reported(J):
    cfg = synth.config(1, layers=1, tokens=64, heads=2, groups=1)
    K, V = synth.gen_cache_numpy(cfg)
    K[0, 1, 5, 7] = np.nan
    with pytest.raises(J.JoltError) as e:
        gpu_encode(cfg, K, V, synth.bf16_bytes(cfg) // 2, "sketch")
    assert e.value.status == 6


def test_corrupt_stream_rejected(J):
    cfg = synth.config(1, layers=1, tokens=64, heads=2, groups=1)
    K, V = synth.gen_cache_numpy(cfg)
    _, st, _, _ = gpu_encode(cfg, K, V, synth.bf16_bytes(cfg) // 2, "sketch")
    buf = bytearray(J.jolt_stream_to_host(st))
    buf[len(buf) // 2] ^= 1
    with pytest.raises(J.JoltError) as e:
        J.jolt_stream_from_host(bytes(buf))
    assert e.value.status == 8


# ------------------------------------------------------------------ tensor-core GEMM building block
@pytest.mark.parametrize("a_mn,b_mn", [(0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (200, 136, 200), (256, 384, 128), (1024, 128, 128)])
def test_tcgen05_gemm_transposed_operands(J, M, N, K, a_mn, b_mn):
    """Operands stored [K][M] / [K][N] (MN-major in the MMA, as the analysis feeds its bases)
    against float64, including ragged M, N and K."""
    import torch
    g = torch.Generator(device="cuda").manual_seed(M * 11 + N * 5 + K + 3 * a_mn + b_mn)
    A = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn((N, K), generator=g, device="cuda").to(torch.bfloat16)
    C = torch.full((M, N), float("nan"), device="cuda", dtype=torch.float32)
    J.jolt_selftest_gemm_bf16_layout(A.T.contiguous() if a_mn else A, a_mn, B.T.contiguous() if b_mn else B, b_mn, C)
    ref = A.double() @ B.double().T
    err = (C.double() - ref).abs().max().item()
    scale = (A.double().abs() @ B.double().abs().T).max().item()
    assert torch.isfinite(C).all()
    assert err <= 1e-5 * scale, (err, scale)


@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (200, 136, 200), (256, 128, 1024), (384, 256, 72)])
def test_tcgen05_gemm_matches_float64(J, M, N, K):
    import torch
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn((N, K), generator=g, device="cuda").to(torch.bfloat16)
    C = torch.full((M, N), float("nan"), device="cuda", dtype=torch.float32)
    J.jolt_selftest_gemm_bf16(A, B, C)
    ref = (A.double() @ B.double().T)
    err = (C.double() - ref).abs().max().item()
    scale = (A.double().abs() @ B.double().abs().T).max().item()
    assert torch.isfinite(C).all()
    assert err <= 1e-5 * scale, (err, scale)
