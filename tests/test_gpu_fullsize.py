"""Full-size workloads through the C ABI, checked on sampled layer-tensors.

The whole cache of each workload (Mistral-7B shape at T = 1024, LLaMA-2-13B shape at
T = 4096, the 32k-token Mistral shape, two sequences of the 8k-token decode sweep) is encoded
and decoded on the GPU in the launch configuration bench.py times. The oracle cannot redo whole
multi-GB caches in float64 within a test, so it checks:
* the allocation: the oracle's dual fed the GPU's exported tables reproduces it exactly, every
  budget pool is respected and the byte formula equals the stored sizes (whole cache);
* on one or two sampled layer-tensors: principal angles of U_D and U_T against the oracle's
  factors (leading columns with relative eigengap >= 1e-3), residual codes bit-exact except
  within 1e-6 s of a cell boundary with scales bit-exact, the GPU decode against the oracle's
  decode of the GPU's stream, and the layer-tensor's relative error within 1% of the oracle's at
  the GPU's allocation.
"""
import copy

import numpy as np
import pytest

import synth
from gpu_common import (ANGLE_TOL, REL_ERR_TOL, check_allocation, codes_parity, decode_tol, host,
                        leading_count, oracle_lt_reconstruction, oracle_plan)
from oracle import jolt as oj
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


def _fullsize(J, cfg, ratio, sample, seq=0, encoder="sketch", seed=42):
    import torch
    dev = torch.device("cuda", 0)
    K, V = synth.gen_cache_torch(cfg, dev, seq=seq)
    budget = synth.kv.budget_bytes(cfg, ratio)
    c = J.jolt_config_default()
    c.encoder = J.JOLT_ENC_SKETCH if encoder == "sketch" else J.JOLT_ENC_EXACT
    c.split_kv_budget = int(cfg.split_kv)
    mask = 0
    for b in cfg.bits:
        mask |= 1 << b
    c.bits_mask = mask
    plan = J.jolt_plan(cfg.layers, cfg.heads, cfg.tokens, cfg.head_dim, cfg.has_v, J.JOLT_BF16, budget,
                       cfg.groups, c)
    st = J.jolt_encode(plan, K, V, seed)
    J.jolt_stream_status(st)
    Ko, Vo = torch.empty_like(K), torch.empty_like(V)
    J.jolt_decode(st, Ko, Vo)
    torch.cuda.synchronize()
    ost = ostream.parse(J.jolt_stream_to_host(st), lts=set(sample))
    op = oracle_plan(cfg, budget, encoder)
    assert ost.rt_max == op.R()
    check_allocation(J, st, ost, op, cfg)
    Pi = J.jolt_export_debug(st, J.JOLT_DBG_PI).reshape(128, 128).astype(np.float64)
    report = {"alloc": ost.alloc.tolist()}
    for lt in sample:
        l, k = lt // 2, lt % 2
        X = host((K if k == 0 else V)[l])
        a = oj.analyse_layer_tensor(op, X, seed, lt, spec=False)
        # factors
        worst, where = 0.0, None
        UD = J.jolt_export_debug(st, J.JOLT_DBG_UD_F32, lt).reshape(128, 128).astype(np.float64)
        kd = leading_count(a["wD"], 128)
        if kd:
            ang = oj.principal_angles(UD[:, :kd], a["U_D"][:, :kd]).max()
            if ang > worst:
                worst, where = ang, ("U_D", kd)
        if op.R():
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
        # codes of this layer-tensor
        out_band, in_band, scale_bad, total = codes_parity(_only(ost, lt), {lt: X}, Pi)
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


def _only(ost, lt):
    """A shallow copy of the parsed stream that holds one layer-tensor (codes_parity walks all)."""
    one = copy.copy(ost)
    one.lts = {lt: ost.lts[lt]}
    return one


def test_mistral7b_t1024_2x_sketch_full(J):
    """The bench workload: 32 layers x 8 KV heads x 1024 tokens, K and V, 2x, 4 groups."""
    r = _fullsize(J, synth.config(1), 2.0, sample=[0, 63])
    print(r)


def test_llama13b_t4096_2x_sketch_full(J):
    """LLaMA-2-13B shape: 40 layers x 40 heads x 4096 tokens, K and V, 2x, 5 groups."""
    r = _fullsize(J, synth.config(2), 2.0, sample=[1, 78])
    print(r)


def test_mistral7b_t32768_3x_low_bits_full(J):
    """32k tokens, 3x, residual bits restricted to 1..4."""
    r = _fullsize(J, synth.config(3), 3.0, sample=[30])
    print(r)


@pytest.mark.parametrize("seq,ratio", [(0, 2.5), (15, 3.0)])
def test_decode_sweep_sequences(J, seq, ratio):
    """Sequences of the 16-sequence, 8k-token sweep, each its own stream."""
    r = _fullsize(J, synth.config(4), ratio, sample=[5], seq=seq)
    print(r)
