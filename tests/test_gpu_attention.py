"""Attention over the compressed cache on the GPU (through the C ABI) against the oracle's plain
definition: softmax(scale q K_hat^T) V_hat with K_hat, V_hat the float64 reconstructions of the
GPU's own stream.

Tolerance: the kernel works in float32 on stored values that are exact in float32 (bf16 factors,
codes, fp16 scales); Pi^T q and G_h U_D^T q carry ~1e-7 relative error, scores and the softmax
inherit it, and the weighted sums run over up to 8192 tokens in float32 (~1e-6 relative). The bound
is 1e-4 of the largest output magnitude of the layer plus 1e-6, two orders above that estimate.
"""
import math

import numpy as np
import pytest

import synth
from gpu_common import RT_MAX, gpu_encode, host
from oracle import attention as oa
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


def _queries(L, Hq, n, seed):
    import torch
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((L, Hq, n, 128), generator=g, device="cuda").to(torch.bfloat16)


def _check(J, st, Q, layers, scale):
    import torch
    out = torch.full(Q.shape, float("nan"), dtype=torch.float32, device="cuda")
    J.jolt_attention(st, Q, out, scale)
    torch.cuda.synchronize()
    ost = ostream.parse(J.jolt_stream_to_host(st), lts={2 * l + k for l in layers for k in (0, 1)})
    Qh, got = host(Q), host(out)
    worst = 0.0
    for l in layers:
        ref = oa.attention_over_stream(ost, l, Qh[l], scale)
        err = np.abs(got[l] - ref).max()
        tol = 1e-4 * np.abs(ref).max() + 1e-6
        assert err <= tol, (l, err, tol)
        worst = max(worst, err / np.abs(ref).max())
    return worst


@pytest.mark.parametrize("tokens,Hq,n", [(600, 32, 1), (600, 8, 3), (256, 16, 2)])
def test_attention_matches_the_definition(J, tokens, Hq, n):
    """Grouped-query (4 query heads per KV head) and multi-head, one to three queries per head,
    token counts across whole and ragged 256-token chunks."""
    cfg = synth.config(1, layers=3, tokens=tokens, heads=8, seed=1707, groups=3)
    K, V = synth.gen_cache_numpy(cfg)
    _, st, _, _ = gpu_encode(cfg, K, V, synth.bf16_bytes(cfg) // 2, "sketch")
    Q = _queries(cfg.layers, Hq, n, tokens + Hq + n)
    print(_check(J, st, Q, range(cfg.layers), 1.0 / math.sqrt(128)))


def test_attention_full_mistral_cache(J):
    """The Mistral-7B workload (32 layers, 8 KV heads, 32 query heads, T = 1024) at 2x: the whole
    cache in one call, the first and last layers checked."""
    import torch
    cfg = synth.config(1)
    K, V = synth.gen_cache_torch(cfg, torch.device("cuda", 0))
    c = J.jolt_config_default()
    c.encoder = J.JOLT_ENC_SKETCH
    c.rt_max = RT_MAX
    c.split_kv_budget = 1
    plan = J.jolt_plan(cfg.layers, cfg.heads, cfg.tokens, 128, True, J.JOLT_BF16, synth.kv.budget_bytes(cfg, 2.0),
                       cfg.groups, c)
    st = J.jolt_encode(plan, K, V, 42)
    J.jolt_stream_status(st)
    Q = _queries(cfg.layers, 32, 1, 77)
    print(_check(J, st, Q, (0, 31), 1.0 / math.sqrt(128)))
