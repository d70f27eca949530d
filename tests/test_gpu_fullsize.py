"""Full-size workloads through the C ABI, checked on sampled layer-tensors.

The whole cache of each workload (Mistral-7B shape at T = 1024 with both encoders, LLaMA-2-13B
shape at T = 4096, the 32k-token Mistral shape, sequences of the 8k-token decode sweep at each of
its three budgets) is encoded and decoded on the GPU in the launch configuration bench.py times.
The oracle cannot redo whole multi-GB caches in float64 within a test, so it checks:
* the allocation: the oracle's dual fed the GPU's exported tables reproduces it exactly, every
  budget pool is respected and the byte formula equals the stored sizes (whole cache);
* on sampled layer-tensors, the first (K) and the last (V) layer-tensor of every layer group:
  principal angles of U_D and U_T against the oracle's factors (leading columns with relative
  eigengap >= 1e-4), residual codes bit-exact except within 1e-6 s of a cell boundary with scales
  bit-exact, the GPU decode against the oracle's decode of the GPU's stream, and the layer-tensor's
  relative error within 1% of the oracle's at the GPU's allocation.
"""
import numpy as np
import pytest

import synth
from gpu_common import fullsize_check
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


def group_edges(cfg):
    """Layer-tensors lt = 2 layer + kind: the first layer's K and the last layer's V of each group."""
    out = []
    for lay in oj.group_ranges(cfg.layers, cfg.groups):
        out += [2 * lay[0], 2 * lay[-1] + 1]
    return out


def _report(r):
    """Largest principal angle and boundary-band code count over the sampled layer-tensors."""
    lts = [k for k in r if isinstance(k, int)]
    print({"alloc": r["alloc"], "max_angle": max(r[k]["max_angle"] for k in lts),
           "boundary_mismatches": sum(r[k]["boundary_mismatches"] for k in lts),
           "codes": sum(r[k]["codes"] for k in lts), "err": {k: r[k]["err"] for k in lts}})


@pytest.mark.parametrize("ratio", [2.0, 3.0])
def test_mistral7b_t1024_sketch_full(J, ratio):
    """The bench workload: 32 layers x 8 KV heads x 1024 tokens, K and V, 4 groups, sketch."""
    cfg = synth.config(1)
    _report(fullsize_check(J, cfg, ratio, sample=group_edges(cfg)))


@pytest.mark.parametrize("ratio", [2.0, 3.0])
def test_mistral7b_t1024_exact_full(J, ratio):
    """The same cache with the exact token factor (all 32 layers)."""
    cfg = synth.config(1)
    _report(fullsize_check(J, cfg, ratio, sample=group_edges(cfg), encoder="exact"))


def test_llama13b_t4096_2x_sketch_full(J):
    """LLaMA-2-13B shape: 40 layers x 40 heads x 4096 tokens, K and V, 2x, 5 groups."""
    cfg = synth.config(2)
    _report(fullsize_check(J, cfg, 2.0, sample=group_edges(cfg)))


def test_mistral7b_t32768_3x_low_bits_full(J):
    """32k tokens, 3x, residual bits restricted to 1..4."""
    cfg = synth.config(3)
    _report(fullsize_check(J, cfg, 3.0, sample=group_edges(cfg)))


@pytest.mark.parametrize("seq,ratio", [(0, 2.0), (7, 2.5), (15, 3.0)])
def test_decode_sweep_sequences(J, seq, ratio):
    """Sequences of the 16-sequence, 8k-token sweep at each of its budgets, each its own stream."""
    cfg = synth.config(4)
    _report(fullsize_check(J, cfg, ratio, sample=group_edges(cfg), seq=seq))
