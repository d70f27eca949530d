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


def test_mistral7b_t1024_2x_sketch_full(J):
    """The bench workload: 32 layers x 8 KV heads x 1024 tokens, K and V, 2x, 4 groups."""
    r = fullsize_check(J, synth.config(1), 2.0, sample=[0, 63])
    print(r)


def test_llama13b_t4096_2x_sketch_full(J):
    """LLaMA-2-13B shape: 40 layers x 40 heads x 4096 tokens, K and V, 2x, 5 groups."""
    r = fullsize_check(J, synth.config(2), 2.0, sample=[1, 78])
    print(r)


def test_mistral7b_t32768_3x_low_bits_full(J):
    """32k tokens, 3x, residual bits restricted to 1..4."""
    r = fullsize_check(J, synth.config(3), 3.0, sample=[30])
    print(r)


@pytest.mark.parametrize("seq,ratio", [(0, 2.5), (15, 3.0)])
def test_decode_sweep_sequences(J, seq, ratio):
    """Sequences of the 16-sequence, 8k-token sweep, each its own stream."""
    r = fullsize_check(J, synth.config(4), ratio, sample=[5], seq=seq)
    print(r)
