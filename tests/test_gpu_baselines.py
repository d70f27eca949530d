"""In-codec baselines on the GPU through the C ABI, checked against the oracle.

Residual only (jolt_config.factors = 0, bits_mask = 1 << 4): per-row 4-bit quantisation of the
rotated cache, r_t = r_d = 0 everywhere. Tucker only (bits_mask = 1): the dual picks the ranks
and no residual is stored. Both run the same kernels as the JoLT allocation ("A JoLT for the KV
Cache", Abstract: the joint allocation against quantisation-only and decomposition-only
methods) and are checked like the full workloads: allocation, factors where present, codes,
decode, and the relative error within 1% of the oracle's at the GPU's allocation.
"""
import pytest

import synth
from gpu_common import fullsize_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_decomposition_b200 import build
    build.build()
    from tensor_decomposition_b200 import jolt
    return jolt


def _units(report):
    return [tuple(u) for grp in report["alloc"] for u in grp]


@pytest.mark.parametrize("cfg_idx,sample", [(1, [0, 63]), (2, [1])])
def test_residual_only_4bit(J, cfg_idx, sample):
    cfg = synth.config(cfg_idx)
    r = fullsize_check(J, cfg, 2.0, sample=sample, bits=(4,), factors=0)
    assert all(u == (0, 0, 4) for u in _units(r)), r["alloc"]
    print(r)


@pytest.mark.parametrize("cfg_idx,sample", [(1, [0, 63]), (2, [78])])
def test_tucker_only(J, cfg_idx, sample):
    cfg = synth.config(cfg_idx)
    r = fullsize_check(J, cfg, 2.0, sample=sample, bits=(0,))
    assert all(u[2] == 0 and u[0] > 0 for u in _units(r)), r["alloc"]
    print(r)
