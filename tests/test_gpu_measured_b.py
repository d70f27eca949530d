"""Measured-b refinement on the GPU through the C ABI (jolt_config.measured_b = 1).

After the first dual, one extra pass of the residual coder measures the exact squared error of
every allowed width at each unit's chosen ranks, and a second dual re-chooses the widths with
those errors. Checked on full workloads like the JoLT allocation: the oracle's dual fed the
GPU's refined tables reproduces the allocation, the measured errors of sampled layer-tensors
equal the oracle's measurement from the same stored factors, and codes, decode and relative
error match the oracle at the GPU's allocation.
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


@pytest.mark.parametrize("cfg_idx,ratio,sample", [(1, 2.0, [0, 63]), (3, 3.0, [30])])
def test_measured_b_refinement(J, cfg_idx, ratio, sample):
    r = fullsize_check(J, synth.config(cfg_idx), ratio, sample=sample, measured_b=1)
    print(r)
