"""Randomized Hadamard rotation on the GPU through the C ABI (jolt_config.rotation = 1).

Pi = diag(s) H / sqrt(D) with the signs of the seed's rotation stream: the GPU's float32 Pi is
bit-identical to the oracle's float64 one rounded to float32, the full workload passes the same
checks as with the Haar rotation (allocation, factors, codes, decode, error at the GPU's
allocation), and the stream records the rotation so that a stream read back from host memory
decodes to the same values.
"""
import numpy as np
import pytest

import synth
from gpu_common import fullsize_check
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


def test_hadamard_full_workload_and_stream_round_trip(J):
    import torch
    r = fullsize_check(J, synth.config(1), 2.0, sample=[0, 63], rotation=1, keep=True)
    Ko, Vo, st = r["_keep"]
    Pi = J.jolt_export_debug(st, J.JOLT_DBG_PI).reshape(128, 128)
    assert np.array_equal(Pi, onum.hadamard_rotation(42, 128).astype(np.float32))
    buf = J.jolt_stream_to_host(st)
    assert ostream.parse(buf, lts=set()).rotation == "hadamard"
    st2 = J.jolt_stream_from_host(buf)
    K2, V2 = torch.empty_like(Ko), torch.empty_like(Vo)
    J.jolt_decode(st2, K2, V2)
    torch.cuda.synchronize()
    assert torch.equal(K2, Ko) and torch.equal(V2, Vo)
