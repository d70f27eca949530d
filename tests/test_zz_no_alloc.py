"""The allocation-free relative-error entry point against the allocating one.

Collected last (file name), so it also runs after every other GPU test has used the library;
it passes on its own as well. Both calls go through the C ABI; the two entry points run the
same kernels in the same reduction order, so their results must be bit-identical.
"""
import numpy as np
import pytest

from gpu_common import to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from tensor_decomposition_b200 import build
    build.build()
    from tensor_decomposition_b200 import jolt
    return jolt


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n", [1, 2047, 1_000_003, 3_000_000])
def test_noalloc_matches_allocating_entry_point(J, dtype, n):
    rng = np.random.default_rng(n)
    a = rng.standard_normal(n).astype(np.float32)
    b = (a + 0.01 * rng.standard_normal(n)).astype(np.float32)
    ta, tb = to_torch(a, dtype), to_torch(b, dtype)
    want = J.jolt_rel_frob_error(ta, tb)
    before = J.jolt_alloc_count()
    first = J.jolt_rel_frob_error_noalloc(ta, tb)
    second = J.jolt_rel_frob_error_noalloc(ta, tb)          # twice in a row: scratch reused
    assert first == want and second == want
    assert J.jolt_alloc_count() == before                   # no device allocation by the library
    z = to_torch(np.zeros(16, np.float32), dtype)
    assert J.jolt_rel_frob_error_noalloc(z, z) == 0.0       # zero reference -> 0 (same rule)


def test_noalloc_rejects_oversized_n(J):
    import ctypes
    t = to_torch(np.ones(4, np.float32), "f32")
    out = ctypes.c_double()
    too_big = (1 << 62) + 1
    st = J._lib.jolt_rel_frob_error_noalloc(J._dptr(t), J._dptr(t), too_big, J._dtype_code(t),
                                            J._stream_ptr(None), ctypes.byref(out))
    assert J.STATUS_NAMES[st] == "INVALID_ARG"       # rejected before any device work
    assert "exceeds the limit" in J._lib.jolt_last_error().decode()
