"""C-ABI library checks that need no GPU: it builds, loads, exports every declared symbol,
and rejects bad requests before touching the device."""
import ctypes
import os
import re
import struct

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def jolt():
    from tensor_decomposition_b200 import build as b
    b.build()
    from tensor_decomposition_b200 import jolt as j
    return j


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "jolt.h")).read()
    return re.findall(r"JOLT_API\s+[\w\s\*]+?\b(jolt_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    for n in ("jolt_plan", "jolt_encode", "jolt_decode", "jolt_rel_frob_error"):
        assert n in names


def test_library_exports_every_declared_symbol(jolt):
    lib = ctypes.CDLL(jolt.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(declared_symbols()) == set(jolt.EXPORTED)


def test_config_defaults(jolt):
    c = jolt.jolt_config_default()
    assert (c.encoder, c.oversample, c.power_iters, c.rank_step, c.rt_max, c.bits_mask,
            c.split_kv_budget, c.max_jacobi_sweeps, c.factors, c.measured_b) == (0, 16, 1, 16, 0, 0x1FF, 0, 30, 1, 0)
    assert c.eig_solver == jolt.JOLT_EIG_TRIDIAG


@pytest.mark.parametrize("args", [
    dict(layers=0, heads=8, tokens=64, head_dim=128),
    dict(layers=2, heads=8, tokens=64, head_dim=64),
    dict(layers=2, heads=8, tokens=64, head_dim=128, groups=3),
    dict(layers=200, heads=8, tokens=64, head_dim=128),
])
def test_plan_rejects_bad_shapes(jolt, args):
    groups = args.pop("groups", 1)
    with pytest.raises(jolt.JoltError) as e:
        jolt.jolt_plan(args["layers"], args["heads"], args["tokens"], args["head_dim"], True,
                       jolt.JOLT_BF16, 10 ** 6, groups)
    assert e.value.status == 1


def test_plan_rejects_infeasible_budget(jolt):
    c = jolt.jolt_config_default()
    c.bits_mask = 0b11110            # b in 1..4 only: the residual alone needs H T (D/8 + 2) bytes
    with pytest.raises(jolt.JoltError) as e:
        jolt.jolt_plan(2, 8, 64, 128, True, jolt.JOLT_BF16, 1000, 1, c)
    assert e.value.status == 2


def test_plan_rejects_bad_options(jolt):
    c = jolt.jolt_config_default()
    c.bits_mask = 0
    with pytest.raises(jolt.JoltError):
        jolt.jolt_plan(2, 8, 64, 128, True, jolt.JOLT_BF16, 10 ** 6, 1, c)
    c = jolt.jolt_config_default()
    c.rank_step = 48
    with pytest.raises(jolt.JoltError):
        jolt.jolt_plan(2, 8, 64, 128, True, jolt.JOLT_BF16, 10 ** 6, 1, c)
    c = jolt.jolt_config_default()
    c.factors = 2                    # 0 (residual only) or 1
    with pytest.raises(jolt.JoltError):
        jolt.jolt_plan(2, 8, 64, 128, True, jolt.JOLT_BF16, 10 ** 6, 1, c)
    c = jolt.jolt_config_default()
    c.eig_solver = 2                 # TRIDIAG (0) or JACOBI (1)
    with pytest.raises(jolt.JoltError):
        jolt.jolt_plan(2, 8, 64, 128, True, jolt.JOLT_BF16, 10 ** 6, 1, c)


@pytest.mark.parametrize("batch,n,solver", [(0, 16, 0), (1, 0, 0), (1, 129, 0), (1, 16, 2)])
def test_eig_small_selftest_rejects_bad_sizes(jolt, batch, n, solver):
    """The small eigensolver self-test checks its arguments before any device call."""
    lib = ctypes.CDLL(jolt.LIB_PATH)
    f = lib.jolt_selftest_eig_small
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int32, ctypes.c_void_p]
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert f(batch, n, p, p, p, solver, None) == 1


def test_stream_from_host_rejects_corrupt_buffers(jolt):
    with pytest.raises(jolt.JoltError) as e:
        jolt.jolt_stream_from_host(b"NOPE" + bytes(100), cuda_stream=0)
    assert e.value.status == 8
    # well-formed header, wrong CRC
    import zlib
    hb = 64 + 24
    hb = (hb + 15) // 16 * 16
    head = bytearray(hb)
    struct.pack_into("<4sIII", head, 0, b"JOLT", 1, hb, 0)
    struct.pack_into("<8i", head, 16, 1, 8, 64, 128, 1, 16, 0, 0)
    struct.pack_into("<QQ", head, 48, 42, 0)
    data = bytes(head)
    good = data + struct.pack("<I", zlib.crc32(data))
    bad = data + struct.pack("<I", zlib.crc32(data) ^ 1)
    with pytest.raises(jolt.JoltError) as e:
        jolt.jolt_stream_from_host(bad, cuda_stream=0)
    assert e.value.status == 8
    # version mismatch
    v2 = bytearray(good)
    struct.pack_into("<I", v2, 4, 2)
    with pytest.raises(jolt.JoltError) as e:
        jolt.jolt_stream_from_host(bytes(v2), cuda_stream=0)
    assert e.value.status == 8


@pytest.mark.parametrize("M,N,K,a_mn,b_mn", [
    (0, 128, 64, 0, 0),      # empty
    (128, 128, 60, 0, 0),    # K not a multiple of 8
    (100, 128, 64, 1, 0),    # transposed A needs M a multiple of 8
    (128, 100, 64, 0, 1),    # transposed B needs N a multiple of 8
])
def test_gemm_selftest_rejects_bad_sizes(jolt, M, N, K, a_mn, b_mn):
    """The layout self-test checks its sizes before any device call (no GPU needed)."""
    lib = ctypes.CDLL(jolt.LIB_PATH)
    f = lib.jolt_selftest_gemm_bf16_layout
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                  ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert f(M, N, K, p, a_mn, p, b_mn, p, None) == 1


@pytest.mark.parametrize("tokens,heads,encoder,rank", [
    (1024, 8, 2, 256),     # Mistral-7B shape, sketch at 2x: the grid's own cap, 256
    (1024, 8, 1, 512),     # the same with the exact encoder: budget / (2T) = 512
    (256, 8, 0, 256),      # single layer, automatic (exact) encoder: T = 256
])
def test_plan_refuses_token_ranks_beyond_the_kernels(jolt, tokens, heads, encoder, rank):
    """The default grid follows the method's reading; a grid above the implemented rank 112 is
    refused before any device call, with the rank in the message."""
    c = jolt.jolt_config_default()
    c.encoder = encoder
    budget = 2 * heads * tokens * 128 * 2 // 2          # 2 layer-tensors at 2x
    with pytest.raises(jolt.JoltError) as e:
        jolt.jolt_plan(1, heads, tokens, 128, True, jolt.JOLT_BF16, budget, 1, c)
    assert e.value.status == 9
    assert f"token rank {rank}" in str(e.value) and "rt_max" in str(e.value)


def test_entry_points_reject_null_handles_without_device_work(jolt):
    """Every entry point that takes a plan, a stream or device buffers rejects null ones with
    JOLT_ERR_INVALID_ARG and a message, before any launch or device allocation; the destroy
    calls accept null."""
    L = jolt._lib
    launches, allocs = L.jolt_launch_count(), L.jolt_alloc_count()
    i32, u64, dbl = ctypes.c_int32(), ctypes.c_uint64(), ctypes.c_double()
    out = ctypes.c_void_p()
    calls = {
        "jolt_plan_info": lambda: L.jolt_plan_info(None, ctypes.byref(i32), ctypes.byref(i32), ctypes.byref(i32),
                                                   ctypes.byref(u64)),
        "jolt_encode": lambda: L.jolt_encode(None, None, None, 42, None, ctypes.byref(out)),
        "jolt_decode": lambda: L.jolt_decode(None, None, None, None),
        "jolt_attention": lambda: L.jolt_attention(None, None, 32, 1, 1.0, None, None),
        "jolt_rel_frob_error": lambda: L.jolt_rel_frob_error(None, None, 16, jolt.JOLT_BF16, None, ctypes.byref(dbl)),
        "jolt_rel_frob_error_noalloc": lambda: L.jolt_rel_frob_error_noalloc(None, None, 16, jolt.JOLT_BF16, None,
                                                                             ctypes.byref(dbl)),
        "jolt_stream_status": lambda: L.jolt_stream_status(None),
        "jolt_stream_info": lambda: L.jolt_stream_info(None, ctypes.byref(u64), ctypes.byref(i32), ctypes.byref(dbl)),
        "jolt_stream_to_host": lambda: L.jolt_stream_to_host(None, None, ctypes.byref(u64)),
        "jolt_export_debug": lambda: L.jolt_export_debug(None, 0, 0, None, ctypes.byref(u64)),
        "jolt_profile_report": lambda: L.jolt_profile_report(None, None),
    }
    for name, call in calls.items():
        assert call() == 1, name
        msg = L.jolt_last_error().decode()
        assert msg.startswith(name) and "null" in msg, (name, msg)
    L.jolt_stream_destroy(None)
    L.jolt_plan_destroy(None)
    assert L.jolt_launch_count() == launches
    assert L.jolt_alloc_count() == allocs


def test_error_calls_reject_bad_dtype_and_size(jolt):
    """The relative-error entry points check the element type, and the allocation-free one its
    size limit, on the host (the buffers below are never dereferenced)."""
    L = jolt._lib
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    d = ctypes.c_double()
    for f in (L.jolt_rel_frob_error, L.jolt_rel_frob_error_noalloc):
        assert f(p, p, 16, 7, None, ctypes.byref(d)) == 1
        assert "dtype" in L.jolt_last_error().decode()
    too_big = (1 << 62) + 1
    assert L.jolt_rel_frob_error_noalloc(p, p, too_big, jolt.JOLT_BF16, None, ctypes.byref(d)) == 1
    assert "exceeds the limit" in L.jolt_last_error().decode()


@pytest.mark.parametrize("batch,n,R", [
    (0, 256, 16),       # empty batch
    (1, 1, 1),          # order below 2
    (1, 4097, 16),      # above the exact encoder's 4096 tokens
    (1, 256, 0),        # no eigenpair asked for
    (1, 100, 101),      # more eigenpairs than the order
    (1, 1024, 129),     # more than the 128 leading eigenpairs the solver returns
])
def test_dense_eig_selftest_rejects_bad_sizes(jolt, batch, n, R):
    L = jolt._lib
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert L.jolt_selftest_eig_dense(batch, n, R, p, p, p, None) == 1
    assert "jolt_selftest_eig_dense" in L.jolt_last_error().decode()


def test_dense_eig_selftest_rejects_null_buffers(jolt):
    L = jolt._lib
    assert L.jolt_selftest_eig_dense(1, 256, 16, None, None, None, None) == 1


def test_profile_switch_needs_no_device(jolt):
    L = jolt._lib
    assert L.jolt_profile_enable(1) == 0
    assert L.jolt_profile_enable(0) == 0
