"""Python binding of the JoLT codec library (libjolt.so), argument marshalling only.

Every function has the name of the C entry point it calls (include/jolt.h). Tensors are
PyTorch CUDA tensors used as plain device memory; CUDA streams default to torch's current
stream. All computation happens in the library's CUDA kernels: if the library is missing
or fails to load, importing this module raises, there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjolt.so")

JOLT_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "BUDGET_INFEASIBLE", 3: "OOM", 4: "CUDA",
                5: "NOT_CONVERGED", 6: "NONFINITE", 7: "TIMEOUT", 8: "CORRUPT_STREAM",
                9: "UNSUPPORTED"}
JOLT_BF16, JOLT_F32 = 0, 1
JOLT_ENC_AUTO, JOLT_ENC_EXACT, JOLT_ENC_SKETCH = 0, 1, 2
JOLT_EIG_TRIDIAG, JOLT_EIG_JACOBI = 0, 1
JOLT_ROT_HAAR, JOLT_ROT_HADAMARD = 0, 1
JOLT_DBG_PI, JOLT_DBG_UT_F32, JOLT_DBG_UD_F32, JOLT_DBG_TABLE, JOLT_DBG_XX, JOLT_DBG_LAMBDA, \
    JOLT_DBG_OMEGA, JOLT_DBG_MEAS = range(8)
PART_NAMES = ("U_T", "U_D", "G", "scales", "codes")

EXPORTED = ["jolt_config_default", "jolt_plan", "jolt_plan_info", "jolt_encode", "jolt_decode",
            "jolt_rel_frob_error", "jolt_rel_frob_error_noalloc", "jolt_stream_status",
            "jolt_stream_info", "jolt_stream_to_host", "jolt_stream_from_host", "jolt_export_debug", "jolt_stream_destroy",
            "jolt_plan_destroy", "jolt_last_error", "jolt_profile_enable", "jolt_profile_report",
            "jolt_launch_count", "jolt_alloc_count", "jolt_selftest_gemm_bf16", "jolt_selftest_gemm_bf16_layout",
            "jolt_selftest_eig_dense", "jolt_selftest_eig_small", "jolt_attention"]


class JoltError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int32), ("heads", ctypes.c_int32), ("tokens", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("has_v", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class Config(ctypes.Structure):
    _fields_ = [("encoder", ctypes.c_int32), ("oversample", ctypes.c_int32),
                ("power_iters", ctypes.c_int32), ("rank_step", ctypes.c_int32),
                ("rt_max", ctypes.c_int32), ("bits_mask", ctypes.c_uint32),
                ("split_kv_budget", ctypes.c_int32), ("max_jacobi_sweeps", ctypes.c_int32),
                ("factors", ctypes.c_int32), ("measured_b", ctypes.c_int32), ("rotation", ctypes.c_int32),
                ("eig_solver", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m tensor_decomposition_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, u64, i32, st = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int32, ctypes.c_int
    sig = {
        "jolt_config_default": (None, [ctypes.POINTER(Config)]),
        "jolt_plan": (st, [ctypes.POINTER(Shape), u64, i32, ctypes.POINTER(Config), ctypes.POINTER(vp)]),
        "jolt_plan_info": (st, [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32),
                                ctypes.POINTER(u64)]),
        "jolt_encode": (st, [vp, vp, vp, u64, vp, ctypes.POINTER(vp)]),
        "jolt_decode": (st, [vp, vp, vp, vp]),
        "jolt_rel_frob_error": (st, [vp, vp, u64, i32, vp, ctypes.POINTER(ctypes.c_double)]),
        "jolt_rel_frob_error_noalloc": (st, [vp, vp, u64, i32, vp, ctypes.POINTER(ctypes.c_double)]),
        "jolt_stream_status": (st, [vp]),
        "jolt_stream_info": (st, [vp, ctypes.POINTER(u64), ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_double)]),
        "jolt_stream_to_host": (st, [vp, vp, ctypes.POINTER(u64)]),
        "jolt_stream_from_host": (st, [vp, u64, vp, ctypes.POINTER(vp)]),
        "jolt_export_debug": (st, [vp, i32, i32, vp, ctypes.POINTER(u64)]),
        "jolt_stream_destroy": (None, [vp]),
        "jolt_plan_destroy": (None, [vp]),
        "jolt_last_error": (ctypes.c_char_p, []),
        "jolt_profile_enable": (st, [i32]),
        "jolt_profile_report": (st, [ctypes.c_char_p, ctypes.POINTER(u64)]),
        "jolt_launch_count": (u64, []),
        "jolt_alloc_count": (u64, []),
        "jolt_selftest_gemm_bf16": (st, [i32, i32, i32, vp, vp, vp, vp]),
        "jolt_selftest_gemm_bf16_layout": (st, [i32, i32, i32, vp, i32, vp, i32, vp, vp]),
        "jolt_selftest_eig_dense": (st, [i32, i32, i32, vp, vp, vp, vp]),
        "jolt_selftest_eig_small": (st, [i32, i32, vp, vp, vp, i32, vp]),
        "jolt_attention": (st, [vp, vp, i32, i32, ctypes.c_float, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def _check(status: int):
    if status != JOLT_OK:
        raise JoltError(status, _lib.jolt_last_error().decode())


def _stream_ptr(cuda_stream):
    if cuda_stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if hasattr(cuda_stream, "cuda_stream"):
        return ctypes.c_void_p(cuda_stream.cuda_stream)
    return ctypes.c_void_p(int(cuda_stream))


def _dptr(t, dtype=None):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return JOLT_BF16
    if t.dtype == torch.float32:
        return JOLT_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def jolt_config_default() -> Config:
    c = Config()
    _lib.jolt_config_default(ctypes.byref(c))
    return c


class Plan:
    def __init__(self, handle, shape: Shape, budget: int, groups: int, cfg: Config):
        self.handle, self.shape, self.budget, self.groups, self.cfg = handle, shape, budget, groups, cfg

    def __del__(self):
        if getattr(self, "handle", None):
            _lib.jolt_plan_destroy(self.handle)
            self.handle = None


class Stream:
    def __init__(self, handle, plan=None, keep=()):
        self.handle, self.plan, self._keep = handle, plan, keep

    def __del__(self):
        if getattr(self, "handle", None):
            _lib.jolt_stream_destroy(self.handle)
            self.handle = None


def jolt_plan(layers, heads, tokens, head_dim, has_v, dtype, byte_budget, num_groups, config=None) -> Plan:
    sh = Shape(layers, heads, tokens, head_dim, int(bool(has_v)), dtype)
    cfg = config if config is not None else jolt_config_default()
    h = ctypes.c_void_p()
    _check(_lib.jolt_plan(ctypes.byref(sh), int(byte_budget), int(num_groups), ctypes.byref(cfg), ctypes.byref(h)))
    return Plan(h, sh, int(byte_budget), int(num_groups), cfg)


def jolt_plan_info(plan: Plan) -> dict:
    r, l, e = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    w = ctypes.c_uint64()
    _check(_lib.jolt_plan_info(plan.handle, ctypes.byref(r), ctypes.byref(l), ctypes.byref(e), ctypes.byref(w)))
    return dict(rt_max=r.value, sketch_l=l.value, encoder=e.value, workspace_bytes=w.value)


def jolt_encode(plan: Plan, K, V, seed: int, cuda_stream=None) -> Stream:
    h = ctypes.c_void_p()
    _check(_lib.jolt_encode(plan.handle, _dptr(K), _dptr(V), int(seed) & (2 ** 64 - 1),
                            _stream_ptr(cuda_stream), ctypes.byref(h)))
    return Stream(h, plan)


def jolt_decode(stream: Stream, K_out, V_out=None, cuda_stream=None):
    _check(_lib.jolt_decode(stream.handle, _dptr(K_out), _dptr(V_out), _stream_ptr(cuda_stream)))


def jolt_rel_frob_error(ref, approx, cuda_stream=None) -> float:
    if ref.shape != approx.shape or ref.dtype != approx.dtype:
        raise ValueError("ref and approx must share shape and dtype")
    out = ctypes.c_double()
    _check(_lib.jolt_rel_frob_error(_dptr(ref), _dptr(approx), ref.numel(), _dtype_code(ref),
                                    _stream_ptr(cuda_stream), ctypes.byref(out)))
    return out.value


def jolt_rel_frob_error_noalloc(ref, approx, cuda_stream=None) -> float:
    if ref.shape != approx.shape or ref.dtype != approx.dtype:
        raise ValueError("ref and approx must share shape and dtype")
    out = ctypes.c_double()
    _check(_lib.jolt_rel_frob_error_noalloc(_dptr(ref), _dptr(approx), ref.numel(), _dtype_code(ref),
                                            _stream_ptr(cuda_stream), ctypes.byref(out)))
    return out.value


def jolt_stream_status(stream: Stream):
    _check(_lib.jolt_stream_status(stream.handle))


def jolt_stream_info(stream: Stream, groups: int) -> dict:
    bp = (ctypes.c_uint64 * 5)()
    al = (ctypes.c_int32 * (groups * 6))()
    lam = (ctypes.c_double * 2)()
    _check(_lib.jolt_stream_info(stream.handle, bp, al, lam))
    return dict(bytes_by_part=dict(zip(PART_NAMES, list(bp))),
                alloc=np.array(list(al), dtype=np.int64).reshape(groups, 2, 3), lambdas=list(lam))


def jolt_stream_to_host(stream: Stream) -> bytes:
    n = ctypes.c_uint64()
    _check(_lib.jolt_stream_to_host(stream.handle, None, ctypes.byref(n)))
    buf = ctypes.create_string_buffer(n.value)
    _check(_lib.jolt_stream_to_host(stream.handle, buf, ctypes.byref(n)))
    return buf.raw[: n.value]


def jolt_stream_from_host(data: bytes, cuda_stream=None) -> Stream:
    h = ctypes.c_void_p()
    buf = ctypes.create_string_buffer(data, len(data))
    _check(_lib.jolt_stream_from_host(buf, len(data), _stream_ptr(cuda_stream), ctypes.byref(h)))
    return Stream(h)


def jolt_export_debug(stream: Stream, what: int, lt: int = 0) -> np.ndarray:
    n = ctypes.c_uint64()
    _check(_lib.jolt_export_debug(stream.handle, what, lt, None, ctypes.byref(n)))
    buf = ctypes.create_string_buffer(n.value)
    _check(_lib.jolt_export_debug(stream.handle, what, lt, buf, ctypes.byref(n)))
    raw = buf.raw[: n.value]
    if what in (JOLT_DBG_PI, JOLT_DBG_UT_F32, JOLT_DBG_UD_F32):
        return np.frombuffer(raw, dtype=np.float32).copy()
    if what == JOLT_DBG_OMEGA:
        return np.frombuffer(raw, dtype=np.uint16).copy()
    return np.frombuffer(raw, dtype=np.float64).copy()


def jolt_profile_enable(on: bool = True):
    _check(_lib.jolt_profile_enable(1 if on else 0))


def jolt_profile_report() -> dict:
    import json
    n = ctypes.c_uint64()
    _check(_lib.jolt_profile_report(None, ctypes.byref(n)))
    buf = ctypes.create_string_buffer(n.value)
    _check(_lib.jolt_profile_report(buf, ctypes.byref(n)))
    return json.loads(buf.value.decode())


def jolt_launch_count() -> int:
    return int(_lib.jolt_launch_count())


def jolt_alloc_count() -> int:
    return int(_lib.jolt_alloc_count())


def jolt_selftest_gemm_bf16(A, B, C, cuda_stream=None):
    """C = A B^T on the tensor cores; A [M][K], B [N][K] bf16, C [M][N] float32 (CUDA tensors)."""
    M, K = A.shape
    N = B.shape[0]
    _check(_lib.jolt_selftest_gemm_bf16(M, N, K, _dptr(A), _dptr(B), _dptr(C), _stream_ptr(cuda_stream)))


def jolt_selftest_gemm_bf16_layout(A, a_mn, B, b_mn, C, cuda_stream=None):
    """C = A B^T on the tensor cores with either operand stored transposed: A is [M][K] (a_mn
    false) or [K][M] (a_mn true), B is [N][K] or [K][N]; C [M][N] float32 (CUDA tensors)."""
    M, K = (A.shape[1], A.shape[0]) if a_mn else A.shape
    N = B.shape[1] if b_mn else B.shape[0]
    _check(_lib.jolt_selftest_gemm_bf16_layout(M, N, K, _dptr(A), int(bool(a_mn)), _dptr(B), int(bool(b_mn)),
                                               _dptr(C), _stream_ptr(cuda_stream)))


def jolt_selftest_eig_small(A, V, lam, solver=0, cuda_stream=None):
    """A: [batch][n][n] float64 CUDA tensor; V: [batch][n][n] and lam: [batch][n] float32 outputs."""
    _check(_lib.jolt_selftest_eig_small(int(A.shape[0]), int(A.shape[1]), _dptr(A), _dptr(V), _dptr(lam),
                                        int(solver), _stream_ptr(cuda_stream)))


def jolt_selftest_eig_dense(A, R, V, lam, cuda_stream=None):
    """A: [batch][n][n] float64 CUDA tensor; V: [batch][n][R] and lam: [batch][R] float64 outputs."""
    _check(_lib.jolt_selftest_eig_dense(int(A.shape[0]), int(A.shape[1]), int(R), _dptr(A), _dptr(V), _dptr(lam),
                                        _stream_ptr(cuda_stream)))


def jolt_attention(stream: Stream, Q, out, scale: float, cuda_stream=None):
    """Q: bf16 CUDA tensor [layers][q_heads][n][head_dim]; out: float32 CUDA tensor of the same shape."""
    if Q.dim() != 4 or tuple(out.shape) != tuple(Q.shape):
        raise ValueError("Q and out must be [layers][q_heads][n][head_dim] of the same shape")
    _check(_lib.jolt_attention(stream.handle, _dptr(Q), int(Q.shape[1]), int(Q.shape[2]), float(scale), _dptr(out),
                               _stream_ptr(cuda_stream)))
