"""Python binding of libmoeq.so (include/moeq.h): argument marshalling only.

Every function here forwards to the C entry point of the same name; device
buffers are passed as torch CUDA tensors (their data pointers) and streams
as torch streams.  There is no fallback: if the library is missing this
module fails to import, and a non-OK status raises MoeqError.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libmoeq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python -m quantized_mixture_experts_affine_b200._build`"
                      " (nvcc, sm_100a) before using the layer library")

_lib = C.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, \
    ERR_RANGE = range(8)
MODE_AUTO, MODE_DECODE, MODE_PREFILL = 0, 1, 2

EXPORTS = ("moeq_dequant", "moeq_qmv", "moeq_route_topk", "moeq_expert_ffn", "moeq_layer_forward",
           "moeq_workspace_bytes", "moeq_device_status", "moeq_status_str", "moeq_version",
           "moeq_set_profile_events", "moeq_launch_count", "moeq_layer_forward_static",
           "moeq_static_workspace_capacity", "moeq_selftest_wait_timeout",
           "moeq_layer_forward_norm", "moeq_cache_create", "moeq_cache_workspace_bytes",
           "moeq_cache_forward", "moeq_cache_stats", "moeq_cache_destroy")


class MoeqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_str(status)} (status {status})")


class QTensor(C.Structure):
    """moeq_qtensor."""
    _fields_ = [("w", C.c_void_p), ("scales", C.c_void_p), ("biases", C.c_void_p),
                ("out_dim", C.c_int32), ("in_dim", C.c_int32), ("bits", C.c_int32),
                ("group_size", C.c_int32), ("expert_stride_w", C.c_int64),
                ("expert_stride_sb", C.c_int64), ("format", C.c_int32)]


class Layer(C.Structure):
    """moeq_layer."""
    _fields_ = [("router", QTensor), ("gate", QTensor), ("up", QTensor), ("down", QTensor),
                ("has_shared", C.c_int32), ("sh_gate", QTensor), ("sh_up", QTensor),
                ("sh_down", QTensor), ("sh_expert_gate", QTensor), ("hidden", C.c_int32),
                ("inter", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("renorm", C.c_int32), ("router_scale", C.c_float)]


_P = C.c_void_p
_lib.moeq_dequant.argtypes = [C.POINTER(QTensor), C.c_int32, _P, _P, _P]
_lib.moeq_qmv.argtypes = [C.POINTER(QTensor), C.c_int32, _P, C.c_int32, _P, _P]
_lib.moeq_route_topk.argtypes = [_P, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_float, _P,
                                 _P, _P]
_lib.moeq_expert_ffn.argtypes = [C.POINTER(Layer), _P, C.c_int32, _P, _P, _P, _P, _P, C.c_size_t,
                                 C.c_int32, _P]
_lib.moeq_layer_forward.argtypes = [C.POINTER(Layer), _P, C.c_int32, _P, _P, _P, _P, _P,
                                    C.c_size_t, C.c_int32, _P]
_lib.moeq_layer_forward_static.argtypes = [C.POINTER(Layer), _P, C.c_int32, _P, _P, _P, _P, _P]
_lib.moeq_cache_create.argtypes = [C.POINTER(Layer), C.c_int32, C.c_int32, C.POINTER(C.c_void_p)]
_lib.moeq_cache_create.restype = C.c_int
_lib.moeq_cache_workspace_bytes.argtypes = [C.c_void_p, C.c_int32]
_lib.moeq_cache_workspace_bytes.restype = C.c_size_t
_lib.moeq_cache_forward.argtypes = [C.c_void_p, _P, C.c_int32, _P, _P, _P, _P, _P, C.c_size_t, _P]
_lib.moeq_cache_forward.restype = C.c_int
_lib.moeq_cache_stats.argtypes = [C.c_void_p, C.POINTER(C.c_uint64), C.POINTER(C.c_uint64),
                                  C.POINTER(C.c_uint64)]
_lib.moeq_cache_stats.restype = C.c_int
_lib.moeq_cache_destroy.argtypes = [C.c_void_p]
_lib.moeq_cache_destroy.restype = None
_lib.moeq_layer_forward_norm.argtypes = [C.POINTER(Layer), _P, C.c_int32, _P, _P, _P, C.c_float,
                                         _P, _P, _P, _P, C.c_size_t, C.c_int32, _P]
_lib.moeq_static_workspace_capacity.restype = C.c_size_t
_lib.moeq_workspace_bytes.argtypes = [C.POINTER(Layer), C.c_int32, C.c_int32]
_lib.moeq_workspace_bytes.restype = C.c_size_t
_lib.moeq_device_status.argtypes = [_P, C.POINTER(C.c_int32)]
_lib.moeq_selftest_wait_timeout.argtypes = [_P]
_lib.moeq_status_str.argtypes = [C.c_int32]
_lib.moeq_status_str.restype = C.c_char_p
_lib.moeq_version.restype = C.c_char_p
_lib.moeq_set_profile_events.argtypes = [_P, _P]
_lib.moeq_set_profile_events.restype = C.c_int
_lib.moeq_launch_count.restype = C.c_uint64
for _f in ("moeq_dequant", "moeq_qmv", "moeq_route_topk", "moeq_expert_ffn", "moeq_layer_forward",
           "moeq_layer_forward_static", "moeq_device_status", "moeq_selftest_wait_timeout",
           "moeq_layer_forward_norm"):
    getattr(_lib, _f).restype = C.c_int


def lib() -> C.CDLL:
    return _lib


def status_str(status: int) -> str:
    return _lib.moeq_status_str(int(status)).decode()


def version() -> str:
    return _lib.moeq_version().decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, rc):
    if rc != OK:
        raise MoeqError(fn, rc)


FMT_AFFINE, FMT_MXFP4 = 0, 1


def qtensor(w, scales, biases, out_dim, in_dim, bits, group_size=64, n_mats=1,
            fmt: int = FMT_AFFINE) -> QTensor:
    """Descriptor of a bank of n_mats packed matrices stored back to back
    (MX FP4: scales are the uint8 exponents, biases unused)."""
    sw = out_dim * in_dim * bits // 32 if n_mats > 1 else 0
    ssb = out_dim * (in_dim // group_size) if n_mats > 1 else 0
    return QTensor(_ptr(w), _ptr(scales), _ptr(biases) if fmt == FMT_AFFINE else None, out_dim,
                   in_dim, bits, group_size, sw, ssb, fmt)


def moeq_dequant(t: QTensor, expert: int, q_out=None, w_out=None, stream=None) -> None:
    _check("moeq_dequant", _lib.moeq_dequant(C.byref(t), expert, _ptr(q_out), _ptr(w_out),
                                             _stream(stream)))


def moeq_qmv(t: QTensor, expert: int, x, M: int, y, stream=None) -> None:
    _check("moeq_qmv", _lib.moeq_qmv(C.byref(t), expert, _ptr(x), M, _ptr(y), _stream(stream)))


def moeq_route_topk(logits, M: int, E: int, K: int, renorm: bool, router_scale: float, idx, w,
                    stream=None) -> None:
    _check("moeq_route_topk", _lib.moeq_route_topk(_ptr(logits), M, E, K, int(renorm),
                                                   float(router_scale), _ptr(idx), _ptr(w),
                                                   _stream(stream)))


def moeq_workspace_bytes(L: Layer, M: int, mode: int = MODE_AUTO) -> int:
    return int(_lib.moeq_workspace_bytes(C.byref(L), M, mode))


def moeq_expert_ffn(L: Layer, x, M: int, idx, w, residual, y, ws, ws_bytes: int,
                    mode: int = MODE_AUTO, stream=None) -> None:
    _check("moeq_expert_ffn", _lib.moeq_expert_ffn(C.byref(L), _ptr(x), M, _ptr(idx), _ptr(w),
                                                   _ptr(residual), _ptr(y), _ptr(ws), ws_bytes,
                                                   mode, _stream(stream)))


def moeq_layer_forward(L: Layer, x, M: int, y, residual=None, idx_out=None, w_out=None, ws=None,
                       ws_bytes: int = 0, mode: int = MODE_AUTO, stream=None) -> None:
    _check("moeq_layer_forward",
           _lib.moeq_layer_forward(C.byref(L), _ptr(x), M, _ptr(y), _ptr(residual),
                                   _ptr(idx_out), _ptr(w_out), _ptr(ws), ws_bytes, mode,
                                   _stream(stream)))


def moeq_layer_forward_norm(L: Layer, x, M: int, y, gamma, eps: float, y_norm, residual=None,
                            idx_out=None, w_out=None, ws=None, ws_bytes: int = 0,
                            mode: int = MODE_AUTO, stream=None) -> None:
    """moeq_layer_forward plus y_norm = bf16 RMS norm of y with weights gamma."""
    _check("moeq_layer_forward_norm",
           _lib.moeq_layer_forward_norm(C.byref(L), _ptr(x), M, _ptr(y), _ptr(residual),
                                        _ptr(gamma), float(eps), _ptr(y_norm), _ptr(idx_out),
                                        _ptr(w_out), _ptr(ws), ws_bytes, mode, _stream(stream)))


def moeq_layer_forward_static(L: Layer, x, M: int, y, residual=None, idx_out=None, w_out=None,
                              stream=None) -> None:
    """Decode layer forward on the library's fixed per-device workspace."""
    _check("moeq_layer_forward_static",
           _lib.moeq_layer_forward_static(C.byref(L), _ptr(x), M, _ptr(y), _ptr(residual),
                                          _ptr(idx_out), _ptr(w_out), _stream(stream)))


def moeq_static_workspace_capacity() -> int:
    return int(_lib.moeq_static_workspace_capacity())


def moeq_set_profile_events(start=None, stop=None) -> None:
    """start/stop: torch.cuda.Event (or None to turn profiling off)."""
    _check("moeq_set_profile_events",
           _lib.moeq_set_profile_events(None if start is None else start.cuda_event,
                                        None if stop is None else stop.cuda_event))


def moeq_launch_count() -> int:
    return int(_lib.moeq_launch_count())


def moeq_selftest_wait_timeout(stream=None) -> None:
    _check("moeq_selftest_wait_timeout", _lib.moeq_selftest_wait_timeout(_stream(stream)))


def moeq_device_status(stream=None) -> int:
    v = C.c_int32(0)
    _check("moeq_device_status", _lib.moeq_device_status(_stream(stream), C.byref(v)))
    return int(v.value)


class ExpertCache:
    """moeq_expert_cache: routed expert banks in host memory, `slots` of
    them cached in HBM (see include/moeq.h).  Keeps the layer descriptor
    alive; frees the cache on close()."""

    def __init__(self, L: Layer, slots: int, max_tokens: int):
        self._L = L
        self._h = C.c_void_p()
        _check("moeq_cache_create", _lib.moeq_cache_create(C.byref(L), slots, max_tokens,
                                                           C.byref(self._h)))

    def workspace_bytes(self, M: int) -> int:
        return int(_lib.moeq_cache_workspace_bytes(self._h, M))

    def forward(self, x, M: int, y, ws, ws_bytes: int, residual=None, idx_out=None, w_out=None,
                stream=None) -> None:
        _check("moeq_cache_forward",
               _lib.moeq_cache_forward(self._h, _ptr(x), M, _ptr(y), _ptr(residual),
                                       _ptr(idx_out), _ptr(w_out), _ptr(ws), ws_bytes,
                                       _stream(stream)))

    def stats(self):
        h, m, b = C.c_uint64(), C.c_uint64(), C.c_uint64()
        _check("moeq_cache_stats", _lib.moeq_cache_stats(self._h, C.byref(h), C.byref(m),
                                                         C.byref(b)))
        return int(h.value), int(m.value), int(b.value)

    def close(self) -> None:
        if self._h:
            _lib.moeq_cache_destroy(self._h)
            self._h = C.c_void_p()
