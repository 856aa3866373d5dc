"""ctypes wrapper of the C oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
Arguments are numpy arrays in host memory; nothing here touches a GPU.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def lib_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2, no fp contraction, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Tensor(C.Structure):
    _fields_ = [("w", C.c_void_p), ("s", C.c_void_p), ("b", C.c_void_p),
                ("out", C.c_int32), ("inn", C.c_int32), ("bits", C.c_int32), ("G", C.c_int32),
                ("stride_w", C.c_int64), ("stride_sb", C.c_int64), ("format", C.c_int32)]


class _Layer(C.Structure):
    _fields_ = [("router", _Tensor), ("gate", _Tensor), ("up", _Tensor), ("down", _Tensor),
                ("has_shared", C.c_int32),
                ("sh_gate", _Tensor), ("sh_up", _Tensor), ("sh_down", _Tensor),
                ("sh_expert_gate", _Tensor),
                ("H", C.c_int32), ("I", C.c_int32), ("E", C.c_int32), ("K", C.c_int32),
                ("renorm", C.c_int32), ("router_scale", C.c_double)]


@dataclass
class OracleTensor:
    """Packed tensor (or bank) in host memory: w [mats][out][in*bits/32] u32,
    s/b [mats][out][in/G] bf16 bits (u16)."""
    w: np.ndarray
    s: np.ndarray
    b: np.ndarray
    out_dim: int
    in_dim: int
    bits: int
    group_size: int
    fmt: int = 0   # 0 affine; 1 MX FP4 (s: uint8 E8M0 exponents, b unused)

    @classmethod
    def of(cls, t) -> "OracleTensor":
        """Accept any object with the same attribute names (e.g. a generated tensor)."""
        return cls(t.w, t.s, t.b, t.out_dim, t.in_dim, t.bits, t.group_size,
                   getattr(t, "fmt", 0))

    def _c(self) -> _Tensor:
        sdt = np.uint16 if self.fmt == 0 else np.uint8
        arrays = ((self.w, np.uint32), (self.s, sdt)) + (((self.b, np.uint16),) if self.fmt == 0
                                                         else ())
        for a, dt in arrays:
            assert a.dtype == dt and a.flags.c_contiguous, (a.dtype, dt)
        wpr = self.in_dim * self.bits // 32
        gpr = self.in_dim // self.group_size
        return _Tensor(self.w.ctypes.data, self.s.ctypes.data,
                       self.b.ctypes.data if self.fmt == 0 else None,
                       self.out_dim, self.in_dim, self.bits, self.group_size,
                       self.out_dim * wpr, self.out_dim * gpr, self.fmt)

    @property
    def n_mats(self) -> int:
        return self.w.size // (self.out_dim * self.in_dim * self.bits // 32)


@dataclass
class OracleLayer:
    router: OracleTensor
    gate: OracleTensor
    up: OracleTensor
    down: OracleTensor
    H: int
    I: int
    E: int
    K: int
    renorm: bool = True
    router_scale: float = 1.0
    sh_gate: OracleTensor | None = None
    sh_up: OracleTensor | None = None
    sh_down: OracleTensor | None = None
    sh_expert_gate: OracleTensor | None = None

    def _c(self) -> _Layer:
        has = self.sh_gate is not None
        z = _Tensor()
        return _Layer(self.router._c(), self.gate._c(), self.up._c(), self.down._c(), int(has),
                      self.sh_gate._c() if has else z, self.sh_up._c() if has else z,
                      self.sh_down._c() if has else z, self.sh_expert_gate._c() if has else z,
                      self.H, self.I, self.E, self.K, int(self.renorm), float(self.router_scale))


def _L():
    global _lib
    if _lib is None:
        build()
        _lib = C.CDLL(_LIB)
        P = C.c_void_p
        _lib.oracle_set_threads.argtypes = [C.c_int]
        _lib.oracle_get_threads.restype = C.c_int
        _lib.oracle_unpack.argtypes = [C.POINTER(_Tensor), C.c_int, P]
        _lib.oracle_dequant_f32.argtypes = [C.POINTER(_Tensor), C.c_int, P]
        _lib.oracle_qmv.argtypes = [C.POINTER(_Tensor), C.c_int, P, C.c_int, P]
        _lib.oracle_qmv_f64.argtypes = [C.POINTER(_Tensor), C.c_int, P, C.c_int, P]
        _lib.oracle_route.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_double, P, P, P]
        _lib.oracle_route_f32.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_double, P,
                                          P, P]
        _lib.oracle_expert_ffn.argtypes = [C.POINTER(_Layer), P, C.c_int, P, P, P, P]
        _lib.oracle_layer.argtypes = [C.POINTER(_Layer), P, C.c_int, P, P, P, P, P, P]
        _lib.oracle_rmsnorm.argtypes = [P, C.c_int, C.c_int, P, C.c_double, P]
    return _lib


def set_threads(n: int) -> None:
    _L().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_L().oracle_get_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data


def unpack(t, mat: int = 0) -> np.ndarray:
    t = OracleTensor.of(t)
    q = np.empty((t.out_dim, t.in_dim), np.uint8)
    _L().oracle_unpack(C.byref(t._c()), mat, _ptr(q))
    return q


def dequant_f32(t, mat: int = 0) -> np.ndarray:
    t = OracleTensor.of(t)
    w = np.empty((t.out_dim, t.in_dim), np.float32)
    _L().oracle_dequant_f32(C.byref(t._c()), mat, _ptr(w))
    return w


def qmv(t, x_bf16: np.ndarray, mat: int = 0) -> np.ndarray:
    """x_bf16: uint16 [M][in] (bf16 bits).  Returns fp64 [M][out]."""
    t = OracleTensor.of(t)
    x = np.ascontiguousarray(x_bf16, np.uint16).reshape(-1, t.in_dim)
    y = np.empty((x.shape[0], t.out_dim), np.float64)
    _L().oracle_qmv(C.byref(t._c()), mat, _ptr(x), x.shape[0], _ptr(y))
    return y


def qmv_f64(t, x: np.ndarray, mat: int = 0) -> np.ndarray:
    t = OracleTensor.of(t)
    x = np.ascontiguousarray(x, np.float64).reshape(-1, t.in_dim)
    y = np.empty((x.shape[0], t.out_dim), np.float64)
    _L().oracle_qmv_f64(C.byref(t._c()), mat, _ptr(x), x.shape[0], _ptr(y))
    return y


def route(logits: np.ndarray, K: int, renorm: bool = True, router_scale: float = 1.0):
    """logits fp64 [M][E] -> (idx int32 [M][K], w fp64 [M][K], gap fp64 [M])."""
    l = np.ascontiguousarray(logits, np.float64)
    M, E = l.shape
    idx = np.empty((M, K), np.int32)
    w = np.empty((M, K), np.float64)
    gap = np.empty(M, np.float64)
    _L().oracle_route(_ptr(l), M, E, K, int(renorm), float(router_scale), _ptr(idx), _ptr(w),
                      _ptr(gap))
    return idx, w, gap


def route_f32(logits: np.ndarray, K: int, renorm: bool = True, router_scale: float = 1.0):
    l = np.ascontiguousarray(logits, np.float32)
    M, E = l.shape
    idx = np.empty((M, K), np.int32)
    w = np.empty((M, K), np.float64)
    gap = np.empty(M, np.float64)
    _L().oracle_route_f32(_ptr(l), M, E, K, int(renorm), float(router_scale), _ptr(idx),
                          _ptr(w), _ptr(gap))
    return idx, w, gap


def expert_ffn(L: OracleLayer, x_bf16: np.ndarray, idx: np.ndarray, w: np.ndarray,
               residual: np.ndarray | None = None) -> np.ndarray:
    x = np.ascontiguousarray(x_bf16, np.uint16).reshape(-1, L.H)
    M = x.shape[0]
    idx = np.ascontiguousarray(idx, np.int32).reshape(M, L.K)
    w = np.ascontiguousarray(w, np.float64).reshape(M, L.K)
    res = None if residual is None else np.ascontiguousarray(residual, np.float32).reshape(M, L.H)
    out = np.empty((M, L.H), np.float64)
    cl = L._c()
    _L().oracle_expert_ffn(C.byref(cl), _ptr(x), M, _ptr(idx), _ptr(w), _ptr(res), _ptr(out))
    return out


def layer(L: OracleLayer, x_bf16: np.ndarray, residual: np.ndarray | None = None):
    """Full layer.  Returns dict(out fp64 [M][H], idx, w, gap, logits)."""
    x = np.ascontiguousarray(x_bf16, np.uint16).reshape(-1, L.H)
    M = x.shape[0]
    res = None if residual is None else np.ascontiguousarray(residual, np.float32).reshape(M, L.H)
    out = np.empty((M, L.H), np.float64)
    idx = np.empty((M, L.K), np.int32)
    w = np.empty((M, L.K), np.float64)
    gap = np.empty(M, np.float64)
    logits = np.empty((M, L.E), np.float64)
    cl = L._c()
    _L().oracle_layer(C.byref(cl), _ptr(x), M, _ptr(res), _ptr(out), _ptr(idx), _ptr(w),
                      _ptr(gap), _ptr(logits))
    return dict(out=out, idx=idx, w=w, gap=gap, logits=logits)


def rmsnorm(y: np.ndarray, gamma_bf16: np.ndarray, eps: float) -> np.ndarray:
    """RMS norm of each row of y (fp64 [M][H]) with the bf16 weights gamma
    ([H] bit patterns): y / sqrt(mean(y^2) + eps) * gamma, in fp64."""
    y = np.ascontiguousarray(y, np.float64)
    M, H = y.reshape(-1, y.shape[-1]).shape
    g = np.ascontiguousarray(gamma_bf16, np.uint16).reshape(H)
    out = np.empty((M, H), np.float64)
    _L().oracle_rmsnorm(_ptr(y), M, H, _ptr(g), float(eps), _ptr(out))
    return out
