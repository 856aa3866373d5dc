"""Seeded synthetic inputs for the layer: packed weights, activations, logits.

Host functions return numpy arrays; device functions fill torch CUDA
tensors with the same bytes (``synth_core.h`` states why they agree).
This module is the only one that serves both the CUDA library and the
CPU oracle; it holds no step of the layer forward.

Streams are named by a 64-bit tag: ``tag(kind, copy)``; matrix m of a bank
uses stream ``tag + m``.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_LIB_PATH = os.path.join(_PKG, "lib", "libmoeq_synth.so")
_lib = None

ROUTER, GATE, UP, DOWN, SH_GATE, SH_UP, SH_DOWN, SH_EXPERT_GATE, X, LOGITS, RESIDUAL = range(1, 12)


def tag(kind: int, copy: int = 0) -> int:
    return (int(kind) << 48) | (int(copy) << 32)


def _L():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            from .. import _build
            _build.build_synth()
        _lib = C.CDLL(_LIB_PATH)
        u64, i32, i64, P = C.c_uint64, C.c_int, C.c_int64, C.c_void_p
        _lib.moeq_synth_tensor_host.argtypes = [u64, u64, i32, i32, i32, i32, i32, i32, P, P, P,
                                                i32]
        _lib.moeq_synth_tensor_dev.argtypes = [u64, u64, i32, i32, i32, i32, i32, i32, P, P, P,
                                               P]
        _lib.moeq_synth_tensor_mx_host.argtypes = [u64, u64, i32, i32, i32, P, P, i32]
        _lib.moeq_synth_tensor_mx_dev.argtypes = [u64, u64, i32, i32, i32, P, P, P]
        _lib.moeq_synth_normal_bf16_host.argtypes = [u64, u64, i64, P, i32]
        _lib.moeq_synth_normal_bf16_dev.argtypes = [u64, u64, i64, P, P]
        _lib.moeq_synth_zipf_logits_host.argtypes = [u64, u64, i32, i32, C.c_double, P, P]
        _lib.moeq_synth_weights_f32_host.argtypes = [u64, u64, i32, i32, i32, P]
    return _lib


@dataclass
class HostQ:
    """Packed bank in host memory.  w: u32 [n_mats][out][in*bits/32];
    s, b: u16 (bf16 bits) [n_mats][out][in/G].  fmt 1 (MX FP4): s holds the
    u8 E8M0 exponents, b is empty."""
    w: np.ndarray
    s: np.ndarray
    b: np.ndarray
    out_dim: int
    in_dim: int
    bits: int
    group_size: int
    n_mats: int
    fmt: int = 0

    @property
    def nbytes(self) -> int:
        return self.w.nbytes + self.s.nbytes + self.b.nbytes

    def mat(self, m: int) -> "HostQ":
        return HostQ(self.w[m:m + 1], self.s[m:m + 1], self.b[m:m + 1] if self.fmt == 0 else self.b,
                     self.out_dim, self.in_dim, self.bits, self.group_size, 1, self.fmt)


@dataclass
class DevQ:
    """Packed bank in device memory (torch tensors; w int32 storage of u32,
    s/b int16 storage of bf16 bits; fmt 1 (MX FP4): s uint8 exponents, b
    empty)."""
    w: "object"
    s: "object"
    b: "object"
    out_dim: int
    in_dim: int
    bits: int
    group_size: int
    n_mats: int
    fmt: int = 0

    @property
    def nbytes(self) -> int:
        return (self.w.numel() * 4 + self.s.numel() * self.s.element_size() +
                self.b.numel() * self.b.element_size())

    @property
    def bytes_per_mat(self) -> int:
        return self.nbytes // self.n_mats

    def to_host(self) -> HostQ:
        sd = np.uint16 if self.fmt == 0 else np.uint8
        return HostQ(self.w.cpu().numpy().view(np.uint32), self.s.cpu().numpy().view(sd),
                     self.b.cpu().numpy().view(np.uint16), self.out_dim, self.in_dim, self.bits,
                     self.group_size, self.n_mats, self.fmt)


def tensor_mx_host(seed: int, tg: int, n_mats: int, out_dim: int, in_dim: int, threads: int = 0,
                   first_mat: int = 0) -> HostQ:
    """MX FP4 bank (4-bit E2M1 codes, one E8M0 byte per 32 values) from the
    same weight streams as tensor_host."""
    ws, ss = _shapes(n_mats, out_dim, in_dim, 4, 32)
    w = np.empty(ws, np.uint32)
    e = np.empty(ss, np.uint8)
    rc = _L().moeq_synth_tensor_mx_host(seed, tg + first_mat, n_mats, out_dim, in_dim,
                                        w.ctypes.data, e.ctypes.data, threads)
    if rc:
        raise ValueError(f"moeq_synth_tensor_mx_host rc={rc}")
    return HostQ(w, e, np.zeros(0, np.uint16), out_dim, in_dim, 4, 32, n_mats, 1)


def tensor_mx_dev(seed: int, tg: int, n_mats: int, out_dim: int, in_dim: int, device="cuda",
                  stream=None) -> DevQ:
    import torch
    ws, ss = _shapes(n_mats, out_dim, in_dim, 4, 32)
    w = torch.empty(ws, dtype=torch.int32, device=device)
    e = torch.empty(ss, dtype=torch.uint8, device=device)
    st = stream if stream is not None else torch.cuda.current_stream(device)
    rc = _L().moeq_synth_tensor_mx_dev(seed, tg, n_mats, out_dim, in_dim, w.data_ptr(),
                                       e.data_ptr(), st.cuda_stream)
    if rc:
        raise RuntimeError(f"moeq_synth_tensor_mx_dev rc={rc}")
    return DevQ(w, e, torch.zeros(0, dtype=torch.int16, device=device), out_dim, in_dim, 4, 32,
                n_mats, 1)


def packed_bytes(out_dim: int, in_dim: int, bits: int, group_size: int = 64) -> int:
    """Bytes of one packed matrix: codes + bf16 scale + bf16 bias per group."""
    return out_dim * in_dim * bits // 8 + 2 * 2 * out_dim * (in_dim // group_size)


def _shapes(n_mats, out_dim, in_dim, bits, G):
    if (in_dim * bits) % 32 or in_dim % G:
        raise ValueError("in_dim must fill whole words and whole groups")
    return (n_mats, out_dim, in_dim * bits // 32), (n_mats, out_dim, in_dim // G)


def tensor_host(seed: int, tg: int, n_mats: int, out_dim: int, in_dim: int, bits: int,
                group_size: int = 64, requant_from4: bool = False, threads: int = 0,
                first_mat: int = 0) -> HostQ:
    """Matrices first_mat .. first_mat+n_mats-1 of the bank with stream tag tg."""
    ws, ss = _shapes(n_mats, out_dim, in_dim, bits, group_size)
    w = np.empty(ws, np.uint32)
    s = np.empty(ss, np.uint16)
    b = np.empty(ss, np.uint16)
    rc = _L().moeq_synth_tensor_host(seed, tg + first_mat, n_mats, out_dim, in_dim, bits,
                                     group_size, int(requant_from4), w.ctypes.data,
                                     s.ctypes.data, b.ctypes.data, threads)
    if rc:
        raise ValueError(f"moeq_synth_tensor_host rc={rc}")
    return HostQ(w, s, b, out_dim, in_dim, bits, group_size, n_mats)


def tensor_dev(seed: int, tg: int, n_mats: int, out_dim: int, in_dim: int, bits: int,
               group_size: int = 64, requant_from4: bool = False, device="cuda",
               stream=None) -> DevQ:
    import torch
    ws, ss = _shapes(n_mats, out_dim, in_dim, bits, group_size)
    w = torch.empty(ws, dtype=torch.int32, device=device)
    s = torch.empty(ss, dtype=torch.int16, device=device)
    b = torch.empty(ss, dtype=torch.int16, device=device)
    st = stream if stream is not None else torch.cuda.current_stream(device)
    rc = _L().moeq_synth_tensor_dev(seed, tg, n_mats, out_dim, in_dim, bits, group_size,
                                    int(requant_from4), w.data_ptr(), s.data_ptr(), b.data_ptr(),
                                    st.cuda_stream)
    if rc:
        raise RuntimeError(f"moeq_synth_tensor_dev rc={rc}")
    return DevQ(w, s, b, out_dim, in_dim, bits, group_size, n_mats)


def normal_bf16_host(seed: int, tg: int, n: int, threads: int = 0) -> np.ndarray:
    out = np.empty(n, np.uint16)
    rc = _L().moeq_synth_normal_bf16_host(seed, tg, n, out.ctypes.data, threads)
    if rc:
        raise ValueError(f"moeq_synth_normal_bf16_host rc={rc}")
    return out


def normal_bf16_dev(seed: int, tg: int, n: int, device="cuda", stream=None):
    """bf16 tensor of n values (same bits as normal_bf16_host)."""
    import torch
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    st = stream if stream is not None else torch.cuda.current_stream(device)
    rc = _L().moeq_synth_normal_bf16_dev(seed, tg, n, out.data_ptr(), st.cuda_stream)
    if rc:
        raise RuntimeError(f"moeq_synth_normal_bf16_dev rc={rc}")
    return out


def zipf_logits_host(seed: int, tg: int, M: int, E: int, zipf_s: float = 1.1):
    """fp32 [M][E] logits ln p_e + Gumbel, p_e ~ rank^-zipf_s; also the ranks."""
    logits = np.empty((M, E), np.float32)
    rank = np.empty(E, np.int32)
    rc = _L().moeq_synth_zipf_logits_host(seed, tg, M, E, float(zipf_s), logits.ctypes.data,
                                          rank.ctypes.data)
    if rc:
        raise ValueError(f"moeq_synth_zipf_logits_host rc={rc}")
    return logits, rank


def weights_f32_host(seed: int, tg: int, mat: int, out_dim: int, in_dim: int) -> np.ndarray:
    """The fp32 draws of one matrix before quantisation, [out][in]."""
    w = np.empty((out_dim, in_dim), np.float32)
    rc = _L().moeq_synth_weights_f32_host(seed, tg, mat, out_dim, in_dim, w.ctypes.data)
    if rc:
        raise ValueError(f"moeq_synth_weights_f32_host rc={rc}")
    return w


def bf16_bits_to_f32(x: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp32."""
    return (np.asarray(x, np.uint16).astype(np.uint32) << 16).view(np.float32)
