"""The C ABI loads, exports every declared symbol, and rejects bad arguments
on the host before launching anything (no GPU needed: every call here fails
its argument checks; fake device addresses are never dereferenced)."""
import ctypes as C
import os
import re

import pytest

from quantized_mixture_experts_affine_b200 import moeq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moeq.h")

A = 1 << 20  # fake, 256-byte aligned device address (never dereferenced)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moeq_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert set(moeq.EXPORTS) <= set(names) and len(names) >= 9
    lib = C.CDLL(moeq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for s in range(8):
        assert moeq.status_str(s) and moeq.status_str(s) != "unknown status"
    assert moeq.status_str(99) == "unknown status"
    assert "sm_100a" in moeq.version()


def qt(out=128, inn=256, bits=4, G=64, w=A, s=A, b=A, n_mats=1):
    return moeq.qtensor(w, s, b, out, inn, bits, G, n_mats)


def rc_qmv(t, M=1, x=A, y=A, expert=0):
    return moeq.lib().moeq_qmv(C.byref(t), expert, x, M, y, None)


def test_qmv_argument_checks():
    assert rc_qmv(qt(bits=7)) == moeq.ERR_UNSUPPORTED
    assert rc_qmv(qt(bits=1)) == moeq.ERR_UNSUPPORTED
    assert rc_qmv(qt(bits=5, inn=192)) == moeq.ERR_ALIGNMENT      # 5-bit rows: in_dim % 128
    assert rc_qmv(qt(bits=3, inn=192)) == moeq.ERR_ALIGNMENT      # 3-bit rows: in_dim % 128
    assert rc_qmv(qt(bits=6, inn=96, G=32)) == moeq.ERR_ALIGNMENT  # 6-bit rows: in_dim % 64
    assert rc_qmv(qt(G=48)) == moeq.ERR_UNSUPPORTED
    assert rc_qmv(qt(inn=96, G=64)) == moeq.ERR_ALIGNMENT
    assert rc_qmv(qt(w=A + 4)) == moeq.ERR_ALIGNMENT
    assert rc_qmv(qt(), x=A + 2) == moeq.ERR_ALIGNMENT
    assert rc_qmv(qt(w=0)) == moeq.ERR_INVALID_ARG
    assert rc_qmv(qt(), M=0) == moeq.ERR_INVALID_ARG
    assert rc_qmv(qt(), M=65) == moeq.ERR_UNSUPPORTED
    assert rc_qmv(qt(), expert=-1) == moeq.ERR_INVALID_ARG
    assert rc_qmv(qt(inn=16384, bits=8)) == moeq.ERR_UNSUPPORTED   # > 8 slices of 512 B
    assert moeq.lib().moeq_qmv(None, 0, A, 1, A, None) == moeq.ERR_INVALID_ARG


def test_dequant_argument_checks():
    lib = moeq.lib()
    assert lib.moeq_dequant(C.byref(qt()), 0, None, None, None) == moeq.ERR_INVALID_ARG
    assert lib.moeq_dequant(C.byref(qt(bits=7)), 0, A, None, None) == moeq.ERR_UNSUPPORTED
    # expert > 0 needs expert strides
    assert lib.moeq_dequant(C.byref(qt()), 1, A, None, None) == moeq.ERR_INVALID_ARG


def test_route_argument_checks():
    lib = moeq.lib()
    assert lib.moeq_route_topk(A, 4, 8, 9, 1, 1.0, A, A, None) == moeq.ERR_INVALID_ARG
    assert lib.moeq_route_topk(A, 4, 64, 33, 1, 1.0, A, A, None) == moeq.ERR_UNSUPPORTED
    assert lib.moeq_route_topk(A, 4, 5000, 4, 1, 1.0, A, A, None) == moeq.ERR_UNSUPPORTED
    assert lib.moeq_route_topk(A, -1, 8, 2, 1, 1.0, A, A, None) == moeq.ERR_INVALID_ARG
    assert lib.moeq_route_topk(A, 0, 8, 2, 1, 1.0, None, None, None) == moeq.OK  # nothing to do
    assert lib.moeq_route_topk(None, 3, 8, 2, 1, 1.0, A, A, None) == moeq.ERR_INVALID_ARG


def layer(H=256, I=128, E=8, K=2, bits=4, shared=False):
    L = moeq.Layer()
    L.router = qt(E, H, 8)
    L.gate = qt(I, H, bits, n_mats=E)
    L.up = qt(I, H, bits, n_mats=E)
    L.down = qt(H, I, bits, n_mats=E)
    L.has_shared = int(shared)
    if shared:
        L.sh_gate, L.sh_up, L.sh_down = qt(I, H, bits), qt(I, H, bits), qt(H, I, bits)
        L.sh_expert_gate = qt(1, H, 8)
    L.hidden, L.inter, L.n_experts, L.top_k, L.renorm, L.router_scale = H, I, E, K, 1, 1.0
    return L


def test_workspace_bytes():
    L = layer()
    assert moeq.moeq_workspace_bytes(L, 1, moeq.MODE_DECODE) > 0
    assert moeq.moeq_workspace_bytes(L, 65, moeq.MODE_DECODE) == 0
    assert moeq.moeq_workspace_bytes(L, 0, moeq.MODE_DECODE) == 0
    Ls = layer(shared=True)
    assert moeq.moeq_workspace_bytes(Ls, 5, moeq.MODE_DECODE) > moeq.moeq_workspace_bytes(L, 5, moeq.MODE_DECODE)
    bad = layer()
    bad.top_k = 9
    assert moeq.moeq_workspace_bytes(bad, 1, moeq.MODE_DECODE) == 0
    bad = layer()
    bad.down = qt(255, 128, 4, n_mats=8)  # down must be [H][I]
    assert moeq.moeq_workspace_bytes(bad, 1, moeq.MODE_DECODE) == 0


def fwd(L, M=1, x=A, y=A, ws=A, ws_bytes=None, mode=moeq.MODE_DECODE):
    if ws_bytes is None:
        ws_bytes = moeq.moeq_workspace_bytes(L, max(M, 1), mode) - 256
    return moeq.lib().moeq_layer_forward(C.byref(L), x, M, y, None, None, None, ws, ws_bytes,
                                         mode, None)


def test_forward_argument_checks():
    L = layer()
    assert fwd(L) == moeq.ERR_WORKSPACE                 # workspace too small
    assert fwd(L, ws=None, ws_bytes=1 << 30) == moeq.ERR_WORKSPACE
    assert fwd(L, x=A + 2, ws_bytes=1 << 30) == moeq.ERR_ALIGNMENT
    assert fwd(L, ws=A + 16, ws_bytes=1 << 30) == moeq.ERR_ALIGNMENT
    assert fwd(L, mode=7, ws_bytes=1 << 30) == moeq.ERR_INVALID_ARG
    assert fwd(L, M=0) == moeq.OK                       # nothing to do
    assert fwd(L, M=-1) == moeq.ERR_INVALID_ARG
    assert fwd(L, M=65, ws_bytes=1 << 30) == moeq.ERR_UNSUPPORTED  # decode limit
    bad = layer()
    bad.gate = qt(128, 256, 3, n_mats=8)
    assert fwd(bad, ws_bytes=1 << 30) == moeq.ERR_UNSUPPORTED
    bad = layer()
    bad.n_experts = 4                                    # router rows != E
    assert fwd(bad, ws_bytes=1 << 30) == moeq.ERR_INVALID_ARG
    lib = moeq.lib()
    # expert_ffn needs the routing
    assert lib.moeq_expert_ffn(C.byref(L), A, 2, None, None, None, A, A, 1 << 30,
                               moeq.MODE_DECODE, None) == moeq.ERR_INVALID_ARG


def test_device_status_needs_output():
    assert moeq.lib().moeq_device_status(None, None) == moeq.ERR_INVALID_ARG


def fwd_static(L, M=1, x=A, y=A, residual=None):
    return moeq.lib().moeq_layer_forward_static(C.byref(L), x, M, y, residual, None, None, None)


def test_static_entry_checks_arguments_before_capacity():
    """The fixed-workspace entry runs moeq_layer_forward's argument checks
    before its capacity check: an oversized layer with a bad pointer reports
    the pointer, not the workspace."""
    big = layer(H=8192, I=2048, E=512, K=8)
    assert moeq.moeq_workspace_bytes(big, 64, moeq.MODE_DECODE) > \
        moeq.moeq_static_workspace_capacity()
    assert fwd_static(big, M=64, x=0) == moeq.ERR_INVALID_ARG
    assert fwd_static(big, M=64, y=0) == moeq.ERR_INVALID_ARG
    assert fwd_static(big, M=64, x=A + 2) == moeq.ERR_ALIGNMENT
    assert fwd_static(big, M=64, y=A + 4) == moeq.ERR_ALIGNMENT
    assert fwd_static(big, M=64, residual=A + 8) == moeq.ERR_ALIGNMENT
    assert fwd_static(big, M=-1) == moeq.ERR_INVALID_ARG
    bad = layer()
    bad.n_experts = 4
    assert fwd_static(bad) == moeq.ERR_INVALID_ARG
    assert fwd_static(big, M=0) == moeq.OK
    # valid pointers: now the capacity decides (nothing launched, no device needed)
    assert fwd_static(big, M=64) == moeq.ERR_WORKSPACE
    assert fwd_static(layer(), M=65) == moeq.ERR_UNSUPPORTED


def test_norm_entry_argument_checks():
    """moeq_layer_forward_norm: the forward's checks first, then gamma,
    y_norm and eps; nothing is launched on a failed check."""
    L = layer()
    f = moeq.lib().moeq_layer_forward_norm

    def call(x=A, y=A, gamma=A, eps=1e-6, y_norm=A, M=1):
        return f(C.byref(L), x, M, y, None, gamma, eps, y_norm, None, None, A, 1 << 30,
                 moeq.MODE_DECODE, None)
    assert call(x=0) == moeq.ERR_INVALID_ARG
    assert call(gamma=0) == moeq.ERR_INVALID_ARG
    assert call(y_norm=0) == moeq.ERR_INVALID_ARG
    assert call(eps=0.0) == moeq.ERR_INVALID_ARG
    assert call(eps=-1.0) == moeq.ERR_INVALID_ARG
    assert call(eps=float("inf")) == moeq.ERR_INVALID_ARG
    assert call(eps=float("nan")) == moeq.ERR_INVALID_ARG
    assert call(gamma=A + 2) == moeq.ERR_ALIGNMENT
    assert call(y_norm=A + 8) == moeq.ERR_ALIGNMENT
    assert call(M=0, gamma=0) == moeq.OK


def test_cache_create_argument_checks():
    """moeq_cache_create refuses before touching the device: a missing
    layer or output, slots outside [K, E], too many tokens for the slots."""
    f = moeq.lib().moeq_cache_create
    L = layer(E=8, K=2)
    h = C.c_void_p()
    assert f(None, 4, 1, C.byref(h)) == moeq.ERR_INVALID_ARG
    assert f(C.byref(L), 4, 1, None) == moeq.ERR_INVALID_ARG
    assert f(C.byref(L), 1, 1, C.byref(h)) == moeq.ERR_INVALID_ARG     # slots < K
    assert f(C.byref(L), 9, 1, C.byref(h)) == moeq.ERR_INVALID_ARG     # slots > E
    assert f(C.byref(L), 4, 3, C.byref(h)) == moeq.ERR_INVALID_ARG     # 3 tokens x 2 > 4 slots
    assert f(C.byref(L), 4, 65, C.byref(h)) == moeq.ERR_INVALID_ARG
    bad = layer(E=8, K=2)
    bad.n_experts = 4
    assert f(C.byref(bad), 4, 1, C.byref(h)) == moeq.ERR_UNSUPPORTED
    assert not h.value
