"""MX FP4 expert weights (the mlx issue page's mode="mxfp4": 4-bit E2M1
codes, one E8M0 exponent byte per 32 values) through the C ABI, against the
oracle.

Bars: dequantised codes and fp32 weights bit-exact; the device generator's
bytes equal the host generator's.
"""
import numpy as np
import pytest

import oracle
from quantized_mixture_experts_affine_b200 import moeq, synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0


def test_mx_generator_and_dequant_bit_exact():
    d = synth.tensor_mx_dev(SEED, synth.tag(synth.UP, 40), 3, 72, 512)
    h = synth.tensor_mx_host(SEED, synth.tag(synth.UP, 40), 3, 72, 512)
    host = d.to_host()
    assert np.array_equal(host.w, h.w) and np.array_equal(host.s, h.s)
    t = moeq.qtensor(d.w, d.s, None, 72, 512, 4, 32, 3, moeq.FMT_MXFP4)
    for e in (0, 2):
        codes = torch.empty((72, 512), dtype=torch.uint8, device="cuda")
        w = torch.empty((72, 512), dtype=torch.float32, device="cuda")
        moeq.moeq_dequant(t, e, codes, w)
        torch.cuda.synchronize()
        assert np.array_equal(codes.cpu().numpy(), oracle.unpack(h, e))
        assert np.array_equal(w.cpu().numpy().view(np.uint32),
                              oracle.dequant_f32(h, e).view(np.uint32))
    assert moeq.moeq_device_status() == 0


def test_mx_every_code_and_scale_byte():
    """All 16 codes under exponent bytes 0 (2^-127, subnormal), 1, 100, 127,
    200 and 254 (6 * 2^127), bit-exact against the oracle."""
    codes = np.tile(np.arange(16, dtype=np.uint32), 2)
    w = np.zeros((6, 4), np.uint32)
    for j in range(8):
        w |= codes[j::8][None, :4] << (4 * j)
    ebytes = np.array([[0], [1], [100], [127], [200], [254]], np.uint8)
    host = synth.HostQ(w.reshape(1, 6, 4), ebytes.reshape(1, 6, 1), np.zeros(0, np.uint16),
                       6, 32, 4, 32, 1, 1)
    wd = torch.from_numpy(host.w.view(np.int32)).cuda()
    ed = torch.from_numpy(host.s).cuda()
    t = moeq.qtensor(wd, ed, None, 6, 32, 4, 32, 1, moeq.FMT_MXFP4)
    out = torch.empty((6, 32), dtype=torch.float32, device="cuda")
    moeq.moeq_dequant(t, 0, None, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32),
                          oracle.dequant_f32(host).view(np.uint32))


# ------------------------------------------------------------------ qmv and layers
from helpers import check_routing, weights_for  # noqa: E402
from quantized_mixture_experts_affine_b200.layer import (DeviceLayer, LayerConfig,  # noqa: E402
                                                         Workspace, layer_forward)

D, P = moeq.MODE_DECODE, moeq.MODE_PREFILL


def test_mx_qmv_parity():
    """moeq_qmv on an MX bank (3-limb fixed-point input, exact integer sums):
    relative L2 <= 1e-5 against the oracle's fp64 product."""
    d = synth.tensor_mx_dev(SEED, synth.tag(synth.DOWN, 41), 2, 300, 1024)
    h = d.to_host()
    t = moeq.qtensor(d.w, d.s, None, 300, 1024, 4, 32, 2, moeq.FMT_MXFP4)
    for M in (1, 5):
        xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 90 + M), M * 1024).reshape(M, 1024)
        x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        y = torch.empty((M, 300), device="cuda")
        moeq.moeq_qmv(t, 1, x, M, y)
        torch.cuda.synchronize()
        ref = oracle.qmv(oracle.OracleTensor.of(h), xb, mat=1)
        got = y.cpu().numpy()
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-5
    assert moeq.moeq_device_status() == 0


MXCFG = LayerConfig("mx", H=1024, I=512, E=32, K=4, expert_bits=4, shared=True, shared_I=512,
                    shared_bits=4, G=32)


def mx_layer(cfg, shared_mx=False):
    """MX FP4 routed experts (gate/up/down) beside an 8-bit affine router and
    shared-expert gate; the shared expert affine 4-bit, or MX too."""
    A = lambda kind, n, o, i, b, G: synth.tensor_dev(SEED, synth.tag(kind), n, o, i, b, G)
    X = lambda kind, n, o, i: synth.tensor_mx_dev(SEED, synth.tag(kind), n, o, i)
    t = dict(router=A(synth.ROUTER, 1, cfg.E, cfg.H, 8, 64),
             gate=X(synth.GATE, cfg.E, cfg.I, cfg.H), up=X(synth.UP, cfg.E, cfg.I, cfg.H),
             down=X(synth.DOWN, cfg.E, cfg.H, cfg.I),
             sh_expert_gate=A(synth.SH_EXPERT_GATE, 1, 1, cfg.H, 8, 64))
    if shared_mx:
        t.update(sh_gate=X(synth.SH_GATE, 1, cfg.shared_I, cfg.H),
                 sh_up=X(synth.SH_UP, 1, cfg.shared_I, cfg.H),
                 sh_down=X(synth.SH_DOWN, 1, cfg.H, cfg.shared_I))
    else:
        t.update(sh_gate=A(synth.SH_GATE, 1, cfg.shared_I, cfg.H, 4, 64),
                 sh_up=A(synth.SH_UP, 1, cfg.shared_I, cfg.H, 4, 64),
                 sh_down=A(synth.SH_DOWN, 1, cfg.H, cfg.shared_I, 4, 64))
    L = DeviceLayer(cfg, **t)
    O = lambda v: oracle.OracleTensor.of(v.to_host())
    OL = oracle.OracleLayer(H=cfg.H, I=cfg.I, E=cfg.E, K=cfg.K, renorm=cfg.renorm,
                            router_scale=cfg.router_scale, **{k: O(v) for k, v in t.items()})
    return L, OL


def check_mx(cfg, OL, xb, y, idx, w):
    ref = oracle.layer(OL, xb)
    check_routing(idx, ref["idx"], ref["gap"], ref["logits"], cfg)
    wref = weights_for(idx, ref["logits"], cfg)
    out = oracle.expert_ffn(OL, xb, idx, wref)
    r = np.linalg.norm(y - out) / np.linalg.norm(out)
    assert r <= 2e-3 and np.abs(y - out).max() <= 1e-2, (r, np.abs(y - out).max())


@pytest.mark.parametrize("shared_mx", [False, True])
def test_mx_layer_both_paths(shared_mx):
    cfg = MXCFG
    L, OL = mx_layer(cfg, shared_mx)
    for M, mode in ((1, D), (5, D), (24, D), (300, P)):
        xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 95 + M), M * cfg.H).reshape(M, cfg.H)
        x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        y, idx, w = layer_forward(L, x, mode=mode)
        torch.cuda.synchronize()
        assert moeq.moeq_device_status() == 0, (M, mode)
        check_mx(cfg, OL, xb, y.cpu().numpy().astype(np.float64), idx.cpu().numpy(),
                 w.cpu().numpy().astype(np.float64))
    # chunked prefill: bitwise the one-shot rows
    M = 2100
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 96), M * cfg.H).reshape(M, cfg.H)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    y1, _, _ = layer_forward(L, x, mode=P)
    ws = Workspace(L, 2048, P)
    yc = torch.cat([layer_forward(L, x[t0:t0 + 2048], ws=ws, mode=P)[0]
                    for t0 in range(0, M, 2048)])
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    assert torch.equal(y1.view(torch.int32), yc.view(torch.int32))
