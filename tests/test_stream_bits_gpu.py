"""3-, 5- and 6-bit codes (affine widths that do not divide 32; the mlx
issue page's table runs an affine 5-bit model): each row is one
little-endian bit stream, value i at bits [i*b, (i+1)*b), so a value may
straddle two 32-bit words.  Through the C ABI, against the oracle.

Bars: the device generator's words equal the host generator's; unpacked
codes and dequantised fp32 weights bit-exact; qmv relative L2 <= 1e-5;
layer outputs at the layer tolerance of every other layer test (routing
equal except at near-ties, relative L2 <= 2e-3, max abs <= 1e-2).  These
widths run on the decode path only: MOEQ_MODE_PREFILL refuses the layer
with MOEQ_ERR_UNSUPPORTED and MOEQ_MODE_AUTO keeps it on decode up to 64
tokens, whatever M * top_k.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from helpers import check_layer_outputs, rel_l2
from quantized_mixture_experts_affine_b200 import moeq, synth
from quantized_mixture_experts_affine_b200.layer import (CONFIGS, Workspace, layer_forward,
                                                         synthetic_layer)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0
D, P, A = moeq.MODE_DECODE, moeq.MODE_PREFILL, moeq.MODE_AUTO


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("bits,G,inn,rq", [(3, 32, 512, False), (3, 64, 384, False),
                                           (3, 128, 256, True), (6, 32, 192, False),
                                           (6, 64, 512, True), (6, 128, 640, False),
                                           (5, 32, 384, False), (5, 64, 256, True),
                                           (5, 128, 512, False)])
def test_generator_and_dequant_bit_exact(bits, G, inn, rq):
    tg = synth.tag(synth.UP, 30 + bits)
    q = synth.tensor_dev(SEED, tg, 3, 72, inn, bits, G, rq)
    host = q.to_host()
    h = synth.tensor_host(SEED, tg, 3, 72, inn, bits, G, rq)
    assert np.array_equal(host.w, h.w) and np.array_equal(host.s, h.s)
    assert np.array_equal(host.b, h.b)
    t = moeq.qtensor(q.w, q.s, q.b, 72, inn, bits, G, 3)
    for e in (0, 2):
        codes = torch.empty((72, inn), dtype=torch.uint8, device="cuda")
        w = torch.empty((72, inn), dtype=torch.float32, device="cuda")
        moeq.moeq_dequant(t, e, codes, w)
        torch.cuda.synchronize()
        ref = oracle.unpack(host, e)
        assert ref.max() == (1 << bits) - 1 and ref.min() == 0
        assert np.array_equal(codes.cpu().numpy(), ref)
        assert np.array_equal(w.cpu().numpy().view(np.uint32),
                              oracle.dequant_f32(host, e).view(np.uint32))
    assert moeq.moeq_device_status() == 0


QMV_CASES = [  # (bits, G, out, in, M, requant)
    (3, 64, 1024, 4096, 1, False),   # 397B-like gate/up width, four slices
    (3, 32, 130, 384, 7, False),     # ragged rows, 12 chunks in one slice
    (3, 128, 768, 2048, 64, True),   # max decode M
    (6, 64, 512, 2048, 3, False),
    (6, 128, 96, 4096, 2, False),    # 3 KB rows
    (6, 32, 33, 192, 4, False),      # 144-byte rows, 6 chunks
    (6, 64, 2048, 768, 5, True),     # down width
    (5, 64, 512, 4096, 1, False),    # 20-byte runs, four slices
    (5, 32, 70, 384, 9, True),       # ragged rows
    (5, 128, 2048, 1024, 64, False), # max decode M
]


@pytest.mark.parametrize("bits,G,out,inn,M,rq", QMV_CASES)
def test_qmv_parity(bits, G, out, inn, M, rq):
    tg = synth.tag(synth.ROUTER, 40 + bits)
    q = synth.tensor_dev(SEED, tg, 2, out, inn, bits, G, rq)
    t = moeq.qtensor(q.w, q.s, q.b, out, inn, bits, G, 2)
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 9), M * inn).reshape(M, inn)
    x = dev(xb.view(np.int16))
    host = q.to_host()
    for e in (0, 1):
        y = torch.full((M, out), float("nan"), device="cuda")
        moeq.moeq_qmv(t, e, x, M, y)
        torch.cuda.synchronize()
        ref = oracle.qmv(host, xb, mat=e)
        assert rel_l2(y.cpu().numpy(), ref) <= 1e-5, rel_l2(y.cpu().numpy(), ref)
    assert moeq.moeq_device_status() == 0


def shape(name, **kw):
    tag = "_".join(f"{k}{v}" for k, v in kw.items())
    return dataclasses.replace(CONFIGS[name], name=f"{name}_{tag}", **kw)


LAYERS = [
    shape("decode_30b", expert_bits=3),
    shape("decode_30b", expert_bits=6, G=32),
    shape("decode_397b", expert_bits=6, shared_bits=3, G=128),
    shape("mixed_2bit", expert_bits=3),   # 4 -> 3 bit requantised experts, 4-bit shared
    shape("decode_397b", expert_bits=5, shared_bits=5),
]


def tokens(cfg, M, copy):
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, copy), M * cfg.H).reshape(M, cfg.H)
    return xb, dev(xb.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("cfg", LAYERS, ids=lambda c: c.name)
def test_layer_decode(cfg):
    L = synthetic_layer(cfg, SEED, 0)
    for M in (1, 5, 24):
        xb, x = tokens(cfg, M, 80 + M)
        y, idx, w = layer_forward(L, x, mode=D)
        torch.cuda.synchronize()
        assert moeq.moeq_device_status() == 0
        check_layer_outputs(cfg, SEED, 0, xb, y.cpu().numpy(), idx.cpu().numpy(),
                            w.cpu().numpy())


def test_auto_stays_on_decode_and_prefill_refuses():
    cfg = LAYERS[0]                       # top-8: 64 tokens are 512 pairs
    L = synthetic_layer(cfg, SEED, 0)
    M = 64
    xb, x = tokens(cfg, M, 90)
    assert moeq.moeq_workspace_bytes(L.desc, M, P) == 0
    assert moeq.moeq_workspace_bytes(L.desc, M, A) == moeq.moeq_workspace_bytes(L.desc, M, D) > 0
    ya, idx, w = layer_forward(L, x, mode=A)
    yd = layer_forward(L, x, mode=D)[0]
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    assert torch.equal(ya.view(torch.int32), yd.view(torch.int32))
    check_layer_outputs(cfg, SEED, 0, xb, ya.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy())
    # beyond the decode path's 64 tokens AUTO has no path for the layer
    assert moeq.moeq_workspace_bytes(L.desc, M + 1, A) == 0
    y = torch.empty((M, cfg.H), device="cuda")
    with pytest.raises(moeq.MoeqError) as e:
        moeq.moeq_layer_forward(L.desc, x, M, y, None, None, None,
                                torch.empty(1 << 20, dtype=torch.uint8, device="cuda"), 1 << 20,
                                P, None)
    assert e.value.status == moeq.ERR_UNSUPPORTED


def test_decode_chunks_match_one_shot():
    """Two calls of 32 tokens give the rows of one call of 64 bitwise (each
    token's sums run in the same order whatever M)."""
    cfg = LAYERS[1]
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = tokens(cfg, 64, 91)
    y1 = layer_forward(L, x, mode=D)[0]
    ws = Workspace(L, 32, D)
    yc = torch.cat([layer_forward(L, x[t0:t0 + 32], ws=ws, mode=D)[0] for t0 in (0, 32)])
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), yc.view(torch.int32))
