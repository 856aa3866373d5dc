"""moeq_layer_forward_norm on the GPU against the oracle, through the C ABI.

The output RMS norm of the flash-moe-inference page's per-layer pipeline
("CMD3: expert forward + combine + norm"): y_norm = bf16(y / sqrt(mean(y^2)
+ eps) * gamma).  Bars:
  * y is bit for bit the output of moeq_layer_forward (the norm adds an
    output and changes nothing else);
  * y_norm against oracle.rmsnorm of the oracle's layer output (fp64, on the
    GPU's routing): relative L2 <= 2e-3 per token, and per element within
    2^-8 |ref| + 2e-3 * rms(ref) -- one bf16 rounding (at most 2^-9 relative)
    on top of the layer tolerance;
  * prefill: one-shot and 2048-token chunked y_norm bitwise equal.
"""
import numpy as np
import pytest

import oracle
from helpers import check_layer_outputs, oracle_expert_outputs, weights_for, oracle_routing
from quantized_mixture_experts_affine_b200 import moeq, synth
from quantized_mixture_experts_affine_b200.layer import (CONFIGS, Workspace, layer_forward,
                                                         layer_forward_norm, synthetic_layer)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0
EPS = 1e-6


def bf16_bits(v):
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def gamma_of(cfg):
    g = 1.0 + 0.25 * (synth.normal_bf16_host(SEED, synth.tag(synth.RESIDUAL, 99), cfg.H)
                      .astype(np.uint32) << 16).view(np.float32)
    gb = bf16_bits(g)
    return gb, torch.from_numpy(gb.view(np.int16)).cuda()


def tokens(cfg, M, copy):
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, copy), M * cfg.H).reshape(M, cfg.H)
    return xb, torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)


def check_norm(cfg, xb, y, yn, idx, w, gb, residual=None, copy=0):
    logits, _, _, _ = oracle_routing(cfg, SEED, copy, xb)
    ref_y = oracle_expert_outputs(cfg, SEED, copy, xb, idx, weights_for(idx, logits, cfg),
                                  residual)
    ref = oracle.rmsnorm(ref_y, gb, EPS)
    got = (yn.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(got.shape[0]):
        rms = np.sqrt((ref[t] ** 2).mean())
        rel = np.linalg.norm(got[t] - ref[t]) / np.linalg.norm(ref[t])
        assert rel <= 2e-3, (t, rel)
        assert (np.abs(got[t] - ref[t]) <= 2.0 ** -8 * np.abs(ref[t]) + 2e-3 * rms).all(), t


@pytest.mark.parametrize("name,M,mode", [("tiny", 3, moeq.MODE_DECODE),
                                         ("decode_397b", 1, moeq.MODE_DECODE),
                                         ("decode_30b", 5, moeq.MODE_DECODE),
                                         ("prefill_8bit", 300, moeq.MODE_PREFILL),
                                         ("mixed_2bit", 256, moeq.MODE_PREFILL)])
def test_layer_forward_norm(name, M, mode):
    cfg = CONFIGS[name]
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = tokens(cfg, M, 40 + M)
    gb, g = gamma_of(cfg)
    res_np = np.linspace(-2, 2, M * cfg.H, dtype=np.float32).reshape(M, cfg.H)
    res = torch.from_numpy(res_np).cuda()
    y0, i0, w0 = layer_forward(L, x, residual=res, mode=mode)
    y, yn, idx, w = layer_forward_norm(L, x, g, EPS, residual=res, mode=mode)
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    assert torch.equal(y.view(torch.int32), y0.view(torch.int32)) and torch.equal(idx, i0)
    ig, wg = idx.cpu().numpy(), w.cpu().numpy()
    # the oracle on every row of small calls, on 12 spread rows of larger ones
    rows = np.arange(M) if M <= 16 else np.unique(np.linspace(0, M - 1, 12).astype(int))
    yn_np = yn.view(torch.int16).cpu().numpy().view(np.uint16)
    check_layer_outputs(cfg, SEED, 0, xb, y.cpu().numpy(), ig, wg, residual=res_np, rows=rows)
    check_norm(cfg, xb[rows], None, yn_np[rows], ig[rows], wg[rows], gb, residual=res_np[rows])


def test_layer_forward_norm_one_launch_decode(monkeypatch):
    monkeypatch.setenv("MOEQ_FUSED_DECODE", "1")
    cfg = CONFIGS["decode_397b"]
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = tokens(cfg, 1, 61)
    gb, g = gamma_of(cfg)
    y, yn, idx, w = layer_forward_norm(L, x, g, EPS, mode=moeq.MODE_DECODE)
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    ig, wg = idx.cpu().numpy(), w.cpu().numpy()
    check_norm(cfg, xb, y.cpu().numpy(), yn.view(torch.int16).cpu().numpy().view(np.uint16),
               ig, wg, gb)


def test_prefill_norm_chunk_invariance():
    """4097 tokens (n = 8 * 4097 crosses the 32768 seam): one call and calls
    of 2048 tokens give bitwise the same y and y_norm."""
    cfg = CONFIGS["prefill_8bit"]
    L = synthetic_layer(cfg, SEED, 0)
    M = 4097
    xb, x = tokens(cfg, M, 88)
    gb, g = gamma_of(cfg)
    P = moeq.MODE_PREFILL
    y1, n1, _, _ = layer_forward_norm(L, x, g, EPS, mode=P)
    ws = Workspace(L, 2048, P)
    parts = [layer_forward_norm(L, x[t0:t0 + 2048], g, EPS, ws=ws, mode=P)
             for t0 in range(0, M, 2048)]
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    y2 = torch.cat([p[0] for p in parts])
    n2 = torch.cat([p[1] for p in parts])
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    assert torch.equal(n1.view(torch.int16), n2.view(torch.int16))
    rows = np.array([0, 1, 2047, 2048, 4095, 4096])
    ig = np.concatenate([p[2].cpu().numpy() for p in parts])[rows]
    wg = np.concatenate([p[3].cpu().numpy() for p in parts])[rows]
    check_norm(cfg, xb[rows], None, n1.view(torch.int16).cpu().numpy().view(np.uint16)[rows],
               ig, wg, gb)
