"""Edge cases of both layer paths against the fp64 oracle, through the C ABI.

The decode path turns every 32-value block of its inputs (the token, the
SwiGLU outputs h) into block fixed point, and the prefill path runs fp16
tensor-core operands.  Both are exact or tightly bounded on iid normal
inputs; these cases push the regions where they are weakest, the class of
input behind the mlx issue page ("Silent numerical corruption in single long
forward on quantized MoE when sequence length % 32 != 0"): corruption that
only inputs the tests never drew would show.

  * massive activations: a few channels at 2^8..2^12 times the rest, and a
    block holding a single nonzero value;
  * heavy-tailed h: gate/up rows scaled up so that a few SwiGLU outputs per
    expert are ~2^8 times the rest (the down projection's input blocks);
  * groups with scale 0 (constant groups) and all-zero groups;
  * 8-bit groups with scales below the fp16 normal range (2^-17 .. 2^-14,
    exactly representable in fp16) and one not representable, which prefill
    must refuse with MOEQ_ERR_RANGE while decode computes it;
  * a token value beyond the fp16 range: prefill refuses, decode computes.

Bars (the layer tolerance, per token since the inputs span orders of
magnitude): relative L2 <= 2e-3 and max abs <= 1e-2 * max(1, max |ref|) for
every token; routing equal to the oracle's except at near-ties.
"""
import numpy as np
import pytest

import oracle
from helpers import check_routing, weights_for
from quantized_mixture_experts_affine_b200 import moeq, synth
from quantized_mixture_experts_affine_b200.layer import (DeviceLayer, LayerConfig, layer_forward)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0
D, P = moeq.MODE_DECODE, moeq.MODE_PREFILL

EDGE4 = LayerConfig("edge4", H=1024, I=512, E=16, K=4, expert_bits=4, shared=True, shared_I=512,
                    shared_bits=4)
EDGE8 = LayerConfig("edge8", H=1024, I=512, E=16, K=4, expert_bits=8)


# ------------------------------------------------------------------ host-built layers

def host_layer(cfg, copy=0):
    """Host tensors of a whole layer from the seeded streams (a dict)."""
    T = lambda kind, n, o, i, b: synth.tensor_host(SEED, synth.tag(kind, copy), n, o, i, b, cfg.G)
    t = dict(router=T(synth.ROUTER, 1, cfg.E, cfg.H, cfg.router_bits),
             gate=T(synth.GATE, cfg.E, cfg.I, cfg.H, cfg.expert_bits),
             up=T(synth.UP, cfg.E, cfg.I, cfg.H, cfg.expert_bits),
             down=T(synth.DOWN, cfg.E, cfg.H, cfg.I, cfg.expert_bits))
    if cfg.shared:
        t.update(sh_gate=T(synth.SH_GATE, 1, cfg.shared_I, cfg.H, cfg.shared_bits),
                 sh_up=T(synth.SH_UP, 1, cfg.shared_I, cfg.H, cfg.shared_bits),
                 sh_down=T(synth.SH_DOWN, 1, cfg.H, cfg.shared_I, cfg.shared_bits),
                 sh_expert_gate=T(synth.SH_EXPERT_GATE, 1, 1, cfg.H, cfg.shared_gate_bits))
    return t


def to_device(cfg, t):
    def dq(h):
        return synth.DevQ(torch.from_numpy(h.w.view(np.int32)).cuda(),
                          torch.from_numpy(h.s.view(np.int16)).cuda(),
                          torch.from_numpy(h.b.view(np.int16)).cuda(),
                          h.out_dim, h.in_dim, h.bits, h.group_size, h.n_mats)
    return DeviceLayer(cfg, **{k: dq(v) for k, v in t.items()})


def to_oracle(cfg, t):
    O = oracle.OracleTensor.of
    return oracle.OracleLayer(H=cfg.H, I=cfg.I, E=cfg.E, K=cfg.K, renorm=cfg.renorm,
                              router_scale=cfg.router_scale, **{k: O(v) for k, v in t.items()})


def bf16_bits(v):
    """Round-to-nearest-even bf16 bits of float values."""
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def bf16_float(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def scale_rows(h, rows, f):
    """Multiply the scales and biases of the given rows (every matrix of the
    bank) by f, a power of two (exact in bf16)."""
    for arr in (h.s, h.b):
        arr[:, rows, :] = bf16_bits(bf16_float(arr[:, rows, :]) * f)


# ------------------------------------------------------------------ running and checking

def run(L, xb, mode, residual=None):
    """The layer on tokens xb in one call (decode: calls of at most 64
    tokens, its limit); returns y, idx, w and the device status."""
    M = xb.shape[0]
    step = 64 if mode == D else M
    ys, ids, ws = [], [], []
    for t0 in range(0, M, step):
        xc = np.ascontiguousarray(xb[t0:t0 + step])
        x = torch.from_numpy(xc.view(np.int16)).cuda().view(torch.bfloat16)
        y = torch.full((xc.shape[0], L.cfg.H), float("nan"), device="cuda")
        res = None if residual is None else torch.from_numpy(
            np.ascontiguousarray(residual[t0:t0 + step])).cuda()
        y, idx, w = layer_forward(L, x, y=y, residual=res, mode=mode)
        torch.cuda.synchronize()
        ys.append(y.cpu().numpy())
        ids.append(idx.cpu().numpy())
        ws.append(w.cpu().numpy())
    return (np.concatenate(ys), np.concatenate(ids), np.concatenate(ws),
            moeq.moeq_device_status())


def check(cfg, OL, xb, y, idx, w, residual=None):
    ref = oracle.layer(OL, xb, residual)
    check_routing(idx, ref["idx"], ref["gap"], ref["logits"], cfg)
    wref = weights_for(idx, ref["logits"], cfg)
    assert np.abs(w - wref).max() < 1e-4
    out = oracle.expert_ffn(OL, xb, idx, wref, residual)
    y = np.asarray(y, np.float64)
    assert np.isfinite(y).all()
    for t in range(y.shape[0]):
        err = y[t] - out[t]
        rel = np.linalg.norm(err) / max(np.linalg.norm(out[t]), 1e-300)
        mx = np.abs(err).max()
        assert rel <= 2e-3 and mx <= 1e-2 * max(1.0, np.abs(out[t]).max()), (t, rel, mx)


def both_paths(cfg, t, xb, residual=None, modes=(D, P)):
    L, OL = to_device(cfg, t), to_oracle(cfg, t)
    for mode in modes:
        y, idx, w, status = run(L, xb, mode, residual)
        assert status == 0, (mode, moeq.status_str(status))
        check(cfg, OL, xb, y, idx, w, residual)


def normal_tokens(cfg, M, copy):
    return synth.normal_bf16_host(SEED, synth.tag(synth.X, copy), M * cfg.H).reshape(M, cfg.H)


def massive_tokens(cfg, M, copy, top=12):
    """N(0,1) tokens with massive activations: four fixed channels at
    2^8..2^top times the rest in every token, one more random channel per
    token at 2^9, and in token 0 a block holding a single nonzero value."""
    xf = bf16_float(normal_tokens(cfg, M, copy)).copy()
    rng = np.random.default_rng(copy)
    for c, mag in ((3, 2.0 ** 8), (129, 2.0 ** (top - 2)), (500, 2.0 ** top),
                   (1000, 2.0 ** (top - 1))):
        xf[:, c] = mag * np.where(rng.random(M) < 0.5, -1.0, 1.0) * (1 + 0.5 * rng.random(M))
    xf[np.arange(M), rng.integers(0, cfg.H, M)] = 2.0 ** 9
    xf[0, 64:96] = 0.0
    xf[0, 77] = 3.0
    return bf16_bits(xf)


# ------------------------------------------------------------------ the cases

@pytest.mark.parametrize("M", [1, 5, 80])
@pytest.mark.parametrize("top", [10, 12])
def test_massive_activations(M, top):
    """Decode computes every case.  Prefill computes the 2^10 case; at 2^12
    its SwiGLU outputs (about 2^12 * 0.02 squared, times the tails) may pass
    the fp16 maximum, and then it must refuse with MOEQ_ERR_RANGE, never
    return silently wrong rows."""
    cfg = EDGE4
    t = host_layer(cfg)
    xb = massive_tokens(cfg, M, 600 + M, top)
    L, OL = to_device(cfg, t), to_oracle(cfg, t)
    y, idx, w, status = run(L, xb, D)
    assert status == 0
    check(cfg, OL, xb, y, idx, w)
    y, idx, w, status = run(L, xb, P)
    assert status == 0 if top == 10 else status in (0, moeq.ERR_RANGE)
    if status == 0:
        check(cfg, OL, xb, y, idx, w)


@pytest.mark.parametrize("M", [1, 7, 96])
def test_heavy_tailed_hidden(M):
    """Rows 0, 77 and 200 of every gate and up matrix (routed and shared)
    scaled by 2^4: their SwiGLU outputs are ~2^8 times the rest, so every
    down projection sees input blocks with one dominant value."""
    cfg = EDGE4
    t = host_layer(cfg, copy=1)
    for k in ("gate", "up", "sh_gate", "sh_up"):
        scale_rows(t[k], [0, 77, 200], 16.0)
    both_paths(cfg, t, normal_tokens(cfg, M, 700 + M),
               residual=np.linspace(-3, 3, M * cfg.H, dtype=np.float32).reshape(M, cfg.H))


@pytest.mark.parametrize("M", [1, 64, 130])
def test_zero_scale_groups(M):
    """Groups with scale 0 (every weight equals the bias) and groups with
    scale and bias 0, in every tensor, at both group positions of a row."""
    cfg = EDGE4
    t = host_layer(cfg, copy=2)
    rng = np.random.default_rng(M)
    for k, h in t.items():
        n, o, g = h.s.shape
        for _ in range(max(4, o // 8)):
            m, r, j = rng.integers(0, n), rng.integers(0, o), rng.integers(0, g)
            h.s[m, r, j] = 0
            if rng.random() < 0.3:
                h.b[m, r, j] = 0
        h.s[:, 0, 0] = 0          # first group of row 0
        h.s[:, o - 1, g - 1] = 0  # last group of the last row
    both_paths(cfg, t, normal_tokens(cfg, M, 800 + M))


def tiny_scale_layer(exact=True):
    """8-bit experts whose group scales lie in [2^-17, 2^-14) (below the fp16
    normal range, exact as fp16 subnormals) with biases of ordinary size;
    with exact=False the first group of every gate row gets 1.5 * 2^-24,
    which fp16 cannot hold (its subnormal step is 2^-24)."""
    cfg = EDGE8
    t = host_layer(cfg, copy=3)
    rng = np.random.default_rng(11)
    for k in ("gate", "up", "down"):
        h = t[k]
        sel = rng.random(h.s.shape) < 0.25
        mag = 2.0 ** rng.integers(-17, -14, h.s.shape) * (1 + rng.integers(0, 8, h.s.shape) / 8)
        h.s[sel] = bf16_bits(mag[sel])
    if not exact:
        t["gate"].s[:, :, 0] = bf16_bits(1.5 * 2.0 ** -24)
    return cfg, t


@pytest.mark.parametrize("M", [1, 70])
def test_tiny_scales_8bit(M):
    cfg, t = tiny_scale_layer(exact=True)
    both_paths(cfg, t, normal_tokens(cfg, M, 900 + M))


def test_scale_beyond_fp16_precision_is_refused_by_prefill():
    """A scale fp16 cannot represent exactly: prefill reports MOEQ_ERR_RANGE
    in the device status; decode computes the layer."""
    cfg, t = tiny_scale_layer(exact=False)
    xb = normal_tokens(cfg, 70, 950)
    L, OL = to_device(cfg, t), to_oracle(cfg, t)
    _, _, _, status = run(L, xb, P)
    assert status == moeq.ERR_RANGE
    for M in (1, 70):
        y, idx, w, status = run(L, xb[:M], D)
        assert status == 0
        check(cfg, OL, xb[:M], y, idx, w)


def test_token_beyond_fp16_range():
    """A token value of 2^17 (a finite bf16 value above the fp16 maximum):
    prefill reports MOEQ_ERR_RANGE; decode computes the layer."""
    cfg = EDGE4
    t = host_layer(cfg, copy=4)
    xb = normal_tokens(cfg, 66, 960)
    xb[5, 321] = bf16_bits(2.0 ** 17)
    L, OL = to_device(cfg, t), to_oracle(cfg, t)
    _, _, _, status = run(L, xb, P)
    assert status == moeq.ERR_RANGE
    for rows in (slice(5, 6), slice(0, 9)):
        y, idx, w, status = run(L, xb[rows], D)
        assert status == 0
        check(cfg, OL, xb[rows], y, idx, w)
