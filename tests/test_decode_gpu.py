"""Decode path on the GPU against the fp64 oracle (through the C ABI).

Bars: unpacked codes and dequantised fp32 weights bit-exact; qmv relative
L2 <= 1e-5 (24-bit fixed-point input, fp32 sums); routing equal except at
near-ties; layer outputs relative L2 <= 2e-3 and max abs <= 1e-2.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from helpers import check_layer_outputs, rel_l2, NEAR_TIE
from quantized_mixture_experts_affine_b200 import moeq, synth
from quantized_mixture_experts_affine_b200.layer import (CONFIGS, expert_ffn, layer_forward,
                                                         synthetic_layer, Workspace)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def x_tokens(cfg, M, copy=0, seed=SEED):
    xb = synth.normal_bf16_host(seed, synth.tag(synth.X, copy), M * cfg.H).reshape(M, cfg.H)
    return xb, dev(xb.view(np.int16)).view(torch.bfloat16)


# ------------------------------------------------------------------ generator

@pytest.mark.parametrize("bits,G,rq", [(2, 64, False), (4, 64, False), (8, 64, False),
                                       (2, 64, True), (4, 32, False), (8, 128, False)])
def test_device_generator_matches_host(bits, G, rq):
    tg = synth.tag(synth.GATE, 3)
    d = synth.tensor_dev(7, tg, 3, 40, 512, bits, G, rq).to_host()
    h = synth.tensor_host(7, tg, 3, 40, 512, bits, G, rq)
    assert np.array_equal(d.w, h.w) and np.array_equal(d.s, h.s) and np.array_equal(d.b, h.b)
    xd = synth.normal_bf16_dev(7, synth.tag(synth.X), 10001).cpu().view(torch.int16).numpy()
    assert np.array_equal(xd.view(np.uint16), synth.normal_bf16_host(7, synth.tag(synth.X), 10001))


# ------------------------------------------------------------------ dequant

@pytest.mark.parametrize("bits,G", [(2, 64), (4, 64), (8, 64), (4, 32), (8, 128), (2, 128)])
def test_dequant_bit_exact(bits, G):
    q = synth.tensor_dev(SEED, synth.tag(synth.UP, bits), 3, 72, 512, bits, G)
    t = moeq.qtensor(q.w, q.s, q.b, 72, 512, bits, G, 3)
    host = q.to_host()
    for e in (0, 2):
        codes = torch.empty((72, 512), dtype=torch.uint8, device="cuda")
        w = torch.empty((72, 512), dtype=torch.float32, device="cuda")
        moeq.moeq_dequant(t, e, codes, w)
        torch.cuda.synchronize()
        assert np.array_equal(codes.cpu().numpy(), oracle.unpack(host, e))
        assert np.array_equal(w.cpu().numpy().view(np.uint32),
                              oracle.dequant_f32(host, e).view(np.uint32))
    assert moeq.moeq_device_status() == 0


# ------------------------------------------------------------------ qmv

QMV_CASES = [  # (bits, G, out, in, M, requant)
    (8, 64, 128, 2816, 1, False),    # standalone router 2816 -> 128
    (8, 64, 512, 4096, 3, False),    # 397B-like router
    (4, 64, 1024, 4096, 2, False),
    (2, 64, 1024, 4096, 1, True),
    (4, 64, 4096, 1024, 5, False),
    (8, 32, 130, 256, 64, False),    # ragged rows, max decode M
    (4, 128, 96, 768, 7, False),
    (2, 32, 33, 128, 4, False),
    (4, 64, 40, 192, 3, False),      # 3 groups per row: scale/bias runs not 16-byte multiples
    # 128 row blocks: each block's tokens are split over units in runs
    (8, 64, 1024, 4096, 7, False),   # runs of 3, 3, 1 tokens
    (4, 64, 1024, 4096, 5, False),   # runs of 2, 2, 1 tokens
]


@pytest.mark.parametrize("bits,G,out,inn,M,rq", QMV_CASES)
def test_qmv_parity(bits, G, out, inn, M, rq):
    tg = synth.tag(synth.ROUTER, 100 + bits)
    q = synth.tensor_dev(SEED, tg, 2, out, inn, bits, G, rq)
    t = moeq.qtensor(q.w, q.s, q.b, out, inn, bits, G, 2)
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 5), M * inn).reshape(M, inn)
    x = dev(xb.view(np.int16))
    host = q.to_host()
    for e in (0, 1):
        y = torch.full((M, out), float("nan"), device="cuda")
        moeq.moeq_qmv(t, e, x, M, y)
        torch.cuda.synchronize()
        ref = oracle.qmv(host, xb, mat=e)
        assert rel_l2(y.cpu().numpy(), ref) <= 1e-5, rel_l2(y.cpu().numpy(), ref)
    assert moeq.moeq_device_status() == 0


@pytest.mark.parametrize("bits,out,M", [(8, 1024, 7), (4, 1024, 5), (8, 512, 3), (4, 96, 7)])
def test_qmv_token_split_matches_single_tokens(bits, out, M):
    """With few row blocks the M tokens of a block are split over several
    work units (runs of tokens).  Each token's output row must be bitwise
    the row a one-token call produces: the split only regroups whole vector
    computations, so a misplaced run shows up as a wrong row."""
    inn = 4096 if out >= 512 else 768
    G = 64
    q = synth.tensor_dev(SEED, synth.tag(synth.ROUTER, 300 + bits), 1, out, inn, bits, G, False)
    t = moeq.qtensor(q.w, q.s, q.b, out, inn, bits, G, 1)
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 31), M * inn).reshape(M, inn)
    x = dev(xb.view(np.int16))
    y = torch.full((M, out), float("nan"), device="cuda")
    moeq.moeq_qmv(t, 0, x, M, y)
    for m in range(M):
        y1 = torch.full((1, out), float("nan"), device="cuda")
        moeq.moeq_qmv(t, 0, x[m:m + 1], 1, y1)
        torch.cuda.synchronize()
        assert torch.equal(y[m:m + 1], y1), m
    assert moeq.moeq_device_status() == 0


def test_qmv_unaligned_scales():
    """Scale/bias arrays only 2-byte aligned (offset by one entry): the rows
    are copied entry by entry instead of in bulk; same results."""
    bits, G, out, inn, M = 4, 64, 96, 512, 2
    q = synth.tensor_dev(SEED, synth.tag(synth.ROUTER, 77), 1, out, inn, bits, G)
    n = q.s.numel()
    s_buf = torch.zeros(n + 8, dtype=q.s.dtype, device="cuda")
    b_buf = torch.zeros(n + 8, dtype=q.b.dtype, device="cuda")
    s_buf[1:n + 1].copy_(q.s.reshape(-1))
    b_buf[1:n + 1].copy_(q.b.reshape(-1))
    t = moeq.qtensor(q.w, s_buf[1:].data_ptr(), b_buf[1:].data_ptr(), out, inn, bits, G, 1)
    xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 6), M * inn).reshape(M, inn)
    y = torch.full((M, out), float("nan"), device="cuda")
    moeq.moeq_qmv(t, 0, dev(xb.view(np.int16)), M, y)
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    ref = oracle.qmv(q.to_host(), xb, mat=0)
    assert rel_l2(y.cpu().numpy(), ref) <= 1e-5


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("M,E,K,renorm,scale", [(37, 128, 8, True, 1.0), (5, 512, 4, True, 1.0),
                                                (64, 8, 2, False, 0.5), (3, 4096, 32, True, 2.0),
                                                (1, 16, 16, True, 1.0)])
def test_route_topk_parity(M, E, K, renorm, scale):
    logits, _ = synth.zipf_logits_host(SEED, synth.tag(synth.LOGITS, E), M, E, 1.1)
    lg = dev(logits)
    idx = torch.empty((M, K), dtype=torch.int32, device="cuda")
    w = torch.empty((M, K), dtype=torch.float32, device="cuda")
    moeq.moeq_route_topk(lg, M, E, K, renorm, scale, idx, w)
    torch.cuda.synchronize()
    # the decision is taken on the same fp32 logits on both sides
    io, wo, gap = oracle.route_f32(logits, K, renorm, scale)
    ig, wg = idx.cpu().numpy(), w.cpu().numpy()
    for t in range(M):
        if np.array_equal(ig[t], io[t]):
            continue
        if set(ig[t]) != set(io[t]):
            # another set only where the K-th choice is a near-tie
            assert gap[t] < NEAR_TIE, (t, ig[t], io[t], gap[t])
        else:
            # the same set in another order: only between near-equal logits
            l = scale * logits[t].astype(np.float64)
            for a, b in zip(ig[t], io[t]):
                if a != b:
                    assert abs(l[a] - l[b]) <= NEAR_TIE * max(1.0, abs(l[a])), (t, ig[t], io[t])
    assert np.abs(wg - wo).max() < 2e-6
    if renorm:
        assert np.allclose(wg.sum(1), 1.0, atol=1e-6)
    assert (np.diff(wg, axis=1) <= 1e-7).all()


def test_route_ties_lower_index():
    logits = np.zeros((2, 8), np.float32)
    logits[1, 3] = 1.0
    idx = torch.empty((2, 3), dtype=torch.int32, device="cuda")
    w = torch.empty((2, 3), dtype=torch.float32, device="cuda")
    moeq.moeq_route_topk(dev(logits), 2, 8, 3, True, 1.0, idx, w)
    assert idx.cpu().numpy().tolist() == [[0, 1, 2], [3, 0, 1]]
    assert np.allclose(w.cpu().numpy()[0], 1 / 3)


# ------------------------------------------------------------------ layer forward (decode)

def run_decode(cfg_name, Ms, copy=0, residual=False):
    cfg = CONFIGS[cfg_name]
    L = synthetic_layer(cfg, SEED, copy)
    out = []
    for M in Ms:
        xb, x = x_tokens(cfg, M, copy=M)
        res = None
        res_np = None
        if residual:
            res_np = np.linspace(-1, 1, M * cfg.H, dtype=np.float32).reshape(M, cfg.H)
            res = dev(res_np)
        y = torch.full((M, cfg.H), float("nan"), device="cuda")
        y, idx, w = layer_forward(L, x, y=y, residual=res, mode=moeq.MODE_DECODE)
        torch.cuda.synchronize()
        assert moeq.moeq_device_status() == 0
        r = check_layer_outputs(cfg, SEED, copy, xb, y.cpu().numpy(), idx.cpu().numpy(),
                                w.cpu().numpy(), residual=res_np)
        out.append(r)
    return out


def test_decode_tiny():
    run_decode("tiny", [1, 3, 5])


def test_decode_tiny_residual():
    run_decode("tiny", [3], residual=True)


def test_decode_30b_like():
    run_decode("decode_30b", [1, 4])


def test_decode_397b_like():
    run_decode("decode_397b", [1, 8])


def test_decode_30b_like_planned_apart():
    """M*K = 128 pairs: the plan runs as a launch of its own (above the size
    the gate/up launch plans itself) while the down launch still combines."""
    run_decode("decode_30b", [16], residual=True)


@pytest.mark.slow
def test_decode_397b_like_batch64():
    run_decode("decode_397b", [64])


def test_decode_mixed_2bit():
    run_decode("mixed_2bit", [1, 3])


def test_expert_ffn_zipf_routing_decode():
    """Mixed bank with router logits drawn for a skewed (Zipf 1.1) expert load."""
    cfg = CONFIGS["mixed_2bit"]
    L = synthetic_layer(cfg, SEED, 0)
    M = 64
    logits, _ = synth.zipf_logits_host(SEED, synth.tag(synth.LOGITS), M, cfg.E, 1.1)
    idx = torch.empty((M, cfg.K), dtype=torch.int32, device="cuda")
    w = torch.empty((M, cfg.K), dtype=torch.float32, device="cuda")
    moeq.moeq_route_topk(dev(logits), M, cfg.E, cfg.K, True, 1.0, idx, w)
    xb, x = x_tokens(cfg, M, copy=11)
    y = expert_ffn(L, x, idx, w, mode=moeq.MODE_DECODE)
    torch.cuda.synchronize()
    from helpers import oracle_expert_outputs, weights_for
    ig = idx.cpu().numpy()
    io, _, gap = oracle.route_f32(logits, cfg.K, True, 1.0)
    assert ((np.sort(ig, 1) == np.sort(io, 1)).all(1) | (gap < NEAR_TIE)).all()
    rows = np.arange(0, M, 4)
    # fp64 weights of the GPU's selection from the same drawn logits
    wref = weights_for(ig[rows], logits[rows], cfg)
    ref = oracle_expert_outputs(cfg, SEED, 0, xb[rows], ig[rows], wref)
    got = y.cpu().numpy()[rows]
    assert rel_l2(got, ref) <= 2e-3 and np.abs(got - ref).max() <= 1e-2


def test_workspace_reuse_and_poison():
    """Two calls into the same workspace, outputs poisoned with two values,
    agree bitwise (no unwritten rows, no dependence on stale workspace)."""
    cfg = CONFIGS["decode_30b"]
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = x_tokens(cfg, 4, copy=3)
    ws = Workspace(L, 4, moeq.MODE_DECODE)
    ys = []
    for poison in (float("nan"), 1e30):
        ws.buf.fill_(0xA5)
        y = torch.full((4, cfg.H), poison, device="cuda")
        layer_forward(L, x, y=y, ws=ws, mode=moeq.MODE_DECODE)
        ys.append(y.cpu().numpy())
    assert np.isfinite(ys[0]).all()
    assert np.array_equal(ys[0].view(np.uint32), ys[1].view(np.uint32))


# ------------------------------------------------------------------ single token (M = 1)
# The three decode paths for one token (environment read on every call):
#   single      the default: three lean launches (router, top-K + gate/up,
#               down + combine) for the layers whose formats they take;
#   launches    MOEQ_SINGLE_DECODE=0: the general decode launches with the
#               in-kernel plan;
#   one_launch  MOEQ_FUSED_DECODE=1: the opt-in one-launch kernel (every
#               group 64 wide, rows of whole 8-group runs).
# A layer a path does not take runs on the general launches.

@pytest.fixture(params=["single", "launches", "one_launch"])
def decode_path(request, monkeypatch):
    monkeypatch.delenv("MOEQ_FUSED_DECODE", raising=False)
    monkeypatch.delenv("MOEQ_SINGLE_DECODE", raising=False)
    if request.param == "one_launch":
        monkeypatch.setenv("MOEQ_FUSED_DECODE", "1")
    elif request.param == "launches":
        monkeypatch.setenv("MOEQ_SINGLE_DECODE", "0")
    return request.param


@pytest.mark.parametrize("name", ["tiny", "decode_30b", "decode_397b", "mixed_2bit"])
def test_single_token_poisoned_workspace(name, decode_path):
    """The one-launch kernel keeps its inter-CTA flags in the workspace: a
    workspace filled with three different poisons, then reused for a chain
    of calls (each call's tag derives from the previous one's), gives
    bitwise the same output every time, on either path."""
    cfg = CONFIGS[name]
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = x_tokens(cfg, 1, copy=21)
    ws = Workspace(L, 1, moeq.MODE_DECODE)
    outs = []
    for poison in (0xA5, 0x00, 0xFF):
        ws.buf.fill_(poison)
        for _ in range(3):
            y = torch.full((1, cfg.H), float("nan"), device="cuda")
            y, idx, w = layer_forward(L, x, y=y, ws=ws, mode=moeq.MODE_DECODE)
            outs.append(y.cpu().numpy().copy())
    assert moeq.moeq_device_status() == 0
    check_layer_outputs(cfg, SEED, 0, xb, outs[0], idx.cpu().numpy(), w.cpu().numpy())
    for o in outs[1:]:
        assert np.array_equal(o.view(np.uint32), outs[0].view(np.uint32))


@pytest.mark.parametrize("name", ["decode_397b", "decode_30b"])
def test_single_token_many_tokens_in_a_row(name, decode_path):
    """Different tokens through one workspace, one call each (as a decode
    loop does); every output matches the oracle."""
    cfg = CONFIGS[name]
    L = synthetic_layer(cfg, SEED, 1)
    ws = Workspace(L, 1, moeq.MODE_DECODE)
    for t in range(6):
        xb, x = x_tokens(cfg, 1, copy=400 + t)
        y, idx, w = layer_forward(L, x, ws=ws, mode=moeq.MODE_DECODE)
        torch.cuda.synchronize()
        assert moeq.moeq_device_status() == 0
        check_layer_outputs(cfg, SEED, 1, xb, y.cpu().numpy(), idx.cpu().numpy(),
                            w.cpu().numpy())


@pytest.mark.parametrize("name,G", [("decode_30b", 64), ("decode_30b", 128), ("decode_397b", 32),
                                    ("prefill_8bit", 64), ("prefill_8bit", 32), ("tiny", 64)])
def test_single_token_residual_group_sizes(name, G, decode_path):
    """One token with a residual, 4- and 8-bit layers at group sizes 32, 64
    and 128 (row blocks whose scale runs are 24, 48 or 6 entries per row),
    against the oracle; a second call into the same workspace is bitwise
    the same."""
    cfg = dataclasses.replace(CONFIGS[name], name=f"{name}_g{G}", G=G)
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = x_tokens(cfg, 1, copy=51)
    res_np = np.linspace(-1, 1, cfg.H, dtype=np.float32)[None, :]
    ws = Workspace(L, 1, moeq.MODE_DECODE)
    y, idx, w = layer_forward(L, x, residual=dev(res_np), ws=ws, mode=moeq.MODE_DECODE)
    y2 = layer_forward(L, x, residual=dev(res_np), ws=ws, mode=moeq.MODE_DECODE)[0]
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    check_layer_outputs(cfg, SEED, 0, xb, y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(),
                        residual=res_np)
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))


@pytest.mark.parametrize("name,be,bs", [("decode_397b", 2, 2), ("decode_397b", 2, 4),
                                       ("decode_397b", 4, 2), ("decode_397b", 8, 8),
                                       ("decode_30b", 2, 2), ("decode_30b", 8, 8)])
def test_single_token_code_widths(name, be, bs, decode_path):
    """One token through routed / shared code widths the single-token
    launches take (equal widths, 2-bit routed with a 4-bit shared expert)
    and ones they leave to the general launches (4-bit routed with a 2-bit
    shared expert; 8-bit 397B-like rows beyond their shared memory), against
    the oracle."""
    cfg = dataclasses.replace(CONFIGS[name], name=f"{name}_b{be}s{bs}", expert_bits=be,
                              shared_bits=bs)
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = x_tokens(cfg, 1, copy=52)
    y, idx, w = layer_forward(L, x, mode=moeq.MODE_DECODE)
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    check_layer_outputs(cfg, SEED, 0, xb, y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy())


@pytest.mark.parametrize("name,kw", [
    ("decode_397b", dict(renorm=False, router_scale=0.7)),
    ("decode_30b", dict(renorm=False)),
    ("decode_30b", dict(K=1)),
    ("decode_30b", dict(E=32, K=4)),
    ("decode_30b", dict(E=40, K=3, router_scale=1.5)),
], ids=["397b_softmax_w_scale", "30b_softmax_w", "30b_top1", "30b_e32", "30b_e40_k3_scale"])
def test_routing_variants(name, kw, decode_path):
    """Weights without renormalisation (softmax over all experts), a router
    scale, top-1 routing and small or ragged expert counts, on every
    single-token path (M = 1) and on the general launches (M = 3), against
    the oracle."""
    cfg = dataclasses.replace(CONFIGS[name], name=name + "_" + "_".join(f"{k}{v}" for k, v in kw.items()),
                              **kw)
    L = synthetic_layer(cfg, SEED, 0)
    for M in (1, 3):
        xb, x = x_tokens(cfg, M, copy=60 + M)
        y, idx, w = layer_forward(L, x, mode=moeq.MODE_DECODE)
        torch.cuda.synchronize()
        assert moeq.moeq_device_status() == 0
        check_layer_outputs(cfg, SEED, 0, xb, y.cpu().numpy(), idx.cpu().numpy(),
                            w.cpu().numpy())


def test_single_token_expert_index_out_of_range(decode_path):
    """A given routing with an expert index out of range: every decode path
    reports MOEQ_ERR_INVALID_ARG in the device status and reads the index
    as expert 0 (no access outside the bank)."""
    cfg = CONFIGS["decode_397b"]
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = x_tokens(cfg, 1, copy=33)
    ig = np.array([[5, cfg.E, 17, 200]], dtype=np.int32)
    wg = np.array([[0.4, 0.3, 0.2, 0.1]], dtype=np.float32)
    y = expert_ffn(L, x, dev(ig), dev(wg), mode=moeq.MODE_DECODE)
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == moeq.ERR_INVALID_ARG
    from helpers import oracle_expert_outputs
    used = np.array([[5, 0, 17, 200]], dtype=np.int32)
    ref = oracle_expert_outputs(cfg, SEED, 0, xb, used, wg.astype(np.float64), None)
    got = y.cpu().numpy()
    assert rel_l2(got, ref) <= 2e-3 and np.abs(got - ref).max() <= 1e-2


@pytest.mark.parametrize("name", ["decode_397b", "mixed_2bit", "tiny"])
def test_single_token_given_routing(name, decode_path):
    """moeq_expert_ffn with M = 1 (routing passed in): experts, shared expert
    and combine against the oracle, with a residual."""
    cfg = CONFIGS[name]
    L = synthetic_layer(cfg, SEED, 0)
    xb, x = x_tokens(cfg, 1, copy=31)
    rng = np.random.default_rng(5)
    ig = np.sort(rng.choice(cfg.E, cfg.K, replace=False)).astype(np.int32)[None, :]
    wg = rng.random((1, cfg.K)).astype(np.float32)
    wg /= wg.sum()
    res_np = np.linspace(-2, 2, cfg.H, dtype=np.float32)[None, :]
    y = expert_ffn(L, x, dev(ig), dev(wg), residual=dev(res_np), mode=moeq.MODE_DECODE)
    torch.cuda.synchronize()
    assert moeq.moeq_device_status() == 0
    from helpers import oracle_expert_outputs
    ref = oracle_expert_outputs(cfg, SEED, 0, xb, ig, wg.astype(np.float64), res_np)
    got = y.cpu().numpy()
    assert rel_l2(got, ref) <= 2e-3 and np.abs(got - ref).max() <= 1e-2
