"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden, each with its source), closed forms, brute-force
dense products built here by other code, invariants, and special cases that
reduce to textbook results.  A plausible mistake anywhere in the oracle
(dropped bias, wrong bit order, transposed operand, softmax/scale order,
SiLU on the wrong half, shared gate misplaced) fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
from quantized_mixture_experts_affine_b200 import synth

BF16_ONE = 0x3F80


def bf16_bits(v):
    """fp32 -> bf16 bits, round to nearest even (numpy, independent of the C code)."""
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def f32_of_bf16(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def pack(codes, bits):
    """codes [out][in] (ints) -> u32 words [out][in*bits/32]: value j of a
    row at bits [j*b, (j+1)*b) of the row as one little-endian integer (for
    3 and 6 bits values straddle words), built with Python big integers."""
    codes = np.asarray(codes, np.int64)
    out, n = codes.shape
    nw = n * bits // 32
    words = np.zeros((out, nw), np.uint32)
    for r in range(out):
        big = 0
        for j in range(n):
            big |= int(codes[r, j]) << (j * bits)
        for k in range(nw):
            words[r, k] = (big >> (32 * k)) & 0xFFFFFFFF
    return words


def unpack_np(words, bits, in_dim):
    """Inverse of pack, by Python big integers (independent of the oracle)."""
    words = np.asarray(words, np.uint32).reshape(-1, in_dim * bits // 32)
    out = np.zeros((words.shape[0], in_dim), np.int64)
    for r in range(words.shape[0]):
        big = 0
        for k, wv in enumerate(words[r]):
            big |= int(wv) << (32 * k)
        for j in range(in_dim):
            out[r, j] = (big >> (j * bits)) & ((1 << bits) - 1)
    return out


class T:
    """Minimal packed tensor for hand-built cases (one matrix)."""

    def __init__(self, codes, s_bits, b_bits, bits, G):
        codes = np.asarray(codes)
        self.out_dim, self.in_dim = codes.shape
        self.bits, self.group_size = bits, G
        self.w = pack(codes, bits)
        gshape = (self.out_dim, self.in_dim // G)
        self.s = np.ascontiguousarray(np.broadcast_to(np.asarray(s_bits, np.uint16), gshape))
        self.b = np.ascontiguousarray(np.broadcast_to(np.asarray(b_bits, np.uint16), gshape))


def dense_f64(t, mat=0):
    """Dense fp64 weights built here: codes by numpy bit extraction, then q*s+b."""
    q = unpack_np(t.w.reshape(-1, t.w.shape[-1])[mat * t.out_dim:(mat + 1) * t.out_dim],
                  t.bits, t.in_dim).astype(np.float64)
    s = f32_of_bf16(t.s.reshape(-1, t.s.shape[-1])[mat * t.out_dim:(mat + 1) * t.out_dim])
    b = f32_of_bf16(t.b.reshape(-1, t.b.shape[-1])[mat * t.out_dim:(mat + 1) * t.out_dim])
    s = np.repeat(s.astype(np.float64), t.group_size, axis=1)
    b = np.repeat(b.astype(np.float64), t.group_size, axis=1)
    return q * s + b


# ---------------------------------------------------------------- format

def test_packed_sizes_match_pages(golden):
    g = golden("format.json")
    e = g["expert_397b_4bit"]
    H, I = e["hidden"], e["intermediate"]
    per_expert = 2 * synth.packed_bytes(I, H, 4) + synth.packed_bytes(H, I, 4)
    assert per_expert == e["bytes_expected"] == 7077888
    assert per_expert / 2**20 == 6.75
    # fp32 scales/biases would give 7.5 MiB, not the printed ~6.75MB
    assert (per_expert + 2 * 2 * (2 * I * H // 64 + H * I // 64)) / 2**20 == 7.5
    # generated banks have exactly these sizes
    q = synth.tensor_host(0, synth.tag(synth.GATE), 1, I, H, 4)
    d = synth.tensor_host(0, synth.tag(synth.DOWN), 1, H, I, 4)
    assert 2 * q.nbytes + d.nbytes == e["bytes_expected"]
    # 2-bit / 4-bit ratio consistent with the printed pack totals (within 5%)
    two = 2 * synth.packed_bytes(I, H, 2) + synth.packed_bytes(H, I, 2)
    pt = g["pack_totals_gb"]
    assert abs(two / per_expert - pt["two_bit"] / pt["four_bit"]) < 0.05 * pt["two_bit"] / pt["four_bit"]
    gs = g["gate_shape"]
    assert gs["u32_shape"][1] * g["per_word"][str(gs["bits"])] == gs["in_dim_expected"]


def test_words_unpack_low_bits_first(golden):
    for c in golden("words.json")["cases"]:
        bits = c["bits"]
        per = 32 // bits
        word = int(c["word"], 16)
        t = T(np.zeros((1, 64)), BF16_ONE, 0, bits, 64)
        t.w[:] = 0
        t.w[0, 0] = word
        q = oracle.unpack(t)
        assert list(q[0, :per]) == c["codes"], c
        assert not q[0, per:].any()


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_unpack_matches_independent_extraction(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(7, 256))
    t = T(codes, BF16_ONE, 0, bits, 64)
    assert np.array_equal(oracle.unpack(t), codes)
    assert np.array_equal(unpack_np(t.w, bits, 256), codes)


# ---------------------------------------------------------------- dequant

@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
def test_dequant_endpoints_bit_exact(bits):
    """q = 0 -> bias and q = 2^b-1 -> bias + (2^b-1)*scale, exactly in fp32."""
    rng = np.random.default_rng(10 + bits)
    levels = (1 << bits) - 1
    codes = np.zeros((4, 128), np.int64)
    codes[:, 1::2] = levels
    s = bf16_bits(rng.uniform(1e-4, 1e-2, size=(4, 2)).astype(np.float32))
    b = bf16_bits(rng.uniform(-0.1, 0.0, size=(4, 2)).astype(np.float32))
    t = T(codes, s, b, bits, 64)
    w = oracle.dequant_f32(t)
    sf = np.repeat(f32_of_bf16(s), 64, 1).astype(np.float64)
    bf = np.repeat(f32_of_bf16(b), 64, 1).astype(np.float64)
    assert np.array_equal(w[:, 0::2], bf[:, 0::2].astype(np.float32))
    # exact value in fp64, rounded once to fp32
    assert np.array_equal(w[:, 1::2], (bf + levels * sf)[:, 1::2].astype(np.float32))


def test_dequant_matches_single_rounding_everywhere():
    q = synth.tensor_host(3, synth.tag(synth.UP), 1, 64, 256, 4)
    w = oracle.dequant_f32(q)
    assert np.array_equal(w, dense_f64(q).astype(np.float32))


@pytest.mark.parametrize("bits,G", [(2, 64), (4, 64), (8, 64), (4, 32), (8, 128), (3, 64),
                                    (6, 32), (3, 128), (5, 64), (5, 32)])
def test_quantiser_reconstruction_pins_format(bits, G):
    """Generator and oracle agree on the format: dequantised codes sit within
    half a quantisation step of the fp32 draws (a wrong bit order or group
    indexing would be off by many steps)."""
    tg = synth.tag(synth.GATE, 7)
    q = synth.tensor_host(5, tg, 2, 96, 512, bits, G)
    for m in range(2):
        w = synth.weights_f32_host(5, tg, m, 96, 512).astype(np.float64)
        dq = oracle.dequant_f32(q, m).astype(np.float64)
        s = np.repeat(f32_of_bf16(q.s[m]).astype(np.float64), G, 1)
        wg = w.reshape(96, -1, G)
        slack = np.repeat(2.0**-7 * np.abs(wg).max(-1), G, 1)
        assert (np.abs(dq - w) <= 0.5 * s + slack + 1e-12).all()
        # and the draws are N(0, 0.02)-like
        assert abs(w.std() - 0.02) < 0.002


def test_requantised_2bit_reconstruction():
    """4->2 bit requantisation: 2-bit codes reconstruct the 4-bit dequantised
    values within half a 2-bit step."""
    tg = synth.tag(synth.DOWN, 3)
    q4 = synth.tensor_host(9, tg, 1, 32, 256, 4)
    q2 = synth.tensor_host(9, tg, 1, 32, 256, 2, requant_from4=True)
    w4 = oracle.dequant_f32(q4).astype(np.float64)
    w2 = oracle.dequant_f32(q2).astype(np.float64)
    s2 = np.repeat(f32_of_bf16(q2.s[0]).astype(np.float64), 64, 1)
    slack = np.repeat(2.0**-7 * np.abs(w4.reshape(32, -1, 64)).max(-1), 64, 1)
    assert (np.abs(w2 - w4) <= 0.5 * s2 + slack).all()


# ---------------------------------------------------------------- qmv

@pytest.mark.parametrize("bits,G,out,inn", [(4, 64, 40, 256), (8, 64, 17, 320), (2, 64, 33, 128),
                                            (4, 32, 9, 96), (8, 128, 5, 384), (3, 64, 11, 256),
                                            (6, 32, 7, 192), (3, 32, 5, 96)])
def test_qmv_equals_bruteforce_dense(bits, G, out, inn):
    tg = synth.tag(synth.ROUTER, bits)
    q = synth.tensor_host(11, tg, 2, out, inn, bits, G)
    x = synth.normal_bf16_host(11, synth.tag(synth.X, bits), 3 * inn).reshape(3, inn)
    xf = f32_of_bf16(x).astype(np.float64)
    for m in range(2):
        W = dense_f64(q, m)
        ref = xf @ W.T
        y = oracle.qmv(q, x, mat=m)
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
        # a transposed or mis-strided operand would not match a non-square product
        assert W.shape == (out, inn)


def test_fma_factoring_agrees():
    """fma(q, s*x, b*x), (q*s + b)*x and the group form s*sum(q x) + b*sum(x)
    agree to rounding (flash-moe-inference, matvec_4bit_fma listing)."""
    q = synth.tensor_host(13, synth.tag(synth.GATE, 1), 1, 24, 512, 4)
    x = f32_of_bf16(synth.normal_bf16_host(13, synth.tag(synth.X, 1), 512)).astype(np.float64)
    codes = unpack_np(q.w[0], 4, 512).astype(np.float64)
    s = np.repeat(f32_of_bf16(q.s[0]).astype(np.float64), 64, 1)
    b = np.repeat(f32_of_bf16(q.b[0]).astype(np.float64), 64, 1)
    naive = ((codes * s + b) * x).sum(1)
    fma = (codes * (s * x) + (b * x)).sum(1)
    grp = ((codes * x).reshape(24, -1, 64).sum(-1) * s[:, ::64]
           + x.reshape(-1, 64).sum(-1)[None] * b[:, ::64]).sum(1)
    mag = (np.abs(codes * s * x) + np.abs(b * x)).sum(1)
    y = oracle.qmv_f64(q, x[None])[0]
    for v in (naive, fma, grp):
        assert (np.abs(v - y) <= 64 * np.finfo(np.float64).eps * mag).all()


def test_integer_special_case_exact():
    """8-bit, scale 1, bias 0: the product is an exact integer matvec."""
    rng = np.random.default_rng(21)
    codes = rng.integers(0, 256, size=(13, 192))
    t = T(codes, BF16_ONE, 0, 8, 64)
    xi = rng.integers(-8, 9, size=(2, 192))
    x = bf16_bits(xi.astype(np.float32))
    y = oracle.qmv(t, x)
    assert np.array_equal(y, (xi @ codes.T).astype(np.float64))


def test_one_hot_returns_dequantised_column():
    q = synth.tensor_host(17, synth.tag(synth.DOWN, 2), 1, 48, 256, 4)
    w = oracle.dequant_f32(q)
    for c in (0, 63, 64, 200, 255):
        x = np.zeros((1, 256), np.uint16)
        x[0, c] = BF16_ONE
        y = oracle.qmv(q, x)
        assert np.array_equal(y[0], w[:, c].astype(np.float64))


# ---------------------------------------------------------------- routing

def test_route_closed_forms(golden):
    g = golden("router.json")
    for c in g["cases"]:
        logits = np.log(np.array([c["p"]], np.float64))
        idx, w, gap = oracle.route(logits, c["K"], c["renorm"], c["scale"])
        assert list(idx[0]) == c["idx"], c
        assert np.allclose(w[0], c["w"], rtol=1e-14, atol=1e-15), c
    c = g["scaled"]
    logits = np.log(np.array([c["p"]], np.float64)) / c["scale"]
    idx, w, _ = oracle.route(logits, c["K"], True, c["scale"])
    assert list(idx[0]) == c["idx"]
    assert np.allclose(w[0], c["w"], rtol=1e-14)
    # scale applied BEFORE softmax: with scale 1 the same logits give other weights
    _, w1, _ = oracle.route(logits, c["K"], True, 1.0)
    assert not np.allclose(w1[0], c["w"], rtol=1e-3)


def test_route_k_equals_e_is_softmax():
    rng = np.random.default_rng(3)
    l = rng.normal(size=(5, 16))
    idx, w, _ = oracle.route(l, 16, True, 1.0)
    sm = np.exp(l - l.max(1, keepdims=True))
    sm /= sm.sum(1, keepdims=True)
    for t in range(5):
        assert np.allclose(w[t], sm[t][idx[t]], rtol=1e-13)
        assert sorted(idx[t]) == list(range(16))


def test_route_renorm_is_softmax_over_selected():
    rng = np.random.default_rng(4)
    l = rng.normal(size=(20, 64)) * 2
    idx, w, gap = oracle.route(l, 6, True, 1.0)
    for t in range(20):
        sel = l[t, idx[t]]
        sm = np.exp(sel - sel.max())
        sm /= sm.sum()
        assert np.allclose(w[t], sm, rtol=1e-13)
        assert abs(w[t].sum() - 1) < 1e-12
        assert (np.diff(w[t]) <= 0).all()
        assert len(set(idx[t])) == 6 and idx[t].min() >= 0 and idx[t].max() < 64
        rest = np.delete(l[t], idx[t])
        assert l[t, idx[t]].min() >= rest.max()
        p = np.exp(l[t] - l[t].max())
        p /= p.sum()
        ps = np.sort(p)[::-1]
        assert np.isclose(gap[t], (ps[5] - ps[6]) / ps[5], rtol=1e-10)


def test_route_ties_lower_index():
    l = np.array([[1.0, 1.0, 1.0, 0.0, 1.0]])
    idx, w, gap = oracle.route(l, 2, True, 1.0)
    assert list(idx[0]) == [0, 1]
    assert gap[0] == 0.0


# ---------------------------------------------------------------- experts / layer

def _const_tensor(out, inn, bias, bits=4, G=64):
    return T(np.zeros((out, inn), np.int64), BF16_ONE, bf16_bits(np.float32(bias)), bits, G)


def _bank(ts):
    """Stack single-matrix tensors into a bank."""
    t0 = ts[0]
    b = T(np.zeros((1, t0.in_dim), np.int64), BF16_ONE, 0, t0.bits, t0.group_size)
    b.out_dim, b.in_dim = t0.out_dim, t0.in_dim
    b.w = np.ascontiguousarray(np.stack([t.w for t in ts]))
    b.s = np.ascontiguousarray(np.stack([t.s for t in ts]))
    b.b = np.ascontiguousarray(np.stack([t.b for t in ts]))
    return b


def test_swiglu_layer_golden(golden):
    g = golden("swiglu_layer.json")
    H = 64
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = BF16_ONE
    router = _const_tensor(1, H, 0.0, bits=8)
    for c in g["cases"]:
        I = c["I"]
        L = oracle.OracleLayer(router=oracle.OracleTensor.of(router),
                               gate=oracle.OracleTensor.of(_const_tensor(I, H, c["bias_gate"])),
                               up=oracle.OracleTensor.of(_const_tensor(I, H, c["bias_up"])),
                               down=oracle.OracleTensor.of(_const_tensor(H, I, c["bias_down"])),
                               H=H, I=I, E=1, K=1)
        r = oracle.layer(L, x)
        assert np.allclose(r["out"], c["out"], rtol=1e-15), (r["out"][0, :3], c)
        assert list(r["idx"][0]) == [0] and r["w"][0, 0] == 1.0
    s = g["shared"]
    I = 64
    L = oracle.OracleLayer(
        router=oracle.OracleTensor.of(router),
        gate=oracle.OracleTensor.of(_const_tensor(I, H, s["routed"]["bias_gate"])),
        up=oracle.OracleTensor.of(_const_tensor(I, H, s["routed"]["bias_up"])),
        down=oracle.OracleTensor.of(_const_tensor(H, I, s["routed"]["bias_down"])),
        H=H, I=I, E=1, K=1,
        sh_gate=oracle.OracleTensor.of(_const_tensor(I, H, s["shared"]["bias_gate"])),
        sh_up=oracle.OracleTensor.of(_const_tensor(I, H, s["shared"]["bias_up"])),
        sh_down=oracle.OracleTensor.of(_const_tensor(H, I, s["shared"]["bias_down"])),
        sh_expert_gate=oracle.OracleTensor.of(_const_tensor(1, H, 0.0, bits=8)))
    r = oracle.layer(L, x)
    assert np.allclose(r["out"], s["out"], rtol=1e-15)


def _rand_layer(seed, H, I, E, K, shared, ebits=4, rbits=8):
    mk = lambda kind, n, o, i, b: oracle.OracleTensor.of(
        synth.tensor_host(seed, synth.tag(kind), n, o, i, b))
    kw = {}
    if shared:
        kw = dict(sh_gate=mk(synth.SH_GATE, 1, I, H, ebits), sh_up=mk(synth.SH_UP, 1, I, H, ebits),
                  sh_down=mk(synth.SH_DOWN, 1, H, I, ebits),
                  sh_expert_gate=mk(synth.SH_EXPERT_GATE, 1, 1, H, 8))
    return oracle.OracleLayer(router=mk(synth.ROUTER, 1, E, H, rbits),
                              gate=mk(synth.GATE, E, I, H, ebits), up=mk(synth.UP, E, I, H, ebits),
                              down=mk(synth.DOWN, E, H, I, ebits), H=H, I=I, E=E, K=K, **kw)


def test_layer_equals_dense_composition():
    """Tiny random layer vs a dense fp64 composition built here from the
    numpy-unpacked weights: router -> softmax -> top-K -> renorm ->
    SwiGLU experts -> weighted sum + sigmoid-gated shared expert."""
    H, I, E, K = 128, 64, 6, 2
    L = _rand_layer(23, H, I, E, K, shared=True)
    x = synth.normal_bf16_host(23, synth.tag(synth.X), 4 * H).reshape(4, H)
    xf = f32_of_bf16(x).astype(np.float64)
    r = oracle.layer(L, x)
    Wr = dense_f64(L.router)
    sig = lambda v: 1 / (1 + np.exp(-v))
    for t in range(4):
        lg = Wr @ xf[t]
        p = np.exp(lg - lg.max())
        p /= p.sum()
        top = np.argsort(-p, kind="stable")[:K]
        w = p[top] / p[top].sum()
        assert list(r["idx"][t]) == list(top)
        out = np.zeros(H)
        for k, e in enumerate(top):
            g = dense_f64(L.gate, e) @ xf[t]
            u = dense_f64(L.up, e) @ xf[t]
            out += w[k] * (dense_f64(L.down, e) @ (g * sig(g) * u))
        g = dense_f64(L.sh_gate) @ xf[t]
        u = dense_f64(L.sh_up) @ xf[t]
        out += sig(dense_f64(L.sh_expert_gate) @ xf[t])[0] * (dense_f64(L.sh_down) @ (g * sig(g) * u))
        assert np.allclose(r["out"][t], out, rtol=1e-11, atol=1e-12 * np.abs(out).max())


def test_expert_ffn_matches_layer_given_its_routing():
    L = _rand_layer(29, 128, 64, 8, 3, shared=False)
    x = synth.normal_bf16_host(29, synth.tag(synth.X), 3 * 128).reshape(3, 128)
    r = oracle.layer(L, x)
    y = oracle.expert_ffn(L, x, r["idx"], r["w"])
    assert np.array_equal(y, r["out"])


def test_per_token_independence():
    """A token's output does not depend on the other tokens of the batch
    (Silent numerical corruption ... % 32 != 0, mlx issue 3856: one-shot and
    chunked prefill must agree)."""
    L = _rand_layer(31, 128, 64, 8, 2, shared=True)
    x = synth.normal_bf16_host(31, synth.tag(synth.X), 7 * 128).reshape(7, 128)
    full = oracle.layer(L, x)["out"]
    for t in range(7):
        one = oracle.layer(L, x[t:t + 1])["out"]
        assert np.array_equal(one[0], full[t])
    chunks = np.concatenate([oracle.layer(L, x[i:i + 3])["out"] for i in range(0, 7, 3)])
    assert np.array_equal(chunks, full)


def test_residual_adds_through():
    L = _rand_layer(37, 128, 64, 4, 2, shared=False)
    x = synth.normal_bf16_host(37, synth.tag(synth.X), 2 * 128).reshape(2, 128)
    res = np.linspace(-1, 1, 256, dtype=np.float32).reshape(2, 128)
    a = oracle.layer(L, x)["out"]
    b = oracle.layer(L, x, residual=res)["out"]
    assert np.allclose(b - a, res.astype(np.float64), rtol=0, atol=1e-12)


def test_threads_do_not_change_results():
    L = _rand_layer(41, 128, 64, 8, 2, shared=True)
    x = synth.normal_bf16_host(41, synth.tag(synth.X), 6 * 128).reshape(6, 128)
    oracle.set_threads(1)
    a = oracle.layer(L, x)["out"]
    oracle.set_threads(4)
    b = oracle.layer(L, x)["out"]
    oracle.set_threads(0)
    assert np.array_equal(a, b)


def test_route_under_exp_underflow_selects_by_logit():
    """Scores that underflow to 0 in fp64 (logit gaps of ~1000) still rank
    by their logits, as the strictly increasing softmax ranks them; the
    near-tie gap stays defined (1 - exp(l_next - l_K))."""
    l = np.array([[0.0, -3000.0, -2000.0, -1000.0, 5.0]])
    idx, w, gap = oracle.route(l, 3, True, 1.0)
    assert idx[0].tolist() == [4, 0, 3]
    e5 = np.exp(-5.0)
    assert np.allclose(w[0], [1 / (1 + e5), e5 / (1 + e5), 0.0], rtol=1e-14, atol=1e-300)
    assert gap[0] == 1.0
    # a negative router scale reverses the order of the logits
    idx, _, _ = oracle.route(l, 2, True, -1.0)
    assert idx[0].tolist() == [1, 2]


# ------------------------------------------------------------------ RMS norm of the output

def _bf16(v):
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_rmsnorm_worked_row():
    """(3, 4): mean square 12.5, so with eps 0 and unit weights the row
    becomes (3, 4) / sqrt(12.5); weights 2 and 0.5 scale each column."""
    out = oracle.rmsnorm(np.array([[3.0, 4.0]]), _bf16([1.0, 1.0]), 0.0)
    assert np.allclose(out, [[3 / np.sqrt(12.5), 4 / np.sqrt(12.5)]], rtol=1e-15)
    out = oracle.rmsnorm(np.array([[3.0, 4.0]]), _bf16([2.0, 0.5]), 0.0)
    assert np.allclose(out, [[6 / np.sqrt(12.5), 2 / np.sqrt(12.5)]], rtol=1e-15)


def test_rmsnorm_invariants():
    """With eps 0 and unit weights every output row has mean square 1, and
    the result does not change when a row is scaled by a positive factor;
    with eps > 0 a constant row c gives c / sqrt(c^2 + eps)."""
    rng = np.random.default_rng(3)
    y = rng.normal(size=(5, 64)) * rng.uniform(0.1, 100, size=(5, 1))
    one = _bf16(np.ones(64))
    out = oracle.rmsnorm(y, one, 0.0)
    assert np.allclose((out ** 2).mean(axis=1), 1.0, rtol=1e-13)
    assert np.allclose(oracle.rmsnorm(7.5 * y, one, 0.0), out, rtol=1e-13)
    c = oracle.rmsnorm(np.full((1, 8), 0.5), _bf16(np.ones(8)), 1e-2)
    assert np.allclose(c, 0.5 / np.sqrt(0.25 + 1e-2), rtol=1e-15)
    # rows are independent of one another
    assert np.allclose(oracle.rmsnorm(y[2:3], one, 1e-6), oracle.rmsnorm(y, one, 1e-6)[2:3])


# ------------------------------------------------------------------ MX FP4 codes

# The E2M1 element values of the OCP Microscaling Formats specification
# (v1.0, FP4 E2M1 table): codes 0..7 and their negatives 8..15.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
              -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def _mx_tensor(codes, ebytes):
    """Host MX FP4 tensor from unpacked codes [out][in] and exponent bytes
    [out][in/32] (packed here independently of the oracle: 8 codes per word,
    low nibble first)."""
    codes = np.asarray(codes, np.uint32)
    out, inn = codes.shape
    w = np.zeros((1, out, inn // 8), np.uint32)
    for j in range(8):
        w[0] |= codes[:, j::8] << (4 * j)
    e = np.ascontiguousarray(np.asarray(ebytes, np.uint8).reshape(1, out, inn // 32))
    return oracle.OracleTensor(w, e, np.zeros(0, np.uint16), out, inn, 4, 32, 1)


def test_mxfp4_element_table_and_scale_bytes():
    codes = np.tile(np.arange(16), 2)[None, :]            # one row of 32 values
    for x, f in ((127, 1.0), (128, 2.0), (126, 0.5), (120, 2.0 ** -7), (140, 2.0 ** 13)):
        w = oracle.dequant_f32(_mx_tensor(codes, [[x]]))
        assert np.array_equal(w[0], np.array(E2M1_TABLE * 2, np.float32) * np.float32(f)), x
        assert np.array_equal(np.signbit(w[0]), np.signbit(np.array(E2M1_TABLE * 2)))
    assert np.isnan(oracle.dequant_f32(_mx_tensor(codes, [[255]]))).all()
    q = oracle.unpack(_mx_tensor(codes, [[127]]))
    assert np.array_equal(q[0], codes[0])


def test_mxfp4_qmv_brute_force():
    """Random codes and exponents (several groups per row): the oracle's
    qmv equals a dense fp64 product of the table-decoded weights."""
    rng = np.random.default_rng(7)
    out, inn = 5, 128
    codes = rng.integers(0, 16, (out, inn))
    eb = rng.integers(110, 140, (out, inn // 32))
    t = _mx_tensor(codes, eb)
    dense = np.array(E2M1_TABLE)[codes] * np.ldexp(1.0, np.repeat(eb, 32, axis=1) - 127)
    xb = _bf16(rng.normal(size=(3, inn)))
    x = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    got = oracle.qmv(t, xb)
    assert np.allclose(got, x @ dense.T, rtol=1e-13, atol=1e-300)


def test_mxfp4_generator_round_trip():
    """The generator's MX quantiser: every element within half an E2M1 step
    (at its magnitude) times the group scale of the fp32 weight, the group
    maximum mapped into [4, 6], and host and device streams equal by
    construction (shared recipe)."""
    H, O = 256, 6
    t = synth.tensor_mx_host(3, synth.tag(synth.GATE), 1, O, H)
    w32 = synth.weights_f32_host(3, synth.tag(synth.GATE), 0, O, H)
    deq = oracle.dequant_f32(oracle.OracleTensor.of(t))
    scale = np.ldexp(1.0, np.repeat(t.s[0].astype(int), 32, axis=1) - 127)
    v = np.abs(w32 / scale)
    step = np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0))
    over = np.maximum(v - 6.0, 0.0)
    assert (np.abs(deq - w32) <= (step / 2 + over) * scale + 1e-12).all()
    amax = np.abs(deq).reshape(O, H // 32, 32).max(axis=2) / scale[:, ::32]
    assert ((amax >= 4.0) & (amax <= 6.0)).all()



def test_cross_word_packing_by_hand():
    """3 bits: 32 values in 3 words, value 10 straddling words 0 and 1 (bits
    30..32) and value 21 words 1 and 2 (bits 63..65); 6 bits: value 5 at bits
    30..35 straddles words 0 and 1; 5 bits: value 6 at bits 30..34 straddles
    words 0 and 1, value 12 at bits 60..64 words 1 and 2."""
    codes = np.zeros((1, 32), np.int64)
    codes[0, 10] = 0b110      # bits 30, 31 = 0, 1 ; bit 32 = 1
    codes[0, 21] = 0b011      # bit 63 = 1 ; bits 64, 65 = 1, 0
    t = T(codes, BF16_ONE, 0, 3, 32)
    assert t.w.tolist() == [[0x80000000, 0x80000001, 0x00000001]]
    assert np.array_equal(oracle.unpack(t), codes)
    c6 = np.zeros((1, 32), np.int64)
    c6[0, 5] = 0b101101       # bits 30, 31 = 1, 0 ; bits 32..35 = 1, 1, 0, 1
    t6 = T(c6, BF16_ONE, 0, 6, 32)
    assert t6.w[0, 0] == 0x40000000 and t6.w[0, 1] == 0x0000000B
    assert np.array_equal(oracle.unpack(t6), c6)
    c5 = np.zeros((1, 32), np.int64)
    c5[0, 6] = 0b10111        # bits 30, 31 = 1, 1 ; bits 32..34 = 1, 0, 1
    c5[0, 12] = 0b11001       # bits 60..63 = 1, 0, 0, 1 ; bit 64 = 1
    t5 = T(c5, BF16_ONE, 0, 5, 32)
    assert t5.w.tolist() == [[0xC0000000, 0x90000005, 0x00000001, 0, 0]]
    assert np.array_equal(oracle.unpack(t5), c5)
