"""Shared test helpers: host copies of synthetic layers for the oracle, and
the parity comparison of device layer outputs against the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle
from oracle.synthetic import host_router, host_tensor, oracle_layer  # noqa: F401

# Pass criteria for layer outputs against the fp64 oracle on the same bf16 inputs.
REL_L2 = 2e-3
MAX_ABS = 1e-2
# Routing: the GPU's choice may differ only where the oracle's K-th and
# (K+1)-th probabilities are within this relative margin.
NEAR_TIE = 1e-5


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def oracle_expert_outputs(cfg, seed, copy, x_bits, idx, wts, residual=None):
    """Oracle experts+combine for the given routing (compact bank of the
    experts that appear in idx)."""
    experts = np.unique(idx)
    remap = {int(e): i for i, e in enumerate(experts)}
    L = oracle_layer(cfg, seed, copy, experts)
    idx_c = np.vectorize(lambda e: remap[int(e)])(idx).astype(np.int32)
    return oracle.expert_ffn(L, x_bits, idx_c, wts, residual)


def oracle_routing(cfg, seed, copy, x_bits):
    """fp64 router logits and routing of the oracle."""
    R = host_router(cfg, seed, copy)
    logits = oracle.qmv(R, x_bits)
    idx, w, gap = oracle.route(logits, cfg.K, cfg.renorm, cfg.router_scale)
    return logits, idx, w, gap


def check_routing(idx_gpu, idx_o, gap_o, logits_o, cfg):
    """GPU top-K equals the oracle's except at near-ties; returns the mask of
    tokens whose choice differs (all of them near-ties)."""
    idx_gpu = np.asarray(idx_gpu)
    l = cfg.router_scale * np.asarray(logits_o, np.float64)
    p = np.exp(l - l.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    diff = np.any(idx_gpu != idx_o, axis=1)
    for t in np.nonzero(diff)[0]:
        g, o = idx_gpu[t], idx_o[t]
        assert len(set(g)) == cfg.K and g.min() >= 0 and g.max() < cfg.E
        if set(g) != set(o):
            # a different set only where the K-th choice is a near-tie
            assert gap_o[t] < NEAR_TIE, (t, g, o, gap_o[t])
        else:
            # same set, other order: only between near-equal probabilities
            for a, b in zip(g, o):
                if a != b:
                    assert abs(p[t, a] - p[t, b]) < NEAR_TIE * max(p[t, a], p[t, b]), (t, g, o)
    return diff


def weights_for(idx, logits_o, cfg):
    """fp64 routing weights of a given selection from the oracle's logits."""
    l = cfg.router_scale * np.asarray(logits_o, np.float64)
    p = np.exp(l - l.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    w = np.take_along_axis(p, np.asarray(idx, np.int64), axis=1)
    if cfg.renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return w


def check_layer_outputs(cfg, seed, copy, x_bits, y_gpu, idx_gpu, w_gpu, residual=None,
                        rows=None):
    """Full parity check of a layer forward (optionally on a subset of rows).
    Returns (rel_l2, max_abs, n_near_tie_tokens)."""
    x_bits = np.asarray(x_bits, np.uint16).reshape(-1, cfg.H)
    y_gpu = np.asarray(y_gpu, np.float64).reshape(-1, cfg.H)
    idx_gpu = np.asarray(idx_gpu).reshape(-1, cfg.K)
    w_gpu = np.asarray(w_gpu, np.float64).reshape(-1, cfg.K)
    if rows is not None:
        x_bits, y_gpu, idx_gpu, w_gpu = x_bits[rows], y_gpu[rows], idx_gpu[rows], w_gpu[rows]
        if residual is not None:
            residual = np.asarray(residual).reshape(-1, cfg.H)[rows]
    logits_o, idx_o, w_o, gap_o = oracle_routing(cfg, seed, copy, x_bits)
    diff = check_routing(idx_gpu, idx_o, gap_o, logits_o, cfg)
    # routing weights of the GPU's own selection agree with the fp64 ones
    w_ref = weights_for(idx_gpu, logits_o, cfg)
    assert np.abs(w_gpu - w_ref).max() < 1e-4, np.abs(w_gpu - w_ref).max()
    out_o = oracle_expert_outputs(cfg, seed, copy, x_bits, idx_gpu, w_ref, residual)
    r = rel_l2(y_gpu, out_o)
    m = float(np.abs(y_gpu - out_o).max())
    assert r <= REL_L2 and m <= MAX_ABS, (r, m)
    return r, m, int(diff.sum())
