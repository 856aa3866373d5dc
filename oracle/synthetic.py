"""Oracle layers over the seeded synthetic weights.

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).  The
host copies come from the seeded input generator (the same bytes the device
generator writes); `cfg` is any object with the layer-shape fields (H, I,
E, K, G, bit widths, shared-expert fields, renorm, router_scale,
requant_from4).
"""
from __future__ import annotations

import numpy as np

from quantized_mixture_experts_affine_b200 import synth

from .oracle import OracleLayer, OracleTensor


def host_tensor(cfg, seed: int, kind: int, copy: int, out_dim: int, in_dim: int, bits: int,
                mats=None, requant=False):
    """Host copy of a bank (all matrices, or the listed ones stacked in order)."""
    tg = synth.tag(kind, copy)
    if mats is None:
        return synth.tensor_host(seed, tg, 1, out_dim, in_dim, bits, cfg.G, requant)
    parts = [synth.tensor_host(seed, tg, 1, out_dim, in_dim, bits, cfg.G, requant, first_mat=int(m))
             for m in mats]
    return synth.HostQ(np.ascontiguousarray(np.concatenate([p.w for p in parts])),
                       np.ascontiguousarray(np.concatenate([p.s for p in parts])),
                       np.ascontiguousarray(np.concatenate([p.b for p in parts])),
                       out_dim, in_dim, bits, cfg.G, len(parts))


def host_router(cfg, seed, copy=0):
    return host_tensor(cfg, seed, synth.ROUTER, copy, cfg.E, cfg.H, cfg.router_bits)


def oracle_layer(cfg, seed: int, copy: int, experts):
    """Oracle layer whose banks hold only `experts` (in that order)."""
    rq = cfg.requant_from4
    O = OracleTensor.of
    kw = {}
    if cfg.shared:
        kw = dict(
            sh_gate=O(host_tensor(cfg, seed, synth.SH_GATE, copy, cfg.shared_I, cfg.H, cfg.shared_bits)),
            sh_up=O(host_tensor(cfg, seed, synth.SH_UP, copy, cfg.shared_I, cfg.H, cfg.shared_bits)),
            sh_down=O(host_tensor(cfg, seed, synth.SH_DOWN, copy, cfg.H, cfg.shared_I, cfg.shared_bits)),
            sh_expert_gate=O(host_tensor(cfg, seed, synth.SH_EXPERT_GATE, copy, 1, cfg.H,
                                         cfg.shared_gate_bits)))
    return OracleLayer(
        router=O(host_router(cfg, seed, copy)),
        gate=O(host_tensor(cfg, seed, synth.GATE, copy, cfg.I, cfg.H, cfg.expert_bits, experts, rq)),
        up=O(host_tensor(cfg, seed, synth.UP, copy, cfg.I, cfg.H, cfg.expert_bits, experts, rq)),
        down=O(host_tensor(cfg, seed, synth.DOWN, copy, cfg.H, cfg.I, cfg.expert_bits, experts, rq)),
        H=cfg.H, I=cfg.I, E=len(experts), K=cfg.K, renorm=cfg.renorm,
        router_scale=cfg.router_scale, **kw)
