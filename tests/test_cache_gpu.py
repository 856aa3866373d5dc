"""Expert streaming from host memory through an HBM expert cache
(moeq_cache_*), against the device-resident layer and the oracle.

Bars: every step's routing equals the device-resident layer's and its
output agrees with it and with the oracle within the layer tolerance; the
cache's hit and miss counts and copied bytes equal a Python replay of the
same least-recently-used policy on the same selections.
"""
import numpy as np
import pytest

import oracle
from helpers import check_layer_outputs
from quantized_mixture_experts_affine_b200 import moeq, synth
from quantized_mixture_experts_affine_b200.layer import (DeviceLayer, LayerConfig, layer_forward,
                                                         synthetic_layer)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
SEED = 0
CFG = LayerConfig("stream", H=1024, I=512, E=64, K=4, expert_bits=4, shared=True, shared_I=512,
                  shared_bits=4)


def host_copy(d):
    """The same bank in page-locked host memory."""
    return synth.DevQ(d.w.cpu().pin_memory(), d.s.cpu().pin_memory(), d.b.cpu().pin_memory(),
                      d.out_dim, d.in_dim, d.bits, d.group_size, d.n_mats, d.fmt)


def replay_lru(selections, slots):
    """Hits, misses of the cache policy on a sequence of per-step selections."""
    where, last, owner = {}, [0] * slots, [-1] * slots
    hits = misses = 0
    for step, sel in enumerate(selections, start=1):
        for e in sel:
            if e in where:
                if last[where[e]] != step:
                    hits += 1
            else:
                free = [q for q in range(slots) if last[q] != step]
                empty = [q for q in free if owner[q] < 0]
                v = empty[0] if empty else min(free, key=lambda q: (last[q], q))
                if owner[v] >= 0:
                    del where[owner[v]]
                owner[v], where[e] = e, v
                misses += 1
            last[where[e]] = step
    return hits, misses


@pytest.mark.parametrize("M,slots", [(1, 8), (2, 8), (1, 4)])
def test_cache_streams_experts(M, slots):
    cfg = CFG
    L = synthetic_layer(cfg, SEED, 0)
    hb = {k: host_copy(getattr(L, k)) for k in ("gate", "up", "down")}
    host = DeviceLayer(cfg, router=L.router, gate=hb["gate"], up=hb["up"], down=hb["down"],
                       sh_gate=L.sh_gate, sh_up=L.sh_up, sh_down=L.sh_down,
                       sh_expert_gate=L.sh_expert_gate)
    cache = moeq.ExpertCache(host.desc, slots, M)
    ws = torch.empty(cache.workspace_bytes(M), dtype=torch.uint8, device="cuda")
    sels = []
    try:
        for step in range(8):
            xb = synth.normal_bf16_host(SEED, synth.tag(synth.X, 500 + step), M * cfg.H)
            xb = xb.reshape(M, cfg.H)
            x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
            y = torch.full((M, cfg.H), float("nan"), device="cuda")
            idx = torch.empty((M, cfg.K), dtype=torch.int32, device="cuda")
            w = torch.empty((M, cfg.K), device="cuda")
            cache.forward(x, M, y, ws, ws.numel(), idx_out=idx, w_out=w)
            y0, i0, w0 = layer_forward(L, x, mode=moeq.MODE_DECODE)
            torch.cuda.synchronize()
            assert moeq.moeq_device_status() == 0
            assert torch.equal(idx, i0)
            got, ref = y.cpu().numpy(), y0.cpu().numpy()
            assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-5
            if step % 3 == 0:
                check_layer_outputs(cfg, SEED, 0, xb, got, idx.cpu().numpy(), w.cpu().numpy())
            ig = idx.cpu().numpy()
            sels.append([int(e) for e in ig.reshape(-1)])
        hits, misses, nbytes = cache.stats()
        assert (hits, misses) == replay_lru(sels, slots)
        per_expert = 3 * synth.packed_bytes(cfg.I, cfg.H, 4, cfg.G)
        assert nbytes == misses * per_expert
    finally:
        cache.close()
