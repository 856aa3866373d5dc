"""Layer descriptors over device-resident packed weights.

``DeviceLayer`` owns the torch tensors of one layer and the ``moeq_layer``
struct that points at them.  ``synthetic_layer`` fills one from the seeded
generator; real weights can be wrapped the same way with ``moeq.qtensor``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from . import moeq
from . import synth
from .config import CONFIGS, LayerConfig  # noqa: F401  (re-exported)


@dataclass
class DeviceLayer:
    cfg: LayerConfig
    router: synth.DevQ
    gate: synth.DevQ
    up: synth.DevQ
    down: synth.DevQ
    sh_gate: synth.DevQ | None = None
    sh_up: synth.DevQ | None = None
    sh_down: synth.DevQ | None = None
    sh_expert_gate: synth.DevQ | None = None
    desc: moeq.Layer = field(default=None)

    def __post_init__(self):
        c = self.cfg

        def q(t: synth.DevQ):
            return moeq.qtensor(t.w, t.s, t.b, t.out_dim, t.in_dim, t.bits, t.group_size,
                                t.n_mats, getattr(t, "fmt", 0))
        z = moeq.QTensor()
        self.desc = moeq.Layer(q(self.router), q(self.gate), q(self.up), q(self.down),
                               int(c.shared), q(self.sh_gate) if c.shared else z,
                               q(self.sh_up) if c.shared else z,
                               q(self.sh_down) if c.shared else z,
                               q(self.sh_expert_gate) if c.shared else z,
                               c.H, c.I, c.E, c.K, int(c.renorm), float(c.router_scale))

    def nbytes(self) -> int:
        ts = [self.router, self.gate, self.up, self.down]
        if self.cfg.shared:
            ts += [self.sh_gate, self.sh_up, self.sh_down, self.sh_expert_gate]
        return sum(t.nbytes for t in ts)


def synthetic_layer(cfg: LayerConfig, seed: int = 0, copy: int = 0, device="cuda") -> DeviceLayer:
    """All tensors of one layer drawn on the device from the seeded streams
    (stream tag = (tensor kind, copy), matrix m of a bank = tag + m)."""
    T = lambda kind: synth.tag(kind, copy)
    mk = lambda kind, n, o, i, b, rq=False: synth.tensor_dev(seed, T(kind), n, o, i, b, cfg.G, rq,
                                                             device)
    kw = {}
    if cfg.shared:
        kw = dict(sh_gate=mk(synth.SH_GATE, 1, cfg.shared_I, cfg.H, cfg.shared_bits),
                  sh_up=mk(synth.SH_UP, 1, cfg.shared_I, cfg.H, cfg.shared_bits),
                  sh_down=mk(synth.SH_DOWN, 1, cfg.H, cfg.shared_I, cfg.shared_bits),
                  sh_expert_gate=mk(synth.SH_EXPERT_GATE, 1, 1, cfg.H, cfg.shared_gate_bits))
    return DeviceLayer(cfg,
                       router=mk(synth.ROUTER, 1, cfg.E, cfg.H, cfg.router_bits),
                       gate=mk(synth.GATE, cfg.E, cfg.I, cfg.H, cfg.expert_bits, cfg.requant_from4),
                       up=mk(synth.UP, cfg.E, cfg.I, cfg.H, cfg.expert_bits, cfg.requant_from4),
                       down=mk(synth.DOWN, cfg.E, cfg.H, cfg.I, cfg.expert_bits, cfg.requant_from4),
                       **kw)


class Workspace:
    """A device workspace sized for a layer, a token count and a mode."""

    def __init__(self, L: DeviceLayer, M: int, mode: int = moeq.MODE_AUTO, device="cuda"):
        import torch
        self.bytes = moeq.moeq_workspace_bytes(L.desc, M, mode)
        if self.bytes == 0:
            raise moeq.MoeqError("moeq_workspace_bytes", moeq.ERR_UNSUPPORTED)
        # 256-byte aligned (torch's caching allocator aligns to 512)
        self.buf = torch.empty(self.bytes, dtype=torch.uint8, device=device)


def layer_forward(L: DeviceLayer, x, y=None, residual=None, idx=None, w=None, ws=None,
                  mode: int = moeq.MODE_AUTO, stream=None):
    """y = layer(x) for bf16 x [M][H] on the device; returns (y, idx, w)."""
    import torch
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, L.cfg.H), dtype=torch.float32, device=x.device)
    if idx is None:
        idx = torch.empty((M, L.cfg.K), dtype=torch.int32, device=x.device)
    if w is None:
        w = torch.empty((M, L.cfg.K), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = Workspace(L, M, mode, x.device)
    moeq.moeq_layer_forward(L.desc, x, M, y, residual, idx, w, ws.buf, ws.bytes, mode, stream)
    return y, idx, w


def layer_forward_norm(L: DeviceLayer, x, gamma, eps: float, y=None, y_norm=None, residual=None,
                       idx=None, w=None, ws=None, mode: int = moeq.MODE_AUTO, stream=None):
    """y = layer(x) and y_norm = bf16 RMS norm of y with weights gamma (bf16
    [H]); returns (y, y_norm, idx, w)."""
    import torch
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, L.cfg.H), dtype=torch.float32, device=x.device)
    if y_norm is None:
        y_norm = torch.empty((M, L.cfg.H), dtype=torch.bfloat16, device=x.device)
    if idx is None:
        idx = torch.empty((M, L.cfg.K), dtype=torch.int32, device=x.device)
    if w is None:
        w = torch.empty((M, L.cfg.K), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = Workspace(L, M, mode, x.device)
    moeq.moeq_layer_forward_norm(L.desc, x, M, y, gamma, eps, y_norm, residual, idx, w, ws.buf,
                                 ws.bytes, mode, stream)
    return y, y_norm, idx, w


def expert_ffn(L: DeviceLayer, x, idx, w, y=None, residual=None, ws=None,
               mode: int = moeq.MODE_AUTO, stream=None):
    import torch
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, L.cfg.H), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = Workspace(L, M, mode, x.device)
    moeq.moeq_expert_ffn(L.desc, x, M, idx, w, residual, y, ws.buf, ws.bytes, mode, stream)
    return y
