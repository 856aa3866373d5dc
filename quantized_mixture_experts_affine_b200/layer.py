"""Layer descriptors over device-resident packed weights.

``DeviceLayer`` owns the torch tensors of one layer and the ``moeq_layer``
struct that points at them.  ``synthetic_layer`` fills one from the seeded
generator; real weights can be wrapped the same way with ``moeq.qtensor``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from . import moeq
from . import synth


@dataclass(frozen=True)
class LayerConfig:
    name: str
    H: int                 # hidden
    I: int                 # expert intermediate
    E: int                 # experts
    K: int                 # top-K
    expert_bits: int
    router_bits: int = 8
    shared: bool = False
    shared_I: int = 0
    shared_bits: int = 4
    shared_gate_bits: int = 8
    G: int = 64
    renorm: bool = True
    router_scale: float = 1.0
    requant_from4: bool = False   # experts requantised 4 -> expert_bits

    def expert_bytes(self) -> int:
        return 3 * synth.packed_bytes(self.I, self.H, self.expert_bits, self.G)

    def router_bytes(self) -> int:
        return synth.packed_bytes(self.E, self.H, self.router_bits, self.G)

    def shared_bytes(self) -> int:
        if not self.shared:
            return 0
        return (3 * synth.packed_bytes(self.shared_I, self.H, self.shared_bits, self.G)
                + synth.packed_bytes(1, self.H, self.shared_gate_bits, self.G))

    def decode_bytes_per_token(self) -> int:
        """Weight bytes one token needs (router + K experts + shared expert)."""
        return self.router_bytes() + self.K * self.expert_bytes() + self.shared_bytes()

    def flops_per_token(self) -> int:
        f = 2 * self.E * self.H + self.K * 3 * 2 * self.H * self.I
        if self.shared:
            f += 3 * 2 * self.H * self.shared_I + 2 * self.H
        return f


# The workloads: hidden / experts / top-K / intermediate / bit widths.
CONFIGS = {
    "tiny": LayerConfig("tiny", H=256, I=128, E=8, K=2, expert_bits=4),
    "decode_30b": LayerConfig("decode_30b", H=2048, I=768, E=128, K=8, expert_bits=4),
    "decode_397b": LayerConfig("decode_397b", H=4096, I=1024, E=512, K=4, expert_bits=4,
                               shared=True, shared_I=1024, shared_bits=4),
    # the 397B-like shapes with a 16-expert bank (profiling captures)
    "decode_397b_e16": LayerConfig("decode_397b_e16", H=4096, I=1024, E=16, K=4, expert_bits=4,
                                   shared=True, shared_I=1024, shared_bits=4),
    "prefill_8bit": LayerConfig("prefill_8bit", H=2048, I=768, E=128, K=8, expert_bits=8),
    "mixed_2bit": LayerConfig("mixed_2bit", H=4096, I=1024, E=512, K=4, expert_bits=2,
                              shared=True, shared_I=1024, shared_bits=4, requant_from4=True),
}


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
                                t.n_mats)
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
