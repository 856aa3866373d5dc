"""Layer shapes: the dimensions and bit widths of one MoE FFN layer, and the
named shapes of the pages' model families.  Plain data and arithmetic only:
importing this module loads no library.
"""
from __future__ import annotations

from dataclasses import dataclass


def packed_bytes(out_dim: int, in_dim: int, bits: int, group_size: int) -> int:
    """Bytes of one packed matrix: codes plus one bf16 scale and one bf16
    bias per group."""
    return out_dim * in_dim * bits // 8 + 2 * 2 * out_dim * (in_dim // group_size)


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
        return 3 * packed_bytes(self.I, self.H, self.expert_bits, self.G)

    def router_bytes(self) -> int:
        return packed_bytes(self.E, self.H, self.router_bits, self.G)

    def shared_bytes(self) -> int:
        if not self.shared:
            return 0
        return (3 * packed_bytes(self.shared_I, self.H, self.shared_bits, self.G)
                + packed_bytes(1, self.H, self.shared_gate_bits, self.G))

    def decode_bytes_per_token(self) -> int:
        """Weight bytes one token needs (router + K experts + shared expert)."""
        return self.router_bytes() + self.K * self.expert_bytes() + self.shared_bytes()

    def flops_per_token(self) -> int:
        f = 2 * self.E * self.H + self.K * 3 * 2 * self.H * self.I
        if self.shared:
            f += 3 * 2 * self.H * self.shared_I + 2 * self.H
        return f


# Named shapes (hidden / intermediate / experts / top-K / bit widths): a tiny
# test layer, the 30B-A3B-like and 397B-A17B-like decode layers, the 8-bit
# prefill layer and the mixed bank of 2-bit experts with a 4-bit shared expert.
CONFIGS = {
    "tiny": LayerConfig("tiny", H=256, I=128, E=8, K=2, expert_bits=4),
    "decode_30b": LayerConfig("decode_30b", H=2048, I=768, E=128, K=8, expert_bits=4),
    "decode_397b": LayerConfig("decode_397b", H=4096, I=1024, E=512, K=4, expert_bits=4,
                               shared=True, shared_I=1024, shared_bits=4),
    "prefill_8bit": LayerConfig("prefill_8bit", H=2048, I=768, E=128, K=8, expert_bits=8),
    "mixed_2bit": LayerConfig("mixed_2bit", H=4096, I=1024, E=512, K=4, expert_bits=2,
                              shared=True, shared_I=1024, shared_bits=4, requant_from4=True),
}
