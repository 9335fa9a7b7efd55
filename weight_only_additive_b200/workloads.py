"""Named AQLM layer workloads: layer shapes, codebook schemes and batch sizes.

Scheme names follow the AQLM convention ``MxB gG``: M codebooks of 2^B entries,
codewords of g weights (so M*B/g bits per weight before codebook overhead).
The shapes are the linear layers of the model families the AQLM pages say the
format targets (Llama 2, Mixtral), at the sizes of their public architectures.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple


@dataclass(frozen=True)
class Scheme:
    M: int
    B: int
    g: int

    @property
    def name(self) -> str:
        return f"{self.M}x{self.B}g{self.g}"

    @property
    def bits_per_weight(self) -> float:
        return self.M * self.B / self.g

    @property
    def code_bytes(self) -> int:
        return 1 if self.B <= 8 else 2


S1x16g8 = Scheme(1, 16, 8)
S2x8g8 = Scheme(2, 8, 8)
S1x16g16 = Scheme(1, 16, 16)
SCHEMES = {s.name: s for s in (S1x16g8, S2x8g8, S1x16g16)}


@dataclass(frozen=True)
class Layer:
    name: str
    N: int          # output features (rows of W)
    K: int          # input features
    scheme: Scheme

    @property
    def G(self) -> int:
        return self.K // self.scheme.g

    def algorithmic_bytes(self, batch: int) -> int:
        """Bytes a perfect kernel moves: codes + codebooks + scales + x + y."""
        s = self.scheme
        codes = self.N * self.G * s.M * s.code_bytes
        codebooks = s.M * (1 << s.B) * s.g * 2
        return codes + codebooks + 2 * self.N + 2 * batch * self.K + 2 * batch * self.N

    def flops(self, batch: int) -> int:
        return 2 * batch * self.N * self.K


@dataclass(frozen=True)
class Workload:
    index: int                 # 1-based position in the published config list
    name: str
    layers: Tuple[Layer, ...]
    batches: Tuple[int, ...]
    description: str = ""
    extra: dict = field(default_factory=dict, compare=False, hash=False)


def _llama2_7b(s: Scheme) -> Tuple[Layer, ...]:
    return (Layer("q_proj", 4096, 4096, s), Layer("k_proj", 4096, 4096, s),
            Layer("v_proj", 4096, 4096, s), Layer("o_proj", 4096, 4096, s),
            Layer("gate_proj", 11008, 4096, s), Layer("up_proj", 11008, 4096, s),
            Layer("down_proj", 4096, 11008, s))


def _llama2_70b_shapes(s: Scheme) -> Tuple[Layer, ...]:
    return (Layer("q_proj", 8192, 8192, s), Layer("k_proj", 1024, 8192, s),
            Layer("gate_proj", 28672, 8192, s), Layer("down_proj", 8192, 28672, s))


def _mixtral_experts(s: Scheme) -> Tuple[Layer, ...]:
    out: List[Layer] = []
    for e in range(8):
        out += [Layer(f"expert{e}.w1", 14336, 4096, s), Layer(f"expert{e}.w3", 14336, 4096, s),
                Layer(f"expert{e}.w2", 4096, 14336, s)]
    return tuple(out)


def _sweep_layers() -> Tuple[Layer, ...]:
    out: List[Layer] = []
    for s in (S1x16g8, S2x8g8):
        out += [Layer(f"up_11008x4096.{s.name}", 11008, 4096, s),
                Layer(f"down_4096x11008.{s.name}", 4096, 11008, s)]
    return tuple(out)


WORKLOADS = (
    Workload(1, "single_4096x4096_1x16g8", (Layer("linear", 4096, 4096, S1x16g8),), (1,),
             "one 4096x4096 AQLM linear, 1x16 g8 (2 bit), batch 1"),
    Workload(2, "llama2_7b_layer_set_2x8g8", _llama2_7b(S2x8g8), (1,),
             "Llama-2-7B decoder linears q/k/v/o/gate/up/down, 2x8 g8 (2 bit), batch 1"),
    Workload(3, "llama2_70b_layers_1x16g8", _llama2_70b_shapes(S1x16g8), (1, 4),
             "Llama-2-70B linear shapes 8192x8192, 1024x8192, 28672x8192, 8192x28672, 1x16 g8"),
    Workload(4, "batch_sweep_11008x4096", _sweep_layers(), (1, 4, 16, 64, 256),
             "batch sweep on 11008x4096 and 4096x11008, 1x16 g8 and 2x8 g8"),
    Workload(5, "mixtral_8x7b_experts_1x16g16", _mixtral_experts(S1x16g16), (1,),
             "Mixtral-8x7B expert FFNs, 8 experts x w1/w3/w2, 1x16 g16 (1 bit), batch 1"),
    Workload(5, "mixtral_8x7b_experts_2x8g8", _mixtral_experts(S2x8g8), (1,),
             "Mixtral-8x7B expert FFNs, 8 experts x w1/w3/w2, 2x8 g8 (2 bit), batch 1"),
)

BY_NAME = {w.name: w for w in WORKLOADS}


def get(name: str) -> Workload:
    return BY_NAME[name]
