"""The five synthetic workloads of the routed-MoE FFN, as data.

Shapes follow a Qwen3.8-Flash-Next-shaped layer (48 layers x 512 experts,
hidden 2048, expert intermediate 768, top-10; "24,576 experts ... about ten"
per token, hexlives "Commitment is a speedup", first paragraph; 48 captured
layer graphs, pyshine Strata tour, "Understanding the Architecture").

Block formats are self-defined (32 weights per block along the reduction
axis, fp16 scale ``d`` and fp16 min ``m``, ``w = d*q + m``):

* Q2: 2-bit codes, d ~ U(0.005, 0.02), m = -1.5 d  -> 12 bytes per block
* Q4: 4-bit codes, d ~ U(0.002, 0.01), m = -7.5 d  -> 20 bytes per block
"""
from __future__ import annotations

from dataclasses import dataclass, replace

Q2, Q4 = 2, 4
BLOCK = 32

# stream tags ("what" word of a stream key)
GATE, UP, DOWN = 0, 1, 2
WHAT_CODES = {GATE: 1, UP: 2, DOWN: 3}
WHAT_SCALES = {GATE: 4, UP: 5, DOWN: 6}
WHAT_ROUTER = 7
WHAT_BIAS = 8
WHAT_X = 9
WHAT_NOISE = 10
WHAT_NGRAM_CODES = 11
WHAT_NGRAM_SCALES = 12
WHAT_NGRAM_IDS = 13


@dataclass(frozen=True)
class Fmt:
    bits: int
    d_lo: float
    d_hi: float
    m_coef: float  # m = -m_coef * d

    @property
    def code_bytes_per_block(self) -> int:
        return BLOCK * self.bits // 8

    @property
    def bytes_per_block(self) -> int:
        return self.code_bytes_per_block + 4


FORMATS = {
    Q2: Fmt(bits=2, d_lo=0.005, d_hi=0.02, m_coef=1.5),
    Q4: Fmt(bits=4, d_lo=0.002, d_hi=0.01, m_coef=7.5),
}


@dataclass(frozen=True)
class Config:
    cid: int
    name: str
    L: int          # layers
    E: int          # experts per layer
    H: int          # hidden size
    I: int          # expert intermediate size
    k: int          # experts per token
    T: int          # tokens per step
    fmt: int        # Q2 or Q4
    x_kind: str     # "normal" | "correlated" | "bf16"
    bias: bool      # per-expert router logit bias ~ N(0, 1)
    residual: bool  # x <- RMSNorm(x + y) between layers
    eps: float = 1e-6
    router_std: float = 0.02
    fmt_layers: tuple = ()   # per-layer block format (mixed-bit stack); empty: every layer is `fmt`

    @property
    def format(self) -> Fmt:
        return FORMATS[self.fmt]

    def expert_bytes(self) -> int:
        """Packed bytes of one expert (gate + up + down)."""
        blocks = 3 * self.H * self.I // BLOCK
        return blocks * self.format.bytes_per_block

    def router_bytes(self) -> int:
        return self.E * self.H * 4

    def for_layer(self, layer: int) -> "Config":
        """This configuration with layer ``layer``'s block format (a mixed-bit
        stack gives its layers different formats; the streams do not depend
        on the format)."""
        if not self.fmt_layers:
            return self
        return replace(self, fmt=self.fmt_layers[layer], fmt_layers=())

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


CONFIGS = {
    0: Config(0, "tiny layer: 64 experts, hidden 256, intermediate 128, top-4, Q2, 1 token",
              L=1, E=64, H=256, I=128, k=4, T=1, fmt=Q2, x_kind="normal",
              bias=False, residual=False),
    1: Config(1, "decode layer: 512 experts, hidden 2048, intermediate 768, top-10, Q2, 1 token",
              L=1, E=512, H=2048, I=768, k=10, T=1, fmt=Q2, x_kind="normal",
              bias=False, residual=False),
    2: Config(2, "48-layer decode stack: 24,576 Q2 experts, top-10, 1 token, residual RMSNorm",
              L=48, E=512, H=2048, I=768, k=10, T=1, fmt=Q2, x_kind="normal",
              bias=False, residual=True),
    3: Config(3, "48-layer verify batch: 8 correlated tokens, Q4 experts, top-10, residual RMSNorm",
              L=48, E=512, H=2048, I=768, k=10, T=8, fmt=Q4, x_kind="correlated",
              bias=False, residual=True),
    4: Config(4, "prefill chunk: 4096 bf16 tokens, 512 Q4 experts, top-10, biased router",
              L=1, E=512, H=2048, I=768, k=10, T=4096, fmt=Q4, x_kind="bf16",
              bias=True, residual=False),
}


def get(cid: int) -> Config:
    return CONFIGS[cid]


@dataclass(frozen=True)
class NgramConfig:
    """An n-gram row table of one layer and a chunk of tokens that read it.

    The pages size the whole table at 51.2 billion elements (about 28.8 GB)
    for 48 layers (pyshine Strata tour, "Understanding the Architecture"),
    about a billion elements a layer; 2^22 rows of 256 give 2^30.  Rows use
    the Q4 block format; ids are uniform over a 2^17-token vocabulary."""
    cid: int = 5
    R: int = 1 << 22
    D: int = 256
    T: int = 4096
    vocab: int = 1 << 17
    fmt: int = Q4

    @property
    def format(self) -> Fmt:
        return FORMATS[self.fmt]

    def row_bytes(self) -> int:
        return self.D // BLOCK * self.format.bytes_per_block

    def with_(self, **kw) -> "NgramConfig":
        return replace(self, **kw)


NGRAM = NgramConfig()


def mixed(cfg: Config, every: int = 4) -> Config:
    """``cfg`` as a mixed-bit stack: layers 0, every, 2 every, ... in Q4, the
    others in Q2. Same configuration id, so its Q2 layers are ``cfg``'s own
    when ``cfg`` is a Q2 stack."""
    return cfg.with_(fmt_layers=tuple(Q4 if l % every == 0 else Q2 for l in range(cfg.L)))
