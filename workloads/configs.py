"""The five synthetic verify-step shapes (plus the sliding-window variant of the
long-context shape).

Each one fixes the attention shape (batch B, query/KV heads, head_dim D,
prefix length), the draft tree (depth d, top-k k, kept nodes m), the
vocabulary V and logit storage type, the target-noise scale sigma and the
acceptance modes that run on it.

The draft tree terms follow the EAGLE-2 notes ("s1mplewind eagle" page,
EAGLE-2 sections "Expansion of tree" and "Reranking Nodes"): depth = number of
expansion levels, k = children kept per expanded node and frontier width per
level, m = nodes kept by the rerank (the root not counted).
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Config:
    name: str
    B: int            # sequences in the batch
    Hq: int           # query heads
    Hkv: int          # key/value heads (GQA group G = Hq // Hkv)
    D: int            # head_dim
    L: int            # prefix length (for a ragged batch: the upper bound)
    depth: int        # tree depth d
    k: int            # top-k per expanded node and frontier width
    m: int            # tree nodes kept by the rerank (root excluded)
    V: int            # vocabulary
    logits_dtype: str  # "f32" or "bf16": storage of draft and target logits
    sigma: float      # std of the target-minus-draft logit noise
    accept: tuple = ("greedy",)
    L_min: int = 0    # ragged batch: prefix lengths uniform in [L_min, L]
    window: int = 0   # sliding-window width for attention (0 = none)
    seeds: tuple = field(default=(0,))

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def R(self) -> int:
        """Draft rows: the root row plus k rows per expanded level."""
        return 1 + (self.depth - 1) * self.k

    @property
    def P(self) -> int:
        """Candidate pool: k root children plus k*k per deeper level."""
        return self.k + (self.depth - 1) * self.k * self.k

    @property
    def ragged(self) -> bool:
        return self.L_min > 0 and self.L_min != self.L


_SEEDS10 = tuple(range(10))

CONFIGS = {
    "tiny": Config(
        name="tiny", B=1, Hq=4, Hkv=4, D=64, L=128, depth=3, k=2, m=10,
        V=1000, logits_dtype="f32", sigma=1.0, accept=("greedy",), seeds=(0,)),
    "7b": Config(
        name="7b", B=1, Hq=32, Hkv=32, D=128, L=2048, depth=6, k=10, m=60,
        V=32000, logits_dtype="f32", sigma=1.0,
        accept=("greedy", "stochastic"), seeds=_SEEDS10),
    "l3-8b": Config(
        name="l3-8b", B=4, Hq=32, Hkv=8, D=128, L=8192, depth=6, k=8, m=64,
        V=128256, logits_dtype="bf16", sigma=0.5, accept=("stochastic",),
        seeds=_SEEDS10),
    "long": Config(
        name="long", B=1, Hq=32, Hkv=8, D=128, L=32768, depth=8, k=10, m=80,
        V=128256, logits_dtype="bf16", sigma=1.0, accept=("greedy",),
        seeds=_SEEDS10),
    "long-window": Config(
        name="long-window", B=1, Hq=32, Hkv=8, D=128, L=32768, depth=8, k=10,
        m=80, V=128256, logits_dtype="bf16", sigma=1.0, accept=("greedy",),
        window=2048, seeds=_SEEDS10),
    "serve": Config(
        name="serve", B=32, Hq=32, Hkv=8, D=128, L=4096, L_min=512, depth=5,
        k=4, m=32, V=128256, logits_dtype="bf16", sigma=1.0,
        accept=("stochastic",), seeds=_SEEDS10),
}


def get_config(name: str, **overrides) -> Config:
    cfg = CONFIGS[name]
    if overrides:
        d = dict(cfg.__dict__)
        d.update(overrides)
        cfg = Config(**d)
    return cfg
