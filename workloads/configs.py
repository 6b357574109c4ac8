"""Workload shapes of the reconciliation point.

Each workload is a sequence of reconciliation points. A point is one
row-parallel projection (attention out-proj or FFN down-proj) whose N partial
products are summed across the tensor-parallel group and added to the
residual stream ("Interconnects e clusters", section 01 Conceito: two
reconciliation points per layer, one after the out-projection that follows the
sequence mixer and one after the FFN down-projection).

Shapes:
  N  tensor-parallel ranks (the group is emulated inside one GPU's memory)
  M  tokens reconciled per call (1 for single-token decode)
  H  hidden size (the reconciled vector's width)
  K  projection input width; rank r owns the K/N slice r*K/N .. (r+1)*K/N-1

Distributions (all drawn in bf16): x ~ N(0, 1), W ~ N(0, 0.02^2) (standard
deviation 0.02, the usual weight-initialisation convention), residual ~ N(0, 1).
Every point draws its own x, W and residual.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple


@dataclass(frozen=True)
class Point:
    """One reconciliation point: a row-parallel projection of input width k."""

    index: int          # position in the step (0-based); selects the substreams
    kind: str           # "out_proj" or "down_proj"
    k: int              # projection input width K


@dataclass(frozen=True)
class Config:
    name: str
    n_ranks: int
    tokens: int
    hidden: int
    seed: int
    # (kind, K, layers): each layer contributes one point of each listed kind,
    # in the order listed (out-proj first, then down-proj).
    layer_points: Tuple[Tuple[str, int], ...]
    layers: int
    sigma_x: float = 1.0
    sigma_w: float = 0.02
    sigma_res: float = 1.0
    description: str = ""
    points: List[Point] = field(default_factory=list, compare=False)

    def __post_init__(self):
        pts = []
        idx = 0
        for _layer in range(self.layers):
            for kind, k in self.layer_points:
                pts.append(Point(index=idx, kind=kind, k=k))
                idx += 1
        object.__setattr__(self, "points", pts)

    @property
    def n_points(self) -> int:
        return len(self.points)

    def shard(self, k: int) -> int:
        return k // self.n_ranks

    @property
    def chunk(self) -> int:
        return self.hidden // self.n_ranks

    def weight_bytes(self) -> int:
        return sum(p.k * self.hidden * 2 for p in self.points)

    def algorithmic_bytes(self, staged_partials: bool) -> int:
        """Bytes one pass over all points must move through HBM.

        Per point: every shard of W read once (K*H*2), x read (M*K*2), the
        residual read and the output written (2*M*H*2). When the N partials
        are staged through memory between the partial and the ring kernel,
        they are written once and read once (2*N*M*H*2).
        """
        m, h, n = self.tokens, self.hidden, self.n_ranks
        total = 0
        for p in self.points:
            total += p.k * h * 2 + m * p.k * 2 + 2 * m * h * 2
            if staged_partials:
                total += 2 * n * m * h * 2
        return total

    def flops(self) -> int:
        return sum(2 * self.tokens * p.k * self.hidden for p in self.points)


CONFIGS = {
    "tiny": Config(
        name="tiny", n_ranks=2, tokens=1, hidden=256, seed=0,
        layer_points=(("out_proj", 1024), ("down_proj", 1024)), layers=2,
        description="N=2, M=1, H=256, K=1024 (shard 512), 2 layers x 2 points",
    ),
    "decode_n2": Config(
        name="decode_n2", n_ranks=2, tokens=1, hidden=5120, seed=1,
        layer_points=(("out_proj", 5120), ("down_proj", 17408)), layers=64,
        description="single-token decode, H=5120 bf16, N=2, 64 layers x 2 points "
                    "(out-proj K=5120, down-proj K=17408) = 128 reconciliations/token",
    ),
    "decode_n4_m32": Config(
        name="decode_n4_m32", n_ranks=4, tokens=32, hidden=5120, seed=2,
        layer_points=(("out_proj", 5120), ("down_proj", 17408)), layers=64,
        description="decode batch M=32 at N=4, H=5120, 128 reconciliations/token",
    ),
    "decode_n8_m64": Config(
        name="decode_n8_m64", n_ranks=8, tokens=64, hidden=4096, seed=3,
        layer_points=(("out_proj", 4096), ("down_proj", 14336)), layers=48,
        description="decode batch M=64 at N=8, H=4096, 48 layers x 2 points "
                    "(out-proj K=4096, down-proj K=14336)",
    ),
    "prefill_n4": Config(
        name="prefill_n4", n_ranks=4, tokens=4096, hidden=5120, seed=4,
        layer_points=(("down_proj", 17408),), layers=1,
        description="prefill of a 4096-token prompt: N=4, M=4096, H=5120, "
                    "down-proj K=17408 (shard 4352), 1 point",
    ),
}

CONFIG_ORDER = ["tiny", "decode_n2", "decode_n4_m32", "decode_n8_m64", "prefill_n4"]


def get_config(name: str) -> Config:
    try:
        return CONFIGS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {CONFIG_ORDER}") from None
