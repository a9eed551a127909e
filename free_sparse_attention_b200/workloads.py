"""Workload shapes for the SCOPE per-layer hot path.

Each workload is one attention layer of a video diffusion transformer: post-RoPE
Q, K, V of a T x Hg x Wg token grid per head, with the head dimension split into the
temporal / height / width channel ranges of 3D RoPE.  The shapes follow the model
families the SCOPE paper evaluates (Wan2.1/2.2 and HunyuanVideo at 720p, abstract and
"Implementation details"); the hyperparameters Cq=300, Cm=333 per subspace and the
fixed Top-k fraction alpha=0.1 are the ones the paper's implementation details give.
The Top-p threshold rho is not reported by the paper; 0.9 is this library's default.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    Hg: int
    Wg: int
    d_t: int
    d_h: int
    d_w: int
    dtype: str          # "f32" or "bf16"
    Cq: int
    Cm: int
    seed: int
    rho: float = 0.9
    alpha: float = 0.1
    iters: int = 5
    rho_sweep: tuple = field(default=())

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def d(self) -> int:
        return self.d_t + self.d_h + self.d_w

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny", 1, 1, 4, 8, 8, 16, 24, 24, "f32", 8, 8, seed=0)
COGVIDEOX = Workload("cogvideox", 1, 48, 13, 30, 45, 16, 24, 24, "bf16", 100, 100, seed=1)
WAN480 = Workload("wan480p", 1, 40, 21, 30, 52, 44, 42, 42, "bf16", 300, 333, seed=2)
HUNYUAN720 = Workload("hunyuan720p", 1, 24, 33, 45, 80, 16, 56, 56, "bf16", 300, 333, seed=3)
WAN720 = Workload("wan720p", 1, 40, 21, 45, 80, 44, 42, 42, "bf16", 300, 333, seed=4,
                  rho_sweep=(0.5, 0.7, 0.9, 0.95, 0.99))

ALL = {w.name: w for w in (TINY, COGVIDEOX, WAN480, HUNYUAN720, WAN720)}
