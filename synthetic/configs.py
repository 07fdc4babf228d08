"""The five synthetic decode-attention workloads (shapes only; no arithmetic of the method).

Sizes follow the Windowed-MTP pages' setting: million-token context on one GPU, a 4K
sink-plus-recent draft window (4 sink + 4092 recent), GQA attention with head_dim 128, chain
drafts of depth gamma and a small speculation tree.  The pages' workloads are RULER-style tasks
on trained models; attention cost depends only on shapes, so seeded N(0, 1) tensors of these
shapes stand in for them.
"""
from dataclasses import dataclass, field
from typing import Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int                      # committed context per sequence (cfg 4: see contexts)
    Hq: int
    Hkv: int
    D: int = 128
    page_size: int = 64
    n_sink: int = 4
    windows: Tuple[int, ...] = (4092,)   # recent-window sizes W (ring capacity = n_sink + W)
    gammas: Tuple[int, ...] = (3,)
    verify_layers: int = 1
    tree_nodes: int = 0         # 0 = chain verify
    seed: int = 0
    k_scale: float = 1.0        # K multiplied by this before bf16 rounding
    sm_scale: float = 128 ** -0.5
    outlier_p: float = 0.0      # probability a (token, kv head) row of K and V is an outlier
    outlier_factor: float = 8.0
    vocab: int = 1024
    ragged: Tuple[int, int] = field(default=(0, 0))   # (lo, hi) of per-sequence contexts

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def capacity(self, window: int) -> int:
        return self.n_sink + window


TINY = Workload(
    name="tiny-2k", B=1, L=2048, Hq=8, Hkv=2, windows=(252,), gammas=(3,), verify_layers=1,
    seed=0, k_scale=128 ** -0.5, sm_scale=1.0,
)
CTX128K = Workload(
    name="ctx128k", B=1, L=131072, Hq=16, Hkv=2, windows=(4092,), gammas=(3,), verify_layers=8,
    seed=1,
)
CTX1M = Workload(
    name="ctx1m", B=1, L=1 << 20, Hq=32, Hkv=4, windows=(4092,), gammas=(1, 3, 5, 7),
    verify_layers=12, seed=2,
)
BATCH8_TREE = Workload(
    name="batch8-tree", B=8, L=262144, Hq=32, Hkv=4, windows=(4092,), gammas=(7,),
    verify_layers=12, tree_nodes=8, seed=3, ragged=(65536, 262144),
)
NOPE1M = Workload(
    name="nope1m-outlier", B=1, L=1 << 20, Hq=64, Hkv=8, windows=(1020, 2044, 4092, 8188, 16380),
    gammas=(5,), verify_layers=12, seed=4, outlier_p=0.01,
)

ALL = (TINY, CTX128K, CTX1M, BATCH8_TREE, NOPE1M)
BY_NAME = {w.name: w for w in ALL}
