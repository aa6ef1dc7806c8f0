"""The five latent-point workloads: shapes, budgets and generator settings.

Sizes follow the view counts the pages scale over (from about a hundred to
1,024 views of a VGGT-style backbone, "Zebra3D" abstract and "AVGGT" results):
S frames of N = 1 camera + 4 register + 37x37 patch tokens, 16 heads of
d = 64.  Sparsity percentages become per-query-tile budgets as follows:
  * "keep 20 % of key tiles plus own frame": k = round(0.20 * nt);
  * "x % tile sparsity": kept = round((1 - x) * nt) including the own frame's
    tiles, so k = kept - tiles_per_frame.
"""
from __future__ import annotations

import dataclasses
import math


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    frames: int          # S
    tokens: int          # N per frame
    heads: int           # H (batch folded in)
    head_dim: int        # d
    tile: int            # T
    n_sink: int          # camera + register tokens per frame
    dtype: str           # "f32" or "bf16"
    k: int               # extra key tiles per query tile beyond the own frame's
    landmark: bool       # fold unselected tiles into mean-K/mean-V tokens
    streamed: bool       # select without materialising the score matrix
    n_points: int        # P shared 3-D points
    window: int          # visibility window in frames (0 = all frames)
    p_assign: float      # probability that a non-sink token is tied to a point
    seed: int = 0

    @property
    def L(self) -> int:
        return self.frames * self.tokens

    @property
    def tpf(self) -> int:
        return -(-self.tokens // self.tile)

    @property
    def nt(self) -> int:
        return self.frames * self.tpf

    @property
    def max_kept(self) -> int:
        return self.tpf + min(self.k, self.nt - self.tpf)

    @property
    def sparsity(self) -> float:
        return 1.0 - self.max_kept / self.nt

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _k_from_sparsity(frames: int, tokens: int, tile: int, sparsity: float) -> int:
    tpf = -(-tokens // tile)
    nt = frames * tpf
    kept = int(round((1.0 - sparsity) * nt))
    return kept - tpf


TINY = Workload("tiny_s4_n256", 4, 256, 2, 64, 64, 0, "f32", 4, False, False, 128, 0, 1.0)
VGGT_S16 = Workload("vggt_s16_n1374", 16, 1374, 16, 64, 128, 5, "bf16",
                    int(round(0.20 * 16 * 11)), False, False, 4096, 0, 0.7)
VGGT_S128 = Workload("vggt_s128_n1374", 128, 1374, 16, 64, 128, 5, "bf16",
                     _k_from_sparsity(128, 1374, 128, 0.90), False, False, 32768, 16, 0.7)
VGGT_S512 = Workload("vggt_s512_n1374_landmark", 512, 1374, 16, 64, 128, 5, "bf16",
                     _k_from_sparsity(512, 1374, 128, 0.94), True, False, 131072, 16, 0.7)
VGGT_S1024 = Workload("vggt_s1024_n1374_streamed", 1024, 1374, 16, 64, 128, 5, "bf16",
                      _k_from_sparsity(1024, 1374, 128, 0.97), False, True, 262144, 32, 0.7)

ALL = [TINY, VGGT_S16, VGGT_S128, VGGT_S512, VGGT_S1024]
BY_NAME = {w.name: w for w in ALL}

# generator constants of the recipe
A_LAT = 0.8
A_NOISE = 0.6
SINK_K_SCALE = 4.0


def softmax_scale(w: Workload) -> float:
    return 1.0 / math.sqrt(w.head_dim)
