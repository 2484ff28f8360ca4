"""The five PT-DiT attention workloads (token grid, proxy ratio, TCM window and shift).

The ratio schedule follows the compression ratios of the Qihoo-T2X reading note
(§3 Method, "compression ratios"), one step finer than the page's own schedule so
that the larger grids keep 256 proxies; video uses p_f = 1.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    grid: tuple          # (f, h, w) token grid
    D: int               # model width
    heads: int
    dtype: str           # "f32" | "bf16": storage and MMA input type
    ratio: tuple         # proxy window (p_f, p_h, p_w)
    window: tuple        # TCM window (w_f, w_h, w_w)
    shift: tuple         # SWSA cyclic shift (s_f, s_h, s_w)

    @property
    def N(self) -> int:
        f, h, w = self.grid
        return f * h * w

    @property
    def M(self) -> int:
        pf, ph, pw = self.ratio
        return self.N // (pf * ph * pw)

    @property
    def n(self) -> int:
        wf, wh, ww = self.window
        return wf * wh * ww

    @property
    def d(self) -> int:
        return self.D // self.heads

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_16x16_f32", 1, (1, 16, 16), 64, 2, "f32", (1, 2, 2), (1, 4, 4), (0, 2, 2)),
        Workload("t2i_1024px_64x64_b4", 4, (1, 64, 64), 1152, 16, "bf16", (1, 4, 4), (1, 8, 8), (0, 4, 4)),
        Workload("t2i_2048px_128x128", 1, (1, 128, 128), 1152, 16, "bf16", (1, 8, 8), (1, 8, 8), (0, 4, 4)),
        Workload("t2v_16x32x48", 1, (16, 32, 48), 1152, 16, "bf16", (1, 4, 4), (2, 8, 8), (1, 4, 4)),
        Workload("video_32x64x64", 1, (32, 64, 64), 1152, 16, "bf16", (1, 16, 16), (2, 8, 8), (1, 4, 4)),
        # the pages' own video setting: temporal compression p_f = 4 (§3 Method,
        # compression-ratio paragraph) on the T2V clip and on the long video
        Workload("t2v_pf4_16x32x48", 1, (16, 32, 48), 1152, 16, "bf16", (4, 4, 4), (2, 8, 8), (1, 4, 4)),
        Workload("video_pf4_32x64x64", 1, (32, 64, 64), 1152, 16, "bf16", (4, 8, 8), (2, 8, 8), (1, 4, 4)),
        # text-to-multiview: 24 views of one object treated as the frames of a
        # video (T2MV section), 512 px views -> 32 x 32 tokens, p_f = 4
        Workload("t2mv_24x32x32", 1, (24, 32, 32), 1152, 16, "bf16", (4, 4, 4), (2, 8, 8), (1, 4, 4)),
    ]
}
ORDER = list(WORKLOADS)
# The five workloads of the scope (the others are the pages' video / multiview settings).
CORE = ORDER[:5]
# The headline bench workload: the largest grid, the long high-resolution video
# (32 x 64 x 64 tokens).
HEADLINE = "video_32x64x64"
# Ratio sweep on the long video grid.
RATIO_SWEEP = [(1, 2, 2), (1, 4, 4), (1, 8, 8), (1, 16, 16)]
