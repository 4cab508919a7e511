"""Seeded synthetic workloads shared by the tests, the bench and the oracle checks.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Every tensor is drawn in fp32 from a seeded
``torch.Generator`` on the CPU and rounded once to bf16, so the GPU library and
the fp64 oracle receive identical bf16 bits.  Pad tokens (the tail of every
segment past ``seg_len``) are zero.

The workloads follow the shapes the source pages talk about:

* ``tiny``    -- 2 heads, d=64, 4 frames of 8x8 tokens (256 tokens), SLA with
                 25 % critical / 25 % negligible.
* ``wan``     -- Wan2.1-1.3B-shaped layer: 12 heads, d=128, 21 frames of 30x52
                 = 32,760 tokens padded to 32,768; frame-correlated inputs;
                 5 % critical / 10 % negligible (SLA page, section 3).
* ``hunyuan`` -- HunyuanVideo-shaped: 24 heads, d=128, 30 frames of 48x80 =
                 115,200 tokens; frame-correlated; 5 % / 10 %.
* ``lvsa``    -- LVSA frame mask: 12 heads, d=128, 121 frames of 30x52 = 1,560
                 tokens, each frame padded to 1,600 (25 blocks of 64); N(0,1);
                 budget C=21, window W=3, denoising steps s=0..3.
* ``ropeslr`` -- RoPeSLR-shaped gated local + far field: 16 heads, d=128,
                 8x64x64 = 32,768 tokens; N(0,1); 4x4x4 tiles, 3x3x3 tile
                 neighbourhood, 2x16x16 pooling cells, gate g=0.55.
* ``sta``     -- VORTA's sliding tile attention on the same 8x64x64 latent,
                 windows of 12x28x20 tokens.
* ``svoo``    -- SVOO's co-clustered block-sparse attention on the wan layer:
                 64 query and 64 key clusters from sampled anchors
                 (``make_anchors``), 2 iterations, 20 % of the key blocks kept.

Frame-correlated recipe (wan, hunyuan): for head h, frame f, position p and
channel c, ``x = sqrt(0.5)*s[h,f,c] + sqrt(0.5)*e[h,f,p,c]`` with s, e ~ N(0,1),
which gives correlation 0.5 between tokens of one frame in one channel.
"""
from __future__ import annotations

import dataclasses
import math

import torch

BLOCK = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int          # 1-based position in the workload list; seeds derive from it
    heads: int
    d: int
    frames: int         # latent frames (segments for padding purposes)
    fh: int             # latent height per frame
    fw: int             # latent width per frame
    seg_stride: int     # padded tokens per segment
    n_seg: int          # number of padded segments
    seg_len: int        # valid tokens per segment
    mode: str           # "sla", "lvsa", "tile3d", "sta" or "svoo"
    correlated: bool
    crit_frac: float = 0.05
    negl_frac: float = 0.10
    # LVSA
    lvsa_C: int = 0
    lvsa_W: int = 0
    lvsa_steps: tuple = ()
    # TILE3D
    tile: tuple = (4, 4, 4)
    radius: int = 1
    cell: tuple = (2, 16, 16)
    gate: float = 0.55
    rope: bool = False  # 3-D rotary embedding of q and k before both branches
    # STA: sliding tile window in tokens per axis (odd multiples of the 4-token tile)
    window: tuple = (12, 12, 12)
    # SVOO: query and key cluster counts, co-clustering iterations, kept fraction of key blocks
    clusters: tuple = (64, 64)
    iters: int = 2
    keep_frac: float = 0.2
    batch: int = 1

    @property
    def n_pad(self) -> int:
        return self.n_seg * self.seg_stride

    @property
    def n_valid(self) -> int:
        return self.n_seg * self.seg_len

    @property
    def n_blocks(self) -> int:
        return self.n_pad // BLOCK

    def seq(self) -> dict:
        return dict(B=self.batch, H=self.heads, d=self.d, block=BLOCK,
                    n_seg=self.n_seg, seg_len=self.seg_len, seg_stride=self.seg_stride)


TINY = Workload("tiny", 1, heads=2, d=64, frames=4, fh=8, fw=8,
                seg_stride=256, n_seg=1, seg_len=256, mode="sla", correlated=False,
                crit_frac=0.25, negl_frac=0.25)
WAN = Workload("wan", 2, heads=12, d=128, frames=21, fh=30, fw=52,
               seg_stride=32768, n_seg=1, seg_len=32760, mode="sla", correlated=True)
HUNYUAN = Workload("hunyuan", 3, heads=24, d=128, frames=30, fh=48, fw=80,
                   seg_stride=115200, n_seg=1, seg_len=115200, mode="sla", correlated=True)
LVSA = Workload("lvsa", 4, heads=12, d=128, frames=121, fh=30, fw=52,
                seg_stride=1600, n_seg=121, seg_len=1560, mode="lvsa", correlated=False,
                lvsa_C=21, lvsa_W=3, lvsa_steps=(0, 1, 2, 3))
ROPESLR = Workload("ropeslr", 5, heads=16, d=128, frames=8, fh=64, fw=64,
                   seg_stride=32768, n_seg=1, seg_len=32768, mode="tile3d", correlated=False, rope=True)

# VORTA's local heads: 3-D sliding tile attention on the same 8x64x64 latent, windows of
# 3 x 7 x 5 tiles (12 x 28 x 20 tokens, ~14 % of the keys); not one of the quoted configurations
STA = Workload("sta", 6, heads=16, d=128, frames=8, fh=64, fw=64,
               seg_stride=32768, n_seg=1, seg_len=32768, mode="sta", correlated=False, window=(12, 28, 20))

# SVOO's co-clustered block-sparse attention on the Wan2.1-1.3B-shaped layer (the model the
# SVOO summary reports first): 64 query and 64 key clusters, 2 iterations, 20 % of the key
# blocks kept per query block (the summary's example of a robust layer that loses 80 % of
# its attention); not one of the quoted configurations
SVOO = Workload("svoo", 7, heads=12, d=128, frames=21, fh=30, fw=52,
                seg_stride=32768, n_seg=1, seg_len=32760, mode="svoo", correlated=True,
                clusters=(64, 64), iters=2, keep_frac=0.2)

ALL = (TINY, WAN, HUNYUAN, LVSA, ROPESLR, STA, SVOO)
BY_NAME = {w.name: w for w in ALL}


def _valid_rows(n_seg: int, seg_len: int, seg_stride: int) -> torch.Tensor:
    t = torch.arange(n_seg * seg_stride)
    return (t % seg_stride) < seg_len


def _frame_correlated(gen: torch.Generator, heads: int, frames: int, per_frame: int, d: int) -> torch.Tensor:
    s = torch.randn(heads, frames, 1, d, generator=gen, dtype=torch.float32)
    e = torch.randn(heads, frames, per_frame, d, generator=gen, dtype=torch.float32)
    r = math.sqrt(0.5)
    return (r * s + r * e).reshape(heads, frames * per_frame, d)


def make_tensor(w: Workload, which: str, heads: int | None = None) -> torch.Tensor:
    """One of q, k, v as a bf16 CPU tensor [B, H, N_pad, d] with zero pads.

    ``heads`` limits the draw to the first heads (the draw for head h does not
    depend on how many heads are drawn when the workload is not correlated;
    correlated draws are made per head for the same reason).
    """
    seed = {"q": 1000, "k": 2000, "v": 3000}[which] + w.index
    H = w.heads if heads is None else heads
    out = torch.zeros(w.batch, H, w.n_pad, w.d, dtype=torch.bfloat16)
    valid = _valid_rows(w.n_seg, w.seg_len, w.seg_stride)
    for b in range(w.batch):
        for h in range(H):
            gen = torch.Generator().manual_seed(seed * 1_000_003 + b * 1009 + h)
            if w.correlated:
                x = _frame_correlated(gen, 1, w.frames, w.fh * w.fw, w.d)[0]
            else:
                x = torch.randn(w.n_valid, w.d, generator=gen, dtype=torch.float32)
            out[b, h, valid] = x.to(torch.bfloat16)
    return out


def make_w_proj(w: Workload) -> torch.Tensor:
    """W_proj [d, d] bf16 with entries ~ N(0, 1/d)."""
    gen = torch.Generator().manual_seed(4000 + w.index)
    x = torch.randn(w.d, w.d, generator=gen, dtype=torch.float32) / math.sqrt(w.d)
    return x.to(torch.bfloat16)


def make_qkv(w: Workload, heads: int | None = None):
    return make_tensor(w, "q", heads), make_tensor(w, "k", heads), make_tensor(w, "v", heads)


def small_variant(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (used for reduced-size parity cases)."""
    return dataclasses.replace(w, **changes)


def random_bf16(shape, seed: int, scale: float = 1.0) -> torch.Tensor:
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=gen, dtype=torch.float32) * scale).to(torch.bfloat16)


def make_anchors(w: Workload, which: str, heads: int | None = None) -> torch.Tensor:
    """SVOO anchor tokens: int32 [B, H, C], C distinct valid tokens per (b, h) drawn
    uniformly without replacement (C = clusters[0] for "q", clusters[1] for "k")."""
    C = w.clusters[0] if which == "q" else w.clusters[1]
    seed = {"q": 5000, "k": 6000}[which] + w.index
    H = w.heads if heads is None else heads
    valid = torch.nonzero(_valid_rows(w.n_seg, w.seg_len, w.seg_stride)).reshape(-1)
    out = torch.zeros(w.batch, H, C, dtype=torch.int32)
    for b in range(w.batch):
        for h in range(H):
            gen = torch.Generator().manual_seed(seed * 1_000_003 + b * 1009 + h)
            out[b, h] = valid[torch.randperm(valid.numel(), generator=gen)[:C]].to(torch.int32)
    return out


def make_mixture(n: int, d: int, n_comp: int, seed: int, spread: float = 0.05):
    """Well-separated Gaussian mixture: (x bf16 [n, d], component [n] int64, anchors [n_comp]).

    Component means ~ N(0, 1)^d, each token = its component's mean + spread * N(0, 1)^d.
    Every component holds at least one token; anchors[m] is the first token of component m.
    """
    gen = torch.Generator().manual_seed(seed)
    mu = torch.randn(n_comp, d, generator=gen, dtype=torch.float32)
    comp = torch.randint(n_comp, (n,), generator=gen)
    comp[torch.randperm(n, generator=gen)[:n_comp]] = torch.arange(n_comp)
    x = mu[comp] + spread * torch.randn(n, d, generator=gen, dtype=torch.float32)
    anchors = torch.tensor([int(torch.nonzero(comp == m)[0]) for m in range(n_comp)], dtype=torch.int64)
    return x.to(torch.bfloat16), comp, anchors
