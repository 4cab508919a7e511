"""LVSA oracle (fp64 / integer, CPU) -- test infrastructure only.

Source: rainbus paper-digest page "LVSA：面向长视频扩散模型的无训练稀疏注意力"
(arXiv 2605.31057), sections "核心方法" and "方法步骤详情":

* the budget C and window half-width W fix the global period
  T_per = ceil(T / (C - (2W + 1)));
* at denoising step s the global set is G_s = {(s mod T_per + i T_per) mod T},
  of constant size ceil(T / T_per), so each frame is global at least once in
  any T_per consecutive steps;
* the local window of query frame t starts at w_lo = max(0, min(t - W, T-1-2W))
  and spans 2W + 1 frames;
* the window is expanded, toward the side with more room, until it holds
  min(2W + 1, T - |G|) frames that are not global, so every frame attends
  |G| + min(2W + 1, T - |G|) unique frames;
* A(t) = G_s u W(t), and every query token of frame t attends, with one exact
  softmax, every key token of the frames in A(t) (step 6 formula).

Readings where the page is silent:

* "the side with the most room": room_lo = w_lo frames to the left, room_hi =
  T - 1 - w_hi to the right; grow w_hi when room_hi >= room_lo (a tie grows the
  right side), otherwise grow w_lo.  The page's "at most 8 iterations" is an
  observation, not a rule.
* when T < 2W + 1 the window is clipped to [0, T - 1].
* pad tokens of a frame (past its valid length) are excluded from the softmax;
  pad queries give 0.

Parity status: every function is pinned (tests/test_oracle_lvsa.py) by the
page's printed constants, its stated invariants and hand-worked small cases.
"""
from __future__ import annotations

import math

import numpy as np

from .sla import block_sparse_attention, valid_tokens


def global_period(T: int, C: int, W: int) -> int:
    """T_per = ceil(T / (C - (2W + 1))); requires C > 2W + 1."""
    if C <= 2 * W + 1:
        raise ValueError("budget C must exceed the window 2W+1")
    return -(-T // (C - (2 * W + 1)))


def global_set(T: int, T_per: int, s: int) -> list[int]:
    """G_s = {(s mod T_per + i*T_per) mod T : i = 0 .. ceil(T/T_per) - 1}, sorted."""
    n = -(-T // T_per)
    return sorted({(s % T_per + i * T_per) % T for i in range(n)})


def adaptive_window(T: int, W: int, t: int) -> tuple[int, int]:
    """[w_lo, w_hi] with w_lo = max(0, min(t - W, T - 1 - 2W)), w_hi = w_lo + 2W (clipped)."""
    lo = max(0, min(t - W, T - 1 - 2 * W))
    hi = min(T - 1, lo + 2 * W)
    return lo, hi


def expanded_window(T: int, W: int, t: int, G: list[int]) -> tuple[int, int, int]:
    """Grow the window until it holds min(2W+1, T-|G|) non-global frames.

    Returns (w_lo, w_hi, iterations).
    """
    gset = set(G)
    lo, hi = adaptive_window(T, W, t)
    target = min(2 * W + 1, T - len(gset))

    def non_global(a, b):
        return sum(1 for f in range(a, b + 1) if f not in gset)

    it = 0
    while non_global(lo, hi) < target:
        room_lo, room_hi = lo, T - 1 - hi
        if room_hi >= room_lo and room_hi > 0:
            hi += 1
        elif room_lo > 0:
            lo -= 1
        else:  # cannot happen: target <= number of non-global frames
            raise AssertionError("window cannot grow")
        it += 1
    return lo, hi, it


def attention_sets(T: int, C: int, W: int, s: int) -> list[list[int]]:
    """A(t) = G_s u W(t) for every query frame t, each sorted ascending."""
    T_per = global_period(T, C, W)
    G = global_set(T, T_per, s)
    out = []
    for t in range(T):
        lo, hi, _ = expanded_window(T, W, t, G)
        out.append(sorted(set(G) | set(range(lo, hi + 1))))
    return out


def frame_mask_attention(q, k, v, n_seg, seg_len, seg_stride, sets, rows=None, block: int = 64):
    """Exact softmax of each query token of frame t over the valid keys of frames A(t).

    q, k, v are one head [N_pad, d]; frames are segments of ``seg_stride`` tokens.
    ``rows`` restricts the work to some query blocks.
    """
    valid = valid_tokens(n_seg, seg_len, seg_stride)
    bpf = seg_stride // block
    nb = q.shape[0] // block
    key_blocks = []
    for i in range(nb):
        t = i // bpf
        key_blocks.append([f * bpf + b for f in sets[t] for b in range(bpf)])
    return block_sparse_attention(q, k, v, valid, key_blocks, rows, block)
