"""Sliding tile attention oracle (fp64, CPU) -- test infrastructure only.

Source: VORTA paper notes (zhaoyang97 Paper-Notes, NeurIPS 2025, arXiv 2505.18809),
section "方法详解", design 1 (sliding-window attention for local heads): the 3-D
sliding tile attention mask

    M = { m_ij } = { j in (tau(i) - w, tau(i) + w] },   tau(i) = floor(i / t) * t + ceil(t / 2),

tau(i) being the centre of the tile of size t that holds position i, applied on
each of the frame, height and width axes; the page's window is (18, 27, 24) and
its stated purpose is to turn the jagged sliding-window mask into block-dense
tiles.

Readings:

* both sides of the membership test are tile centres: key j is attended by query
  i when, on every axis, tau(j) lies in (tau(i) - w, tau(i) + w] with w = W / 2,
  W the window on that axis.  With W an odd number of tiles, W = (2r + 1) t,
  this keeps exactly the key tiles within r tiles of the query's tile, so every
  (query tile, key tile) block of the mask is all-true or all-false -- the
  block-dense property the page names.  Reading j itself (not its centre) would
  cut tiles at a one-token offset, which contradicts that property;
* one softmax over all attended keys of a query (plain attention restricted to
  the mask), scale 1/sqrt(d);
* the tile is 4 x 4 x 4 tokens (one 64-token block of the library), so the
  window on each axis is an odd multiple of 4; the page's (18, 27, 24) belongs to
  its own tile size and is not reproduced.

Parity status: pinned (tests/test_oracle_sta.py) -- hand-worked tile centres and
key sets on one axis against the formula, the block-dense property, windows of 3
tiles equal to the tile neighbourhood of oracle/tile3d.py, a window covering the
grid equal to dense attention (torch SDPA), and brute-force attention of single
queries.
"""
from __future__ import annotations

import math

import numpy as np

from .sla import row_softmax


def tile_centre(x, t: int):
    """tau(x) = floor(x / t) * t + ceil(t / 2) (elementwise over integer positions)."""
    x = np.asarray(x)
    return (x // t) * t + (t + 1) // 2


def axis_allowed(n: int, t: int, window: int) -> np.ndarray:
    """[n, n] boolean: query position i attends key position j on one axis of length n."""
    tau = tile_centre(np.arange(n), t).astype(np.float64)
    w = window / 2.0
    diff = tau[None, :] - tau[:, None]               # tau(j) - tau(i), rows i, columns j
    return (diff > -w) & (diff <= w)


def sta_mask(F: int, Hh: int, Ww: int, tile=(4, 4, 4), window=(12, 12, 12)) -> np.ndarray:
    """[N, N] boolean mask over raster tokens (f, h, w), N = F * Hh * Ww."""
    mf = axis_allowed(F, tile[0], window[0])
    mh = axis_allowed(Hh, tile[1], window[1])
    mw = axis_allowed(Ww, tile[2], window[2])
    m = mf[:, None, None, :, None, None] & mh[None, :, None, None, :, None] & mw[None, None, :, None, None, :]
    n = F * Hh * Ww
    return m.reshape(n, n)


def sliding_tile_attention(q, k, v, F, Hh, Ww, tile=(4, 4, 4), window=(12, 12, 12), rows=None):
    """Softmax attention of every query over the keys the mask allows.

    q, k, v: one head, [F*Hh*Ww, d] in raster order.  ``rows`` is an optional list
    of raster token indices to compute (others left 0).  Queries of one tile share
    their key set, so they are evaluated together.
    """
    n, d = q.shape
    mf = axis_allowed(F, tile[0], window[0])
    mh = axis_allowed(Hh, tile[1], window[1])
    mw = axis_allowed(Ww, tile[2], window[2])
    f, h, w = (a.reshape(-1) for a in np.meshgrid(np.arange(F), np.arange(Hh), np.arange(Ww), indexing="ij"))
    out = np.zeros((n, v.shape[1]))
    scale = 1.0 / math.sqrt(d)
    rows = range(n) if rows is None else rows
    groups = {}
    for r in rows:
        groups.setdefault((f[r] // tile[0], h[r] // tile[1], w[r] // tile[2]), []).append(r)
    for _, qs in groups.items():
        r0 = qs[0]
        keys = np.nonzero(mf[f[r0]][f] & mh[h[r0]][h] & mw[w[r0]][w])[0]
        qs = np.asarray(qs)
        out[qs] = row_softmax((q[qs] @ k[keys].T) * scale) @ v[keys]
    return out
