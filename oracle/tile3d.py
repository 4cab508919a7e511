"""RoPeSLR-style gated local + far-field oracle (fp64, CPU) -- test infrastructure only.

Source: aixinbiao blog page "RoPeSLR 把视频扩散里的 attention 砍了一半"
(arXiv 2605.20659), section "稀疏邻域加低秩远场，两路并行":

* a sparse neighbourhood branch: each token attends its 3x3x3 spatio-temporal
  neighbourhood;
* a low-rank far-field branch: K and V are compressed to a small set of pooled
  tokens (rank 64) and every token attends to them;
* the two outputs are fused by a gate: g * local + (1 - g) * global
  (g = 0.55 at convergence on that page).

Readings:

* the neighbourhood is taken at tile granularity: tokens are grouped in
  4x4x4 tiles of the (frame, h, w) raster; a query attends every token of the
  tiles within Chebyshev distance ``radius`` (=1, so 3x3x3 tiles, clipped at
  the borders), with one softmax over those keys;
* the far field is one mean pool of K and V over cells of 2x16x16 tokens,
  giving 64 pooled tokens for an 8x64x64 latent; the page's pyramid text is
  garbled (2k + 128 tokens cannot make rank 64), so the single pool is used;
* the far-field branch has its own softmax over the pooled tokens;
* the gate multiplies the two normalised outputs;
* RoPE (the page: the neighbourhood branch "encodes relative position with
  RoPE") is optional here (``rope=True``) and reads as the usual 3-D rotary
  embedding: the d channels of q and k split into three contiguous groups for
  the frame, height and width axes -- with P = d/2 channel pairs, the height
  and width groups take floor(P/3) pairs each and the frame group the rest
  (d = 128: 44, 42, 42 channels) -- and pair i of a group of n pairs (channels
  2i, 2i+1 inside the group) is rotated by the angle pos * base^(-i/n), pos the
  token's coordinate on that axis, base 10000.  As in a video transformer that
  rotates q and k at the start of its attention block, the rotation is applied
  to q and k before both branches: the neighbourhood sees rotated q and k, and
  the far field pools the rotated K (and V as it is).  With ``rope=False`` q and
  k are taken as given (rotated upstream, or not at all).

Parity status: every function is pinned (tests/test_oracle_tile3d.py): g = 1
and g = 0 special cases, a tile grid of at most 2 per dimension (local equals
dense attention), one pooling cell (global equals mean of V); the rotary
embedding by hand-worked rotations, norm preservation, the identity at the
origin and the invariance of rotated dot products under a common shift of
both positions.
"""
from __future__ import annotations

import math

import numpy as np

from .sla import row_softmax


def raster_index(F: int, Hh: int, Ww: int) -> np.ndarray:
    """Token index of every (f, h, w) of the raster: [F, Hh, Ww] -> int."""
    return np.arange(F * Hh * Ww).reshape(F, Hh, Ww)


def tile_of_tokens(F, Hh, Ww, tile):
    """Tile coordinates (tf, th, tw) of every raster token, as three [N] arrays."""
    f, h, w = np.meshgrid(np.arange(F), np.arange(Hh), np.arange(Ww), indexing="ij")
    return (f // tile[0]).reshape(-1), (h // tile[1]).reshape(-1), (w // tile[2]).reshape(-1)


def local_attention(q, k, v, F, Hh, Ww, tile=(4, 4, 4), radius=1, rows=None):
    """Exact softmax of each query over the tokens of its (2r+1)^3 tile neighbourhood.

    q, k, v: one head, [F*Hh*Ww, d] in raster order.  ``rows`` is an optional
    list of raster token indices to compute (others left 0).
    """
    n, d = q.shape
    tf, th, tw = tile_of_tokens(F, Hh, Ww, tile)
    out = np.zeros((n, v.shape[1]))
    scale = 1.0 / math.sqrt(d)
    tiles = np.stack([tf, th, tw], axis=1)
    # group queries by tile: all queries of one tile share a neighbourhood
    keyset = {}
    rows = range(n) if rows is None else rows
    by_tile = {}
    for t in rows:
        by_tile.setdefault(tuple(tiles[t]), []).append(t)
    for tq, qs in by_tile.items():
        if tq not in keyset:
            near = np.all(np.abs(tiles - np.array(tq)[None, :]) <= radius, axis=1)
            keyset[tq] = np.nonzero(near)[0]
        keys = keyset[tq]
        qs = np.asarray(qs)
        s = (q[qs] @ k[keys].T) * scale
        out[qs] = row_softmax(s) @ v[keys]
    return out


def far_field(k, v, F, Hh, Ww, cell=(2, 16, 16)):
    """Mean-pool K and V over cells of cell[0] x cell[1] x cell[2] tokens.

    Returns (kbar, vbar), each [n_cells, d], cells in raster order of the cell grid.
    """
    d = k.shape[1]
    cf, ch, cw = F // cell[0], Hh // cell[1], Ww // cell[2]
    kk = k.reshape(cf, cell[0], ch, cell[1], cw, cell[2], d)
    vv = v.reshape(cf, cell[0], ch, cell[1], cw, cell[2], v.shape[1])
    kbar = kk.mean(axis=(1, 3, 5)).reshape(cf * ch * cw, d)
    vbar = vv.mean(axis=(1, 3, 5)).reshape(cf * ch * cw, v.shape[1])
    return kbar, vbar


def global_attention(q, kbar, vbar, rows=None):
    """softmax(q kbar^T / sqrt(d)) vbar for every query (own softmax)."""
    d = q.shape[1]
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(list(rows))
    out = np.zeros((q.shape[0], vbar.shape[1]))
    s = (q[rows] @ kbar.T) / math.sqrt(d)
    out[rows] = row_softmax(s) @ vbar
    return out


def rope_split(d: int) -> tuple[int, int, int]:
    """Channel pairs of the (frame, height, width) groups of the rotary embedding."""
    pairs = d // 2
    n_hw = pairs // 3
    return pairs - 2 * n_hw, n_hw, n_hw


def rope_3d(x, F, Hh, Ww, base: float = 10000.0):
    """The 3-D rotary embedding of one head's rows x [F*Hh*Ww, d] in raster order.

    Pair i of an axis group with n pairs is rotated by pos * base^(-i/n), pos the
    token's coordinate on that axis: (a, b) -> (a cos - b sin, a sin + b cos).
    """
    n, d = x.shape
    f, h, w = np.meshgrid(np.arange(F), np.arange(Hh), np.arange(Ww), indexing="ij")
    pos = [f.reshape(-1).astype(np.float64), h.reshape(-1).astype(np.float64), w.reshape(-1).astype(np.float64)]
    out = np.array(x, dtype=np.float64, copy=True)
    c0 = 0
    for axis, n_pairs in enumerate(rope_split(d)):
        for i in range(n_pairs):
            ang = pos[axis] * base ** (-i / n_pairs)
            a, b = x[:, c0 + 2 * i], x[:, c0 + 2 * i + 1]
            out[:, c0 + 2 * i] = a * np.cos(ang) - b * np.sin(ang)
            out[:, c0 + 2 * i + 1] = a * np.sin(ang) + b * np.cos(ang)
        c0 += 2 * n_pairs
    return out


def gated_head(q, k, v, F, Hh, Ww, tile=(4, 4, 4), radius=1, cell=(2, 16, 16), gate=0.55, rows=None,
               rope: bool = False):
    """O = g * local + (1 - g) * global for one head (RoPeSLR page); with ``rope`` q and
    k are first rotated by the 3-D rotary embedding."""
    if rope:
        q, k = rope_3d(q, F, Hh, Ww), rope_3d(k, F, Hh, Ww)
    loc = local_attention(q, k, v, F, Hh, Ww, tile, radius, rows)
    kbar, vbar = far_field(k, v, F, Hh, Ww, cell)
    glob = global_attention(q, kbar, vbar, rows)
    return dict(local=loc, glob=glob, kbar=kbar, vbar=vbar, o=gate * loc + (1.0 - gate) * glob)
