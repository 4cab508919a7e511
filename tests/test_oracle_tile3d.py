"""Pins for the RoPeSLR-style gated oracle: gate special cases, a tile grid small
enough that the neighbourhood is everything (local == dense, checked against
torch SDPA), far-field pooling against torch avg_pool3d, one pooling cell
(global == mean of V)."""
import math

import numpy as np
import torch

from oracle import tile3d


def _qkv(seed, n, d):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((n, d)) for _ in range(3))


def _sdpa(q, k, v):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None], torch.tensor(k)[None, None], torch.tensor(v)[None, None])[0, 0].numpy()


def test_small_grid_local_is_dense():
    F, Hh, Ww, d = 8, 8, 8, 8          # 2x2x2 tiles: every tile neighbours every tile
    q, k, v = _qkv(1, F * Hh * Ww, d)
    loc = tile3d.local_attention(q, k, v, F, Hh, Ww)
    np.testing.assert_allclose(loc, _sdpa(q, k, v), rtol=0, atol=1e-12)


def test_far_field_matches_avg_pool3d():
    F, Hh, Ww, d = 4, 32, 32, 4
    _, k, v = _qkv(2, F * Hh * Ww, d)
    kbar, vbar = tile3d.far_field(k, v, F, Hh, Ww, (2, 16, 16))
    for x, xbar in ((k, kbar), (v, vbar)):
        t = torch.tensor(x).reshape(F, Hh, Ww, d).permute(3, 0, 1, 2)[None]
        ref = torch.nn.functional.avg_pool3d(t, (2, 16, 16))[0]          # [d, 2, 2, 2]
        ref = ref.permute(1, 2, 3, 0).reshape(-1, d).numpy()
        np.testing.assert_allclose(xbar, ref, rtol=1e-13, atol=1e-14)


def test_gate_special_cases():
    F, Hh, Ww, d = 8, 16, 16, 8
    q, k, v = _qkv(3, F * Hh * Ww, d)
    r1 = tile3d.gated_head(q, k, v, F, Hh, Ww, gate=1.0, cell=(2, 8, 8))
    np.testing.assert_array_equal(r1["o"], r1["local"])
    r0 = tile3d.gated_head(q, k, v, F, Hh, Ww, gate=0.0, cell=(2, 8, 8))
    np.testing.assert_array_equal(r0["o"], r0["glob"])
    # g = 0: textbook attention of every query over the pooled tokens
    np.testing.assert_allclose(r0["glob"], _sdpa(q, r0["kbar"], r0["vbar"]), rtol=0, atol=1e-12)


def test_single_cell_global_is_mean_of_values():
    F, Hh, Ww, d = 4, 8, 8, 4
    q, k, v = _qkv(4, F * Hh * Ww, d)
    r = tile3d.gated_head(q, k, v, F, Hh, Ww, cell=(4, 8, 8), gate=0.0)
    np.testing.assert_allclose(r["o"], np.tile(v.mean(axis=0), (q.shape[0], 1)), rtol=1e-13, atol=1e-14)


def test_local_neighbourhood_brute_force():
    F, Hh, Ww, d = 8, 12, 16, 4
    q, k, v = _qkv(5, F * Hh * Ww, d)
    loc = tile3d.local_attention(q, k, v, F, Hh, Ww)
    idx = np.arange(F * Hh * Ww).reshape(F, Hh, Ww)
    for (f, h, w) in [(0, 0, 0), (7, 11, 15), (3, 5, 9), (4, 4, 4), (0, 11, 3)]:
        tf, th, tw = f // 4, h // 4, w // 4
        keys = [int(idx[a, b, c]) for a in range(F) for b in range(Hh) for c in range(Ww)
                if abs(a // 4 - tf) <= 1 and abs(b // 4 - th) <= 1 and abs(c // 4 - tw) <= 1]
        t = int(idx[f, h, w])
        lg = np.array([q[t] @ k[u] for u in keys]) / math.sqrt(d)
        p = np.exp(lg - lg.max())
        p /= p.sum()
        np.testing.assert_allclose(loc[t], p @ v[keys], rtol=1e-12, atol=1e-13)
