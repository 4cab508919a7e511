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


# ---------------------------------------------------------------- rotary embedding

def test_rope_split_of_the_head_sizes():
    assert tile3d.rope_split(128) == (22, 21, 21)       # 44 + 42 + 42 channels
    assert tile3d.rope_split(64) == (12, 10, 10)


def test_rope_hand_rotations():
    # d = 12: 6 pairs -> frame 2, height 2, width 2 pairs; pair 0 of a group has angle = pos
    F, Hh, Ww, d = 2, 3, 4, 12
    x = np.zeros((F * Hh * Ww, d))
    t = (1 * Hh + 2) * Ww + 3                      # token (f, h, w) = (1, 2, 3)
    x[t, 0] = 1.0                                 # frame pair 0 (channels 0, 1): (1, 0)
    x[t, 2] = 1.0                                 # frame pair 1 (channels 2, 3): (1, 0), angle 10000^(-1/2)
    x[t, 4] = 2.0                                 # height pair 0 (channels 4, 5): (2, 1)
    x[t, 5] = 1.0
    x[t, 9] = -1.0                                # width pair 0 (channels 8, 9): (0, -1)
    r = tile3d.rope_3d(x, F, Hh, Ww)
    # frame pair 0 rotated by 1
    assert np.allclose(r[t, 0:2], [math.cos(1.0), math.sin(1.0)], atol=1e-15)
    # frame pair 1: f = 1 times 10000^(-1/2) = 0.01
    assert np.allclose(r[t, 2:4], [math.cos(0.01), math.sin(0.01)], atol=1e-15)
    # height pair 0 = (2, 1), angle 2
    a, b = 2.0, 1.0
    assert np.allclose(r[t, 4:6], [a * math.cos(2) - b * math.sin(2), a * math.sin(2) + b * math.cos(2)], atol=1e-14)
    # width pair 0 = channels 8, 9 = (0, -1), angle 3
    assert np.allclose(r[t, 8:10], [math.sin(3.0), -math.cos(3.0)], atol=1e-14)


def test_rope_identity_at_origin_and_norm_preserved():
    q, _, _ = _qkv(11, 2 * 8 * 8, 64)
    r = tile3d.rope_3d(q, 2, 8, 8)
    assert np.allclose(r[0], q[0], atol=0)        # token (0, 0, 0) is not rotated
    pair_norm = lambda x: x[:, 0::2] ** 2 + x[:, 1::2] ** 2  # noqa: E731
    assert np.allclose(pair_norm(r), pair_norm(q), rtol=1e-12, atol=1e-12)


def test_rope_dot_products_depend_on_relative_position_only():
    # the same q at (1, 2, 3) and k at (0, 5, 1), and both shifted by (2, 1, 4): equal dot products
    F, Hh, Ww, d = 4, 8, 8, 128
    rng = np.random.default_rng(12)
    qv, kv = rng.standard_normal(d), rng.standard_normal(d)
    tok = lambda f, h, w: (f * Hh + h) * Ww + w  # noqa: E731
    x = np.zeros((F * Hh * Ww, d))
    y = np.zeros((F * Hh * Ww, d))
    x[tok(1, 2, 3)] = qv
    x[tok(3, 3, 7)] = qv
    y[tok(0, 5, 1)] = kv
    y[tok(2, 6, 5)] = kv
    rq, rk = tile3d.rope_3d(x, F, Hh, Ww), tile3d.rope_3d(y, F, Hh, Ww)
    a = rq[tok(1, 2, 3)] @ rk[tok(0, 5, 1)]
    b = rq[tok(3, 3, 7)] @ rk[tok(2, 6, 5)]
    assert abs(a - b) < 1e-10 * (1 + abs(a))
    assert abs(a - qv @ kv) > 1e-3                 # and the rotation did change it


def test_gated_head_with_rope_equals_rotating_q_and_k_first():
    F, Hh, Ww, d = 4, 8, 8, 32
    q, k, v = _qkv(13, F * Hh * Ww, d)
    r = tile3d.gated_head(q, k, v, F, Hh, Ww, cell=(2, 4, 4), gate=0.55, rope=True)
    qr, kr = tile3d.rope_3d(q, F, Hh, Ww), tile3d.rope_3d(k, F, Hh, Ww)
    ref = tile3d.gated_head(qr, kr, v, F, Hh, Ww, cell=(2, 4, 4), gate=0.55)
    assert np.allclose(r["o"], ref["o"], rtol=1e-12, atol=1e-12)
    # the far field pools the rotated keys
    kb, _ = tile3d.far_field(kr, v, F, Hh, Ww, (2, 4, 4))
    assert np.allclose(r["kbar"], kb)
