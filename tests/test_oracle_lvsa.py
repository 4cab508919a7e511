"""Pins for the LVSA oracle: the page's printed constants, its stated invariants,
hand-worked attention sets, and the dense special case (T_per = 1)."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import lvsa, sla


def _constants(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "lvsa_constants.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            rows.append((parts[0], [int(x) for x in parts[1:]]))
    return rows


def test_printed_constants(golden_dir):
    for kind, vals in _constants(golden_dir):
        if kind == "wan_budget":
            frames, temporal_stride, budget, T, W = vals
            assert (frames - 1) // temporal_stride + 1 == budget
            for s in range(4):
                assert {len(A) for A in lvsa.attention_sets(T, budget, W, s)} == {budget}
        elif kind == "period":
            T, C, W, tper = vals
            assert lvsa.global_period(T, C, W) == tper
        elif kind == "global_size":
            T, tper, size = vals
            for s in range(3 * tper):
                assert len(lvsa.global_set(T, tper, s)) == size
        elif kind == "set_size":
            T, C, W, size = vals
            for s in range(4):
                for A in lvsa.attention_sets(T, C, W, s):
                    assert len(A) == size
        elif kind == "global_set":
            T, tper, s, *members = vals
            assert lvsa.global_set(T, tper, s) == members
        else:
            raise AssertionError(kind)


def _hand_sets(golden_dir):
    cases, cur = [], None
    with open(os.path.join(golden_dir, "lvsa_sets.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            if line.startswith("case"):
                cur = (tuple(int(x) for x in line.split()[1:]), [])
                cases.append(cur)
            else:
                t, frames = line.split(":")
                cur[1].append([int(x) for x in frames.split()])
    return cases


def test_hand_worked_sets(golden_dir):
    for (T, C, W, s), expect in _hand_sets(golden_dir):
        assert lvsa.attention_sets(T, C, W, s) == expect, (T, C, W, s)


@pytest.mark.parametrize("T,C,W", [(121, 21, 3), (100, 21, 3), (81, 21, 3), (37, 9, 2),
                                   (10, 6, 1), (5, 6, 1), (200, 30, 4), (13, 8, 3)])
def test_invariants(T, C, W):
    tper = lvsa.global_period(T, C, W)
    nG = math.ceil(T / tper)
    for s in range(2 * tper + 1):
        G = lvsa.global_set(T, tper, s)
        assert len(G) == nG                                   # constant size
        sets = lvsa.attention_sets(T, C, W, s)
        for t, A in enumerate(sets):
            assert t in A                                     # own frame
            assert set(G) <= set(A)
            assert len(A) == nG + min(2 * W + 1, T - nG)      # unique-frame count
            assert len(A) == len(set(A))
            nonglob = sorted(set(A) - set(G))
            lo, hi, _ = lvsa.expanded_window(T, W, t, G)
            assert all(lo <= f <= hi for f in nonglob)        # non-globals form the window
            if T >= C:
                assert C - (tper - 1) <= len(A) <= C          # budget band of the page
    # every frame is global at least once in any T_per consecutive steps
    for s0 in range(tper):
        seen = set()
        for s in range(s0, s0 + tper):
            seen |= set(lvsa.global_set(T, tper, s))
        assert seen == set(range(T))


def test_window_at_borders_has_2w_plus_1_frames():
    for T, W in [(121, 3), (10, 1), (9, 4)]:
        for t in range(T):
            lo, hi = lvsa.adaptive_window(T, W, t)
            assert hi - lo == 2 * W and 0 <= lo and hi <= T - 1
            assert lo <= t <= hi


def test_period_one_is_dense_attention():
    # C - (2W+1) >= T gives T_per = 1: every frame is global, attention is dense
    T, C, W = 4, 9, 1
    assert lvsa.global_period(T, C, W) == 1
    rng = np.random.default_rng(3)
    seg_len, stride, d = 50, 64, 8
    n = T * stride
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    valid = sla.valid_tokens(T, seg_len, stride)
    q[~valid] = k[~valid] = v[~valid] = 0
    sets = lvsa.attention_sets(T, C, W, 0)
    assert all(A == list(range(T)) for A in sets)
    out = lvsa.frame_mask_attention(q, k, v, T, seg_len, stride, sets)
    mask = torch.tensor(valid)[None, None, None, :].expand(1, 1, n, n)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None], torch.tensor(k)[None, None], torch.tensor(v)[None, None],
        attn_mask=mask)[0, 0].numpy()
    ref[~valid] = 0
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_frame_attention_matches_token_loop():
    # brute force: token-by-token softmax over the frames of A(t)
    T, C, W = 6, 5, 1
    rng = np.random.default_rng(4)
    stride, seg_len, d = 64, 40, 4
    n = T * stride
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    valid = sla.valid_tokens(T, seg_len, stride)
    sets = lvsa.attention_sets(T, C, W, 1)
    out = lvsa.frame_mask_attention(q, k, v, T, seg_len, stride, sets)
    for tok in itertools.chain(range(0, 40, 7), range(64 * 3, 64 * 3 + 40, 9)):
        f = tok // stride
        keys = [u for u in range(n) if valid[u] and (u // stride) in sets[f]]
        lg = np.array([q[tok] @ k[u] for u in keys]) / math.sqrt(d)
        p = np.exp(lg - lg.max())
        p /= p.sum()
        np.testing.assert_allclose(out[tok], p @ v[keys], rtol=1e-12, atol=1e-13)
    assert np.abs(out[~valid]).max() == 0
