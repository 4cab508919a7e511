"""GPU parity of slr_frame_mask_attn against the fp64 oracle: LVSA frame masks
(small case in full for four denoising steps and with two batch entries, the
121-frame workload on 64 sampled query blocks of every head, including the
first and last blocks and frame tails) and the gated tile neighbourhood + far
field (small grids in full, including an odd tile count and two batch entries,
and the 8x64x64 workload on sampled tokens), with and without the 3-D rotary
embedding of q and k; the sliding tile mask (small grids in full with windows of
one to seven tiles per axis, two batch entries, 8x64x64 on sampled tokens, and a
window covering the grid against the dense call)."""
import numpy as np
import pytest
import torch

import block_sparse_linear_02_b200 as slr
import workloads
from gpu_common import assert_close, cuda, make_inputs, rows_of_blocks, status_ok, to64, valid_np
from oracle import lvsa as olvsa
from oracle import sta as osta
from oracle import tile3d as otile

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("step", [0, 1, 2, 3])
def test_lvsa_small_full(step):
    T, C, W, seg_len, stride, H, d = 10, 6, 1, 100, 128, 2, 128
    q, k, v = make_inputs(1, H, d, T, seg_len, stride, seed=41)
    seq = slr.make_seq(1, H, d, T, seg_len, stride)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.lvsa_mask(T, C, W, step))
    status_ok()
    sets = olvsa.attention_sets(T, C, W, step)
    for h in range(H):
        ref = olvsa.frame_mask_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), T, seg_len, stride, sets)
        assert_close(to64(out[0, h]), ref, f"step {step} head {h}")


def test_lvsa_two_batch_entries():
    B, T, C, W, seg_len, stride, H, d = 2, 9, 6, 1, 150, 192, 2, 128
    q, k, v = make_inputs(B, H, d, T, seg_len, stride, seed=43)
    seq = slr.make_seq(B, H, d, T, seg_len, stride)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.lvsa_mask(T, C, W, 2))
    status_ok()
    sets = olvsa.attention_sets(T, C, W, 2)
    outs, refs = [], []
    for b in range(B):
        for h in range(H):
            outs.append(to64(out[b, h]))
            refs.append(olvsa.frame_mask_attention(to64(q[b, h]), to64(k[b, h]), to64(v[b, h]), T, seg_len, stride,
                                                   sets))
    assert_close(np.concatenate(outs), np.concatenate(refs), "lvsa B=2")


@pytest.mark.parametrize("step", [0, 3])
def test_lvsa_workload_sampled(step):
    w = workloads.LVSA
    q, k, v = workloads.make_qkv(w)
    seq = slr.make_seq(1, w.heads, w.d, w.n_seg, w.seg_len, w.seg_stride)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.lvsa_mask(w.frames, w.lvsa_C, w.lvsa_W, step))
    status_ok()
    sets = olvsa.attention_sets(w.frames, w.lvsa_C, w.lvsa_W, step)
    bpf = w.seg_stride // 64
    outs, refs = [], []
    for h in range(w.heads):
        rng = np.random.default_rng(100 * step + h)
        rows = sorted(set([0, 24, 25, 60 * bpf + 7, 120 * bpf + 24, w.n_blocks - 1] +
                          rng.choice(w.n_blocks, 58, replace=False).tolist()))
        sel = rows_of_blocks(rows)
        ref = olvsa.frame_mask_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), w.n_seg, w.seg_len,
                                         w.seg_stride, sets, rows=rows)
        outs.append(to64(out[0, h])[sel])
        refs.append(ref[sel])
    assert_close(np.concatenate(outs), np.concatenate(refs), "lvsa workload")
    pad = ~valid_np(w.n_seg, w.seg_len, w.seg_stride)
    assert torch.count_nonzero(out[0, 0, torch.from_numpy(pad)]).item() == 0


@pytest.mark.parametrize("F,Hh,Ww,cell,gate", [(8, 16, 16, (2, 4, 4), 0.55), (12, 8, 8, (3, 2, 2), 0.3),
                                               (4, 16, 32, (1, 4, 8), 1.0), (8, 8, 16, (2, 2, 4), 0.0)])
def test_tile3d_small_full(F, Hh, Ww, cell, gate):
    H, d = 2, 128
    n = F * Hh * Ww
    q, k, v = make_inputs(1, H, d, 1, n, n, seed=51)
    seq = slr.make_seq(1, H, d, 1, n, n)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.tile3d_mask(F, Hh, Ww, 1, cell, gate))
    status_ok()
    for h in range(H):
        r = otile.gated_head(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), F, Hh, Ww, cell=cell, gate=gate)
        assert_close(to64(out[0, h]), r["o"], f"tile3d head {h}")


def test_tile3d_two_batch_entries():
    B, H, d, F, Hh, Ww, cell = 2, 2, 128, 8, 8, 16, (2, 2, 4)
    n = F * Hh * Ww
    q, k, v = make_inputs(B, H, d, 1, n, n, seed=53)
    seq = slr.make_seq(B, H, d, 1, n, n)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.tile3d_mask(F, Hh, Ww, 1, cell, 0.55))
    status_ok()
    outs, refs = [], []
    for b in range(B):
        for h in range(H):
            r = otile.gated_head(to64(q[b, h]), to64(k[b, h]), to64(v[b, h]), F, Hh, Ww, cell=cell, gate=0.55)
            outs.append(to64(out[b, h]))
            refs.append(r["o"])
    assert_close(np.concatenate(outs), np.concatenate(refs), "tile3d B=2")


def test_tile3d_workload_sampled():
    w = workloads.ROPESLR
    q, k, v = workloads.make_qkv(w)
    seq = slr.make_seq(1, w.heads, w.d, 1, w.seg_len, w.seg_stride)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq,
                                  slr.tile3d_mask(w.frames, w.fh, w.fw, w.radius, w.cell, w.gate))
    status_ok()
    rng = np.random.default_rng(5)
    toks = sorted(set(rng.choice(w.n_pad, 300, replace=False).tolist() + [0, w.n_pad - 1, 64 * 64 * 4 - 1]))
    outs, refs = [], []
    for h in range(0, w.heads, 3):
        r = otile.gated_head(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), w.frames, w.fh, w.fw,
                             w.tile, w.radius, w.cell, w.gate, rows=toks)
        outs.append(to64(out[0, h])[toks])
        refs.append(r["o"][toks])
    assert_close(np.concatenate(outs), np.concatenate(refs), "tile3d workload")


@pytest.mark.parametrize("F,Hh,Ww,cell,d", [(8, 16, 16, (2, 4, 4), 128), (12, 8, 8, (3, 2, 2), 64),
                                            (4, 16, 32, (1, 4, 8), 128)])
def test_tile3d_rope_small_full(F, Hh, Ww, cell, d):
    H, n = 2, F * Hh * Ww
    q, k, v = make_inputs(1, H, d, 1, n, n, seed=57)
    seq = slr.make_seq(1, H, d, 1, n, n)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq,
                                  slr.tile3d_mask(F, Hh, Ww, 1, cell, 0.55, rope=True))
    status_ok()
    for h in range(H):
        r = otile.gated_head(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), F, Hh, Ww, cell=cell, gate=0.55,
                             rope=True)
        assert_close(to64(out[0, h]), r["o"], f"tile3d rope head {h}")
    # the rotation changes the result: the same call without it is far from the rotated oracle
    plain = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.tile3d_mask(F, Hh, Ww, 1, cell, 0.55))
    r = otile.gated_head(to64(q[0, 0]), to64(k[0, 0]), to64(v[0, 0]), F, Hh, Ww, cell=cell, gate=0.55, rope=True)
    assert np.abs(to64(plain[0, 0]) - r["o"]).max() > 0.05


def test_tile3d_rope_two_batch_entries():
    B, H, d, F, Hh, Ww, cell = 2, 2, 128, 8, 8, 16, (2, 2, 4)
    n = F * Hh * Ww
    q, k, v = make_inputs(B, H, d, 1, n, n, seed=59)
    seq = slr.make_seq(B, H, d, 1, n, n)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq,
                                  slr.tile3d_mask(F, Hh, Ww, 1, cell, 0.3, rope=True))
    status_ok()
    outs, refs = [], []
    for b in range(B):
        for h in range(H):
            r = otile.gated_head(to64(q[b, h]), to64(k[b, h]), to64(v[b, h]), F, Hh, Ww, cell=cell, gate=0.3,
                                 rope=True)
            outs.append(to64(out[b, h]))
            refs.append(r["o"])
    assert_close(np.concatenate(outs), np.concatenate(refs), "tile3d rope B=2")


def test_tile3d_rope_workload_sampled():
    w = workloads.ROPESLR
    q, k, v = workloads.make_qkv(w)
    seq = slr.make_seq(1, w.heads, w.d, 1, w.seg_len, w.seg_stride)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq,
                                  slr.tile3d_mask(w.frames, w.fh, w.fw, w.radius, w.cell, w.gate, rope=True))
    status_ok()
    rng = np.random.default_rng(7)
    # sampled tokens plus the raster's corners, where the height and width angles are largest
    toks = sorted(set(rng.choice(w.n_pad, 300, replace=False).tolist()
                      + [0, w.fw - 1, w.fh * w.fw - 1, w.n_pad - 1]))
    outs, refs = [], []
    for h in range(1, w.heads, 4):
        r = otile.gated_head(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), w.frames, w.fh, w.fw,
                             w.tile, w.radius, w.cell, w.gate, rows=toks, rope=True)
        outs.append(to64(out[0, h])[toks])
        refs.append(r["o"][toks])
    assert_close(np.concatenate(outs), np.concatenate(refs), "tile3d rope workload")


@pytest.mark.parametrize("F,Hh,Ww,window,d", [(8, 16, 16, (12, 12, 12), 128), (8, 16, 24, (4, 20, 12), 128),
                                              (12, 8, 32, (20, 4, 28), 64), (4, 16, 16, (4, 4, 4), 128)])
def test_sta_small_full(F, Hh, Ww, window, d):
    H, n = 2, F * Hh * Ww
    q, k, v = make_inputs(1, H, d, 1, n, n, seed=61)
    seq = slr.make_seq(1, H, d, 1, n, n)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.sta_mask(F, Hh, Ww, window))
    status_ok()
    for h in range(H):
        ref = osta.sliding_tile_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), F, Hh, Ww, window=window)
        assert_close(to64(out[0, h]), ref, f"sta head {h}")


def test_sta_two_batch_entries():
    B, H, d, F, Hh, Ww, window = 2, 2, 128, 8, 8, 16, (12, 4, 20)
    n = F * Hh * Ww
    q, k, v = make_inputs(B, H, d, 1, n, n, seed=63)
    seq = slr.make_seq(B, H, d, 1, n, n)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.sta_mask(F, Hh, Ww, window))
    status_ok()
    outs, refs = [], []
    for b in range(B):
        for h in range(H):
            refs.append(osta.sliding_tile_attention(to64(q[b, h]), to64(k[b, h]), to64(v[b, h]), F, Hh, Ww,
                                                    window=window))
            outs.append(to64(out[b, h]))
    assert_close(np.concatenate(outs), np.concatenate(refs), "sta B=2")


def test_sta_workload_sampled():
    w = workloads.STA
    q, k, v = workloads.make_qkv(w)
    seq = slr.make_seq(1, w.heads, w.d, 1, w.seg_len, w.seg_stride)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.sta_mask(w.frames, w.fh, w.fw, w.window))
    status_ok()
    rng = np.random.default_rng(9)
    toks = sorted(set(rng.choice(w.n_pad, 300, replace=False).tolist()
                      + [0, w.fw - 1, w.fh * w.fw - 1, w.n_pad - 1]))
    outs, refs = [], []
    for h in range(0, w.heads, 5):
        ref = osta.sliding_tile_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), w.frames, w.fh, w.fw,
                                          window=w.window, rows=toks)
        outs.append(to64(out[0, h])[toks])
        refs.append(ref[toks])
    assert_close(np.concatenate(outs), np.concatenate(refs), "sta workload")


def test_sta_window_covering_the_grid_is_dense_attention():
    # every tile within reach on every axis: the sliding tile call equals the library's dense
    # block-sparse call on the same (raster) tokens, and both equal plain softmax attention
    H, d, F, Hh, Ww = 2, 128, 8, 16, 16
    n = F * Hh * Ww
    q, k, v = make_inputs(1, H, d, 1, n, n, seed=67)
    seq = slr.make_seq(1, H, d, 1, n, n)
    out = slr.slr_frame_mask_attn(cuda(q), cuda(k), cuda(v), seq, slr.sta_mask(F, Hh, Ww, (12, 28, 28)))
    status_ok()
    dense, _ = slr.slr_block_sparse_attn(cuda(q), cuda(k), cuda(v), seq)
    status_ok()
    for h in range(H):
        ref = osta.sliding_tile_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), F, Hh, Ww, window=(12, 28, 28))
        assert_close(to64(out[0, h]), ref, f"sta covering head {h}")
        assert_close(to64(dense[0, h]), ref, f"dense head {h}")
