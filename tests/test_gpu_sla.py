"""GPU parity of slr_sparse_linear_attn (the full SLA forward) against the fp64
oracle: the tiny workload and ragged cases in full (one with two batch
entries), the 32k-token workload at full size (all masks of all heads, outputs
on 64 sampled query blocks of every head), the 115k-token workload (all masks
of all 24 heads, outputs on 64 sampled query blocks of every head), the 32k
workload with one or two critical blocks per query block (one- and two-step
tiles, many per CTA) and the dense mode.

Where the library's label row differs from the oracle's (only inside the 1e-5
threshold band, which check_mask enforces), that query block's output is
compared with the oracle run on the library's own labels, so that every
sampled block is still checked."""
import numpy as np
import pytest
import torch

import block_sparse_linear_02_b200 as slr
import workloads
from gpu_common import assert_close, check_mask, cuda, make_inputs, rows_of_blocks, status_ok, to64, valid_np
from oracle import sla as osla
from workloads import random_bf16

pytestmark = pytest.mark.gpu


def _seq(w):
    return slr.make_seq(w.batch, w.heads, w.d, w.n_seg, w.seg_len, w.seg_stride)


def _compare(q, k, v, wp, seq, crit, negl, out, mask, heads, sample=None, seed=0, batches=(0,), phi="elu1"):
    """Masks of every listed (b, h) in full; outputs on all or `sample` query blocks.
    Returns the number of query blocks whose label row differed (checked on the
    library's labels)."""
    valid = valid_np(seq.n_seg, seq.seg_len, seq.seg_stride)
    nb = seq.n_seg * seq.seg_stride // 64
    flipped = 0
    outs, refs = [], []
    w64 = to64(wp)
    for b in batches:
        for h in heads:
            rows = None
            if sample is not None:
                rng = np.random.default_rng(seed + 100 * b + h)
                rows = sorted(set([0, nb - 1] + list(rng.choice(nb, sample, replace=False))))
            q64, k64, v64 = to64(q[b, h]), to64(k[b, h]), to64(v[b, h])
            r = osla.sla_head(q64, k64, v64, w64, valid, crit, negl, rows=rows, phi=phi)
            gm = mask[b, h].cpu().numpy()
            check_mask(gm, r["mask"], r["p"], r["tau_c"], r["tau_n"], r["kc"], r["kn"])
            rows = list(range(nb)) if rows is None else rows
            o_ref = r["o"]
            moved = [i for i in rows if not (gm[i] == r["mask"][i]).all()]
            if moved:
                # the oracle's forward on the library's labels for those query blocks
                o_s = osla.block_sparse_attention(q64, k64, v64, valid, osla.lists_from_mask(gm, 1), rows=moved)
                o_l = osla.linear_attention(q64, k64, v64, valid, gm == 0, rows=moved, phi=phi)
                sel = rows_of_blocks(moved)
                o_ref = o_ref.copy()
                o_ref[sel] = (o_s + o_l @ w64)[sel]
                flipped += len(moved)
            sel = rows_of_blocks(rows)
            outs.append(to64(out[b, h])[sel])
            refs.append(o_ref[sel])
    assert_close(np.concatenate(outs), np.concatenate(refs), "sla output")
    return flipped


def test_tiny_workload_full():
    w = workloads.TINY
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), w.crit_frac,
                                           w.negl_frac, mask_out=True)
    status_ok()
    assert _compare(q, k, v, wp, _seq(w), w.crit_frac, w.negl_frac, out, mask, range(w.heads)) == 0


@pytest.mark.parametrize("d", [64, 128])
def test_ragged_full(d):
    H, n_seg, seg_len, stride = 2, 3, 600, 640
    q, k, v = make_inputs(1, H, d, n_seg, seg_len, stride, seed=31 + d)
    wp = random_bf16((d, d), 7, 1.0 / np.sqrt(d))
    seq = slr.make_seq(1, H, d, n_seg, seg_len, stride)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), seq, 0.1, 0.2, mask_out=True)
    status_ok()
    assert _compare(q, k, v, wp, seq, 0.1, 0.2, out, mask, range(H)) == 0
    # pad query rows are zero
    pad = ~valid_np(n_seg, seg_len, stride)
    assert torch.count_nonzero(out[0, :, torch.from_numpy(pad)]).item() == 0


@pytest.mark.parametrize("d", [64, 128])
def test_softmax_feature_map_ragged_full(d):
    # the linear branch with phi = softmax over each q and k row's channels
    H, n_seg, seg_len, stride = 2, 3, 600, 640
    q, k, v = make_inputs(1, H, d, n_seg, seg_len, stride, seed=41 + d)
    wp = random_bf16((d, d), 8, 1.0 / np.sqrt(d))
    seq = slr.make_seq(1, H, d, n_seg, seg_len, stride)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), seq, 0.1, 0.2, mask_out=True,
                                           phi=slr.SLR_PHI_SOFTMAX)
    status_ok()
    assert _compare(q, k, v, wp, seq, 0.1, 0.2, out, mask, range(H), phi="softmax") == 0


def test_softmax_feature_map_tiny_and_wan_sampled():
    # the tiny workload in full and the 32k-token workload on 16 sampled blocks of 4 heads
    w = workloads.TINY
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), w.crit_frac,
                                           w.negl_frac, mask_out=True, phi=slr.SLR_PHI_SOFTMAX)
    status_ok()
    assert _compare(q, k, v, wp, _seq(w), w.crit_frac, w.negl_frac, out, mask, range(w.heads), phi="softmax") == 0
    w = workloads.WAN
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), w.crit_frac,
                                           w.negl_frac, mask_out=True, phi=slr.SLR_PHI_SOFTMAX)
    status_ok()
    flipped = _compare(q, k, v, wp, _seq(w), w.crit_frac, w.negl_frac, out, mask, [0, 5, 6, 11], sample=16,
                       phi="softmax")
    assert flipped <= 2


def test_two_batch_entries_full():
    # B = 2: the library folds (b, h) into one index for its lists, states and TMA coordinates
    B, H, d, n_seg, seg_len, stride = 2, 3, 128, 2, 1000, 1024
    q, k, v = make_inputs(B, H, d, n_seg, seg_len, stride, seed=37)
    wp = random_bf16((d, d), 8, 1.0 / np.sqrt(d))
    seq = slr.make_seq(B, H, d, n_seg, seg_len, stride)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), seq, 0.15, 0.2, mask_out=True)
    status_ok()
    assert _compare(q, k, v, wp, seq, 0.15, 0.2, out, mask, range(H), batches=range(B)) == 0


def test_wan_workload_full_size():
    w = workloads.WAN
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), w.crit_frac,
                                           w.negl_frac, mask_out=True)
    status_ok()
    flipped = _compare(q, k, v, wp, _seq(w), w.crit_frac, w.negl_frac, out, mask, range(w.heads), sample=64)
    assert flipped <= 2


def test_hunyuan_workload_sampled():
    w = workloads.HUNYUAN
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), w.crit_frac,
                                           w.negl_frac, mask_out=True)
    status_ok()
    flipped = _compare(q, k, v, wp, _seq(w), w.crit_frac, w.negl_frac, out, mask, range(w.heads), sample=64)
    assert flipped <= 4


@pytest.mark.parametrize("crit", [0.001, 0.003])
def test_one_and_two_step_tiles_many_per_cta(crit):
    # one or two critical blocks per query block: every pair's tile walks one or two steps,
    # and each CTA takes ~21 such tiles in a row (a short tile hands its Q buffer back after
    # its only QK, so the next tile's Q and Z can land before this tile's softmax starts)
    w = workloads.WAN
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    kc, kn = slr.slr_block_counts(w.n_blocks, crit, w.negl_frac)
    assert kc == (1 if crit == 0.001 else 2)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), crit, w.negl_frac,
                                           mask_out=True)
    status_ok()
    flipped = _compare(q, k, v, wp, _seq(w), crit, w.negl_frac, out, mask, [0, 5, 11], sample=32, seed=7)
    assert flipped <= 2


@pytest.mark.parametrize("name", ["tiny", "wan"])
def test_dense_mode(name):
    w = workloads.BY_NAME[name]
    heads = min(w.heads, 2)
    q, k, v = workloads.make_qkv(w, heads=heads)
    seq = slr.make_seq(1, heads, w.d, w.n_seg, w.seg_len, w.seg_stride)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), None, seq, 1.0, 0.0, mask_out=True)
    status_ok()
    assert (mask == 1).all()
    valid = valid_np(w.n_seg, w.seg_len, w.seg_stride)
    nb = w.n_blocks
    rows = [0, 1, nb // 2, nb - 1]
    sel = rows_of_blocks(rows)
    for h in range(heads):
        ref = osla.block_sparse_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), valid,
                                          [list(range(nb))] * nb, rows=rows)
        assert_close(to64(out[0, h])[sel], ref[sel], f"dense head {h}")
