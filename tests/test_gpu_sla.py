"""GPU parity of slr_sparse_linear_attn (the full SLA forward) against the fp64
oracle: the tiny workload and a ragged case in full, the 32k-token workload at
full size (all masks, outputs on sampled query blocks of every head), the
115k-token workload (all masks of all heads, outputs on sampled blocks of four
heads) and the dense mode."""
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


def _compare(q, k, v, wp, seq, crit, negl, out, mask, heads, sample=None, seed=0):
    valid = valid_np(seq.n_seg, seq.seg_len, seq.seg_stride)
    nb = seq.n_seg * seq.seg_stride // 64
    skipped = 0
    outs, refs = [], []
    for h in heads:
        rows = None
        if sample is not None:
            rng = np.random.default_rng(seed + h)
            rows = sorted(set([0, nb - 1] + list(rng.choice(nb, sample, replace=False))))
        r = osla.sla_head(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), to64(wp), valid, crit, negl, rows=rows)
        gm = mask[0, h].cpu().numpy()
        check_mask(gm, r["mask"], r["p"], r["tau_c"], r["tau_n"], r["kc"], r["kn"])
        rows = list(range(nb)) if rows is None else rows
        keep = [i for i in rows if (gm[i] == r["mask"][i]).all()]
        skipped += len(rows) - len(keep)
        sel = rows_of_blocks(keep)
        outs.append(to64(out[0, h])[sel])
        refs.append(r["o"][sel])
    assert_close(np.concatenate(outs), np.concatenate(refs), "sla output")
    return skipped


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


def test_wan_workload_full_size():
    w = workloads.WAN
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), w.crit_frac,
                                           w.negl_frac, mask_out=True)
    status_ok()
    skipped = _compare(q, k, v, wp, _seq(w), w.crit_frac, w.negl_frac, out, mask, range(w.heads), sample=14)
    assert skipped <= 2


def test_hunyuan_workload_sampled():
    w = workloads.HUNYUAN
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    out, mask = slr.slr_sparse_linear_attn(cuda(q), cuda(k), cuda(v), cuda(wp), _seq(w), w.crit_frac,
                                           w.negl_frac, mask_out=True)
    status_ok()
    skipped = _compare(q, k, v, wp, _seq(w), w.crit_frac, w.negl_frac, out, mask, [0, 7, 15, 23], sample=6)
    assert skipped <= 2


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
