"""GPU parity of slr_block_sparse_attn (tcgen05 block-sparse flash attention)
against the fp64 oracle: explicit ragged lists with duplicates and empty sets,
dense mode with an odd number of blocks, d = 64 and 128, the log-sum-exp
output, the maximum block count, and the out-of-range index error path."""
import numpy as np
import pytest
import torch

import block_sparse_linear_02_b200 as slr
from gpu_common import assert_close, cuda, make_inputs, status_ok, to64, valid_np
from oracle import sla as osla

pytestmark = pytest.mark.gpu


def _random_lists(BH, nb, kv_max, seed):
    rng = np.random.default_rng(seed)
    idx = np.zeros((BH, nb, kv_max), np.int32)
    cnt = np.zeros((BH, nb), np.int32)
    for h in range(BH):
        for i in range(nb):
            c = int(rng.integers(0, kv_max + 1))
            if i % 7 == 3:
                c = 0                                   # empty set
            idx[h, i, :c] = rng.integers(0, nb, c)      # may repeat
            cnt[h, i] = c
    return idx, cnt


@pytest.mark.parametrize("d", [64, 128])
def test_explicit_lists_ragged(d):
    H, n_seg, seg_len, stride, kv_max = 2, 3, 600, 640, 12
    q, k, v = make_inputs(1, H, d, n_seg, seg_len, stride, seed=1 + d)
    nb = n_seg * stride // 64
    idx, cnt = _random_lists(H, nb, kv_max, seed=d)
    seq = slr.make_seq(1, H, d, n_seg, seg_len, stride)
    o, lse = slr.slr_block_sparse_attn(cuda(q), cuda(k), cuda(v), seq,
                                       cuda(torch.from_numpy(idx).reshape(1, H, nb, kv_max)),
                                       cuda(torch.from_numpy(cnt).reshape(1, H, nb)), lse=True)
    status_ok()
    valid = valid_np(n_seg, seg_len, stride)
    for h in range(H):
        lists = [list(idx[h, i, :cnt[h, i]]) for i in range(nb)]
        ref, ref_lse = osla.block_sparse_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), valid, lists,
                                                   return_lse=True)
        assert_close(to64(o[0, h]), ref, f"head {h}")
        got = lse[0, h].cpu().double().numpy()
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(got), fin)
        assert np.abs(got[fin] - ref_lse[fin]).max() < 1e-3


def test_explicit_lists_two_batch_entries():
    # B = 2: lists, valid-key counts and TMA coordinates are indexed by b * H + h
    B, H, d, n_seg, seg_len, stride, kv_max = 2, 3, 128, 2, 450, 512, 9
    q, k, v = make_inputs(B, H, d, n_seg, seg_len, stride, seed=11)
    nb = n_seg * stride // 64
    idx, cnt = _random_lists(B * H, nb, kv_max, seed=12)
    seq = slr.make_seq(B, H, d, n_seg, seg_len, stride)
    o, _ = slr.slr_block_sparse_attn(cuda(q), cuda(k), cuda(v), seq,
                                     cuda(torch.from_numpy(idx).reshape(B, H, nb, kv_max)),
                                     cuda(torch.from_numpy(cnt).reshape(B, H, nb)))
    status_ok()
    valid = valid_np(n_seg, seg_len, stride)
    outs, refs = [], []
    for b in range(B):
        for h in range(H):
            lists = [list(idx[b * H + h, i, :cnt[b * H + h, i]]) for i in range(nb)]
            refs.append(osla.block_sparse_attention(to64(q[b, h]), to64(k[b, h]), to64(v[b, h]), valid, lists))
            outs.append(to64(o[b, h]))
    assert_close(np.concatenate(outs), np.concatenate(refs), "explicit lists B=2")


@pytest.mark.parametrize("d", [64, 128])
def test_dense_odd_block_count(d):
    H, seg_len, stride = 2, 300, 320           # 5 blocks -> the last pair has one block
    q, k, v = make_inputs(1, H, d, 1, seg_len, stride, seed=3 + d)
    seq = slr.make_seq(1, H, d, 1, seg_len, stride)
    o, _ = slr.slr_block_sparse_attn(cuda(q), cuda(k), cuda(v), seq)
    status_ok()
    valid = valid_np(1, seg_len, stride)
    for h in range(H):
        ref = osla.block_sparse_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), valid, [list(range(5))] * 5)
        assert_close(to64(o[0, h]), ref, f"head {h}")


def test_all_sets_empty_gives_zero_and_minus_inf_lse():
    H, d, n = 1, 128, 256
    q, k, v = make_inputs(1, H, d, 1, n, n, seed=5)
    seq = slr.make_seq(1, H, d, 1, n, n)
    idx = torch.zeros(1, H, 4, 3, dtype=torch.int32)
    cnt = torch.zeros(1, H, 4, dtype=torch.int32)
    o, lse = slr.slr_block_sparse_attn(cuda(q), cuda(k), cuda(v), seq, cuda(idx), cuda(cnt), lse=True)
    status_ok()
    assert torch.count_nonzero(o).item() == 0
    assert torch.isinf(lse).all() and (lse < 0).all()


def test_out_of_range_index_reports_error():
    H, d, n = 1, 64, 256
    q, k, v = make_inputs(1, H, d, 1, n, n, seed=6)
    seq = slr.make_seq(1, H, d, 1, n, n)
    idx = torch.tensor([[[[0, 4], [1, 2], [3, -1], [2, 2]]]], dtype=torch.int32)
    cnt = torch.full((1, H, 4), 2, dtype=torch.int32)
    o, _ = slr.slr_block_sparse_attn(cuda(q), cuda(k), cuda(v), seq, cuda(idx), cuda(cnt))
    torch.cuda.synchronize()
    assert slr.slr_check_status() == slr.SLR_ERR_INDEX
    # the valid entries were still attended: block 1 attends {1, 2}
    valid = np.ones(n, bool)
    ref = osla.block_sparse_attention(to64(q[0, 0]), to64(k[0, 0]), to64(v[0, 0]), valid, [[0], [1, 2], [3], [2]])
    assert_close(to64(o[0, 0]), ref, "valid entries")
    assert slr.slr_check_status() == slr.SLR_OK


def test_maximum_block_count_dense_sampled():
    H, d, n = 1, 64, 8192 * 64                 # 8192 key blocks, the library maximum
    q, k, v = make_inputs(1, H, d, 1, n, n, seed=7)
    seq = slr.make_seq(1, H, d, 1, n, n)
    o, _ = slr.slr_block_sparse_attn(cuda(q), cuda(k), cuda(v), seq)
    status_ok()
    valid = np.ones(n, bool)
    rows = [0, 4097, 8191]
    all_blocks = [list(range(8192))] * 8192
    ref = osla.block_sparse_attention(to64(q[0, 0]), to64(k[0, 0]), to64(v[0, 0]), valid, all_blocks, rows=rows)
    sel = np.concatenate([np.arange(b * 64, b * 64 + 64) for b in rows])
    assert_close(to64(o[0, 0])[sel], ref[sel], "sampled blocks")
