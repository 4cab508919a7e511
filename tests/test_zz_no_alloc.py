"""slr_block_sparse_attn_noalloc: the workspace-free attention call for callers
that cannot allocate device memory for the library (a host application that
owns the whole device-memory budget, or a plug-in whose interface only passes
inputs and outputs).  Its scratch is a static device array inside libslr.

Checked through the C ABI against the workspace entry point
slr_block_sparse_attn on two calls in a row (different shapes, so stale lists
left in the shared scratch by the first call would show in the second), plus
the dense mode, the size limit, one direct comparison with the fp64 oracle and
the status word read through slr_check_status(NULL) when no status tensor is
passed.  Every call here runs after the previous one on one stream: calls that
overlap on the GPU race on the shared array and are not exercised.  Collected
last so that a failure here cannot hide the other GPU tests."""
import numpy as np
import pytest
import torch

import block_sparse_linear_02_b200 as slr
from gpu_common import MAX_ABS, RMS_REL, assert_close, cuda, make_inputs, to64, valid_np
from oracle import sla as osla

pytestmark = pytest.mark.gpu


def _lists(BH, nb, kv_max, seed):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, nb, (1, BH, nb, kv_max)).astype(np.int32)
    cnt = rng.integers(0, kv_max + 1, (1, BH, nb)).astype(np.int32)
    return cuda(torch.from_numpy(idx)), cuda(torch.from_numpy(cnt))


def test_noalloc_matches_workspace_call_on_two_calls_in_a_row():
    cases = [(2, 128, 3, 600, 640, 12, 71), (1, 64, 2, 250, 256, 5, 72)]
    for H, d, n_seg, seg_len, stride, kv_max, seed in cases:
        q, k, v = (cuda(x) for x in make_inputs(1, H, d, n_seg, seg_len, stride, seed))
        seq = slr.make_seq(1, H, d, n_seg, seg_len, stride)
        idx, cnt = _lists(H, n_seg * stride // 64, kv_max, seed)
        status = torch.full((1,), -7, dtype=torch.int32, device="cuda")
        o_na, l_na = slr.slr_block_sparse_attn_noalloc(q, k, v, seq, idx, cnt, lse=True, status=status)
        o_ws, l_ws = slr.slr_block_sparse_attn(q, k, v, seq, idx, cnt, lse=True)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close(to64(o_na), to64(o_ws), f"noalloc H={H} d={d}", MAX_ABS, RMS_REL)
        fin = torch.isfinite(l_ws)
        assert torch.equal(torch.isfinite(l_na), fin)
        assert (l_na[fin] - l_ws[fin]).abs().max().item() < 1e-3


def test_noalloc_dense_mode():
    q, k, v = (cuda(x) for x in make_inputs(1, 1, 128, 1, 300, 320, 73))
    seq = slr.make_seq(1, 1, 128, 1, 300, 320)
    o_na, _ = slr.slr_block_sparse_attn_noalloc(q, k, v, seq)
    o_ws, _ = slr.slr_block_sparse_attn(q, k, v, seq)
    torch.cuda.synchronize()
    assert_close(to64(o_na), to64(o_ws), "noalloc dense", MAX_ABS, RMS_REL)


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    # 64 heads x 256 pairs x (512 + 1) x 4 bytes = 33.6 MB > 4 MiB of static scratch
    H, n = 64, 512 * 64
    q = torch.zeros(1, H, n, 64, dtype=torch.bfloat16, device="cuda")
    seq = slr.make_seq(1, H, 64, 1, n, n)
    idx = torch.zeros(1, H, 512, 256, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, H, 512, dtype=torch.int32, device="cuda")
    with pytest.raises(slr.SlrError) as e:
        slr.slr_block_sparse_attn_noalloc(q, q, q, seq, idx, cnt)
    assert e.value.code == slr.SLR_ERR_WORKSPACE


def test_noalloc_matches_oracle_directly():
    """The no-workspace call against the fp64 oracle itself (ragged segments, duplicates in a set)."""
    H, d, n_seg, seg_len, stride = 2, 128, 2, 500, 512
    q, k, v = make_inputs(1, H, d, n_seg, seg_len, stride, seed=74)
    seq = slr.make_seq(1, H, d, n_seg, seg_len, stride)
    nb = n_seg * stride // 64
    idx_np = np.random.default_rng(74).integers(0, nb, (1, H, nb, 6)).astype(np.int32)
    cnt_np = np.random.default_rng(75).integers(0, 7, (1, H, nb)).astype(np.int32)
    idx_np[0, 0, 3, :3] = 5                      # a duplicated entry counts once
    cnt_np[0, 0, 3] = 3
    o, _ = slr.slr_block_sparse_attn_noalloc(cuda(q), cuda(k), cuda(v), seq, cuda(torch.from_numpy(idx_np)),
                                             cuda(torch.from_numpy(cnt_np)))
    assert slr.slr_check_noalloc_status() == slr.SLR_OK
    valid = valid_np(n_seg, seg_len, stride)
    for h in range(H):
        sets = [idx_np[0, h, i, :cnt_np[0, h, i]].tolist() for i in range(nb)]
        ref = osla.block_sparse_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), valid, sets)
        assert_close(to64(o[0, h]), ref, f"noalloc vs oracle head {h}")


def test_noalloc_status_without_status_tensor():
    """An out-of-range entry, with no status tensor passed: the error lands in the static
    scratch's status word and slr_check_status(NULL) (slr_check_noalloc_status) reports it."""
    H, d, n = 1, 64, 256
    q, k, v = (cuda(x) for x in make_inputs(1, H, d, 1, n, n, seed=76))
    seq = slr.make_seq(1, H, d, 1, n, n)
    idx = cuda(torch.tensor([[[[0, 4], [1, 2], [3, -1], [2, 2]]]], dtype=torch.int32))
    cnt = cuda(torch.full((1, H, 4), 2, dtype=torch.int32))
    o, _ = slr.slr_block_sparse_attn_noalloc(q, k, v, seq, idx, cnt)
    assert slr.slr_check_noalloc_status() == slr.SLR_ERR_INDEX
    assert slr.slr_check_noalloc_status() == slr.SLR_OK            # read and cleared
    ref = osla.block_sparse_attention(to64(q[0, 0]), to64(k[0, 0]), to64(v[0, 0]), np.ones(n, bool),
                                      [[0], [1, 2], [3], [2]])
    assert_close(to64(o[0, 0]), ref, "valid entries still attended")
    # the next call starts from a cleared word
    good = cuda(torch.tensor([[[[0, 1], [1, 2], [3, 0], [2, 2]]]], dtype=torch.int32))
    slr.slr_block_sparse_attn_noalloc(q, k, v, seq, good, cnt)
    assert slr.slr_check_noalloc_status() == slr.SLR_OK
