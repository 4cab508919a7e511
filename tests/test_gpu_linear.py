"""GPU parity of slr_linear_marginal (tcgen05 key states, mask-weighted
contraction and apply/projection) against the fp64 oracle, on ragged segments
with random three-way masks, with and without W_proj, d = 64 and 128, plus the
all-marginal and no-marginal special cases."""
import numpy as np
import pytest
import torch

import block_sparse_linear_02_b200 as slr
from gpu_common import assert_close, cuda, make_inputs, status_ok, to64, valid_np
from oracle import sla as osla
from workloads import random_bf16

pytestmark = pytest.mark.gpu


def _check(q, k, v, seq, mask, w, phi="elu1"):
    code = {"elu1": slr.SLR_PHI_ELU1, "softmax": slr.SLR_PHI_SOFTMAX}[phi]
    o = slr.slr_linear_marginal(cuda(q), cuda(k), cuda(v), seq, cuda(mask),
                                None if w is None else cuda(w), phi=code)
    status_ok()
    valid = valid_np(seq.n_seg, seq.seg_len, seq.seg_stride)
    for h in range(seq.H):
        ref = osla.linear_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), valid,
                                    mask[0, h].numpy() == 0, phi=phi)
        if w is not None:
            ref = ref @ to64(w)
        assert_close(o[0, h].cpu().double().numpy(), ref, f"head {h}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("proj", [False, True])
def test_random_masks_ragged(d, proj):
    H, n_seg, seg_len, stride = 2, 3, 600, 640
    q, k, v = make_inputs(1, H, d, n_seg, seg_len, stride, seed=21 + d)
    nb = n_seg * stride // 64
    rng = np.random.default_rng(d + proj)
    mask = torch.from_numpy(rng.integers(-1, 2, (1, H, nb, nb)).astype(np.int8))
    mask[0, 0, 5] = 1                     # a row with no marginal block -> 0
    w = random_bf16((d, d), 99, 1.0 / np.sqrt(d)) if proj else None
    _check(q, k, v, slr.make_seq(1, H, d, n_seg, seg_len, stride), mask, w)


def test_all_marginal():
    H, d, n = 2, 128, 1024
    q, k, v = make_inputs(1, H, d, 1, n - 20, n, seed=23)
    nb = n // 64
    mask = torch.zeros(1, H, nb, nb, dtype=torch.int8)
    _check(q, k, v, slr.make_seq(1, H, d, 1, n - 20, n), mask, None)


@pytest.mark.parametrize("d", [64, 128])
def test_softmax_feature_map_random_masks(d):
    H, n_seg, seg_len, stride = 2, 3, 600, 640
    q, k, v = make_inputs(1, H, d, n_seg, seg_len, stride, seed=51 + d)
    nb = n_seg * stride // 64
    rng = np.random.default_rng(70 + d)
    mask = torch.from_numpy(rng.integers(-1, 2, (1, H, nb, nb)).astype(np.int8))
    w = random_bf16((d, d), 98, 1.0 / np.sqrt(d))
    _check(q, k, v, slr.make_seq(1, H, d, n_seg, seg_len, stride), mask, w, phi="softmax")
