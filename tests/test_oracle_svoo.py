"""Pins of the SVOO co-clustering oracle (oracle/svoo.py) against values the
mathematics fixes: a hand-worked example, mixture ground truth, exact special
cases, a library k-means step, invariances and dense attention."""
import math
import os

import numpy as np
import pytest
import torch

import workloads
from oracle import svoo


def _golden(golden_dir):
    q, k, qa, ka, it = {}, {}, None, None, {}
    with open(os.path.join(golden_dir, "svoo_cocluster_tiny.txt")) as f:
        for line in f:
            w = line.split()
            if not w or w[0].startswith("#"):
                continue
            if w[0] in ("q", "k"):
                (q if w[0] == "q" else k)[int(w[1])] = (float(w[2]), float(w[3]))
            elif w[0] == "qa":
                qa = [int(x) for x in w[1:]]
            elif w[0] == "ka":
                ka = [int(x) for x in w[1:]]
            elif w[0] == "iter":
                it[(int(w[1]), w[2])] = [int(x) for x in w[3:]]
    to_arr = lambda m: np.array([m[i] for i in range(len(m))])
    return to_arr(q), to_arr(k), qa, ka, it


def test_hand_worked_example(golden_dir):
    q, k, qa, ka, expect = _golden(golden_dir)
    _, _, hist = svoo.co_cluster(q, k, qa, ka, iters=2, return_history=True)
    for i, (kl, ql) in enumerate(hist, start=1):
        assert kl.tolist() == expect[(i, "k")], f"iteration {i}, step A"
        assert ql.tolist() == expect[(i, "q")], f"iteration {i}, step B"
    ql1, kl1 = svoo.co_cluster(q, k, qa, ka, iters=1)
    assert ql1.tolist() == expect[(1, "q")] and kl1.tolist() == expect[(1, "k")]


def test_affinity_distance_hand_example():
    # query centres (2, 0) and (0, 1): a key's affinity vector is (2x, y)
    # key centres (0, 0) -> A0 = (0, 0) and (1, 3) -> A1 = (2, 3)
    # key (0.4, 2) -> (0.8, 2): |.-A0|^2 = 0.64 + 4 = 4.64, |.-A1|^2 = 1.44 + 1 = 2.44 -> 1
    # (a metric squared once more, 16 dx^2 + dy^2, would give 6.56 against 6.76 -> 0)
    q = np.array([[2.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    k = np.array([[0.0, 0.0], [1.0, 3.0], [0.4, 2.0]])
    _, kl, hist = svoo.co_cluster(q, k, [0, 1], [0, 1], iters=1, return_history=True)
    assert hist[0][0].tolist() == [0, 1, 1]


@pytest.mark.parametrize("iters", [1, 2, 3])
@pytest.mark.parametrize("d,n_comp", [(16, 6), (64, 12)])
def test_mixture_components_recovered(iters, d, n_comp):
    xq, cq, aq = workloads.make_mixture(700, d, n_comp, seed=11 + d)
    xk, ck, ak = workloads.make_mixture(700, d, n_comp, seed=29 + d)
    q = xq.double().numpy()
    k = xk.double().numpy()
    ql, kl = svoo.co_cluster(q, k, aq.numpy(), ak.numpy(), iters=iters)
    assert np.array_equal(ql, cq.numpy())
    assert np.array_equal(kl, ck.numpy())


def test_directions_no_query_centre_sees_merge_exactly():
    # queries live in the first half of the channels; two key groups differ only in the second
    rng = np.random.default_rng(3)
    d = 8
    q = np.zeros((40, d))
    q[:, :4] = rng.standard_normal((40, 4))
    base = rng.standard_normal((1, d))
    k = np.repeat(base, 40, axis=0) + 0.3 * rng.standard_normal((40, d)) * np.r_[np.zeros(4), np.ones(4)]
    k[20:, 4:] += 5.0                       # every key has the same first half
    _, kl = svoo.co_cluster(q, k, [0, 1], [0, 20], iters=1)
    assert (kl == 0).all()          # equal affinity vectors for both key centres: ties go to 0
    # the two groups are far apart in the plain Euclidean sense, so the case is not trivial
    eu = np.argmin(((k[:, None, :] - k[[0, 20]][None]) ** 2).sum(-1), axis=1)
    assert (eu[:20] == 0).all() and (eu[20:] == 1).all()


def test_step_a_with_orthonormal_query_centres_is_a_kmeans_step():
    from scipy.cluster.vq import kmeans2
    rng = np.random.default_rng(5)
    d, n, ck_n = 8, 300, 7
    q = rng.standard_normal((n, d))
    q[:d] = np.eye(d)                       # anchors 0..d-1: the query centres are the identity
    k = rng.standard_normal((n, d))
    ka = rng.choice(n, ck_n, replace=False)
    cq = svoo.initial_centres(q, np.arange(d))
    ck = svoo.initial_centres(k, ka)
    kl = svoo.assign(k, ck, cq, np.ones(n, dtype=bool))
    ck_new = svoo.update_centres(k, kl, ck)
    ref_centres, ref_labels = kmeans2(k, ck.copy(), iter=1, minit="matrix", missing="warn")
    assert np.array_equal(kl, ref_labels)
    np.testing.assert_allclose(ck_new, ref_centres, rtol=0, atol=1e-12)


def test_invariances():
    rng = np.random.default_rng(9)
    n, d = 400, 16
    q = rng.standard_normal((n, d))
    k = rng.standard_normal((n, d))
    qa = rng.choice(n, 10, replace=False)
    ka = rng.choice(n, 12, replace=False)
    ql, kl = svoo.co_cluster(q, k, qa, ka, iters=2)
    # sign and power-of-two scale of either side (exact in fp64)
    for qq, kk in ((-q, k), (q, -k), (2.0 * q, k), (q, 0.5 * k)):
        a, b = svoo.co_cluster(qq, kk, qa, ka, iters=2)
        assert np.array_equal(a, ql) and np.array_equal(b, kl)
    # relabelling the tokens relabels the result
    p = rng.permutation(n)
    inv = np.argsort(p)
    a, b = svoo.co_cluster(q[p], k[p], inv[qa], inv[ka], iters=2)
    assert np.array_equal(a, ql[p]) and np.array_equal(b, kl[p])
    # a centre that loses all its tokens keeps its value: duplicate anchors tie, the second never wins
    a, b = svoo.co_cluster(q, k, np.r_[qa, qa[:1]], ka, iters=1)
    assert not (a == 10).any()


def test_pads_take_label_c_and_enter_no_centre():
    rng = np.random.default_rng(13)
    n, d = 256, 8
    q = rng.standard_normal((n, d))
    k = rng.standard_normal((n, d))
    valid = np.arange(n) < 250
    qa, ka = rng.choice(250, 6, replace=False), rng.choice(250, 5, replace=False)
    ref = svoo.co_cluster(q[:250], k[:250], qa, ka, iters=2)
    q[250:] = 1e6
    k[250:] = -1e6
    ql, kl = svoo.co_cluster(q, k, qa, ka, iters=2, valid=valid)
    assert (ql[250:] == 6).all() and (kl[250:] == 5).all()
    assert np.array_equal(ql[:250], ref[0]) and np.array_equal(kl[:250], ref[1])
    order = svoo.cluster_order(ql, 6)
    assert (order[250:] >= 250).all()


def test_cluster_order_is_a_stable_sort():
    rng = np.random.default_rng(17)
    labels = rng.integers(0, 9, 1000)
    assert np.array_equal(svoo.cluster_order(labels, 8), np.argsort(labels, kind="stable"))


def test_keep_one_is_dense_attention_in_any_order():
    gen = torch.Generator().manual_seed(21)
    n, d = 320, 32
    q, k, v = (torch.randn(n, d, generator=gen, dtype=torch.float64) for _ in range(3))
    qa = torch.randperm(n, generator=gen)[:5].numpy()
    ka = torch.randperm(n, generator=gen)[:4].numpy()
    ql, kl = svoo.co_cluster(q.numpy(), k.numpy(), qa, ka, iters=2)
    qp, kp = svoo.cluster_order(ql, 5), svoo.cluster_order(kl, 4)
    assert not np.array_equal(qp, np.arange(n))          # the order really moved
    out, mask, _ = svoo.svoo_attention(q.numpy(), k.numpy(), v.numpy(), qp, kp, keep=1.0)
    assert (mask == 1).all()
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0]
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def test_skipped_key_blocks_do_not_reach_the_output():
    rng = np.random.default_rng(23)
    n, d = 512, 16
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    ql, kl = svoo.co_cluster(q, k, rng.choice(n, 4, replace=False), rng.choice(n, 4, replace=False))
    qp, kp = svoo.cluster_order(ql, 4), svoo.cluster_order(kl, 4)
    out, mask, pc = svoo.svoo_attention(q, k, v, qp, kp, keep=0.25)
    nb = n // 64
    assert (mask.sum(axis=1) == math.ceil(0.25 * nb)).all()
    # the kept blocks are the highest compressed scores of their row
    for i in range(nb):
        assert pc[i][mask[i] == 1].min() >= pc[i][mask[i] == 0].max()
    i = 3
    rows = qp[i * 64:(i + 1) * 64]                       # the tokens of reordered query block 3
    skipped = [j for j in range(nb) if mask[i, j] == 0]
    kept = [j for j in range(nb) if mask[i, j] == 1]
    v2 = v.copy()
    for j in skipped:
        v2[kp[j * 64:(j + 1) * 64]] += 100.0
    out2, _, _ = svoo.svoo_attention(q, k, v2, qp, kp, keep=0.25)
    np.testing.assert_allclose(out2[rows], out[rows], rtol=0, atol=1e-12)
    v3 = v.copy()
    v3[kp[kept[0] * 64]] += 100.0
    out3, _, _ = svoo.svoo_attention(q, k, v3, qp, kp, keep=0.25)
    assert np.abs(out3[rows] - out[rows]).max() > 1e-3
