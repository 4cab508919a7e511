"""GPU parity of the SVOO calls against the fp64 oracle (oracle/svoo.py).

Co-clustering: on well-separated mixtures the labels and orders equal the oracle's
(and the mixture's own components) exactly, for one to three iterations.  On plain
N(0, 1) and frame-correlated inputs the oracle replays every step on the GPU's own
labels of the earlier steps (the call is deterministic, so the labels after i
iterations are those of a call with iters = i) and each GPU label must be the
oracle's, or a near tie: its affinity distance within 1e-5 (relative to the
magnitude of the terms) of the oracle's nearest.  The orders must be the stable
sort of the labels, exactly.  Attention: the kept block pairs must be the oracle's
top-kc of the reordered blocks except inside the 1e-5 band of P_c, and the output
must match the oracle evaluated on the GPU's orders and kept pairs; keep = 1 must
equal dense attention whatever the orders.  The Wan-shaped layer (12 heads,
32,760 tokens, 64 + 64 clusters, 2 iterations, 20 % kept) is checked on two heads'
replay, every head's order and mask, and 32 sampled query blocks of every head."""
import numpy as np
import pytest
import torch

import block_sparse_linear_02_b200 as slr
import workloads
from gpu_common import BAND, assert_close, check_mask, cuda, make_inputs, status_ok, to64, valid_np
from oracle import sla as osla
from oracle import svoo as osvoo

pytestmark = pytest.mark.gpu

TIE = 1e-5


def _anchors(B, H, C, n_valid, seed):
    gen = torch.Generator().manual_seed(seed)
    return torch.stack([torch.stack([torch.randperm(n_valid, generator=gen)[:C] for _ in range(H)])
                        for _ in range(B)]).to(torch.int32)


def _check_step(gpu, ref, x, own, other, valid, C):
    """GPU labels of one step against the oracle's assignment from the same centres."""
    assert (gpu[~valid] == C).all()
    diff = np.nonzero((gpu != ref) & valid)[0]
    if diff.size:
        _, dist = osvoo.assign(x[diff], own, other, np.ones(diff.size, dtype=bool), return_dist=True)
        alpha = osvoo.affinity(x[diff], other)
        a_c = osvoo.affinity(own, other)
        scale = (alpha ** 2).sum(axis=1) + (a_c ** 2).sum(axis=1).max()
        gap = dist[np.arange(diff.size), gpu[diff]] - dist[np.arange(diff.size), ref[diff]]
        assert (gap <= TIE * scale).all(), f"{int((gap > TIE * scale).sum())} labels off a near tie"
    return int(diff.size)


def _replay(q, k, qa, ka, hist, valid, n_qc, n_kc):
    """Oracle steps from the GPU's own earlier labels; returns the number of near-tie flips."""
    cq = osvoo.initial_centres(q, qa)
    ck = osvoo.initial_centres(k, ka)
    flips = 0
    for gk, gq in hist:
        flips += _check_step(gk, osvoo.assign(k, ck, cq, valid), k, ck, cq, valid, n_kc)
        ck = osvoo.update_centres(k, gk, ck)
        flips += _check_step(gq, osvoo.assign(q, cq, ck, valid), q, cq, ck, valid, n_qc)
        cq = osvoo.update_centres(q, gq, cq)
    return flips


def _cocluster_history(qd, kd, seq, qa, ka, iters):
    hist = []
    for it in range(1, iters + 1):
        ql, kl, qp, kp = slr.slr_svoo_cocluster(qd, kd, seq, qa, ka, iters=it)
        status_ok()
        hist.append((kl.cpu().numpy(), ql.cpu().numpy(), qp.cpu().numpy(), kp.cpu().numpy()))
    return hist


def _check_orders(hist):
    for kl, ql, qp, kp in hist:
        for b in range(ql.shape[0]):
            for h in range(ql.shape[1]):
                assert np.array_equal(qp[b, h], np.argsort(ql[b, h], kind="stable"))
                assert np.array_equal(kp[b, h], np.argsort(kl[b, h], kind="stable"))


@pytest.mark.parametrize("iters", [1, 2, 3])
@pytest.mark.parametrize("B,H,d,n_qc,n_kc,seg_len,stride", [
    (1, 2, 128, 8, 12, 4096, 4096),
    (2, 1, 64, 16, 5, 2017, 2048),       # ragged tail, two batch entries, odd cluster counts
])
def test_cocluster_mixture_exact(iters, B, H, d, n_qc, n_kc, seg_len, stride):
    q = torch.zeros(B, H, stride, d, dtype=torch.bfloat16)
    k = torch.zeros_like(q)
    comp_q, comp_k = {}, {}
    qa = torch.zeros(B, H, n_qc, dtype=torch.int32)
    ka = torch.zeros(B, H, n_kc, dtype=torch.int32)
    for b in range(B):
        for h in range(H):
            xq, cq_, aq = workloads.make_mixture(seg_len, d, n_qc, seed=100 + 10 * b + h)
            xk, ck_, ak = workloads.make_mixture(seg_len, d, n_kc, seed=200 + 10 * b + h)
            q[b, h, :seg_len], k[b, h, :seg_len] = xq, xk
            comp_q[b, h], comp_k[b, h] = cq_.numpy(), ck_.numpy()
            qa[b, h], ka[b, h] = aq.to(torch.int32), ak.to(torch.int32)
    seq = slr.make_seq(B, H, d, 1, seg_len, stride)
    ql, kl, qp, kp = slr.slr_svoo_cocluster(cuda(q), cuda(k), seq, cuda(qa), cuda(ka), iters=iters)
    status_ok()
    valid = valid_np(1, seg_len, stride)
    for b in range(B):
        for h in range(H):
            rq, rk = osvoo.co_cluster(to64(q[b, h]), to64(k[b, h]), qa[b, h].numpy(), ka[b, h].numpy(), iters=iters,
                                      valid=valid)
            assert np.array_equal(ql[b, h].cpu().numpy(), rq)
            assert np.array_equal(kl[b, h].cpu().numpy(), rk)
            assert np.array_equal(rq[:seg_len], comp_q[b, h]) and np.array_equal(rk[:seg_len], comp_k[b, h])
            assert np.array_equal(qp[b, h].cpu().numpy(), osvoo.cluster_order(rq, n_qc))
            assert np.array_equal(kp[b, h].cpu().numpy(), osvoo.cluster_order(rk, n_kc))


@pytest.mark.parametrize("B,H,d,n_qc,n_kc,seg_len,stride,iters,correlated", [
    (1, 2, 128, 16, 16, 4096, 4096, 2, False),
    (2, 2, 64, 24, 9, 2100, 2112, 3, False),
    (1, 1, 128, 128, 100, 8192, 8192, 2, True),
])
def test_cocluster_replay(B, H, d, n_qc, n_kc, seg_len, stride, iters, correlated):
    if correlated:
        w = workloads.small_variant(workloads.WAN, heads=H, d=d, frames=8, fh=32, fw=32, seg_stride=stride,
                                    seg_len=seg_len, batch=B)
        q, k, _ = workloads.make_qkv(w)
    else:
        q, k, _ = make_inputs(B, H, d, 1, seg_len, stride, seed=61 + d)
    qa = _anchors(B, H, n_qc, seg_len, 7)
    ka = _anchors(B, H, n_kc, seg_len, 8)
    seq = slr.make_seq(B, H, d, 1, seg_len, stride)
    qd, kd = cuda(q), cuda(k)
    hist = _cocluster_history(qd, kd, seq, cuda(qa), cuda(ka), iters)
    again = slr.slr_svoo_cocluster(qd, kd, seq, cuda(qa), cuda(ka), iters=iters)
    for a, b_ in zip(again, (hist[-1][1], hist[-1][0], hist[-1][2], hist[-1][3])):
        assert np.array_equal(a.cpu().numpy(), b_), "the call is not deterministic"
    _check_orders(hist)
    valid = valid_np(1, seg_len, stride)
    flips = 0
    for b in range(B):
        for h in range(H):
            per = [(kl[b, h], ql[b, h]) for kl, ql, _, _ in hist]
            flips += _replay(to64(q[b, h]), to64(k[b, h]), qa[b, h].numpy(), ka[b, h].numpy(), per, valid, n_qc,
                             n_kc)
    assert flips <= max(2, B * H * iters * seg_len // 2000), flips


def _attn_check(q, k, v, qp, kp, keep, out, mask, seg_len, rows=None):
    """Output and kept pairs of one head against the oracle on the GPU's orders."""
    valid = valid_np(1, seg_len, q.shape[0])
    q64, k64, v64 = to64(q), to64(k), to64(v)
    qpn = qp.cpu().numpy().astype(np.int64)
    kpn = kp.cpu().numpy().astype(np.int64)
    ref_mask, pc = osvoo.block_selection(q64[qpn], k64[kpn], valid, keep)
    nb = ref_mask.shape[0]
    kc, _ = osla.block_counts(nb, keep, 0.0)
    gm = mask.cpu().numpy()
    tau_c, tau_n = osla.threshold_band(pc, ref_mask)
    flips = check_mask(gm, ref_mask, pc, tau_c, tau_n, kc, 0)
    ref, _, _ = osvoo.svoo_attention(q64, k64, v64, qpn, kpn, keep, valid=valid, rows=rows, mask=gm)
    got = to64(out)
    if rows is not None:
        toks = qpn[np.concatenate([np.arange(r * 64, (r + 1) * 64) for r in rows])]
        got, ref = got[toks], ref[toks]
    return got, ref, flips


@pytest.mark.parametrize("B,H,d,seg_len,stride,keep", [
    (1, 2, 128, 4096, 4096, 0.25),
    (2, 1, 64, 3000, 3008, 0.1),
    (1, 2, 128, 2560, 2560, 0.5),
])
def test_svoo_attn_small(B, H, d, seg_len, stride, keep):
    q, k, v = make_inputs(B, H, d, 1, seg_len, stride, seed=71 + B)
    qa = _anchors(B, H, 12, seg_len, 9)
    ka = _anchors(B, H, 10, seg_len, 10)
    seq = slr.make_seq(B, H, d, 1, seg_len, stride)
    qd, kd, vd = cuda(q), cuda(k), cuda(v)
    _, _, qp, kp = slr.slr_svoo_cocluster(qd, kd, seq, cuda(qa), cuda(ka), iters=2)
    out, mask = slr.slr_svoo_attn(qd, kd, vd, seq, qp, kp, keep, mask_out=True)
    status_ok()
    outs, refs = [], []
    for b in range(B):
        for h in range(H):
            got, ref, _ = _attn_check(q[b, h], k[b, h], v[b, h], qp[b, h], kp[b, h], keep, out[b, h], mask[b, h],
                                      seg_len)
            outs.append(got)
            refs.append(ref)
    assert_close(np.concatenate(outs), np.concatenate(refs), f"svoo keep {keep}")


def test_svoo_attn_keep_one_is_dense_attention():
    B, H, d, seg_len, stride = 1, 2, 128, 1990, 2048
    q, k, v = make_inputs(B, H, d, 1, seg_len, stride, seed=77)
    seq = slr.make_seq(B, H, d, 1, seg_len, stride)
    qd, kd, vd = cuda(q), cuda(k), cuda(v)
    _, _, qp, kp = slr.slr_svoo_cocluster(qd, kd, seq, cuda(_anchors(B, H, 7, seg_len, 3)),
                                          cuda(_anchors(B, H, 6, seg_len, 4)), iters=2)
    out, mask = slr.slr_svoo_attn(qd, kd, vd, seq, qp, kp, 1.0, mask_out=True)
    status_ok()
    assert (mask.cpu() == 1).all()
    valid = valid_np(1, seg_len, stride)
    nb = stride // 64
    for h in range(H):
        ref = osla.block_sparse_attention(to64(q[0, h]), to64(k[0, h]), to64(v[0, h]), valid, [range(nb)] * nb)
        assert_close(to64(out[0, h]), ref, f"keep 1 head {h}")


def test_svoo_bad_indices_are_reported():
    B, H, d, n = 1, 1, 64, 1024
    q, k, v = make_inputs(B, H, d, 1, n, n, seed=79)
    seq = slr.make_seq(B, H, d, 1, n, n)
    qd, kd, vd = cuda(q), cuda(k), cuda(v)
    qa = _anchors(B, H, 4, n, 5)
    qa[0, 0, 2] = n + 3                         # not a token
    slr.slr_svoo_cocluster(qd, kd, seq, cuda(qa), cuda(_anchors(B, H, 4, n, 6)), iters=1)
    assert slr.slr_check_status() == slr.SLR_ERR_INDEX
    perm = torch.arange(n, dtype=torch.int32).reshape(1, 1, n)
    bad = perm.clone()
    bad[0, 0, 17] = -4
    slr.slr_svoo_attn(qd, kd, vd, seq, cuda(bad), cuda(perm), 0.5)
    assert slr.slr_check_status() == slr.SLR_ERR_INDEX
    out, _ = slr.slr_svoo_attn(qd, kd, vd, seq, cuda(perm), cuda(perm), 0.5)
    status_ok()


def test_svoo_workload_sampled():
    w = workloads.SVOO
    q, k, v = workloads.make_qkv(w)
    qa, ka = workloads.make_anchors(w, "q"), workloads.make_anchors(w, "k")
    seq = slr.make_seq(w.batch, w.heads, w.d, w.n_seg, w.seg_len, w.seg_stride)
    qd, kd, vd = cuda(q), cuda(k), cuda(v)
    hist = _cocluster_history(qd, kd, seq, cuda(qa), cuda(ka), w.iters)
    _check_orders(hist)
    valid = valid_np(1, w.seg_len, w.seg_stride)
    flips = 0
    for h in (0, w.heads - 1):
        per = [(kl[0, h], ql[0, h]) for kl, ql, _, _ in hist]
        flips += _replay(to64(q[0, h]), to64(k[0, h]), qa[0, h].numpy(), ka[0, h].numpy(), per, valid,
                         w.clusters[0], w.clusters[1])
    assert flips <= 20, flips
    qp = torch.from_numpy(hist[-1][2]).to("cuda")
    kp = torch.from_numpy(hist[-1][3]).to("cuda")
    out, mask = slr.slr_svoo_attn(qd, kd, vd, seq, qp, kp, w.keep_frac, mask_out=True)
    status_ok()
    nb = w.n_blocks
    rows = sorted({0, nb - 1} | set(np.random.default_rng(5).choice(nb, 30, replace=False).tolist()))
    outs, refs, band = [], [], 0
    for h in range(w.heads):
        got, ref, f = _attn_check(q[0, h], k[0, h], v[0, h], qp[0, h], kp[0, h], w.keep_frac, out[0, h], mask[0, h],
                                  w.seg_len, rows=rows)
        outs.append(got)
        refs.append(ref)
        band += f
    assert_close(np.concatenate(outs), np.concatenate(refs), "svoo wan layer, sampled blocks")
