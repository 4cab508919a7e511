"""SVOO co-clustered block-sparse attention oracle (fp64, CPU) -- test infrastructure only.

Source: gist.science summary of SVOO (arXiv 2603.18636), section 3 "方法论：SVOO
框架", stage 2 "在线双向协同聚类" (online bidirectional co-clustering):

* query and key centres start from randomly sampled query and key anchor tokens;
* step A (query-aware key partitioning): every key gets an affinity vector
  against the current query centres and joins the nearest key centre;
* step B (key-aware query partitioning): with the key centres just updated,
  every query does the same against the key centres and joins the nearest
  query centre;
* a few iterations (the page: about 2) give aligned Q and K blocks whose tokens
  share their attention preferences;
* dense attention is then computed only for the top block pairs, as many as the
  layer's offline sparsity schedule allows; the clusters may be reused for
  several denoising steps.

Readings where the page is silent (each is listed with the design notes):

1. The affinity vector of a token (or of a centre) is the vector of its dot
   products with the centres of the other side.  "Nearest" is the Euclidean
   distance between affinity vectors; ties go to the lower centre index.
2. A centre is initialised to its anchor token and, after each assignment, set
   to the mean of the tokens assigned to it; a centre with no token keeps its
   previous value.  The anchors (sampled token indices) are inputs.
3. One iteration is step A then step B; the labels of the last steps are the
   result.  Centres are kept in fp64 here.
4. The co-clustered blocks on a 64-token block engine: the tokens of each side
   are put in ascending order of their cluster label, keeping the original
   order inside a cluster (a stable sort), and the blocks are consecutive runs
   of 64 tokens of that order.  A cluster of s tokens then spans at most
   ceil(s / 64) + 1 blocks.
5. The top block pairs: within each query block of the reordered queries, the
   key blocks of the reordered keys are ranked by the SLA page's compressed
   score (block mean pooling, softmax(pool(Q) pool(K)^T / sqrt(d))) and the top
   kc = max(1, ceil(keep * Nb)) are computed; keep = 1 - the layer's sparsity is
   an input.  The rest are skipped: SVOO has no linear branch.
6. Attention is exact softmax over every key of the computed blocks, scale
   1 / sqrt(d); the output is returned in the original token order.
7. Pad tokens (the tail of a single segment) take the label C, past every
   cluster, so that they end the order; they take part in no centre.

Parity status: pinned (tests/test_oracle_svoo.py) -- a hand-worked 2-D example
whose query-aware metric disagrees with the Euclidean one (tests/golden/
svoo_cocluster_tiny.txt), recovery of well-separated mixture components, the
exact merge of key groups that differ only in directions no query centre sees,
step A with orthonormal query centres equal to a k-means step of scipy's
kmeans2, invariances (token order, sign and scale of q or k), the stable order
against numpy's stable argsort, and keep = 1 equal to dense attention (torch
SDPA) whatever the clusters.
"""
from __future__ import annotations

import numpy as np

from .sla import (BLOCK, block_counts, block_logits, block_sparse_attention, classify, compressed_scores,
                  lists_from_mask, pool_blocks)


def initial_centres(x: np.ndarray, anchors) -> np.ndarray:
    """Centres start as copies of the anchor tokens (reading 2): [C, d] fp64."""
    return np.array(x[np.asarray(anchors, dtype=np.int64)], dtype=np.float64)


def affinity(x: np.ndarray, other_centres: np.ndarray) -> np.ndarray:
    """Affinity vectors (reading 1): row t holds x_t . c for every centre c of the other side."""
    return np.asarray(x, dtype=np.float64) @ other_centres.T


def assign(x: np.ndarray, own_centres: np.ndarray, other_centres: np.ndarray, valid: np.ndarray,
           return_dist: bool = False, chunk: int = 4096):
    """Nearest own centre of every valid token in affinity space (reading 1).

    The distance is ||a_t - A_n||^2 with a_t the token's affinity vector and A_n
    the affinity vector of own centre n; ties go to the lower n (numpy's argmin
    returns the first minimum).  Pads get the label C (reading 7).  With
    ``return_dist`` also returns the [N, C] distances (inf for pads).
    """
    n_tok = x.shape[0]
    C = own_centres.shape[0]
    a_c = affinity(own_centres, other_centres)                    # [C, C_other]
    labels = np.full(n_tok, C, dtype=np.int64)
    dist_all = np.full((n_tok, C), np.inf) if return_dist else None
    idx = np.nonzero(valid)[0]
    for s in range(0, idx.size, chunk):
        rows = idx[s:s + chunk]
        a_t = affinity(x[rows], other_centres)                    # [rows, C_other]
        dist = ((a_t[:, None, :] - a_c[None, :, :]) ** 2).sum(axis=2)
        labels[rows] = np.argmin(dist, axis=1)
        if return_dist:
            dist_all[rows] = dist
    return (labels, dist_all) if return_dist else labels


def update_centres(x: np.ndarray, labels: np.ndarray, centres: np.ndarray) -> np.ndarray:
    """Mean of the tokens of each cluster; an empty cluster keeps its centre (reading 2)."""
    new = centres.copy()
    for c in range(centres.shape[0]):
        members = labels == c
        if members.any():
            new[c] = np.asarray(x[members], dtype=np.float64).mean(axis=0)
    return new


def co_cluster(q, k, q_anchor, k_anchor, iters: int = 2, valid=None, return_history: bool = False):
    """Bidirectional co-clustering of one head's queries and keys (steps A and B, reading 3).

    q, k: [N, d]; anchors: token indices of the initial centres.  Returns the
    final (q_labels, k_labels); with ``return_history`` also the list of
    per-iteration (k_labels, q_labels) pairs.
    """
    assert q.shape[0] == k.shape[0], "queries and keys are tokens of one sequence"
    if valid is None:
        valid = np.ones(q.shape[0], dtype=bool)
    cq = initial_centres(q, q_anchor)
    ck = initial_centres(k, k_anchor)
    history = []
    ql = kl = None
    for _ in range(iters):
        kl = assign(k, ck, cq, valid)          # step A: keys against the query centres
        ck = update_centres(k, kl, ck)
        ql = assign(q, cq, ck, valid)          # step B: queries against the updated key centres
        cq = update_centres(q, ql, cq)
        history.append((kl, ql))
    return (ql, kl, history) if return_history else (ql, kl)


def cluster_order(labels: np.ndarray, n_clusters: int) -> np.ndarray:
    """Position -> token: tokens by ascending label, original order within a label (reading 4)."""
    buckets = [[] for _ in range(n_clusters + 1)]
    for t, lab in enumerate(np.asarray(labels).tolist()):
        buckets[lab].append(t)
    return np.array([t for b in buckets for t in b], dtype=np.int64)


def block_selection(qp: np.ndarray, kp: np.ndarray, valid: np.ndarray, keep: float):
    """Reading 5 on the reordered tensors: (mask [Nb, Nb] with 1 = computed, 0 = skipped, P_c)."""
    nb = qp.shape[0] // BLOCK
    kc, _ = block_counts(nb, keep, 0.0)
    qbar = pool_blocks(qp, valid)
    kbar = pool_blocks(kp, valid)
    mask = classify(block_logits(qbar, kbar), kc, 0)
    return mask, compressed_scores(qbar, kbar)


def svoo_attention(q, k, v, q_perm, k_perm, keep: float, valid=None, rows=None, mask=None):
    """Attention of one head over the top block pairs of the co-clustered order (readings 4-6).

    q, k, v: [N, d] in the original token order; q_perm, k_perm: position ->
    token permutations whose first valid-count positions hold the valid tokens.
    ``rows`` restricts the work to some query blocks of the reordered queries;
    ``mask`` replaces the block selection (1 = computed).  Returns (out in the
    original order, mask, P_c).
    """
    n = q.shape[0]
    if valid is None:
        valid = np.ones(n, dtype=bool)
    q_perm = np.asarray(q_perm, dtype=np.int64)
    k_perm = np.asarray(k_perm, dtype=np.int64)
    qp, kp, vp = q[q_perm], k[k_perm], v[k_perm]
    scores = None
    if mask is None:
        mask, scores = block_selection(qp, kp, valid, keep)
    out_p = block_sparse_attention(qp, kp, vp, valid, lists_from_mask(mask, 1), rows=rows)
    out = np.zeros_like(out_p)
    out[q_perm] = out_p
    return out, mask, scores
