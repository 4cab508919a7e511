"""SLA oracle (fp64, CPU) -- test infrastructure only.

Source: techwalker page "清华大学破解视频生成卡顿难题" (SLA, arXiv 2509.24006),
section 3 "SLA方法的核心机制":

* Q and K are mean-pooled per token block and a compressed attention-weight
  matrix P_c = softmax(pool(Q) pool(K)^T / sqrt(d)) is formed;
* each position of P_c is labelled critical (1, top 5 %), negligible (-1,
  bottom 10 %) or marginal (0, the rest);
* critical pairs get exact softmax (FlashAttention-style) attention;
* marginal pairs get linear attention with a feature map phi, evaluated by
  forming K^T V first and multiplying by Q afterwards;
* negligible pairs are skipped;
* a learnable projection is applied to the linear-attention output before it
  is added to the sparse output (same section, the paragraph on the projection layer).

Readings where the page is silent:

1. Percentiles are taken per query-block row of P_c.
2. kc = max(1, ceil(p_c * Nkb)), kn = floor(p_n * Nkb), capped so that
   kc + kn <= Nkb; the fractions are first rounded to fp32 (the C ABI takes
   ``float``) and a 1e-3 slack absorbs that rounding.
3. Rows are ranked by (P_c descending, key-block index ascending).  Softmax is
   strictly increasing within a row, so this ranks the fp64 logits; the oracle
   ranks the logits so that exp rounding cannot invent ties.
4. Linear attention is normalised: O_l = phi(q) H / (phi(q) . Z) with
   H = sum phi(k)^T v, Z = sum phi(k) over the marginal keys; phi = elu + 1;
   a row with no marginal key gives O_l = 0.
4b. The page also reports (the paragraph on the linear branch's activation
   function) that a softmax feature map worked better than elu + 1 or ReLU,
   without defining it.  The plainest reading, available here as
   ``phi="softmax"``: each q and k row is mapped by a softmax over its d
   channels, applied to Q and K separately; the rest of the branch is
   unchanged.  (Not on the library's path yet: its feature map is elu + 1.)
5. The projection is a right product O_l @ W_proj with W_proj [d, d], no bias.
6. Pad tokens (past ``seg_len`` in a segment) are excluded from every sum; pad
   query rows give 0.  Pooled means use valid tokens only.
7. Blocks are 64 consecutive tokens of the raster (frame, h, w) sequence.

Parity status: every function here is pinned (tests/test_oracle_sla.py).
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64


def valid_tokens(n_seg: int, seg_len: int, seg_stride: int) -> np.ndarray:
    """Boolean [n_seg*seg_stride]: token t is valid iff (t mod seg_stride) < seg_len."""
    t = np.arange(n_seg * seg_stride)
    return (t % seg_stride) < seg_len


def block_counts(n_kb: int, crit_frac: float, negl_frac: float) -> tuple[int, int]:
    """(kc, kn): how many key blocks of a row are critical and negligible (reading 2)."""
    pc = float(np.float32(crit_frac))
    pn = float(np.float32(negl_frac))
    kc = min(n_kb, max(1, math.ceil(pc * n_kb - 1e-3)))
    kn = min(n_kb - kc, max(0, math.floor(pn * n_kb + 1e-3)))
    return kc, kn


def pool_blocks(x: np.ndarray, valid: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Mean of the valid tokens of every block: x [N, d] -> [N/block, d] (SLA page, sec. 3)."""
    n, d = x.shape
    nb = n // block
    xb = x.reshape(nb, block, d)
    vb = valid.reshape(nb, block)
    out = np.zeros((nb, d))
    for i in range(nb):
        rows = xb[i][vb[i]]
        out[i] = rows.sum(axis=0) / rows.shape[0]
    return out


def block_logits(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """pool(Q) pool(K)^T / sqrt(d): the argument of the compressed softmax."""
    d = qbar.shape[1]
    return (qbar @ kbar.T) / math.sqrt(d)


def row_softmax(s: np.ndarray) -> np.ndarray:
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def compressed_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """P_c = softmax(pool(Q) pool(K)^T / sqrt(d)), row-wise (SLA page, sec. 3)."""
    return row_softmax(block_logits(qbar, kbar))


def classify(logits: np.ndarray, kc: int, kn: int) -> np.ndarray:
    """Three-way block mask: 1 = critical (top kc), -1 = negligible (bottom kn), 0 = marginal.

    Each row is ordered by (score descending, index ascending); the first kc
    entries are critical and the last kn negligible (readings 1-3).
    """
    nq, nk = logits.shape
    mask = np.zeros((nq, nk), dtype=np.int8)
    idx = np.arange(nk)
    for i in range(nq):
        order = np.lexsort((idx, -logits[i]))      # primary key: -score, then index
        mask[i, order[:kc]] = 1
        if kn > 0:
            mask[i, order[nk - kn:]] = -1
    return mask


def threshold_band(p: np.ndarray, mask: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per row: tau_c = smallest critical P_c, tau_n = largest negligible P_c (nan if none)."""
    nq = p.shape[0]
    tau_c = np.full(nq, np.nan)
    tau_n = np.full(nq, np.nan)
    for i in range(nq):
        c = p[i][mask[i] == 1]
        n = p[i][mask[i] == -1]
        if c.size:
            tau_c[i] = c.min()
        if n.size:
            tau_n[i] = n.max()
    return tau_c, tau_n


def lists_from_mask(mask: np.ndarray, value: int) -> list[np.ndarray]:
    """Per row, the ascending key-block indices whose mask equals ``value``."""
    return [np.nonzero(mask[i] == value)[0] for i in range(mask.shape[0])]


def block_sparse_attention(q, k, v, valid, key_blocks, rows=None, block: int = BLOCK, return_lse=False):
    """Exact softmax attention of every query block over the listed key blocks.

    ``key_blocks[i]`` is a set of key-block indices for query block i (duplicates
    count once).  Only valid keys enter the softmax; pad queries and query blocks
    with no valid key give 0 (SLA page sec. 3, critical branch; LVSA page step 6
    writes the same normalised sum).  ``rows`` restricts the work to some query
    blocks; the others are left 0.  With ``return_lse`` also returns the natural
    log-sum-exp of each valid query's scaled logits (-inf with no key, 0 for pads).
    """
    n, d = q.shape
    nb = n // block
    out = np.zeros((n, v.shape[1]))
    lse = np.zeros(n)
    scale = 1.0 / math.sqrt(d)
    rows = range(nb) if rows is None else rows
    for i in rows:
        t0 = i * block
        qrows = np.arange(t0, t0 + block)
        qrows = qrows[valid[qrows]]
        blocks = np.unique(np.asarray(key_blocks[i], dtype=np.int64))
        keys = (blocks[:, None] * block + np.arange(block)[None, :]).reshape(-1)
        keys = keys[valid[keys]] if keys.size else keys
        if keys.size == 0 or qrows.size == 0:
            lse[qrows] = -np.inf
            continue
        s = (q[qrows] @ k[keys].T) * scale
        out[qrows] = row_softmax(s) @ v[keys]
        m = s.max(axis=1)
        lse[qrows] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return (out, lse) if return_lse else out


def phi_elu1(x: np.ndarray) -> np.ndarray:
    """phi(x) = elu(x) + 1 = x + 1 for x > 0, exp(x) otherwise (always > 0)."""
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def phi_softmax(x: np.ndarray) -> np.ndarray:
    """phi(x) = softmax of each row over its channels (reading 4b); shifted by the
    row max before the exponential, which does not change the result."""
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


FEATURE_MAPS = {"elu1": phi_elu1, "softmax": phi_softmax}


def key_block_states(k, v, valid, block: int = BLOCK, phi: str = "elu1"):
    """Per key block j: h_j = phi(K_j)^T V_j [d, dv] and z_j = sum_t phi(K_j,t) [d].

    The linear branch is evaluated "K^T V first, then Q" (SLA page sec. 3);
    pad keys contribute nothing.
    """
    n, d = k.shape
    nb = n // block
    dv = v.shape[1]
    h = np.zeros((nb, d, dv))
    z = np.zeros((nb, d))
    for j in range(nb):
        r = np.arange(j * block, (j + 1) * block)
        r = r[valid[r]]
        fk = FEATURE_MAPS[phi](k[r])
        h[j] = fk.T @ v[r]
        z[j] = fk.sum(axis=0)
    return h, z


def linear_attention(q, k, v, valid, marginal, rows=None, block: int = BLOCK, phi: str = "elu1"):
    """Linear attention of every query block over its marginal key blocks.

    ``marginal`` is a boolean [Nqb, Nkb] selector.  For query block i,
    H_i = sum_{j marginal} h_j and Z_i = sum z_j, then for each valid query t,
    O_l,t = phi(q_t) H_i / (phi(q_t) . Z_i); 0 when i has no marginal block or t
    is a pad (readings 4 and 6).
    """
    n, d = q.shape
    nb = n // block
    h, z = key_block_states(k, v, valid, block, phi)
    sel = np.asarray(marginal, dtype=np.float64)
    out = np.zeros((n, v.shape[1]))
    rows = range(nb) if rows is None else rows
    for i in rows:
        if not sel[i].any():
            continue
        H = np.tensordot(sel[i], h, axes=(0, 0))
        Z = sel[i] @ z
        t = np.arange(i * block, (i + 1) * block)
        t = t[valid[t]]
        fq = FEATURE_MAPS[phi](q[t])
        out[t] = (fq @ H) / (fq @ Z)[:, None]
    return out


def sla_head(q, k, v, w_proj, valid, crit_frac, negl_frac, rows=None, block: int = BLOCK, phi: str = "elu1"):
    """The SLA forward of one head: O = O_s + O_l @ W_proj (SLA page sec. 3 and 5).

    Returns a dict with the pooled means, logits, P_c, the mask, the per-row
    thresholds and the three outputs.
    """
    qbar = pool_blocks(q, valid, block)
    kbar = pool_blocks(k, valid, block)
    logits = block_logits(qbar, kbar)
    p = row_softmax(logits)
    kc, kn = block_counts(kbar.shape[0], crit_frac, negl_frac)
    mask = classify(logits, kc, kn)
    o_s = block_sparse_attention(q, k, v, valid, lists_from_mask(mask, 1), rows, block)
    o_l = linear_attention(q, k, v, valid, mask == 0, rows, block, phi)
    o = o_s + o_l @ np.asarray(w_proj, dtype=np.float64)
    tau_c, tau_n = threshold_band(p, mask)
    return dict(qbar=qbar, kbar=kbar, logits=logits, p=p, mask=mask, kc=kc, kn=kn,
                tau_c=tau_c, tau_n=tau_n, o_s=o_s, o_l=o_l, o=o)


def sla(q, k, v, w_proj, n_seg, seg_len, seg_stride, crit_frac, negl_frac, rows=None, phi: str = "elu1"):
    """SLA over [B, H, N, d] fp64 arrays; returns a list (over b, h) of ``sla_head`` dicts."""
    valid = valid_tokens(n_seg, seg_len, seg_stride)
    res = []
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            res.append(sla_head(q[b, h], k[b, h], v[b, h], w_proj, valid,
                                crit_frac, negl_frac, rows, phi=phi))
    return res
