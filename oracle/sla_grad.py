"""SLA backward oracle (fp64, CPU) -- test infrastructure only.

Source: techwalker page "清华大学破解视频生成卡顿难题" (SLA, arXiv 2509.24006),
section 3 "SLA方法的核心机制", last paragraph: SLA has a backward pass as well as a
forward one, split the same way -- the sparse part takes the usual FlashAttention
gradients, the linear part gradients of its own -- so that the method can be used
for fine-tuning.

What is differentiated is the forward of oracle/sla.py for one head with the block
mask held fixed:

    O = O_s + O_l W_proj
    O_s[t] = softmax_j(q_t . k_j / sqrt(d)) v_j        over the critical keys of t's block
    O_l[t] = phi(q_t) H_i / (phi(q_t) . Z_i)           H_i = sum phi(k)^T v, Z_i = sum phi(k)
                                                       over the marginal keys of block i

Readings:

1. The classification is a ranking of pooled scores: piecewise constant in Q and K,
   so the mask carries no gradient.  The gradients are those of the forward with
   the mask as given (the same convention as any block-sparse attention trained
   with a selected mask).
2. The sparse part's gradient is the exact gradient of softmax attention over the
   kept keys: with P the attention weights, dV = P^T dO_s, dP = dO_s V^T,
   dS = P * (dP - rowsum(dO_s * O_s)), dQ = dS K / sqrt(d), dK = dS^T Q / sqrt(d)
   (the quantities a FlashAttention backward forms tile by tile).
3. The linear part's gradient is that of the normalised form of reading 4 of
   oracle/sla.py, through phi = elu + 1 (derivative 1 above 0, exp(x) at or below)
   or the channel softmax (y * (dy - dy . y)); a query block with no marginal key
   block gives no gradient.
4. W_proj gets dW = O_l^T dO; pad tokens get zero gradients.

Parity status: pinned (tests/test_oracle_sla_grad.py) -- directional finite
differences of the pinned forward of oracle/sla.py for q, k, v and W_proj with both
feature maps, and the all-critical case against torch autograd through
scaled_dot_product_attention.
"""
from __future__ import annotations

import math

import numpy as np

from .sla import BLOCK, phi_elu1, phi_softmax, row_softmax


def sparse_attention_backward(q, k, v, valid, key_blocks, d_out, block: int = BLOCK):
    """Gradients (dq, dk, dv) of ``sla.block_sparse_attention`` for the upstream
    gradient ``d_out`` of its output, the key-block sets held fixed (readings 1, 2)."""
    n, d = q.shape
    nb = n // block
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    for i in range(nb):
        qrows = np.arange(i * block, (i + 1) * block)
        qrows = qrows[valid[qrows]]
        blocks = np.unique(np.asarray(key_blocks[i], dtype=np.int64))
        keys = (blocks[:, None] * block + np.arange(block)[None, :]).reshape(-1)
        keys = keys[valid[keys]] if keys.size else keys
        if keys.size == 0 or qrows.size == 0:
            continue
        p = row_softmax((q[qrows] @ k[keys].T) * scale)
        o = p @ v[keys]
        do = d_out[qrows]
        dv[keys] += p.T @ do
        dp = do @ v[keys].T
        ds = p * (dp - (do * o).sum(axis=1, keepdims=True))
        dq[qrows] += (ds @ k[keys]) * scale
        dk[keys] += (ds.T @ q[qrows]) * scale
    return dq, dk, dv


def _phi(x, phi):
    return phi_elu1(x) if phi == "elu1" else phi_softmax(x)


def _phi_vjp(x, y, dy, phi):
    """x -> y = phi(x): the gradient with respect to x for the gradient dy of y."""
    if phi == "elu1":
        return dy * np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))
    return y * (dy - (dy * y).sum(axis=-1, keepdims=True))


def linear_attention_backward(q, k, v, valid, marginal, d_out_l, block: int = BLOCK, phi: str = "elu1"):
    """Gradients (dq, dk, dv) of ``sla.linear_attention`` for the upstream gradient
    ``d_out_l`` of O_l, with ``marginal`` [Nb, Nb] (True = marginal) held fixed (reading 3)."""
    n, d = q.shape
    nb = n // block
    fq = _phi(q, phi) * valid[:, None]
    fk = _phi(k, phi) * valid[:, None]
    vv = v * valid[:, None]
    h = np.stack([fk[j * block:(j + 1) * block].T @ vv[j * block:(j + 1) * block] for j in range(nb)])
    z = np.stack([fk[j * block:(j + 1) * block].sum(axis=0) for j in range(nb)])
    dfq = np.zeros_like(fq)
    dH = np.zeros((nb, d, v.shape[1]))
    dZ = np.zeros((nb, d))
    for i in range(nb):
        js = np.nonzero(marginal[i])[0]
        if js.size == 0:
            continue
        H = h[js].sum(axis=0)
        Z = z[js].sum(axis=0)
        rows = np.arange(i * block, (i + 1) * block)
        rows = rows[valid[rows]]
        num = fq[rows] @ H                                  # [rows, dv]
        den = fq[rows] @ Z                                  # [rows]
        o = num / den[:, None]
        do = d_out_l[rows]
        dnum = do / den[:, None]
        dden = -(do * o).sum(axis=1) / den
        dfq[rows] = dnum @ H.T + dden[:, None] * Z[None, :]
        dHi = fq[rows].T @ dnum                             # [d, dv]
        dZi = (dden[:, None] * fq[rows]).sum(axis=0)        # [d]
        dH[js] += dHi[None]
        dZ[js] += dZi[None]
    dfk = np.zeros_like(fk)
    dv = np.zeros_like(vv)
    for j in range(nb):
        s = slice(j * block, (j + 1) * block)
        dfk[s] = vv[s] @ dH[j].T + dZ[j][None, :]
        dv[s] = fk[s] @ dH[j]
    dq = _phi_vjp(q, _phi(q, phi), dfq, phi) * valid[:, None]
    dk = _phi_vjp(k, _phi(k, phi), dfk, phi) * valid[:, None]
    return dq, dk, dv * valid[:, None]


def sla_head_backward(q, k, v, w_proj, valid, mask, d_out, block: int = BLOCK, phi: str = "elu1"):
    """Gradients of the SLA forward of one head, O = O_s + O_l W_proj, for the mask
    ``mask`` (1 critical, 0 marginal, -1 negligible) held fixed.  Returns a dict with
    dq, dk, dv and dw (reading 4)."""
    from .sla import linear_attention, lists_from_mask
    crit = lists_from_mask(mask, 1)
    marginal = mask == 0
    dq_s, dk_s, dv_s = sparse_attention_backward(q, k, v, valid, crit, d_out, block)
    d_out_l = d_out @ w_proj.T
    dq_l, dk_l, dv_l = linear_attention_backward(q, k, v, valid, marginal, d_out_l, block, phi)
    o_l = linear_attention(q, k, v, valid, marginal, block=block, phi=phi)
    return {"dq": dq_s + dq_l, "dk": dk_s + dk_l, "dv": dv_s + dv_l, "dw": o_l.T @ d_out}
