"""Pins of the SLA backward oracle (oracle/sla_grad.py): directional finite
differences of the pinned forward of oracle/sla.py with the block mask held fixed,
and the all-critical case against torch autograd through SDPA."""
import numpy as np
import pytest
import torch

from oracle import sla as osla
from oracle import sla_grad as ograd


def _mask(rng, nb):
    """A fixed three-class mask: every row has a critical block; some rows have no marginal one."""
    m = rng.choice([1, 0, -1], size=(nb, nb), p=[0.3, 0.4, 0.3]).astype(np.int8)
    for i in range(nb):
        m[i, rng.integers(nb)] = 1
    m[1] = np.where(m[1] == 0, -1, m[1])            # row 1: critical and negligible only
    return m


def _forward(q, k, v, w, valid, mask, phi):
    o_s = osla.block_sparse_attention(q, k, v, valid, osla.lists_from_mask(mask, 1))
    o_l = osla.linear_attention(q, k, v, valid, mask == 0, phi=phi)
    return o_s + o_l @ w


@pytest.mark.parametrize("phi", ["elu1", "softmax"])
@pytest.mark.parametrize("seg_len", [256, 230])
def test_directional_finite_differences(phi, seg_len):
    rng = np.random.default_rng(3 if phi == "elu1" else 4)
    n, d, nb = 256, 16, 4
    valid = np.arange(n) < seg_len
    q, k, v = (rng.standard_normal((n, d)) * valid[:, None] for _ in range(3))
    w = rng.standard_normal((d, d)) / np.sqrt(d)
    mask = _mask(rng, nb)
    d_out = rng.standard_normal((n, d)) * valid[:, None]
    g = ograd.sla_head_backward(q, k, v, w, valid, mask, d_out, phi=phi)
    f = lambda q_, k_, v_, w_: float((d_out * _forward(q_, k_, v_, w_, valid, mask, phi)).sum())  # noqa: E731
    eps = 1e-5
    for name, idx in (("dq", 0), ("dk", 1), ("dv", 2), ("dw", 3)):
        for _ in range(3):
            args = [q, k, v, w]
            u = rng.standard_normal(args[idx].shape)
            if idx < 3:
                u *= valid[:, None]
            plus = list(args)
            minus = list(args)
            plus[idx] = args[idx] + eps * u
            minus[idx] = args[idx] - eps * u
            fd = (f(*plus) - f(*minus)) / (2 * eps)
            an = float((g[name] * u).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
    # pads get no gradient
    for name in ("dq", "dk", "dv"):
        assert not g[name][~valid].any()


def test_all_critical_equals_sdpa_autograd():
    gen = torch.Generator().manual_seed(7)
    n, d, nb = 192, 32, 3
    q, k, v = (torch.randn(n, d, generator=gen, dtype=torch.float64, requires_grad=True) for _ in range(3))
    d_out = torch.randn(n, d, generator=gen, dtype=torch.float64)
    o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0]
    o.backward(d_out)
    valid = np.ones(n, dtype=bool)
    dq, dk, dv = ograd.sparse_attention_backward(q.detach().numpy(), k.detach().numpy(), v.detach().numpy(), valid,
                                                 [range(nb)] * nb, d_out.numpy())
    for mine, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)


def test_linear_part_vanishes_without_marginal_blocks():
    rng = np.random.default_rng(11)
    n, d = 128, 8
    valid = np.ones(n, dtype=bool)
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    none = np.zeros((2, 2), dtype=bool)
    dq, dk, dv = ograd.linear_attention_backward(q, k, v, valid, none, rng.standard_normal((n, d)))
    assert not dq.any() and not dk.any() and not dv.any()
