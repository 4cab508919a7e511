"""Shared helpers of the GPU parity tests (imported by tests/test_gpu_*.py).

Tolerances: masks are compared exactly, except that a disagreement is allowed
for a pair whose compressed score P_c lies within 1e-5 of its row's percentile
threshold; attention outputs on bf16 inputs with fp32 accumulation must be
within max-abs 2e-2 and RMS-relative 5e-3 of the fp64 oracle.
"""
from __future__ import annotations

import numpy as np
import torch

MAX_ABS = 2e-2
RMS_REL = 5e-3
BAND = 1e-5

# (test id, what, max-abs, rms-rel) of every output comparison, printed at the end of
# the session (tests/conftest.py) so that the margin to the tolerances is visible.
ERRORS: list = []


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).double().numpy()


def cuda(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda").contiguous()


def assert_close(out: np.ndarray, ref: np.ndarray, what: str = "", max_abs: float = MAX_ABS,
                 rms_rel: float = RMS_REL) -> tuple[float, float]:
    """max-abs and RMS-relative error of out vs ref (any matching shapes)."""
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = out - ref
    ma = float(np.abs(err).max()) if err.size else 0.0
    denom = float(np.sqrt(np.mean(ref * ref))) if ref.size else 1.0
    rr = float(np.sqrt(np.mean(err * err)) / max(denom, 1e-30)) if err.size else 0.0
    import os
    ERRORS.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], what, ma, rr))
    assert ma <= max_abs, f"{what}: max-abs {ma:.3e} > {max_abs}"
    assert rr <= rms_rel, f"{what}: rms-rel {rr:.3e} > {rms_rel}"
    return ma, rr


def rows_of_blocks(blocks, block: int = 64) -> np.ndarray:
    return np.concatenate([np.arange(b * block, (b + 1) * block) for b in blocks])


def check_mask(gpu: np.ndarray, ref: np.ndarray, p: np.ndarray, tau_c: np.ndarray, tau_n: np.ndarray,
               kc: int, kn: int) -> int:
    """Row counts exact; entries equal except inside the threshold band.  Returns #band flips."""
    assert ((gpu == 1).sum(axis=1) == kc).all()
    assert ((gpu == -1).sum(axis=1) == kn).all()
    diff = gpu != ref
    if not diff.any():
        return 0
    i, j = np.nonzero(diff)
    near = (np.abs(p[i, j] - tau_c[i]) <= BAND) | (np.abs(p[i, j] - tau_n[i]) <= BAND)
    assert near.all(), f"{(~near).sum()} mask disagreements outside the threshold band"
    return int(diff.sum())


def make_inputs(B: int, H: int, d: int, n_seg: int, seg_len: int, stride: int, seed: int, scale: float = 1.0):
    """Seeded bf16 q, k, v [B, H, n_seg*stride, d] on the CPU with zero pads."""
    from workloads import random_bf16
    n = n_seg * stride
    out = []
    valid = torch.from_numpy((np.arange(n) % stride) < seg_len)
    for w in range(3):
        x = random_bf16((B, H, n, d), seed * 10 + w, scale)
        x[:, :, ~valid] = 0
        out.append(x)
    return out


def valid_np(n_seg: int, seg_len: int, stride: int) -> np.ndarray:
    return (np.arange(n_seg * stride) % stride) < seg_len


def status_ok():
    import block_sparse_linear_02_b200 as slr
    torch.cuda.synchronize()
    assert slr.slr_check_status() == slr.SLR_OK
