"""CPU tests of the C ABI: the library loads, exports every symbol include/slr.h
declares, its host-only helpers agree with the oracle, and argument errors are
rejected on the host before any CUDA call (no GPU is needed for these)."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_linear_02_b200 as slr
from oracle import lvsa as olvsa
from oracle import sla as osla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_symbols():
    text = open(os.path.join(ROOT, "include", "slr.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(slr_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(slr.LIB_PATH):
        from block_sparse_linear_02_b200 import build
        build.build()
    return slr.lib()


def test_exports_every_declared_symbol(lib):
    syms = _header_symbols()
    assert len(syms) >= 11
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(slr.EXPORTS)


def test_version_and_strings(lib):
    assert lib.slr_version() == 201            # the SVOO calls
    for code in range(0, -7, -1):
        assert slr.status_string(code) not in ("", "unknown status")


@pytest.mark.parametrize("nkb", [1, 2, 3, 4, 7, 64, 100, 512, 1800, 3025, 4096])
@pytest.mark.parametrize("fr", [(0.05, 0.10), (0.25, 0.25), (1.0, 0.0), (0.0, 0.0), (0.5, 0.5), (0.33, 0.2)])
def test_block_counts_match_oracle(lib, nkb, fr):
    assert slr.slr_block_counts(nkb, *fr) == osla.block_counts(nkb, *fr)


def test_block_counts_rejects_bad_fractions(lib):
    for fr in [(-0.1, 0.1), (0.5, 0.6), (1.5, 0.0), (float("nan"), 0.1)]:
        with pytest.raises(slr.SlrError):
            slr.slr_block_counts(100, *fr)


@pytest.mark.parametrize("T,C,W", [(121, 21, 3), (10, 6, 1), (9, 6, 1), (5, 6, 1), (37, 9, 2), (200, 30, 4),
                                   (4, 9, 1), (13, 8, 3), (3, 9, 2), (1, 5, 1), (64, 12, 2)])
def test_lvsa_sets_match_oracle(lib, T, C, W):
    tper = olvsa.global_period(T, C, W)
    for s in range(0, 2 * tper + 2):
        assert slr.slr_lvsa_attention_sets(T, C, W, s) == olvsa.attention_sets(T, C, W, s), (T, C, W, s)


def test_lvsa_sets_rejects_bad_budget(lib):
    with pytest.raises(slr.SlrError):
        slr.slr_lvsa_attention_sets(10, 3, 1, 0)     # C <= 2W+1


def test_workspace_bytes(lib):
    good = slr.make_seq(1, 12, 128, 1, 32760, 32768)
    n = slr.slr_workspace_bytes(slr.SLR_OP_SPARSE_LINEAR, good, slr.SlrFracs(0.05, 0.10))
    # at least h and H (bf16, (d+1)d per block per head)
    assert n >= 2 * 12 * 512 * 129 * 128 * 2
    dense = slr.slr_workspace_bytes(slr.SLR_OP_SPARSE_LINEAR, good, slr.SlrFracs(1.0, 0.0))
    assert 0 < dense <= 4096
    for bad in [slr.make_seq(1, 1, 96, 1, 64, 64),          # d unsupported
                slr.make_seq(1, 1, 64, 1, 60, 100),         # stride not a multiple of 64
                slr.make_seq(1, 1, 64, 1, 10, 128),         # a block with no valid token
                slr.make_seq(0, 1, 64, 1, 64, 64)]:
        assert slr.slr_workspace_bytes(slr.SLR_OP_SPARSE_LINEAR, bad, slr.SlrFracs(0.05, 0.1)) == 0
    m = slr.lvsa_mask(121, 21, 3, 0)
    assert slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, slr.make_seq(1, 12, 128, 121, 1560, 1600), m) > 0
    assert slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, slr.make_seq(1, 12, 128, 120, 1560, 1600), m) == 0
    t3 = slr.tile3d_mask(8, 64, 64)
    assert slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, slr.make_seq(1, 16, 128, 1, 32768, 32768), t3) > 0
    t3bad = slr.tile3d_mask(8, 64, 64, cell=(2, 8, 8))      # 256 cells, not 64
    assert slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, slr.make_seq(1, 16, 128, 1, 32768, 32768), t3bad) == 0
    # tile-major K and V (bf16 [B*H][N][d] each) live in the workspace; with the rotary
    # embedding the rotated q (raster order) does too
    seq3 = slr.make_seq(1, 16, 128, 1, 32768, 32768)
    plain = slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, seq3, t3)
    assert plain >= 2 * 16 * 32768 * 128 * 2
    roped = slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, seq3, slr.tile3d_mask(8, 64, 64, rope=True))
    assert roped - plain >= 16 * 32768 * 128 * 2
    t3bad = slr.tile3d_mask(8, 64, 64)
    t3bad.rope = 2
    assert slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, seq3, t3bad) == 0
    # sliding tile mask: lists only (no far field); windows must be odd numbers of 4-token tiles
    sta = slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, seq3, slr.sta_mask(8, 64, 64, (12, 20, 28)))
    assert 0 < sta < plain
    for bad in [(12, 16, 12), (10, 12, 12), (0, 12, 12), (12, 12, -4)]:
        assert slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, seq3, slr.sta_mask(8, 64, 64, bad)) == 0
    sta_rope = slr.sta_mask(8, 64, 64)
    sta_rope.rope = 1
    assert slr.slr_workspace_bytes(slr.SLR_OP_FRAME_MASK, seq3, sta_rope) == 0


def test_block_sparse_list_cap_clamps_without_overflow(lib):
    # the pair lists hold min(Nb, 2 kv_max) entries; 2 kv_max must not overflow int for huge kv_max
    seq = slr.make_seq(1, 2, 64, 1, 64 * 40, 64 * 40)
    full = slr.slr_workspace_bytes(slr.SLR_OP_BLOCK_SPARSE, seq, ctypes.c_int(40))
    for km in (2 ** 30 + 1, 2 ** 31 - 1):
        assert slr.slr_workspace_bytes(slr.SLR_OP_BLOCK_SPARSE, seq, ctypes.c_int(km)) == full
    assert 0 < slr.slr_workspace_bytes(slr.SLR_OP_BLOCK_SPARSE, seq, ctypes.c_int(3)) < full


def test_invalid_arguments_rejected_before_cuda(lib):
    seq = slr.make_seq(1, 1, 64, 1, 256, 256)
    vp = ctypes.c_void_p
    fake = vp(0x1000)           # never dereferenced: validation fails first
    ws = vp(0x100000)
    # null q
    assert lib.slr_block_sparse_attn(None, fake, fake, ctypes.byref(seq), None, None, 0, fake, None, ws, 1 << 20,
                                     None) == slr.SLR_ERR_ARG
    # misaligned output
    assert lib.slr_block_sparse_attn(fake, fake, fake, ctypes.byref(seq), None, None, 0, vp(0x1001), None, ws,
                                     1 << 20, None) == slr.SLR_ERR_ARG
    # workspace too small / misaligned
    assert lib.slr_block_sparse_attn(fake, fake, fake, ctypes.byref(seq), None, None, 0, fake, None, ws, 16,
                                     None) == slr.SLR_ERR_WORKSPACE
    assert lib.slr_block_sparse_attn(fake, fake, fake, ctypes.byref(seq), None, None, 0, fake, None, vp(0x100010),
                                     1 << 20, None) == slr.SLR_ERR_WORKSPACE
    # unsupported head size
    bad = slr.make_seq(1, 1, 32, 1, 256, 256)
    assert lib.slr_sparse_linear_attn(fake, fake, fake, fake, ctypes.byref(bad), 0.05, 0.1, 0, fake, None, ws,
                                      1 << 20, None) == slr.SLR_ERR_UNSUPPORTED
    # fractions that do not fit
    assert lib.slr_sparse_linear_attn(fake, fake, fake, fake, ctypes.byref(seq), 0.7, 0.5, 0, fake, None, ws,
                                      1 << 20, None) == slr.SLR_ERR_ARG
    # unknown feature map
    assert lib.slr_sparse_linear_attn(fake, fake, fake, fake, ctypes.byref(seq), 0.05, 0.1, 7, fake, None, ws,
                                      1 << 20, None) == slr.SLR_ERR_UNSUPPORTED
    # mask kind
    m = slr.SlrMaskDesc()
    m.kind = 9
    assert lib.slr_frame_mask_attn(fake, fake, fake, ctypes.byref(seq), ctypes.byref(m), fake, ws, 1 << 20,
                                   None) == slr.SLR_ERR_ARG
    # LVSA frame count must equal the number of segments
    m = slr.lvsa_mask(5, 6, 1, 0)
    assert lib.slr_frame_mask_attn(fake, fake, fake, ctypes.byref(seq), ctypes.byref(m), fake, ws, 1 << 20,
                                   None) == slr.SLR_ERR_ARG
    # the rotary embedding is defined for the tile neighbourhood only
    m = slr.lvsa_mask(1, 6, 1, 0)
    m.rope = 1
    assert lib.slr_frame_mask_attn(fake, fake, fake, ctypes.byref(seq), ctypes.byref(m), fake, ws, 1 << 20,
                                   None) == slr.SLR_ERR_UNSUPPORTED
    # linear branch needs a mask
    assert lib.slr_linear_marginal(fake, fake, fake, ctypes.byref(seq), None, 0, None, fake, ws, 1 << 20,
                                   None) == slr.SLR_ERR_ARG


def test_svoo_workspace_and_arguments(lib):
    seq = slr.make_seq(1, 12, 128, 1, 32760, 32768)
    cl = lambda a, b: (ctypes.c_int * 2)(a, b)
    n = slr.slr_workspace_bytes(slr.SLR_OP_SVOO_COCLUSTER, seq, cl(64, 64))
    # centres (fp32) and the metric (bf16, 3 terms) of up to 64 clusters, the sort counts
    assert 2 * 12 * 64 * 128 * 4 < n < 8 << 20
    for a, b in ((1, 64), (64, 129), (0, 0)):
        assert slr.slr_workspace_bytes(slr.SLR_OP_SVOO_COCLUSTER, seq, cl(a, b)) == 0
    two = slr.make_seq(1, 12, 128, 2, 16380, 16384)
    assert slr.slr_workspace_bytes(slr.SLR_OP_SVOO_COCLUSTER, two, cl(64, 64)) == 0
    rows = 12 * 32768 * 128 * 2
    dense = slr.slr_workspace_bytes(slr.SLR_OP_SVOO_ATTN, seq, ctypes.c_float(1.0))
    assert 4 * rows <= dense < 4 * rows + 4096          # the reordered q, k, v and output
    sparse = slr.slr_workspace_bytes(slr.SLR_OP_SVOO_ATTN, seq, ctypes.c_float(0.2))
    assert sparse > dense                                 # plus the classification and the lists
    for bad in (0.0, -0.5, 1.5, float("nan")):
        assert slr.slr_workspace_bytes(slr.SLR_OP_SVOO_ATTN, seq, ctypes.c_float(bad)) == 0
    vp = ctypes.c_void_p
    fake, ws = vp(0x1000), vp(0x100000)
    small = slr.make_seq(1, 1, 64, 1, 256, 256)
    args = lambda nq, nk, it, anc: (fake, fake, ctypes.byref(small), nq, nk, it, anc, anc, fake, fake, fake, fake,
                                    ws, 1 << 30, None)
    assert lib.slr_svoo_cocluster(*args(1, 4, 2, fake)) == slr.SLR_ERR_ARG
    assert lib.slr_svoo_cocluster(*args(4, 200, 2, fake)) == slr.SLR_ERR_ARG
    assert lib.slr_svoo_cocluster(*args(4, 4, 0, fake)) == slr.SLR_ERR_ARG
    assert lib.slr_svoo_cocluster(*args(4, 4, 2, None)) == slr.SLR_ERR_ARG
    assert lib.slr_svoo_cocluster(*args(4, 4, 2, fake)[:13], 16, None) == slr.SLR_ERR_WORKSPACE
    segs = slr.make_seq(1, 1, 64, 2, 128, 128)
    assert lib.slr_svoo_cocluster(fake, fake, ctypes.byref(segs), 4, 4, 2, fake, fake, fake, fake, fake, fake, ws,
                                  1 << 30, None) == slr.SLR_ERR_UNSUPPORTED
    for keep in (0.0, 1.25):
        assert lib.slr_svoo_attn(fake, fake, fake, ctypes.byref(small), fake, fake, keep, fake, None, ws, 1 << 30,
                                 None) == slr.SLR_ERR_ARG
    assert lib.slr_svoo_attn(fake, fake, fake, ctypes.byref(small), None, fake, 0.5, fake, None, ws, 1 << 30,
                             None) == slr.SLR_ERR_ARG
    assert lib.slr_svoo_attn(fake, fake, fake, ctypes.byref(segs), fake, fake, 0.5, fake, None, ws, 1 << 30,
                             None) == slr.SLR_ERR_UNSUPPORTED


def test_svoo_binding_rejects_host_tensors_and_bad_shapes(lib):
    import torch
    seq = slr.make_seq(1, 1, 64, 1, 256, 256)
    q = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16)
    anchors = torch.zeros(1, 1, 4, dtype=torch.int32)
    with pytest.raises(ValueError):           # host tensors never reach the library
        slr.slr_svoo_cocluster(q, q, seq, anchors, anchors)
    perm = torch.arange(256, dtype=torch.int32).reshape(1, 1, 256)
    with pytest.raises(ValueError):
        slr.slr_svoo_attn(q, q, q, seq, perm, perm, 0.5)
