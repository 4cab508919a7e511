"""Python binding of libslr: block-sparse + linear video attention on B200.

A thin ctypes layer over the C ABI in ``include/slr.h``: it checks tensor
dtypes and shapes, allocates outputs and the scratch workspace with torch on the
tensors' device, and passes raw pointers plus torch's current CUDA stream.  All
arithmetic happens in the library's kernels; there is no fallback path, and a
missing ``libslr.so`` raises immediately.

Function names match the C entry points: ``slr_pool_classify``,
``slr_block_sparse_attn``, ``slr_linear_marginal``, ``slr_sparse_linear_attn``,
``slr_frame_mask_attn``, ``slr_svoo_cocluster`` and ``slr_svoo_attn``; host helpers ``slr_block_counts``,
``slr_lvsa_attention_sets``, ``slr_workspace_bytes`` and ``slr_check_status``.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libslr.so")

SLR_OK = 0
SLR_ERR_ARG = -1
SLR_ERR_UNSUPPORTED = -2
SLR_ERR_WORKSPACE = -3
SLR_ERR_CUDA = -4
SLR_ERR_TIMEOUT = -5
SLR_ERR_INDEX = -6

SLR_PHI_ELU1 = 0
SLR_PHI_SOFTMAX = 1
SLR_MASK_LVSA = 1
SLR_MASK_TILE3D = 2
SLR_MASK_STA = 3
ABI_VERSION = 201          # include/slr.h SLR_ABI_VERSION

SLR_OP_POOL_CLASSIFY = 1
SLR_OP_BLOCK_SPARSE = 2
SLR_OP_LINEAR_MARGINAL = 3
SLR_OP_SPARSE_LINEAR = 4
SLR_OP_FRAME_MASK = 5
SLR_OP_SVOO_COCLUSTER = 6
SLR_OP_SVOO_ATTN = 7

EXPORTS = (
    "slr_pool_classify", "slr_block_sparse_attn", "slr_linear_marginal", "slr_sparse_linear_attn",
    "slr_frame_mask_attn", "slr_workspace_bytes", "slr_check_status", "slr_block_counts",
    "slr_lvsa_attention_sets", "slr_status_string", "slr_version", "slr_profile_enable",
    "slr_profile_collect", "slr_block_sparse_attn_noalloc", "slr_svoo_cocluster", "slr_svoo_attn",
)


class SlrError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: status {code} ({status_string(code)})")
        self.code = code


class SlrSeq(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("block", ctypes.c_int),
                ("n_seg", ctypes.c_int), ("seg_len", ctypes.c_int), ("seg_stride", ctypes.c_int)]


class SlrMaskDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("T", ctypes.c_int), ("C", ctypes.c_int), ("W", ctypes.c_int),
                ("step", ctypes.c_int), ("F", ctypes.c_int), ("Hh", ctypes.c_int), ("Ww", ctypes.c_int),
                ("tile", ctypes.c_int * 3), ("radius", ctypes.c_int), ("cell", ctypes.c_int * 3),
                ("gate", ctypes.c_float), ("rope", ctypes.c_int), ("window", ctypes.c_int * 3)]


class SlrFracs(ctypes.Structure):
    _fields_ = [("crit_frac", ctypes.c_float), ("negl_frac", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libslr.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run block_sparse_linear_02_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        seqp, maskp = ctypes.POINTER(SlrSeq), ctypes.POINTER(SlrMaskDesc)
        L.slr_pool_classify.argtypes = [vp, vp, seqp, f, f, vp, vp, vp, vp, vp, sz, vp]
        L.slr_block_sparse_attn.argtypes = [vp, vp, vp, seqp, vp, vp, i, vp, vp, vp, sz, vp]
        L.slr_linear_marginal.argtypes = [vp, vp, vp, seqp, vp, i, vp, vp, vp, sz, vp]
        L.slr_sparse_linear_attn.argtypes = [vp, vp, vp, vp, seqp, f, f, i, vp, vp, vp, sz, vp]
        L.slr_frame_mask_attn.argtypes = [vp, vp, vp, seqp, maskp, vp, vp, sz, vp]
        L.slr_block_sparse_attn_noalloc.argtypes = [vp, vp, vp, seqp, vp, vp, i, vp, vp, vp, vp]
        L.slr_block_sparse_attn_noalloc.restype = i
        L.slr_svoo_cocluster.argtypes = [vp, vp, seqp, i, i, i, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.slr_svoo_attn.argtypes = [vp, vp, vp, seqp, vp, vp, f, vp, vp, vp, sz, vp]
        L.slr_workspace_bytes.argtypes = [i, seqp, vp]
        L.slr_workspace_bytes.restype = sz
        L.slr_check_status.argtypes = [vp, vp]
        L.slr_block_counts.argtypes = [i, f, f, ctypes.POINTER(i), ctypes.POINTER(i)]
        L.slr_lvsa_attention_sets.argtypes = [i, i, i, i, vp, vp, i]
        L.slr_status_string.argtypes = [i]
        L.slr_status_string.restype = ctypes.c_char_p
        L.slr_version.argtypes = []
        L.slr_profile_enable.argtypes = [i]
        L.slr_profile_enable.restype = i
        L.slr_profile_collect.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(i),
                                          ctypes.POINTER(ctypes.c_double), i]
        L.slr_profile_collect.restype = i
        for name in ("slr_pool_classify", "slr_block_sparse_attn", "slr_linear_marginal",
                     "slr_sparse_linear_attn", "slr_frame_mask_attn", "slr_check_status",
                     "slr_block_counts", "slr_lvsa_attention_sets", "slr_version", "slr_svoo_cocluster",
                     "slr_svoo_attn"):
            getattr(L, name).restype = i
        if L.slr_version() != ABI_VERSION:
            # the structs above mirror include/slr.h of this version; an older build would read them wrongly
            raise RuntimeError(f"{LIB_PATH} has ABI {L.slr_version()}, this binding expects {ABI_VERSION}; rebuild it")
        _lib = L
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().slr_status_string(code).decode()
    except RuntimeError:
        return "library not loaded"


def _check(code: int, what: str) -> None:
    if code != SLR_OK:
        raise SlrError(code, what)


# ------------------------------------------------------------------ descriptors

def make_seq(B: int, H: int, d: int, n_seg: int, seg_len: int, seg_stride: int) -> SlrSeq:
    return SlrSeq(B, H, d, 64, n_seg, seg_len, seg_stride)


def seq_from(q, n_seg: int = 1, seg_len: int | None = None, seg_stride: int | None = None) -> SlrSeq:
    """Sequence descriptor for q [B, H, N_pad, d]; default: one unpadded segment."""
    B, H, n, d = q.shape
    if seg_stride is None:
        seg_stride = n // n_seg
    if seg_len is None:
        seg_len = seg_stride
    return make_seq(B, H, d, n_seg, seg_len, seg_stride)


def lvsa_mask(T: int, C: int, W: int, step: int) -> SlrMaskDesc:
    m = SlrMaskDesc()
    m.kind, m.T, m.C, m.W, m.step = SLR_MASK_LVSA, T, C, W, step
    return m


def tile3d_mask(F: int, Hh: int, Ww: int, radius: int = 1, cell=(2, 16, 16), gate: float = 0.55,
                rope: bool = False) -> SlrMaskDesc:
    m = SlrMaskDesc()
    m.kind, m.F, m.Hh, m.Ww, m.radius, m.gate = SLR_MASK_TILE3D, F, Hh, Ww, radius, gate
    m.rope = 1 if rope else 0
    m.tile[:] = [4, 4, 4]
    m.cell[:] = list(cell)
    return m


def sta_mask(F: int, Hh: int, Ww: int, window=(12, 12, 12)) -> SlrMaskDesc:
    """Sliding tile attention over 4x4x4 tiles; window in tokens per axis (odd multiples of 4)."""
    m = SlrMaskDesc()
    m.kind, m.F, m.Hh, m.Ww = SLR_MASK_STA, F, Hh, Ww
    m.tile[:] = [4, 4, 4]
    m.window[:] = list(window)
    return m


# ------------------------------------------------------------------ host helpers

def slr_block_counts(n_kb: int, crit_frac: float, negl_frac: float) -> tuple[int, int]:
    kc, kn = ctypes.c_int(), ctypes.c_int()
    _check(lib().slr_block_counts(n_kb, crit_frac, negl_frac, ctypes.byref(kc), ctypes.byref(kn)),
           "slr_block_counts")
    return kc.value, kn.value


def slr_lvsa_attention_sets(T: int, C: int, W: int, step: int) -> list[list[int]]:
    cap = T
    sets = (ctypes.c_int32 * (T * cap))()
    cnt = (ctypes.c_int32 * T)()
    _check(lib().slr_lvsa_attention_sets(T, C, W, step, ctypes.cast(sets, ctypes.c_void_p),
                                         ctypes.cast(cnt, ctypes.c_void_p), cap), "slr_lvsa_attention_sets")
    return [list(sets[t * cap: t * cap + cnt[t]]) for t in range(T)]


def slr_profile_enable(on: bool) -> None:
    lib().slr_profile_enable(1 if on else 0)


def slr_profile_collect() -> dict:
    """{kernel name: (launches, total device ms)} since the last collect (synchronises)."""
    n = 32
    names = (ctypes.c_char_p * n)()
    launches = (ctypes.c_int * n)()
    ms = (ctypes.c_double * n)()
    k = lib().slr_profile_collect(names, launches, ms, n)
    return {names[i].decode(): (launches[i], ms[i]) for i in range(k)}


def slr_workspace_bytes(op: int, seq: SlrSeq, params=None) -> int:
    p = None if params is None else ctypes.cast(ctypes.pointer(params), ctypes.c_void_p)
    return int(lib().slr_workspace_bytes(op, ctypes.byref(seq), p))


# ------------------------------------------------------------------ device calls

def _stream(t):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class Workspace:
    """A reusable device scratch buffer (256-byte aligned, grown on demand)."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int, device):
        import torch
        if nbytes <= 0:
            raise SlrError(SLR_ERR_ARG, "slr_workspace_bytes rejected the arguments")
        if self.buf is None or self.buf.numel() < nbytes + 256 or self.buf.device != device:
            self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        off = (-base) % 256
        return ctypes.c_void_p(base + off), ctypes.c_size_t(self.buf.numel() - off)


_default_ws = {}


def _ws(ws, device):
    if ws is None:
        ws = _default_ws.setdefault(str(device), Workspace(device))
    return ws


def _check_qkv(*ts):
    import torch
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors [B, H, N_pad, d]")


def slr_check_noalloc_status(device=None) -> int:
    """Synchronise and return (and clear) the status word that
    slr_block_sparse_attn_noalloc writes into its static scratch when it is given
    no status tensor: slr_check_status(NULL, stream) in the C ABI."""
    import torch
    device = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(device):
        return lib().slr_check_status(None, ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream))


def slr_check_status(ws=None, device=None) -> int:
    """Synchronise and return the device status word of the default workspace."""
    import torch
    device = device or torch.device("cuda", torch.cuda.current_device())
    w = _ws(ws, device)
    if w.buf is None:
        return SLR_OK
    base = w.buf.data_ptr()
    return lib().slr_check_status(ctypes.c_void_p(base + (-base) % 256),
                                  ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream))


def slr_pool_classify(q, k, seq: SlrSeq, crit_frac: float, negl_frac: float, scores: bool = False, ws=None):
    """Returns (mask int8 [B,H,Nb,Nb], crit_idx int32 [B,H,Nb,kc], crit_cnt int32 [B,H,Nb], P_c or None)."""
    import torch
    _check_qkv(q, k)
    nb = seq.n_seg * seq.seg_stride // 64
    kc, _ = slr_block_counts(nb, crit_frac, negl_frac)
    dev = q.device
    mask = torch.empty(seq.B, seq.H, nb, nb, dtype=torch.int8, device=dev)
    crit = torch.empty(seq.B, seq.H, nb, kc, dtype=torch.int32, device=dev)
    cnt = torch.empty(seq.B, seq.H, nb, dtype=torch.int32, device=dev)
    sc = torch.empty(seq.B, seq.H, nb, nb, dtype=torch.float32, device=dev) if scores else None
    need = slr_workspace_bytes(SLR_OP_POOL_CLASSIFY, seq, SlrFracs(crit_frac, negl_frac))
    wp, wn = _ws(ws, dev).get(need, dev)
    _check(lib().slr_pool_classify(_ptr(q), _ptr(k), ctypes.byref(seq), crit_frac, negl_frac, _ptr(mask),
                                   _ptr(crit), _ptr(cnt), _ptr(sc), wp, wn, _stream(q)), "slr_pool_classify")
    return mask, crit, cnt, sc


def slr_block_sparse_attn(q, k, v, seq: SlrSeq, kv_idx=None, kv_cnt=None, out=None, lse: bool = False, ws=None):
    """Exact softmax attention over per-query-block key-block sets; kv_idx None = dense. Returns (o, lse)."""
    import torch
    _check_qkv(q, k, v)
    dev = q.device
    o = torch.empty_like(q) if out is None else out
    l = torch.empty(q.shape[:3], dtype=torch.float32, device=dev) if lse else None
    kv_max = 0
    if kv_idx is not None:
        if kv_idx.dtype != torch.int32 or kv_cnt is None or kv_cnt.dtype != torch.int32:
            raise ValueError("kv_idx and kv_cnt must be int32")
        kv_idx, kv_cnt = kv_idx.contiguous(), kv_cnt.contiguous()
        kv_max = kv_idx.shape[-1]
    km = ctypes.c_int(kv_max if kv_idx is not None else seq.n_seg * seq.seg_stride // 64)
    need = slr_workspace_bytes(SLR_OP_BLOCK_SPARSE, seq, km)
    wp, wn = _ws(ws, dev).get(need, dev)
    _check(lib().slr_block_sparse_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(seq), _ptr(kv_idx), _ptr(kv_cnt),
                                       kv_max, _ptr(o), _ptr(l), wp, wn, _stream(q)), "slr_block_sparse_attn")
    return o, l


def slr_linear_marginal(q, k, v, seq: SlrSeq, mask, w_proj=None, out=None, ws=None, phi: int = SLR_PHI_ELU1):
    """Linear attention over the marginal (mask == 0) key blocks, optionally times W_proj; fp32 output."""
    import torch
    _check_qkv(q, k, v)
    dev = q.device
    o = torch.empty(q.shape, dtype=torch.float32, device=dev) if out is None else out
    if w_proj is not None:
        _check_qkv(w_proj)
    need = slr_workspace_bytes(SLR_OP_LINEAR_MARGINAL, seq, None)
    wp, wn = _ws(ws, dev).get(need, dev)
    _check(lib().slr_linear_marginal(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(seq), _ptr(mask.contiguous()),
                                     phi, _ptr(w_proj), _ptr(o), wp, wn, _stream(q)),
           "slr_linear_marginal")
    return o


def slr_sparse_linear_attn(q, k, v, w_proj, seq: SlrSeq, crit_frac: float, negl_frac: float,
                           out=None, mask_out: bool = False, ws=None, phi: int = SLR_PHI_ELU1):
    """The full SLA forward; returns (out bf16, mask int8 or None)."""
    import torch
    _check_qkv(q, k, v)
    dev = q.device
    o = torch.empty_like(q) if out is None else out
    nb = seq.n_seg * seq.seg_stride // 64
    m = torch.empty(seq.B, seq.H, nb, nb, dtype=torch.int8, device=dev) if mask_out else None
    need = slr_workspace_bytes(SLR_OP_SPARSE_LINEAR, seq, SlrFracs(crit_frac, negl_frac))
    wp, wn = _ws(ws, dev).get(need, dev)
    _check(lib().slr_sparse_linear_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(w_proj), ctypes.byref(seq), crit_frac,
                                        negl_frac, phi, _ptr(o), _ptr(m), wp, wn, _stream(q)),
           "slr_sparse_linear_attn")
    return o, m


def slr_frame_mask_attn(q, k, v, seq: SlrSeq, mask: SlrMaskDesc, out=None, ws=None):
    """Attention under an LVSA frame mask or the gated tile neighbourhood + far field."""
    import torch
    _check_qkv(q, k, v)
    dev = q.device
    o = torch.empty_like(q) if out is None else out
    need = slr_workspace_bytes(SLR_OP_FRAME_MASK, seq, mask)
    wp, wn = _ws(ws, dev).get(need, dev)
    _check(lib().slr_frame_mask_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(seq), ctypes.byref(mask), _ptr(o),
                                     wp, wn, _stream(q)), "slr_frame_mask_attn")
    return o


def slr_block_sparse_attn_noalloc(q, k, v, seq: SlrSeq, kv_idx=None, kv_cnt=None, out=None, lse: bool = False,
                                  status=None):
    """slr_block_sparse_attn without a workspace (static device scratch); returns (o, lse).

    ``status``: optional int32 CUDA tensor of one element that receives the device status;
    without it the status lands in the static scratch and slr_check_noalloc_status()
    reads it.  Outputs are allocated here only when not given; the library call itself
    allocates nothing.
    """
    import torch
    _check_qkv(q, k, v)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if lse else None
    kv_max = 0
    if kv_idx is not None:
        kv_idx, kv_cnt = kv_idx.contiguous(), kv_cnt.contiguous()
        kv_max = kv_idx.shape[-1]
    _check(lib().slr_block_sparse_attn_noalloc(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(seq), _ptr(kv_idx),
                                               _ptr(kv_cnt), kv_max, _ptr(o), _ptr(l), _ptr(status), _stream(q)),
           "slr_block_sparse_attn_noalloc")
    return o, l


def slr_svoo_cocluster(q, k, seq: SlrSeq, q_anchor, k_anchor, iters: int = 2, ws=None):
    """SVOO's bidirectional co-clustering from anchor tokens (int32 [B, H, n_qc] and
    [B, H, n_kc]); returns (q_label, k_label, q_perm, k_perm), each int32 [B, H, N_pad]."""
    import torch
    _check_qkv(q, k)
    for a in (q_anchor, k_anchor):
        if a.dtype != torch.int32 or not a.is_cuda or a.dim() != 3 or tuple(a.shape[:2]) != (seq.B, seq.H):
            raise ValueError("anchors must be int32 CUDA tensors [B, H, clusters]")
    q_anchor, k_anchor = q_anchor.contiguous(), k_anchor.contiguous()
    n_qc, n_kc = q_anchor.shape[-1], k_anchor.shape[-1]
    dev = q.device
    shape = (seq.B, seq.H, seq.n_seg * seq.seg_stride)
    ql, kl, qp, kp = (torch.empty(shape, dtype=torch.int32, device=dev) for _ in range(4))
    need = slr_workspace_bytes(SLR_OP_SVOO_COCLUSTER, seq, (ctypes.c_int * 2)(n_qc, n_kc))
    wp, wn = _ws(ws, dev).get(need, dev)
    _check(lib().slr_svoo_cocluster(_ptr(q), _ptr(k), ctypes.byref(seq), n_qc, n_kc, iters, _ptr(q_anchor),
                                    _ptr(k_anchor), _ptr(ql), _ptr(kl), _ptr(qp), _ptr(kp), wp, wn, _stream(q)),
           "slr_svoo_cocluster")
    return ql, kl, qp, kp


def slr_svoo_attn(q, k, v, seq: SlrSeq, q_perm, k_perm, keep_frac: float, out=None, mask_out: bool = False,
                  ws=None):
    """Attention over the top keep_frac of the key blocks of the co-clustered orders
    (int32 [B, H, N_pad] permutations); returns (out bf16 in token order, mask int8 or None)."""
    import torch
    _check_qkv(q, k, v)
    for p_ in (q_perm, k_perm):
        if p_.dtype != torch.int32 or not p_.is_cuda or tuple(p_.shape) != tuple(q.shape[:3]):
            raise ValueError("permutations must be int32 CUDA tensors [B, H, N_pad]")
    q_perm, k_perm = q_perm.contiguous(), k_perm.contiguous()
    dev = q.device
    o = torch.empty_like(q) if out is None else out
    nb = seq.n_seg * seq.seg_stride // 64
    m = torch.empty(seq.B, seq.H, nb, nb, dtype=torch.int8, device=dev) if mask_out else None
    need = slr_workspace_bytes(SLR_OP_SVOO_ATTN, seq, ctypes.c_float(keep_frac))
    wp, wn = _ws(ws, dev).get(need, dev)
    _check(lib().slr_svoo_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(seq), _ptr(q_perm), _ptr(k_perm),
                               keep_frac, _ptr(o), _ptr(m), wp, wn, _stream(q)), "slr_svoo_attn")
    return o, m
