"""Benchmark of the sparse video-attention hot path on B200: ms per attention call.

Headline workload (the JSON line's own fields): the Wan2.1-1.3B-shaped SLA layer
(12 heads, d = 128, 21 frames x 30 x 52 = 32,760 tokens padded to 32,768,
frame-correlated bf16 inputs, 5 % critical / 10 % negligible, phi = elu + 1,
W_proj ~ N(0, 1/d)).  One step = one full slr_sparse_linear_attn call: pooling
and the compressed scores (logits on the tensor cores from bf16 hi + lo pooled
means, fp32 accumulation), classification, critical lists, the linear branch
(key states, mask-weighted contraction, apply and projection) and the
block-sparse flash attention with the projected linear output added.

At one GPU the same run also measures the other workloads, each with its own
dense-mode comparison, roofline and bounded CPU-oracle sample, under
``other_configs``: the HunyuanVideo-shaped SLA layer (24 heads, 115,200
tokens), the LVSA frame mask (121 frames x 1,600 tokens, 12 heads, denoising
steps 0..3 in turn), the RoPeSLR-shaped gated tile neighbourhood + far field
(16 heads, 8 x 64 x 64 tokens), VORTA's sliding tile attention on the same
latent, and SVOO's co-clustering + attention over the top 20 % co-clustered block
pairs on the Wan-shaped layer.  ``--workload NAME`` makes that workload the
headline instead.

Printed (rank 0, one JSON line): the device-timed ms per call (inputs resident
in HBM, CUDA events on the call's stream, max over ranks) with the median and
minimum of the per-call times, effective TFLOPS on computed blocks, the
speed-up over the library's own dense mode, the end-to-end time through host
buffers, the roofline of the dominant kernel (timed live with the library's
per-kernel event profiler), SM clocks sampled during the timed regions, and the
fp64 CPU oracle timed on a bounded sample.

Multi-GPU: independent replicas (each rank runs the whole call on its own GPU;
the path has no exchange step).  ``value`` is then the max-over-ranks ms per
call divided by the number of ranks (aggregate time per call).

``--impl reference`` times the fp64 oracle on the host cores instead (rank 0
only), on a bounded sample of the same workload, extrapolated to a full call.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

WORKLOAD = workloads.WAN
OTHER_WORKLOADS = (workloads.HUNYUAN, workloads.LVSA, workloads.ROPESLR, workloads.STA, workloads.SVOO)
METRIC = "ms per sparse attn call & TFLOPS on computed blocks (% BF16 peak); speedup vs dense"
UNIT = "ms/call"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def measured_traffic(kernel: str, workload: str = "wan"):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary,
    or None when the kernel's source has changed since those counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        recs = json.load(f)
    rec = recs.get(f"{kernel}:{workload}")            # records are keyed kernel:workload
    if not rec or rec.get("workload") != workload:
        return None
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["sha256"]:
            return None
    return rec["dram_bytes_per_launch"]


def config_dict(w, phi="elu1"):
    if w.mode == "sla":
        desc = (f"{w.name}: SLA layer B={w.batch} H={w.heads} d={w.d} N={w.n_pad} "
                f"({w.n_valid} valid, {w.frames} frames of {w.fh}x{w.fw}), block 64, "
                f"{int(w.crit_frac * 100)}% critical / {int(w.negl_frac * 100)}% negligible, "
                + ("phi=elu+1" if phi == "elu1" else "phi=softmax over the channels"))
    elif w.mode == "lvsa":
        desc = (f"{w.name}: LVSA frame mask B={w.batch} H={w.heads} d={w.d} T={w.frames} frames of "
                f"{w.fh}x{w.fw}={w.seg_len} tokens padded to {w.seg_stride} (N={w.n_pad}), C={w.lvsa_C}, "
                f"W={w.lvsa_W}, denoising steps {list(w.lvsa_steps)} in turn, no linear branch")
    elif w.mode == "sta":
        desc = (f"{w.name}: sliding tile attention B={w.batch} H={w.heads} d={w.d} "
                f"{w.frames}x{w.fh}x{w.fw}={w.n_pad} tokens, 4x4x4 tiles, window "
                f"{w.window[0]}x{w.window[1]}x{w.window[2]} tokens")
    elif w.mode == "svoo":
        desc = (f"{w.name}: SVOO co-clustered block-sparse attention B={w.batch} H={w.heads} d={w.d} "
                f"N={w.n_pad} ({w.n_valid} valid, {w.frames} frames of {w.fh}x{w.fw}), {w.clusters[0]} query + "
                f"{w.clusters[1]} key clusters from sampled anchors, {w.iters} iterations, top "
                f"{int(round(w.keep_frac * 100))}% key blocks per query block; one call = co-clustering + attention")
    else:
        desc = (f"{w.name}: gated tile neighbourhood + far field B={w.batch} H={w.heads} d={w.d} "
                f"{w.frames}x{w.fh}x{w.fw}={w.n_pad} tokens, 4x4x4 tiles, 3x3x3 tile neighbourhood, "
                f"64 far tokens from {w.cell[0]}x{w.cell[1]}x{w.cell[2]} cells, gate {w.gate}"
                + (", 3-D RoPE on q and k" if w.rope else ""))
    bytes_in = w.n_pad * w.d * 2 * w.heads * w.batch
    return {
        "workload": desc,
        "global_batch": w.batch,
        "seq_len": w.n_pad,
        "heads": w.heads,
        "head_dim": w.d,
        "l2_policy": (f"inputs 3 x {bytes_in / 1e6:.0f} MB bf16 > 126 MB L2; no flush between steps"
                      if 3 * bytes_in > 126e6 * 2 else
                      "a 256 MB buffer is written between steps (L2 flush)"),
    }


def sla_flops(w, kc, kn):
    """Algorithmic FLOPs of one SLA call on computed blocks: (critical pairs, linear branch)."""
    nb = w.n_blocks
    BH = w.batch * w.heads
    d = w.d
    crit = 4.0 * 64 * 64 * d * nb * kc * BH                        # QK^T and PV per critical pair
    km = nb - kc - kn
    contraction = 2.0 * nb * nb * (d + 1) * d * BH if km > 0 else 0.0   # H = M01 h
    precompute = 2.0 * 64 * d * d * nb * BH                         # h_j = phi(K_j)^T V_j
    apply = 2.0 * 64 * d * d * nb * BH * 2                          # phi(Q)H and the W_proj product
    return crit, contraction + precompute + apply


def lvsa_flops(w, sets):
    """FLOPs of one LVSA call on computed blocks: 4*64*64*d per attended (query block,
    key block) pair of 64-token blocks, frame tails included (frames are 25 blocks)."""
    bpf = w.seg_stride // 64
    pairs = sum(bpf * len(A) * bpf for A in sets)
    return 4.0 * 64 * 64 * w.d * pairs * w.heads * w.batch


def tile3d_flops(w):
    """FLOPs of one gated tile call: 4*64*64*d per (query tile, neighbour tile) pair of the
    clipped (2r+1)^3 neighbourhood, plus one 64-token far block per query tile."""
    def extent_sum(n_tiles):
        return sum(min(t + w.radius, n_tiles - 1) - max(t - w.radius, 0) + 1 for t in range(n_tiles))
    tf, th, tw = w.frames // w.tile[0], w.fh // w.tile[1], w.fw // w.tile[2]
    pairs = extent_sum(tf) * extent_sum(th) * extent_sum(tw)
    far = tf * th * tw
    return 4.0 * 64 * 64 * w.d * (pairs + far) * w.heads * w.batch, pairs


def svoo_flops(w, kc):
    """FLOPs of one SVOO attention on computed blocks: 4*64*64*d per kept (query block,
    key block) pair, kc pairs per query block."""
    return 4.0 * 64 * 64 * w.d * w.n_blocks * kc * w.heads * w.batch


def sta_flops(w):
    """FLOPs of one sliding tile call: 4*64*64*d per (query tile, key tile) pair of the
    clipped window, the tile radius on each axis being (window / 4 - 1) / 2."""
    def extent_sum(n_tiles, r):
        return sum(min(t + r, n_tiles - 1) - max(t - r, 0) + 1 for t in range(n_tiles))
    rad = [(x // 4 - 1) // 2 for x in w.window]
    pairs = (extent_sum(w.frames // 4, rad[0]) * extent_sum(w.fh // 4, rad[1]) * extent_sum(w.fw // 4, rad[2]))
    return 4.0 * 64 * 64 * w.d * pairs * w.heads * w.batch, pairs


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples go to $SLR_CLOCKS_CSV when set, else to the temp directory
        self.path = os.environ.get("SLR_CLOCKS_CSV") or os.path.join(tempfile.gettempdir(),
                                                                      f"slr_clocks_rank{gpu_index}.csv")

    def start(self, append: bool = False):
        """Start sampling; append=True continues the log of an earlier start/pause."""
        try:
            os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
            self.f = open(self.path, "a" if append else "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            self.started = True
        except (OSError, FileNotFoundError):
            self.proc = None

    def pause(self):
        """Stop sampling (between timed regions) without summarising."""
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        self.proc = None

    def stop(self):
        """Stop sampling and summarise every sample taken since the first start."""
        if self.proc is not None:
            self.pause()
        elif not getattr(self, "started", False):
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle samples

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return 1


def cpu_oracle_sample(w, q, k, v, wp, rows_per_head=256, heads=12, phi="elu1"):
    """Time the fp64 oracle on a bounded sample of workload `w` and extrapolate to a
    full call.  Only oracle functions run inside the timed spans.

    SLA: per sampled head, pooling, logits, classification in full, plus the sparse
    and linear outputs of `rows_per_head` query blocks.  LVSA: the attention sets in
    full plus `rows_per_head` query blocks per sampled head.  Tile mode: `rows_per_head`
    x 64 query tokens per sampled head.  Returns (ms per call, description, threads).
    """
    from oracle import lvsa as olvsa
    from oracle import sla as osla
    from oracle import sta as osta
    from oracle import svoo as osvoo
    from oracle import tile3d as otile
    heads = min(heads, w.heads)
    nb = w.n_blocks
    rows_per_head = min(rows_per_head, nb)
    rng = np.random.default_rng(0)
    rows = sorted(rng.choice(nb, rows_per_head, replace=False).tolist())
    f64 = lambda x: x.float().double().numpy()  # noqa: E731
    fixed, per_rows = 0.0, 0.0
    if w.mode == "sla":
        valid = osla.valid_tokens(w.n_seg, w.seg_len, w.seg_stride)
        wp64 = f64(wp)
        for h in range(heads):
            qh, kh, vh = (f64(x[0, h]) for x in (q, k, v))
            t0 = time.perf_counter()
            qbar = osla.pool_blocks(qh, valid)
            kbar = osla.pool_blocks(kh, valid)
            lg = osla.block_logits(qbar, kbar)
            osla.row_softmax(lg)
            kc, kn = osla.block_counts(nb, w.crit_frac, w.negl_frac)
            mask = osla.classify(lg, kc, kn)
            t1 = time.perf_counter()
            o_s = osla.block_sparse_attention(qh, kh, vh, valid, osla.lists_from_mask(mask, 1), rows=rows)
            o_l = osla.linear_attention(qh, kh, vh, valid, mask == 0, rows=rows, phi=phi)
            o_s + o_l @ wp64
            t2 = time.perf_counter()
            fixed += t1 - t0
            per_rows += t2 - t1
        what = (f"pooling, fp64 logits, P_c and classification in full, then block_sparse_attention "
                f"and linear_attention (key states over all blocks) for {rows_per_head} of {nb} query blocks")
    elif w.mode == "lvsa":
        step = w.lvsa_steps[0]
        for h in range(heads):
            qh, kh, vh = (f64(x[0, h]) for x in (q, k, v))
            t0 = time.perf_counter()
            sets = olvsa.attention_sets(w.frames, w.lvsa_C, w.lvsa_W, step)
            t1 = time.perf_counter()
            olvsa.frame_mask_attention(qh, kh, vh, w.n_seg, w.seg_len, w.seg_stride, sets, rows=rows)
            t2 = time.perf_counter()
            fixed += t1 - t0
            per_rows += t2 - t1
        what = (f"attention_sets in full, then frame_mask_attention for {rows_per_head} of {nb} query "
                f"blocks (step {step})")
    elif w.mode == "svoo":
        valid = osla.valid_tokens(w.n_seg, w.seg_len, w.seg_stride)
        qa, ka = workloads.make_anchors(w, "q", heads), workloads.make_anchors(w, "k", heads)
        for h in range(heads):
            qh, kh, vh = (f64(x[0, h]) for x in (q, k, v))
            t0 = time.perf_counter()
            ql, kl = osvoo.co_cluster(qh, kh, qa[0, h].numpy(), ka[0, h].numpy(), iters=w.iters, valid=valid)
            qp, kp = osvoo.cluster_order(ql, w.clusters[0]), osvoo.cluster_order(kl, w.clusters[1])
            mask, _ = osvoo.block_selection(qh[qp], kh[kp], valid, w.keep_frac)
            t1 = time.perf_counter()
            osvoo.svoo_attention(qh, kh, vh, qp, kp, w.keep_frac, valid=valid, rows=rows, mask=mask)
            t2 = time.perf_counter()
            fixed += t1 - t0
            per_rows += t2 - t1
        what = (f"co_cluster ({w.iters} iterations), cluster_order and block_selection in full, then "
                f"svoo_attention for {rows_per_head} of {nb} query blocks")
    elif w.mode == "sta":
        toks = sorted(rng.choice(w.n_pad, rows_per_head * 64, replace=False).tolist())
        for h in range(heads):
            qh, kh, vh = (f64(x[0, h]) for x in (q, k, v))
            t0 = time.perf_counter()
            osta.sliding_tile_attention(qh, kh, vh, w.frames, w.fh, w.fw, window=w.window, rows=toks)
            per_rows += time.perf_counter() - t0
        what = f"sliding_tile_attention for {rows_per_head * 64} of {w.n_pad} query tokens"
    else:
        toks = sorted(rng.choice(w.n_pad, rows_per_head * 64, replace=False).tolist())
        for h in range(heads):
            qh, kh, vh = (f64(x[0, h]) for x in (q, k, v))
            t0 = time.perf_counter()
            if w.rope:      # the rotation covers every token whatever the sample
                qh, kh = otile.rope_3d(qh, w.frames, w.fh, w.fw), otile.rope_3d(kh, w.frames, w.fh, w.fw)
            t1 = time.perf_counter()
            otile.gated_head(qh, kh, vh, w.frames, w.fh, w.fw, w.tile, w.radius, w.cell, w.gate, rows=toks)
            fixed += t1 - t0
            per_rows += time.perf_counter() - t1
        what = ((f"rope_3d of q and k in full, then " if w.rope else "")
                + f"gated_head (far-field pooling in full) for {rows_per_head * 64} of {w.n_pad} query tokens")
    per_head = fixed / heads + (per_rows / heads) * (nb / rows_per_head)
    total_ms = per_head * w.heads * w.batch * 1e3
    desc = (f"{heads} of {w.heads} heads: {what}; extrapolated linearly to {w.heads} heads x {nb} blocks "
            f"(sample wall {fixed + per_rows:.1f} s)")
    return total_ms, desc, _blas_threads()


# ------------------------------------------------------------------ one workload on the GPU

class Runner:
    """Inputs, calls and timing of one workload on this rank's GPU."""

    def __init__(self, w, slr, dev, dist, sdist, world, phi="elu1"):
        self.w, self.slr, self.dev, self.dist, self.sdist, self.world = w, slr, dev, dist, sdist, world
        self.phi = slr.SLR_PHI_SOFTMAX if phi == "softmax" else slr.SLR_PHI_ELU1
        self.q_h, self.k_h, self.v_h = workloads.make_qkv(w)
        self.wp_h = workloads.make_w_proj(w)
        self.q, self.k, self.v, self.wp = (x.to(dev) for x in (self.q_h, self.k_h, self.v_h, self.wp_h))
        self.seq = slr.make_seq(w.batch, w.heads, w.d, w.n_seg, w.seg_len, w.seg_stride)
        self.out = torch.empty_like(self.q)
        self.ws, self.ws_dense = slr.Workspace(dev), slr.Workspace(dev)
        self.stream = torch.cuda.current_stream(dev)
        self.flush = None
        if 3 * self.q.numel() * 2 <= 2 * 126e6:     # inputs fit in L2: flush between steps
            self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        if w.mode == "lvsa":
            self.masks = [slr.lvsa_mask(w.frames, w.lvsa_C, w.lvsa_W, s) for s in w.lvsa_steps]
        elif w.mode == "tile3d":
            self.masks = [slr.tile3d_mask(w.frames, w.fh, w.fw, w.radius, w.cell, w.gate, rope=w.rope)]
        elif w.mode == "sta":
            self.masks = [slr.sta_mask(w.frames, w.fh, w.fw, w.window)]
        elif w.mode == "svoo":
            self.qa_h, self.ka_h = workloads.make_anchors(w, "q"), workloads.make_anchors(w, "k")
            self.qa, self.ka = self.qa_h.to(dev), self.ka_h.to(dev)
            self.ws_cl = slr.Workspace(dev)

    def call(self, i=0, o=None, q=None, k=None, v=None, wp=None, ws=None, anchors=None):
        slr, w = self.slr, self.w
        o = self.out if o is None else o
        q, k, v = (self.q if q is None else q), (self.k if k is None else k), (self.v if v is None else v)
        ws = self.ws if ws is None else ws
        if w.mode == "sla":
            slr.slr_sparse_linear_attn(q, k, v, self.wp if wp is None else wp, self.seq, w.crit_frac, w.negl_frac,
                                       out=o, ws=ws, phi=self.phi)
        elif w.mode == "svoo":
            qa, ka = (self.qa, self.ka) if anchors is None else anchors
            _, _, qp, kp = slr.slr_svoo_cocluster(q, k, self.seq, qa, ka, iters=w.iters, ws=self.ws_cl)
            slr.slr_svoo_attn(q, k, v, self.seq, qp, kp, w.keep_frac, out=o, ws=ws)
        else:
            slr.slr_frame_mask_attn(q, k, v, self.seq, self.masks[i % len(self.masks)], out=o, ws=ws)

    def call_dense(self, i=0):
        if self.w.mode == "sla":
            self.slr.slr_sparse_linear_attn(self.q, self.k, self.v, None, self.seq, 1.0, 0.0, out=self.out,
                                            ws=self.ws_dense)
        else:
            self.slr.slr_block_sparse_attn(self.q, self.k, self.v, self.seq, out=self.out, ws=self.ws_dense)

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()
        torch.cuda.synchronize(self.dev)

    def timed(self, fn, steps):
        """(max-over-ranks mean ms per call over the bracketed region, median, min of the
        per-call event times of this rank)."""
        self.barrier()
        E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        a, b = E(), E()
        per = [(E(), E()) for _ in range(steps)]
        a.record(self.stream)
        flush_ms = 0.0
        for i in range(steps):
            if self.flush is not None:
                self.flush.fill_(i & 0xFF)
            per[i][0].record(self.stream)
            fn(i)
            per[i][1].record(self.stream)
        b.record(self.stream)
        self.barrier()
        ts = [x.elapsed_time(y) for x, y in per]
        if self.flush is not None:    # the flush writes are not part of the call
            flush_ms = a.elapsed_time(b) - sum(ts)
        total = (a.elapsed_time(b) - flush_ms) / steps
        return self.sdist.max_over_ranks(total, device=self.dev), statistics.median(ts), min(ts)

    def status_ok(self):
        ok = self.slr.slr_check_status(self.ws, self.dev) == self.slr.SLR_OK
        if self.w.mode == "svoo":
            ok = ok and self.slr.slr_check_status(self.ws_cl, self.dev) == self.slr.SLR_OK
        return ok

    def work(self):
        """(FLOPs of the dominant kernel per call, all FLOPs on computed blocks, details)."""
        w, slr = self.w, self.slr
        if w.mode == "sla":
            kc, kn = slr.slr_block_counts(w.n_blocks, w.crit_frac, w.negl_frac)
            crit, lin = sla_flops(w, kc, kn)
            return crit, crit + lin, {"kc": kc, "kn": kn, "critical_tflop": crit / 1e12,
                                      "linear_branch_tflop": lin / 1e12}
        if w.mode == "lvsa":
            fl = [lvsa_flops(w, slr.slr_lvsa_attention_sets(w.frames, w.lvsa_C, w.lvsa_W, s)) for s in w.lvsa_steps]
            f = sum(fl) / len(fl)
            return f, f, {"computed_tflop_per_step": [x / 1e12 for x in fl]}
        if w.mode == "sta":
            f, pairs = sta_flops(w)
            return f, f, {"tile_pairs_per_head": pairs, "computed_tflop": f / 1e12}
        if w.mode == "svoo":
            kc, _ = slr.slr_block_counts(w.n_blocks, w.keep_frac, 0.0)
            f = svoo_flops(w, kc)
            return f, f, {"kc": kc, "computed_tflop": f / 1e12, "clusters": list(w.clusters), "iters": w.iters}
        f, pairs = tile3d_flops(w)
        return f, f, {"local_tile_pairs_per_head": pairs, "computed_tflop": f / 1e12}

    def measure(self, steps, warmup, peaks, peak_src, with_e2e):
        slr, w = self.slr, self.w
        for i in range(warmup):
            self.call(i)
            self.call_dense(i)
        torch.cuda.synchronize(self.dev)
        if not self.status_ok():
            raise SystemExit(f"{w.name}: device status error during warm-up")
        ms, med, mn = self.timed(self.call, steps)
        dense_steps = max(3, steps // 2) if w.mode == "sla" and w.n_pad <= 65536 else 3
        ms_dense, med_dense, _ = self.timed(self.call_dense, dense_steps)
        slr.slr_profile_enable(True)
        slr.slr_profile_collect()
        ms_prof, _, _ = self.timed(self.call, steps)
        prof = slr.slr_profile_collect()
        slr.slr_profile_enable(False)
        if not self.status_ok():
            raise SystemExit(f"{w.name}: device status error during timing")
        dom_fl, all_fl, details = self.work()
        peak_tf = peaks["bf16_tflops"]
        launches, attn_ms = prof.get("attention", (steps, float("nan")))
        attn_ms_per = attn_ms / max(1, launches)
        attn_tf = dom_fl / (attn_ms_per * 1e-3) / 1e12
        total_tf = all_fl / (ms * 1e-3) / 1e12
        res = {
            "ms_per_call": round(ms, 4), "ms_median": round(med, 4), "ms_min": round(mn, 4),
            "tflops_computed_blocks": round(total_tf, 1),
            "tflops_pct_bf16_peak": round(100 * total_tf / peak_tf, 1),
            "dense_ms_per_call": round(ms_dense, 4), "dense_ms_median": round(med_dense, 4),
            "speedup_vs_dense": round(ms_dense / ms, 2),
            "speedup_vs_dense_median": round(med_dense / med, 2),
            "roofline": {
                "kernel": "attention (block-sparse flash attention, tcgen05)",
                "bound": "tensor",
                "achieved": round(attn_tf, 1),
                "peak": peak_tf,
                "unit": "TFLOP/s",
                "frac": round(attn_tf / peak_tf, 4),
                "peak_source": f"{peak_src} bf16 burst",
                "traffic": measured_traffic("attention", w.name),
                "flops_per_launch": dom_fl,
                "ms_per_launch": round(attn_ms_per, 4),
            },
            "work": details,
            "kernels": {k_: {"launches": n, "ms_per_launch": round(t / max(1, n), 4)} for k_, (n, t) in prof.items()},
            "profiled_ms_per_step": round(ms_prof, 4),
            "gpu_launches": sum(n for n, _ in prof.values()),
        }
        if with_e2e:
            res["e2e"] = self.e2e(steps)
        return res

    def e2e(self, steps):
        """The same call through host buffers: pinned host -> device copies of the
        inputs, the call, and the device -> host copy of the output, every step."""
        hq, hk, hv, hw = (x.pin_memory() for x in (self.q_h, self.k_h, self.v_h, self.wp_h))
        ho = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        dq, dk, dv, dw, do = (torch.empty_like(x, device=self.dev) for x in (self.q_h, self.k_h, self.v_h,
                                                                               self.wp_h, self.out))
        sla = self.w.mode == "sla"
        svoo = self.w.mode == "svoo"
        if svoo:     # the sampled anchor tokens are inputs of the call too
            hqa, hka = self.qa_h.pin_memory(), self.ka_h.pin_memory()
            dqa, dka = torch.empty_like(hqa, device=self.dev), torch.empty_like(hka, device=self.dev)

        def step(i):
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            if sla:
                dw.copy_(hw, non_blocking=True)
            if svoo:
                dqa.copy_(hqa, non_blocking=True)
                dka.copy_(hka, non_blocking=True)
            self.call(i, o=do, q=dq, k=dk, v=dv, wp=dw, anchors=(dqa, dka) if svoo else None)
            ho.copy_(do, non_blocking=True)

        for i in range(2):
            step(i)
        ms, _, _ = self.timed(step, max(3, steps // 4))
        h2d = sum(x.numel() * x.element_size() for x in ((hq, hk, hv, hw) if sla else (hq, hk, hv)))
        if svoo:
            h2d += sum(x.numel() * x.element_size() for x in (hqa, hka))
        d2h = ho.numel() * ho.element_size()
        return {"value": round(self.sdist.aggregate_ms_per_call(ms, self.world), 4), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    def release(self):
        for name in ("q", "k", "v", "wp", "out", "flush", "ws", "ws_dense", "ws_cl", "qa", "ka"):
            setattr(self, name, None)
        torch.cuda.empty_cache()


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="slr", choices=["slr", "reference"])
    ap.add_argument("--workload", default=WORKLOAD.name, choices=sorted(workloads.BY_NAME))
    ap.add_argument("--others", default="auto", choices=["auto", "none"],
                    help="auto: at one GPU also measure the other workloads under other_configs")
    ap.add_argument("--phi", default="elu1", choices=["elu1", "softmax"],
                    help="feature map of the linear branch of the SLA workloads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-rows", type=int, default=None,
                    help="query blocks per head in the CPU oracle sample (default 256; 64 for svoo)")
    ap.add_argument("--oracle-heads", type=int, default=None,
                    help="heads in the CPU oracle sample (default 12; 2 for svoo, whose co-clustering runs in full)")
    args = ap.parse_args()
    w = workloads.BY_NAME[args.workload]
    small = w.mode == "svoo"
    args.oracle_rows = args.oracle_rows or (64 if small else 256)
    args.oracle_heads = args.oracle_heads or (2 if small else 12)
    warmup = max(3, args.warmup)

    from block_sparse_linear_02_b200 import dist as sdist
    rank, world, local = sdist.env_ranks()
    if world > 1 and args.impl == "slr":
        torch.cuda.set_device(local)
    dist = sdist.init("nccl" if args.impl == "slr" else "gloo", timeout_s=300)

    if args.impl == "reference":
        run_reference(args, w, rank, world, warmup)
        if dist is not None:
            dist.destroy_process_group()
        return

    import block_sparse_linear_02_b200 as slr
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()

    # SM clocks are sampled only while a workload's GPU regions run (not while the
    # host generates inputs or runs the oracle)
    clocks = ClockSampler(local)
    r = Runner(w, slr, dev, dist, sdist, world, phi=args.phi)
    clocks.start()
    time.sleep(0.25)
    res = r.measure(args.steps, warmup, peaks, peak_src, with_e2e=not args.no_e2e)
    clocks.pause()
    q_h, k_h, v_h, wp_h = r.q_h, r.k_h, r.v_h, r.wp_h
    r.release()
    others = []
    if world == 1 and args.others == "auto":
        for ow in OTHER_WORKLOADS:
            if ow.name == w.name:
                continue
            ro = Runner(ow, slr, dev, dist, sdist, world, phi=args.phi)
            clocks.start(append=True)
            time.sleep(0.25)
            o = ro.measure(args.steps, warmup, peaks, peak_src, with_e2e=False)
            clocks.pause()
            others.append((ow, {"config": config_dict(ow, args.phi), **o}))
            ro.release()
            del ro
    clk = clocks.stop()
    if rank == 0 and not args.no_cpu_baseline:
        for ow, o in others:
            rows = {"hunyuan": 16, "lvsa": 8, "ropeslr": 8, "sta": 8, "svoo": 16}.get(ow.name, 16)
            qo, ko, vo = workloads.make_qkv(ow, heads=2)
            cms, desc, threads = cpu_oracle_sample(ow, qo, ko, vo, workloads.make_w_proj(ow), rows_per_head=rows,
                                                   heads=2, phi=args.phi)
            o["cpu_baseline"] = {"value": round(cms, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                                 "sample": desc, "extrapolated": True}
    others = [o for _, o in others]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cms, desc, threads = cpu_oracle_sample(w, q_h, k_h, v_h, wp_h, rows_per_head=args.oracle_rows,
                                               heads=args.oracle_heads, phi=args.phi)
        cpu = {"value": round(cms, 1), "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "extrapolated": True, "host_cpus": os.cpu_count()}

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(sdist.aggregate_ms_per_call(res["ms_per_call"], world), 4),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": warmup,
            "ms_per_step": res["ms_per_call"],
            "ms_median": res["ms_median"],
            "ms_min": res["ms_min"],
            "higher_is_better": False,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded bf16; frame-correlated for the SLA workloads)",
            "config": config_dict(w, args.phi),
            **{k_: res[k_] for k_ in ("tflops_computed_blocks", "tflops_pct_bf16_peak", "dense_ms_per_call",
                                      "dense_ms_median", "speedup_vs_dense", "speedup_vs_dense_median",
                                      "roofline", "work", "kernels", "profiled_ms_per_step", "gpu_launches")},
            "clocks": clk,
            "e2e": res.get("e2e"),
            "cpu_baseline": cpu,
            "other_configs": others,
        }
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, w, rank, world, warmup):
    """The reference arm: the fp64 oracle on the host cores, bounded samples."""
    if rank != 0:
        return
    q, k, v = workloads.make_qkv(w)
    wp = workloads.make_w_proj(w)
    rows, heads = args.oracle_rows, args.oracle_heads
    for _ in range(min(warmup, 1)):
        cpu_oracle_sample(w, q, k, v, wp, rows_per_head=rows, heads=heads, phi=args.phi)
    vals = []
    desc, threads = "", 1
    for _ in range(max(1, min(args.steps, 3))):
        ms, desc, threads = cpu_oracle_sample(w, q, k, v, wp, rows_per_head=rows, heads=heads, phi=args.phi)
        vals.append(ms)
    val = statistics.median(vals)
    line = {
        "metric": METRIC, "value": round(val, 1), "unit": UNIT, "n_gpus": world, "steps": len(vals),
        "warmup": warmup, "ms_per_step": round(val, 1), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded bf16; frame-correlated for the SLA workloads)",
        "config": config_dict(w, args.phi), "impl": "reference",
        "cpu_baseline": {"value": round(val, 1), "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
                         "extrapolated": True},
        "e2e": {"value": round(val, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
