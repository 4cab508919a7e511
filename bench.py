"""Benchmark of the SLA hot path on B200: ms per slr_sparse_linear_attn call.

Default workload: the Wan2.1-1.3B-shaped attention layer (12 heads, d = 128,
21 frames x 30 x 52 = 32,760 tokens padded to 32,768, frame-correlated bf16
inputs, 5 % critical / 10 % negligible, phi = elu + 1, W_proj ~ N(0, 1/d)).
One step = one full call: pooling, fp64 scores and classification, critical
lists, the linear branch (key states, mask-weighted contraction, apply and
projection) and the block-sparse flash attention with the projected linear
output added.

Printed (rank 0, one JSON line): the device-timed ms per call (inputs resident
in HBM, CUDA events on the call's stream, max over ranks), effective TFLOPS on
computed blocks, speedup over the library's own dense mode, the end-to-end
time through host buffers, the roofline of the dominant kernel (timed live
with the library's per-kernel event profiler), SM clocks sampled during the
timed region, and the fp64 CPU oracle timed on a bounded sample.

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


def measured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None when
    the kernel's source has changed since those counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["sha256"]:
            return None
    return rec["dram_bytes_per_launch"]


def config_dict(w):
    return {
        "workload": (f"{w.name}: SLA layer B={w.batch} H={w.heads} d={w.d} N={w.n_pad} "
                     f"({w.n_valid} valid, {w.frames} frames of {w.fh}x{w.fw}), block 64, "
                     f"{int(w.crit_frac * 100)}% critical / {int(w.negl_frac * 100)}% negligible, phi=elu+1"),
        "global_batch": w.batch,
        "seq_len": w.n_pad,
        "heads": w.heads,
        "head_dim": w.d,
        "l2_policy": "inputs 3 x %.0f MB bf16 > 126 MB L2; no flush between steps" % (w.n_pad * w.d * 2 * w.heads / 1e6),
    }


def sla_flops(w, kc, kn):
    """Algorithmic FLOPs of one call on computed blocks."""
    nb = w.n_blocks
    BH = w.batch * w.heads
    d = w.d
    crit = 4.0 * 64 * 64 * d * nb * kc * BH                        # QK^T and PV per critical pair
    km = nb - kc - kn
    contraction = 2.0 * nb * nb * (d + 1) * d * BH if km > 0 else 0.0   # H = M01 h
    precompute = 2.0 * 64 * d * d * nb * BH                         # h_j = phi(K_j)^T V_j
    apply = 2.0 * 64 * d * d * nb * BH * 2                          # phi(Q)H and the W_proj product
    return crit, contraction + precompute + apply


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

    def start(self):
        try:
            os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
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


# ------------------------------------------------------------------ CPU oracle sample

def cpu_oracle_sample(w, q, k, v, wp, rows_per_head=256, heads=12):
    """Time the fp64 oracle on `heads` heads: full classification + `rows_per_head` query blocks.

    Returns (extrapolated ms per full call, description, threads).
    """
    from oracle import sla as osla
    valid = osla.valid_tokens(w.n_seg, w.seg_len, w.seg_stride)
    nb = w.n_blocks
    rng = np.random.default_rng(0)
    rows = sorted(rng.choice(nb, rows_per_head, replace=False).tolist())
    wp64 = wp.float().double().numpy()
    fixed, per_rows = 0.0, 0.0
    for h in range(heads):
        qh, kh, vh = (x[0, h].float().double().numpy() for x in (q, k, v))
        t0 = time.perf_counter()
        qbar = osla.pool_blocks(qh, valid)
        kbar = osla.pool_blocks(kh, valid)
        lg = osla.block_logits(qbar, kbar)
        kc, kn = osla.block_counts(nb, w.crit_frac, w.negl_frac)
        mask = osla.classify(lg, kc, kn)
        hs, zs = osla.key_block_states(kh, vh, valid)
        t1 = time.perf_counter()
        crit = osla.lists_from_mask(mask, 1)
        osla.block_sparse_attention(qh, kh, vh, valid, crit, rows=rows)
        marg = (mask == 0).astype(np.float64)
        for i in rows:
            H = np.tensordot(marg[i], hs, axes=(0, 0))
            Z = marg[i] @ zs
            t = np.arange(i * 64, (i + 1) * 64)
            t = t[valid[t]]
            fq = osla.phi_elu1(qh[t])
            ((fq @ H) / (fq @ Z)[:, None]) @ wp64
        t2 = time.perf_counter()
        fixed += t1 - t0
        per_rows += t2 - t1
    per_head = fixed / heads + (per_rows / heads) * (nb / rows_per_head)
    total_ms = per_head * w.heads * w.batch * 1e3
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        threads = 1
    desc = (f"{heads} of {w.heads} heads: pooling, fp64 logits, classification and key states in full, "
            f"sparse + linear outputs of {rows_per_head} of {nb} query blocks; extrapolated linearly to "
            f"{w.heads} heads x {nb} blocks (sample wall {fixed + per_rows:.1f} s)")
    return total_ms, desc, threads


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="slr", choices=["slr", "reference"])
    ap.add_argument("--workload", default=WORKLOAD.name, choices=sorted(workloads.BY_NAME))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-rows", type=int, default=256, help="query blocks per head in the CPU oracle sample")
    ap.add_argument("--oracle-heads", type=int, default=12, help="heads in the CPU oracle sample")
    args = ap.parse_args()
    w = workloads.BY_NAME[args.workload]
    if w.mode != "sla":
        raise SystemExit("bench.py times the SLA call; pick an SLA workload")
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
    q_h, k_h, v_h = workloads.make_qkv(w)
    wp_h = workloads.make_w_proj(w)
    q, k, v, wp = (x.to(dev) for x in (q_h, k_h, v_h, wp_h))
    seq = slr.make_seq(w.batch, w.heads, w.d, w.n_seg, w.seg_len, w.seg_stride)
    out = torch.empty_like(q)
    ws_sparse, ws_dense = slr.Workspace(dev), slr.Workspace(dev)
    stream = torch.cuda.current_stream(dev)

    def call(dense=False, o=out, qq=q, kk=k, vv=v):
        if dense:
            slr.slr_sparse_linear_attn(qq, kk, vv, None, seq, 1.0, 0.0, out=o, ws=ws_dense)
        else:
            slr.slr_sparse_linear_attn(qq, kk, vv, wp, seq, w.crit_frac, w.negl_frac, out=o, ws=ws_sparse)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(fn, steps):
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        barrier()
        return sdist.max_over_ranks(a.elapsed_time(b) / steps, device=dev)

    # warm-up (both modes)
    for _ in range(warmup):
        call()
        call(dense=True)
    torch.cuda.synchronize(dev)
    if slr.slr_check_status(ws_sparse, dev) != slr.SLR_OK:
        raise SystemExit("device status error during warm-up")

    # timed region 1: the sparse call (the metric); clocks are sampled from here
    # through the dense, profiled and end-to-end regions
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.25)
    ms_sparse = timed(call, args.steps)
    ms_dense = timed(lambda: call(dense=True), max(3, args.steps // 4))

    # timed region 2: the same steps with the per-kernel event profiler on
    slr.slr_profile_enable(True)
    slr.slr_profile_collect()
    ms_prof = timed(call, args.steps)
    prof = slr.slr_profile_collect()
    slr.slr_profile_enable(False)
    if slr.slr_check_status(ws_sparse, dev) != slr.SLR_OK:
        raise SystemExit("device status error during timing")

    kc, kn = slr.slr_block_counts(w.n_blocks, w.crit_frac, w.negl_frac)
    crit_fl, lin_fl = sla_flops(w, kc, kn)
    peaks, peak_src = load_peaks()
    peak_tf = peaks["bf16_tflops"]
    total_tf = (crit_fl + lin_fl) / (ms_sparse * 1e-3) / 1e12
    launches, attn_ms = prof.get("attention", (args.steps, float("nan")))
    attn_ms_per = attn_ms / max(1, launches)
    attn_tf = crit_fl / (attn_ms_per * 1e-3) / 1e12
    gpu_launches = sum(n for n, _ in prof.values())

    # end-to-end through host buffers
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hw = (x.pin_memory() for x in (q_h, k_h, v_h, wp_h))
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        dq, dk, dv, dw, do = (torch.empty_like(x, device=dev) for x in (q_h, k_h, v_h, wp_h, out))

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            dw.copy_(hw, non_blocking=True)
            slr.slr_sparse_linear_attn(dq, dk, dv, dw, seq, w.crit_frac, w.negl_frac, out=do, ws=ws_sparse)
            ho.copy_(do, non_blocking=True)

        for _ in range(2):
            e2e_step()
        e2e_ms = timed(e2e_step, max(3, args.steps // 4))
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hw))
        d2h = ho.numel() * ho.element_size()
        e2e = {"value": round(sdist.aggregate_ms_per_call(e2e_ms, world), 4), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    clk = clocks.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cms, desc, threads = cpu_oracle_sample(w, q_h, k_h, v_h, wp_h, rows_per_head=args.oracle_rows,
                                               heads=args.oracle_heads)
        cpu = {"value": round(cms, 1), "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "host_cpus": os.cpu_count()}

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(sdist.aggregate_ms_per_call(ms_sparse, world), 4),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": warmup,
            "ms_per_step": round(ms_sparse, 4),
            "higher_is_better": False,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded, frame-correlated bf16)",
            "config": config_dict(w),
            "tflops_computed_blocks": round(total_tf, 1),
            "tflops_pct_bf16_peak": round(100 * total_tf / peak_tf, 1),
            "dense_ms_per_call": round(ms_dense, 4),
            "speedup_vs_dense": round(ms_dense / ms_sparse, 2),
            "roofline": {
                "kernel": "attention (block-sparse flash attention, tcgen05)",
                "bound": "tensor",
                "achieved": round(attn_tf, 1),
                "peak": peak_tf,
                "unit": "TFLOP/s",
                "frac": round(attn_tf / peak_tf, 4),
                "peak_source": f"{peak_src} bf16 burst",
                "traffic": measured_traffic("attention"),
                "flops_per_launch": crit_fl,
                "ms_per_launch": round(attn_ms_per, 4),
            },
            "kernels": {k_: {"launches": n, "ms_per_launch": round(t / max(1, n), 4)} for k_, (n, t) in prof.items()},
            "profiled_ms_per_step": round(ms_prof, 4),
            "gpu_launches": gpu_launches,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
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
        cpu_oracle_sample(w, q, k, v, wp, rows_per_head=rows, heads=heads)
    vals = []
    desc, threads = "", 1
    for _ in range(max(1, min(args.steps, 3))):
        ms, desc, threads = cpu_oracle_sample(w, q, k, v, wp, rows_per_head=rows, heads=heads)
        vals.append(ms)
    val = statistics.median(vals)
    line = {
        "metric": METRIC, "value": round(val, 1), "unit": UNIT, "n_gpus": world, "steps": len(vals),
        "warmup": warmup, "ms_per_step": round(val, 1), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, frame-correlated bf16)",
        "config": config_dict(w), "impl": "reference",
        "cpu_baseline": {"value": round(val, 1), "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(val, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
