#!/usr/bin/env python
"""Throughput of the SpargeAttn sparse-attention forward on B200.

One step = the whole hot path on one batch of synthetic input resident in HBM:
  [Hilbert table + permute Q, K, V]  (grid workloads only)
  stage 1  sparge_predict_pool        (block means, CosSim, INT8 codes: HBM bound)
           sparge_predict_select      (S_hat, TopCdf, fix rule, skip list)
  stage 2  sparge_attn_fwd           (fp16 V copy, tcgen05 attention)
  [inverse permute O]                (grid workloads only)
The default workload is the 128K causal GQA INT8 configuration
(B1, Hq32, Hkv8, N131072, d128, bf16 I/O).  The metric is dense-equivalent
TOPS = 4 N^2 d Hq (halved when causal) / step time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Multi-GPU (torchrun): every rank runs an independent replica of the workload
(weak scaling, no collective on the data path); the timed region is bracketed
by barriers and the max over ranks is reported.  --impl reference times the
CPU oracle on rank 0 on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import os
import re
import signal
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import get_workload, make_qkv  # noqa: E402

METRIC = "sparse-attn dense-equiv TOPS at N=128K causal; sparsity; % tensor-core peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0
L2_BYTES = 126e6  # B200 L2
ATTN_SRC = os.path.join(ROOT, "free_block_sparse_predict_b200", "csrc", "attn_sm100.cu")


def dense_equiv_ops(w) -> float:
    ops = 4.0 * w.N * w.N * w.d * w.Hq * w.B
    return ops / 2 if w.causal else ops


def pool_bytes(w) -> float:
    """Algorithmic HBM bytes of one predictor pooling stage: one read of Q and
    K, the block means and self-similarities written, and with INT8 the codes
    of Q and K and their block scales."""
    es = 2
    Tm, Tn = -(-w.N // w.bq), -(-w.N // w.bk)
    bq_, bk_ = w.B * w.Hq, w.B * w.Hkv
    b = (bq_ + bk_) * w.N * w.d * es + (bq_ * Tm + bk_ * Tn) * (w.d + 1) * 4
    if w.qk_int8:
        b += bq_ * w.N * w.d + bq_ * Tm * 4                       # Q codes, scales
        b += bk_ * w.N * w.d + bk_ * Tn * 4                       # K codes, scales
    return float(b)


def pool_extra_bytes(w) -> float:
    """Bytes the INT8 pooling stage moves beyond the algorithmic ones: the
    second read of K (the codes of K - kbar need kbar, a mean over all of K)
    and the float64 block sums that kbar is reduced from."""
    if not w.qk_int8:
        return 0.0
    Tn = -(-w.N // w.bk)
    bk_ = w.B * w.Hkv
    return float(bk_ * w.N * w.d * 2 + 2 * bk_ * Tn * w.d * 8)


def attn_peak_tflops(w, peaks, qk_blocks, pv_blocks, key="bf16_tflops_sustained"):
    """The tensor peak for the attention kernel's own mix of contractions: Q K^T
    in INT8 (twice the measured bf16 rate, the nominal dense ratio of the two)
    or in the I/O dtype, P~V in fp16 (the bf16 rate).  The flop-weighted
    harmonic mean: issued flops over the time they need at those peaks."""
    bf = float(peaks[key])
    qk_peak = 2.0 * bf if w.qk_int8 else bf
    tot = qk_blocks + pv_blocks
    if tot == 0:
        return bf
    return tot / (qk_blocks / qk_peak + pv_blocks / bf)


def workload_config(w, world, t_bytes):
    """The config object of the JSON line, shared by both arms."""
    return {"workload": f"{w.name}: B{w.B} Hq{w.Hq} Hkv{w.Hkv} N{w.N} d{w.d} "
                        f"{w.dtype} causal={int(w.causal)} int8_qk={int(w.qk_int8)} "
                        f"tau={w.tau} theta={w.theta} lambda={w.lam}",
            "global_batch": w.B * world, "seq_len": w.N,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (no flush)" if t_bytes > L2_BYTES
            else "inputs fit in L2: 256 MB rewritten, then 256 MB read, between "
                 "steps; steps timed alone"}


def fp32_peak_tflops(peaks) -> float:
    """FP32 FMA peak derived from the unit counts: 148 SMs x 128 FP32 lanes x
    2 flops x the measured maximum SM clock."""
    return 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def profiled_traffic(workload: str, seq_len: int, path=None):
    """dram bytes per attention launch from a committed ncu summary
    (profiles/attn_kernel_*.md, or the one file given) taken on the current
    kernel source and on this workload and length; None if there is none."""
    paths = [path] if path else sorted(glob.glob(os.path.join(ROOT, "profiles",
                                                             "attn_kernel_*.md")))
    cur = hashlib.sha256(open(ATTN_SRC, "rb").read()).hexdigest()
    for pth in paths:
        if not os.path.exists(pth):
            continue
        text = open(pth).read()
        m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
        h = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
        wl = re.search(r"dram_bytes_workload:\s*(\S+)\s+N=(\d+)", text)
        if not m or not h or not wl:
            continue
        if wl.group(1) == workload and int(wl.group(2)) == int(seq_len) and h.group(1) == cur:
            return float(m.group(1))
    return None


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity on one rank).  The
    tensor lives on `device` (the GPU for NCCL, None = CPU for gloo)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tops(world: int, ops_per_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's dense-equivalent ops over the
    slowest rank's time for the timed steps."""
    return world * ops_per_step * steps / (max_ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL, start_new_session=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        try:
            os.killpg(self.proc.pid, signal.SIGTERM)
        except ProcessLookupError:
            pass
        self.proc.wait(timeout=10)
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------
# native arm
# ----------------------------------------------------------------------------

def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import free_block_sparse_predict_b200 as fb

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = _workload(args)
    t = make_qkv(w, seed=0)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16

    def host(a):
        x = torch.from_numpy(a)
        return x.view(torch.bfloat16) if w.dtype == "bf16" else x

    q_h, k_h, v_h = (host(t[x]).pin_memory() for x in ("q", "k", "v"))
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    p = fb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.tau, w.theta, w.lam, causal=w.causal,
                       qk_int8=w.qk_int8, io_dtype=tdt)
    ws = fb.workspace(p, dev)
    mask, idx, cnt, sq_out, _ = fb.predict_outputs(p, dev)
    o = torch.empty(q.shape, dtype=tdt, device=dev)
    stats = torch.zeros(5, dtype=torch.int64, device=dev)
    perm = hws = None
    qp = kp = vp = op = None
    if w.grid:
        perm = torch.empty(w.N, dtype=torch.int32, device=dev)
        hws = torch.zeros(fb.sparge_hilbert_workspace_bytes(*w.grid), dtype=torch.uint8,
                          device=dev)
        qp, kp, vp, op = (torch.empty_like(x) for x in (q, k, v, o))
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    launches_per_step = 0

    def step(qs, ks, vs, os_, timing=None, prm=None):
        nonlocal launches_per_step
        prm = p if prm is None else prm
        n = 0
        if w.grid:
            fb.sparge_hilbert_index(w.N, w.prefix_len, *w.grid, perm, hws, stream)
            fb.sparge_hilbert_permute(qs, qp, perm, stream)
            fb.sparge_hilbert_permute(ks, kp, perm, stream)
            fb.sparge_hilbert_permute(vs, vp, perm, stream)
            qs, ks, vs, dst = qp, kp, vp, op
            n += 2 + 3
        else:
            dst = os_
        if timing:
            timing[0].record(stream)
        fb.sparge_predict_pool(prm, qs, ks, ws, stream)
        n += 4 if w.qk_int8 else 1
        if timing:
            timing[1].record(stream)
        fb.sparge_predict_select(prm, mask, idx, cnt, None, None, ws, stream)
        n += 1
        if timing:
            timing[2].record(stream)
        fb.sparge_attn_fwd(prm, qs, ks, vs, idx, cnt, dst, ws, stats, stream)
        n += 2 if w.dtype == "bf16" else 1
        if timing:
            timing[3].record(stream)
        if w.grid:
            fb.sparge_inverse_permute(op, os_, perm, stream)
            n += 1
        launches_per_step = n

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- device-resident timing
    for _ in range(args.warmup):
        step(q, k, v, o)
    torch.cuda.synchronize()
    stats.zero_()
    step(q, k, v, o)                       # one counted step for the work counters
    torch.cuda.synchronize()
    st = stats.cpu().numpy().astype(np.int64)
    if fb.sparge_device_status(ws) != 0:
        raise RuntimeError("device status reported an error")
    # the select stage's own work on this step's pooled statistics (untimed)
    fb.sparge_predict_select(p, mask, idx, cnt, sq_out, None, ws, stream)
    torch.cuda.synchronize()
    sel_work = select_work(w, sq_out.cpu().numpy(), int(cnt.sum()), w.theta)
    mask_h0 = mask[:, 0].cpu().numpy().astype(bool) if rank == 0 else None

    sampler = ClockSampler(_gpu_uuid(torch, dev)) if local_rank == 0 or world > 1 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    # inputs that fit in L2 would stay there from one step to the next: then a
    # 256 MB buffer is rewritten between steps and only the steps are timed.
    # A second 256 MB buffer is read after it, so that the flush's own dirty
    # lines are written back before the step starts instead of inside it.
    flush = flush_rd = None
    if _bytes(t) <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        flush_rd = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    e0, e1 = ev(), ev()
    per = [(ev(), ev(), ev(), ev()) for _ in range(args.steps)]
    span = [(ev(), ev()) for _ in range(args.steps)]
    e0.record(stream)
    for s in range(args.steps):
        if flush is not None:
            flush.fill_(s & 255)
            flush_rd.max()
        span[s][0].record(stream)
        step(q, k, v, o, per[s])
        span[s][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    ms_total = (e0.elapsed_time(e1) if flush is None
                else float(sum(a.elapsed_time(b) for a, b in span)))
    pool_ms = float(np.mean([a.elapsed_time(b) for (a, b, _, _) in per]))
    sel_ms = float(np.mean([a.elapsed_time(b) for (_, a, b, _) in per]))
    attn_ms = float(np.mean([a.elapsed_time(b) for (_, _, a, b) in per]))
    step_median_ms = float(np.median([a.elapsed_time(b) for a, b in span]))
    # grid workloads: Hilbert table + permutes of Q, K, V before the predictor,
    # inverse permute of O after the attention
    perm_ms = float(np.mean([sp[0].elapsed_time(pe[0]) for sp, pe in zip(span, per)]))
    inv_ms = float(np.mean([pe[3].elapsed_time(sp[1]) for sp, pe in zip(span, per)]))
    pred_ms = pool_ms + sel_ms
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / args.steps
    ops_step = dense_equiv_ops(w)
    value = aggregate_tops(world, ops_step, args.steps, ms_total)

    # ---- the same workload in a sparse regime: theta = -1 makes every block
    # selective and tau = 0.5 lets TopCdf drop blocks, so the skipping of Eq. 2
    # is what gets timed.  Reported beside the headline, never instead of it.
    sparse = None
    if not args.no_sparse_regime:
        ps = fb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, 0.5, -1.0, w.lam, causal=w.causal,
                            qk_int8=w.qk_int8, io_dtype=tdt)
        for _ in range(args.warmup):
            step(q, k, v, o, prm=ps)
        torch.cuda.synchronize()
        stats.zero_()
        step(q, k, v, o, prm=ps)
        torch.cuda.synchronize()
        sst = [int(x) for x in stats.cpu()]
        fb.sparge_predict_select(ps, mask, idx, cnt, sq_out, None, ws, stream)
        torch.cuda.synchronize()
        s_sel_work = select_work(w, sq_out.cpu().numpy(), int(cnt.sum()), -1.0)
        pk, _ = load_peaks()
        sper = [(ev(), ev(), ev(), ev()) for _ in range(args.steps)]
        sspan = [(ev(), ev()) for _ in range(args.steps)]
        for s_ in range(args.steps):
            if flush is not None:
                flush.fill_(s_ & 255)
                flush_rd.max()
            sspan[s_][0].record(stream)
            step(q, k, v, o, sper[s_], prm=ps)
            sspan[s_][1].record(stream)
        torch.cuda.synchronize()
        if fb.sparge_device_status(ws) != 0:
            raise RuntimeError("device status reported an error")
        s_step = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in sspan])), world, dev)
        s_attn = float(np.mean([a.elapsed_time(b) for (_, _, a, b) in sper]))
        s_pred = float(np.mean([a.elapsed_time(c) for (a, _, c, _) in sper]))
        s_sel = float(np.mean([b.elapsed_time(c) for (_, b, c, _) in sper]))
        vis = _visible_blocks(w)
        sparse = {
            "tau": 0.5, "theta": -1.0, "lambda": w.lam, "steps": args.steps,
            "value": round(aggregate_tops(world, dense_equiv_ops(w), 1, s_step), 3), "unit": "TOPS",
            "latency_ms": {"step": round(s_step, 4), "predict": round(s_pred, 4),
                           "predict_select": round(s_sel, 4), "attention": round(s_attn, 4)},
            "select_roofline": select_roofline(s_sel_work, s_sel, fp32_peak_tflops(pk),
                                               float(pk["hbm_gbs"])),
            "sparsity": {"mg": round(1.0 - sst[1] / vis, 6),
                         "pv_slices_skipped": round(sst[4] / max(1, sst[3] + sst[4]), 6),
                         "total": round(1.0 - (sst[1] + sst[3] / 4.0) / (2.0 * vis), 6)},
            "work": {"qk_blocks": sst[1], "pv_blocks": sst[2], "visible_blocks": vis},
            "attention_tflops": round((sst[1] + sst[2]) * 2.0 * w.bq * w.bk * w.d
                                      / (s_attn * 1e-3) / 1e12, 2),
            "what": "the same workload and step with theta = -1 (every block selective) and "
                    "tau = 0.5: TopCdf drops blocks, Q K^T and P~V are skipped for them "
                    "(Eq. 2); dense-equivalent TOPS over the step time; not the headline"}

    # ---- end to end through the public API with host buffers.  Every step
    # copies its inputs from pinned host memory and its output back, pipelined
    # as a serving loop would: two device buffer sets, the H2D copy of step s+1
    # and the D2H copy of step s on their own streams while step s computes.
    e2e = None
    if not args.no_e2e:
        cs_in, cs_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        bufs = [(q, k, v, o), tuple(torch.empty_like(x) for x in (q, k, v, o))]
        o_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]

        def run_e2e(nsteps):
            ready = [torch.cuda.Event() for _ in range(nsteps)]
            done = [torch.cuda.Event() for _ in range(nsteps)]
            out = [torch.cuda.Event() for _ in range(nsteps)]
            start, end = ev(), ev()
            start.record(stream)
            cs_in.wait_event(start)
            for s_ in range(nsteps):
                qb, kb, vb, ob = bufs[s_ % 2]
                with torch.cuda.stream(cs_in):
                    if s_ >= 2:
                        cs_in.wait_event(done[s_ - 2])      # step s-2 has read these
                    qb.copy_(q_h, non_blocking=True)
                    kb.copy_(k_h, non_blocking=True)
                    vb.copy_(v_h, non_blocking=True)
                    ready[s_].record(cs_in)
                stream.wait_event(ready[s_])
                if s_ >= 2:
                    stream.wait_event(out[s_ - 2])          # O of step s-2 is on the host
                step(qb, kb, vb, ob)
                done[s_].record(stream)
                with torch.cuda.stream(cs_out):
                    cs_out.wait_event(done[s_])
                    o_h[s_ % 2].copy_(ob, non_blocking=True)
                    out[s_].record(cs_out)
            stream.wait_event(out[nsteps - 1])
            end.record(stream)
            return start, end

        run_e2e(2)
        torch.cuda.synchronize()
        barrier()
        a, b = run_e2e(args.steps)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        nb = lambda x: x.numel() * x.element_size()
        e2e = {"value": round(aggregate_tops(world, ops_step, args.steps, e2e_ms), 3),
               "unit": "TOPS", "h2d_bytes_per_step": nb(q) + nb(k) + nb(v),
               "d2h_bytes_per_step": nb(o), "ms_per_step": round(e2e_ms / args.steps, 3),
               "pipelined": "H2D of step s+1 and D2H of step s overlap the compute of step s"}

    # ---- optional: the same step captured once into a CUDA graph and replayed
    graph_line = None
    if args.graph:
        from free_block_sparse_predict_b200.graph import SpargeGraph
        g = SpargeGraph(p, grid=(w.prefix_len, *w.grid) if w.grid else None, device=dev)
        g.q.copy_(q)
        g.k.copy_(k)
        g.v.copy_(v)
        for _ in range(args.warmup):
            g.run()
        torch.cuda.synchronize()
        gspan = [(ev(), ev()) for _ in range(args.steps)]
        g0, g1 = ev(), ev()
        g0.record(stream)
        for s_ in range(args.steps):
            if flush is not None:
                flush.fill_(s_ & 255)
                flush_rd.max()
            gspan[s_][0].record(stream)
            g.run()
            gspan[s_][1].record(stream)
        g1.record(stream)
        torch.cuda.synchronize()
        g_ms = (g0.elapsed_time(g1) if flush is None
                else float(sum(a.elapsed_time(b) for a, b in gspan)))
        g_ms = max_over_ranks(g_ms, world, dev)
        graph_line = {"value": round(aggregate_tops(world, dense_equiv_ops(w), args.steps, g_ms), 3),
                      "unit": "TOPS", "ms_per_step": round(g_ms / args.steps, 4),
                      "what": "the same step (permutes, predictor, attention) captured once "
                              "into a CUDA graph and replayed"}
        del g

    if rank != 0:
        return None

    # ---- work accounting and roofline of the attention kernel
    tiles, qk_blocks, pv_blocks, pv_slices, skipped = (int(x) for x in st)
    vis = _visible_blocks(w)
    blk_flops = 2.0 * w.bq * w.bk * w.d
    mma_flops = (qk_blocks + pv_blocks) * blk_flops
    achieved = mma_flops / (attn_ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    # the kernel runs back to back for seconds: the sustained (power-capped)
    # peak applies; the burst figure is reported beside it
    peak = attn_peak_tflops(w, peaks, qk_blocks, pv_blocks)
    peak_burst = attn_peak_tflops(w, peaks, qk_blocks, pv_blocks, key="bf16_tflops")
    peak_bf16 = float(peaks["bf16_tflops_sustained"])
    traffic = profiled_traffic(w.name, w.N)
    pbytes = pool_bytes(w)
    hbm_peak = float(peaks["hbm_gbs"])
    fp32_peak = fp32_peak_tflops(peaks)
    sparsity = {
        "mg": round(1.0 - qk_blocks / vis, 6),
        "pv_slices_skipped": round(skipped / max(1, pv_slices + skipped), 6),
        "total": round(1.0 - (qk_blocks + pv_slices / 4.0) / (2.0 * vis), 6),
    }
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8-qk/f16-pv" if w.qk_int8 else ("bf16" if w.dtype == "bf16" else "f16"),
        "data": "synthetic (seeded generators; no model weights)",
        "config": workload_config(w, world, _bytes(t)),
        "latency_ms": {"predict": round(pred_ms, 4), "predict_pool": round(pool_ms, 4),
                       "predict_select": round(sel_ms, 4), "attention": round(attn_ms, 4),
                       "step": round(ms_step, 4), "step_median": round(step_median_ms, 4),
                       **({"permute": round(perm_ms, 4), "inverse_permute": round(inv_ms, 4)}
                          if w.grid else {})},
        "predict_roofline": {
            "pool": {"bound": "hbm", "achieved": round(pbytes / (pool_ms * 1e-3) / 1e9, 1),
                     "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(pbytes / (pool_ms * 1e-3) / 1e9 / hbm_peak, 4),
                     "bytes_per_launch": pbytes,
                     "extra_bytes": pool_extra_bytes(w),
                     "kernel": "pooling stage (pool_kernel; with INT8 also k-bar and the codes "
                               "of K - k-bar): algorithmic bytes (one read of Q and K, means, "
                               "self-similarities, codes, scales) / stage time; extra_bytes: "
                               "the second read of K and the k-bar sums, not counted"},
            **({"permute": {"bound": "hbm", "unit": "GB/s", "peak": hbm_peak,
                            "bytes_per_launch": 2 * _bytes(t),
                            "achieved": round(2 * _bytes(t) / (perm_ms * 1e-3) / 1e9, 1),
                            "frac": round(2 * _bytes(t) / (perm_ms * 1e-3) / 1e9 / hbm_peak, 4),
                            "kernel": "Hilbert table + gather of Q, K, V: each read once and "
                                      "written once / stage time"},
                "inverse_permute": {"bound": "hbm", "unit": "GB/s", "peak": hbm_peak,
                                    "bytes_per_launch": 2 * o.numel() * o.element_size(),
                                    "achieved": round(2 * o.numel() * o.element_size()
                                                      / (inv_ms * 1e-3) / 1e9, 1),
                                    "frac": round(2 * o.numel() * o.element_size()
                                                  / (inv_ms * 1e-3) / 1e9 / hbm_peak, 4),
                                    "kernel": "scatter of O back to token order: read once, "
                                              "written once / stage time"}}
               if w.grid else {}),
            "select": select_roofline(sel_work, sel_ms, fp32_peak, hbm_peak),
        },
        "sparsity": sparsity,
        "work": {"tiles": tiles, "qk_blocks": qk_blocks, "pv_blocks": pv_blocks,
                 "pv_slices": pv_slices, "skipped_slices": skipped, "visible_blocks": vis},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic,
                     "peak_source": (f"{peak_src} sustained peaks (MEASURED_PEAKS.json) of each "
                                     "contraction's dtype: "
                                     + ("Q K^T INT8 at 2x the bf16 rate, " if w.qk_int8
                                        else "Q K^T at the bf16 rate, ")
                                     + "P~V fp16 at the bf16 rate; flop-weighted harmonic mean"),
                     "frac_of_burst_peak": round(achieved / peak_burst, 4),
                     # Q K^T counted at the bf16 rate (as if it were a bf16 product)
                     "frac_bf16_counted": round(achieved / peak_bf16, 4),
                     # NVIDIA's B200 datasheet: 2.25 PFLOP/s dense bf16 per GPU (the
                     # 4.5 figure printed beside it assumes 2:4 sparsity)
                     "frac_of_datasheet_bf16": round(achieved / DATASHEET_BF16_TFLOPS, 4),
                     "kernel": "attn_kernel (tcgen05), issued MMA flops per launch / launch time"},
        "gpu_launches": launches_per_step * args.steps,
        **({"sparse_regime": sparse} if sparse else {}),
        **({"graph": graph_line} if graph_line else {}),
        "clocks": clocks,
        "e2e": e2e,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"], line["parity_sample"] = cpu_baseline(
            w, t, tiles_per_sample=args.cpu_tiles, gpu_mask_h0=mask_h0)
    return line


def _workload(args):
    w = get_workload(args.workload)
    return w.replace(N=args.seq_len) if args.seq_len > 0 else w


def _bytes(t):
    return sum(t[x].nbytes for x in ("q", "k", "v"))


def _gpu_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index)


def _visible_per_row(w):
    """Visible key blocks of each query block (all of them unless causal)."""
    Tm, Tn = -(-w.N // w.bq), -(-w.N // w.bk)
    if not w.causal:
        return np.full(Tm, Tn, dtype=np.int64)
    last = np.minimum(w.N, (np.arange(Tm) + 1) * w.bq) - 1
    return np.minimum(Tn, last // w.bk + 1).astype(np.int64)


def select_work(w, s_q, kept, theta):
    """The select stage's algorithmic work on one step: S_hat's 2*d flops for
    every visible (i, j) of a query block that is not a fix block (Eq. 9: a
    fix block's row is all ones and its S_hat decides nothing), and its HBM
    bytes: the block means and self-similarities read once, the mask, the
    kept entries of the skip list and the counts written."""
    Tm, Tn = -(-w.N // w.bq), -(-w.N // w.bk)
    vis = _visible_per_row(w)
    nonfix = np.asarray(s_q).reshape(w.B * w.Hq, Tm) >= theta
    pairs = int((nonfix * vis[None, :]).sum())
    nbytes = (4 * (w.B * w.Hq * Tm * (w.d + 1) + w.B * w.Hkv * Tn * (w.d + 1))
              + w.B * w.Hq * Tm * Tn + 4 * kept + 4 * w.B * w.Hq * Tm)
    return {"flops": 2.0 * w.d * pairs, "bytes": float(nbytes),
            "nonfix_rows": int(nonfix.sum()), "rows": int(nonfix.size)}


def select_roofline(work, ms, fp32_peak, hbm_peak):
    """Roofline of the select stage: its S_hat flops against the FP32 FMA
    peak and its bytes against HBM; the larger of the two ideal times bounds
    the stage."""
    t_f = work["flops"] / (fp32_peak * 1e12)
    t_b = work["bytes"] / (hbm_peak * 1e9)
    sec = ms * 1e-3
    if t_f >= t_b:
        out = {"bound": "fp32", "achieved": round(work["flops"] / sec / 1e12, 2),
               "peak": round(fp32_peak, 1), "unit": "TFLOP/s"}
    else:
        out = {"bound": "hbm", "achieved": round(work["bytes"] / sec / 1e9, 1),
               "peak": hbm_peak, "unit": "GB/s"}
    out.update({"frac": round(max(t_f, t_b) / sec, 4), "flops_per_launch": work["flops"],
                "bytes_per_launch": work["bytes"], "nonfix_rows": work["nonfix_rows"],
                "rows": work["rows"],
                "kernel": "select_kernel: 2*d flops per visible (i, j) of a non-fix query "
                          "block for S_hat (peak 148 SMs x 128 FP32 lanes x 2 x max SM "
                          "clock), bytes: means and self-similarities read, mask, kept "
                          "skip-list entries and counts written"})
    return out


def _visible_blocks(w):
    Tm, Tn = -(-w.N // w.bq), -(-w.N // w.bk)
    if not w.causal:
        return Tm * Tn * w.Hq * w.B
    tot = 0
    for i in range(Tm):
        last = min(w.N, (i + 1) * w.bq) - 1
        tot += min(Tn, last // w.bk + 1)
    return tot * w.Hq * w.B


# ----------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ----------------------------------------------------------------------------

def _oracle_sample(w, t, n_tiles, head=0, details=False):
    """Oracle time for head `head`: the whole-sequence predictor prorated to
    n_tiles tiles, plus attention on n_tiles evenly spaced query tiles.
    Returns (dense-equivalent ops of those tiles, seconds, tiles) and, with
    details, the oracle's prediction and attention counters too."""
    from oracle import sparge_oracle as orc
    from synth import to_f64
    hk = head // (w.Hq // w.Hkv)
    Q = to_f64(t["q"][:, head:head + 1], w.dtype)
    K = to_f64(t["k"][:, hk:hk + 1], w.dtype)
    V = to_f64(t["v"][:, hk:hk + 1], w.dtype)
    if w.grid:
        perm = orc.hilbert_permutation(w.N, w.prefix_len, *w.grid)
        Q, K, V = (orc.permute_tokens(x, perm) for x in (Q, K, V))
    Tm = -(-w.N // w.bq)
    t0 = time.perf_counter()
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    t_pred = time.perf_counter() - t0
    idx, cnt = orc.mask_compact(pr["M"])
    quant = orc.quantize_qk(Q.astype(np.float32), K.astype(np.float32), w.bq, w.bk) \
        if w.qk_int8 else None
    tiles = sorted({int(x) for x in np.linspace(0, Tm - 1, n_tiles)})
    t1 = time.perf_counter()
    _, ost = orc.sparse_attention(Q, K, V, idx, cnt, w.bq, w.bk, w.lam, w.causal, w.scale,
                                  quant=quant, tiles=[(0, 0, i) for i in tiles])
    t_attn = time.perf_counter() - t1
    pairs = 0
    for i in tiles:
        r0, r1 = i * w.bq, min(w.N, (i + 1) * w.bq)
        pairs += sum((r + 1) if w.causal else w.N for r in range(r0, r1))
    ops = 4.0 * w.d * pairs
    out = (ops, t_attn + t_pred * len(tiles) / Tm, len(tiles))
    return out + ((pr, ost),) if details else out


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads", 1) for x in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, t, tiles_per_sample=64, gpu_mask_h0=None):
    """The oracle timed on a bounded sample, and the parity counts that the
    sample yields for head 0: the oracle's ambiguous mask entries, where the
    GPU's mask differs from it, and the lambda decisions near the threshold
    on the sampled tiles (the INT8 path's decisions use exact scores here)."""
    ops, sec, n, (pr, ost) = _oracle_sample(w, t, tiles_per_sample, details=True)
    base = {"value": round(ops / sec / 1e12, 9), "unit": "TOPS", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"head 0: float64 oracle predictor over all {w.N} tokens (time prorated "
                      f"to the sample) + attention on {n} evenly spaced query tiles; "
                      f"{sec:.1f} s of CPU"}
    vis = int(pr["visible"].sum()) * w.B
    par = {"head": 0, "visible_blocks": vis, "kept_oracle": int(pr["M"].sum()),
           "ambiguous_near_cut": int(pr["amb_cut"].sum()),
           "ambiguous_near_theta": int(pr["amb_theta"].sum()),
           "near_lambda_decisions": int(ost["near_lambda"]), "sampled_tiles": n}
    if gpu_mask_h0 is not None:
        diff = gpu_mask_h0 != pr["M"][:, 0]
        par["mask_differing"] = int(diff.sum())
        par["mask_differing_outside_ambiguous"] = int((diff & ~pr["amb"][:, 0]).sum())
    return base, par


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = _workload(args)
    t = make_qkv(w, seed=0)
    n = max(1, args.ref_tiles)
    for _ in range(args.warmup):
        _oracle_sample(w, t, n)
    tot_ops = tot_s = 0.0
    for _ in range(args.steps):
        ops, sec, n_t = _oracle_sample(w, t, n)
        tot_ops += ops
        tot_s += sec
    value = tot_ops / tot_s / 1e12
    cores = _blas_threads()
    sample = (f"head 0: float64 oracle predictor over all {w.N} tokens (time prorated) + "
              f"attention on {n_t} evenly spaced query tiles per step")
    return {"metric": METRIC, "value": round(value, 9), "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            # the time each sampled step took; the whole workload would take
            # ms_per_step_full_workload at the same rate
            "ms_per_step": round(1e3 * tot_s / args.steps, 1),
            "ms_per_step_full_workload": round(1e3 * dense_equiv_ops(w) / (value * 1e12), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded generators; no model weights)",
            "config": workload_config(w, world, _bytes(t)),
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 9), "unit": "TOPS", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 9), "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------
# sweeps: the pages' ablations on the synthetic workloads (one JSON line each)
# ----------------------------------------------------------------------------

def _measure(w, steps=3, warmup=2, perm=None, want_output=False, seed=0, tensors=None):
    """Times predict + attention for workload w (grid permutation applied
    outside the timed region when perm is given).  Returns counters, times and
    optionally the float32 output and the self-similarities."""
    import torch
    import free_block_sparse_predict_b200 as fb
    dev = torch.device("cuda", 0)
    t = tensors if tensors is not None else make_qkv(w, seed=seed)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16

    def dv(a):
        x = torch.from_numpy(a).to(dev)
        return x.view(torch.bfloat16) if w.dtype == "bf16" else x
    q, k, v = dv(t["q"]), dv(t["k"]), dv(t["v"])
    if perm is not None:
        pt = torch.from_numpy(perm.astype(np.int32)).to(dev)
        q2, k2, v2 = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        fb.sparge_hilbert_permute(q, q2, pt)
        fb.sparge_hilbert_permute(k, k2, pt)
        fb.sparge_hilbert_permute(v, v2, pt)
        q, k, v = q2, k2, v2
    p = fb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.tau, w.theta, w.lam, causal=w.causal,
                       qk_int8=w.qk_int8, io_dtype=tdt,
                       o_dtype=torch.float32 if want_output else tdt)
    ws = fb.workspace(p, dev)
    mask, idx, cnt, sq, sk = fb.predict_outputs(p, dev)
    o = torch.empty(q.shape, dtype=torch.float32 if want_output else tdt, device=dev)
    stats = torch.zeros(5, dtype=torch.int64, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(warmup):
        fb.sparge_predict_mask(p, q, k, mask, idx, cnt, sq, sk, ws)
        fb.sparge_attn_fwd(p, q, k, v, idx, cnt, o, ws)
    torch.cuda.synchronize()
    a, b, c = ev(), ev(), ev()
    pm = am = 0.0
    for i in range(steps):
        a.record()
        fb.sparge_predict_mask(p, q, k, mask, idx, cnt, sq, sk, ws)
        b.record()
        fb.sparge_attn_fwd(p, q, k, v, idx, cnt, o, ws, stats if i == 0 else None)
        c.record()
        torch.cuda.synchronize()
        pm += a.elapsed_time(b)
        am += b.elapsed_time(c)
    st = [int(x) for x in stats.cpu()]
    vis = _visible_blocks(w)
    step_ms = (pm + am) / steps
    out = {"N": w.N, "tau": w.tau, "theta": w.theta, "lambda": w.lam,
           "predict_ms": round(pm / steps, 4), "attention_ms": round(am / steps, 4),
           "tops": round(dense_equiv_ops(w) / (step_ms * 1e-3) / 1e12, 2),
           "sparsity": {"mg": round(1 - st[1] / vis, 5),
                        "pv_slices_skipped": round(st[4] / max(1, st[3] + st[4]), 5),
                        "total": round(1 - (st[1] + st[3] / 4) / (2 * vis), 5)}}
    extra = {"o": o.float() if want_output else None, "s_q": sq, "s_k": sk, "perm_q": q}
    return out, extra


SWEEP_LENGTHS = (8192, 16384, 32768, 65536, 131072)
SWEEP_TAUS = (0.3, 0.5, 0.7, 0.8, 0.9, 0.95, 0.99, 1.0)


def permutation_tables(w, rng_seed=0):
    """Token orders of the permutation sweep on a grid workload: random,
    row-major (the stored order), time-major, and the Hilbert curve (from the
    library, which matches the oracle's curve bit for bit)."""
    T, H, W = w.grid
    P, L = w.prefix_len, T * H * W
    rng = np.random.default_rng(rng_seed)
    lin = np.arange(L)
    tt, rem = np.divmod(lin, H * W)
    yy, xx = np.divmod(rem, W)
    return {
        "random": np.concatenate([np.arange(P), P + rng.permutation(L)]),
        "rowmajor": np.arange(w.N),
        "timemajor": np.concatenate([np.arange(P), P + np.lexsort((tt, xx, yy))]),
        "hilbert": None,
    }


def sweep_points(kind, base):
    """The configurations one sweep visits, as (label, workload, permutation
    name or None): Table 6's split (paper review, section 六) at the
    configuration's theta and at lower ones where blocks are selective; the
    length sweep; the tau sweep with every block selective (theta = -1), the
    speed-against-sparsity curve; and the token orders of Table 4."""
    pts = []
    if kind == "table6":
        for theta in (base.theta, 0.3, 0.0):
            for name, over in (("only_mg", {"lam": float("-inf")}), ("only_mpv", {"theta": 2.0}),
                               ("both", {})):
                pts.append((f"{name} theta={theta}", base.replace(**{"theta": theta, **over}),
                            None))
    elif kind == "length":
        for n in SWEEP_LENGTHS:
            pts.append((f"N={n}", base.replace(N=n), None))
    elif kind == "tau":
        for tau in SWEEP_TAUS:
            pts.append((f"tau={tau}", base.replace(tau=tau, theta=-1.0), None))
    elif kind == "permutation":
        for name in ("random", "rowmajor", "timemajor", "hilbert"):
            for theta in (base.theta, 0.3):
                pts.append((f"{name} theta={theta}", base.replace(theta=theta), name))
    return pts


def run_sweep(args):
    import torch
    kind = args.sweep
    base = _workload(args)
    if kind == "permutation" and not base.grid:
        base = get_workload("video_dit")
    dev = torch.device("cuda", 0)
    sampler = ClockSampler(_gpu_uuid(torch, dev))
    t_base = make_qkv(base, seed=0)
    perms = permutation_tables(base) if kind == "permutation" else {}
    if kind == "permutation":
        import free_block_sparse_predict_b200 as fb
        T, H, W = base.grid
        hp = torch.empty(base.N, dtype=torch.int32, device=dev)
        hws = torch.zeros(fb.sparge_hilbert_workspace_bytes(T, H, W), dtype=torch.uint8,
                          device=dev)
        fb.sparge_hilbert_index(base.N, base.prefix_len, T, H, W, hp, hws)
        perms["hilbert"] = hp.cpu().numpy()
    dense = {}
    for label, w, pname in sweep_points(kind, base):
        tensors = t_base if w.N == base.N else make_qkv(w, seed=0)
        perm = perms.get(pname) if pname else None
        sampler.start()
        r, extra = _measure(w, perm=perm, want_output=kind == "permutation", tensors=tensors)
        clocks = sampler.stop()
        r.update(sweep=kind, point=label, clocks=clocks, workload=w.name)
        if kind == "table6":
            r.update(theta_setting=w.theta)
        if kind == "permutation":
            # Table 4's columns: block self-similarity and L1 against dense attention
            if pname not in dense:
                _, d_extra = _measure(w.replace(theta=2.0, lam=float("-inf")), steps=1, warmup=1,
                                      perm=perm, want_output=True, tensors=tensors)
                dense[pname] = d_extra["o"]
            O, O2 = dense[pname], extra["o"]
            nq, nk = w.prefix_len // w.bq, w.prefix_len // w.bk
            r.update(permutation=pname,
                     sim_q=round(float(extra["s_q"][..., nq:].mean()), 4),
                     sim_k=round(float(extra["s_k"][..., nk:].mean()), 4),
                     l1=round(float((O - O2).abs().sum() / O.abs().sum()), 5))
        print(json.dumps(r), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--workload", default="llm_128k",
                    choices=("tiny", "image_dit", "video_dit", "llm_32k", "llm_128k"))
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override N of the workload (profiling a smaller case)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="also time the step captured into a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sparse-regime", action="store_true")
    ap.add_argument("--cpu-tiles", type=int, default=64)
    ap.add_argument("--ref-tiles", type=int, default=4)
    ap.add_argument("--sweep", choices=("table6", "length", "tau", "permutation"), default=None,
                    help="run an ablation sweep instead of the benchmark (one JSON line per point)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        if world > 1:
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local_rank))
        try:
            line = run_native(args, rank, world, local_rank)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
