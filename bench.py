#!/usr/bin/env python
"""Forward throughput of pyramid selection + causal block-sparse attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path over one batch of synthetic input:
pyr_build (key pyramid) -> pyr_select (coarse-to-fine LogSumExp top-K) ->
bsa_forward (causal block-sparse attention), through the C ABI. The default
workload is the 32K-token bf16 MHA prefill (B=1, H=16, N=32768, d=128, b=64,
top-K=16 + diagonal, cap 32). Inputs (Q, K, V: 384 MiB) are larger than the
126 MB L2, so consecutive steps do not run from cache.

Prints ONE JSON line on rank 0. `value` is tokens/s = B*N per step, summed over
ranks, divided by the max over ranks of the device time of the K timed steps.
With N > 1 (torchrun, one process per GPU) every rank runs its own workload
instance: the path shards by (batch, kv head) with no exchange step, so the
scaling is weak and there is no collective on the data path.

--impl reference times the CPU oracle (test infrastructure, plain C in double)
on the host cores, on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "fwd tokens/s (select+attn) at 32K–1M ctx; % HBM & tensor roofline vs CPU oracle"
DEFAULT_WORKLOAD = "mha_bf16_32k"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "hierarchical_block_sparse_pyr_b200", "csrc")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


# ------------------------------------------------------------ work counts --

def level_sizes(w):
    nb = w.nb
    out, l = [], 0
    while True:
        n = -(-nb // (1 << l))
        out.append(n)
        if n == 1:
            break
        l += 1
    return out


def work_counts(w):
    """Algorithmic bytes / FLOPs of one step from the method's definition.

    Attention pairs are exact; selection counts every node that can be a candidate
    at each level, an upper bound on the nodes the walk actually scores (a few
    percent above it: a kept node whose second child starts at or after the
    query block contributes one child, not two)."""
    elt = 4 if w.dtype == synth.F32 else 2
    lv = level_sizes(w)
    P = sum(lv)
    U = w.B * w.Hkv
    first = w.q_offset // w.b
    nqb = (w.q_offset + w.Nq - 1) // w.b - first + 1
    s0 = 0
    while lv[s0] > w.cap:
        s0 += 1
    # selection: candidates scored per level (upper bound per level: all valid nodes at s0, then <= cap)
    sel_flops = 0
    sel_exps = 0
    sel_nodes = 0  # candidate node rows read, summed over query blocks
    att_pairs = 0
    for qb in range(nqb):
        i = first + qb
        p0, p1 = max(i * w.b, w.q_offset), min((i + 1) * w.b, w.q_offset + w.Nq)
        rows = w.G * (p1 - p0)
        nc = -(-i // (1 << s0))  # valid nodes at s0: those starting before block i
        for l in range(s0, -1, -1):
            sel_flops += 2 * rows * nc * w.d
            sel_exps += rows * nc
            sel_nodes += nc
            keep = min(w.cap // 2 if l > 0 else w.topk, nc)
            if l > 0:
                # children of the kept nodes that start before i (at most 2 per kept node)
                nc = min(2 * keep, -(-i // (1 << (l - 1))))
        nsel = min(w.topk, i)
        # selected blocks are strictly before i (full blocks); the diagonal is causal
        n = p1 - p0
        att_pairs += w.G * (n * nsel * w.b + (p0 - i * w.b + 1 + p1 - i * w.b) * n // 2)
    sel_flops *= U
    sel_exps *= U
    att_pairs *= U
    att_flops = 4 * w.d * att_pairs
    if w.decode:
        # one decode step: re-pool the last block and its ancestors (one node per level)
        pyr_bytes = U * (min(w.b, w.N) * w.d * elt + len(lv) * w.d * 4)
    else:
        pyr_bytes = U * (w.N * w.d * elt + P * w.d * 4)
    q_bytes = w.B * w.Hq * w.Nq * w.d * elt
    # Q once + the pyramid once (each node a bf16 (hi, lo) pair: 4 bytes per element) + idx; a walk that
    # touches fewer nodes than the pyramid holds (decode: one query block per unit) reads only those
    sel_bytes = q_bytes + U * min(P, sel_nodes) * w.d * 4 + U * nqb * w.topk * 4
    # attention: Q + O once; K, V of the selected + diagonal blocks once per query block and kv head
    kv_blocks = 0
    for qb in range(nqb):
        i = first + qb
        kv_blocks += min(w.topk, i) + 1
    att_bytes = 2 * q_bytes + U * kv_blocks * 2 * w.b * w.d * elt
    return dict(pyr_bytes=pyr_bytes, sel_flops=sel_flops, sel_exps=sel_exps, sel_bytes=sel_bytes,
                att_flops=att_flops, att_bytes=att_bytes, att_pairs=att_pairs, tokens=w.B * w.Nq)


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    p = dict(FALLBACK_PEAKS)
    p["source"] = "fallback"
    return p


def src_hash(files):
    h = hashlib.sha256()
    for fn in files:
        with open(os.path.join(CSRC, fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def kernel_source(kernel, w):
    """The .cu file whose code runs as `kernel` for workload w (its hash keys the ncu traffic record)."""
    if kernel == "pyramid":
        return "pyramid.cu"
    if kernel == "select":
        if w.decode:
            return "select_decode.cu" if w.G <= 8 else "select.cu"  # the decode walk (G <= 8), else the SIMT walk
        return "select_tc.cu" if tc_select(w) else "select.cu"
    if w.decode:
        return "attn_decode_warp.cu" if w.G <= 8 else "attn_decode.cu"
    if tc_attention(w) and w.G == 1 and w.b == 64:
        return "attn_pair.cu"  # 64-row MHA query blocks, two per CTA over their own lists
    return "attn_tc.cu" if tc_attention(w) else "attn_simt.cu"


def tc_attention(w):
    """True when bsa_forward takes the tcgen05 kernel for this workload (bf16, d=128, b in {64,128},
    G*b in {64,128,256}, not decode)."""
    return (w.dtype == synth.BF16 and w.d == 128 and w.b in (64, 128) and w.Nq > 1
            and w.G * w.b in (64, 128, 256))


def tc_select(w):
    """True when pyr_select scores on the tensor cores (bf16, d=128, prefill, G*b in {64,128,256})."""
    return (w.dtype == synth.BF16 and w.d == 128 and w.Nq > 1 and w.b % 64 == 0
            and w.G * w.b in (64, 128, 256))


def peak_source(bound, peaks):
    if bound == "alu":
        return "derived: 148 SMs x 128 FP32 lanes x 2 FLOP x median SM clock under load"
    tag = "measured" if peaks["source"] == "measured" else "fallback"
    if bound == "tensor":
        return f"{tag}: dense bf16 cuBLAS, burst (the timed region lasts well under a second)"
    return f"{tag}: HBM copy bandwidth"


def measured_traffic(kernel, workload):
    """dram bytes per launch from a committed ncu summary, if the kernel source is unchanged since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    rec = t.get(workload.name, {}).get(kernel)
    if not rec or rec.get("src_sha") != src_hash([kernel_source(kernel, workload)]):
        return None
    return rec.get("bytes_per_launch")


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, pw, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
                pw.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [s for s, p in zip(sm, pw) if p > 200] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(pw) if pw else None}


# ------------------------------------------------------ multi-rank logic --

def replica_workload(w, rank):
    """The workload instance of one rank: same shape, its own seed (independent problems)."""
    return w if rank == 0 else w.scaled(seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (the job's device time is the slowest rank's)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_max_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own instance in the max-over-ranks time."""
    return world * tokens_per_rank / (ms_max_per_step * 1e-3)


# ----------------------------------------------------------- dense path --

def dense_flops(w):
    """4 d FLOPs per attended (query, key) pair of plain causal attention."""
    pairs = 0
    for t in range(w.Nq) if w.Nq <= 4 else []:
        pairs += w.q_offset + t + 1
    if w.Nq > 4:
        p0, p1 = w.q_offset, w.q_offset + w.Nq  # positions [p0, p1): sum of (p + 1)
        pairs = (p1 * (p1 + 1) - p0 * (p0 + 1)) // 2
    return 4 * w.d * pairs * w.B * w.Hq


def time_dense(P, s, w, Q, K, V, buf, stream, steps, warmup):
    """Event-timed dense_forward (plain causal attention) on the same inputs."""
    steps = max(3, min(steps, 10)) if dense_flops(w) < 1e14 else 2  # a 1M-token dense pass takes seconds
    for _ in range(1 if dense_flops(w) >= 1e14 else max(1, warmup // 2)):
        P.dense_forward(s, Q, K, V, buf.O, buf.lse, buf.status, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        P.dense_forward(s, Q, K, V, buf.O, buf.lse, buf.status, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"ms": round(ms, 4), "tflops": round(dense_flops(w) / (ms * 1e-3) / 1e12, 2)}


def time_backward(P, s, w, Q, K, V, buf, stream, steps, warmup):
    """Event-timed backward (route inversion + gradients) of the forward pass held in buf.

    Algorithmic FLOPs: 8 d per attended (query, key) pair (S and dP recomputed, dQ, dK, dV products).
    """
    dO = synth.grad_output(w).cuda()
    bwd = P.BackwardBuffers(s)
    P.run(s, Q, K, V, buf, stream)
    for _ in range(max(1, warmup)):
        P.run_backward(s, Q, K, V, dO, buf, bwd, stream)
    torch.cuda.synchronize()
    steps = max(2, min(steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        P.run_backward(s, Q, K, V, dO, buf, bwd, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"device status {buf.status.item()}")
    ms = e0.elapsed_time(e1) / steps
    flops = 2 * work_counts(w)["att_flops"]
    del bwd, dO
    return {"ms": round(ms, 4), "algorithmic_tflop": round(flops / 1e12, 4),
            "tflops": round(flops / (ms * 1e-3) / 1e12, 2), "path": "tcgen05 (bf16, d=128, b in {64, 128}) else fp32 CUDA cores"}


def phba_counts(w, M, idx):
    """Algorithmic bytes of the state build and FLOPs of the state-aware attention (PHBA branch).

    State build: read the state keys and values once, the two fp32 gates once, write the two states
    (the fp32 workspace between its two passes is not counted). Attention: 4 d FLOPs per token pair
    (as bsa_forward) plus 4 d per (row, slot) pair, M slots per attended state: the current block's
    state and each routed block's, blocks >= 1 (block 0 has no state). idx: the routes of the step
    ([B, Hkv, nqb, topk], numpy), which decide how many routed blocks are >= 1."""
    elt = 2 if w.dtype == synth.BF16 else 4
    U = w.B * w.Hkv
    build_bytes = U * (2 * w.N * w.d * elt + 2 * w.N * M * 4 + 2 * w.nb * M * w.d * elt)
    first = w.q_offset // w.b
    nqb = idx.shape[2]
    qbs = np.arange(nqb)
    i = first + qbs
    rows = w.G * (np.minimum((i + 1) * w.b, w.q_offset + w.Nq) - np.maximum(i * w.b, w.q_offset))
    n_states = (idx >= 1).sum(axis=-1) + (i >= 1)[None, None, :]  # [B, Hkv, nqb]
    slot_pairs = int((n_states * rows[None, None, :]).sum()) * M
    return build_bytes, 4 * w.d * slot_pairs


def time_phba(args, w, dev, stream, peaks, M=128):
    """The PHBA prefix-state branch on a workload: pyramid + selection + state build + attention over
    tokens and state slots, event-timed per call (1 GPU)."""
    import hierarchical_block_sparse_pyr_b200 as P

    s = P.shape_of(w)
    Qh, Kh, Vh, _ = synth.generate(w)
    Ah, Wh = synth.phba_gates(w, M)
    Q, K, V, A, W = (t.to(dev) for t in (Qh, Kh, Vh, Ah, Wh))
    buf = P.Buffers(s, dev)
    st = P.PhbaStates(s, M, dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        P.pyr_build(s, K, buf.pyr, buf.status, stream)
        P.pyr_select(s, Q, buf.pyr, buf.idx, None, buf.status, stream)
        if ev:
            ev[1].record(stream)
        P.phba_state_build(s, M, K, V, A, W, st.PK, st.PV, st.workspace, buf.status, stream)
        if ev:
            ev[2].record(stream)
        P.phba_forward(s, Q, K, V, buf.idx, buf.O, buf.lse, M=M, PK=st.PK, PV=st.PV, status=buf.status,
                       stream=stream)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"phba: device status {buf.status.item()}")
    steps = max(3, min(args.steps, 10))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for k in range(steps):
        step(evs[k])
    torch.cuda.synchronize()
    sel = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    bld = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    att = sum(e[2].elapsed_time(e[3]) for e in evs) / steps
    build_bytes, slot_flops = phba_counts(w, M, buf.idx.cpu().numpy())
    att_flops = work_counts(w)["att_flops"] + slot_flops
    ms = sel + bld + att
    del Q, K, V, A, W, buf, st
    torch.cuda.empty_cache()
    return {"workload": w.name, "M": M, "ms_per_step": round(ms, 4),
            "value": round(w.B * w.Nq / (ms * 1e-3), 1), "unit": "tokens/s",
            "pyramid_select_ms": round(sel, 4),
            "state_build": {"ms": round(bld, 4), "bound": "hbm", "algorithmic_bytes": build_bytes,
                            "achieved_gbs": round(build_bytes / (bld * 1e-3) / 1e9, 1),
                            "frac": round(build_bytes / (bld * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
            "attention": {"ms": round(att, 4), "bound": "tensor", "algorithmic_tflop": round(att_flops / 1e12, 4),
                          "achieved_tflops": round(att_flops / (att * 1e-3) / 1e12, 1),
                          "frac": round(att_flops / (att * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}}


def break_even(args, w):
    """Sparse step (pyramid + selection + attention) vs dense causal attention over context lengths."""
    import hierarchical_block_sparse_pyr_b200 as P
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    points = []
    for n in (2048, 4096, 8192, 16384, 32768, 65536):
        wn = w.scaled(name=f"{w.name}@N={n}", N=n, Nq=n, q_offset=0)
        s = P.shape_of(wn)
        Qh, Kh, Vh, _ = synth.generate(wn)
        Q, K, V = Qh.cuda(), Kh.cuda(), Vh.cuda()
        buf = P.Buffers(s)
        for _ in range(3):
            P.run(s, Q, K, V, buf, stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(10):
            P.run(s, Q, K, V, buf, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        sparse_ms = e0.elapsed_time(e1) / 10
        dense = time_dense(P, s, wn, Q, K, V, buf, stream, 10, 3)
        points.append({"N": n, "sparse_step_ms": round(sparse_ms, 4), "dense_ms": dense["ms"]})
        del Q, K, V, buf
        torch.cuda.empty_cache()
    be = next((p["N"] for p in points if p["sparse_step_ms"] < p["dense_ms"]), None)
    return {"metric": "break-even context length: pyramid + select + block-sparse attention vs dense causal",
            "workload": w.name, "points": points, "break_even_N": be}


# --------------------------------------------------------------- our arm --

def count_launches(step):
    """Kernels of libpyr launched by one step (profiled outside the timed region)."""
    try:
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
        ours = [n for n in names if any(k in n for k in ("pyr_", "select_", "attn_"))]
        return len(ours), sorted(set(ours))
    except Exception as ex:  # profiler unavailable: report unknown
        return None, [f"profiler unavailable: {ex}"]


def make_step(P, s, w, Q, K, V, buf, stream):
    """One step of the path on resident inputs; ev (4 events) brackets the three calls."""
    def step(ev=None):
        if ev:
            ev[0].record(stream)
        if w.decode:
            # a decode step refreshes only the nodes over the appended position
            P.pyr_update(s, K, buf.pyr, w.N - 1, buf.status, stream)
        else:
            P.pyr_build(s, K, buf.pyr, buf.status, stream)
        if ev:
            ev[1].record(stream)
        P.pyr_select(s, Q, buf.pyr, buf.idx, buf.gap, buf.status, stream)
        if ev:
            ev[2].record(stream)
        P.bsa_forward(s, Q, K, V, buf.idx, buf.O, buf.lse, buf.status, stream)
        if ev:
            ev[3].record(stream)
    return step


def time_steps(step, steps, world, dev, stream, clock_index):
    """K event-timed steps between barriers + synchronize, clocks sampled meanwhile.
    Returns (ms per step of this rank, max over ranks, per-kernel ms lists, clocks)."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(clock_index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record(stream)
    for k in range(steps):
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    per = {"pyramid": [], "select": [], "attention": []}
    for ev in evs:
        per["pyramid"].append(ev[0].elapsed_time(ev[1]))
        per["select"].append(ev[1].elapsed_time(ev[2]))
        per["attention"].append(ev[2].elapsed_time(ev[3]))
    return ms_total / steps, max_over_ranks(ms_total, world, dev) / steps, per, clk


def kernel_report(w, per, ms_step, peaks, sm_clock):
    """Per-kernel roofline figures from the kernels' average event-timed durations.

    Tensor-core kernels are rated against the burst dense bf16 peak (the timed regions last well
    under a second); frac_sustained, against the sustained peak, is context. Selection is also
    rated against HBM with its bytes counted once (Q, the pyramid, idx), and pyramid + selection
    together against HBM."""
    wc = work_counts(w)
    avg = {k: sum(v) / len(v) for k, v in per.items()}
    alu_peak = 148 * 128 * 2 * sm_clock * 1e6 / 1e12
    tc_burst, tc_sus = peaks["bf16_tflops"], peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    sel_tc, att_tc = tc_select(w), tc_attention(w)
    kernels = {
        "pyramid": dict(ms=avg["pyramid"], bound="hbm", kernel="pyr_update" if w.decode else "pyr_build",
                        achieved=wc["pyr_bytes"] / (avg["pyramid"] * 1e-3) / 1e9, peak=peaks["hbm_gbs"], unit="GB/s",
                        algorithmic=wc["pyr_bytes"], traffic=measured_traffic("pyramid", w)),
        "select": dict(ms=avg["select"], bound="tensor" if sel_tc else "alu",
                       achieved=wc["sel_flops"] / (avg["select"] * 1e-3) / 1e12,
                       peak=tc_burst if sel_tc else alu_peak, unit="TFLOP/s", algorithmic=wc["sel_flops"],
                       hbm_bytes=wc["sel_bytes"], hbm_gbs=wc["sel_bytes"] / (avg["select"] * 1e-3) / 1e9,
                       hbm_frac=wc["sel_bytes"] / (avg["select"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                       traffic=measured_traffic("select", w)),
    }
    if w.decode:
        kernels["attention"] = dict(ms=avg["attention"], bound="hbm",
                                    achieved=wc["att_bytes"] / (avg["attention"] * 1e-3) / 1e9,
                                    peak=peaks["hbm_gbs"], unit="GB/s", algorithmic=wc["att_bytes"],
                                    traffic=measured_traffic("attention", w))
    else:
        kernels["attention"] = dict(ms=avg["attention"], bound="tensor" if att_tc else "alu",
                                    achieved=wc["att_flops"] / (avg["attention"] * 1e-3) / 1e12,
                                    peak=tc_burst if att_tc else alu_peak, unit="TFLOP/s",
                                    algorithmic=wc["att_flops"], traffic=measured_traffic("attention", w))
    for name, k in kernels.items():
        k["frac"] = k["achieved"] / k["peak"]
        k["share"] = k["ms"] / ms_step
        if k["bound"] == "tensor":
            k["frac_sustained"] = k["achieved"] / tc_sus
    both_ms = avg["pyramid"] + avg["select"]
    pyr_sel = {"bytes": wc["pyr_bytes"] + wc["sel_bytes"], "ms": both_ms,
               "achieved_gbs": (wc["pyr_bytes"] + wc["sel_bytes"]) / (both_ms * 1e-3) / 1e9}
    pyr_sel["hbm_frac"] = pyr_sel["achieved_gbs"] / peaks["hbm_gbs"]
    return wc, kernels, pyr_sel


def rounded(d):
    return {k: (round(v, 5) if isinstance(v, float) else v) for k, v in d.items()}


def roofline_of(kernels, peaks):
    dom_name = max(kernels, key=lambda k: kernels[k]["ms"])
    dom = kernels[dom_name]
    return {"kernel": dom_name, "bound": dom["bound"], "achieved": round(dom["achieved"], 3),
            "peak": round(dom["peak"], 3), "unit": dom["unit"], "frac": round(dom["frac"], 4),
            "traffic": dom["traffic"], "peak_source": peak_source(dom["bound"], peaks)}


def sub_workload(args, name, dev, stream, local_rank, peaks):
    """One more workload of the metric's range, timed on the device like the headline one (1 GPU)."""
    import hierarchical_block_sparse_pyr_b200 as P

    w = synth.BY_NAME[name]
    t_gen = time.perf_counter()
    Qh, Kh, Vh, _ = synth.generate(w)
    t_gen = time.perf_counter() - t_gen
    s = P.shape_of(w)
    Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
    buf = P.Buffers(s, dev)
    if w.decode:
        P.pyr_build(s, K, buf.pyr, buf.status, stream)
    step = make_step(P, s, w, Q, K, V, buf, stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"{name}: device status {buf.status.item()}")
    steps = max(3, min(args.steps, 10 if not w.decode else 50))
    ms_rank, ms_step, per, clk = time_steps(step, steps, 1, dev, stream, local_rank)
    sm_clock = clk.get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    wc, kernels, pyr_sel = kernel_report(w, per, ms_step, peaks, sm_clock)
    del Q, K, V, buf
    torch.cuda.empty_cache()
    out = {"workload": name, "tokens_per_step": wc["tokens"], "steps": steps, "ms_per_step": round(ms_step, 4),
           "value": round(wc["tokens"] / (ms_step * 1e-3), 1), "unit": "tokens/s",
           "roofline": roofline_of(kernels, peaks),
           "kernels": {k: rounded(v) for k, v in kernels.items()}, "pyramid_select_hbm": rounded(pyr_sel),
           "clocks": clk, "input_generation_s": round(t_gen, 1)}
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, budget_s=5.0, QKV=(Qh, Kh, Vh))
    del Qh, Kh, Vh
    return out


def run_ours(args, w, rank, world, local_rank):
    import hierarchical_block_sparse_pyr_b200 as P

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = replica_workload(w, rank)
    s = P.shape_of(w)
    Qh, Kh, Vh, _ = synth.generate(w, pin=True)
    Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
    buf = P.Buffers(s, dev)
    stream = torch.cuda.current_stream(dev)

    # prefill builds the pyramid from K; a decode step refreshes only the nodes over the
    # appended position (the pyramid of the prefilled context is built once, untimed)
    if w.decode:
        P.pyr_build(s, K, buf.pyr, buf.status, stream)
    step = make_step(P, s, w, Q, K, V, buf, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"device status {buf.status.item()}: {P.strerror(int(buf.status.item()))}")
    launches_per_step, kernel_names = count_launches(step)

    # timed region: K steps, per-kernel events on the launching stream
    _, ms_step, per, clk = time_steps(step, args.steps, world, dev, stream, local_rank)

    # end to end through the binding: pinned host inputs -> device -> path -> O back to pinned host.
    # Prefill: a step's inputs are Q, K and V. Decode: they are the new token's q, k and v; k and v
    # are written into the device-resident cache at the last position (the cache is state, not input).
    O_host = torch.empty(buf.O.shape, dtype=buf.O.dtype, pin_memory=True)
    if w.decode:
        Kn_h = Kh[:, :, w.N - 1].contiguous().pin_memory()
        Vn_h = Vh[:, :, w.N - 1].contiguous().pin_memory()
        h2d = (Qh.numel() * Qh.element_size() + Kn_h.numel() * Kn_h.element_size() +
               Vn_h.numel() * Vn_h.element_size())
    else:
        h2d = Qh.numel() * Qh.element_size() + Kh.numel() * Kh.element_size() + Vh.numel() * Vh.element_size()
    d2h = O_host.numel() * O_host.element_size()

    if w.decode:
        e2e_call = "pyr_update + pyr_select + bsa_forward on the resident cache"

        def e2e_step():
            Q.copy_(Qh, non_blocking=True)
            K[:, :, w.N - 1].copy_(Kn_h, non_blocking=True)
            V[:, :, w.N - 1].copy_(Vn_h, non_blocking=True)
            step()
            O_host.copy_(buf.O, non_blocking=True)
    else:
        # the host-buffer entry point: units stream through the device in chunks, copies overlap compute
        e2e_call = "bsa_forward_host"
        workspace = torch.empty(P.host_workspace_bytes(s, 0, False), dtype=torch.uint8, device=dev)

        def e2e_step():
            P.bsa_forward_host(s, Qh, Kh, Vh, O_host, None, units_per_chunk=0, workspace=workspace,
                               status=buf.status, stream=stream)

    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(3, min(args.steps, 10))
    e0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"device status {buf.status.item()}")
    if not w.decode:
        # the host path computes each unit with the same kernels: its output equals the device path's bit for bit
        step()
        torch.cuda.synchronize()
        if not torch.equal(O_host, buf.O.cpu()):
            raise RuntimeError("bsa_forward_host output differs from the device path")

    dense = time_dense(P, s, w, Q, K, V, buf, stream, args.steps, args.warmup)
    backward = (time_backward(P, s, w, Q, K, V, buf, stream, args.steps, args.warmup)
                if args.backward and not w.decode else None)

    peaks = load_peaks()
    sm_clock = clk.get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    wc, kernels, pyr_sel = kernel_report(w, per, ms_step, peaks, sm_clock)
    value = job_throughput(wc["tokens"], world, ms_step)
    if backward:
        backward["bound"] = "tensor"
        backward["frac"] = round(backward["tflops"] / peaks["bf16_tflops"], 4)  # burst peak, as the forward
    l2_mib = (Qh.numel() + Kh.numel() + Vh.numel()) * Qh.element_size() >> 20
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == synth.BF16 else "f32", "data": "synthetic",
        "config": config_of(w, world, l2_mib),
        "e2e": {"value": round(job_throughput(wc["tokens"], world, e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "call": e2e_call},
        "gpu_launches": None if launches_per_step is None else launches_per_step * args.steps,
        "roofline": roofline_of(kernels, peaks),
        "kernels": {k: rounded(v) for k, v in kernels.items()},
        "pyramid_select_hbm": rounded(pyr_sel),
        "dense": dict(dense, speedup_of_sparse_step=round(dense["ms"] / ms_step, 3)),
        **({"backward": backward} if backward else {}),
        "kernel_names": kernel_names,
        "clocks": clk,
        "peaks_source": peaks["source"],
    }
    del Q, K, V, buf, O_host
    if w.decode:
        del Kn_h, Vn_h
    else:
        del workspace
    torch.cuda.empty_cache()
    if world == 1 and rank == 0 and args.sub_workloads:
        # the rest of the metric's 32K-1M range, each timed like the headline workload
        out["workloads"] = {}
        for name in args.sub_workloads:
            if name != w.name:
                out["workloads"][name] = sub_workload(args, name, dev, stream, local_rank, peaks)
    if world == 1 and rank == 0 and args.with_break_even and not w.decode:
        out["break_even"] = break_even(args, w)
    if world == 1 and rank == 0 and args.phba_slots > 0 and not w.decode and w.dtype == synth.BF16:
        out["phba"] = time_phba(args, w, dev, stream, peaks, args.phba_slots)
    return out


def config_of(w, world, l2_mib=None):
    """The workload's config dict (the same for both arms)."""
    c = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "Nq": w.Nq, "d": w.d, "b": w.b,
         "topk": w.topk, "cap": w.cap, "seed": w.seed, "global_batch": w.B * world, "seq_len": w.N,
         "parallelism": f"replicas{world}" if world > 1 else "single"}
    if l2_mib is None:
        elt = 2 if w.dtype == synth.BF16 else 4
        l2_mib = (w.B * w.Hq * w.Nq + 2 * w.B * w.Hkv * w.N) * w.d * elt >> 20
    c["l2"] = "inputs larger than L2 (Q+K+V %d MiB > 126 MB)" % l2_mib
    return c


# -------------------------------------------------------- oracle baseline --

def oracle_sample(w, n_qb, seed=0, Q=None, K=None, V=None, n_units=1):
    """Time the oracle on n_units consecutive (batch, kv head) units starting at unit `seed`: their
    pyramids and n_qb evenly spaced query blocks of each (selection + attention of all their rows).
    Returns (seconds, est. seconds for the whole job, desc); with every unit and every query block in
    the sample the estimate is the measured time itself."""
    import oracle

    if Q is None:
        Q, K, V, _ = synth.generate(w)
    nqb = oracle.num_qblocks(w)
    U = w.B * w.Hkv
    units = [(seed + k) % U for k in range(min(max(1, n_units), U))]
    qbs = np.unique(np.linspace(0, nqb - 1, num=min(n_qb, nqb)).round().astype(int))
    t0 = time.perf_counter()
    pyr = oracle.pyramid(w, K, units)
    t1 = time.perf_counter()
    idx_u, _, _ = oracle.select(w, Q, pyr, units, [(k, int(q)) for k in range(len(units)) for q in qbs])
    t2 = time.perf_counter()
    full_idx = -np.ones((w.B, w.Hkv, nqb, w.topk), dtype=np.int32)
    rows = []
    first = w.q_offset // w.b
    for k, unit in enumerate(units):
        bi, hk = divmod(unit, w.Hkv)
        full_idx[bi, hk, qbs] = idx_u[k * len(qbs):(k + 1) * len(qbs)]
        for q in qbs:
            i = first + int(q)
            p0, p1 = max(i * w.b, w.q_offset), min((i + 1) * w.b, w.q_offset + w.Nq)
            for g in range(w.G):
                hq = hk * w.G + g
                rows += [((bi * w.Hq + hq) * w.Nq + (p - w.q_offset)) for p in range(p0, p1)]
    oracle.attend(w, Q, K, V, full_idx, np.array(rows, dtype=np.int64))
    t3 = time.perf_counter()
    nu = len(units)
    per_qb = ((t2 - t1) + (t3 - t2)) / (len(qbs) * nu)
    est = U * ((t1 - t0) / nu + per_qb * nqb)
    if nu == U and len(qbs) == nqb:
        desc = f"the whole job: all {U} units, pyramid + selection + attention of all {nqb} query blocks each"
    else:
        desc = (f"units {units[0]}..{units[-1]} of {U}: pyramid + {len(qbs)} of {nqb} query blocks each (evenly "
                f"spaced; selection + attention of all their rows); whole-job time extrapolated")
    return t3 - t0, est, desc


def cpu_baseline(w, budget_s=15.0, QKV=None):
    """The oracle on a sample of about budget_s * 0.4 .. budget_s seconds: more query blocks of one unit
    first, then more units, up to the whole job. QKV: the workload's host tensors, if at hand."""
    Q, K, V = QKV if QKV is not None else synth.generate(w)[:3]
    nqb = oracle_nqb(w)
    U = w.B * w.Hkv
    n, nu = 4, 1
    took, est, desc = oracle_sample(w, n, Q=Q, K=K, V=V)
    while took < budget_s * 0.4 and (n < min(nqb, 4096) or nu < U):
        grow = max(2.0, budget_s / max(took, 1e-3) * 0.9)
        if n < min(nqb, 4096):
            n = min(nqb, 4096, int(n * grow))
        else:
            nu = min(U, int(nu * grow))
        took, est, desc = oracle_sample(w, n, Q=Q, K=K, V=V, n_units=nu)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(w.B * w.Nq / est, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": desc, "sample_seconds": round(took, 2), "extrapolated": "extrapolated" in desc}


def oracle_nqb(w):
    import oracle

    return oracle.num_qblocks(w)


def run_reference(args, w):
    """The oracle, as it stands, on the host cores: each step times a bounded sample of the workload
    (pyramids of one unit and a set of its query blocks). ms_per_step is the time those samples
    actually took; the whole-job time they extrapolate to is given beside it."""
    Q, K, V, _ = synth.generate(w)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    n_qb = 8
    took, _, _ = oracle_sample(w, n_qb, Q=Q, K=K, V=V)
    # size each step to ~4 s of host time so that the whole run ends within minutes
    n_qb = max(1, min(4096, int(n_qb * 4.0 / max(took, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample(w, max(1, n_qb // 4), Q=Q, K=K, V=V)
    ests, tooks, desc = [], [], ""
    for k in range(args.steps):
        took, est, desc = oracle_sample(w, n_qb, seed=k, Q=Q, K=K, V=V)
        ests.append(est)
        tooks.append(took)
    est = statistics.mean(ests)
    ms_timed = statistics.mean(tooks) * 1e3
    value = w.B * w.Nq / est
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_timed, 1),
            "ms_per_step_meaning": "host time of one step's sample (timed); value extrapolates it to the whole job",
            "whole_job_ms_extrapolated": round(est * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, 1),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc + f"; {args.steps} steps, mean sample {statistics.mean(tooks):.2f} s"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", dest="backward", action="store_false",
                    help="skip timing the backward pass (route inversion + gradients) of the forward step")
    ap.add_argument("--break-even", action="store_true",
                    help="sweep the context length and report where the sparse step beats dense attention")
    ap.add_argument("--sub-workloads", default="gqa_bf16_64k,mha_bf16_1m,decode_gqa_bf16_128k",
                    help="comma-separated workloads timed after the headline one and reported under "
                         "'workloads' (1 GPU only); empty for none")
    ap.add_argument("--phba-slots", type=int, default=128,
                    help="also time the PHBA prefix-state branch with this many slots per state, reported under "
                         "'phba' (0: skip)")
    ap.add_argument("--no-break-even", dest="with_break_even", action="store_false",
                    help="skip the sparse-vs-dense context-length sweep reported under 'break_even'")
    ap.add_argument("--n", type=int, default=None,
                    help="shrink the context length (and query rows) of the workload: for profiling the same "
                         "kernels on a smaller case; the default JSON line always uses the full workload")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.sub_workloads = [x for x in args.sub_workloads.split(",") if x]
    for x in args.sub_workloads:
        if x not in synth.BY_NAME:
            ap.error(f"unknown workload {x}")
    w = synth.BY_NAME[args.workload]
    if args.n:
        w = w.scaled(name=f"{w.name}@N={args.n}", N=args.n, Nq=1 if w.decode else args.n,
                     q_offset=args.n - 1 if w.decode else 0)
        args.sub_workloads, args.with_break_even, args.phba_slots, args.backward = [], False, 0, False

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.break_even:
        print(json.dumps(break_even(args, w)), flush=True)
        return

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, w, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(w)
        elif rank == 0:
            out["cpu_baseline"] = None
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
