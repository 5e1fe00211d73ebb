"""Benchmark: zigzag context-parallel causal attention on B200.

One step = the whole hot path on one batch of seeded synthetic input already in
HBM: cp_plan_shards (plan + gather of Q, K, V, dO into shard order),
cp_attn_fwd (per-rank attention over the K/V shards in visit order, partials
combined by the LSE-merge kernel), cp_attn_bwd (dQ, dK, dV).

Metric: causal CP-attention TFLOPS, fwd+bwd, on the workload named in
config.workload (default: 128k tokens, 32/8 GQA heads, head_dim 128, cp 8,
all-gather order).  FLOPs follow the convention 4*D*Hq per unmasked pair for the
forward and 3x that for forward + backward; the unmasked pair count comes from
the library's own planner.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--rotate allgather|ring] [--impl native|reference]
With N > 1 (launched by torchrun) every rank runs its own replica of the
workload on its own GPU: the path has no cross-GPU exchange on one GPU's worth
of virtual ranks, so there is no data-path collective; the barrier and the
max-over-ranks timing use torch.distributed.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------- distributed plumbing

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(world: int, backend: str):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    return dist


def dist_barrier(dist, device=None):
    if dist is not None:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def dist_max(dist, x: float, device=None) -> float:
    """Max of a float over ranks (identity on one rank)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(value_per_rank_units: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return value_per_rank_units * world / (ms_max * 1e-3)


# --------------------------------------------------------------------- peaks and clocks

def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return dict(bf16=float(p["bf16_tflops"]), bf16_sustained=float(p["bf16_tflops_sustained"]),
                    hbm=float(p["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=1400.0, hbm=FALLBACK_HBM_GBS,
                    source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------- CPU baseline (oracle)

def cpu_baseline(w: synth.Workload, budget_tokens: int = 5120):
    """The oracle, as it stands, on a bounded sample of the workload: forward and
    backward of the first `budget_tokens` tokens of one KV group (all its query
    heads), FLOPs by the same convention."""
    import oracle  # test infrastructure: the only place the benchmark runs it
    import torch
    oracle.build()
    g = w.num_heads // w.num_kv_heads
    S = budget_tokens
    t = synth.attn_inputs(1, g, 1, S, w.head_dim, w.seed, amp=w.amp, with_dout=True)
    q, k, v, do = (t[n].to(torch.float64).numpy() for n in ("q", "k", "v", "do"))
    cu = None
    if w.docs:
        lens = synth.doc_lengths(S, w.seed, w.doc_median, w.doc_sigma, w.doc_clip)
        cu = synth.cu_seqlens(lens)
    ds = oracle.doc_start(S, cu)
    t0 = time.perf_counter()
    o, lse = oracle.fwd(q, k, v, ds)
    oracle.bwd(q, k, v, o, lse, do, ds)
    dt = time.perf_counter() - t0
    pairs = oracle.causal_pairs(S, cu)
    flops = oracle.flops(g, w.head_dim, pairs, backward=True)
    return dict(value=flops / dt / 1e12, unit="TFLOPS", cores=oracle.num_threads(), kind="oracle",
                sample=f"fwd+bwd of the first {S} tokens of KV group 0 ({g} query heads, "
                       f"head_dim {w.head_dim}), fp64 C oracle, {dt:.1f} s"), dt


def config_dict(w: synth.Workload, rotate: str, world: int) -> dict:
    q_mib = w.batch * w.num_heads * w.seq_len * w.head_dim * 2 / 2 ** 20
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seq_len, "cp": w.cp,
            "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
            "rotate": rotate, "mask": "doc" if w.docs else "causal", "merge": "separate",
            "l2": "inputs larger than L2 (Q alone is %.0f MiB)" % q_mib,
            "parallelism": f"replicas x{world}"}


# --------------------------------------------------------------------- native arm

# algorithmic FLOPs per unmasked pair and query head, x D: the forward's two products;
# the one-pass backward's four (dV, dP, dK, dQ; S recomputed, not counted); the
# two-pass backward's dK/dV pass (dP, dV, dK) and dQ pass (dQ)
KERNEL_FLOP_SHARE = {"fwd": 4.0, "bwd_fused": 8.0, "bwd_dkdv": 6.0, "bwd_dq": 2.0}

# DRAM bytes (read + write) per launch of a kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum).
# A figure is reported only while the kernel's source is the one it was taken on:
# first 16 hex digits of the sha256 of the file's code lines (text after "//" and
# blank lines dropped, so comment edits keep it); after any code change it reads
# as null.
MEASURED_TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum (1 pass) on the timed step's
    # dK/dV pass of `bench.py --steps 1 --warmup 3 --no-cpu-baseline` (long128k); the
    # median of three captures (reads 21.7, 25.8 and 31.1 GB)
    ("long128k", "allgather", "bwd_dkdv"): {"bytes": 25.77e9 + 0.67201e9,
                                             "src": "context_zigzag_cp_b200/csrc/bwd.cuh",
                                             "sha256_16": "19777449033dea5b"},
}



def measured_traffic(workload: str, rotate: str, kernel: str):
    import hashlib
    rec = MEASURED_TRAFFIC.get((workload, rotate, kernel))
    if rec is None:
        return None
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), rec["src"])
    try:
        digest = code_digest(path)
    except OSError:
        return None
    return rec["bytes"] if digest == rec["sha256_16"] else None


def code_digest(path: str) -> str:
    """sha256 (16 hex digits) of a source file's code: each line cut at "//" and
    stripped, empty lines dropped."""
    import hashlib
    with open(path, encoding="utf-8") as f:
        lines = [ln.split("//", 1)[0].strip() for ln in f]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()[:16]


def forward_at(args, name, device, dist, peaks, reps=5):
    """The forward alone (cp_attn_fwd, both merge modes) on another workload, so the
    low end of the 32k-128k range is measured in the same run: device time per
    call over `reps` calls after 3 warm-up calls, max over ranks."""
    import torch
    import context_zigzag_cp_b200 as cz
    w = synth.WORKLOADS[name]
    t = synth.workload_inputs(w, device=device, with_dout=False)
    cu = None if t["cu_seqlens"] is None else torch.from_numpy(t["cu_seqlens"]).to(device)
    out = {"workload": name, "rotate": w.rotate}
    prob = cz.Problem(w.batch, w.seq_len, w.cp, w.num_heads, w.num_kv_heads, w.head_dim,
                      w.rotate, cu, merge="separate", shard=w.shard)
    plan = cz.Plan(prob)
    qs, ks, vs = plan.shard([t["q"], t["k"], t["v"]])
    o = torch.empty_like(qs)
    lse = torch.empty(qs.shape[:-1], dtype=torch.float32, device=device)
    ws = torch.empty(max(cz.fwd_workspace_bytes(prob), 256), dtype=torch.uint8, device=device)
    flops = 4.0 * w.head_dim * w.num_heads * int(plan.pairs.sum().item()) * w.batch
    for merge in ("separate", "fused"):
        pr = prob.with_merge(merge)
        for _ in range(3):
            cz.attn_fwd(pr, plan, qs, ks, vs, o, lse, ws=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            cz.attn_fwd(pr, plan, qs, ks, vs, o, lse, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        ms = dist_max(dist, e0.elapsed_time(e1) / reps, device)
        out[merge] = {"ms": round(ms, 3), "tflops": round(flops / 1e9 / ms, 1),
                      "frac_of_peak": round(flops / 1e9 / ms / peaks["bf16"], 4)}
    if cz.get_device_status() != 0:
        raise RuntimeError("device status after the 32k forward")
    return out


def run_native(args, w, rank, world, local_rank):
    import torch
    import context_zigzag_cp_b200 as cz

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if args.wait_limit_ms > 0:
        cz.set_wait_limit_ns(int(args.wait_limit_ms) * 1_000_000)
    dist = dist_init(world, "nccl")
    peaks = load_peaks()
    rotate = args.rotate or w.rotate

    t = synth.workload_inputs(w, device=device, with_dout=True)
    cu = None if t["cu_seqlens"] is None else torch.from_numpy(t["cu_seqlens"]).to(device)
    prob = cz.Problem(w.batch, w.seq_len, w.cp, w.num_heads, w.num_kv_heads, w.head_dim, rotate,
                      cu, merge="separate", shard=w.shard)
    prob_fused = prob.with_merge("fused")
    plan = cz.Plan(prob)
    q, k, v, do = t["q"], t["k"], t["v"], t["do"]
    qs, ks, vs, dos = (torch.empty_like(x) for x in (q, k, v, do))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_f = torch.empty(max(cz.fwd_workspace_bytes(prob), 256), dtype=torch.uint8, device=device)
    ws_b = torch.empty(max(cz.bwd_workspace_bytes(prob), 256), dtype=torch.uint8, device=device)

    def step():
        plan.build([q, k, v, do], [qs, ks, vs, dos])
        cz.attn_fwd(prob, plan, qs, ks, vs, o, lse, ws=ws_f)
        cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos, dq, dk, dv, ws=ws_b)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = cz.get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    pairs_rank = plan.pairs.cpu().to(torch.float64)
    pairs = int(pairs_rank.sum().item()) * w.batch
    # unmasked pairs per virtual rank, max over mean: 1 for the plain causal zigzag;
    # packed documents leave the sequence-level zigzag unbalanced
    rank_imbalance = float(pairs_rank.max() / pairs_rank.mean())
    fwd_flops = 4.0 * w.head_dim * w.num_heads * pairs
    step_flops = 3.0 * fwd_flops

    # ---- timed region: K steps, barrier + synchronize on both sides
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_launch0 = cz.launch_count()
    with ClockSampler(local_rank) as clocks:
        dist_barrier(dist, device)
        torch.cuda.synchronize()
        ev0.record()
        for _ in range(args.steps):
            step()
        ev1.record()
        torch.cuda.synchronize()
        dist_barrier(dist, device)
    launches = (cz.launch_count() - n_launch0)
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = dist_max(dist, ms, device)
    value = aggregate(step_flops / 1e12, world, ms_max)

    # ---- per-kernel times inside one traced step (same stream)
    with cz.LaunchTrace(256) as tr:
        step()
    per = {}
    for name, kms in tr.launches():
        a = per.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += kms
    kernels = {n: {"launches": c, "ms": round(t_, 4)} for n, (c, t_) in per.items()}
    # a share is the step's work of that kernel name over all its launches (at head_dim
    # 256 the dK/dV work is two launches, the dV pass and the dK pass)
    for n, share in KERNEL_FLOP_SHARE.items():
        if n in kernels:
            kernels[n]["tflops"] = round(share * w.head_dim * w.num_heads * pairs /
                                         kernels[n]["ms"] / 1e9, 1)
    # HBM-bound kernels: achieved GB/s from their algorithmic bytes
    rows = w.batch * w.num_heads * w.seq_len
    row_bytes = w.head_dim * 2
    n_q = w.batch * w.num_heads * w.seq_len * row_bytes
    n_kv = w.batch * w.num_kv_heads * w.seq_len * row_bytes
    lse_off = int(round(w.cp * rows * w.head_dim * 4 / 256 + 0.4999)) * 256
    lse_parts = ws_f[lse_off:lse_off + w.cp * rows * 4].view(torch.float32)
    live = int(torch.isfinite(lse_parts).sum().item())
    hbm_bytes = {
        "gather": 2 * (2 * n_q + 2 * n_kv),                       # read + write Q, dO, K, V
        "merge": rows * w.cp * 4 + live * w.head_dim * 4 + rows * (row_bytes + 4),
        # O, dO, LSE in; delta, -LSE*log2(e) out (+ the dQ accumulator zeroed when the
        # step runs the one-pass backward)
        "bwd_prep": rows * (2 * row_bytes + 4) + rows * 8
                    + (rows * w.head_dim * 4 if prob.bwd_one_pass else 0),
        "dq_convert": rows * w.head_dim * (4 + 2),                # fp32 accumulator in, bf16 dQ out
    }
    for n, b in hbm_bytes.items():
        if n in kernels and kernels[n]["ms"] > 0:
            kernels[n]["gbs"] = round(b / (kernels[n]["ms"] * 1e-3) / 1e9, 1)
            kernels[n]["frac_of_hbm_peak"] = round(kernels[n]["gbs"] / peaks["hbm"], 4)
    dom = max(kernels, key=lambda n: kernels[n]["ms"])
    dom_flops = KERNEL_FLOP_SHARE.get(dom, 0.0) * w.head_dim * w.num_heads * pairs
    achieved = dom_flops / kernels[dom]["ms"] / 1e9 if dom_flops else 0.0
    peak = peaks["bf16_sustained"]

    # ---- forward alone, both merge modes (device time of the cp_attn_fwd call), with
    # the clocks of that stretch and the time of each call: the forward alone runs
    # several calls back to back under the power cap, the in-step figure one call
    def time_fwd(pr, n=3):
        cz.attn_fwd(pr, plan, qs, ks, vs, o, lse, ws=ws_f)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        ev[0].record()
        for i in range(n):
            cz.attn_fwd(pr, plan, qs, ks, vs, o, lse, ws=ws_f)
            ev[i + 1].record()
        torch.cuda.synchronize()
        calls = [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
        return sum(calls) / n, calls

    with ClockSampler(local_rank) as fwd_clocks:
        fwd_ms, fwd_calls = time_fwd(prob)
    fwd_ms = dist_max(dist, fwd_ms, device)
    fused_ms = dist_max(dist, time_fwd(prob_fused)[0], device)

    # ---- the backward alone, both forms (one pass with dQ reductions; two passes)
    def time_bwd(pr, n=3):
        wb = torch.empty(max(cz.bwd_workspace_bytes(pr), 256), dtype=torch.uint8, device=device)
        cz.attn_bwd(pr, plan, qs, ks, vs, o, lse, dos, dq, dk, dv, ws=wb)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            cz.attn_bwd(pr, plan, qs, ks, vs, o, lse, dos, dq, dk, dv, ws=wb)
        e1.record()
        torch.cuda.synchronize()
        del wb
        return e0.elapsed_time(e1) / n

    bwd_ms = dist_max(dist, time_bwd(prob), device)
    # the one-pass option exists at head_dim 64 and 128 only
    bwd1_ms = dist_max(dist, time_bwd(prob.with_one_pass(True)), device) if w.head_dim != 256 else None
    fwd_32k = forward_at(args, "gqa32k", device, dist, peaks) if w.name != "gqa32k" else None

    # ---- end to end through the public API with pinned host buffers
    hq, hk, hv, hdo = (x.cpu().pin_memory() for x in (q, k, v, do))
    ho, hl = torch.empty_like(o, device="cpu").pin_memory(), torch.empty_like(lse, device="cpu").pin_memory()
    hdq, hdk, hdv = (torch.empty_like(x, device="cpu").pin_memory() for x in (dq, dk, dv))
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hdo))
    d2h = sum(x.numel() * x.element_size() for x in (ho, hl, hdq, hdk, hdv))

    # The same work as step(), step after step, with the copies pipelined the way a
    # training loop would run them: the device holds two sets of input and gradient
    # buffers, step i+1's Q, K, V, dO go up on a side stream while step i computes
    # (dO last: only the backward waits for it), and step i's O, LSE (during its
    # backward) and dQ, dK, dV (during step i+1) come down on another.  Every step's copies are inside the timed region: it starts
    # before the first upload and ends after the last download has landed.
    main_s = torch.cuda.current_stream(device)
    up_s, down_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ins = [(q, k, v, do), tuple(torch.empty_like(x) for x in (q, k, v, do))]
    grads = [(dq, dk, dv), tuple(torch.empty_like(x) for x in (dq, dk, dv))]
    qkv_ready, do_ready = [None, None], [None, None]
    in_free, grads_out, o_out = [None, None], [None, None], [None]

    def upload(i):
        # Q, K, V first (the forward waits for them), then dO (only the backward does)
        b = i % 2
        with torch.cuda.stream(up_s):
            if in_free[b] is not None:            # step i-2 has gathered these buffers
                up_s.wait_event(in_free[b])
            for dst, src in zip(ins[b][:3], (hq, hk, hv)):
                dst.copy_(src, non_blocking=True)
            qkv_ready[b] = up_s.record_event()
            ins[b][3].copy_(hdo, non_blocking=True)
            do_ready[b] = up_s.record_event()

    def compute(i):
        b = i % 2
        xq, xk, xv, xdo = ins[b]
        main_s.wait_event(qkv_ready[b])
        if o_out[0] is not None:                  # the previous O / LSE have come down
            main_s.wait_event(o_out[0])
        plan.build([xq, xk, xv], [qs, ks, vs])
        cz.attn_fwd(prob, plan, qs, ks, vs, o, lse, ws=ws_f)
        fwd_done = main_s.record_event()
        with torch.cuda.stream(down_s):
            down_s.wait_event(fwd_done)
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            o_out[0] = down_s.record_event()
        main_s.wait_event(do_ready[b])
        plan.build([xdo], [dos])
        in_free[b] = main_s.record_event()
        gq, gk, gv = grads[b]
        if grads_out[b] is not None:              # step i-2's gradients have come down
            main_s.wait_event(grads_out[b])
        cz.attn_bwd(prob, plan, qs, ks, vs, o, lse, dos, gq, gk, gv, ws=ws_b)
        bwd_done = main_s.record_event()
        with torch.cuda.stream(down_s):
            down_s.wait_event(bwd_done)
            hdq.copy_(gq, non_blocking=True)
            hdk.copy_(gk, non_blocking=True)
            hdv.copy_(gv, non_blocking=True)
            grads_out[b] = down_s.record_event()

    def e2e_run(n):
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
        main_s.wait_event(o_out[0])
        for ev in grads_out:
            if ev is not None:
                main_s.wait_event(ev)

    n_e2e = max(2, args.steps)
    e2e_run(2)                                    # warm-up of the same pipeline
    torch.cuda.synchronize()
    dist_barrier(dist, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    e2e_run(n_e2e)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = dist_max(dist, e0.elapsed_time(e1) / n_e2e, device)
    st = cz.get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region")

    out = None
    if rank == 0:
        clk = clocks.summary()
        base, _ = cpu_baseline(w) if not args.no_cpu_baseline else (None, 0)
        out = {
            "metric": "causal CP-attention TFLOPS fwd+bwd on 1 B200",
            "value": round(value, 2),
            "unit": "TFLOPS",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_max, 3),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 Q/K/V/dO)",
            "config": config_dict(w, rotate, world),
            "fwd_tflops": round(fwd_flops / 1e9 / fwd_ms, 1),
            "fwd_frac_of_peak": round(fwd_flops / 1e9 / fwd_ms / peaks["bf16"], 4),
            "fwd_alone_calls_ms": [round(c, 3) for c in fwd_calls],
            "fwd_alone_clocks": fwd_clocks.summary(),
            "fwd_fused_tflops": round(fwd_flops / 1e9 / fused_ms, 1),
            "fwd_fused_frac_of_peak": round(fwd_flops / 1e9 / fused_ms / peaks["bf16"], 4),
            # the forward and its merge as they ran inside the traced step; the figures
            # above time the forward alone, three calls back to back
            "fwd_in_step_tflops": round(fwd_flops / 1e9 / (kernels["fwd"]["ms"] + kernels.get(
                "merge", {"ms": 0.0})["ms"]), 1),
            "fwd_32k": fwd_32k,
            "bwd_tflops": round(2.0 * fwd_flops / 1e9 / bwd_ms, 1),
            "bwd_ms": round(bwd_ms, 3),
            "bwd_one_pass_tflops": round(2.0 * fwd_flops / 1e9 / bwd1_ms, 1) if bwd1_ms else None,
            "bwd_one_pass_ms": round(bwd1_ms, 3) if bwd1_ms else None,
            "step_frac_of_peak": round(value / world / peaks["bf16_sustained"], 4),
            "peak_source": peaks["source"],
            "pairs": pairs,
            "rank_pairs_max_over_mean": round(rank_imbalance, 4),
            "kernels": kernels,
            "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "traffic": measured_traffic(w.name, rotate, dom)},
            "e2e": {"value": round(step_flops * world / 1e9 / e2e_ms, 2), "unit": "TFLOPS",
                    "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "overlap": "inputs of step i+1 up and gradients of step i down while "
                               "step i / i+1 compute (two buffer sets); dO up after Q/K/V "
                               "(the forward waits for Q/K/V only); O/LSE down during the "
                               "backward"},
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": base,
        }
    if dist is not None:
        dist_barrier(dist, device)
        dist.destroy_process_group()
    return out


# --------------------------------------------------------------------- reference arm (oracle)

def run_reference(args, w, rank, world):
    """The oracle timed on the host cores; rank 0 only."""
    if rank != 0:
        return None
    base, _ = cpu_baseline(w)           # warm-up / first call builds the oracle
    vals = []
    for _ in range(args.warmup):
        cpu_baseline(w, budget_tokens=1024)
    for _ in range(args.steps):
        b, dt = cpu_baseline(w, budget_tokens=1536)
        vals.append((b, dt))
    tot_flops = sum(b["value"] * dt for b, dt in vals) * 1e12
    tot_t = sum(dt for _, dt in vals)
    value = tot_flops / tot_t / 1e12
    return {
        "impl": "reference",
        "metric": "causal CP-attention TFLOPS fwd+bwd on 1 B200",
        "value": round(value, 6), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(tot_t / len(vals) * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, args.rotate or w.rotate, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": base["cores"],
                         "kind": "oracle", "sample": vals[0][0]["sample"]},
        "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="long128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--rotate", default=None, choices=["allgather", "ring"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # the kernels' bounded waits give up after 2 s by default; a profiler that
    # instruments them (ncu --set full) can slow a launch past that
    ap.add_argument("--wait-limit-ms", type=int, default=0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local_rank = dist_env()
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        out = run_reference(args, w, rank, world)
    else:
        out = run_native(args, w, rank, world, local_rank)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
