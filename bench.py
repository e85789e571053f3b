#!/usr/bin/env python
"""Benchmark of the KDA forward on B200: chunked prefill and single-token decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]

Prints ONE JSON line on rank 0.

* ``value``: prefill tokens/s of the long-context workload (B=1, H=32,
  T=65536, dk=dv=128, bf16 inputs, fp32 final state), whole job: the tokens
  every rank processed divided by the slowest rank's device time for K steps.
  One step is one ``kda_forward`` over the whole batch (chunk staging, decay
  cumsum and scaling, intra-chunk products, UT solve, inter-chunk scan,
  output, state I/O).  Inputs (3.77 GB per step) are far larger than the
  126 MB L2, so no flush is needed between steps.
* ``decode``: the decode workload (B=256, H=32, d=128, 537 MB fp32 state),
  1024 sequential ``kda_decode_step`` calls timed as one region.
* ``e2e``: the same metrics through the public Python API with host-resident
  pinned inputs: every step copies that step's inputs host->device and reads
  the outputs back device->host inside the timed region.
* ``roofline``: the prefill kernel's algorithmic bytes per launch over its
  CUDA-event launch time, against the measured HBM copy bandwidth.
* ``cpu_baseline``: the fp64 CPU oracle timed on this host on a bounded slice
  of the same workload (rank 0, N=1 only).

With N > 1 (launched by torchrun) every rank runs its own independent batch
of the same size (weak scaling); no collective touches the data path, only
the timing (barrier, max over ranks).

``--impl reference`` times the fp64 CPU oracle instead (the reference arm).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (H32,d128,T64K) & decode tok/s; % of roofline"
HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0

# Algorithmic cost model of the prefill per token and head (d = dk = dv):
# bytes read/written once: q, k, v (input dtype), log_alpha (fp32), beta (fp32), out (fp32).
# FLOPs: 5*C*d + 6*d^2 per token-head with C = 64 (triangular products counted half).
def prefill_bytes_per_token_head(dk, dv, in_bytes):
    return (2 * dk + dv) * in_bytes + 4 * dk + 4 + 4 * dv


def prefill_flops_per_token_head(d, C=64):
    return 5 * C * d + 6 * d * d


def decode_bytes_per_head(dk, dv, in_bytes):
    return 2 * 4 * dk * dv + (2 * dk + dv) * in_bytes + 4 * dk + 4 + 4 * dv


# ncu DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch,
# keyed by (kernel source, workload) -> (source digest at capture, bytes).
# Reported only while the kernel source is unchanged (profiles/ holds the captures).
MEASURED_TRAFFIC = {
    ("kda_decode.cu", "decode_bf16_b256_h32_d128_1024steps"): ("bdf76c3b9b0ab14c", 1.0285e9),
    # captured on B4 H32 T4096 (938.4 MB = 0.979 of its algorithmic bytes) and scaled to
    # the long-context launch by token-heads processed (the kernel streams its inputs once)
    ("kda_prefill_tc.cu", "prefill_bf16_b1_h32_t65536_d128"): ("411803dd646a1f7c", 0.979 * 3768582144),
    ("kda_prefill_tc.cu", "prefill_bf16_b4_h32_t16384_d128_state_T4096"): ("411803dd646a1f7c", 938.4e6),
    # two-kernel prefill, one kda_forward_ws call with the pipelined schedule (blocks of
    # 32, 64 and 32 chunks: prep 187.6, 427.8, 183.2 MB and per-head chain 169.6, 357.8,
    # 171.3 MB), captured on B1 H32 T8192 and scaled by 8 to T = 65536: every term
    # (inputs, chunk records, outputs) grows with the token count
    ("kda_prefill_split.cu", "prefill_bf16_b1_h32_t65536_d128"): ("e1d6d30bca00be24", 8 * 1497.4e6),
    ("kda_prefill_split.cu", "prefill_bf16_b1_h32_t65536_d128_T8192"): ("e1d6d30bca00be24", 1497.4e6),
    # Gated DeltaNet two-kernel prefill (kda_gdn_forward_ws, same schedule): chunk-local
    # kernel 143.2, 344.9, 141.3 MB and the chain's kScalar instance 169.8, 356.4, 171.2 MB
    # on B1 H32 T8192, scaled by 8; the chunk-local kernel lives in kda_prep_scalar.cuh
    ("kda_prefill_split.cu", "gdn_prefill_bf16_b1_h32_t65536_d128"):
        ("e1d6d30bca00be24", 8 * 1326.85e6, {"kda_prep_scalar.cuh": "ad7bde3e303a7b31"}),
}


def measured_traffic(src, workload):
    """Captured bytes per launch while the kernel source (and any header named with
    the entry) is the one the capture ran, else None."""
    ent = MEASURED_TRAFFIC.get((src, workload))
    if ent is None:
        return None
    csrc = os.path.join(ROOT, "gated_delta_rule_109_b200", "csrc")
    same = {src: ent[0], **(ent[2] if len(ent) > 2 else {})}
    return ent[1] if all(source_digest(os.path.join(csrc, f)) == d for f, d in same.items()) else None


def source_digest(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def cpu_model():
    """The host CPU's model name (first processor in /proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, BF16_FALLBACK_TFLOPS, BF16_FALLBACK_TFLOPS, "fallback"


# ---------------------------------------------------------------- multi-rank plumbing
def rank_workload(w, rank):
    """Weak scaling: rank r processes its own independent batch (seed + 1000 r)."""
    from gated_delta_rule_109_b200 import inputs as I
    return I.scaled(w, seed=w.seed + 1000 * rank)


def max_over_ranks(value, device=None):
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def init_distributed(backend="nccl", timeout_s=300):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, local, world


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons, every 200 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        import torch
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.ident = str(device.index or 0)

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="kda_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------- prefill
def bench_prefill(w, K, W, device, gate="channel", workspace=None):
    """K timed launches of the prefill.  gate="channel": KDA (kda_forward, or
    kda_forward_ws when a workspace is given); "scalar": Gated DeltaNet
    (kda_gdn_forward, or kda_gdn_forward_ws) with channel 0 of the draw as the gate."""
    import torch
    import gated_delta_rule_109_b200 as kda
    from gated_delta_rule_109_b200 import inputs as I
    x = I.make_inputs(w, device)
    out = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=device)
    sT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=device) if w.final_state else None
    fwd = kda.forward
    if workspace is not None:
        fwd = lambda *a, **kw: kda.forward(*a, workspace=workspace, **kw)
    if gate == "scalar":
        x["log_alpha"] = x["log_alpha"][..., 0].contiguous()
        fwd = kda.gdn_forward
        if workspace is not None:
            fwd = lambda *a, **kw: kda.gdn_forward(*a, workspace=workspace, **kw)
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    for _ in range(W):
        fwd(*args, out=out, final_state=sT, return_final_state=sT is not None)
    torch.cuda.synchronize(device)
    kda.check_status(device)
    stream = torch.cuda.current_stream(device)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    barrier(device)
    torch.cuda.synchronize(device)
    n0 = kda.launch_count()
    evs[0].record(stream)
    for i in range(K):
        fwd(*args, out=out, final_state=sT, return_final_state=sT is not None)
        evs[i + 1].record(stream)
    torch.cuda.synchronize(device)
    launches = kda.launch_count() - n0
    barrier(device)
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(K)]
    kda.check_status(device)
    # per-head Frobenius norm of the final state (a health diagnostic of the recurrence)
    norms = None
    if sT is not None:
        n = torch.linalg.vector_norm(sT, dim=(-2, -1)).flatten()
        norms = {"max": float(n.max()), "mean": float(n.mean()), "min": float(n.min())}
    return {"ms_total": sum(per), "ms_per_launch": per, "launches": launches, "x": x, "state_norm": norms}


def bench_prefill_e2e(w, K, W, device, x, workspace=None, block_tokens=4096):
    """Same metric through the public API with pinned host inputs, copies inside the
    timed region.  With a workspace: kda_forward_host, which overlaps the copies of
    one block of tokens with the kernels of the next; else device copies around
    kda_forward."""
    import torch
    import gated_delta_rule_109_b200 as kda
    names = ("q", "k", "v", "log_alpha", "beta")
    host = {n: x[n].cpu().pin_memory() for n in names}
    s0h = x["initial_state"].cpu().pin_memory() if x["initial_state"] is not None else None
    out_h = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32).pin_memory()
    sT_h = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32).pin_memory() if w.final_state else None
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + (s0h.numel() * 4 if s0h is not None else 0)
    d2h = out_h.numel() * 4 + (sT_h.numel() * 4 if sT_h is not None else 0)
    host_path = workspace is not None
    if host_path:
        # the host path sizes its own workspace (one block of records)
        hws = torch.empty(kda.forward_host_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype, block_tokens),
                          dtype=torch.uint8, device=device)

        def step():
            kda.forward_host(*(host[n] for n in names), s0h, out=out_h, final_state=sT_h,
                             return_final_state=sT_h is not None, block_tokens=block_tokens, workspace=hws,
                             device=device, synchronize=False)
    else:
        dev = {n: torch.empty_like(x[n]) for n in names}
        s0d = torch.empty_like(x["initial_state"]) if s0h is not None else None
        out = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=device)
        sT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=device) if w.final_state else None

        def step():
            for n in names:
                dev[n].copy_(host[n], non_blocking=True)
            if s0h is not None:
                s0d.copy_(s0h, non_blocking=True)
            kda.forward(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], s0d,
                        out=out, final_state=sT, return_final_state=sT is not None)
            out_h.copy_(out, non_blocking=True)
            if sT is not None:
                sT_h.copy_(sT, non_blocking=True)

    for _ in range(W):
        step()
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    assert torch.isfinite(out_h[0, -1]).all()
    return {"ms_total": e0.elapsed_time(e1), "h2d": h2d, "d2h": d2h,
            "path": "kda_forward_host (copies and kernels overlapped per %d-token block)" % block_tokens
            if host_path else "device copies around kda_forward"}


# ---------------------------------------------------------------- decode
def bench_decode(w, steps, W, device, e2e_steps):
    import torch
    import gated_delta_rule_109_b200 as kda
    from gated_delta_rule_109_b200 import inputs as I
    x = I.make_inputs(w, device, steps=steps)
    state = x["initial_state"].clone()
    outs = torch.empty((steps, w.B, w.H, w.dv), dtype=torch.float32, device=device)

    def run(s, st, o):
        kda.decode_step(x["q"][s], x["k"][s], x["v"][s], x["log_alpha"][s], x["beta"][s], st, out=o)

    warm_state = x["initial_state"].clone()
    for s in range(W):
        run(s % steps, warm_state, outs[s % steps])
    del warm_state
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    n0 = kda.launch_count()
    e0.record(stream)
    for s in range(steps):
        run(s, state, outs[s])
    e1.record(stream)
    torch.cuda.synchronize(device)
    launches = kda.launch_count() - n0
    barrier(device)
    kda.check_status(device)
    ms = e0.elapsed_time(e1)

    # end to end: each step's inputs from pinned host memory, its output read back
    names = ("q", "k", "v", "log_alpha", "beta")
    n_e2e = min(e2e_steps, steps)
    host = {n: x[n][:n_e2e].cpu().pin_memory() for n in names}
    dbuf = {n: torch.empty_like(x[n][0]) for n in names}
    out_h = torch.empty((n_e2e, w.B, w.H, w.dv), dtype=torch.float32).pin_memory()
    h2d = sum(host[n][0].numel() * host[n].element_size() for n in names)
    d2h = w.B * w.H * w.dv * 4
    o = torch.empty((w.B, w.H, w.dv), dtype=torch.float32, device=device)
    st2 = x["initial_state"].clone()
    del x
    torch.cuda.synchronize(device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    f0.record(stream)
    for s in range(n_e2e):
        for n in names:
            dbuf[n].copy_(host[n][s], non_blocking=True)
        kda.decode_step(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["log_alpha"], dbuf["beta"], st2, out=o)
        out_h[s].copy_(o, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    return {"ms": ms, "launches": launches, "e2e_ms": f0.elapsed_time(f1), "e2e_steps": n_e2e,
            "h2d": h2d, "d2h": d2h}


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w, x, budget_s, max_tokens=None, chunk_tokens=2048):
    """Time the fp64 oracle on the first tokens of every head until ``budget_s``."""
    import numpy as np
    import oracle
    T = x["q"].shape[1] if max_tokens is None else min(x["q"].shape[1], max_tokens)
    state = None if x["initial_state"] is None else x["initial_state"].cpu().double().numpy()
    done, elapsed = 0, 0.0
    threads = min(os.cpu_count() or 1, w.B * w.H)
    while done < T and (elapsed < budget_s or done == 0):
        n = min(chunk_tokens, T - done)
        sub = {k: x[k][:, done:done + n].cpu() for k in ("q", "k", "v", "log_alpha", "beta")}
        t0 = time.perf_counter()
        _, state = oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], state,
                                  nthreads=threads)
        elapsed += time.perf_counter() - t0
        done += n
    return {"tokens": done * w.B, "seconds": elapsed, "threads": threads,
            "value": done * w.B / elapsed}


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on this host, bounded per step."""
    rank, _, world = int(os.environ.get("RANK", "0")), 0, int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import torch
    from gated_delta_rule_109_b200 import inputs as I
    w = I.PREFILL_H32_T64K
    per_step = args.ref_tokens_per_step
    steps_total = args.warmup + args.steps
    T = min(w.T, per_step * steps_total)
    ws = I.scaled(w, T=T)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = I.make_inputs(ws, dev)
    x = {k: (v.cpu() if v is not None else None) for k, v in x.items()}
    import oracle
    threads = min(os.cpu_count() or 1, w.B * w.H)
    state = None
    t_timed = 0.0
    for s in range(steps_total):
        lo, hi = (s * per_step) % T, (s * per_step) % T + per_step
        sub = {k: x[k][:, lo:hi] for k in ("q", "k", "v", "log_alpha", "beta")}
        t0 = time.perf_counter()
        _, state = oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], state,
                                  nthreads=threads)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            t_timed += dt
    tokens = per_step * w.B * args.steps
    value = tokens / t_timed
    sample = ("fp64 oracle, %s workload, all %d heads, %d consecutive tokens per step "
              "(state carried), %d threads" % (w.name, w.H, per_step, threads))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t_timed / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "tokens_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model(),
                             "host_cores_online": os.cpu_count()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _add_other_prefills(line, args, world, device, hbm, rank=0):
    """The two other bf16 prefill workloads (B1 H16 T4096; B4 H32 T16384 with a
    carried state), each through kda_forward_ws with its whole-sequence workspace,
    timed like the headline and reported with its own roofline."""
    import torch
    import gated_delta_rule_109_b200 as kda
    from gated_delta_rule_109_b200 import inputs as I
    res = {}
    for base in (I.PREFILL_H16_T4K, I.PREFILL_B4_T16K_STATE):
        w = rank_workload(base, rank)
        nb = kda.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype)
        ws = torch.empty(nb, dtype=torch.uint8, device=device)
        K = max(args.steps, 10)
        pre = bench_prefill(w, K, args.warmup, device, workspace=ws)
        ms_total = max_over_ranks(pre["ms_total"], device)
        ms_launch = statistics.mean(pre["ms_per_launch"])
        alg = (w.B * w.T * w.H * prefill_bytes_per_token_head(w.dk, w.dv, 2)
               + (4 * w.B * w.H * w.dk * w.dv if w.final_state else 0)
               + (4 * w.B * w.H * w.dk * w.dv if w.state_sd is not None else 0))
        achieved = alg / (ms_launch / 1e3) / 1e9
        res[w.name] = {"value": w.B * w.T * K * world / (ms_total / 1e3), "unit": "tokens/s",
                       "ms_per_call": ms_total / K, "steps": K, "gpu_launches": pre["launches"],
                       "path": "kda_forward_ws, whole-sequence workspace (%.2f GB)" % (nb / 1e9),
                       "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                                    "frac": achieved / hbm, "traffic": None,
                                    "algorithmic_bytes_per_launch": alg, "ms_per_launch": ms_launch}}
        del pre, ws
        torch.cuda.empty_cache()
    line["other_prefills"] = res


def _add_decode(line, args, rank, world, device, hbm):
    from gated_delta_rule_109_b200 import inputs as I
    wd = rank_workload(I.DECODE_B256, rank)
    dec = bench_decode(wd, args.decode_steps, args.warmup, device, e2e_steps=64)
    dms = max_over_ranks(dec["ms"], device)
    d_e2e = max_over_ranks(dec["e2e_ms"], device)
    dbytes = wd.B * wd.H * decode_bytes_per_head(wd.dk, wd.dv, 2)
    d_ach = dbytes * args.decode_steps / (dms / 1e3) / 1e9
    line["decode"] = {
        "workload": wd.name, "value": wd.B * args.decode_steps * world / (dms / 1e3),
        "unit": "tokens/s", "steps": args.decode_steps, "ms_per_step": dms / args.decode_steps,
        "gpu_launches": dec["launches"],
        "roofline": {"bound": "hbm", "achieved": d_ach, "peak": hbm, "unit": "GB/s",
                     "frac": d_ach / hbm, "traffic": measured_traffic("kda_decode.cu", wd.name),
                     "kernel": "decode_step_kernel",
                     "algorithmic_bytes_per_launch": dbytes,
                     "vs_8TBs_spec": d_ach / 8000.0},
        "e2e": {"value": wd.B * dec["e2e_steps"] * world / (d_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": dec["h2d"], "d2h_bytes_per_step": dec["d2h"],
                "steps": dec["e2e_steps"]}}


def _add_noalloc(line, args, w, world, device, hbm):
    """The long-context prefill without a caller workspace, each call timed like the
    headline: kda_forward (the two-kernel prefill on a workspace from the library's
    pool), kda_forward_ws with no workspace (the one-kernel prefill) and
    kda_forward_noalloc (the two-kernel prefill on the library's static scratch)."""
    import functools
    import torch
    import gated_delta_rule_109_b200 as kda
    from gated_delta_rule_109_b200 import inputs as I
    x = I.make_inputs(w, device)
    args_ = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["initial_state"])
    out = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=device)
    sT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=device)
    res = {}
    alg = (w.B * w.T * w.H * prefill_bytes_per_token_head(w.dk, w.dv, 2) + 4 * w.B * w.H * w.dk * w.dv)
    calls = (("kda_forward", kda.forward),
             ("kda_forward_ws (no workspace: one kernel)", functools.partial(kda.forward, one_kernel=True)),
             ("kda_forward_noalloc", kda.forward_noalloc))
    for name, fn in calls:
        for _ in range(args.warmup):
            fn(*args_, out=out, final_state=sT)
        torch.cuda.synchronize(device)
        kda.check_status(device)
        stream = torch.cuda.current_stream(device)
        K = max(3, min(args.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(device)
        e0.record(stream)
        for _ in range(K):
            fn(*args_, out=out, final_state=sT)
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms = max_over_ranks(e0.elapsed_time(e1), device) / K
        res[name] = {"ms_per_call": ms, "value": w.B * w.T * world / (ms / 1e3), "unit": "tokens/s",
                     "roofline_frac": alg / (ms / 1e3) / 1e9 / hbm}
    res["scratch_bytes"] = kda.noalloc_scratch_bytes()
    res["pool_bytes"] = kda.workspace_pool_bytes(device)
    line["noalloc_prefill"] = res


def _add_gdn(line, args, w, world, device, hbm, use_workspace=True):
    """The Gated DeltaNet specialisation timed on the same workload shape (the
    two-kernel path with a workspace when the shape has one)."""
    import torch
    import gated_delta_rule_109_b200 as kda
    ws = kda.make_workspace(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype, device=device) if use_workspace else None
    pre = bench_prefill(w, args.steps, args.warmup, device, gate="scalar", workspace=ws)
    del pre["x"]
    del ws
    torch.cuda.empty_cache()
    ms_total = max_over_ranks(pre["ms_total"], device)
    ms_launch = statistics.mean(pre["ms_per_launch"])
    in_bytes = 2 if w.dtype == "bf16" else 4
    per_tok_head = (2 * w.dk + w.dv) * in_bytes + 4 + 4 + 4 * w.dv
    alg_bytes = (w.B * w.T * w.H * per_tok_head
                 + (4 * w.B * w.H * w.dk * w.dv if w.final_state else 0)
                 + (4 * w.B * w.H * w.dk * w.dv if w.state_sd is not None else 0))
    ach = alg_bytes / (ms_launch / 1e3) / 1e9
    tc = (w.dtype == "bf16" and w.dk == 128 and w.dv == 128)
    line["gated_deltanet_prefill"] = {
        "workload": w.name, "gate": "one log_alpha per token and head (channel 0 of the KDA draw)",
        "value": w.B * w.T * args.steps * world / (ms_total / 1e3), "unit": "tokens/s",
        "ms_per_step": ms_total / args.steps, "gpu_launches": pre["launches"],
        "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                     "traffic": (measured_traffic("kda_prefill_split.cu", "gdn_" + w.name)
                                 if tc and use_workspace else None),
                     "kernel": ("prefill_prep_scalar_kernel + prefill_chain_t_kernel<kScalar> (pipelined)"
                                if tc and use_workspace
                                else "prefill_gdn_tc_kernel" if tc else "prefill_simt_kernel"),
                     "algorithmic_bytes_per_launch": alg_bytes}}


def _add_raw(line, args, w, world, device, hbm):
    """The prefill on raw activations (gate pre-activations, unnormalised q and k):
    the steps before the path fused (kda_forward_raw) against the same steps as
    separate torch passes followed by kda_forward_ws."""
    import torch
    import gated_delta_rule_109_b200 as kda
    from gated_delta_rule_109_b200 import inputs as I
    x = I.make_raw_inputs(w, device)
    ws = kda.make_workspace(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype, device=device)
    out = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.float32, device=device)
    sT = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=device)
    names = ("q", "k", "v", "gate", "beta")

    def fused():
        kda.forward_raw(*(x[n] for n in names), x["initial_state"], workspace=ws, out=out, final_state=sT)

    def unfused():
        la = torch.nn.functional.logsigmoid(x["gate"])
        qn = torch.nn.functional.normalize(x["q"].float(), dim=-1).to(x["q"].dtype)
        kn = torch.nn.functional.normalize(x["k"].float(), dim=-1).to(x["k"].dtype)
        kda.forward(qn, kn, x["v"], la, x["beta"], x["initial_state"], out=out, final_state=sT, workspace=ws)

    res = {}
    for name, fn in (("fused", fused), ("unfused", unfused)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(device)
        stream = torch.cuda.current_stream(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(device)
        torch.cuda.synchronize(device)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        res[name] = max_over_ranks(e0.elapsed_time(e1), device) / args.steps
    kda.check_status(device)
    del ws
    tokens = w.B * w.T
    line["raw_activation_prefill"] = {
        "workload": w.name,
        "inputs": "gate pre-activations x ~ N(%g,%g) and unnormalised q, k ~ N(0,1)" % (w.alpha_mu, w.alpha_sd),
        "value": tokens * world / (res["fused"] / 1e3), "unit": "tokens/s",
        "ms_per_step": res["fused"],
        "unfused_ms_per_step": res["unfused"],
        "unfused": "torch logsigmoid + two normalize passes, then kda_forward_ws",
        "kernel": "prefill_prep_kernel (with the fused steps) + prefill_chain_kernel"}


def _add_time_split(line, args, w, device, segments=8):
    """One sequence of the prefill workload cut into `segments` contiguous
    segments (time-axis split), run one after another on this GPU.  Timed: the
    phases of the last segment, the one with the most work (its local run and
    transfer, the fold over all earlier segments, the correction).  Checked: the
    concatenated outputs and the last final state against one kda_forward_ws
    call on the whole sequence."""
    import torch
    import gated_delta_rule_109_b200 as kda
    from gated_delta_rule_109_b200 import inputs as I
    if w.T % segments or w.dk != w.dv:
        return
    Ts = w.T // segments
    x = I.make_inputs(w, device)
    names = ("q", "k", "v", "log_alpha", "beta")
    segs = [{n: x[n][:, r * Ts:(r + 1) * Ts].contiguous() for n in names} for r in range(segments)]
    ws = kda.make_workspace(w.B, Ts, w.H, w.dk, w.dv, w.torch_dtype, device=device, segment=True)
    outs, Ps, Fs, final = [], [], [], None
    for r in range(segments):
        o, lf, P = kda.segment_local(*(segs[r][n] for n in names), x["initial_state"] if r == 0 else None,
                                     workspace=ws)
        final = lf
        if r:
            start = kda.segment_start_state(torch.stack(Ps), torch.stack(Fs))
            final = kda.segment_correct(start, lf, o, workspace=ws)
        outs.append(o); Ps.append(P); Fs.append(lf)
    whole_ws = kda.make_workspace(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype, device=device)
    o_w, s_w = kda.forward(*(x[n] for n in names), x["initial_state"], workspace=whole_ws)
    del whole_ws
    out = torch.cat(outs, dim=1)
    rel = lambda a, b: float((a - b).abs().max() / b.pow(2).mean().sqrt())
    check = {"out": rel(out, o_w), "final_state": rel(final, s_w)}
    del out, o_w, outs

    last = segs[-1]
    Pst, Fst = torch.stack(Ps[:-1]), torch.stack(Fs[:-1])
    phases = {
        "local": lambda: kda.segment_local(*(last[n] for n in names), None, workspace=ws),
        "fold": lambda: kda.segment_start_state(Pst, Fst),
    }
    o_l, lf_l, _ = phases["local"]()
    start = phases["fold"]()
    phases["correct"] = lambda: kda.segment_correct(start, lf_l, o_l, workspace=ws)
    ms = {}
    for name, fn in phases.items():
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(device)
        stream = torch.cuda.current_stream(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms[name] = e0.elapsed_time(e1) / args.steps
    kda.check_status(device)
    per_rank = ms["local"] + ms["fold"] + ms["correct"]
    line["time_split"] = {
        "workload": w.name, "segments": segments, "segment_tokens": Ts,
        "emulation": "segments run one after another on one GPU; per-rank phases timed on the last segment",
        "local_ms": ms["local"], "fold_ms": ms["fold"], "correct_ms": ms["correct"],
        "per_rank_ms_without_exchange": per_rank,
        "exchange_bytes_per_rank": 2 * w.B * w.H * w.dk * w.dv * 4,
        "whole_sequence_ms": line.get("ms_per_step"),
        "max_abs_err_over_rms_vs_whole_sequence": check}


def backward_bytes_per_token_head(dk, dv, in_bytes):
    """Algorithmic HBM bytes of the backward per token and head: q, k (dk) and v (dv)
    in the input dtype, log_alpha (dk) and the output cotangent (dv) in fp32, beta,
    and the fp32 gradients of q, k, v, log_alpha and beta."""
    return in_bytes * (2 * dk + dv) + 4 * (dk + dv) + 4 + 4 * (3 * dk + dv) + 4


def _add_backward(line, args, device, hbm, world=1, w=None):
    """kda_backward on the short-context prefill workload (B1 H16 T4096 d128 bf16):
    every gradient, with the forward inputs and the output cotangent resident."""
    import torch
    import gated_delta_rule_109_b200 as kda
    from gated_delta_rule_109_b200 import inputs as I
    w = w or I.PREFILL_H16_T4K
    x = I.make_inputs(w, device)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 500)
    d_out = torch.randn((w.B, w.T, w.H, w.dv), generator=g, device=device)
    ws = torch.empty(kda.backward_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv), dtype=torch.uint8, device=device)
    names = ("q", "k", "v", "log_alpha", "beta")
    fn = lambda: kda.backward(*(x[n] for n in names), d_out, x["initial_state"], None, workspace=ws)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    n0 = kda.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(device)
    launches = kda.launch_count() - n0
    kda.check_status(device)
    ms = max_over_ranks(e0.elapsed_time(e1), device) / args.steps
    in_bytes = 2 if w.dtype == "bf16" else 4
    alg = w.B * w.T * w.H * backward_bytes_per_token_head(w.dk, w.dv, in_bytes)
    achieved = alg / (ms / 1e3) / 1e9
    line["backward"] = {
        "workload": w.name, "value": w.B * w.T * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
        "gpu_launches": launches,
        "kernels": "bwd_state_kernel + bwd_adjoint_kernel + bwd_chunk_grad_kernel (fp32 CUDA cores)",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": None, "algorithmic_bytes_per_launch": alg,
                     "launch": "one kda_backward call (three kernels)"}}


# ---------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--workload", default="prefill_bf16_b1_h32_t65536_d128",
                    help="prefill workload to time (name from gated_delta_rule_109_b200.inputs)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override T of the prefill workload (profiling runs on a shorter case)")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--ref-tokens-per-step", type=int, default=1024)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "backward"], default="all",
                    help="time only one kernel (profiling runs); the default times both")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workspace", action="store_true",
                    help="time kda_forward without a workspace (the one-kernel prefill)")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the Gated DeltaNet timing on the prefill workload")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        return run_reference(args)

    import torch
    from gated_delta_rule_109_b200 import build as kbuild, inputs as I
    import gated_delta_rule_109_b200 as kda
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    kda.load()          # fails loudly if libkda.so is missing
    rank, local, world = init_distributed()
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d (launch N>1 with torchrun)" % (args.gpus, world))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    byname = {w.name: w for w in I.WORKLOADS}
    w = rank_workload(byname[args.workload], rank)
    if args.seq_len > 0:
        w = I.scaled(w, T=args.seq_len, name=w.name + "_T%d" % args.seq_len)
    hbm, tf_burst, tf_sust, peak_src = load_peaks()
    in_bytes = 2 if w.dtype == "bf16" else 4

    if args.only in ("decode", "backward"):
        line = {"metric": METRIC, "unit": "tokens/s", "n_gpus": world, "impl": "kda", "only": args.only}
        if args.only == "decode":
            _add_decode(line, args, rank, world, device, hbm)
        else:
            _add_backward(line, args, device, hbm, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0

    # the two-kernel prefill's workspace, allocated once outside every timed region
    ws_bytes = 0 if args.no_workspace else kda.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.torch_dtype)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device) if ws_bytes else None
    split = ws is not None

    clocks = ClockSampler(device)
    clocks.start()
    pre = bench_prefill(w, args.steps, args.warmup, device, workspace=ws)
    clk = clocks.stop()
    ms_total = max_over_ranks(pre["ms_total"], device)
    tokens_per_step = w.B * w.T
    value = tokens_per_step * args.steps * world / (ms_total / 1e3)

    # roofline of the prefill kernel (one launch per step)
    ms_launch = statistics.mean(pre["ms_per_launch"])
    alg_bytes = (w.B * w.T * w.H * prefill_bytes_per_token_head(w.dk, w.dv, in_bytes)
                 + (4 * w.B * w.H * w.dk * w.dv if w.final_state else 0)
                 + (4 * w.B * w.H * w.dk * w.dv if w.state_sd is not None else 0))
    achieved = alg_bytes / (ms_launch / 1e3) / 1e9
    tc = (w.dtype == "bf16" and w.dk == 128 and w.dv == 128)   # the library's dispatch rule
    kname, ksrc = ("prefill_tc_kernel", "kda_prefill_tc.cu") if tc else ("prefill_simt_kernel", "kda_prefill_simt.cu")
    # the library's schedule rule: few heads (2 B H <= SMs) and >= 128 chunks pipeline the
    # chunk-local kernel beside a per-head chain; else the chain runs after it
    pipelined = split and 2 * w.B * w.H <= torch.cuda.get_device_properties(device).multi_processor_count \
        and (w.T + 63) // 64 >= 128
    if split:
        kname, ksrc = ("prefill_prep_kernel + prefill_chain_t_kernel (pipelined)" if pipelined
                       else "prefill_prep_kernel + prefill_chain_kernel"), "kda_prefill_split.cu"
    traffic = measured_traffic(ksrc, w.name)
    alg_flops = w.B * w.T * w.H * prefill_flops_per_token_head(w.dk)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic,
                "kernel": kname, "algorithmic_bytes_per_launch": alg_bytes,
                "ms_per_launch": ms_launch,
                "launch": "one kda_forward_ws call (both kernels)" if split else "one kernel launch", "peak_source": peak_src + " HBM copy (MEASURED_PEAKS.json hbm_gbs)",
                "tensor_view": {"algorithmic_flops_per_launch": alg_flops,
                                "achieved_tflops": alg_flops / (ms_launch / 1e3) / 1e12,
                                "peak_tflops": tf_burst,
                                "frac": alg_flops / (ms_launch / 1e3) / 1e12 / tf_burst}}

    e2e = bench_prefill_e2e(w, args.e2e_steps, 1, device, pre["x"], workspace=ws)
    e2e_ms = max_over_ranks(e2e["ms_total"], device)
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(w, pre["x"], args.cpu_budget_s)
    del pre["x"]
    del ws
    torch.cuda.empty_cache()

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if tc else "f32", "data": "synthetic",
            "arithmetic": ("tcgen05 bf16 products of hi/lo-split operands (3 terms), fp32 accumulation "
                           "in tensor memory, fp32 CUDA-core solve and scans") if tc else "fp32 CUDA cores",
            "path": (("two kernels per block of up to 64 chunks (first and last 32), pipelined: the per-head "
                      "state chain of block i "
                      "beside the chunk-local kernel of block i+1 (records in two slots of a %.2f GB caller "
                      "workspace)" if pipelined else
                      "two kernels per call (chunk-local records in a %.2f GB caller workspace, then the "
                      "state chain)") % (ws_bytes / 1e9)) if split else "one fused kernel per call",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "input_dtype": w.dtype, "chunk": 64, "final_state": w.final_state,
                       "l2": "no flush: inputs %.2f GB per step > 126 MB L2" % (alg_bytes / 1e9),
                       "per_rank": "independent batch per rank (seed + 1000*rank)",
                       "inputs": "seeded N(0,1) q,k,v (q,k L2-normalised); log_alpha=logsigmoid(N(%g,%g)); "
                                 "beta=sigmoid(N(%g,%g))" % (w.alpha_mu, w.alpha_sd, w.beta_mu, w.beta_sd)},
            "roofline": roofline,
            "e2e": {"value": tokens_per_step * args.e2e_steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "steps": args.e2e_steps, "path": e2e["path"]},
            "gpu_launches": pre["launches"],
            "clocks": clk,
            "final_state_norm_per_head": pre.get("state_norm")}

    if not args.no_decode and args.only == "all":
        _add_decode(line, args, rank, world, device, hbm)
    if not args.no_variants and args.only == "all":
        _add_other_prefills(line, args, world, device, hbm, rank)
        if ws_bytes:
            _add_noalloc(line, args, w, world, device, hbm)
        _add_gdn(line, args, w, world, device, hbm)
        if ws_bytes:
            _add_raw(line, args, w, world, device, hbm)
            if world == 1:
                _add_time_split(line, args, w, device)
        _add_backward(line, args, device, hbm, world)

    if cb is not None:
        line["cpu_baseline"] = {"value": cb["value"], "unit": "tokens/s", "cores": cb["threads"],
                                "kind": "oracle", "cpu_model": cpu_model(),
                                "host_cores_online": os.cpu_count(),
                                "sample": "fp64 oracle on the first %d tokens of all %d heads of the %s "
                                          "workload (%.1f s)" % (cb["tokens"], w.H, w.name, cb["seconds"])}
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
