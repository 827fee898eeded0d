#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200: chunkwise prefill (headline) and the decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

A step is one ``kda_chunk_fwd`` over the 128K-token, 32-head bf16 workload (B=1, T=131072,
H=32, d_k=d_v=128, chunk 64, fp32 state, S0 ~ N(0, 0.1^2)); the decode step (256 sequences x 32
heads, 512 MiB fp32 state, 1000 consecutive steps) is measured in the same run and reported
under ``decode``. Inputs are synthetic (``kda_inputs``), resident in HBM before timing; one step
reads 5.4 GB of inputs, far more than the 126 MB L2, so no flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs its own copy of the workload: the
heads and sequences are independent, so there is no collective on the data path (weak scaling);
only the timing uses a MAX all-reduce. ``--impl reference`` times the float64 CPU oracle on a
bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_inputs as K  # noqa: E402

METRIC = "KDA prefill Mtok/s @T=128K,H=32 (% TC peak); decode-step HBM GB/s vs peak"
WORKLOAD = "bf16_t128k_h32"
DECODE = "decode_n256_h32"
C = 64
D = 128
# algorithmic HBM bytes per token*head of the prefill: q, k, v bf16 (3 x 256 B), out bf16
# (256 B; the output takes the inputs' dtype), log_alpha fp32 (512 B), beta fp32 (4 B)
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * D * 2 + D * 2 + D * 4 + 4
# kernels one prefill step launches: the chunk-preparation pass and the state scan
# the same algorithmic bytes, split by the pass that moves them: the preparation pass reads q, k,
# log_alpha and beta; the scan reads v and writes out (its other traffic is the workspace)
PREP_BYTES_PER_TOKEN_HEAD = 2 * D * 2 + D * 4 + 4
SCAN_BYTES_PER_TOKEN_HEAD = D * 2 + D * 2
# DRAM traffic per token*head measured by Nsight Compute (profiles/dram_traffic.json), valid for
# the kernel source it was taken from
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
CSRC = os.path.join(ROOT, "kimi_delta_attention_25_b200", "csrc")
# useful tensor flops per token*head (chunk C): 6 d^2 (W.S, Q.S, Kend^T.U) + 5 C d (triangular
# K K^T, Q K^T, T.(beta K), T.(beta V), M.U) + C^2 / 3 (triangular inverse)
PREFILL_FLOPS_PER_TOKEN_HEAD = 6 * D * D + 5 * C * D + C * C // 3
# backward (kda_chunk_bwd, fp32 arithmetic on CUDA cores): flops per (64-token chunk, head) that
# each of its three phases must do in this design, triangular products counted once
# (TRI = a 64 x 64 triangle times 128 columns, FULL = 64 x 128 x 128, 2 flops per multiply-add):
#   forward records: A, the solve for U (TRI each); Kt S, Ke^T U (FULL each) (for bf16 inputs the
#                    forward's tensor-core passes do this work; the count is the fp32 design's)
#   state gradient:  A (with Kt Kh^T, kept for the per-chunk kernel), M, M^T dO, the solves for Y0
#                    and Kp (TRI); Qt^T dO, then per chunk of the reverse scan Kp dS' and Bk^T Y (FULL)
#   per chunk:       dO U^T, Y U^T, dM Kh, dP Kh, dM^T Qt, dP^T Kt (TRI); dO S^T, Y S^T, U dS'^T (FULL)
BWD_TRI = C * C // 2 * D * 2
BWD_FULL = C * D * D * 2
BWD_FLOPS_PER_CHUNK_HEAD = {"bwd_forward_records": 2 * BWD_TRI + 2 * BWD_FULL,
                            "bwd_scan": 5 * BWD_TRI + 3 * BWD_FULL,
                            "bwd_local": 6 * BWD_TRI + 3 * BWD_FULL}
# algorithmic HBM bytes per token*head: q, k, v, dout bf16 and log_alpha, beta read; dq, dk, dv,
# dlog_alpha, dbeta fp32 written
BWD_BYTES_PER_TOKEN_HEAD = 4 * D * 2 + D * 4 + 4 + 4 * D * 4 + 4
# fp32 FMA peak of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz (max SM clock)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# decode: state read + written once per step
DECODE_STATE_BYTES_PER_HEAD = 2 * D * D * 4
DECODE_IO_BYTES_PER_HEAD = 3 * D * 2 + D * 4 + 4 + D * 4


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sus=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.p is None:
            return False
        time.sleep(0.2)
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
            out, _ = self.p.communicate()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                self.rows.append(f)
        return False

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            for i, n in enumerate(names):
                if "Active" in r[5 + i] and "Not" not in r[5 + i]:
                    reasons.add(n)
        # median under load: drop idle samples below half of max
        top = max(mx) if mx else None
        load = [s for s in sm if top is None or s > 0.3 * top] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": top,
                "reasons": sorted(reasons), "samples": len(self.rows)}


def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x, ws):
    from kimi_delta_attention_25_b200 import shard
    return shard.max_over_ranks(x, device="cuda") if ws > 1 else x


def measured_traffic(kernel, unit="dram_bytes_per_token_head"):
    """DRAM bytes per unit of `kernel` from the committed ncu summary, or None when the kernel's
    source has changed since the counters were taken."""
    import hashlib
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)[kernel]
        with open(os.path.join(CSRC, t["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    return float(t[unit]) if sha == t["source_sha256"] else None


def time_loop(fn, steps, warmup, ws):
    """CUDA-event time of `steps` calls of fn on the current stream, after `warmup` calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    barrier(ws)
    return s.elapsed_time(e) / steps      # ms per call


# ---------------------------------------------------------------------------------------------

def cpu_oracle_sample(budget_s=12.0, workload=WORKLOAD):
    """Times the float64 oracle (as it stands) on a bounded sample of a prefill workload:
    the first T' tokens of H' heads, with T' sized from a short calibration run so that the
    whole sample takes about `budget_s` seconds on all host cores. Returns a dict in Mtok/s."""
    from oracle import ref
    cores = ref.online_cores()
    w = K.WORKLOADS[workload]
    Hs = w.H
    cal_T = 1024
    def run(d, nthreads):
        args = [d[x].float().numpy() for x in ("q", "k", "v", "log_alpha", "beta")]
        S0 = None if d["S0"] is None else d["S0"].double().numpy()
        cu = None if d["cu_seqlens"] is None else d["cu_seqlens"].numpy()
        t0 = time.perf_counter()
        ref.forward(*args, S0=S0, cu_seqlens=cu, nthreads=nthreads)
        return time.perf_counter() - t0

    per_tok_head = run(K.make_prefill(w, T=cal_T, H=1), 1) / cal_T
    Ts = int(max(1024, min(w.T, budget_s / per_tok_head * min(Hs, cores) / Hs)))
    Ts -= Ts % C
    dt = run(K.make_prefill(w, T=Ts, H=Hs), min(Hs, cores))
    tok_equiv = Ts * Hs / w.H                 # tokens of the full 32-head workload
    return {"value": tok_equiv / dt / 1e6, "unit": "Mtok/s", "cores": min(Hs, cores),
            "kind": "oracle",
            "sample": "float64 C recurrence on the first %d tokens of %d of the %d heads "
                      "(%.1f s; scaled to tokens of all %d heads)" % (Ts, Hs, w.H, dt, w.H),
            "seconds": dt, "host_cores": cores}


def cpu_oracle_backward_sample(tokens=8192):
    """Times the float64 backward oracle (token-level reverse sweep, numpy, one thread) as it
    stands on the first `tokens` tokens of one head of the prefill workload; scaled to tokens of
    the full 32-head workload per second."""
    from oracle import backward as bw
    w = K.WORKLOADS[WORKLOAD]
    d = K.make_prefill(w, T=tokens, H=1)
    g = torch.Generator().manual_seed(1234)
    dout = torch.randn(d["v"].shape, generator=g).to(torch.bfloat16)
    f = lambda t: t.float().numpy()  # noqa: E731
    t0 = time.perf_counter()
    bw.backward(f(d["q"]), f(d["k"]), f(d["v"]), f(d["log_alpha"]), f(d["beta"]), f(dout),
                S0=d["S0"].double().numpy())
    dt = time.perf_counter() - t0
    return {"value": tokens / w.H / dt / 1e6, "unit": "Mtok/s", "cores": 1, "kind": "oracle",
            "sample": "float64 numpy reverse sweep on the first %d tokens of 1 of the %d heads "
                      "(%.1f s; scaled to tokens of all %d heads)" % (tokens, w.H, dt, w.H),
            "seconds": dt}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = K.WORKLOADS[WORKLOAD]
    vals = []
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(budget_s=budget)
        if i >= args.warmup:
            vals.append(r)
    v = statistics.median([r["value"] for r in vals])
    ms = w.T / (v * 1e6) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "Mtok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": w.T, "heads": w.H,
                       "head_dim": D, "chunk": C, "parallelism": "none (host cores)"},
            "cpu_baseline": {"kind": "oracle", "cores": vals[-1]["cores"], "sample": vals[-1]["sample"],
                             "value": v, "unit": "Mtok/s"},
            "e2e": {"value": v, "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------

def run_native(args):
    ws, rank, local = dist_setup(args.gpus)
    import kimi_delta_attention_25_b200 as kda
    kda.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()
    w = K.WORKLOADS[WORKLOAD]
    from kimi_delta_attention_25_b200 import shard
    d = K.make_prefill(w, device=dev, seed=shard.rank_seed(w.seed, rank))
    B, T, H = w.B, w.T, w.H
    out = torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev)
    Sf = torch.empty(B, H, D, D, dtype=torch.float32, device=dev)
    wsz = kda.chunk_fwd_workspace_size(B, T, H, B)
    work = torch.empty(max(256, wsz), dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"],
                      out=out, S_final=Sf, workspace=work)

    def prep():
        kda.chunk_prep(d["q"], d["k"], d["log_alpha"], d["beta"], work)

    def scan():
        kda.chunk_scan(d["v"], work, S0=d["S0"], out=out, S_final=Sf)

    step()
    torch.cuda.synchronize()
    assert kda.workspace_status(work) == kda.KDA_OK
    # the step is the public call (one timed step = one chunk_fwd); each pass is also timed alone
    ms, ms_prep, ms_scan, clk = time_prefill(kda, ws, args, step, prep, scan, args.steps, local)
    assert kda.workspace_status(work) == kda.KDA_OK
    launches = kda.chunk_fwd_kernel_launches(B, T, H, B)
    tokens = B * T
    value = ws * tokens / (ms * 1e-3) / 1e6                   # Mtok/s, whole job
    th = B * T * H
    alg_bytes = th * PREFILL_BYTES_PER_TOKEN_HEAD
    flops = th * PREFILL_FLOPS_PER_TOKEN_HEAD
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    tfs = flops / (ms * 1e-3) / 1e12
    kern = {}
    for name, t_ms, per in (("chunk_prep", ms_prep, PREP_BYTES_PER_TOKEN_HEAD),
                            ("chunk_scan", ms_scan, SCAN_BYTES_PER_TOKEN_HEAD)):
        tr = measured_traffic(name)
        a = th * per / (t_ms * 1e-3) / 1e9
        kern[name] = {"ms": t_ms, "achieved": a, "frac": a / pk["hbm"],
                      "algorithmic_bytes_per_launch": th * per,
                      "traffic": None if tr is None else tr * th}
    dom = max(kern, key=lambda k: kern[k]["ms"])

    # ---- end to end through the public call with pinned host buffers
    host = {x: d[x].cpu().pin_memory() for x in ("q", "k", "v", "log_alpha", "beta", "S0")}
    dbuf = {x: torch.empty_like(d[x]) for x in host}
    h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h_sf = torch.empty(Sf.shape, dtype=Sf.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = h_out.numel() * h_out.element_size() + h_sf.numel() * h_sf.element_size()

    def e2e_step():
        for x in host:
            dbuf[x].copy_(host[x], non_blocking=True)
        kda.chunk_fwd(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["log_alpha"], dbuf["beta"],
                      S0=dbuf["S0"], out=out, S_final=Sf, workspace=work)
        h_out.copy_(out, non_blocking=True)
        h_sf.copy_(Sf, non_blocking=True)

    e2e_steps = max(1, min(args.steps, 5))
    ms_e2e = max_over_ranks(time_loop(e2e_step, e2e_steps, 1, ws), ws)
    e2e_val = ws * tokens / (ms_e2e * 1e-3) / 1e6
    del host, dbuf, h_out, h_sf

    # ---- the same workload as a full layer step (gate producers and output norm fused)
    del work
    torch.cuda.empty_cache()
    layer_step = run_layer_step(kda, dev, pk, ws, rank, args, d)

    # ---- the other prefill workloads: 8K tokens x 16 heads, and 8 packed sequences (262K tokens)
    other = {name: run_prefill_config(kda, dev, pk, ws, rank, args, name, 6.0)
             for name in ("bf16_t8k_h16", "bf16_varlen8_262k_h32")}

    # ---- decode step
    dec = run_decode(kda, dev, pk, ws, local, args)

    # ---- backward of the same prefill
    bwd = run_backward(kda, dev, pk, ws, local, args, d)

    del d, out
    torch.cuda.empty_cache()
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample()
        bwd["cpu_baseline"] = cpu_oracle_backward_sample()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Mtok/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": ws * B, "seq_len": T, "heads": H,
                       "head_dim": D, "chunk": C, "state": "fp32", "gates": "fp32", "out": "bf16",
                       "l2": "inputs larger than L2 (5.4 GB read per step), no flush",
                       "parallelism": "dp%d (independent heads/sequences per GPU)" % ws},
            "roofline": {"bound": "hbm", "achieved": kern[dom]["achieved"], "peak": pk["hbm"],
                         "unit": "GB/s", "frac": kern[dom]["frac"], "traffic": kern[dom]["traffic"],
                         "peak_source": "of %s" % pk["src"], "kernel": dom,
                         "ms_per_launch": kern[dom]["ms"],
                         "algorithmic_bytes_per_launch": kern[dom]["algorithmic_bytes_per_launch"],
                         "kernels": kern,
                         "step": {"achieved": gbs, "frac": gbs / pk["hbm"],
                                  "algorithmic_bytes": alg_bytes,
                                  "tensor_tflops_useful": tfs, "tensor_frac_useful": tfs / pk["bf16"]}},
            "e2e": {"value": e2e_val, "unit": "Mtok/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
            "gpu_launches": args.steps * launches,
            "clocks": clk.summary(),
            "layer_step": layer_step,
            "configs": other,
            "decode": dec,
            "backward": bwd,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def time_prefill(kda, ws, args, fwd, prep, scan, steps, local):
    """Times `steps` calls of the public prefill call fwd() between a barrier + synchronize on both
    sides (the step; with few (sequence, head) chains the library runs its two passes as a
    pipeline over token ranges, so they overlap inside the call), then the two passes alone, each
    between CUDA events on the launching stream, for the per-kernel rooflines. Returns the step time
    (max over ranks), the mean time of each pass and the clock record of the step's timed region."""
    with Clocks(local) as clk:
        for _ in range(args.warmup):
            fwd()
        torch.cuda.synchronize()
        barrier(ws)
        torch.cuda.synchronize()
        t_s, t_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_s.record()
        for _ in range(steps):
            fwd()
        t_e.record()
        torch.cuda.synchronize()
        barrier(ws)
    ms = max_over_ranks(t_s.elapsed_time(t_e) / steps, ws)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    prep()
    scan()
    for ev in evs:
        ev[0].record()
        prep()
        ev[1].record()
        scan()
        ev[2].record()
    torch.cuda.synchronize()
    ms_prep = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    ms_scan = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    return ms, ms_prep, ms_scan, clk


def run_prefill_config(kda, dev, pk, ws, rank, args, name, cpu_budget_s):
    """One more prefill workload (two passes, bf16 outputs), timed like the headline step: Mtok/s,
    the roofline of each pass and of the step, and the oracle on a bounded sample of it."""
    from kimi_delta_attention_25_b200 import shard
    w = K.WORKLOADS[name]
    d = K.make_prefill(w, device=dev, seed=shard.rank_seed(w.seed, rank))
    B, T, H = w.B, w.T, w.H
    cu = d.get("cu_seqlens")
    N = B if cu is None else cu.shape[0] - 1
    if cu is not None:
        cu = cu.to(dev)
    out = torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev)
    Sf = torch.empty(N, H, D, D, dtype=torch.float32, device=dev)
    work = torch.empty(max(256, kda.chunk_fwd_workspace_size(B, T, H, N)), dtype=torch.uint8, device=dev)
    steps = max(3, args.steps)

    def fwd():
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], cu_seqlens=cu,
                      out=out, S_final=Sf, workspace=work)

    def prep():
        kda.chunk_prep(d["q"], d["k"], d["log_alpha"], d["beta"], work, cu_seqlens=cu)

    def scan():
        kda.chunk_scan(d["v"], work, S0=d["S0"], cu_seqlens=cu, out=out, S_final=Sf)

    ms, ms_prep, ms_scan, clk = time_prefill(kda, ws, args, fwd, prep, scan, steps,
                                             int(os.environ.get("LOCAL_RANK", "0")))
    assert kda.workspace_status(work) == kda.KDA_OK
    th = B * T * H
    kern = {}
    for kname, t_ms, per in (("chunk_prep", ms_prep, PREP_BYTES_PER_TOKEN_HEAD),
                             ("chunk_scan", ms_scan, SCAN_BYTES_PER_TOKEN_HEAD)):
        a = th * per / (t_ms * 1e-3) / 1e9
        kern[kname] = {"ms": t_ms, "achieved": a, "frac": a / pk["hbm"]}
    gbs = th * PREFILL_BYTES_PER_TOKEN_HEAD / (ms * 1e-3) / 1e9
    tfs = th * PREFILL_FLOPS_PER_TOKEN_HEAD / (ms * 1e-3) / 1e12
    res = {"workload": name, "tokens": B * T, "heads": H, "sequences": N, "ms_per_step": ms,
           "Mtok_s": ws * B * T / (ms * 1e-3) / 1e6, "steps": steps, "out": "bf16",
           "l2": "inputs %.2f GB per step (%s L2)" % (th * PREFILL_BYTES_PER_TOKEN_HEAD / 1e9,
                                                      "larger than" if th * 1540 > 126e6 else "within"),
           "roofline": {"bound": "hbm", "peak": pk["hbm"], "unit": "GB/s", "peak_source": "of %s" % pk["src"],
                        "kernels": kern,
                        "step": {"achieved": gbs, "frac": gbs / pk["hbm"], "tensor_tflops_useful": tfs,
                                 "tensor_frac_useful": tfs / pk["bf16"]}},
           "gpu_launches": steps * kda.chunk_fwd_kernel_launches(B, T, H, N), "clocks": clk.summary()}
    del d, out, Sf, work
    torch.cuda.empty_cache()
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_oracle_sample(budget_s=cpu_budget_s, workload=name)
    return res


# the layer step: q, k, v, out bf16 (4 x 256 B), the decay-gate input f bf16 (256 B) in place of
# fp32 log_alpha, the write-gate logits bf16 (2 B) in place of fp32 beta, the output gate g bf16 (256 B)
LAYER_BYTES_PER_TOKEN_HEAD = 4 * D * 2 + D * 2 + 2 + D * 2


def run_layer_step(kda, dev, pk, ws, rank, args, d):
    """The same 128K x 32 prefill as a full KDA layer step: gates produced inside the preparation
    pass from f, A_log, dt_bias and the beta logits, and the gated RMSNorm applied in the scan's
    output epilogue; bf16 outputs. Timed like the headline step (the public call, and each pass
    alone)."""
    B, T, H = d["v"].shape[:3]
    lay = K.make_layer_inputs(B, T, H, dtype="bf16", device=dev, seed=5)
    opts = dict(lay, norm_eps=1e-5)
    out = torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev)
    Sf = torch.empty(B, H, D, D, dtype=torch.float32, device=dev)
    work = torch.empty(max(256, kda.chunk_fwd_workspace_size(B, T, H, B)), dtype=torch.uint8, device=dev)
    steps = max(3, args.steps)

    def fwd():
        kda.chunk_fwd(d["q"], d["k"], d["v"], None, None, S0=d["S0"], out=out, S_final=Sf, workspace=work,
                      layer=opts)

    def prep():
        kda.chunk_prep(d["q"], d["k"], None, None, work, layer=opts)

    def scan():
        kda.chunk_scan(d["v"], work, S0=d["S0"], out=out, S_final=Sf, layer=opts)

    ms, ms_prep, ms_scan, clk = time_prefill(kda, ws, args, fwd, prep, scan, steps,
                                             int(os.environ.get("LOCAL_RANK", "0")))
    assert kda.workspace_status(work) == kda.KDA_OK
    th = B * T * H
    gbs = th * LAYER_BYTES_PER_TOKEN_HEAD / (ms * 1e-3) / 1e9
    kern = {"chunk_prep_gates": {"ms": ms_prep}, "chunk_scan_norm": {"ms": ms_scan}}
    del out, Sf, work, lay, opts
    torch.cuda.empty_cache()
    return {"workload": WORKLOAD, "ms_per_step": ms, "Mtok_s": ws * B * T / (ms * 1e-3) / 1e6, "steps": steps,
            "fused": "decay gate from f, A_log, dt_bias and beta from logits in the preparation pass; "
                     "gated RMSNorm (sigmoid gate) in the scan's output epilogue",
            "algorithmic_bytes_per_token_head": LAYER_BYTES_PER_TOKEN_HEAD,
            "roofline_step": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                              "frac": gbs / pk["hbm"], "peak_source": "of %s" % pk["src"]},
            "kernels": kern, "gpu_launches": steps * kda.chunk_fwd_kernel_launches(B, T, H, B),
            "clocks": clk.summary()}


def run_decode(kda, dev, pk, ws, local, args):
    w = K.WORKLOADS[DECODE]
    N, H = w.B, w.H
    S = K.make_decode_state(w, device=dev)
    nsteps = w.decode_steps
    xs = [K.make_decode_step(w, s, device=dev) for s in range(nsteps)]
    out = torch.empty(N, H, D, dtype=torch.float32, device=dev)
    it = [0]

    def one():
        x = xs[it[0] % nsteps]
        it[0] += 1
        kda.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, out=out)

    with Clocks(local) as clk:
        ms = time_loop(one, nsteps, 5, ws)
    ms = max_over_ranks(ms, ws)

    # the same 1000 launches captured once in a CUDA graph and replayed (launch overhead removed)
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        with torch.cuda.graph(g, stream=cs):
            for x in xs:
                kda.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, out=out)
    torch.cuda.current_stream().wait_stream(cs)
    g.replay()
    torch.cuda.synchronize()
    gs, ge = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gs.record()
    g.replay()
    ge.record()
    torch.cuda.synchronize()
    ms_graph = max_over_ranks(gs.elapsed_time(ge) / nsteps, ws)
    del g
    heads = N * H
    state_b = heads * DECODE_STATE_BYTES_PER_HEAD
    io_b = heads * DECODE_IO_BYTES_PER_HEAD
    us = ms * 1e3
    gbs = state_b / (ms * 1e-3) / 1e9
    return {"workload": DECODE, "us_per_step": us, "steps": nsteps,
            "graph_us_per_step": ms_graph * 1e3,
            "state_gbs": gbs, "total_gbs": (state_b + io_b) / (ms * 1e-3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": gbs / pk["hbm"], "peak_source": "of %s" % pk["src"],
                         "traffic": (lambda t: None if t is None else t * heads)(
                             measured_traffic("decode", "dram_bytes_per_head"))},
            "tokens_per_s_whole_job": ws * N / (ms * 1e-3),
            "gpu_launches": nsteps, "clocks": clk.summary()}


def run_backward(kda, dev, pk, ws, local, args, d):
    """kda_chunk_bwd on the headline workload (gradients of every input for a random output
    gradient and final-state gradient), its three kernels timed one by one with CUDA events."""
    B, T, H = d["v"].shape[:3]
    g = torch.Generator(device=dev).manual_seed(1234)
    dout = torch.randn(B, T, H, D, generator=g, device=dev).to(torch.bfloat16)
    dSf = torch.randn(B, H, D, D, generator=g, device=dev)
    args_ = (d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout)
    kw = dict(S0=d["S0"], dS_final=dSf)
    grads, work = kda.chunk_bwd(*args_, **kw, return_workspace=True)
    torch.cuda.synchronize()
    assert kda.workspace_status(work) == kda.KDA_OK
    steps = max(1, min(args.steps, 3))
    names = ("bwd_forward_records", "bwd_scan", "bwd_local")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]

    def step(ev=None):
        for p in range(3):
            if ev is not None:
                ev[p].record()
            kda.chunk_bwd(*args_, **kw, grads=grads, workspace=work, phase=p)
        if ev is not None:
            ev[3].record()

    with Clocks(local) as clk:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        barrier(ws)
        torch.cuda.synchronize()
        t_s, t_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_s.record()
        for i in range(steps):
            step(evs[i])
        t_e.record()
        torch.cuda.synchronize()
        barrier(ws)
    assert kda.workspace_status(work) == kda.KDA_OK
    ms = max_over_ranks(t_s.elapsed_time(t_e) / steps, ws)
    chunk_heads = B * (T // C) * H
    kern = {}
    for p, name in enumerate(names):
        t_ms = statistics.mean(e[p].elapsed_time(e[p + 1]) for e in evs)
        fl = chunk_heads * BWD_FLOPS_PER_CHUNK_HEAD[name]
        a = fl / (t_ms * 1e-3) / 1e12
        kern[name] = {"ms": t_ms, "achieved": a, "frac": a / FP32_ALU_TFLOPS, "flops_per_launch": fl}
    dom = max(kern, key=lambda k: kern[k]["ms"])
    th = B * T * H
    gbs = th * BWD_BYTES_PER_TOKEN_HEAD / (ms * 1e-3) / 1e9
    del grads, work, dout
    torch.cuda.empty_cache()
    return {"workload": WORKLOAD, "ms_per_step": ms, "Mtok_s": ws * B * T / (ms * 1e-3) / 1e6,
            "steps": steps, "grads": "fp32", "arithmetic": "fp32 (CUDA cores)",
            "roofline": {"bound": "alu", "achieved": kern[dom]["achieved"], "peak": FP32_ALU_TFLOPS,
                         "unit": "TFLOP/s", "frac": kern[dom]["frac"], "traffic": None,
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz",
                         "kernel": dom, "ms_per_launch": kern[dom]["ms"],
                         "flops_per_launch": kern[dom]["flops_per_launch"], "kernels": kern,
                         "step": {"hbm_gbs_algorithmic": gbs, "hbm_frac": gbs / pk["hbm"],
                                  "algorithmic_bytes": th * BWD_BYTES_PER_TOKEN_HEAD}},
            "gpu_launches": 3 * steps, "clocks": clk.summary()}


def run_profile_case(args):
    """One small invocation for Nsight Compute captures: `step` runs the headline step (the public
    call kda_chunk_fwd, full size) `--steps` times; `prefill` runs the two passes kda_chunk_prep and
    kda_chunk_scan, one full launch each, on the first `--tokens` tokens of the 32-head bf16 workload
    (inputs > L2, a few GB at most) twice;
    `backward` runs kda_chunk_bwd twice on the same tokens; `decode` runs 8 decode steps of the
    256 x 32 decode workload."""
    import kimi_delta_attention_25_b200 as kda
    kda.load()
    dev = torch.device("cuda", 0)
    if args.profile == "step":
        # the headline step as timed (the public call, bf16 outputs), full size, `--steps` times
        w = K.WORKLOADS[WORKLOAD]
        d = K.make_prefill(w, device=dev)
        out = torch.empty(w.B, w.T, w.H, D, dtype=torch.bfloat16, device=dev)
        Sf = torch.empty(w.B, w.H, D, D, dtype=torch.float32, device=dev)
        ws = torch.empty(kda.chunk_fwd_workspace_size(w.B, w.T, w.H, w.B), dtype=torch.uint8, device=dev)
        for _ in range(args.steps):
            kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], out=out, S_final=Sf,
                          workspace=ws)
        torch.cuda.synchronize()
        assert kda.workspace_status(ws) == kda.KDA_OK
    elif args.profile == "prefill":
        w = K.WORKLOADS[WORKLOAD]
        d = K.make_prefill(w, device=dev, T=args.tokens)
        ws = torch.empty(kda.chunk_fwd_workspace_size(w.B, args.tokens, w.H, w.B), dtype=torch.uint8, device=dev)
        for _ in range(2):
            kda.chunk_prep(d["q"], d["k"], d["log_alpha"], d["beta"], ws)
            kda.chunk_scan(d["v"], ws, S0=d["S0"], out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        assert kda.workspace_status(ws) == kda.KDA_OK
    elif args.profile == "backward":
        w = K.WORKLOADS[WORKLOAD]
        d = K.make_prefill(w, device=dev, T=args.tokens)
        g = torch.Generator(device=dev).manual_seed(1234)
        dout = torch.randn(d["v"].shape, generator=g, device=dev).to(torch.bfloat16)
        for _ in range(2):
            _, ws = kda.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout, S0=d["S0"],
                                  return_workspace=True)
        torch.cuda.synchronize()
        assert kda.workspace_status(ws) == kda.KDA_OK
    else:
        w = K.WORKLOADS[DECODE]
        S = K.make_decode_state(w, device=dev)
        xs = [K.make_decode_step(w, s, device=dev) for s in range(8)]
        for x in xs:
            kda.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
        torch.cuda.synchronize()
    print("profile case %s done" % args.profile)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["step", "prefill", "decode", "backward"], default=None,
                    help="run one small case for an Nsight Compute capture instead of the benchmark")
    ap.add_argument("--tokens", type=int, default=32768, help="tokens of the --profile prefill case")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
