#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet chunked-prefill operator on B200.

One step = one pass of the operator over one batch of the dense bf16 workload
(B=4, T=4096, H=16, dk=dv=128): gdn_chunk_fwd, and with STEP = "fwdbwd" also
gdn_chunk_bwd on the same inputs with incoming gradients dO, dhT. In the fwd+bwd step the
forward also writes the bf16 chunk start states (gdn_options.states) and the backward
reads them instead of recomputing its forward pass. Inputs are synthetic (seeded, see the workloads module)
and resident in HBM when the timed region starts; the working set is larger
than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--mode fwd]

Prints one JSON line (rank 0). Under torchrun each rank runs its own replica
(the operator shards by independent (sequence, head) units; no collective on
the data path) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_chunked_prefill_b200.workloads import CONFIGS, make_inputs  # noqa: E402

METRIC = "GDN chunk fwd/bwd tokens/s and TFLOP/s on 1 B200; % of roofline"
WORKLOAD = "dense_bf16"
STEP = "fwdbwd"       # what one step runs: "fwd" or "fwdbwd"
C = 64


def flops(w, fwd=True, bwd=True):
    """Chunked-algorithm FLOPs: dense GEMMs at 2 flop/MAC, triangular inverse C^3/3 MAC/chunk."""
    ntok = w.B * w.T
    gemm_v = 6 * w.dk * w.dv + 2 * C * (w.dk + 2 * w.dv)      # per token per v-head
    gram = 4 * C * w.dk                                       # per token per q/k head
    inv = (2.0 / 3.0) * C * C                                 # per token per v-head
    f = ntok * (w.Hv * (gemm_v + inv) + w.Hqk * gram)
    b = ntok * (2 * (w.Hv * gemm_v + w.Hqk * gram) + w.Hv * 4 * C * C)
    return (f if fwd else 0.0) + (b if bwd else 0.0)


def alg_bytes(w, fwd=True, bwd=True):
    """Algorithmic minimum bytes: every input read once, every output written once."""
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T
    qk = ntok * w.Hqk * w.dk * es
    vv = ntok * w.Hv * w.dv * es
    gb = ntok * w.Hv * (4 + es)
    st = w.num_seqs * w.Hv * w.dk * w.dv * 4
    h0 = st if w.h0_std is not None else 0
    f = 2 * qk + vv + gb + h0 + vv + st                       # q k v g beta h0 | o hT
    b = 2 * qk + vv + gb + h0 + vv + st + 2 * qk + vv + gb + h0   # + dO dhT | dq dk dv dg dbeta dh0
    return (f if fwd else 0) + (b if bwd else 0)


def kernel_alg_bytes(w):
    """Algorithmic bytes of one launch of each kernel (inputs read once, outputs written once;
    scratch such as the per-chunk states is not counted), per the workload."""
    es = 2 if w.dtype == "bf16" else 4
    ntok = w.B * w.T
    qk = ntok * w.Hqk * w.dk * es            # q or k (or dq, dk)
    vv = ntok * w.Hv * w.dv * es             # v, o, dO or dv
    gb = ntok * w.Hv * (4 + es)              # g and beta (or dg, dbeta)
    st = w.num_seqs * w.Hv * w.dk * w.dv * 4
    h0 = st if w.h0_std is not None else 0
    return {
        # forward call: q k v g beta h0 -> o hT ; the backward's state pass reads the same inputs
        "gdn_fwd_tc_kernel": [2 * qk + vv + gb + h0 + vv + st, 2 * qk + vv + gb + h0],
        # reverse chain: q k dO g beta dhT -> dh0
        "gdn_bwd_chain_kernel": [2 * qk + vv + gb + st + st],
        # gradients: q k v dO g beta -> dq dk dv dg dbeta
        "gdn_bwd_grad_kernel": [2 * qk + 2 * vv + gb + 2 * qk + vv + gb],
    }


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) every 20 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.time(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.02)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if not inside:
            inside, window = self.samples, "warmup+timed"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = float(np.median([s[1] for s in inside]))
        bits = 0
        for s in inside:
            bits |= int(s[2])
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(inside), "window": window}


def traffic_record(kernel_name, workload, mode):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary of the same workload and
    step, if its sources are unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        recs = json.load(fh)
    for r in recs:
        if r.get("kernel") == kernel_name and r.get("workload") == workload and r.get("step") == mode:
            if sources_sha(r["sources"]) != r.get("sources_sha256_16"):
                return None                      # the kernel changed since the capture
            return float(r["bytes_per_launch"])
    return None


def sources_sha(paths):
    """First 16 hex digits of the SHA-256 of the concatenated files' code (None if one is missing).
    Comments, trailing blanks and empty lines are dropped first, so that only a change of code
    invalidates a capture."""
    h = hashlib.sha256()
    for rel in paths:
        path = os.path.join(ROOT, rel)
        if not os.path.exists(path):
            return None
        with open(path) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        for line in text.splitlines():
            line = re.sub(r"//.*$", "", line).rstrip()
            if line:
                h.update(line.encode() + b"\n")
    return h.hexdigest()[:16]


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The largest value of x over all ranks (the step time of the slowest rank)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank times its own replica of the workload, drawn from its own seed."""
    return base + 17 * rank


# ------------------------------------------------------------------------------------- oracle arm
def oracle_sample(w, x, mode, budget_s):
    """Time the fp64 oracle on whole (sequence, head) units of the workload until `budget_s`."""
    from oracle import bwd_token, fwd_chunk  # the CPU baseline is the oracle as it stands
    hq_of = lambda j: j // (w.Hv // w.Hqk)
    units, tok, t0 = 0, 0, time.perf_counter()
    if x["cu_seqlens"] is not None:         # packed: sequence n is tokens cu[n]..cu[n+1] of batch row 0
        cu = x["cu_seqlens"].tolist()
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    else:
        spans = [(n, 0, w.T) for n in range(w.B)]
    order = [(n, j) for n in range(len(spans)) for j in range(w.Hv)]
    for n, j in order:
        bi, s0, e0 = spans[n]
        sl = lambda a, h: a[bi:bi + 1, s0:e0, h:h + 1]
        q, k, v = sl(x["q"], hq_of(j)), sl(x["k"], hq_of(j)), sl(x["v"], j)
        g, b = sl(x["g"], j), sl(x["beta"], j)
        h0 = None if x["h0"] is None else x["h0"][n:n + 1, j:j + 1]
        fwd_chunk(q, k, v, g, b, x["scale"], h0, chunk=C)
        if mode == "fwdbwd":
            bwd_token(q, k, v, g, b, x["scale"], sl(x["dO"], j), h0, x["dhT"][n:n + 1, j:j + 1])
        units += 1
        tok += e0 - s0
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    # one workload token carries all Hv heads: unit-tokens / Hv = workload tokens
    return (tok / w.Hv) / el, el, units, tok


def run_reference(args, w, x):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cores = 1
    per_step = []
    for _ in range(args.warmup):
        oracle_sample(w, x, args.mode, budget_s=0.0)
    for _ in range(args.steps):
        v, el, units, unit_tok = oracle_sample(w, x, args.mode, budget_s=0.0)
        per_step.append(el)
    tok = unit_tok / w.Hv
    value = tok * len(per_step) / sum(per_step)
    sample = f"one (sequence, head) unit of {unit_tok} tokens per step ({args.mode}), fp64 numpy oracle"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * sum(per_step) / len(per_step), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.description + f"; step = {args.mode}", "mode": args.mode},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------------------------- GPU arm
# Decode step workload: a serving batch whose fp32 states (268 MB) exceed the 126 MB L2.
DECODE = dict(N=256, Hqk=16, Hv=16, dk=128, dv=128)


def decode_bytes(N, Hqk, Hv, dk, dv):
    """Algorithmic bytes of one decode step (bf16 I/O): each state read and written once (fp32),
    v, o, g, beta per v-head and q, k per q/k head once."""
    return N * Hv * (2 * dk * dv * 4 + 2 * dv * 2 + 4 + 2) + N * Hqk * 2 * dk * 2


def decode_oracle_sample(x, Hv, budget_s):
    """The fp64 oracle's token form, one token of 8 sequences per repetition, for `budget_s`."""
    from oracle import fwd_token  # the CPU baseline is the oracle as it stands
    n_s = 8
    t0 = time.time()
    reps = 0
    while reps == 0 or time.time() - t0 < budget_s:
        fwd_token(x["q"][:n_s], x["k"][:n_s], x["v"][:n_s], x["g"][:n_s], x["beta"][:n_s], x["scale"],
                  x["h0"][:n_s])
        reps += 1
    el = time.time() - t0
    return {"value": n_s * reps / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n_s} sequences x {Hv} heads, one token each, fp64 numpy oracle, {reps} reps, {el:.1f} s"}


def run_decode(args):
    """One step = gdn_recurrent_step over every sequence of the batch (one token each). With
    --impl reference the oracle's token form alone is timed (rank 0)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    c = DECODE
    if args.impl == "reference":
        if rank != 0:
            return
        x = make_inputs(c["N"], 1, c["Hqk"], c["Hv"], c["dk"], c["dv"], "bf16", 2000, h0_std=0.1)
        cpu = decode_oracle_sample(x, c["Hv"], 5.0)
        print(json.dumps({"impl": "reference", "metric": "GDN recurrent decode step tokens/s on 1 B200; % of HBM "
                          "roofline", "value": cpu["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                          "steps": 1, "warmup": 0, "higher_is_better": True, "scaling": "weak",
                          "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                          "config": {"workload": "decode step (oracle sample)", "step": "decode"},
                          "cpu_baseline": cpu, "e2e": {"value": cpu["value"], "unit": "tokens/s",
                                                       "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return
    import gated_deltanet_chunked_prefill_b200 as gdn

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    N, Hqk, Hv, dk, dv = c["N"], c["Hqk"], c["Hv"], c["dk"], c["dv"]
    x = make_inputs(N, 1, Hqk, Hv, dk, dv, "bf16", rank_seed(2000, rank), h0_std=0.1)
    tok = {n: x[n][:, 0].contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")}
    state = x["h0"].to(dev)
    o = torch.empty((N, Hv, dv), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.gdn_recurrent_step(tok["q"], tok["k"], tok["v"], tok["g"], tok["beta"], state, x["scale"], o=o)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if args.single:
        step()
        torch.cuda.synchronize()
        return
    sampler = ClockSampler(local)
    sampler.start()
    n0 = gdn.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    tw0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    tw1 = time.time()
    if dist:
        dist.barrier()
    sampler.stop()
    launches = gdn.launch_count() - n0
    ms_step = max_over_ranks(ev0.elapsed_time(ev1), dist, dev) / args.steps
    hbm, _, src = peaks()
    nbytes = decode_bytes(N, Hqk, Hv, dk, dv)
    gbs = nbytes / (ms_step / 1e3) / 1e9
    # the oracle's token form on a bounded sample of the same batch (rank 0, N = 1 only)
    cpu = decode_oracle_sample(x, Hv, min(args.cpu_budget, 5.0)) \
        if rank == 0 and world == 1 and args.cpu_budget > 0 else None
    if rank == 0:
        line = {"metric": "GDN recurrent decode step tokens/s on 1 B200; % of HBM roofline",
                "value": N * world / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": f"decode step: {N} sequences, Hqk={Hqk} Hv={Hv}, dk=dv={dk}, bf16 I/O, "
                                       f"fp32 state", "step": "decode", "parallelism": "single" if world == 1
                           else f"replicas{world}", "l2": "states (268 MB) larger than the 126 MB L2; no flush"},
                "roofline": {"bound": "hbm", "kernel": "gdn_step_kernel", "achieved": gbs, "peak": hbm,
                             "unit": "GB/s", "frac": gbs / hbm, "peak_source": src,
                             "traffic": traffic_record("gdn_step_kernel", "decode", "decode"),
                             "alg_bytes_per_launch": nbytes, "avg_launch_ms": ms_step},
                "cpu_baseline": cpu, "gpu_launches": launches, "clocks": sampler.summary(tw0, tw1)}
        print(json.dumps(line))
    if dist:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--mode", default=STEP, choices=["fwd", "fwdbwd", "decode"],
                    help="decode: the recurrent decode step on its own batch (a separate line)")
    ap.add_argument("--single", action="store_true",
                    help="only warm-up steps plus one step, no report (for profiler launch lists)")
    ap.add_argument("--workload", default=WORKLOAD, choices=list(CONFIGS))
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle CPU baseline")
    ap.add_argument("--cp", type=int, default=0, help="cp_segment_chunks option (0 = automatic)")
    args = ap.parse_args()

    w = CONFIGS[args.workload]
    if args.mode == "decode":
        run_decode(args)
        return
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        x = make_inputs(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.seed, h0_std=w.h0_std, lengths=w.lengths,
                        backward=True)
        run_reference(args, w, x)
        return

    import gated_deltanet_chunked_prefill_b200 as gdn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    x = make_inputs(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, rank_seed(w.seed, rank), h0_std=w.h0_std,
                    lengths=w.lengths,
                    backward=True)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    stream = torch.cuda.current_stream(dev)

    mode = args.mode

    ws_f = torch.zeros(gdn.fwd_workspace_size(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.num_seqs, args.cp),
                       dtype=torch.uint8, device=dev)
    states = gdn.chunk_states(d["q"], d["v"], d["cu_seqlens"]) if mode == "fwdbwd" else None
    ws_b = torch.zeros(gdn.bwd_workspace_size(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.num_seqs, args.cp,
                                              states=states), dtype=torch.uint8, device=dev)
    o = torch.empty_like(d["v"])
    hT = torch.empty((w.num_seqs, w.Hv, w.dk, w.dv), dtype=torch.float32, device=dev)

    def step(dd):
        gdn.gdn_chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["scale"], dd["h0"],
                          dd["cu_seqlens"], cp_segment_chunks=args.cp, workspace=ws_f, o=o, hT=hT, states=states)
        if mode == "fwdbwd":
            return gdn.gdn_chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["dO"], dd["scale"],
                                     dd["h0"], dd["dhT"], dd["cu_seqlens"], cp_segment_chunks=args.cp,
                                     workspace=ws_b, states=states)
        return None

    # ---- device-resident timing
    for _ in range(max(args.warmup, 3)):
        step(d)
    torch.cuda.synchronize()
    if args.single:
        step(d)
        torch.cuda.synchronize()
        return
    if dist:
        dist.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    n0 = gdn.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    tw0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step(d)
    ev1.record(stream)
    torch.cuda.synchronize()
    tw1 = time.time()
    if dist:
        dist.barrier()
    sampler.stop()
    launches = gdn.launch_count() - n0
    ms = max_over_ranks(ev0.elapsed_time(ev1), dist, dev)
    ms_step = ms / args.steps
    tokens = w.B * w.T * world
    value = tokens / (ms_step / 1e3)

    # ---- per-kernel times (CUDA events on the launch stream, library-recorded)
    per_kernel = {}
    with gdn.KernelTrace(capacity=64) as tr:
        for _ in range(5):
            step(d)
    for name, t in tr.launches:
        per_kernel.setdefault(name, []).append(t)
    fwd_ms = bwd_ms = None
    with gdn.KernelTrace(capacity=64) as trf:
        for _ in range(5):
            gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                              d["cu_seqlens"], cp_segment_chunks=args.cp, workspace=ws_f, o=o, hT=hT, states=states)
    fwd_ms = sum(t for _, t in trf.launches) / 5
    bwd_recompute_ms = None
    if mode == "fwdbwd":
        bwd_ms = sum(t for _, t in tr.launches) / 5 - fwd_ms
        # the backward alone once more, recomputing the chunk states itself (no cache)
        ws_r = torch.zeros(gdn.bwd_workspace_size(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.num_seqs, args.cp),
                           dtype=torch.uint8, device=dev)
        with gdn.KernelTrace(capacity=64) as trb:
            for _ in range(5):
                gdn.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["scale"], d["h0"],
                                  d["dhT"], d["cu_seqlens"], cp_segment_chunks=args.cp, workspace=ws_r)
        bwd_recompute_ms = sum(t for _, t in trb.launches) / 5
        del ws_r

    hbm, tc_peak, src = peaks()
    # per-launch algorithmic bytes, matched to the launches of one step in order
    kb = kernel_alg_bytes(w)
    seen = {}
    per_kernel_bytes = {}
    for name, t in tr.launches[: len(tr.launches) // 5]:
        k = seen.get(name, 0)
        seen[name] = k + 1
        opts = kb.get(name)
        if opts:
            per_kernel_bytes.setdefault(name, []).append(opts[min(k, len(opts) - 1)])
    dom = max(per_kernel, key=lambda k: sum(per_kernel[k]))
    dom_ms = float(np.mean(per_kernel[dom]))
    dom_bytes = float(np.mean(per_kernel_bytes.get(dom, [0])))
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_source": src,
                "traffic": traffic_record(dom, args.workload, mode),
                "alg_bytes_per_launch": dom_bytes, "avg_launch_ms": dom_ms}
    step_bytes = alg_bytes(w, fwd=True, bwd=mode == "fwdbwd")
    step_roofline = {"alg_bytes": step_bytes, "achieved_gbs": step_bytes / (ms_step / 1e3) / 1e9,
                     "frac_hbm": step_bytes / (ms_step / 1e3) / 1e9 / hbm,
                     "tflops": flops(w, fwd=True, bwd=mode == "fwdbwd") / (ms_step / 1e3) / 1e12,
                     "frac_tensor": flops(w, fwd=True, bwd=mode == "fwdbwd") / (ms_step / 1e3) / 1e12 / tc_peak}

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region
    host_in = {k: x[k].pin_memory() for k in ("q", "k", "v", "g", "beta", "h0", "dO", "dhT", "cu_seqlens")
               if x.get(k) is not None}
    dev_in = {k: torch.empty_like(d[k]) for k in host_in}
    dev_in["scale"] = d["scale"]
    for k in ("h0", "dO", "dhT", "cu_seqlens"):
        dev_in.setdefault(k, None)
    h2d = sum(t.numel() * t.element_size() for k, t in host_in.items()
              if mode == "fwdbwd" or k not in ("dO", "dhT"))
    out_host = {"o": torch.empty(o.shape, dtype=o.dtype, pin_memory=True),
                "hT": torch.empty(hT.shape, dtype=hT.dtype, pin_memory=True)}

    def e2e_step():
        for k, t in host_in.items():
            if mode == "fwdbwd" or k not in ("dO", "dhT"):
                dev_in[k].copy_(t, non_blocking=True)
        gr = step(dev_in)
        out_host["o"].copy_(o, non_blocking=True)
        out_host["hT"].copy_(hT, non_blocking=True)
        nbytes = o.numel() * o.element_size() + hT.numel() * 4
        if gr is not None:
            for k2, t2 in gr.items():
                if t2 is None:
                    continue
                if k2 not in out_host:
                    out_host[k2] = torch.empty(t2.shape, dtype=t2.dtype, pin_memory=True)
                out_host[k2].copy_(t2, non_blocking=True)
                nbytes += t2.numel() * t2.element_size()
        return nbytes

    for _ in range(2):
        d2h = e2e_step()
    torch.cuda.synchronize()
    e_steps = max(3, min(args.steps, 20))
    if dist:
        dist.barrier()
    ev0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(ev0.elapsed_time(ev1), dist, dev)
    e2e = {"value": tokens / (e_ms / e_steps / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    # ---- CPU baseline: the oracle on the host cores (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_budget > 0:
        v_cpu, el, units, unit_tok = oracle_sample(w, x, mode, args.cpu_budget)
        cpu = {"value": v_cpu, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{units} (sequence, head) units, {unit_tok} unit-tokens of the same workload "
                         f"({mode}), fp64 numpy oracle, {el:.1f} s"}

    fl = flops(w, fwd=True, bwd=mode == "fwdbwd") * world
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": w.description, "step": mode, "global_batch": w.B * world,
                      "seq_len": w.T, "heads_qk": w.Hqk, "heads_v": w.Hv, "dk": w.dk, "dv": w.dv,
                      "chunk": C, "parallelism": f"replicas x{world}" if world > 1 else "single",
                      "l2": "working set larger than the 126 MB L2; no flush",
                      "bwd_states": "cached by the forward (bf16 chunk start states)" if mode == "fwdbwd" else None,
                      "cp_segment_chunks": args.cp},
           "tflops": fl / (ms_step / 1e3) / 1e12,
           "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "bwd_recompute_ms": bwd_recompute_ms,
           "per_kernel_ms": {k: float(np.mean(v)) for k, v in per_kernel.items()},
           "roofline": roofline, "step_roofline": step_roofline, "cpu_baseline": cpu, "e2e": e2e,
           "gpu_launches": int(launches),
           "clocks": sampler.summary(tw0, tw1)}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
