#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet chunked-prefill operator on B200.

Headline step: one pass of the whole operator -- gdn_chunk_fwd then gdn_chunk_bwd -- over the
packed variable-length workload (24 sequences, 65536 tokens, H=16, dk=dv=128, bf16), the largest
single-GPU configuration. The forward writes the chunk-state cache (gdn_options.states) and the
backward reads it. Inputs are synthetic (seeded, see the workloads module) and resident in HBM
when the timed region starts; the working set is larger than the 126 MB L2.

The same JSON line carries, under "per_config", every named workload measured the same way:
the tiny fp32 forward, the dense forward, the long grouped-value forward (context parallelism),
the packed forward, the backward configuration (backward alone, reading the forward's cache;
its forward is timed separately) and the recurrent decode step. Each entry has its roofline
fraction (the slower of bf16 tensor peak and HBM bytes, against the measured peaks), the
dominant kernel's achieved bandwidth, an end-to-end number through the public API with host
buffers, and the fp64 oracle timed on a bounded sample on all host cores.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--only NAME]

Prints one JSON line (rank 0). Under torchrun each rank runs its own replica (the operator
shards by independent (sequence, head) units; no collective on the data path) and the time is
the max over ranks.
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
HEADLINE = ("varlen_bf16", "fwdbwd")
# (workload, step) of the per-configuration entries; "bwd" = backward alone with the cache
SUBS = [("tiny_fp32", "fwd"), ("tiny_fp32", "bwd"), ("dense_bf16", "fwd"), ("long_gqa_bf16", "fwd"),
        ("varlen_bf16", "fwd"), ("bwd_bf16", "bwd")]
C = 64
L2_BYTES = 126 * 1024 * 1024
# datasheet peaks of a B200 (HGX), reported beside the measured ones
DATASHEET_HBM_GBS, DATASHEET_BF16_TFLOPS = 7700.0, 2250.0


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
    fwd_call = 2 * qk + vv + gb + h0 + vv + st
    return {
        # forward call: q k v g beta h0 -> o hT ; the backward's state pass reads the same inputs
        "gdn_fwd_tc_kernel": [fwd_call, 2 * qk + vv + gb + h0],
        "gdn_fwd_simt_kernel": [fwd_call],
        # reverse chain: q k dO g beta dhT -> dh0
        "gdn_bwd_chain_kernel": [2 * qk + vv + gb + st + st],
        # gradients: q k v dO g beta -> dq dk dv dg dbeta
        "gdn_bwd_grad_kernel": [2 * qk + 2 * vv + gb + 2 * qk + vv + gb],
        # CUDA-core backward (fp32, head dims 64), one launch: q k v g beta h0 dO dhT -> dq dk dv dg dbeta dh0
        "gdn_bwd_simt_kernel": [2 * qk + 2 * vv + gb + h0 + st + 2 * qk + vv + gb + st],
    }


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def roofline_fraction(w, step, ms):
    """Fraction of the roofline time (the slower of bf16 tensor peak and HBM bytes) that one step
    of `ms` milliseconds reaches, against the measured peaks and against the datasheet ones."""
    fwd, bwd = step in ("fwd", "fwdbwd"), step in ("bwd", "fwdbwd")
    fl, by = flops(w, fwd, bwd), alg_bytes(w, fwd, bwd)
    hbm, tc, src = peaks()
    fp32_tc = w.dtype == "f32"       # fp32 I/O runs on CUDA cores; its flops are still counted on bf16 peak
    t_hbm, t_tc = by / (hbm * 1e9), fl / (tc * 1e12)
    t_dhbm, t_dtc = by / (DATASHEET_HBM_GBS * 1e9), fl / (DATASHEET_BF16_TFLOPS * 1e12)
    t = ms / 1e3
    return {"alg_bytes": by, "alg_flop": fl, "bound": "hbm" if t_hbm >= t_tc else "tensor",
            "roofline_ms": 1e3 * max(t_hbm, t_tc), "frac": max(t_hbm, t_tc) / t,
            "frac_datasheet": max(t_dhbm, t_dtc) / t, "achieved_gbs": by / t / 1e9,
            "achieved_tflops": fl / t / 1e12, "peak_source": src,
            "note": "fp32 I/O on CUDA cores" if fp32_tc else None}


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


# ------------------------------------------------------------------------------ oracle (CPU) legs
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _pool_init():
    # one BLAS thread per worker: the pool itself spreads the units over the cores
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def make_pool(cores: int):
    """Worker processes for the oracle, forked before this process touches CUDA (a pool forked
    after the first GPU call is not safe)."""
    import multiprocessing as mp
    return mp.get_context("fork").Pool(cores, initializer=_pool_init)


def _oracle_unit(task):
    """One (sequence, v-head) unit through the oracle as it stands; returns its token count."""
    from oracle import bwd_token, fwd_chunk, fwd_token  # the CPU baseline is the oracle as it stands
    kind, a = task
    if kind == "decode":
        fwd_token(a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"], a["h0"])
        return a["q"].shape[0]
    ex = lambda t: None if t is None else t[None, :, None]
    q, k, v, g, b = ex(a["q"]), ex(a["k"]), ex(a["v"]), ex(a["g"]), ex(a["beta"])
    h0 = None if a["h0"] is None else a["h0"][None, None]
    if kind in ("fwd", "fwdbwd"):
        fwd_chunk(q, k, v, g, b, a["scale"], h0, chunk=C)
    if kind in ("bwd", "fwdbwd"):
        bwd_token(q, k, v, g, b, a["scale"], ex(a["dO"]), h0, a["dhT"][None, None])
    return a["q"].shape[0]


def unit_tasks(w, x, mode, order_seed=0, by_sequence=False):
    """Oracle tasks, one per (sequence, v-head) unit of the workload, in a fixed shuffled order
    (a bounded sample then covers short and long packed sequences alike). by_sequence: the
    sequences in shuffled order, each with its v-heads in order (consecutive units have equal
    lengths)."""
    f32 = lambda t: None if t is None else t.float().numpy()
    hq_of = lambda j: j // (w.Hv // w.Hqk)
    if x["cu_seqlens"] is not None:
        cu = x["cu_seqlens"].tolist()
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    else:
        spans = [(n, 0, w.T) for n in range(w.B)]
    if by_sequence:
        seqs = list(range(len(spans)))
        np.random.default_rng(order_seed).shuffle(seqs)
        units = [(n, j) for n in seqs for j in range(w.Hv)]
    else:
        units = [(n, j) for n in range(len(spans)) for j in range(w.Hv)]
        np.random.default_rng(order_seed).shuffle(units)
    for n, j in units:
        bi, s0, e0 = spans[n]
        a = {"q": f32(x["q"][bi, s0:e0, hq_of(j)]), "k": f32(x["k"][bi, s0:e0, hq_of(j)]),
             "v": f32(x["v"][bi, s0:e0, j]), "g": f32(x["g"][bi, s0:e0, j]),
             "beta": f32(x["beta"][bi, s0:e0, j]), "scale": x["scale"],
             "h0": None if x["h0"] is None else f32(x["h0"][n, j])}
        if mode in ("bwd", "fwdbwd"):
            a["dO"] = f32(x["dO"][bi, s0:e0, j])
            a["dhT"] = f32(x["dhT"][n, j])
        yield (mode, a)


def oracle_run(pool, tasks, budget_s, max_units=None):
    """Run oracle tasks on the pool, at most one per worker in flight, submitting until
    `budget_s` seconds have passed (or `max_units` were submitted); waits for those in flight.
    Returns (unit-tokens, seconds, units)."""
    cores = pool._processes
    t0 = time.perf_counter()
    inflight, done_tok, units, submitted = [], 0, 0, 0
    it = iter(tasks)
    exhausted = False
    while True:
        while (not exhausted and len(inflight) < cores and time.perf_counter() - t0 < budget_s
               and (max_units is None or submitted < max_units)):
            try:
                task = next(it)
            except StopIteration:
                exhausted = True
                break
            inflight.append(pool.apply_async(_oracle_unit, (task,)))
            submitted += 1
        if not inflight:
            break
        ready = [r for r in inflight if r.ready()]
        if not ready:
            time.sleep(0.002)
            continue
        for r in ready:
            done_tok += r.get()
            units += 1
            inflight.remove(r)
    return done_tok, time.perf_counter() - t0, units


def cpu_baseline(pool, w, x, mode, budget_s):
    tok, el, units = oracle_run(pool, unit_tasks(w, x, mode), budget_s)
    return {"value": (tok / w.Hv) / el, "unit": "tokens/s", "cores": pool._processes, "kind": "oracle",
            "sample": f"{units} (sequence, v-head) units, {tok} unit-tokens of this workload ({mode}), "
                      f"fp64 numpy oracle, {pool._processes} processes, {el:.1f} s; tokens/s counts a "
                      f"workload token as all {w.Hv} v-heads"}


def run_reference(args, pool):
    """The oracle as it stands on the host cores, on the headline workload: each step runs one
    (sequence, v-head) unit per core, v-heads of one sequence together (equal lengths), the
    sequences in a fixed shuffled order."""
    name, mode = HEADLINE
    w = CONFIGS[name]
    x = make_inputs(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.seed, h0_std=w.h0_std, lengths=w.lengths,
                    backward=True)
    cores = pool._processes
    tasks = iter(unit_tasks(w, x, mode, by_sequence=True))
    for _ in range(args.warmup):
        oracle_run(pool, tasks, 1e9, max_units=cores)
    tok_all, t_all, units_all = 0, 0.0, 0
    for _ in range(args.steps):
        tok, el, units = oracle_run(pool, tasks, 1e9, max_units=cores)
        tok_all, t_all, units_all = tok_all + tok, t_all + el, units_all + units
    value = (tok_all / w.Hv) / t_all
    sample = (f"{units_all} (sequence, v-head) units ({tok_all} unit-tokens) of the packed workload, "
              f"{cores} v-heads of one sequence per step on {cores} processes ({mode}), fp64 numpy oracle")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * t_all / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.description + f"; step = {mode}", "step": mode},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------------------------- GPU arm
# Decode step workloads: serving batches whose fp32 states (268 MB) exceed the 126 MB L2.
DECODE = dict(N=256, Hqk=16, Hv=16, dk=128, dv=128)
DECODE_256 = dict(N=64, Hqk=16, Hv=16, dk=256, dv=256)


def decode_bytes(N, Hqk, Hv, dk, dv):
    """Algorithmic bytes of one decode step (bf16 I/O): each state read and written once (fp32),
    v, o, g, beta per v-head and q, k per q/k head once."""
    return N * Hv * (2 * dk * dv * 4 + 2 * dv * 2 + 4 + 2) + N * Hqk * 2 * dk * 2


def time_steps(step, steps, stream, flush=None):
    """Device time of `steps` calls of step() in ms per step: one event pair around all of them,
    or, with `flush` (a buffer larger than L2), one pair per step with the buffer rewritten between
    steps (outside the pairs)."""
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps
    pairs = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        pairs.append((e0, e1))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in pairs]))


class Case:
    """One workload on the device: its inputs, the step a measurement times, and the same step
    end to end from pinned host buffers."""

    def __init__(self, gdn, name, mode, dev, rank, cp):
        self.gdn, self.name, self.mode, self.dev, self.cp = gdn, name, mode, dev, cp
        self.w = w = CONFIGS[name]
        self.x = make_inputs(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, rank_seed(w.seed, rank),
                             h0_std=w.h0_std, lengths=w.lengths, backward=mode != "fwd")
        self.d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.x.items()}
        d = self.d
        self.o = torch.empty_like(d["v"])
        self.hT = torch.empty((w.num_seqs, w.Hv, w.dk, w.dv), dtype=torch.float32, device=dev)
        self.ws_f = torch.zeros(gdn.fwd_workspace_size(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.num_seqs, cp),
                                dtype=torch.uint8, device=dev)
        # the chunk-state cache exists on the tensor-core sizes (bf16, dk = dv = 128) only
        tc = w.dtype == "bf16" and w.dk == 128 and w.dv == 128
        self.states = gdn.chunk_states(d["q"], d["v"], d["cu_seqlens"]) if mode != "fwd" and tc else None
        self.ws_b = None
        if mode != "fwd":
            self.ws_b = torch.zeros(gdn.bwd_workspace_size(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.num_seqs, cp,
                                                           states=self.states), dtype=torch.uint8, device=dev)
            if mode == "bwd":                   # the cache the timed backward reads
                self.fwd(d)
        self.flush = (torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
                      if alg_bytes(w, mode != "bwd", mode != "fwd") < 2 * L2_BYTES else None)

    def fwd(self, dd):
        self.gdn.gdn_chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["scale"], dd["h0"],
                               dd["cu_seqlens"], cp_segment_chunks=self.cp, workspace=self.ws_f, o=self.o,
                               hT=self.hT, states=self.states, check_status=False)

    def bwd(self, dd, states=True, ws=None):
        return self.gdn.gdn_chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["dO"], dd["scale"],
                                      dd["h0"], dd["dhT"], dd["cu_seqlens"], cp_segment_chunks=self.cp,
                                      workspace=self.ws_b if ws is None else ws,
                                      states=self.states if states else None, check_status=False)

    def step(self, dd=None):
        dd = self.d if dd is None else dd
        if self.mode == "fwd":
            self.fwd(dd)
            return None
        if self.mode == "fwdbwd":
            self.fwd(dd)
        return self.bwd(dd)

    def measure(self, steps, warmup, stream):
        for _ in range(max(warmup, 3)):
            self.step()
        torch.cuda.synchronize()
        ms = time_steps(self.step, steps, stream, self.flush)
        per_kernel, launches_one = {}, []
        with self.gdn.KernelTrace(capacity=256) as tr:
            for _ in range(3):
                if self.flush is not None:
                    self.flush.zero_()
                self.step()
        for name, t in tr.launches:
            per_kernel.setdefault(name, []).append(t)
        launches_one = tr.launches[: len(tr.launches) // 3]
        return ms, per_kernel, launches_one

    def extra_times(self, stream):
        """The forward call alone, and (with a backward) the backward that recomputes its forward
        pass instead of reading the cache."""
        out = {}
        if self.mode == "fwd":
            return out
        with self.gdn.KernelTrace(capacity=256) as trf:
            for _ in range(3):
                self.fwd(self.d)
        out["fwd_ms"] = sum(t for _, t in trf.launches) / 3
        ws_r = torch.zeros(self.gdn.bwd_workspace_size(self.w.B, self.w.T, self.w.Hqk, self.w.Hv, self.w.dk,
                                                       self.w.dv, self.w.num_seqs, self.cp),
                           dtype=torch.uint8, device=self.dev)
        with self.gdn.KernelTrace(capacity=256) as trb:
            for _ in range(3):
                self.bwd(self.d, states=False, ws=ws_r)
        out["bwd_recompute_ms"] = sum(t for _, t in trb.launches) / 3
        with self.gdn.KernelTrace(capacity=256) as trc:
            for _ in range(3):
                self.bwd(self.d)
        out["bwd_ms"] = sum(t for _, t in trc.launches) / 3
        return out

    def e2e(self, steps, stream, dist):
        """The step through the public host-buffer entry point (gdn_chunk_host of the C ABI): inputs
        from pinned host memory, every output back to pinned host memory, all inside the timed
        region. Two scratch buffers and two output sets are used in turn on three streams (kernels,
        copies in, copies out), so that one step's outputs go back while the next step's inputs
        come in. The backward-alone workload recomputes its forward pass (the host holds no
        chunk-state cache)."""
        mode, w, x = self.mode, self.w, self.x
        keys = ["q", "k", "v", "g", "beta", "h0", "cu_seqlens"] + (["dO", "dhT"] if mode != "fwd" else [])
        host = {k: (x[k].contiguous().pin_memory() if isinstance(x.get(k), torch.Tensor) else None) for k in keys}
        h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
        need = self.gdn.host_scratch_size(mode, host["q"].dtype, w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.num_seqs,
                                          self.cp)
        scratch = [torch.empty(need, dtype=torch.uint8, device=self.dev) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(self.dev), torch.cuda.Stream(self.dev)
        outs = [None, None]

        def one(i):
            outs[i % 2] = self.gdn.gdn_chunk_host(
                host["q"], host["k"], host["v"], host["g"], host["beta"], x["scale"], host["h0"],
                host["cu_seqlens"], dO=host.get("dO"), dhT=host.get("dhT"), mode=mode, scratch=scratch[i % 2],
                outputs=outs[i % 2], stream=stream, h2d_stream=s_in, d2h_stream=s_out,
                cp_segment_chunks=self.cp, synchronize=False)

        for i in range(2):                       # also allocates the two output sets
            one(i)
        torch.cuda.synchronize()
        d2h = sum(t.numel() * t.element_size() for t in outs[0].values())
        if dist:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(steps):
            one(i)
        for s_ in (s_in, s_out):                 # the timed region ends when all three streams have
            ev = torch.cuda.Event()
            ev.record(s_)
            stream.wait_event(ev)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, self.dev) / steps
        return e_ms, int(h2d), int(d2h)



def dominant_roofline(case, per_kernel, launches_one, step_label):
    """The roofline object of the kernel with the largest total time in one step: its algorithmic
    bytes per launch over its average CUDA-event launch time."""
    hbm, _, src = peaks()
    kb = kernel_alg_bytes(case.w)
    seen, per_kernel_bytes = {}, {}
    for name, _t in launches_one:
        k = seen.get(name, 0)
        seen[name] = k + 1
        opts = kb.get(name)
        if opts:
            # the backward's state pass is the second forward-kernel launch only in a recompute
            idx = min(k, len(opts) - 1) if case.mode == "fwdbwd" or case.states is None else 0
            per_kernel_bytes.setdefault(name, []).append(opts[idx])
    dom = max(per_kernel, key=lambda k: sum(per_kernel[k]))
    dom_ms = float(np.mean(per_kernel[dom]))
    dom_bytes = float(np.mean(per_kernel_bytes.get(dom, [0])))
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    return {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "frac_datasheet": achieved / DATASHEET_HBM_GBS, "peak_source": src,
            "traffic": traffic_record(dom, case.name, step_label),
            "alg_bytes_per_launch": dom_bytes, "avg_launch_ms": dom_ms}


def measure_case(gdn, name, mode, args, dev, rank, world, dist, stream, pool, budget, e2e_steps):
    case = Case(gdn, name, mode, dev, rank, args.cp)
    w = case.w
    ms, per_kernel, launches_one = case.measure(args.steps, args.warmup, stream)
    ms = max_over_ranks(ms, dist, dev)
    tokens = w.B * w.T
    fwd, bwd = mode in ("fwd", "fwdbwd"), mode in ("bwd", "fwdbwd")
    res = {"workload": name, "description": w.description, "step": mode, "ms_per_step": ms,
           "tokens_per_s": tokens * world / (ms / 1e3),
           "tflops": flops(w, fwd, bwd) * world / (ms / 1e3) / 1e12,
           "step_roofline": roofline_fraction(w, mode, ms),
           "roofline": dominant_roofline(case, per_kernel, launches_one, mode),
           "per_kernel_ms": {k: float(np.mean(v)) for k, v in per_kernel.items()},
           "l2": ("inputs larger than the 126 MB L2; no flush" if case.flush is None else
                  "working set below 2x L2: a 252 MB buffer is rewritten between timed steps")}
    res.update(case.extra_times(stream))
    e_ms, h2d, d2h = case.e2e(e2e_steps, stream, dist)
    res["e2e"] = {"value": tokens * world / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}
    res["cpu_baseline"] = (cpu_baseline(pool, w, case.x, mode, budget)
                           if pool is not None and rank == 0 and world == 1 else None)
    del case
    torch.cuda.empty_cache()
    return res


def measure_weak_decay(gdn, args, dev, rank, world, dist, stream):
    """The long grouped-value forward with weakly decaying heads (g x 0.01: no gate window closes
    within 16 chunks), unsplit and in each context-parallel mode: the restart fallback (default),
    the exact stitch, and the gate-driven start with the exact stitch as fallback."""
    name = "long_gqa_bf16"
    w = CONFIGS[name]
    x = make_inputs(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, rank_seed(w.seed, rank), h0_std=w.h0_std)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    d["g"] = (d["g"] * 0.01).contiguous()
    o = torch.empty_like(d["v"])
    hT = torch.empty((w.num_seqs, w.Hv, w.dk, w.dv), dtype=torch.float32, device=dev)
    out = {"workload": w.description + "; g x 0.01 (weakly decaying heads)", "step": "fwd"}
    for label, cp, cpx in (("unsplit", -1, 0), ("gate_restart", 0, 0), ("exact_stitch", 0, 1),
                           ("gate_exact_fallback", 0, 2)):
        ws = torch.zeros(gdn.fwd_workspace_size(w.B, w.T, w.Hqk, w.Hv, w.dk, w.dv, w.num_seqs, cp, cpx),
                         dtype=torch.uint8, device=dev)

        def step():
            gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], None,
                              cp_segment_chunks=cp, cp_exact=cpx, workspace=ws, o=o, hT=hT, check_status=False)

        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize()
        out[label + "_ms"] = max_over_ranks(time_steps(step, max(3, min(args.steps, 10)), stream), dist, dev)
        del ws
    out["speedup_vs_unsplit"] = {k[:-3]: out["unsplit_ms"] / out[k] for k in list(out) if k.endswith("_ms")}
    del d
    torch.cuda.empty_cache()
    return out


def measure_decode(gdn, args, dev, rank, world, dist, stream, pool, budget, c=DECODE):
    """One step = gdn_recurrent_step over every sequence of the batch (one token each)."""
    N, Hqk, Hv, dk, dv = c["N"], c["Hqk"], c["Hv"], c["dk"], c["dv"]
    x = make_inputs(N, 1, Hqk, Hv, dk, dv, "bf16", rank_seed(2000, rank), h0_std=0.1)
    tok = {n: x[n][:, 0].contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")}
    state = x["h0"].to(dev)
    o = torch.empty((N, Hv, dv), dtype=torch.bfloat16, device=dev)

    def step():
        gdn.gdn_recurrent_step(tok["q"], tok["k"], tok["v"], tok["g"], tok["beta"], state, x["scale"], o=o)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    ms = max_over_ranks(time_steps(step, args.steps, stream), dist, dev)
    hbm, _, src = peaks()
    nbytes = decode_bytes(N, Hqk, Hv, dk, dv)
    gbs = nbytes / (ms / 1e3) / 1e9
    cpu = None
    if pool is not None and rank == 0 and world == 1:
        def tasks():
            for s0 in range(0, N, 8):
                yield ("decode", {n: x[n][s0:s0 + 8].float().numpy() for n in ("q", "k", "v", "g", "beta", "h0")}
                       | {"scale": x["scale"]})
        tk, el, units = oracle_run(pool, tasks(), budget)
        cpu = {"value": tk / el, "unit": "tokens/s", "cores": pool._processes, "kind": "oracle",
               "sample": f"{units} groups of 8 sequences x {Hv} heads, one token each, fp64 numpy oracle "
                         f"(token form), {pool._processes} processes, {el:.1f} s"}
    return {"workload": f"decode step: {N} sequences, Hqk={Hqk} Hv={Hv}, dk=dv={dk}, bf16 I/O, fp32 state",
            "step": "decode", "ms_per_step": ms, "tokens_per_s": N * world / (ms / 1e3),
            "roofline": {"bound": "hbm", "kernel": "gdn_step_kernel", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "frac_datasheet": gbs / DATASHEET_HBM_GBS, "peak_source": src,
                         "traffic": traffic_record("gdn_step_kernel", "decode", "decode"),
                         "alg_bytes_per_launch": nbytes, "avg_launch_ms": ms},
            "l2": f"states ({N * Hv * dk * dv * 4 / 1e6:.0f} MB) larger than the 126 MB L2; no flush",
            "cpu_baseline": cpu}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only", default=None,
                    help="time only this workload (name from the workloads module, or 'decode') as the line")
    ap.add_argument("--mode", default=None, choices=["fwd", "fwdbwd", "bwd"], help="step of --only")
    ap.add_argument("--no-sub", action="store_true", help="skip the per-configuration entries")
    ap.add_argument("--single", action="store_true",
                    help="only warm-up steps plus one step of the headline, no report (profiler launch lists)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle CPU baseline (headline)")
    ap.add_argument("--cp", type=int, default=0, help="cp_segment_chunks option (0 = automatic)")
    args = ap.parse_args()
    assert args.warmup >= 0 and args.steps > 0

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    # the oracle's process pool is forked before anything touches CUDA
    want_cpu = rank == 0 and world == 1 and args.cpu_budget > 0 and not args.single
    if args.impl == "reference":
        if rank != 0:
            return
        pool = make_pool(host_cores())
        try:
            run_reference(args, pool)
        finally:
            pool.terminate()
        return
    pool = make_pool(host_cores()) if want_cpu else None

    import gated_deltanet_chunked_prefill_b200 as gdn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    stream = torch.cuda.current_stream(dev)

    name, mode = HEADLINE
    if args.only in ("decode", "decode_d256"):
        cfg = DECODE if args.only == "decode" else DECODE_256
        if args.single:                          # warm-up steps plus one step, no report
            x = make_inputs(cfg["N"], 1, cfg["Hqk"], cfg["Hv"], cfg["dk"], cfg["dv"], "bf16", 2000, h0_std=0.1)
            tok = {n: x[n][:, 0].contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")}
            state = x["h0"].to(dev)
            for _ in range(max(args.warmup, 3) + 1):
                gdn.gdn_recurrent_step(tok["q"], tok["k"], tok["v"], tok["g"], tok["beta"], state, x["scale"])
            torch.cuda.synchronize()
            return
        line = measure_decode(gdn, args, dev, rank, world, dist, stream, pool, min(args.cpu_budget, 5.0), cfg)
        line.update({"metric": "GDN recurrent decode step tokens/s on 1 B200; % of HBM roofline",
                     "value": line["tokens_per_s"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                     "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                     "dtype": "bf16", "data": "synthetic"})
        if pool is not None:
            pool.terminate()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    if args.only:
        name, mode = args.only, args.mode or ("fwd" if args.only != "bwd_bf16" else "bwd")
    if args.single:
        case = Case(gdn, name, mode, dev, rank, args.cp)
        for _ in range(max(args.warmup, 3)):
            case.step()
        case.step()
        torch.cuda.synchronize()
        return

    # ---- the headline step, device-resident, with clocks sampled during the timed region
    sampler = ClockSampler(local)
    sampler.start()
    case = Case(gdn, name, mode, dev, rank, args.cp)
    w = case.w
    for _ in range(max(args.warmup, 3)):
        case.step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    n0 = gdn.launch_count()
    tw0 = time.time()
    ms = time_steps(case.step, args.steps, stream, case.flush)
    tw1 = time.time()
    launches = gdn.launch_count() - n0
    if dist:
        dist.barrier()
    sampler.stop()
    ms = max_over_ranks(ms, dist, dev)
    tokens = w.B * w.T
    fwd, bwd = mode in ("fwd", "fwdbwd"), mode in ("bwd", "fwdbwd")
    per_kernel = {}
    with gdn.KernelTrace(capacity=256) as tr:
        for _ in range(3):
            case.step()
    for kname, t in tr.launches:
        per_kernel.setdefault(kname, []).append(t)
    roofline = dominant_roofline(case, per_kernel, tr.launches[: len(tr.launches) // 3], mode)
    extra = case.extra_times(stream)
    e_ms, h2d, d2h = case.e2e(max(3, min(args.steps, 10)), stream, dist)
    head_x = case.x
    del case
    torch.cuda.empty_cache()

    out = {"metric": METRIC, "value": tokens * world / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
           "data": "synthetic",
           "config": {"workload": w.description + f"; step = {mode}", "name": name, "step": mode,
                      "global_batch": w.B * world, "seq_len": w.T, "num_seqs": w.num_seqs, "heads_qk": w.Hqk,
                      "heads_v": w.Hv, "dk": w.dk, "dv": w.dv, "chunk": C,
                      "parallelism": f"replicas x{world}" if world > 1 else "single",
                      "l2": "working set larger than the 126 MB L2; no flush",
                      "bwd_states": "cached by the forward (bf16 chunk start states)" if mode == "fwdbwd" else None,
                      "cp_segment_chunks": args.cp},
           "tflops": flops(w, fwd, bwd) * world / (ms / 1e3) / 1e12,
           **extra,
           "per_kernel_ms": {k: float(np.mean(v)) for k, v in per_kernel.items()},
           "roofline": roofline, "step_roofline": roofline_fraction(w, mode, ms),
           "e2e": {"value": tokens * world / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h, "ms_per_step": e_ms},
           "gpu_launches": int(launches), "clocks": sampler.summary(tw0, tw1)}
    out["cpu_baseline"] = cpu_baseline(pool, w, head_x, mode, args.cpu_budget) if pool is not None else None
    del head_x

    # ---- every named workload, measured the same way
    if not args.no_sub and not args.only:
        sub_budget = max(2.0, args.cpu_budget / 3)
        per = {}
        for sname, smode in SUBS:
            per[f"{sname}:{smode}"] = measure_case(gdn, sname, smode, args, dev, rank, world, dist, stream, pool,
                                                   sub_budget, max(3, min(args.steps, 5)))
        per["long_gqa_bf16:fwd:weak_decay"] = measure_weak_decay(gdn, args, dev, rank, world, dist, stream)
        per["decode"] = measure_decode(gdn, args, dev, rank, world, dist, stream, pool, sub_budget)
        per["decode_d256"] = measure_decode(gdn, args, dev, rank, world, dist, stream, pool, sub_budget / 2,
                                            DECODE_256)
        out["per_config"] = per
    if pool is not None:
        pool.terminate()
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
