#!/usr/bin/env python
"""Throughput of the fused exact-attention hot path (forward + backward) on B200.

One step = one forward and one backward pass of causal bf16 attention over one
batch of B=2, H=16, N=4096, d=128 (Q, K, V, dO ~ N(0,1), seeded), i.e. every
kernel of the path: the fused forward, the backward's preprocessing, its
single-pass dK/dV/dQ kernel and the dQ conversion.  FLOPs follow the usual convention: forward
2*B*H*N^2*d for causal (4*B*H*N^2*d non-causal), backward 2.5x the forward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun every rank runs its own batch
(weak scaling, no data-path collective); times are the max over ranks.
``--impl reference`` times the float64 CPU oracle on a bounded sample of the same
workload instead (the only other place this script runs the oracle).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

B, H, N, D = 2, 16, 4096, 128
CAUSAL = True
SEED = 5
METRIC = "causal bf16 attention fwd/bwd TFLOPS at N=4096,d=128; % of B200 tensor peak"
UNIT = "TFLOPS"
WORKLOAD = "causal attention fwd+bwd B2 H16 N4096 d128 bf16, Q/K/V/dO ~ N(0,1)"


def flops_fwd(b=B, h=H, n=N, d=D, causal=CAUSAL):
    return (2.0 if causal else 4.0) * b * h * n * n * d


def flops_bwd(b=B, h=H, n=N, d=D, causal=CAUSAL):
    return 2.5 * flops_fwd(b, h, n, d, causal)


def measured_peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # no NVML: clocks reported as unavailable
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- CPU oracle timing
_ORACLE_INPUTS = None


def time_oracle_sample(n_heads: int):
    """float64 oracle forward + backward on the first n_heads (b, h) slices of the
    workload, all host cores.  Returns (TFLOPS, seconds, cores, sample text)."""
    import oracle
    global _ORACLE_INPUTS
    if _ORACLE_INPUTS is None:  # drawn once, reused by every timed sample
        from attn_inputs import make_dense
        _ORACLE_INPUTS = make_dense(B, H, N, D, seed=SEED, causal=CAUSAL, with_grad=True)
    inp = _ORACLE_INPUTS
    threads = oracle.default_threads()
    picks = list(range(n_heads))
    t0 = time.perf_counter()
    oracle.fwd(inp.q, inp.k, inp.v, inp.scale, CAUSAL, slices=picks, nthreads=threads)
    oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, CAUSAL, slices=picks, nthreads=threads)
    dt = time.perf_counter() - t0
    fl = flops_fwd(1, n_heads) + flops_bwd(1, n_heads)
    return fl / dt / 1e12, dt, threads, f"{n_heads} of {B * H} (b,h) slices at N={N}, d={D}, fwd+bwd"


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    threads = oracle.default_threads()
    vals = []
    for s in range(args.warmup + args.steps):
        v, dt, cores, sample = time_oracle_sample(1)
        if s >= args.warmup:
            vals.append((v, dt))
    value = statistics.median(v for v, _ in vals)
    total_s = sum(dt for _, dt in vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total_s / max(1, len(vals)), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "H": H, "N": N, "d": D, "causal": CAUSAL},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "per step: 1 of 32 (b,h) slices at N=4096, d=128, fwd+bwd, float64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def source_digest():
    """Digest of the kernel sources' code: comments and white space are left out, so
    an edit to a comment does not disown counters taken on the same code."""
    h = hashlib.sha256()
    for f in ("attn_bwd_sm100.cu", "attn_bwd_fused_sm100.cu", "attn_fwd_sm100.cu", "sm100_ptx.cuh", "attn_common.cuh",
              "attn_api.cu"):
        with open(os.path.join(HERE, "exact_attention_123_b200", "csrc", f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_ncu():
    """Per-kernel figures of the committed ncu captures, if they were taken on the
    current kernel code; otherwise None."""
    p = os.path.join(HERE, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    keys = ("tensor_pipe_active_pct", "mufu_pipe_active_pct", "issue_active_pct", "hbm_gbs", "dram_bytes_per_launch",
            "l2_hit_pct", "smem_bank_conflicts_ld", "smem_bank_conflicts_st", "registers_per_thread", "smem_per_cta_kb",
            "duration_us_ncu")
    out = {k: {f: e[f] for f in keys if f in e} for k, e in rec.items()
           if isinstance(e, dict) and e.get("source_digest") == source_digest()}
    return out or None


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on the
    current kernel sources; otherwise None."""
    p = os.path.join(HERE, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    e = rec.get(kernel)
    if not e or e.get("source_digest") != source_digest():
        return None
    return e.get("dram_bytes_per_launch")


# The backward as timed in the headline step: its kernels launched one by one
# through attn_bwd_phase so each gets its own CUDA events.  (name, phase, kernel,
# tensor-core FLOPs of the kernel in units of the forward's count, or None for an
# HBM-bound kernel.)
BWD_PHASES = [
    ("bwd_pre", 3, "attn_bwd_pre_kernel", None),            # D, lse2, zeroed dQ accumulator
    ("bwd_main", 4, "attn_bwd_fused_sm100_kernel", 2.5),    # all five products of every tile pair
    ("bwd_dq_convert", 5, "attn_bwd_dq_convert_kernel", None),
]
# --deterministic: the two-pass backward (attn_bwd_deterministic) in the step instead
BWD_PHASES_DET = [
    ("bwd_pre", 0, "attn_bwd_pre_kernel", None),            # D, lse2
    ("bwd_dkdv", 1, "attn_bwd_dkdv_sm100_kernel", 2.0),     # S^T, dP^T, dV, dK
    ("bwd_dq", 2, "attn_bwd_dq_sm100_kernel", 1.5),         # S, dP (recomputed), dQ
]
MIN_WARMUP = 10  # warm-up calls before any timing (at least, whatever --warmup says)


def _median_ms(fn, flush, stream, reps):
    """Median over `reps` calls of fn(), CUDA events on the launching stream, L2
    flushed before each call outside the bracket."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for e in ev:
        flush.zero_()
        e[0].record(stream)
        fn()
        e[1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(e[0].elapsed_time(e[1]) for e in ev)


def _shape_table(ea, dev, stream, flush, peak, reps, with_oracle):
    """Every workload shape of the pages (sequence length 2048 timing table, codechina
    article §5.2; N = 4096, d = 128 tiling example, §2.2; variable lengths, §6.2): the
    median time, TFLOPS and share of the measured peak of each pass, with the
    oracle's host time on a bounded sample next to it."""
    import torch
    from attn_inputs import draw_lengths, make_dense, make_varlen, padding_key_mask
    out = {}
    threads = None

    def oracle_time(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    def entry(key, ms, flops, osec=None, ofrac=None):
        tf = flops / (ms * 1e-3) / 1e12
        e = {"us": round(ms * 1e3, 1), "tflops": round(tf, 1), "pct": round(100 * tf / peak, 1)}
        if osec is not None:
            # oracle on `ofrac` of the work, scaled up to the whole shape
            e["oracle_s"] = round(osec / ofrac, 2)
            e["oracle_cores"] = threads
        out[key] = e

    if with_oracle:
        import oracle
        threads = oracle.default_threads()
    # (name, B, H, N, d, seed, sigma, causal list, with backward)
    dense = [("c2_n2048_d64", 4, 16, 2048, 64, 2, 1.0, (True, False), True),
             ("c3_n4096_d128", 2, 16, 4096, 128, 3, 1.0, (False,), True),
             ("c3s_n4096_d128_sigma4", 2, 16, 4096, 128, 33, 4.0, (True, False), False)]
    for name, B, H, N, d, seed, sig, causals, with_bwd in dense:
        inp = make_dense(B, H, N, d, seed=seed, qk_sigma=sig, with_grad=with_bwd)
        q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
        do = inp.do.to(dev) if with_bwd else None
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
        ws = ea.workspace_for(q) if with_bwd else None
        for causal in causals:
            kw = dict(scale=inp.scale, causal=causal, stream=stream)
            for _ in range(3):
                ea.attn_fwd(q, k, v, o, lse, **kw)
            f_ms = _median_ms(lambda: ea.attn_fwd(q, k, v, o, lse, **kw), flush, stream, reps)
            ffl = (2.0 if causal else 4.0) * B * H * N * N * d
            tag = f"{name}_{'causal' if causal else 'noncausal'}"
            osec = None
            if with_oracle:
                osec = oracle_time(lambda: oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, slices=[0],
                                                      nthreads=threads))
            entry(tag + "_fwd", f_ms, ffl, osec, 1.0 / (B * H))
            if with_bwd:
                dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
                for _ in range(3):
                    ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, workspace=ws, **kw)
                b_ms = _median_ms(lambda: ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, workspace=ws, **kw),
                                  flush, stream, reps)
                osec = None
                if with_oracle:
                    osec = oracle_time(lambda: oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, causal,
                                                          slices=[0], nthreads=threads))
                entry(tag + "_bwd", b_ms, 2.5 * ffl, osec, 1.0 / (B * H))
        del q, k, v, o, lse, do, ws
    # variable-length workload: 8 sequences of U[256, 4096] tokens, H32 d128, causal,
    # key padding that empties the first 2 % of each sequence's query rows
    lengths = draw_lengths(8, 256, 4096, 40)
    keep = padding_key_mask(lengths, 41)
    vin = make_varlen(lengths, 32, 128, 4, True, keep, with_grad=True)
    q, k, v, do = (t.to(dev) for t in (vin.q, vin.k, vin.v, vin.do))
    cu, kk = vin.cu_seqlens.to(dev), keep.to(dev)
    o, lse = torch.empty_like(q), torch.empty(q.shape[:2], device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = ea.workspace_for(q, cu)
    kw = dict(scale=vin.scale, causal=True, cu_seqlens=cu, key_keep=kk, max_seqlen=max(lengths), stream=stream)
    ffl = 2.0 * 32 * 128 * sum(n * n for n in lengths)
    for _ in range(3):
        ea.attn_fwd(q, k, v, o, lse, **kw)
        ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, workspace=ws, **kw)
    f_ms = _median_ms(lambda: ea.attn_fwd(q, k, v, o, lse, **kw), flush, stream, reps)
    b_ms = _median_ms(lambda: ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, workspace=ws, **kw), flush, stream, reps)
    osf = osb = None
    frac = (lengths[0] ** 2) / (32 * sum(n * n for n in lengths))  # sequence 0, head 0
    if with_oracle:
        osf = oracle_time(lambda: oracle.fwd(vin.q, vin.k, vin.v, vin.scale, True, cu_seqlens=vin.cu_seqlens,
                                             key_keep=keep, slices=[0], nthreads=threads))
        osb = oracle_time(lambda: oracle.bwd(vin.q, vin.k, vin.v, vin.do, vin.scale, True,
                                             cu_seqlens=vin.cu_seqlens, key_keep=keep, slices=[0],
                                             nthreads=threads))
    entry("c4_varlen_8x_h32_d128_causal_fwd", f_ms, ffl, osf, frac)
    entry("c4_varlen_8x_h32_d128_causal_bwd", b_ms, 2.5 * ffl, osb, frac)
    st = ea.attn_status(stream)
    if st != ea.ATTN_OK:
        raise RuntimeError(f"shape table reported status {st}: {ea.attn_strerror(st)}")
    return out


def launch_plan(gpus: int, env) -> tuple:
    """How to honour --gpus: ("run", None) when the process layout already matches,
    ("spawn", argv) to relaunch this script as `gpus` ranks (one process per GPU,
    torchrun on 127.0.0.1) when started as a single plain process, or ("error", text)
    when started under a launcher with another world size."""
    ws = env.get("WORLD_SIZE")
    if gpus < 1:
        return "error", f"--gpus must be >= 1, got {gpus}"
    if ws is None:
        if gpus == 1:
            return "run", None
        argv = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
                "--master-addr=127.0.0.1", "--master-port=29531", os.path.abspath(__file__)] + sys.argv[1:]
        return "spawn", argv
    if int(ws) != gpus:
        return "error", f"--gpus {gpus} but the launcher started WORLD_SIZE={ws} ranks"
    return "run", None


def run_ours(args):
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}), flush=True)
        return 1
    if ws > torch.cuda.device_count():
        print(json.dumps({"error": f"{ws} ranks but {torch.cuda.device_count()} visible GPUs"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    from exact_attention_123_b200 import build
    if rank == 0:
        build.build()
    if ws > 1:
        dist.barrier()
    import exact_attention_123_b200 as ea
    from attn_inputs import make_dense

    inp = make_dense(B, H, N, D, seed=SEED + 1000 * rank, causal=CAUSAL, with_grad=True)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsbuf = ea.workspace_for(q)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream(dev)
    kw = dict(scale=inp.scale, causal=CAUSAL, stream=stream)
    phases = BWD_PHASES_DET if args.deterministic else BWD_PHASES
    n_k = 1 + len(phases)  # kernels per step

    def step(ev=None):
        # attn_bwd == its phases in order; launched one by one here to time each kernel
        if ev is not None:
            ev[0].record(stream)
        ea.attn_fwd(q, k, v, o, lse, **kw)
        for i, (_, ph, _, _) in enumerate(phases):
            if ev is not None:
                ev[1 + i].record(stream)
            ea.attn_bwd_phase(ph, q, k, v, o, lse, do, dq, dk, dv, workspace=wsbuf, **kw)
        if ev is not None:
            ev[n_k].record(stream)

    n_warm = max(MIN_WARMUP, args.warmup)
    for _ in range(n_warm):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    st = ea.attn_status(stream)
    if st != ea.ATTN_OK:
        raise RuntimeError(f"warm-up reported status {st}: {ea.attn_strerror(st)}")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_k + 1)] for _ in range(args.steps)]
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for s in range(args.steps):
            flush.zero_()          # L2 flushed before every step, outside the event bracket
            step(events[s])
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
    if ws > 1:
        dist.barrier()
    st = ea.attn_status(stream)
    if st != ea.ATTN_OK:
        raise RuntimeError(f"timed steps reported status {st}: {ea.attn_strerror(st)}")

    seg = [[e[i].elapsed_time(e[i + 1]) for i in range(n_k)] for e in events]  # ms per kernel per step
    step_ms = [sum(x) for x in seg]
    total_ms = sum(step_ms)
    from exact_attention_123_b200.sharding import max_over_ranks
    total_ms_max = max_over_ranks(total_ms, device=dev)  # the job is as slow as its slowest rank

    # ---- end to end through the public API with host buffers.  Every step copies its
    # inputs in from pinned host memory and its gradients out to pinned host memory.
    # The steps are pipelined over two device buffer sets and three streams (copy in,
    # kernels, copy out) ordered by events, so the copy engines move step s+1's inputs
    # and step s-1's gradients while the SMs run step s.
    pin = {n: x.cpu().pin_memory() for n, x in (("q", q), ("k", k), ("v", v), ("do", do))}
    outs = {n: torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for n, x in (("dq", dq), ("dk", dk), ("dv", dv))}
    h2d = sum(x.numel() * x.element_size() for x in pin.values())
    d2h = sum(x.numel() * x.element_size() for x in outs.values())
    bufs = [dict(q=q, k=k, v=v, do=do, dq=dq, dk=dk, dv=dv)]
    bufs.append({n: torch.empty_like(t) for n, t in bufs[0].items()})
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in, ev_run, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    used = [False, False]

    def e2e_step(i):
        b = bufs[i]
        with torch.cuda.stream(s_in):
            if used[i]:
                s_in.wait_event(ev_run[i])  # the kernels of two steps ago are done with set i
            for n in ("q", "k", "v", "do"):
                b[n].copy_(pin[n], non_blocking=True)
            ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        if used[i]:
            stream.wait_event(ev_out[i])  # the gradients of two steps ago have left set i
        ea.attn_fwd(b["q"], b["k"], b["v"], o, lse, **kw)
        ea.attn_bwd(b["q"], b["k"], b["v"], o, lse, b["do"], b["dq"], b["dk"], b["dv"], workspace=wsbuf,
                    deterministic=args.deterministic, **kw)
        ev_run[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[i])
            for n in ("dq", "dk", "dv"):
                outs[n].copy_(b[n], non_blocking=True)
            ev_out[i].record(s_out)
        used[i] = True

    for s in range(2):
        e2e_step(s % 2)
    torch.cuda.synchronize(dev)
    e2e_n = max(3, args.e2e_steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    e0.record(s_in)  # every stream is idle here; the others start after work ordered behind e0
    for s in range(e2e_n):
        e2e_step(s % 2)
    e1.record(s_out)  # behind the last copy out, which is behind every earlier step's work
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device=dev)
    st = ea.attn_status(stream)
    if st != ea.ATTN_OK:
        raise RuntimeError(f"end-to-end steps reported status {st}")
    # The pipeline's longest stream alone: the steps' host-to-device copies back to back, no
    # kernels and no copies out (which run alongside and only slow them) -- a lower bound on
    # the end-to-end step that the host link sets.
    torch.cuda.synchronize(dev)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(s_in)
    with torch.cuda.stream(s_in):
        for s in range(e2e_n):
            for n in ("q", "k", "v", "do"):
                bufs[s % 2][n].copy_(pin[n], non_blocking=True)
    c1.record(s_in)
    torch.cuda.synchronize(dev)
    copy_ms = max_over_ranks(c0.elapsed_time(c1), device=dev)

    peaks, peak_src = measured_peaks()
    peak = float(peaks["bf16_tflops"])
    reps = max(20, args.shape_reps)

    # ---- block-sparse variant: the same workload with half of the (query tile, key
    # tile) pairs left out by a seeded per-head tile mask; timed after the headline
    # steps, L2 flushed before each call.  FLOPs are those of the pairs computed
    # (causal convention: a diagonal pair counts half, as in the dense count).
    bsp = None
    if not args.no_blocksparse and ws == 1:
        from attn_inputs import tile_mask
        nbt = (N + 127) // 128
        bm = tile_mask(H, N, SEED + 7, 0.5)
        tri = torch.tril(torch.ones(nbt, nbt, dtype=torch.uint8))
        live = bm & tri if CAUSAL else bm
        diag = torch.eye(nbt, dtype=torch.uint8)
        pair_units = float(live.sum().item()) - (0.5 * float((live & diag).sum().item()) if CAUSAL else 0.0)
        fl_fwd = B * pair_units * 4.0 * 128 * 128 * D
        bmd = bm.to(dev)
        for _ in range(3):
            ea.attn_fwd_blocksparse(q, k, v, bmd, o, lse, **kw)
            ea.attn_bwd_blocksparse(q, k, v, o, lse, do, bmd, dq, dk, dv, workspace=wsbuf, **kw)
        f_ms = _median_ms(lambda: ea.attn_fwd_blocksparse(q, k, v, bmd, o, lse, **kw), flush, stream, reps)
        b_ms = _median_ms(lambda: ea.attn_bwd_blocksparse(q, k, v, o, lse, do, bmd, dq, dk, dv, workspace=wsbuf, **kw),
                          flush, stream, reps)
        st = ea.attn_status(stream)
        if st != ea.ATTN_OK:
            raise RuntimeError(f"block-sparse steps reported status {st}")
        dense_units = nbt * (nbt + 1) / 2 - nbt / 2 if CAUSAL else nbt * nbt
        bsp = {"density": 0.5, "seed": SEED + 7, "pairs_frac": round(pair_units / (H * dense_units), 4),
               "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4),
               "fwd_tflops": round(fl_fwd / (f_ms * 1e-3) / 1e12, 1),
               "bwd_tflops": round(2.5 * fl_fwd / (b_ms * 1e-3) / 1e12, 1)}

    # ---- FP8 (e4m3) forward on the same workload: q, k, v quantised per tensor
    # (factor = amax / 448) on the device; timed like the block-sparse variant.
    # FLOPs as the bf16 forward's; the peak is the measured bf16 one times the
    # nominal e4m3 : bf16 dense ratio (2).
    fp8 = None
    if not args.no_fp8 and ws == 1:
        q8s = []
        for t in (q, k, v):
            fct = float(t.abs().max().float().item()) / 448.0
            q8s.append(((t.float() / fct).to(torch.float8_e4m3fn), fct))
        (q8, qf), (k8, kf), (v8, vf) = q8s
        for _ in range(3):
            ea.attn_fwd_fp8(q8, k8, v8, qf, kf, vf, o, lse, **kw)
        f8_ms = _median_ms(lambda: ea.attn_fwd_fp8(q8, k8, v8, qf, kf, vf, o, lse, **kw), flush, stream, reps)
        st = ea.attn_status(stream)
        if st != ea.ATTN_OK:
            raise RuntimeError(f"fp8 forward reported status {st}")
        f8_tf = flops_fwd() / (f8_ms * 1e-3) / 1e12
        pk8 = 2.0 * peak
        fp8 = {"fwd_ms": round(f8_ms, 4), "fwd_tflops": round(f8_tf, 1), "pct_of_2x_bf16_peak": round(100 * f8_tf / pk8, 1)}
        if bsp is not None:
            # e4m3 with the block-sparse variant's tile mask (FLOPs of the pairs computed)
            for _ in range(3):
                ea.attn_fwd_fp8_blocksparse(q8, k8, v8, qf, kf, vf, bmd, o, lse, **kw)
            fs_ms = _median_ms(lambda: ea.attn_fwd_fp8_blocksparse(q8, k8, v8, qf, kf, vf, bmd, o, lse, **kw),
                               flush, stream, reps)
            st = ea.attn_status(stream)
            if st != ea.ATTN_OK:
                raise RuntimeError(f"fp8 block-sparse forward reported status {st}")
            fp8.update({"blocksparse_fwd_ms": round(fs_ms, 4),
                        "blocksparse_fwd_tflops": round(fl_fwd / (fs_ms * 1e-3) / 1e12, 1)})

    shapes = None
    if not args.no_shapes and ws == 1:
        shapes = _shape_table(ea, dev, stream, flush, peak, reps, with_oracle=not args.no_cpu_baseline)

    step_flops = flops_fwd() + flops_bwd()
    value = step_flops * args.steps * ws / (total_ms_max * 1e-3) / 1e12
    e2e_value = step_flops * e2e_n * ws / (e2e_ms * 1e-3) / 1e12

    # per-kernel medians over the timed steps (the headline value above uses the total)
    med = [statistics.median(x[i] for x in seg) for i in range(n_k)]
    fwd_ms = med[0]
    bwd_ms = sum(med[1:])
    fwd_tf = flops_fwd() / (fwd_ms * 1e-3) / 1e12
    bwd_tf = flops_bwd() / (bwd_ms * 1e-3) / 1e12
    per_kernel = {"attn_fwd_sm100_kernel": (fwd_ms, fwd_tf)}
    breakdown = {"fwd": round(fwd_ms * 1e3, 1)}
    hbm_ms = {}
    for (name, _, kname, mult), ms in zip(phases, med[1:]):
        breakdown[name] = round(ms * 1e3, 1)
        if mult is None:
            hbm_ms[kname] = ms
        else:
            per_kernel[kname] = (ms, mult * flops_fwd() / (ms * 1e-3) / 1e12)
    dominant = max(per_kernel, key=lambda kname: per_kernel[kname][0])
    dom_tf = per_kernel[dominant][1]
    # HBM-bound kernels, algorithmic bytes per launch: the preprocess reads O and dO
    # (bf16) and lse, writes D and lse2 and (single pass) zeroes the fp32 dQ accumulator;
    # the conversion reads the accumulator and writes dQ (bf16)
    hbm_bytes = {"attn_bwd_pre_kernel": B * H * N * (2 * D * 2 + 4 + 8 + (0 if args.deterministic else 4 * D)),
                 "attn_bwd_dq_convert_kernel": B * H * N * (4 * D + 2 * D)}
    hbm = {k: {"achieved": round(hbm_bytes[k] / (ms * 1e-3) / 1e9, 1), "bytes_per_launch": hbm_bytes[k]}
           for k, ms in hbm_ms.items() if k in hbm_bytes}

    if ws > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if ws == 1 and not args.no_cpu_baseline:
        cv, cdt, cores, sample = time_oracle_sample(args.cpu_heads)
        cpu = {"value": cv, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
               "seconds": round(cdt, 3)}

    ncu = recorded_ncu()
    if ncu:  # the three headline counters per kernel; the full record is in profiles/
        ncu = {k: {"tensor_pct": round(e.get("tensor_pipe_active_pct", float("nan")), 1),
                   "hbm_gbs": round(e.get("hbm_gbs", float("nan"))),
                   "smem_conflicts": int(e.get("smem_bank_conflicts_ld", 0) + e.get("smem_bank_conflicts_st", 0))}
               for k, e in ncu.items()}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "H": H, "N": N, "d": D, "causal": CAUSAL, "seed": SEED,
                   "l2": "flushed (256 MiB write) before every timed step, outside the timed bracket",
                   "warmup_steps_run": n_warm,
                   "backward": "deterministic (two passes)" if args.deterministic else "single pass",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "roofline": {"kernel": dominant, "bound": "tensor", "achieved": dom_tf, "peak": peak, "unit": "TFLOP/s",
                     "frac": dom_tf / peak, "traffic": recorded_traffic(dominant),
                     "peak_source": ("MEASURED_PEAKS.json bf16_tflops (burst)" if peak_src == "measured" else
                                     "fallback: 1590 TFLOPS measured earlier on this pool "
                                     "(no MEASURED_PEAKS.json beside bench.py)")},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_n, "pipeline": "copy in, kernels, copy out on three streams over two buffer sets",
                "ms_per_step": e2e_ms / e2e_n,
                # the host-to-device copies alone, back to back: the host link's bound on a step
                "h2d_only_ms_per_step": copy_ms / e2e_n,
                "frac_of_copy_bound": (copy_ms / e2e_ms) if e2e_ms > 0 else None},
        "gpu_launches": n_k * args.steps,
        "clocks": clk.summary(),
        "wall_s_timed_region": round(wall, 4),
        "ncu_recorded": ncu,
        "blocksparse": bsp,
        "fp8": fp8,
        "hbm": {k: dict(e, unit="GB/s", frac=round(e["achieved"] / float(peaks["hbm_gbs"]), 4))
                for k, e in hbm.items()},
        "shapes": shapes,
        # last, so that they survive in any tail of the output
        "breakdown_us": breakdown,
        "tflops": {"fwd": round(fwd_tf, 1), "bwd": round(bwd_tf, 1),
                   **{k: round(v[1], 1) for k, v in per_kernel.items() if k != "attn_fwd_sm100_kernel"}},
        "pct_of_peak": {"fwd": round(100 * fwd_tf / peak, 2), "bwd": round(100 * bwd_tf / peak, 2),
                        "step": round(100 * value / ws / peak, 2), "stat": f"median of {args.steps} steps",
                        "peak": f"{peak} TFLOPS bf16 dense ({peak_src}, burst)"},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ncu reports
# Figures read from one `ncu --set full` capture (raw page, CSV), per kernel launch.
NCU_METRICS = {
    "duration_us_ncu": ("gpu__time_duration.sum", "us"),
    "dram_read": ("dram__bytes_read.sum", "bytes"),
    "dram_write": ("dram__bytes_write.sum", "bytes"),
    "tensor_pipe_active_pct": ("sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed", None),
    "mufu_pipe_active_pct": ("sm__inst_executed_pipe_xu.avg.pct_of_peak_sustained_active", None),
    "issue_active_pct": ("smsp__issue_active.avg.pct_of_peak_sustained_active", None),
    "l2_hit_pct": ("lts__t_sector_hit_rate.pct", None),
    "warp_instructions": ("smsp__inst_executed.sum", None),
    "smem_bank_conflicts_ld": ("l1tex__data_bank_conflicts_pipe_lsu_mem_shared_op_ld.sum", None),
    "smem_bank_conflicts_st": ("l1tex__data_bank_conflicts_pipe_lsu_mem_shared_op_st.sum", None),
    "registers_per_thread": ("launch__registers_per_thread", None),
    "smem_per_cta_kb": ("launch__shared_mem_per_block_dynamic", "kb"),
}
_SCALE = {"us": {"nsecond": 1e-3, "usecond": 1.0, "msecond": 1e3, "second": 1e6},
          "bytes": {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9},
          "kb": {"byte": 1e-3, "Kbyte": 1.0, "Mbyte": 1e3}}


def ncu_kernel_key(name: str) -> str:
    """Record key of a kernel: the bare name for the dense bf16 d=128 instantiations
    the bench times, the name with its template arguments otherwise."""
    base = name.split("(")[0].replace("void ", "").replace("attn::", "").strip()
    short, _, args = base.partition("<")
    return short if args.rstrip(">") in ("128, 0", "128, 0, 0", "128, 0, 0, 2, 0") else base


def ncu_rows(csv_text: str):
    """Per-launch figures from `ncu -i REPORT --page raw --csv` output."""
    import csv
    import io
    rows = list(csv.reader(io.StringIO(csv_text)))
    head, units = rows[0], rows[1]
    col = {h: i for i, h in enumerate(head)}
    out = []
    for r in rows[2:]:
        if len(r) != len(head):
            continue
        e = {"kernel": ncu_kernel_key(r[col["Kernel Name"]])}
        for key, (metric, kind) in NCU_METRICS.items():
            if metric not in col or r[col[metric]] in ("", "n/a"):
                continue
            v = float(r[col[metric]].replace(",", ""))
            if kind:
                v *= _SCALE[kind].get(units[col[metric]], 1.0)
            e[key] = v
        if "dram_read" in e and "dram_write" in e:
            e["dram_bytes_per_launch"] = int(round(e["dram_read"] + e["dram_write"]))
            if e.get("duration_us_ncu"):
                e["hbm_gbs"] = e["dram_bytes_per_launch"] / (e["duration_us_ncu"] * 1e-6) / 1e9
        out.append(e)
    return out


def ncu_summary(report: str, record: bool) -> int:
    """Print one JSON line per captured launch; with `record`, store them in
    profiles/ncu_traffic.json under the current kernel-code digest."""
    text = subprocess.run(["ncu", "-i", report, "--page", "raw", "--csv"], capture_output=True, text=True,
                          check=True).stdout
    rows = ncu_rows(text)
    for e in rows:
        print(json.dumps(e), flush=True)
    if record:
        p = os.path.join(HERE, "profiles", "ncu_traffic.json")
        rec = json.load(open(p)) if os.path.exists(p) else {}
        dg = source_digest()
        rec["source_digest"] = dg
        for e in rows:
            ent = {k: v for k, v in e.items() if k != "kernel"}
            ent["source_digest"] = dg
            rec[e["kernel"]] = ent
        with open(p, "w") as f:
            json.dump(rec, f, indent=2)
            f.write("\n")
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--cpu-heads", type=int, default=32,
                    help="(b,h) slices in the CPU-oracle baseline sample (32 = the whole workload, about 14 s on 16 cores)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-blocksparse", action="store_true", help="skip the block-sparse variant's timing")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 forward's timing")
    ap.add_argument("--no-shapes", action="store_true", help="skip the table of the other workload shapes")
    ap.add_argument("--deterministic", action="store_true",
                    help="time the deterministic two-pass backward in the step instead of the single pass")
    ap.add_argument("--shape-reps", type=int, default=30, help="timed calls per entry of the shape table (median)")
    ap.add_argument("--ncu-summary", metavar="REPORT",
                    help="print the per-kernel figures of an ncu --set full report (no GPU needed) and exit")
    ap.add_argument("--record", action="store_true",
                    help="with --ncu-summary: store them in profiles/ncu_traffic.json for the current kernel code")
    args = ap.parse_args()
    if args.ncu_summary:
        return ncu_summary(args.ncu_summary, args.record)
    plan, what = launch_plan(args.gpus, os.environ)
    if plan == "error":
        print(json.dumps({"error": what}), flush=True)
        return 2
    if plan == "spawn":
        return subprocess.run(what).returncode
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
