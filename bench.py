#!/usr/bin/env python
"""Benchmark: exact attention forward + backward on B200 through libfa.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fa|reference]
                    [--workload 2] [--no-e2e] [--no-cpu-baseline]

One step = fa_forward + the three backward steps (preprocess, dK/dV, dQ
finalize) over one batch of the GPT-2-medium-shaped layer (B=64, H=16,
T=1024, d=64, non-causal; the workload the "Efficient attention: memory-bound"
page times), bf16 inputs already resident in HBM.  Each step's inputs
(4 x 128 MiB) exceed the 126 MB L2, so no flush is needed between steps.

Prints one JSON line (rank 0).  `value` is algorithmic TFLOP/s of the whole
job: (4 + 10) * B * Hq * d * pairs per step and GPU, over the slowest rank's
device time.  Under torchrun each rank runs its own batch (the (batch, head)
units are independent; no collective on the data path): weak scaling.

`--impl reference` times the CPU float64 oracle (the reference arm here) on a
bounded sample per step, on rank 0 only.
"""

from __future__ import annotations

import argparse
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

METRIC = "attention fwd+bwd TFLOPS (bf16, 1×B200) and % of dense tensor peak"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["fa", "reference"], default="fa")
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="headline workload only (by default the d=128 prefill and decode workloads are timed too)")
    ap.add_argument("--extra-steps", type=int, default=30,
                    help="timed steps of the T=8192 workload in the extra set (T=32768: a third; decode: x10)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--window", type=int, default=None,
                    help="sliding window of that many keys (prefill: implies causal; decode: last keys)")
    ap.add_argument("--fp8", action="store_true",
                    help="prefill, d = 128 only: the E4M3 forward (fa_forward_fp8) alone")
    ap.add_argument("--dropout", type=float, default=None,
                    help="prefill: forward + backward with fused dropout of this rate (fa_forward_dropout, "
                         "fa_backward_dkdv_dropout)")
    ap.add_argument("--cp", action="store_true",
                    help="decode only: context-parallel, every sequence's cache cut into one share per GPU")
    ap.add_argument("--deterministic", action="store_true",
                    help="prefill: forward + fa_backward_deterministic (dQ from its own pass, the same bits on "
                         "every run); the default step is timed beside it")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (smaller cases for profiler captures only)")
    return ap.parse_args()


def pairs_count(Tq, Tk, causal, window=0):
    """(query, key) pairs entering the softmax; bottom-right causal rule, and
    with a sliding window the `window` most recent keys of each query."""
    if window:
        off = Tk - Tq
        tot = 0
        for i in range(Tq):
            hi = min(Tk - 1, i + off)
            lo = max(0, i + off - window + 1)
            tot += max(0, hi - lo + 1)
        return tot
    if not causal:
        return Tq * Tk
    off = Tk - Tq
    # rows i with i + off + 1 in [1, Tk]: sum of min(Tk, max(0, i + off + 1))
    tot = 0
    first_full = max(0, Tk - off - 1)   # from this row on every key is visible
    for i in range(min(Tq, first_full)):
        tot += max(0, i + off + 1)
    tot += max(0, Tq - first_full) * Tk
    return tot


def flops(w):
    P = pairs_count(w.T, w.T, w.causal, w.window)
    f = 4 * w.B * w.Hq * w.d * P
    b = 10 * w.B * w.Hq * w.d * P
    return f, b


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"bf16_tflops": pk["bf16_tflops"], "bf16_tflops_sustained": pk.get("bf16_tflops_sustained"),
                "hbm_gbs": pk["hbm_gbs"], "source": "measured"}
    except Exception:
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


KERNEL_SOURCES = {
    "fa_fwd_kernel": "fa_fwd.cuh",
    "fa_bwd_dkdv_kernel": "fa_bwd.cuh",
    "fa_decode_split_kernel": "fa_decode.cuh",
}


def kernel_source_hash(kernel):
    """Hash of the source file that holds a kernel's code (the shared PTX
    wrappers only gain functions, so a kernel's file is what changes it)."""
    h = hashlib.sha256()
    f = KERNEL_SOURCES[kernel]
    with open(os.path.join(ROOT, "io_aware_exact_forward_b200", "csrc", f), "rb") as fh:
        h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, only if it was
    taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            data = json.load(f)
        ent = data[kernel][workload]
        if ent.get("source_hash") == kernel_source_hash(kernel):
            return ent["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.out is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
                except ValueError:
                    continue
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [r for r in rows if r[2] > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3][1:5]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(load), "power_w_max": max(r[2] for r in rows), "reasons": reasons}


# ---------------------------------------------------------------------------
# CPU baseline: the float64 oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_heads(w, inp_cpu, heads, budget_s):
    """Run the oracle's forward + backward head by head; stop at the budget.
    Returns (heads done, seconds, algorithmic flops done)."""
    import oracle
    from workloads import to_f64
    G = w.Hq // w.Hkv
    f, b = flops(w)
    per_head = (f + b) / (w.B * w.Hq)
    done, t0 = 0, time.perf_counter()
    for (bi, h) in heads:
        g = h // G
        qh = to_f64(inp_cpu["q"][bi, :, h])
        kh = to_f64(inp_cpu["k"][bi, :, g])
        vh = to_f64(inp_cpu["v"][bi, :, g])
        dh = to_f64(inp_cpu["do"][bi, :, h])
        win = w.window or None
        oracle.head_forward(qh, kh, vh, w.scale, w.causal, window=win)
        oracle.head_backward(qh, kh, vh, dh, w.scale, w.causal, window=win)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done, dt, done * per_head


def oracle_decode(w, q, kc, vc, seqlens, budget_s, max_passes=None):
    """Run the oracle's decode (G query heads of one KV head at a time) over
    the given sequences; stop at the budget.  Returns (groups done, seconds,
    algorithmic bytes done: the K and V rows the query sees, q, o, lse)."""
    import oracle
    from workloads import to_f64
    G = w.Hq // w.Hkv
    done, nbytes, t0 = 0, 0, time.perf_counter()
    passes = 0
    while max_passes is None or passes < max_passes:   # passes until the budget is spent
        passes += 1
        for b in range(q.shape[0]):
            L = int(seqlens[b])
            seen = min(L, w.window) if w.window else L
            qb, kb, vb = to_f64(q[b:b + 1]), to_f64(kc[b:b + 1, :L]), to_f64(vc[b:b + 1, :L])
            for hkv in range(w.Hkv):
                oracle.decode_forward(qb, kb, vb, [L], w.scale, pairs=[(0, hkv * G + i) for i in range(G)],
                                      window=w.window or None)
                done += 1
                nbytes += seen * w.d * 2 * 2 + G * (w.d * 2 * 2 + 4)
                if time.perf_counter() - t0 >= budget_s:
                    return done, time.perf_counter() - t0, nbytes
    return done, time.perf_counter() - t0, nbytes


def cpu_baseline(w, inp_cpu, budget_s):
    heads = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    done, dt, fl = oracle_heads(w, inp_cpu, heads, budget_s)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"float64 oracle forward+backward of {done} of {w.B * w.Hq} heads of {w.name} "
                      f"({dt:.1f} s; same algorithmic FLOP count as the GPU metric)"}


def cpu_sdpa_fp32(w, inp_cpu, budget_s):
    """torch's own CPU scaled_dot_product_attention in fp32, forward and
    backward through autograd, one batch entry (all its heads) at a time
    until the budget is spent: a second, less deliberately slow CPU figure
    beside the float64 oracle (the same algorithmic FLOP count)."""
    import torch
    import torch.nn.functional as F
    G = w.Hq // w.Hkv
    pairs = w.T * (w.T + 1) // 2 if w.causal else w.T * w.T
    fl_one = 14 * w.Hq * w.d * pairs
    done, dt, warm = 0, 0.0, False
    for b in [0] + list(range(w.B)):  # the first pass (batch entry 0) warms up, untimed
        q = inp_cpu["q"][b].float().transpose(0, 1).contiguous().requires_grad_()        # [Hq, T, d]
        k = inp_cpu["k"][b].float().transpose(0, 1).repeat_interleave(G, 0).contiguous().requires_grad_()
        v = inp_cpu["v"][b].float().transpose(0, 1).repeat_interleave(G, 0).contiguous().requires_grad_()
        do = inp_cpu["do"][b].float().transpose(0, 1).contiguous()
        t0 = time.perf_counter()
        o = F.scaled_dot_product_attention(q, k, v, is_causal=w.causal, scale=w.scale)
        o.backward(do)
        if warm:
            dt += time.perf_counter() - t0
            done += 1
            if dt >= budget_s:
                break
        warm = True
    return {"value": fl_one * done / dt / 1e12, "unit": "TFLOP/s", "cores": torch.get_num_threads(),
            "kind": "torch CPU scaled_dot_product_attention, fp32, forward + backward (autograd)",
            "sample": f"{done} of {w.B} batch entries (all {w.Hq} heads each) of {w.name} ({dt:.1f} s)"}


# ---------------------------------------------------------------------------
# reference arm
# ---------------------------------------------------------------------------

def run_reference_decode(args, w):
    """The oracle's decode on the host cores: each step one (sequence, KV
    head) group of two sequences drawn like the workload's."""
    from workloads import decode_inputs
    inp = decode_inputs(w.with_(B=2), device="cpu")
    q, kc, vc, sl = inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"]
    G = w.Hq // w.Hkv
    groups = [(b, hkv) for b in range(2) for hkv in range(w.Hkv)]

    def one(s):
        b, hkv = groups[s % len(groups)]
        sub = w.with_(Hq=G, Hkv=1)
        return oracle_decode(sub, q[b:b + 1, hkv * G:(hkv + 1) * G], kc[b:b + 1, :, hkv:hkv + 1],
                             vc[b:b + 1, :, hkv:hkv + 1], sl[b:b + 1], 1e9, max_passes=1)

    for s in range(args.warmup):
        one(s)
    tot_b, tot_t = 0, 0.0
    for s in range(args.steps):
        _, dt, nb = one(s)
        tot_b += nb
        tot_t += dt
    value = tot_b / tot_t / 1e9
    line = {
        "impl": "reference", "metric": "split-KV decode HBM GB/s (bf16 KV cache, 1xB200) and % of HBM peak",
        "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        # a token decodes all Hkv groups of its sequence
        "tokens_per_s": args.steps / w.Hkv / tot_t,
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Tk_max": w.T, "d": w.d,
                   "chunk": w.chunk, "window": w.window or None,
                   "step": "one (sequence, KV head) group of the workload"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one (sequence, KV head) group of {w.name} per step, float64 numpy"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_fp8(args, w):
    """The oracle's forward on E4M3 inputs on the host cores: each step 256
    query rows of one head (heads and row blocks cycling over the workload),
    decoding that head's codes included."""
    import numpy as np
    import torch
    import oracle
    from workloads import prefill_inputs_e4m3
    inp = prefill_inputs_e4m3(w.with_(B=1), device="cpu")
    codes = {n: inp[n].view(torch.uint8).numpy() for n in ("q", "k", "v")}
    G = w.Hq // w.Hkv
    T, n_blk = w.T, (w.T + 255) // 256

    def one(s):
        h, blk = s % w.Hq, (s * 7919) % n_blk
        rows = np.arange(blk * 256, min(T, blk * 256 + 256))
        t0 = time.perf_counter()
        q = oracle.e4m3_decode(codes["q"][0, :, h]) * inp["q_descale"]
        k = oracle.e4m3_decode(codes["k"][0, :, h // G]) * inp["k_descale"]
        v = oracle.e4m3_decode(codes["v"][0, :, h // G]) * inp["v_descale"]
        oracle.head_forward(q, k, v, w.scale, w.causal, rows=rows)
        dt = time.perf_counter() - t0
        keys = np.minimum(rows + 1, T).sum() if w.causal else len(rows) * T
        return dt, 4.0 * w.d * float(keys)

    for s in range(args.warmup):
        one(s)
    tot_t, tot_f = 0.0, 0.0
    for s in range(args.steps):
        dt, fl = one(s)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": "attention forward TFLOPS (E4M3 inputs, 1xB200) and % of dense E4M3 tensor peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "tokens_per_s": tokens_at_rate(value, flops(w)[0], prefill_tokens(w)),
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d, "causal": w.causal,
                   "inputs": "E4M3 codes, per-tensor amax/448 factors",
                   "step": "256 query rows of one head, forward, codes decoded"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"256 query rows of one head of {w.name} per step, float64 numpy"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_dropout(args, w):
    """The oracle's forward + backward with dropout on P on the host cores:
    each step one (batch, head) of the workload (heads cycling)."""
    from oracle import dropout as dr
    from workloads import prefill_inputs, to_f64
    inp = prefill_inputs(w.with_(B=1), device="cpu")
    G = w.Hq // w.Hkv
    f_fwd, f_bwd = flops(w)
    per_head = (f_fwd + f_bwd) / (w.B * w.Hq)

    def one(s):
        h = s % w.Hq
        qh, kh, vh, dh = (to_f64(inp[n][0, :, h if n in ("q", "do") else h // G]) for n in ("q", "k", "v", "do"))
        t0 = time.perf_counter()
        dr.head_forward_dropout(qh, kh, vh, w.scale, w.causal, args.dropout, 0x5EED0000, 0, h)
        dr.head_backward_dropout(qh, kh, vh, dh, w.scale, w.causal, args.dropout, 0x5EED0000, 0, h)
        return time.perf_counter() - t0

    for s in range(args.warmup):
        one(s)
    tot = sum(one(s) for s in range(args.steps))
    value = per_head * args.steps / tot / 1e12
    line = {
        "impl": "reference",
        "metric": "attention fwd+bwd TFLOPS with fused dropout (bf16, 1xB200) and % of dense tensor peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "tokens_per_s": tokens_at_rate(value, f_fwd + f_bwd, prefill_tokens(w)),
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d, "causal": w.causal,
                   "dropout": args.dropout,
                   "step": "one (batch, head) of the workload, forward and backward with dropout"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one (batch, head) of {w.name} per step, float64 numpy"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args, w, rank):
    if rank != 0:
        return 0
    if args.fp8:
        return run_reference_fp8(args, w)
    if args.dropout is not None:
        return run_reference_dropout(args, w)
    if w.decode:
        return run_reference_decode(args, w)
    from workloads import prefill_inputs
    inp = prefill_inputs(w.with_(B=1), device="cpu")
    heads = [(0, h) for h in range(w.Hq)]
    for s in range(args.warmup):
        oracle_heads(w, inp, [heads[s % len(heads)]], 1e9)
    total_fl, total_t = 0.0, 0.0
    for s in range(args.steps):
        done, dt, fl = oracle_heads(w, inp, [heads[s % len(heads)]], 1e9)
        total_fl += fl
        total_t += dt
    value = total_fl / total_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "tokens_per_s": tokens_at_rate(value, sum(flops(w)), prefill_tokens(w)),
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d,
                   "causal": w.causal, "window": w.window or None,
                   "step": "one head of the workload, forward + backward"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"one (batch, head) of {w.name} per step, float64 numpy"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# timing helpers shared by every rank
# ---------------------------------------------------------------------------

def max_over_ranks(value, dist, device=None):
    """Largest `value` over all ranks (the job's time is the slowest rank's)."""
    if dist is None:
        return value
    import torch
    dev = device if (device is not None and dist.get_backend() == "nccl") else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(work_per_rank_step, world, steps, elapsed_ms):
    """Whole-job rate: every rank's work over the slowest rank's time."""
    return world * work_per_rank_step * steps / (elapsed_ms * 1e-3)


# ---------------------------------------------------------------------------
# libfa arm
# ---------------------------------------------------------------------------

class _PrefillRun:
    """Device buffers and the four launches of one fwd+bwd step of a prefill
    workload, called through the C ABI."""

    def __init__(self, lib, fa, w, dev, seed, dropout=None):
        import ctypes
        import torch
        from workloads import prefill_inputs
        self.fa, self.lib, self.w, self.dev = fa, lib, w, dev
        inp = prefill_inputs(w, device=dev, seed=seed)
        self.q, self.k, self.v, self.do = inp["q"], inp["k"], inp["v"], inp["do"]
        B, Hq, Hkv, T, d = w.B, w.Hq, w.Hkv, w.T, w.d
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        self.ws_bytes = lib.fa_backward_workspace_bytes(B, Hq, Hkv, T, T, d)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        P = ctypes.c_void_p
        self.pq, self.pk, self.pv, self.pdo, self.po, self.plse = (
            P(t.data_ptr()) for t in (self.q, self.k, self.v, self.do, self.o, self.lse))
        self.pdq, self.pdk, self.pdv, self.pws = (P(t.data_ptr()) for t in (self.dq, self.dk, self.dv, self.ws))
        self.stream = torch.cuda.current_stream(dev)
        self.sp = P(self.stream.cuda_stream)
        # with a sliding window the windowed entry points take the window in
        # place of the causal flag; with dropout the dropout entry points take
        # (rate, seed, offset) after it
        self.fwd_fn, self.dkdv_fn, self.mask_arg = lib.fa_forward, lib.fa_backward_dkdv, int(w.causal)
        self.extra = ()
        if w.window:
            self.fwd_fn, self.dkdv_fn, self.mask_arg = lib.fa_forward_window, lib.fa_backward_dkdv_window, w.window
        if dropout is not None:
            self.fwd_fn, self.dkdv_fn = lib.fa_forward_dropout, lib.fa_backward_dkdv_dropout
            self.extra = (float(dropout), 0x5EED0000 + seed, 0)

    def _check(self, st, name):
        if st != 0:
            raise RuntimeError(f"{name}: {self.fa.STATUS.get(st, st)}")

    def step(self, evs=None):
        w, lib, s = self.w, self.lib, self.stream
        B, Hq, Hkv, T, d = w.B, w.Hq, w.Hkv, w.T, w.d
        if evs: evs[0].record(s)
        self._check(self.fwd_fn(self.pq, self.pk, self.pv, self.po, self.plse, B, Hq, Hkv, T, T, d, w.scale,
                                self.mask_arg, *self.extra, self.sp), "fa_forward")
        if evs: evs[1].record(s)
        self._check(lib.fa_backward_preprocess(self.po, self.plse, self.pdo, self.pws, self.ws_bytes, B, Hq, Hkv, T,
                                               T, d, self.sp), "preprocess")
        if evs: evs[2].record(s)
        self._check(self.dkdv_fn(self.pq, self.pk, self.pv, self.pdo, self.pdk, self.pdv, self.pws, self.ws_bytes,
                                 B, Hq, Hkv, T, T, d, w.scale, self.mask_arg, *self.extra, self.sp), "dkdv")
        if evs: evs[3].record(s)
        self._check(lib.fa_backward_dq_finalize(self.pdq, self.pws, self.ws_bytes, B, Hq, Hkv, T, T, d, self.sp),
                    "dq_finalize")
        if evs: evs[4].record(s)

    KERNELS_PER_STEP = 4

    def timed(self, steps, warmup, barrier):
        """Warm-up, then `steps` timed steps with events around every launch.
        Returns (elapsed ms of the whole timed region on this rank, average
        ms of each of the four launches)."""
        import torch
        for _ in range(warmup):
            self.step()
        barrier()
        if self.lib.fa_check(self.sp) != 0:
            raise RuntimeError("device status set during warm-up")
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        barrier()
        t0.record(self.stream)
        for s_ in range(steps):
            self.step(evs[s_])
        t1.record(self.stream)
        barrier()
        if self.lib.fa_check(self.sp) != 0:
            raise RuntimeError("device status set during the timed region")
        seg = [sum(evs[s_][i].elapsed_time(evs[s_][i + 1]) for s_ in range(steps)) / steps for i in range(4)]
        return t0.elapsed_time(t1), seg


def prefill_tokens(w):
    """Tokens of one prefill step: B * T."""
    return w.B * w.T


def tokens_at_rate(tflops, flops_per_step, tokens_per_step):
    """Tokens per second of a run that reaches `tflops` on a workload whose
    step does `flops_per_step` over `tokens_per_step` tokens."""
    return tflops * 1e12 * tokens_per_step / flops_per_step


def extra_workloads(args, lib, fa, dev, rank, world, dist, barrier):
    """The long-context prefill workloads and the decode workload, each timed
    on the device in the same run as the headline workload (fewer steps: a
    step is 10-40 ms there).  Summaries only; each has its own bench line
    with `--workload N`."""
    from workloads import WORKLOADS
    import torch
    peaks = load_peaks()
    out = {}
    for idx, steps in ((3, args.extra_steps), (4, max(3, args.extra_steps // 3))):
        w = WORKLOADS[idx]
        run = _PrefillRun(lib, fa, w, dev, w.seed + rank)
        elapsed, seg = run.timed(steps, 3, barrier)
        elapsed = max_over_ranks(elapsed, dist, dev)
        f_fwd, f_bwd = flops(w)
        value = job_rate(f_fwd + f_bwd, world, steps, elapsed) / 1e12
        ms = elapsed / steps
        out[w.name] = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "ms_per_step": ms, "steps": steps, "warmup": 3,
            "frac": value / world / peaks["bf16_tflops"],
            "tokens_per_s": world * prefill_tokens(w) / (ms * 1e-3),
            "per_kernel_ms": {"fa_fwd_kernel": seg[0], "fa_bwd_preprocess_kernel": seg[1],
                              "fa_bwd_dkdv_kernel": seg[2], "fa_bwd_dq_convert_kernel": seg[3]},
            "fwd_tflops": f_fwd / (seg[0] * 1e-3) / 1e12, "dkdv_tflops": f_bwd / (seg[2] * 1e-3) / 1e12,
            "config": {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d, "causal": w.causal, "seed": w.seed + rank},
        }
        del run
        torch.cuda.empty_cache()
    w = WORKLOADS[5]
    dec = _DecodeRun(lib, fa, w, dev, w.seed + rank)
    steps = args.extra_steps * 10
    ms = max_over_ranks(dec.timed(steps, 3, barrier), dist, dev) / steps
    value = world * dec.alg_bytes / (ms * 1e-3) / 1e9
    out[w.name] = {
        "metric": "split-KV decode HBM GB/s (bf16 KV cache, 1xB200) and % of HBM peak", "value": value,
        "unit": "GB/s", "ms_per_step": ms, "steps": steps, "warmup": 3, "frac": value / world / peaks["hbm_gbs"],
        "tokens_per_s": world * w.B / (ms * 1e-3),
        "config": {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Tk_max": w.T, "d": w.d, "chunk": w.chunk,
                   "total_cached_tokens": dec.total_keys, "seed": w.seed + rank},
    }
    del dec
    torch.cuda.empty_cache()
    return out


def run_fa(args, w, rank, world, dist):
    import torch
    import io_aware_exact_forward_b200 as fa

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = fa.load_library()
    run = _PrefillRun(lib, fa, w, dev, w.seed + rank)
    q, k, v, do, o, lse, dq, dk, dv, ws = (run.q, run.k, run.v, run.do, run.o, run.lse, run.dq, run.dk, run.dv,
                                           run.ws)
    B, Hq, Hkv, T, d = w.B, w.Hq, w.Hkv, w.T, w.d
    scale = w.scale
    kernels_per_step = run.KERNELS_PER_STEP

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    gpu_index = local
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            gpu_index = int(vis.split(",")[local])
        except ValueError:
            pass
    with ClockSampler(gpu_index) as clocks:
        elapsed_ms, seg = run.timed(args.steps, args.warmup, barrier)
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    ms_per_step = elapsed_ms / args.steps
    f_fwd, f_bwd = flops(w)
    value = job_rate(f_fwd + f_bwd, world, args.steps, elapsed_ms) / 1e12

    # roofline of the dominant kernel (largest share of the step)
    peaks = load_peaks()
    names = ["fa_fwd_kernel", "fa_bwd_preprocess_kernel", "fa_bwd_dkdv_kernel", "fa_bwd_dq_convert_kernel"]
    dom = max(range(4), key=lambda i: seg[i])
    if dom == 0:
        alg, bound = f_fwd, "tensor"
    elif dom == 2:
        alg, bound = f_bwd, "tensor"
    else:
        alg, bound = None, "hbm"
    if alg is not None:
        achieved = alg / (seg[dom] * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"kernel": names[dom], "bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": f"{peaks['source']} bf16 dense (burst)",
                "traffic": traffic_from_profile(names[dom], w.name), "traffic_unit": "bytes per launch",
                "algorithmic_per_launch": alg}
    else:
        roof = {"kernel": names[dom], "bound": bound, "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": None, "traffic": None}
    per_kernel = {names[i]: {"ms_avg": seg[i]} for i in range(4)}
    per_kernel["fa_fwd_kernel"]["tflops"] = f_fwd / (seg[0] * 1e-3) / 1e12
    per_kernel["fa_bwd_dkdv_kernel"]["tflops"] = f_bwd / (seg[2] * 1e-3) / 1e12
    per_kernel["backward_total_tflops"] = f_bwd / (sum(seg[1:]) * 1e-3) / 1e12

    # end to end through the public API, host buffers in pinned memory
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        hdq = torch.empty(dq.shape, dtype=dq.dtype, pin_memory=True)
        hdk = torch.empty(dk.shape, dtype=dk.dtype, pin_memory=True)
        hdv = torch.empty(dv.shape, dtype=dv.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
        d2h = sum(t.numel() * t.element_size() for t in (ho, hlse, hdq, hdk, hdv))

        # Two device slots and three streams: step i+1's inputs are copied in
        # (and step i-1's results copied out) while step i computes.  Every
        # step still moves its own inputs in and its own results out.
        win = w.window or None
        slots = []
        for _ in range(2):
            slots.append({"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
                          "do": torch.empty_like(do), "o": torch.empty_like(o), "lse": torch.empty_like(lse),
                          "dq": torch.empty_like(dq), "dk": torch.empty_like(dk), "dv": torch.empty_like(dv)})
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            for i in range(n):
                sl, j = slots[i % 2], i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_comp[j])      # step i-2 has read this slot's inputs
                    sl["q"].copy_(hq, non_blocking=True); sl["k"].copy_(hk, non_blocking=True)
                    sl["v"].copy_(hv, non_blocking=True); sl["do"].copy_(hdo, non_blocking=True)
                    ev_in[j].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(ev_in[j])
                    if i >= 2:
                        s_comp.wait_event(ev_out[j])     # step i-2's results have left this slot
                    fa.forward(sl["q"], sl["k"], sl["v"], scale=scale, causal=w.causal, out=sl["o"], lse=sl["lse"],
                               window=win)
                    fa.backward(sl["q"], sl["k"], sl["v"], sl["o"], sl["lse"], sl["do"], scale=scale, causal=w.causal,
                                workspace=ws, dq=sl["dq"], dk=sl["dk"], dv=sl["dv"], window=win)
                    ev_comp[j].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[j])
                    ho.copy_(sl["o"], non_blocking=True); hlse.copy_(sl["lse"], non_blocking=True)
                    hdq.copy_(sl["dq"], non_blocking=True); hdk.copy_(sl["dk"], non_blocking=True)
                    hdv.copy_(sl["dv"], non_blocking=True)
                    ev_out[j].record(s_out)

        e2e_steps(3)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_steps(args.e2e_steps)
        e1.record(s_out)
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        e2e = {"value": job_rate(f_fwd + f_bwd, world, args.e2e_steps, e_ms) / 1e12, "unit": "TFLOP/s",
               "tokens_per_s": world * prefill_tokens(w) * args.e2e_steps / (e_ms * 1e-3),
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "ms_per_step": e_ms / args.e2e_steps,
               "pipelining": "two device slots; copies of neighbouring steps overlap compute on separate streams"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = {"q": q.cpu(), "k": k.cpu(), "v": v.cpu(), "do": do.cpu()}
        cpu = cpu_baseline(w, inp_cpu, args.cpu_seconds)
        cpu["tokens_per_s"] = cpu["value"] * 1e12 / ((f_fwd + f_bwd) / prefill_tokens(w))
        sdpa = cpu_sdpa_fp32(w, inp_cpu, min(args.cpu_seconds, 10.0))
        sdpa["tokens_per_s"] = sdpa["value"] * 1e12 / ((f_fwd + f_bwd) / prefill_tokens(w))
        cpu["second_baseline"] = sdpa

    extras = None
    if args.workload == 2 and not w.window and args.batch is None and not args.no_extra:
        del run, q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()
        extras = extra_workloads(args, lib, fa, dev, rank, world, dist, barrier)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "tokens_per_s": world * prefill_tokens(w) / (ms_per_step * 1e-3),
            "config": {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "T": T, "d": d, "causal": w.causal,
                       "window": w.window or None,
                       "step": "fa_forward + fa_backward (preprocess, dkdv, dq_finalize)",
                       "l2": "inputs larger than L2 (q, k, v, dO: 4 x %d MiB per step)" % (B * T * Hq * d * 2 >> 20),
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "seed": w.seed},
            "pct_of_peak": {"measured": value / world / peaks["bf16_tflops"], "spec_2250": value / world / 2250.0},
            "roofline": roof,
            "per_kernel": per_kernel,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": kernels_per_step * args.steps,
            "clocks": clocks.summary(),
            "workloads": extras,
        }
        print(json.dumps(line), flush=True)
    return 0


class _DecodeRun:
    """Device buffers and the launch of one split-KV decode step, called
    through the C ABI."""

    def __init__(self, lib, fa, w, dev, seed):
        import ctypes
        import torch
        from workloads import decode_inputs
        self.fa, self.lib, self.w, self.dev = fa, lib, w, dev
        inp = decode_inputs(w, device=dev, seed=seed)
        self.q, self.kc, self.vc, self.sl = inp["q"], inp["k_cache"], inp["v_cache"], inp["seqlens"]
        B, Hq, Hkv, Tk_max, d, chunk = w.B, w.Hq, w.Hkv, w.T, w.d, w.chunk
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        self.wsb = lib.fa_decode_workspace_bytes(B, Hq, Tk_max, d, chunk)
        self.ws = torch.empty(self.wsb, dtype=torch.uint8, device=dev)
        P = ctypes.c_void_p
        self.stream = torch.cuda.current_stream(dev)
        self.sp = P(self.stream.cuda_stream)
        args_c = (P(self.q.data_ptr()), P(self.kc.data_ptr()), P(self.vc.data_ptr()), P(self.sl.data_ptr()),
                  P(self.o.data_ptr()), P(self.lse.data_ptr()), P(self.ws.data_ptr()), self.wsb, B, Hq, Hkv,
                  Tk_max, d, w.scale, chunk)
        self.fn = lib.fa_decode_splitkv
        if w.window:
            self.fn = lib.fa_decode_splitkv_window
            args_c = args_c + (w.window,)
        self.args_c = args_c + (self.sp,)
        # keys the query sees: the whole prefix, or its last `window` keys
        sl = self.sl
        self.total_keys = int(sl.clamp(max=w.window).sum().item()) if w.window else int(sl.sum().item())
        self.alg_bytes = (self.total_keys * Hkv * d * 2 * 2 + self.q.numel() * 2 + self.o.numel() * 2
                          + self.lse.numel() * 4)

    def step(self):
        st = self.fn(*self.args_c)
        if st != 0:
            raise RuntimeError(f"fa_decode_splitkv: {self.fa.STATUS.get(st, st)}")

    KERNELS_PER_STEP = 3   # split, combine, empty-sequence kernels

    def timed(self, steps, warmup, barrier):
        """Elapsed ms of `steps` decode steps on this rank after `warmup`; the
        cache (2 x 4.3 GB) is far larger than L2, so no flush is needed."""
        import torch
        for _ in range(warmup):
            self.step()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(steps):
            self.step()
        e1.record(self.stream)
        barrier()
        if self.lib.fa_check(self.sp) != 0:
            raise RuntimeError("device status set during the timed region")
        return e0.elapsed_time(e1)


def run_decode(args, w, rank, world, dist):
    """Split-KV decode of the B=64, Hq=32, Hkv=8, d=128 batch: one step is
    fa_decode_splitkv (split kernel + combine kernel); value is algorithmic
    HBM GB/s (K and V of every cached token read once, plus q, o, lse)."""
    import torch
    import io_aware_exact_forward_b200 as fa

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = fa.load_library()
    run = _DecodeRun(lib, fa, w, dev, w.seed + rank)
    q, kc, vc, sl, o, lse, ws = run.q, run.kc, run.vc, run.sl, run.o, run.lse, run.ws
    B, Hq, Hkv, Tk_max, d, chunk = w.B, w.Hq, w.Hkv, w.T, w.d, w.chunk
    total_keys, alg_bytes = run.total_keys, run.alg_bytes

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    with ClockSampler(local) as clocks:
        ms = max_over_ranks(run.timed(args.steps, args.warmup, barrier), dist, dev)
    value = job_rate(alg_bytes, world, args.steps, ms) / 1e9

    # End to end through the public binding: per step the query rows and the
    # sequence lengths come in from pinned host memory and O and LSE go back;
    # the KV cache is state that stays resident, as in serving.
    e2e = None
    if not args.no_e2e:
        hq, hsl = q.cpu().pin_memory(), sl.cpu().pin_memory()
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        win = w.window or None

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            sl.copy_(hsl, non_blocking=True)
            fa.decode_splitkv(q, kc, vc, sl, scale=w.scale, chunk=chunk, workspace=ws, out=o, lse=lse, window=win)
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        for _ in range(3):
            e2e_step()
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(run.stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        f1.record(run.stream)
        barrier()
        e_ms = max_over_ranks(f0.elapsed_time(f1), dist, dev)
        e2e = {"value": job_rate(alg_bytes, world, args.e2e_steps, e_ms) / 1e9, "unit": "GB/s",
               "tokens_per_s": world * B * args.e2e_steps / (e_ms * 1e-3),
               "h2d_bytes_per_step": hq.numel() * hq.element_size() + hsl.numel() * hsl.element_size(),
               "d2h_bytes_per_step": ho.numel() * ho.element_size() + hlse.numel() * hlse.element_size(),
               "steps": args.e2e_steps, "ms_per_step": e_ms / args.e2e_steps,
               "note": "the KV cache stays resident on the device"}
    peaks = load_peaks()
    # dominant kernel time: split kernel alone, timed separately on the same stream
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle over the first two sequences' caches, copied to the host
        nb, dt, nbytes = oracle_decode(w, q[:2].cpu(), kc[:2].cpu(), vc[:2].cpu(), sl[:2].cpu(), args.cpu_seconds)
        cpu = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
               "tokens_per_s": nb / w.Hkv / dt,
               "sample": f"float64 oracle decode of {nb} (sequence, KV head) groups, cycling over the first two "
                         f"sequences of {w.name} ({dt:.1f} s; same algorithmic bytes as the GPU metric)"}

    if rank == 0:
        line = {
            "metric": "split-KV decode HBM GB/s (bf16 KV cache, 1xB200) and % of HBM peak",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "tokens_per_s": world * B * args.steps / (ms * 1e-3),
            "config": {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "Tk_max": Tk_max, "d": d, "chunk": chunk,
                       "total_cached_tokens": total_keys, "window": w.window or None,
                       "l2": "KV cache larger than L2", "seed": w.seed},
            "roofline": {"kernel": "fa_decode_split_kernel + fa_decode_combine_kernel", "bound": "hbm",
                         "achieved": value / world, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": value / world / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} HBM copy",
                         "traffic": traffic_from_profile("fa_decode_split_kernel", w.name),
                         "algorithmic_per_launch": alg_bytes},
            "gpu_launches": 3 * args.steps,   # split, combine, empty-sequence kernels
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
            "e2e": e2e,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_fp8_forward(args, w, rank, world, dist):
    """The E4M3 forward on a d = 128 prefill workload: one step is one
    fa_forward_fp8 launch over the whole batch (Q, K, V codes resident).
    value is algorithmic TFLOP/s (4 B Hq d pairs); the roofline denominator is
    the measured bf16 peak times 2, the nominal E4M3:bf16 ratio of the tensor
    cores (4.5 : 2.25 PFLOP/s dense)."""
    import ctypes
    import torch
    import io_aware_exact_forward_b200 as fa
    from workloads import prefill_inputs_e4m3

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = fa.load_library()
    inp = prefill_inputs_e4m3(w, device=dev, seed=w.seed + rank)
    q, k, v = inp["q"], inp["k"], inp["v"]
    qs, ks, vs = inp["q_descale"], inp["k_descale"], inp["v_descale"]
    B, Hq, Hkv, T, d = w.B, w.Hq, w.Hkv, w.T, w.d
    o = torch.empty((B, T, Hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
    P = ctypes.c_void_p
    stream = torch.cuda.current_stream(dev)
    sp = P(stream.cuda_stream)
    args_c = (P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), qs, ks, vs, P(o.data_ptr()), P(lse.data_ptr()),
              B, Hq, Hkv, T, T, d, w.scale, int(w.causal), sp)

    def step():
        st = lib.fa_forward_fp8(*args_c)
        if st != 0:
            raise RuntimeError(f"fa_forward_fp8: {fa.STATUS.get(st, st)}")

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    # L2 is flushed between timed launches by writing a 256 MiB buffer
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        for s_ in range(args.steps):
            flush.fill_(s_ & 0xFF)
            evs[s_][0].record(stream)
            step()
            evs[s_][1].record(stream)
        barrier()
    if lib.fa_check(sp) != 0:
        raise RuntimeError("device status set during the timed region")
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), dist, dev)
    f_fwd, _ = flops(w)
    value = job_rate(f_fwd, world, args.steps, ms) / 1e12
    peaks = load_peaks()
    peak = 2.0 * peaks["bf16_tflops"]

    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            fa.forward_fp8(q, k, v, qs, ks, vs, scale=w.scale, causal=w.causal, out=o, lse=lse)
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        for _ in range(3):
            e2e_step()
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        f1.record(stream)
        barrier()
        e_ms = max_over_ranks(f0.elapsed_time(f1), dist, dev)
        e2e = {"value": job_rate(f_fwd, world, args.e2e_steps, e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hq, hk, hv)),
               "d2h_bytes_per_step": ho.numel() * ho.element_size() + hlse.numel() * hlse.element_size(),
               "steps": args.e2e_steps, "ms_per_step": e_ms / args.e2e_steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        G = Hq // Hkv
        per_head = f_fwd / (B * Hq)
        qc, kc, vc = (t.view(torch.uint8).cpu() for t in (q, k, v))
        done, t0 = 0, time.perf_counter()
        for h in range(Hq):
            oracle.attention_forward_e4m3(qc[:1, :, h:h + 1].numpy(), kc[:1, :, h // G:h // G + 1].numpy(),
                                          vc[:1, :, h // G:h // G + 1].numpy(), qs, ks, vs, w.scale, w.causal)
            done += 1
            if time.perf_counter() - t0 >= args.cpu_seconds:
                break
        dt = time.perf_counter() - t0
        cpu = {"value": done * per_head / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"float64 oracle forward on E4M3 inputs, {done} of {B * Hq} heads of {w.name} "
                         f"({dt:.1f} s; same algorithmic FLOP count as the GPU metric)"}
    if rank == 0:
        line = {
            "metric": "attention forward TFLOPS (E4M3 inputs, 1xB200) and % of dense E4M3 tensor peak",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3", "data": "synthetic",
            "tokens_per_s": world * prefill_tokens(w) * args.steps / (ms * 1e-3),
            "config": {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "T": T, "d": d, "causal": w.causal,
                       "inputs": "E4M3 codes, per-tensor amax/448 factors", "l2": "256 MiB flush between launches",
                       "seed": w.seed},
            "roofline": {"kernel": "fa_fwd_kernel<128, true>", "bound": "tensor", "achieved": value / world,
                         "peak": peak, "unit": "TFLOP/s", "frac": value / world / peak,
                         "peak_source": f"{peaks['source']} bf16 dense (burst) x 2, the nominal E4M3:bf16 ratio",
                         "traffic": None, "algorithmic_per_launch": f_fwd},
            "gpu_launches": args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
            "e2e": e2e,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_dropout(args, w, rank, world, dist):
    """Forward + backward with fused dropout on P (rate args.dropout) on a
    prefill workload: one step is fa_forward_dropout + the three backward
    steps with fa_backward_dkdv_dropout (inputs resident, larger than L2).
    value is algorithmic TFLOP/s (14 B Hq d pairs; the mask's work is not
    counted).  The plain fwd+bwd step is timed the same way in the same run
    for the overhead."""
    import torch
    import io_aware_exact_forward_b200 as fa

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = fa.load_library()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    run = _PrefillRun(lib, fa, w, dev, w.seed + rank, dropout=args.dropout)
    with ClockSampler(local) as clocks:
        elapsed, seg = run.timed(args.steps, args.warmup, barrier)
    del run
    plain = _PrefillRun(lib, fa, w, dev, w.seed + rank)
    elapsed_plain, seg_plain = plain.timed(args.steps, args.warmup, barrier)
    del plain
    elapsed = max_over_ranks(elapsed, dist, dev)
    elapsed_plain = max_over_ranks(elapsed_plain, dist, dev)
    f_fwd, f_bwd = flops(w)
    value = job_rate(f_fwd + f_bwd, world, args.steps, elapsed) / 1e12
    ms = elapsed / args.steps
    peaks = load_peaks()
    names = ["fa_fwd_kernel<d, false, true>", "fa_bwd_preprocess_kernel", "fa_bwd_dkdv_kernel<d, false, true>",
             "fa_bwd_dq_convert_kernel"]
    dom = max(range(4), key=lambda i: seg[i])
    alg = f_fwd if dom == 0 else (f_bwd if dom == 2 else None)
    if rank == 0:
        line = {
            "metric": "attention fwd+bwd TFLOPS with fused dropout (bf16, 1xB200) and % of dense tensor peak",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "tokens_per_s": world * prefill_tokens(w) / (ms * 1e-3),
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d,
                       "causal": w.causal, "dropout": args.dropout,
                       "step": "fa_forward_dropout + preprocess + fa_backward_dkdv_dropout + dq_finalize",
                       "l2": "inputs larger than L2", "seed": w.seed},
            "per_kernel_ms": {names[i]: seg[i] for i in range(4)},
            "fwd_tflops": f_fwd / (seg[0] * 1e-3) / 1e12, "dkdv_tflops": f_bwd / (seg[2] * 1e-3) / 1e12,
            "plain": {"ms_per_step": elapsed_plain / args.steps,
                      "tflops": job_rate(f_fwd + f_bwd, world, args.steps, elapsed_plain) / 1e12,
                      "per_kernel_ms": seg_plain},
            "roofline": {"kernel": names[dom], "bound": "tensor" if alg else "hbm",
                         "achieved": alg / (seg[dom] * 1e-3) / 1e12 if alg else None,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": alg / (seg[dom] * 1e-3) / 1e12 / peaks["bf16_tflops"] if alg else None,
                         "peak_source": f"{peaks['source']} bf16 dense (burst)", "traffic": None,
                         "algorithmic_per_launch": alg},
            "gpu_launches": _PrefillRun.KERNELS_PER_STEP * args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": None,
            "e2e": None,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_deterministic(args, w, rank, world, dist):
    """Forward + the deterministic backward (fa_backward_deterministic: the
    preprocess, the dK/dV kernel without dQ and the dQ pass in one call) on a
    prefill workload, inputs resident and larger than L2; the default step
    (fused dQ) is timed the same way in the same run for comparison."""
    import torch
    import io_aware_exact_forward_b200 as fa

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = fa.load_library()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    run = _PrefillRun(lib, fa, w, dev, w.seed + rank)
    B, Hq, Hkv, T, d = w.B, w.Hq, w.Hkv, w.T, w.d
    causal, window = int(w.causal or bool(w.window)), int(w.window or 0)

    def step(evs=None):
        s = run.stream
        if evs: evs[0].record(s)
        run._check(run.fwd_fn(run.pq, run.pk, run.pv, run.po, run.plse, B, Hq, Hkv, T, T, d, w.scale,
                              run.mask_arg, run.sp), "fa_forward")
        if evs: evs[1].record(s)
        run._check(lib.fa_backward_deterministic(run.pq, run.pk, run.pv, run.po, run.plse, run.pdo, run.pdq, run.pdk,
                                                 run.pdv, run.pws, run.ws_bytes, B, Hq, Hkv, T, T, d, w.scale,
                                                 causal, window, run.sp), "fa_backward_deterministic")
        if evs: evs[2].record(s)

    for _ in range(args.warmup):
        step()
    barrier()
    if lib.fa_check(run.sp) != 0:
        raise RuntimeError("device status set during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(run.stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(run.stream)
        barrier()
    if lib.fa_check(run.sp) != 0:
        raise RuntimeError("device status set in the timed region")
    elapsed = t0.elapsed_time(t1)
    seg = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j in range(2)]
    elapsed_plain, seg_plain = run.timed(args.steps, args.warmup, barrier)
    del run
    elapsed = max_over_ranks(elapsed, dist, dev)
    elapsed_plain = max_over_ranks(elapsed_plain, dist, dev)
    f_fwd, f_bwd = flops(w)
    value = job_rate(f_fwd + f_bwd, world, args.steps, elapsed) / 1e12
    ms = elapsed / args.steps
    peaks = load_peaks()
    bwd_name = "fa_backward_deterministic (preprocess, dK/dV without dQ, dQ pass)"
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "tokens_per_s": world * prefill_tokens(w) / (ms * 1e-3),
            "config": {"workload": w.name, "B": B, "Hq": Hq, "Hkv": Hkv, "T": T, "d": d, "causal": w.causal,
                       "window": w.window or None,
                       "step": "fa_forward + fa_backward_deterministic", "l2": "inputs larger than L2",
                       "seed": w.seed},
            "per_kernel_ms": {"fa_fwd_kernel": seg[0], bwd_name: seg[1]},
            "default": {"ms_per_step": elapsed_plain / args.steps,
                        "tflops": job_rate(f_fwd + f_bwd, world, args.steps, elapsed_plain) / 1e12,
                        "per_kernel_ms": seg_plain},
            # the backward is one call of three launches: its roofline is the
            # call's, against the tensor peak
            "roofline": {"kernel": bwd_name, "bound": "tensor", "achieved": f_bwd / (seg[1] * 1e-3) / 1e12,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": f_bwd / (seg[1] * 1e-3) / 1e12 / peaks["bf16_tflops"],
                         "peak_source": f"{peaks['source']} bf16 dense (burst)", "traffic": None,
                         "algorithmic_per_launch": f_bwd},
            "gpu_launches": 4 * args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": None,
            "e2e": None,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_decode_cp(args, w, rank, world, dist):
    """Context-parallel decode of the same batch: every sequence's cache is
    cut into `world` contiguous shares and rank r holds share r.  One step is
    fa_decode_splitkv_partial on the local share, one NCCL all-gather of the
    packed fp32 (O, LSE) blocks and fa_decode_merge.  The whole batch's
    algorithmic bytes are fixed as N grows (strong scaling); value is those
    bytes per step over the slowest rank's step time."""
    import ctypes
    import torch
    import io_aware_exact_forward_b200 as fa
    from io_aware_exact_forward_b200 import context_parallel as cp
    from workloads import decode_inputs

    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    lib = fa.load_library()
    full = decode_inputs(w, device=dev)            # the same batch on every rank
    B, Hq, Hkv, Tk_max, d, chunk = w.B, w.Hq, w.Hkv, w.T, w.d, w.chunk
    shard_len = (Tk_max + world - 1) // world
    lo = rank * shard_len
    q, sl_full = full["q"], full["seqlens"]
    kc = full["k_cache"][:, lo:lo + shard_len].contiguous()
    vc = full["v_cache"][:, lo:lo + shard_len].contiguous()
    del full
    torch.cuda.empty_cache()
    sl = cp.shard_seqlens(sl_full, rank, shard_len)
    Tk_loc = kc.shape[1]
    total_keys = int(sl_full.sum().item())
    n = cp.packed_block_floats(B, Hq, d)
    n_o = B * Hq * d
    block = torch.empty(n, dtype=torch.float32, device=dev)
    gathered = torch.empty(world * n, dtype=torch.float32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    wsb = lib.fa_decode_workspace_bytes(B, Hq, Tk_loc, d, chunk)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    P = ctypes.c_void_p
    stream = torch.cuda.current_stream(dev)
    sp = P(stream.cuda_stream)
    part_args = (P(q.data_ptr()), P(kc.data_ptr()), P(vc.data_ptr()), P(sl.data_ptr()), P(block.data_ptr()),
                 P(block.data_ptr() + 4 * n_o), P(ws.data_ptr()), wsb, B, Hq, Hkv, Tk_loc, d, w.scale, chunk, sp)
    merge_args = (P(gathered.data_ptr()), n, P(gathered.data_ptr() + 4 * n_o), n, P(o.data_ptr()),
                  P(lse.data_ptr()), world, B, Hq, d, sp)

    def step():
        st = lib.fa_decode_splitkv_partial(*part_args)
        if st != 0:
            raise RuntimeError(f"fa_decode_splitkv_partial: {fa.STATUS.get(st, st)}")
        dist.all_gather_into_tensor(gathered, block)
        st = lib.fa_decode_merge(*merge_args)
        if st != 0:
            raise RuntimeError(f"fa_decode_merge: {fa.STATUS.get(st, st)}")

    alg_bytes = total_keys * Hkv * d * 2 * 2 + q.numel() * 2 + o.numel() * 2 + lse.numel() * 4

    def barrier():
        dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
    if lib.fa_check(sp) != 0:
        raise RuntimeError("device status set during the timed region")
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    value = alg_bytes * args.steps / (ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            oo, ll = fa.decode_splitkv_cp(q, kc, vc, sl, scale=w.scale, chunk=chunk, workspace=ws)
            ho.copy_(oo, non_blocking=True)
            hlse.copy_(ll, non_blocking=True)

        for _ in range(3):
            e2e_step()
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        f1.record(stream)
        barrier()
        e_ms = max_over_ranks(f0.elapsed_time(f1), dist, dev)
        e2e = {"value": alg_bytes * args.e2e_steps / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": hq.numel() * hq.element_size(),
               "d2h_bytes_per_step": ho.numel() * ho.element_size() + hlse.numel() * hlse.element_size(),
               "steps": args.e2e_steps, "ms_per_step": e_ms / args.e2e_steps,
               "note": "each rank's share of the KV cache and the sequence lengths stay resident"}
    peaks = load_peaks()
    if rank == 0:
        line = {
            "metric": "split-KV decode HBM GB/s (bf16 KV cache, 1xB200) and % of HBM peak",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "tokens_per_s": B * args.steps / (ms * 1e-3),
            "config": {"workload": w.name, "context_parallel": True, "B": B, "Hq": Hq, "Hkv": Hkv,
                       "Tk_max": Tk_max, "shard_len": shard_len, "d": d, "chunk": chunk,
                       "total_cached_tokens": total_keys, "l2": "KV cache larger than L2", "seed": w.seed},
            "roofline": {"kernel": "fa_decode_split_kernel + fa_decode_combine_kernel + fa_decode_merge_kernel",
                         "bound": "hbm", "achieved": value / world, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": value / world / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} HBM copy",
                         "traffic": None, "algorithmic_per_launch": alg_bytes / world},
            "gpu_launches": 4 * args.steps,   # split, combine, empty-sequence and merge kernels (plus NCCL's)
            "clocks": clocks.summary(),
            "cpu_baseline": None,
            "e2e": e2e,
        }
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    from workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.batch is not None:
        w = w.with_(B=args.batch)
    if args.window is not None:
        if args.window < 1:
            print("--window must be >= 1", file=sys.stderr)
            return 2
        w = w.with_(window=args.window, causal=not w.decode)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.fp8 and (w.decode or w.d != 128 or w.window):
        print("--fp8 applies to the d = 128 prefill workloads without a window", file=sys.stderr)
        return 2
    if args.dropout is not None and (w.decode or w.window or not (0.0 <= args.dropout < 1.0)):
        print("--dropout takes a rate in [0, 1) and applies to the prefill workloads without a window",
              file=sys.stderr)
        return 2
    if args.deterministic and (w.decode or args.fp8 or args.dropout is not None):
        print("--deterministic applies to the plain prefill workloads (no --fp8 or --dropout)", file=sys.stderr)
        return 2
    if args.cp and (not w.decode or w.window):
        print("--cp applies to the decode workload without a window", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, w, rank)
    if world > 1 or args.cp:
        import datetime
        import torch
        import torch.distributed as tdist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29533")
        tdist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        if args.fp8:
            return run_fp8_forward(args, w, rank, world, dist)
        if args.dropout is not None:
            return run_dropout(args, w, rank, world, dist)
        if args.deterministic:
            return run_deterministic(args, w, rank, world, dist)
        if w.decode and args.cp:
            return run_decode_cp(args, w, rank, world, dist)
        if w.decode:
            return run_decode(args, w, rank, world, dist)
        return run_fa(args, w, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
