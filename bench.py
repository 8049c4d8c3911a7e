#!/usr/bin/env python
"""Benchmark of the fused softmax-weighted average on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * the GRADIENT query (swa_attn_grad): causal attention forward (bf16,
    B=2 H=16 N=16384 D=64, scale 1/8) -- out and lse -- and the gradient of
    loss = 1/2 sum out^2 with respect to q, k, v;
  * the Nadaraya-Watson regrid (fp32, 16384 targets x 16384 sources in
    [0,10]^2, h = 0.5).
The other workloads (the 4x16x4096 forward, the 1x8x65536 forward + gradient
with and without 0.01% of V set to +inf, the float32 256-token call) are
timed after the step, each beside a bounded oracle sample, under "configs".
The metric is attention TFLOP/s with FLOPs counted causally (N(N+1)/2 pairs
per head; forward 4*D per pair, backward 2.5x forward), over the whole
step's device time.  Inputs (201 MB of Q, K, V) exceed the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1: launched by torchrun, one process per GPU; the problem is one batch
of B*N sequences (and N blocks of regrid targets), split across the ranks by
sequences -- rank r computes sequences [rB, rB+B), its heads -- with no
collective in the data path (weak scaling: per-rank work fixed); the
elapsed time is the max over ranks.  --impl reference times the float64
CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal attention fwd+bwd TFLOP/s (bf16, D=64) and % of BF16 tensor peak, 1×B200"
B, H, N, D = 2, 16, 16384, 64
SEED = 4
NW_M = NW_S = 16384
NW_SEED = 2
H_BW = 0.5
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
SM_MAX_MHZ = 1965.0
MUFU_GPAIRS = 148 * 16 * SM_MAX_MHZ * 1e6 / 1e9  # one ex2 per pair, Gpair/s

# kernel id -> (name, source file whose hash keys the recorded ncu traffic)
KERNELS = {
    1: ("attn_fwd", "causal_attention_swa_b200/csrc/attn_fwd_tc.cu"),
    2: ("attn_bwd", "causal_attention_swa_b200/csrc/attn_bwd_tc.cu"),
    3: ("nw_regrid", "causal_attention_swa_b200/csrc/nw_regrid.cu"),
}


def attn_flops(b=B, h=H, n=N, d=D):
    pairs = n * (n + 1) // 2
    fwd = 4 * d * b * h * pairs
    return fwd, 2.5 * fwd


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", 0) or 0),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=0.0, source="fallback")


def source_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel_id):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's source changed since the counters were taken."""
    name, src = KERNELS[kernel_id]
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(name)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha") != source_sha(src):
        return None
    return float(rec["bytes_per_launch"])


# --------------------------------------------------------------------- clocks

NVML_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every 20 ms
    while the timed region runs (read-only queries)."""

    def __init__(self, index):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no clocks rather than guess
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, int(reasons)))
            except Exception:
                pass
            self._stop.wait(0.02)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(name for bit, name in NVML_REASONS.items() if bits & bit)
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle

def host_threads():
    """Threads for the oracle: every core this process may run on (torchrun sets
    OMP_NUM_THREADS=1 for its ranks; the oracle leg runs on rank 0 alone)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except (AttributeError, OSError):
        return max(1, os.cpu_count() or 1)


def oracle_sample(head_tokens, nw_targets, seed=SEED, threads=0):
    """Time the float64 oracle on a bounded sample of the step: one head of
    the attention batch (its first `head_tokens` tokens as a causal problem)
    forward + backward, and `nw_targets` regrid targets against all sources.
    Returns (seconds, attention FLOPs of the sample by the causal count)."""
    import oracle
    from causal_attention_swa_b200 import inputs
    qb, kb, vb, _ = inputs.attn_bf16(1, 1, head_tokens, seed=seed)
    q, k, v = (inputs.bf16_to_f64(b) for b in (qb, kb, vb))
    t, s, y = inputs.nw_grid(NW_M, NW_S, NW_SEED)
    t0 = time.perf_counter()
    out, _ = oracle.attn_fwd(q, k, v, threads=threads)
    oracle.attn_bwd(q, k, v, out, out=out, threads=threads)
    oracle.nw_regrid(t[:nw_targets], s, y, h=H_BW, threads=threads)
    dt = time.perf_counter() - t0
    fwd, bwd = attn_flops(1, 1, head_tokens)
    return dt, fwd + bwd


def run_reference(args, info):
    """--impl reference: the float64 oracle on the host cores, rank 0 only."""
    from causal_attention_swa_b200 import dist as sdist
    if not info.is_root:
        return 0
    threads = host_threads()
    head_tokens, nw_targets = 4096, 128
    for _ in range(args.warmup):
        oracle_sample(1024, 16, threads=threads)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample(head_tokens, nw_targets, threads=threads)
        times.append(dt)
        flops = fl
    mean_s = sum(times) / len(times)
    value = flops / mean_s / 1e12
    sample = (f"per step: head 0 of the {B}x{H}x{N} batch, its first {head_tokens} tokens "
              f"as a causal problem, forward + backward, plus {nw_targets} of {NW_M} regrid "
              f"targets against all {NW_S} sources")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": info.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"causal attention fwd+bwd B={B} H={H} N={N} D={D} + "
                               f"Nadaraya-Watson regrid {NW_M}x{NW_S} (bounded sample)",
                   "global_batch": B, "seq_len": N, "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    sdist.shutdown()
    return 0


# ----------------------------------------------------------------- our arm

def timed_grad(swa, q, k, v, causal, stream, device, ws, reps=5, warm=2):
    """Median of (reps - warm) gradient calls: whole-call, forward-kernel and
    backward-kernel times (CUDA events, the library's profiling hook)."""
    import torch
    out, lse = torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    rows = []
    for rep in range(reps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        for e in ev:
            e.record(stream)
        ev[0].record(stream)
        swa.profile_kernel(swa.SWA_KERNEL_ATTN_FWD, ev[2], ev[3])
        swa.attn_grad(q, k, v, causal=causal, out=out, lse=lse, dq=dq, dk=dk, dv=dv,
                      workspace=ws)
        ev[1].record(stream)
        swa.profile_kernel(swa.SWA_KERNEL_ATTN_BWD, ev[4], ev[5])
        swa.attn_grad(q, k, v, causal=causal, out=out, lse=lse, dq=dq, dk=dk, dv=dv,
                      workspace=ws)
        swa.profile_kernel(swa.SWA_KERNEL_NONE)
        torch.cuda.synchronize(device)
        if rep >= warm:
            rows.append((ev[0].elapsed_time(ev[1]), ev[2].elapsed_time(ev[3]),
                         ev[4].elapsed_time(ev[5])))
    if swa.get_device_error(device) != swa.SWA_OK:
        raise RuntimeError("device error word set during the gradient calls")
    med = lambda i: statistics.median(r[i] for r in rows)  # noqa: E731
    return {"call_ms": med(0), "fwd_ms": med(1), "bwd_ms": med(2)}


def timed_call(fn, stream, device, reps=7, warm=2):
    import torch
    ts = []
    for rep in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize(device)
        if rep >= warm:
            ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def oracle_attn_rate(qb, kb, vb, heads, tokens, backward, threads, v_f64=None):
    """Oracle TFLOP/s (causal count) on heads[...]'s first `tokens` tokens."""
    import oracle
    from causal_attention_swa_b200 import inputs
    q, k, v = (inputs.bf16_to_f64(b[:, :, :tokens]) for b in (qb, kb, vb))
    B_, H_ = qb.shape[:2]
    q, k, v = (a.reshape(B_ * H_, 1, tokens, 64)[heads] for a in (q, k, v))
    t0 = time.perf_counter()
    out, _ = oracle.attn_fwd(q, k, v, threads=threads, allow_underflow=True)
    if backward:
        oracle.attn_bwd(q, k, v, out, threads=threads, allow_underflow=True)
    dt = time.perf_counter() - t0
    fwd, bwd = attn_flops(len(heads), 1, tokens)
    return (fwd + (bwd if backward else 0)) / dt / 1e12, dt


def other_configs(swa, inputs, torch, stream, device, pk, info, cpu):
    """The workloads besides the step's: each timed on the GPU with its
    roofline fraction, and (rank 0, one GPU) the oracle on a bounded sample."""
    peak = pk["bf16_tflops"]
    threads = host_threads()
    res = {}

    def dev16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)

    # 4x16x4096 causal forward (out + lse)
    wl = inputs.WORKLOADS["attn_fwd_b4h16n4096"]
    qb, kb, vb, _ = inputs.attn_bf16(**wl)
    q, k, v = dev16(qb), dev16(kb), dev16(vb)
    ws = torch.empty(max(swa.attn_fwd_workspace_size(wl["B"], wl["H"], wl["N"], D, swa.SWA_BF16),
                         16), dtype=torch.uint8, device=device)
    o, l = torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=device)
    ms = timed_call(lambda: swa.attn_fwd(q, k, v, out=o, lse=l, workspace=ws), stream, device)
    fl, _ = attn_flops(wl["B"], wl["H"], wl["N"])
    entry = {"workload": "causal attention forward B=4 H=16 N=4096 D=64 bf16 (out + lse)",
             "ms": ms, "tflops": fl / (ms * 1e-3) / 1e12,
             "frac": fl / (ms * 1e-3) / 1e12 / peak, "bound": "tensor",
             "timing": "median of 5 calls after 2 warm-up calls (V scan + kernel), CUDA events; "
                       "inputs 101 MB (< L2, not flushed)"}
    if cpu:
        rate, dt = oracle_attn_rate(qb, kb, vb, [0, 1], wl["N"], False, threads)
        entry["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": threads,
                                 "kind": "oracle", "sample": f"2 of 64 heads, forward; {dt:.1f} s"}
    res["fwd_b4h16n4096"] = entry
    del q, k, v, o, l, ws

    # 1x8x65536 forward + gradient, without and with 0.01% +inf in V
    wl = inputs.WORKLOADS["attn_fwdbwd_b1h8n65536"]
    for with_inf in (False, True):
        qb, kb, vb, _ = inputs.attn_bf16(**wl, n_inf=inputs.LONG_CONTEXT_N_INF if with_inf else 0)
        q, k, v = dev16(qb), dev16(kb), dev16(vb)
        ws = torch.empty(swa.attn_grad_workspace_size(wl["B"], wl["H"], wl["N"], D, swa.SWA_BF16),
                         dtype=torch.uint8, device=device)
        t = timed_grad(swa, q, k, v, True, stream, device, ws)
        fwd, bwd = attn_flops(wl["B"], wl["H"], wl["N"])
        entry = {"workload": "causal attention forward + gradient B=1 H=8 N=65536 D=64 bf16, "
                             "Q, K ~ N(0, 0.5^2)" + (", 3355 V entries +inf" if with_inf else ""),
                 "call_ms": t["call_ms"], "fwd_ms": t["fwd_ms"], "bwd_ms": t["bwd_ms"],
                 "tflops": (fwd + bwd) / (t["call_ms"] * 1e-3) / 1e12,
                 "fwd_tflops": fwd / (t["fwd_ms"] * 1e-3) / 1e12,
                 "bwd_tflops": bwd / (t["bwd_ms"] * 1e-3) / 1e12,
                 "fwd_frac": fwd / (t["fwd_ms"] * 1e-3) / 1e12 / peak,
                 "bwd_frac": bwd / (t["bwd_ms"] * 1e-3) / 1e12 / peak, "bound": "tensor",
                 "timing": "median of 3 gradient calls after 2 warm-up calls, CUDA events"}
        if cpu:
            rate, dt = oracle_attn_rate(qb, kb, vb, [0], 8192, True, threads)
            entry["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": threads,
                                     "kind": "oracle",
                                     "sample": f"head 0, first 8192 tokens, forward + gradient; "
                                               f"{dt:.1f} s"}
        res["fwdbwd_b1h8n65536" + ("_inf" if with_inf else "")] = entry
        del q, k, v, ws

    # float32, one head of 256 tokens (the demo's size): latency of the
    # forward + gradient call on CUDA cores
    q64, k64, v64 = inputs.single_head_f64(256)
    q, k, v = (torch.from_numpy(a.astype(np.float32)).to(device) for a in (q64, k64, v64))
    ws = torch.empty(swa.attn_grad_workspace_size(1, 1, 256, D, swa.SWA_F32), dtype=torch.uint8,
                     device=device)
    o, l = torch.empty_like(q), torch.empty((1, 1, 256), dtype=torch.float32, device=device)
    g = [torch.empty_like(q) for _ in range(3)]
    ms = timed_call(lambda: swa.attn_grad(q, k, v, out=o, lse=l, dq=g[0], dk=g[1], dv=g[2],
                                          workspace=ws), stream, device, reps=22)
    fwd, bwd = attn_flops(1, 1, 256)
    entry = {"workload": "causal attention forward + gradient B=1 H=1 N=256 D=64 float32 "
                         "(CUDA cores)",
             "us": ms * 1e3, "tflops": (fwd + bwd) / (ms * 1e-3) / 1e12, "bound": "latency",
             "timing": "median of 20 calls after 2 warm-up calls, CUDA events"}
    if cpu:
        import oracle
        ts = []
        for _ in range(5):
            t0 = time.perf_counter()
            out, _ = oracle.attn_fwd(q64, k64, v64, threads=threads)
            oracle.attn_bwd(q64, k64, v64, out, threads=threads)
            ts.append(time.perf_counter() - t0)
        entry["cpu_baseline"] = {"value": statistics.median(ts) * 1e6, "unit": "us",
                                 "cores": threads, "kind": "oracle",
                                 "sample": "the whole call, median of 5"}
    res["f32_b1h1n256"] = entry

    # the regrid generalised: 3-D points, and the gradient (2-D, loss 1/2 sum out^2)
    t3, s3, v3 = (torch.from_numpy(a).to(device) for a in inputs.nw_grid_nd(NW_M, NW_S, 3))
    ms = timed_call(lambda: swa.nw_regrid_nd(t3, s3, v3, h=H_BW), stream, device)
    rate = NW_M * NW_S / (ms * 1e-3) / 1e9
    entry = {"workload": f"Nadaraya-Watson regrid, 3-D points, {NW_M}x{NW_S} fp32 h={H_BW}",
             "ms": ms, "gpairs_per_s": rate, "points_per_s": NW_M / (ms * 1e-3),
             "frac": rate / MUFU_GPAIRS, "bound": "alu (MUFU: one ex2 per pair)",
             "timing": "median of 5 calls after 2 warm-up calls (both kernels)"}
    if cpu:
        import oracle
        tn, sn, vn = inputs.nw_grid_nd(NW_M, NW_S, 3)
        t0 = time.perf_counter()
        oracle.nw_regrid_nd(tn[:512], sn, vn, h=H_BW, threads=threads)
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": 512 * NW_S / dt / 1e9, "unit": "Gpair/s",
                                 "cores": threads, "kind": "oracle",
                                 "sample": f"512 of {NW_M} targets; {dt:.1f} s"}
    res["nw3d_16384"] = entry
    t2, s2, v2 = (torch.from_numpy(a).to(device) for a in inputs.nw_grid(NW_M, NW_S, NW_SEED))
    g2 = swa.nw_regrid(t2, s2, v2, h=H_BW)
    ms = timed_call(lambda: swa.nw_regrid_bwd(t2, s2, v2, g2, h=H_BW), stream, device)
    rate = 2 * NW_M * NW_S / (ms * 1e-3) / 1e9
    entry = {"workload": f"Nadaraya-Watson regrid gradient (targets, sources, values), 2-D, "
                         f"{NW_M}x{NW_S} fp32, gout = out",
             "ms": ms, "gpairs_per_s": rate, "frac": rate / MUFU_GPAIRS,
             "bound": "alu (MUFU: one ex2 per pair in each of the two passes)",
             "timing": "median of 5 calls after 2 warm-up calls (all four kernels)"}
    if cpu:
        import oracle
        tn, sn, vn = inputs.nw_grid(NW_M, NW_S, NW_SEED)
        sub_t, sub_s = tn[:1024], sn[:1024]
        t0 = time.perf_counter()
        oracle.nw_regrid_bwd(sub_t, sub_s, vn[:1024], np.ones(1024), h=H_BW, threads=threads)
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": 2 * 1024 * 1024 / dt / 1e9, "unit": "Gpair/s",
                                 "cores": threads, "kind": "oracle",
                                 "sample": f"1024 targets x 1024 sources; {dt:.2f} s"}
    res["nw_grad_16384"] = entry
    del t3, s3, v3, t2, s2, v2, g2

    # the QKV projection at the step's shape (x [2*16384, 1024], w [3072, 1024])
    Cq = H * D
    xb, wb = inputs.qkv_inputs(B, N, Cq, H, seed=6)
    x, w = dev16(xb), dev16(wb)
    qo, ko, vo = (torch.empty((B, H, N, D), dtype=torch.bfloat16, device=device) for _ in range(3))
    ms = timed_call(lambda: swa.qkv_proj(x, w, H, q=qo, k=ko, v=vo), stream, device)
    fl = 2.0 * B * N * Cq * 3 * Cq
    entry = {"workload": f"QKV projection B={B} N={N} C={Cq} H={H} bf16 (x w^T into [B,H,N,64])",
             "ms": ms, "tflops": fl / (ms * 1e-3) / 1e12, "frac": fl / (ms * 1e-3) / 1e12 / peak,
             "bound": "tensor", "timing": "median of 5 calls after 2 warm-up calls"}
    if cpu:
        import oracle
        xs = inputs.bf16_to_f64(xb[:, :512])
        t0 = time.perf_counter()
        oracle.qkv_proj(xs, inputs.bf16_to_f64(wb), H)
        dt = time.perf_counter() - t0
        entry["cpu_baseline"] = {"value": 2.0 * B * 512 * Cq * 3 * Cq / dt / 1e12,
                                 "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                 "sample": f"512 of {N} tokens per sequence; {dt:.2f} s"}
    res["qkv_proj_b2n16384c1024"] = entry
    del x, w, qo, ko, vo

    # ring forward: the compute of each rank of an 8-rank ring over one
    # 131072-token sequence, rank after rank on this GPU (each with the K/V
    # chunks its ring steps receive); the K/V transport is not in it
    from causal_attention_swa_b200 import ring
    wl = inputs.WORKLOADS["attn_ring_b1h8n131072"]
    W = 8
    qb, kb, vb, _ = inputs.attn_bf16(**wl)
    q, k, v = dev16(qb), dev16(kb), dev16(vb)
    chunks = [[ring.zigzag_split(t, r, W) for t in (q, k, v)] for r in range(W)]
    kvs = [torch.stack((kc[0], kc[1], vc[0], vc[1])) for _, kc, vc in chunks]
    del q, k, v
    per_rank = []
    for r in range(W):
        state = ring.RingForwardState(chunks[r][0], r, W)

        def run(state=state, r=r):
            for s_ in range(W):
                state.step(s_, kvs[(r - s_) % W])
        per_rank.append(timed_call(run, stream, device, reps=3, warm=1))
    fl, _ = attn_flops(wl["B"], wl["H"], wl["N"])
    ms = max(per_rank)
    entry = {"workload": "ring causal attention forward, 8 ranks, B=1 H=8 N=131072 D=64 bf16, "
                         "Q, K ~ N(0, 0.5^2): the compute of each rank (16 zigzag chunks of "
                         "8192 tokens; 17 chunk calls and merges per rank), ranks timed one "
                         "after another on this GPU; K/V transport not included",
             "ms_per_rank_max": ms, "ms_per_rank_min": min(per_rank),
             "tflops_per_rank": fl / W / (ms * 1e-3) / 1e12,
             "frac": fl / W / (ms * 1e-3) / 1e12 / peak, "bound": "tensor",
             "timing": "median of 2 runs of each rank's steps after 1 warm-up, CUDA events"}
    if cpu:
        rate, dt = oracle_attn_rate(qb, kb, vb, [0], 8192, False, threads)
        entry["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": threads,
                                 "kind": "oracle",
                                 "sample": f"head 0, first 8192 tokens, forward; {dt:.1f} s"}
    res["ring_fwd_b1h8n131072_w8"] = entry
    del chunks, kvs
    if swa.get_device_error(device) != swa.SWA_OK:
        raise RuntimeError("device error word set during the other workloads")
    return res

def run_ours(args, info):
    import torch
    from causal_attention_swa_b200 import dist as sdist
    from causal_attention_swa_b200 import inputs, swa

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    device = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(device)
    sdist.init("nccl", info)
    swa.load_library()

    # this rank's block of one global problem: sequences [rank*B, rank*B + B)
    # of a batch of B*world (every sequence drawn from its own seed) and
    # target block `rank` against the shared source set
    qb, kb, vb = inputs.attn_bf16_batch(B, H, N, seed=SEED,
                                        first=sdist.sequence_block(B, info.rank))
    _, ns, ny = inputs.nw_grid(NW_M, NW_S, NW_SEED)
    nt = inputs.nw_targets_block(NW_M, info.rank, NW_SEED)

    def bf16_host(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)

    host_in = {"q": bf16_host(qb).pin_memory(), "k": bf16_host(kb).pin_memory(),
               "v": bf16_host(vb).pin_memory(), "nt": torch.from_numpy(nt).pin_memory(),
               "ns": torch.from_numpy(ns).pin_memory(), "ny": torch.from_numpy(ny).pin_memory()}
    dev_in = {name: t.to(device) for name, t in host_in.items()}
    q, k, v = dev_in["q"], dev_in["k"], dev_in["v"]
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    nw_out = torch.empty((NW_M,), dtype=torch.float32, device=device)
    ws_g = torch.empty(swa.attn_grad_workspace_size(B, H, N, D, swa.SWA_BF16),
                       dtype=torch.uint8, device=device)
    ws_n = torch.empty(swa.nw_workspace_size(NW_M, NW_S), dtype=torch.uint8, device=device)
    launches = [0]

    main_out = {"out": out, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "nw": nw_out}

    def step(src, dst=None):
        d = main_out if dst is None else dst
        swa.attn_grad(src["q"], src["k"], src["v"], causal=True, out=d["out"], lse=d["lse"],
                      dq=d["dq"], dk=d["dk"], dv=d["dv"], workspace=ws_g)
        launches[0] += swa.last_launch_count()
        swa.nw_regrid(src["nt"], src["ns"], src["ny"], h=H_BW, out=d["nw"], workspace=ws_n)
        launches[0] += swa.last_launch_count()

    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        step(dev_in)
    torch.cuda.synchronize(device)
    if swa.get_device_error(device) != swa.SWA_OK:
        raise RuntimeError("device error word set during warm-up")

    # ---- device-timed region: exactly K steps; each step also brackets one
    # main kernel (rotating fwd, bwd, regrid) with its own pair of events.
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in kev:  # create the events (torch creates them on first record); the
        a.record(stream)  # library's records around the kernel then replace these
        b.record(stream)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches[0] = 0
    with ClockSampler(device.index) as clocks:
        sdist.barrier(device)
        torch.cuda.synchronize(device)
        start.record(stream)
        for i in range(args.steps):
            swa.profile_kernel(1 + i % 3, *kev[i])
            step(dev_in)
        stop.record(stream)
        torch.cuda.synchronize(device)
        swa.profile_kernel(swa.SWA_KERNEL_NONE)
        sdist.barrier(device)
    timed_launches = launches[0]
    elapsed_ms = sdist.max_over_ranks(start.elapsed_time(stop), device)
    if swa.get_device_error(device) != swa.SWA_OK:
        raise RuntimeError("device error word set during the timed region")
    per_kernel = {kid: [] for kid in KERNELS}
    for i, (a, b) in enumerate(kev):
        per_kernel[1 + i % 3].append(a.elapsed_time(b))
    kernel_ms = {kid: (sum(v) / len(v) if v else None) for kid, v in per_kernel.items()}

    fwd_fl, bwd_fl = attn_flops()
    ms_per_step = elapsed_ms / args.steps
    value = (fwd_fl + bwd_fl) * info.world / (elapsed_ms / args.steps * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs in from pinned host memory and its results back out.
    # The copies run on streams of their own with the device side
    # double-buffered, so step s+1's inputs go in and step s-1's results come
    # out while step s computes (the link is full duplex); the bytes each
    # step moves are the same as with no overlap.
    host_out = {"out": torch.empty_like(out, device="cpu").pin_memory(),
                "lse": torch.empty_like(lse, device="cpu").pin_memory(),
                "dq": torch.empty_like(dq, device="cpu").pin_memory(),
                "dk": torch.empty_like(dk, device="cpu").pin_memory(),
                "dv": torch.empty_like(dv, device="cpu").pin_memory(),
                "nw": torch.empty_like(nw_out, device="cpu").pin_memory()}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    bufs = [({name: torch.empty_like(t) for name, t in dev_in.items()},
             {name: torch.empty_like(t) for name, t in main_out.items()}) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    for e in comp_done + out_done:
        e.record(stream)
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sdist.barrier(device)
    torch.cuda.synchronize(device)
    e_start.record(s_in)
    for i in range(args.steps):
        b = i % 2
        ins, outs = bufs[b]
        s_in.wait_event(comp_done[b])  # step i-2, the last reader of these inputs, is done
        with torch.cuda.stream(s_in):
            for name, t in host_in.items():
                ins[name].copy_(t, non_blocking=True)
        in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        stream.wait_event(out_done[b])  # step i-2's results have left this buffer
        step(ins, outs)
        comp_done[b].record(stream)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            for name, t in outs.items():
                host_out[name].copy_(t, non_blocking=True)
        out_done[b].record(s_out)
    e_stop.record(s_out)
    torch.cuda.synchronize(device)
    sdist.barrier(device)
    e2e_ms = sdist.max_over_ranks(e_start.elapsed_time(e_stop), device) / args.steps
    e2e_value = (fwd_fl + bwd_fl) * info.world / (e2e_ms * 1e-3) / 1e12

    # ---- the first widening row: non-causal attention (every pair, the same
    # kernels without tile skipping), timed per kernel group inside the
    # gradient call after the step's measurements
    nc = timed_grad(swa, q, k, v, False, stream, device, ws_g)
    nc_fl = 4 * D * B * H * N * N
    noncausal = {"workload": f"non-causal attention fwd+bwd B={B} H={H} N={N} D={D} bf16",
                 "fwd_ms": nc["fwd_ms"], "bwd_ms": nc["bwd_ms"],
                 "fwd_tflops": nc_fl / (nc["fwd_ms"] * 1e-3) / 1e12,
                 "bwd_tflops": 2.5 * nc_fl / (nc["bwd_ms"] * 1e-3) / 1e12,
                 "timing": "median of 3 gradient calls after 2 warm-up calls; CUDA events "
                           "around the forward and the backward kernels"}

    pk = peaks()
    configs = other_configs(swa, inputs, torch, stream, device, pk, info,
                            cpu=info.is_root and info.world == 1 and not args.no_cpu_baseline)
    dom = 2  # the backward's main kernel dominates the step
    dom_ms = kernel_ms[dom]
    achieved = bwd_fl / (dom_ms * 1e-3) / 1e12 if dom_ms else None
    roofline = {
        "kernel": KERNELS[dom][0], "bound": "tensor", "achieved": achieved,
        "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
        "frac": (achieved / pk["bf16_tflops"]) if achieved else None,
        "traffic": recorded_traffic(dom),
        "peak_source": f"{pk['source']} bf16 dense (burst)",
        "flops_per_launch": bwd_fl, "ms_per_launch": dom_ms,
        "launch": "attn_bwd_dkdv_kernel + attn_bwd_dq_kernel, f16- and bf16-operand "
                  "instances (one event pair around the four launches of the gradient call)",
    }
    if pk.get("bf16_tflops_sustained") and achieved:
        roofline["frac_of_sustained"] = achieved / pk["bf16_tflops_sustained"]
    # the other main kernels against their own bounds: the forward against the
    # bf16 tensor peak, the regrid against MUFU (148 SMs x 16 ex2/clk x max clock)
    mufu_peak = MUFU_GPAIRS
    n_tiles = (N + 127) // 128
    fwd_ex2 = B * H * (n_tiles * (n_tiles + 1) // 2) * 128 * 128
    nw_rate = NW_M * NW_S / (kernel_ms[3] * 1e-3) / 1e9 if kernel_ms[3] else None
    fwd_rate = fwd_fl / (kernel_ms[1] * 1e-3) / 1e12 if kernel_ms[1] else None
    rooflines = {
        "attn_fwd": {"bound": "tensor", "achieved": fwd_rate, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": fwd_rate / pk["bf16_tflops"] if fwd_rate else None,
                     "traffic": recorded_traffic(1),
                     # the forward's actual limit: one MUFU ex2 per element of every causal
                     # 128 x 128 tile it visits, against 148 SMs x 16 ex2/clk x max clock
                     "mufu_frac": (fwd_ex2 / (kernel_ms[1] * 1e-3) / (mufu_peak * 1e9)
                                   if kernel_ms[1] else None)},
        "nw_regrid": {"bound": "alu", "achieved": nw_rate, "peak": mufu_peak, "unit": "Gpair/s",
                      "frac": nw_rate / mufu_peak if nw_rate else None,
                      "traffic": recorded_traffic(3),
                      "peak_source": "148 SMs x 16 MUFU ex2/clk x 1965 MHz (one ex2 per pair)",
                      "timing": "the whole call: pair-grid kernel and final sum"},
    }
    breakdown = {
        "attn_fwd_ms": kernel_ms[1], "attn_bwd_ms": kernel_ms[2], "nw_ms": kernel_ms[3],
        "attn_fwd_tflops": fwd_fl / (kernel_ms[1] * 1e-3) / 1e12 if kernel_ms[1] else None,
        "attn_bwd_tflops": achieved,
        "nw_gpairs_per_s": NW_M * NW_S / (kernel_ms[3] * 1e-3) / 1e9 if kernel_ms[3] else None,
        "nw_points_per_s": NW_M / (kernel_ms[3] * 1e-3) if kernel_ms[3] else None,
    }

    cpu = None
    if info.is_root and info.world == 1 and not args.no_cpu_baseline:
        threads = host_threads()
        dt, fl = oracle_sample(N, NW_M // 32, threads=threads)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
               "kind": "oracle",
               "sample": f"1/32 of one step: head 0 of {B * H} ({N} tokens, forward + "
                         f"backward) and {NW_M // 32} of {NW_M} regrid targets; "
                         f"{dt:.1f} s wall"}

    if info.is_root:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": info.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"causal attention fwd+bwd B={B} H={H} N={N} D={D} bf16 "
                                   f"(dout = out) + Nadaraya-Watson regrid {NW_M}x{NW_S} "
                                   f"fp32 h={H_BW}",
                       "global_batch": B * info.world, "seq_len": N,
                       "parallelism": f"heads split over {info.world} GPU(s): rank r takes "
                                      f"sequences [{B}r, {B}r+{B}) of a {B * info.world}-"
                                      f"sequence batch (no data-path collective)",
                       "l2": "inputs larger than L2 (Q, K, V = 201 MB per rank)"},
            "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": timed_launches, "clocks": clocks.summary(),
            "breakdown": breakdown, "rooflines": rooflines, "noncausal": noncausal,
            "configs": configs,
        }
        print(json.dumps(line), flush=True)
    sdist.shutdown()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from causal_attention_swa_b200 import dist as sdist
    info = sdist.rank_info()
    if info.world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={info.world}")
    if args.impl == "reference":
        return run_reference(args, info)
    return run_ours(args, info)


if __name__ == "__main__":
    sys.exit(main())
