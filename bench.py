#!/usr/bin/env python
"""Benchmark of the fused softmax-weighted average on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * causal attention forward (bf16, B=2 H=16 N=16384 D=64, scale 1/8):
    out and lse;
  * its backward for loss = 1/2 sum out^2 (dout = out): dq, dk, dv;
  * the Nadaraya-Watson regrid (fp32, 16384 targets x 16384 sources in
    [0,10]^2, h = 0.5).
The metric is attention TFLOP/s with FLOPs counted causally (N(N+1)/2 pairs
per head; forward 4*D per pair, backward 2.5x forward), over the whole
step's device time.  Inputs (201 MB of Q, K, V) exceed the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1: launched by torchrun, one process per GPU; each rank runs its own
seeded replica of the batch (weak scaling, no collective in the data path);
the elapsed time is the max over ranks.  --impl reference times the float64
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

def run_ours(args, info):
    import torch
    from causal_attention_swa_b200 import dist as sdist
    from causal_attention_swa_b200 import inputs, swa

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    device = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(device)
    sdist.init("nccl", info)
    swa.load_library()

    seed = sdist.replica_seed(SEED, info.rank)
    qb, kb, vb, _ = inputs.attn_bf16(B, H, N, seed=seed)
    nt, ns, ny = inputs.nw_grid(NW_M, NW_S, sdist.replica_seed(NW_SEED, info.rank))

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
    ws_f = torch.empty(max(swa.attn_fwd_workspace_size(B, H, N, D, swa.SWA_BF16), 16),
                       dtype=torch.uint8, device=device)
    ws_b = torch.empty(swa.attn_bwd_workspace_size(B, H, N, D, swa.SWA_BF16),
                       dtype=torch.uint8, device=device)
    ws_n = torch.empty(swa.nw_workspace_size(NW_M, NW_S), dtype=torch.uint8, device=device)
    launches = [0]

    main_out = {"out": out, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "nw": nw_out}

    def step(src, dst=None):
        d = main_out if dst is None else dst
        swa.attn_fwd(src["q"], src["k"], src["v"], causal=True, out=d["out"], lse=d["lse"],
                     workspace=ws_f)
        launches[0] += swa.last_launch_count()
        swa.attn_bwd(src["q"], src["k"], src["v"], d["out"], d["out"], d["lse"], causal=True,
                     dq=d["dq"], dk=d["dk"], dv=d["dv"], workspace=ws_b)
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
    # kernels without tile skipping), timed per API call after the step's
    # measurements (its calls include the small scan and prep kernels)
    nc_fwd, nc_bwd = [], []
    for rep in range(5):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        swa.attn_fwd(q, k, v, causal=False, out=out, lse=lse, workspace=ws_f)
        e1.record(stream)
        swa.attn_bwd(q, k, v, out, out, lse, causal=False, dq=dq, dk=dk, dv=dv, workspace=ws_b)
        e2.record(stream)
        torch.cuda.synchronize(device)
        if rep >= 2:  # two warm-up calls
            nc_fwd.append(e0.elapsed_time(e1))
            nc_bwd.append(e1.elapsed_time(e2))
    if swa.get_device_error(device) != swa.SWA_OK:
        raise RuntimeError("device error word set during the non-causal calls")
    nc_fl = 4 * D * B * H * N * N
    nc_f_ms, nc_b_ms = sorted(nc_fwd)[1], sorted(nc_bwd)[1]
    noncausal = {"workload": f"non-causal attention fwd+bwd B={B} H={H} N={N} D={D} bf16",
                 "fwd_ms": nc_f_ms, "bwd_ms": nc_b_ms,
                 "fwd_tflops": nc_fl / (nc_f_ms * 1e-3) / 1e12,
                 "bwd_tflops": 2.5 * nc_fl / (nc_b_ms * 1e-3) / 1e12,
                 "timing": "median of 3 API calls after 2 warm-up calls, CUDA events"}

    pk = peaks()
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
        "launch": "attn_bwd_dkdv_kernel + attn_bwd_dq_kernel (one event pair around both)",
    }
    if pk.get("bf16_tflops_sustained") and achieved:
        roofline["frac_of_sustained"] = achieved / pk["bf16_tflops_sustained"]
    # the other main kernels against their own bounds: the forward against the
    # bf16 tensor peak, the regrid against MUFU (148 SMs x 16 ex2/clk x max clock)
    mufu_peak = 148 * 16 * SM_MAX_MHZ * 1e6 / 1e9  # Gpair/s
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
                      "peak_source": "148 SMs x 16 MUFU ex2/clk x 1965 MHz (one ex2 per pair)"},
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
                       "parallelism": f"replicas x{info.world} (independent heads)",
                       "l2": "inputs larger than L2 (Q, K, V = 201 MB per rank)"},
            "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": timed_launches, "clocks": clocks.summary(),
            "breakdown": breakdown, "rooflines": rooflines, "noncausal": noncausal,
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
