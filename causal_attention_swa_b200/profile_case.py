"""A small, repeatable workload for profiler captures of one kernel.

    python -m causal_attention_swa_b200.profile_case grad --B 1 --H 8 --N 16384 --reps 3
    python -m causal_attention_swa_b200.profile_case regrid --M 16384 --S 16384 --reps 3

Runs the named call (through the public binding) `reps` times on cuda:0 on
seeded synthetic inputs and checks the device error word.  The sizes are
chosen on the command line so that a capture can stay on a case of a few
hundred MB (inputs still larger than the 126 MB L2):
  grad        swa_attn_grad, bf16, causal (the GRADIENT query)
  fwd         swa_attn_fwd, bf16, causal
  regrid      swa_nw_regrid (2-D points)
  regrid_bwd  swa_nw_regrid_bwd (2-D points)
  qkv         swa_qkv_proj (C = 64 H)
"""
from __future__ import annotations

import argparse
import sys

import numpy as np
import torch

from causal_attention_swa_b200 import inputs, swa


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description="one call, a few times, for a profiler")
    ap.add_argument("call", choices=("grad", "fwd", "regrid", "regrid_bwd", "qkv"))
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=8)
    ap.add_argument("--N", type=int, default=16384)
    ap.add_argument("--M", type=int, default=16384)
    ap.add_argument("--S", type=int, default=16384)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    def d16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    if a.call in ("grad", "fwd"):
        q, k, v = (d16(b) for b in inputs.attn_bf16_batch(a.B, a.H, a.N, seed=4))
        for _ in range(a.reps):
            if a.call == "grad":
                swa.attn_grad(q, k, v, causal=True)
            else:
                swa.attn_fwd(q, k, v, causal=True)
    elif a.call in ("regrid", "regrid_bwd"):
        t, s, y = (torch.from_numpy(x).to(dev) for x in inputs.nw_grid(a.M, a.S, 2))
        g = swa.nw_regrid(t, s, y)
        for _ in range(a.reps):
            if a.call == "regrid":
                swa.nw_regrid(t, s, y, out=g)
            else:
                swa.nw_regrid_bwd(t, s, y, g)
    else:
        xb, wb = inputs.qkv_inputs(a.B, a.N, 64 * a.H, a.H, seed=6)
        x, w = d16(xb), d16(wb)
        for _ in range(a.reps):
            swa.qkv_proj(x, w, a.H)
    torch.cuda.synchronize()
    st = swa.get_device_error()
    print(f"{a.call}: {a.reps} calls, device error word {swa._status_name(st)}")
    return 0 if st == swa.SWA_OK else 1


if __name__ == "__main__":
    sys.exit(main())
