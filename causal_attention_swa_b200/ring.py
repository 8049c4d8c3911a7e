"""Sequence-sharded causal attention over W ranks (ring): forward and backward.

For sequences too long for one GPU's share of a step, the N tokens of each
(b, h) are split into 2W chunks of C = N / (2W) tokens, and rank r holds
chunks r and 2W-1-r of Q, K and V ("zigzag": with causal attention a chunk
late in the sequence meets more keys, so pairing an early chunk with a late
one gives every rank the same work).  K and V travel around the ring: at
step s rank r holds the chunks of rank (r - s) mod W, sends them to rank
r + 1 and receives the next ones from rank r - 1 while it computes.

Each (query chunk, key chunk) pair is either
  * skipped      key chunk after the query chunk (every pair masked),
  * causal       the same chunk (the diagonal: swa_attn_fwd, causal),
  * full         key chunk before the query chunk (swa_attn_fwd, causal = 0),
and the partial results merge by their log-sum-exp (swa_attn_merge: the
view's weighted average over the union of disjoint key sets, computed
exactly from the sets' own averages and normalisers) into a float32
accumulator; the last partial of a query chunk also writes the bf16 result.

The backward (the GRADIENT query over the sharded sequence) walks the same
plan: each (query chunk, key chunk) pair adds its dq, dk, dv terms to
float32 sums (swa_attn_bwd_acc, with the merged forward's out and lse, so P
and delta are the whole row's); dq stays with its rank, while each key
chunk's dk, dv sums travel around the ring with its K and V and reach their
owner after the last step.  Float32 sums, not bf16 partials: sum_j dS_ij
k_j cancels across key chunks.

Every arithmetic step runs in libswa.so's kernels; this module only
allocates, orders the calls and moves K/V (and the dk, dv sums) with
torch.distributed point-to-point operations (NCCL on GPUs); K/V transfers
overlap the compute.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from causal_attention_swa_b200 import swa


def zigzag_chunks(rank: int, world: int) -> tuple[int, int]:
    """The two chunk indices (of 2 * world) that `rank` holds."""
    return rank, 2 * world - 1 - rank


def pair_mode(q_chunk: int, k_chunk: int) -> str:
    """'skip', 'causal' or 'full' for a query chunk against a key chunk."""
    if k_chunk > q_chunk:
        return "skip"
    return "causal" if k_chunk == q_chunk else "full"


def plan(rank: int, world: int) -> list[list[tuple[int, int, str]]]:
    """Per ring step s, the (query slot, key slot, mode) sub-calls of `rank`
    (slots 0, 1 = the first, second chunk held), skipped pairs left out."""
    steps = []
    for s in range(world):
        src = (rank - s) % world
        calls = []
        for qs, qc in enumerate(zigzag_chunks(rank, world)):
            for ks, kc in enumerate(zigzag_chunks(src, world)):
                mode = pair_mode(qc, kc)
                if mode != "skip":
                    calls.append((qs, ks, mode))
        steps.append(calls)
    return steps


def zigzag_split(x: torch.Tensor, rank: int, world: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Contiguous copies of the two chunks (dim 2, the token axis) of a
    [B, H, N, D] tensor that `rank` holds; N must be a multiple of 2*world."""
    n = x.shape[2]
    if n % (2 * world) != 0:
        raise ValueError(f"N = {n} is not a multiple of 2 * world = {2 * world}")
    c = n // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return (x[:, :, a * c:(a + 1) * c].contiguous(), x[:, :, b * c:(b + 1) * c].contiguous())


def zigzag_join(parts: list[tuple[torch.Tensor, torch.Tensor]], world: int) -> torch.Tensor:
    """Inverse of zigzag_split over all ranks: parts[r] = rank r's two chunks."""
    chunks = [None] * (2 * world)
    for r, (xa, xb) in enumerate(parts):
        a, b = zigzag_chunks(r, world)
        chunks[a], chunks[b] = xa, xb
    return torch.cat(chunks, dim=2)


@dataclass
class RingForwardState:
    """One rank's accumulators: float32 out and lse per held query chunk."""
    q: tuple[torch.Tensor, torch.Tensor]
    rank: int
    world: int

    def __post_init__(self):
        qa = self.q[0]
        B, H, C, D = qa.shape
        self.acc = [torch.empty((B, H, C, D), dtype=torch.float32, device=qa.device)
                    for _ in range(2)]
        self.lse = [torch.empty((B, H, C), dtype=torch.float32, device=qa.device)
                    for _ in range(2)]
        self.out = [torch.empty_like(qa) for _ in range(2)]
        self.plan = plan(self.rank, self.world)
        # the last sub-call of each query slot writes that slot's result
        self.last = {}
        for s, calls in enumerate(self.plan):
            for i, (qs, _, _) in enumerate(calls):
                self.last[qs] = (s, i)
        self.started = [False, False]

    def step(self, s: int, kv: torch.Tensor) -> None:
        """Ring step s with kv = stack(k chunk 0, k chunk 1, v chunk 0, v chunk 1)
        of rank (rank - s) mod world."""
        for i, (qs, ks, mode) in enumerate(self.plan[s]):
            out_p, lse_p = swa.attn_fwd(self.q[qs], kv[ks], kv[2 + ks], causal=(mode == "causal"))
            final = self.out[qs] if self.last[qs] == (s, i) else None
            swa.attn_merge(out_p, lse_p, self.acc[qs], self.lse[qs], first=not self.started[qs],
                           out_final=final)
            self.started[qs] = True

    def result(self):
        """((out chunk 0, out chunk 1), (lse chunk 0, lse chunk 1)); lse natural log."""
        return (self.out[0], self.out[1]), (self.lse[0], self.lse[1])


def ring_attn_fwd(qa, qb, ka, kb, va, vb, group=None, step_fn=None):
    """Causal attention forward of this rank's two zigzag chunks (each
    [B, H, C, 64], bf16 or fp32, CUDA) against the whole sequence held by the
    ranks of `group` (the default group; one rank without torch.distributed).

    Returns ((out_a, out_b), (lse_a, lse_b)).  `step_fn(s, src, kv)`, if
    given, replaces the compute (the ring's transport alone, for tests)."""
    if dist.is_available() and dist.is_initialized():
        rank, world = dist.get_rank(group), dist.get_world_size(group)
    else:
        rank, world = 0, 1
    kv = torch.stack((ka, kb, va, vb))
    nxt = torch.empty_like(kv) if world > 1 else None
    state = None if step_fn is not None else RingForwardState((qa, qb), rank, world)
    for s in range(world):
        src = (rank - s) % world
        reqs = []
        if s + 1 < world:  # pass this step's K/V on while computing with them
            ops = [dist.P2POp(dist.isend, kv, (rank + 1) % world, group),
                   dist.P2POp(dist.irecv, nxt, (rank - 1) % world, group)]
            reqs = dist.batch_isend_irecv(ops)
        if step_fn is not None:
            step_fn(s, src, kv)
        else:
            state.step(s, kv)
        for r in reqs:
            r.wait()
        if s + 1 < world:
            kv, nxt = nxt, kv
    return None if state is None else state.result()


@dataclass
class RingBackwardState:
    """One rank's backward: float32 dq sums per held query chunk, and the
    plan of (query slot, key slot, mode) sub-calls per ring step."""
    q: tuple[torch.Tensor, torch.Tensor]
    out: tuple[torch.Tensor, torch.Tensor]
    dout: tuple[torch.Tensor, torch.Tensor]
    lse: tuple[torch.Tensor, torch.Tensor]
    rank: int
    world: int

    def __post_init__(self):
        self.dq_acc = [torch.zeros(t.shape, dtype=torch.float32, device=t.device) for t in self.q]
        self.plan = plan(self.rank, self.world)

    def step(self, s: int, kv: torch.Tensor, dkv: torch.Tensor) -> None:
        """Ring step s: kv = stack(k0, k1, v0, v1) of rank (rank - s) mod world,
        dkv = the float32 sums (dk0, dk1, dv0, dv1) travelling with them."""
        for qs, ks, mode in self.plan[s]:
            swa.attn_bwd_acc(self.q[qs], kv[ks], kv[2 + ks], self.out[qs], self.dout[qs],
                             self.lse[qs], self.dq_acc[qs], dkv[ks], dkv[2 + ks],
                             causal=(mode == "causal"))

    def dq(self):
        return tuple(swa.f32_to_bf16(a) for a in self.dq_acc)


def ring_attn_bwd(qa, qb, ka, kb, va, vb, outs, douts, lses, group=None, step_fn=None):
    """Backward of ring_attn_fwd for upstream gradients douts = (dout_a, dout_b)
    (douts = outs for loss = 1/2 sum out^2), given the forward's merged
    outs and lses of this rank's two chunks (bf16 inputs).

    Returns ((dq_a, dq_b), (dk_a, dk_b), (dv_a, dv_b)) in bf16.  `step_fn(s,
    src, kv, dkv)`, if given, replaces the compute (for transport tests)."""
    if dist.is_available() and dist.is_initialized():
        rank, world = dist.get_rank(group), dist.get_world_size(group)
    else:
        rank, world = 0, 1
    kv = torch.stack((ka, kb, va, vb))
    dkv = torch.zeros(kv.shape, dtype=torch.float32, device=kv.device)
    nxt = torch.empty_like(kv) if world > 1 else None
    nxt_d = torch.empty_like(dkv) if world > 1 else None
    state = None if step_fn is not None else RingBackwardState(
        (qa, qb), tuple(outs), tuple(douts), tuple(lses), rank, world)
    for s in range(world):
        src = (rank - s) % world
        reqs = []
        if s + 1 < world:  # K/V move on while this step computes with them
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, kv, (rank + 1) % world, group),
                                           dist.P2POp(dist.irecv, nxt, (rank - 1) % world, group)])
        if step_fn is not None:
            step_fn(s, src, kv, dkv)
        else:
            state.step(s, kv, dkv)
        for r in reqs:
            r.wait()
        if world > 1:
            # the updated sums follow their K/V; after the last step they reach
            # their owner (rank src = rank + 1 - world = rank + 1 mod world)
            for r in dist.batch_isend_irecv([
                    dist.P2POp(dist.isend, dkv, (rank + 1) % world, group),
                    dist.P2POp(dist.irecv, nxt_d, (rank - 1) % world, group)]):
                r.wait()
            dkv, nxt_d = nxt_d, dkv
        if s + 1 < world:
            kv, nxt = nxt, kv
    if state is None:
        return None, dkv
    dk = (swa.f32_to_bf16(dkv[0]), swa.f32_to_bf16(dkv[1]))
    dv = (swa.f32_to_bf16(dkv[2]), swa.f32_to_bf16(dkv[3]))
    return state.dq(), dk, dv
