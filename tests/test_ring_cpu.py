"""Host logic of the sequence-sharded (ring) forward on CPU: the zigzag
chunk plan covers every causal pair of the sequence exactly once with the
same work on every rank, the split and join of the token axis are inverse,
and over gloo ranks (2 and 3) the ring delivers, at step s, the K/V chunks
of rank (r - s) mod W to rank r (compute replaced by a recorder)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from causal_attention_swa_b200 import ring


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_plan_covers_each_causal_chunk_pair_once_and_balances_ranks(world):
    seen = {}
    work = []
    for r in range(world):
        units = 0.0
        for s, calls in enumerate(ring.plan(r, world)):
            src = (r - s) % world
            for qs, ks, mode in calls:
                qc = ring.zigzag_chunks(r, world)[qs]
                kc = ring.zigzag_chunks(src, world)[ks]
                assert (qc, kc) not in seen
                seen[(qc, kc)] = mode
                units += 0.5 if mode == "causal" else 1.0
        work.append(units)
    n = 2 * world
    # every chunk pair with key chunk <= query chunk, the diagonal causal
    assert set(seen) == {(q, k) for q in range(n) for k in range(q + 1)}
    assert all((m == "causal") == (q == k) for (q, k), m in seen.items())
    # the same work on every rank: (2W)^2 / 2 chunk-pair units in all (a
    # diagonal pair counts half), 2W per rank
    assert work == [2.0 * world] * world


def test_zigzag_split_join_roundtrip():
    x = torch.arange(2 * 3 * 24 * 4, dtype=torch.float32).reshape(2, 3, 24, 4)
    for world in (1, 2, 3, 4, 6, 12):
        parts = [ring.zigzag_split(x, r, world) for r in range(world)]
        for xa, xb in parts:
            assert xa.is_contiguous() and xb.is_contiguous()
            assert xa.shape == (2, 3, 24 // (2 * world), 4)
        assert torch.equal(ring.zigzag_join(parts, world), x)
    with pytest.raises(ValueError):
        ring.zigzag_split(x, 0, 5)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    # this rank's chunks hold (rank, slot, tensor) tags
    shape = (1, 2, 3, 64)
    t = [torch.full(shape, float(100 * rank + j)) for j in range(6)]
    seen = []

    def record(s, src, kv):
        seen.append((s, src, [float(kv[i].flatten()[0]) for i in range(4)]))

    ring.ring_attn_fwd(t[0], t[1], t[2], t[3], t[4], t[5], step_fn=record)
    q.put((rank, seen))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_delivers_each_ranks_kv_in_order_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        steps = results[r]
        assert [s for s, _, _ in steps] == list(range(world))
        for s, src, tags in steps:
            assert src == (r - s) % world
            # k chunks 0, 1 and v chunks 0, 1 of rank src (tags 2..5)
            assert tags == [100.0 * src + j for j in range(2, 6)]


def _bwd_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    shape = (1, 2, 3, 64)
    t = [torch.full(shape, float(100 * rank + j)) for j in range(6)]
    seen = []

    def add(s, src, kv, dkv):
        seen.append((s, src, float(kv[0].flatten()[0])))
        dkv += 1000.0 * src + rank + 1  # tagged by the sums' owner and this rank

    _, dkv = ring.ring_attn_bwd(t[0], t[1], t[2], t[3], t[4], t[5], None, None, None,
                                step_fn=add)
    q.put((rank, seen, [float(dkv[i].flatten()[0]) for i in range(4)]))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_backward_sums_visit_every_rank_and_return_home_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {r: (seen, sums) for r, seen, sums in (q.get(timeout=120) for _ in procs)}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        seen, sums = results[r]
        assert [(s, src) for s, src, _ in seen] == [(s, (r - s) % world) for s in range(world)]
        assert [k0 for _, _, k0 in seen] == [100.0 * ((r - s) % world) + 2 for s in range(world)]
        # rank r ends with its own chunks' sums: one term from every rank
        want = world * 1000.0 * r + world * (world + 1) / 2
        assert sums == [want] * 4
