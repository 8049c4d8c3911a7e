"""Multi-rank host logic on CPU: two gloo ranks exercise the split of one
batch across ranks (each draws its own sequences; together they are the
global batch), the barrier and the max-over-ranks reduction that bench.py
uses to time a multi-GPU run (no GPU, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    from causal_attention_swa_b200 import dist as sdist
    from causal_attention_swa_b200 import inputs
    info = sdist.rank_info()
    sdist.init("gloo", info, timeout_s=60)
    sdist.barrier()
    elapsed = 10.0 + 5.0 * rank          # rank 1 is the slow one
    mx = sdist.max_over_ranks(elapsed)
    tot = sdist.sum_over_ranks(1.0)
    # this rank's block of the global batch (2 sequences per rank, 3 heads)
    first = sdist.sequence_block(2, rank)
    qb, kb, vb = inputs.attn_bf16_batch(2, 3, 40, seed=4, first=first)
    tb = inputs.nw_targets_block(64, rank)
    q.put((rank, info.world, mx, tot, first, qb, kb, vb, tb))
    sdist.shutdown()


def test_two_gloo_ranks_split_one_batch_and_time_as_max():
    import numpy as np
    from causal_attention_swa_b200 import inputs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted((q.get(timeout=120) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in results] == [0, 1]
    for rank, world, mx, tot, *_ in results:
        assert world == 2 and mx == 15.0 and tot == 2.0
    # the two blocks are sequences 0-1 and 2-3 of one 4-sequence batch
    assert results[0][4] == 0 and results[1][4] == 2
    whole = inputs.attn_bf16_batch(4, 3, 40, seed=4)
    for i in range(3):
        assert np.array_equal(np.concatenate([results[0][5 + i], results[1][5 + i]]), whole[i])
    # rank 0's block is the one-GPU workload itself; the target blocks differ
    assert np.array_equal(results[0][5], inputs.attn_bf16_batch(2, 3, 40, seed=4)[0])
    assert np.array_equal(results[0][8], inputs.nw_grid(64, 64)[0])
    assert not np.array_equal(results[0][8], results[1][8])


def test_shard_partitions_units_in_order():
    from causal_attention_swa_b200 import dist as sdist
    for units in (1, 7, 32, 33):
        for world in (1, 2, 3, 8):
            blocks = [sdist.shard(units, world, r) for r in range(world)]
            pos = 0
            for first, count in blocks:
                assert first == pos and count >= 0
                pos += count
            assert pos == units
            assert max(c for _, c in blocks) - min(c for _, c in blocks) <= 1


def test_single_process_defaults():
    from causal_attention_swa_b200 import dist as sdist
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    info = sdist.rank_info()
    assert (info.rank, info.world, info.local_rank) == (0, 1, 0) and info.is_root
    assert sdist.max_over_ranks(3.5) == 3.5


@pytest.mark.parametrize("argv", [["--warmup", "2"], ["--gpus", "2"]])
def test_bench_rejects_bad_arguments(argv):
    import bench
    with pytest.raises(SystemExit):
        bench.main(argv)
