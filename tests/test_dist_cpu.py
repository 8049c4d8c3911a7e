"""Multi-rank host logic on CPU: two gloo ranks exercise the replica seeds,
the barrier and the max-over-ranks reduction that bench.py uses to time a
multi-GPU run (no GPU, no data-path collective)."""
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
    from causal_attention_swa_b200 import dist as sdist
    info = sdist.rank_info()
    sdist.init("gloo", info, timeout_s=60)
    sdist.barrier()
    elapsed = 10.0 + 5.0 * rank          # rank 1 is the slow one
    mx = sdist.max_over_ranks(elapsed)
    tot = sdist.sum_over_ranks(1.0)
    q.put((rank, info.world, mx, tot, sdist.replica_seed(4, rank)))
    sdist.shutdown()


def test_two_gloo_ranks_time_as_max_and_seed_independently():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in results] == [0, 1]
    for rank, world, mx, tot, seed in results:
        assert world == 2 and mx == 15.0 and tot == 2.0
    assert results[0][4] == 4 and results[1][4] != 4


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
