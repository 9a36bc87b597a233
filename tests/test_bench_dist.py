"""The multi-process plumbing of bench.py on the CPU: two gloo ranks (the same
rendezvous torchrun gives), barrier, and the MAX-over-ranks time reduction that
turns per-rank elapsed times into the job's time."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench

    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
    results[rank] = bench.max_over_ranks(elapsed, w)
    import torch.distributed as dist

    dist.destroy_process_group()


def test_two_rank_max_reduction():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        assert dict(results) == {0: 15.0, 1: 15.0}


def test_single_process_needs_no_process_group():
    import bench

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    r, w, local = bench.dist_setup(1)
    assert (r, w, local) == (0, 1, 0)
    assert bench.max_over_ranks(3.5, w) == 3.5


def test_work_accounting():
    """Visible pairs: non-causal M*N; causal bottom-right sum_i min(N, i + N - M + 1)."""
    import bench
    import synth

    assert bench.visible_pairs(4, 4, False) == 16
    assert bench.visible_pairs(4, 4, True) == 10
    assert bench.visible_pairs(2, 5, True) == 4 + 5
    assert bench.visible_pairs(5, 2, True) == 1 + 2
    p = synth.make_varlen("x", [3, 1], 2, 1, 64, "f16", True, seed=0)
    assert bench.prefill_flops(p) == 4 * 64 * 2 * (6 + 1)
    d = synth.make_decode("d", [10, 0, 5], 8, 2, 128, "bf16", seed=0)
    assert bench.decode_bytes(d) == 2 * 15 * 2 * 128 * 2 + 2 * 3 * 8 * 128 * 2
