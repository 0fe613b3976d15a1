"""The N>1 host logic of bench.py on CPU with the gloo backend (world size 2): every rank runs its
own seeded work (weak scaling, no data-path collective), the timing is the max over ranks, and
the whole-job rate counts the units of all ranks over the slowest rank's time."""
import os
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, str(ROOT))
    import datetime

    import torch.distributed as dist

    import bench
    from block_discrete_diffusion_tcgen05_b200 import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.max_over_ranks(my_ms, dist, "cpu")
        seed = synth.seed_for(2, bench.rank_seed_layer(rank), "q")
        first = float(synth.normal_bf16((4,), seed).f32[0])
        rate = bench.whole_job_rate(1e12, 10, world, mx, 1e12)
        q.put((rank, mx, seed, first, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, mx0, s0, f0, rate0), (r1, mx1, s1, f1, rate1) = res
    assert mx0 == mx1 == 15.0            # both ranks see the slowest rank's time
    assert s0 != s1 and f0 != f1         # each rank works on its own inputs
    assert rate0 == rate1 == pytest.approx(2 * 10 * 1e12 / 15e-3 / 1e12)


def test_single_process_is_identity():
    sys.path.insert(0, str(ROOT))
    import bench

    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_rate(2e9, 4, 1, 2.0, 1e9) == pytest.approx(4000.0)
