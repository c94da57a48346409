"""The N > 1 path of bench.py on CPU: two ranks over gloo (no GPU).

bench.py runs one replica per GPU: every rank works on its own sequences (its
own input seeds), the step has no exchange, and the only collectives are the
barrier and the element-wise maximum of the measured times, from which rank 0
reports the whole-job rate.  These tests run exactly those host functions in
two processes.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from datetime import timedelta

    import torch.distributed as dist

    import bench
    from workloads import gen_draft_logits, get_config

    w, r, local = bench.rank_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=timedelta(seconds=60))
    try:
        # each rank measured different times; every rank must end with the maxima
        mine = [1.0 + r, 10.0 - r, 0.5 * (r + 1)]
        red = bench.max_over_ranks(mine, dist, "cpu")
        dist.barrier()
        cfg = get_config("tiny")
        first = gen_draft_logits(cfg, bench.input_seed(r, 0))
        np.save(os.path.join(out_dir, f"rank{r}_inputs.npy"), first)
        np.save(os.path.join(out_dir, f"rank{r}.npy"),
                np.array(red + [w, r, local, bench.whole_job_rate(w, red[0])], dtype=np.float64))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_ranks_reduce_max_and_work_on_their_own_inputs(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [np.load(tmp_path / f"rank{r}.npy") for r in range(world)]
    for r in range(world):
        red, w, rank, local, rate = res[r][:3], res[r][3], res[r][4], res[r][5], res[r][6]
        assert w == world and rank == r and local == r
        np.testing.assert_array_equal(red, [2.0, 10.0, 1.0])   # max over ranks, element by element
        assert rate == pytest.approx(world * 1000.0 / 2.0)     # whole job: both ranks' steps per max time
    a, b = (np.load(tmp_path / f"rank{r}_inputs.npy") for r in range(world))
    assert a.shape == b.shape and not np.array_equal(a, b)       # distinct sequences per rank


def test_alone_the_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], None, "cpu") == [3.0, 4.0]
    assert bench.whole_job_rate(1, 0.1) == pytest.approx(10000.0)
    assert bench.input_seed(0, 3) != bench.input_seed(1, 3)
