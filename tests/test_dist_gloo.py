"""bench.py's multi-process plumbing on CPU: two gloo ranks.

Under torchrun every rank runs one replica of the workload; the job's rate is
the units of all ranks over the slowest rank's time, and the reference arm runs
on rank 0 only.  These run the same helpers bench.py uses, with world size 2,
on the host (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank), OMP_NUM_THREADS="2")
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup()
    try:
        assert (r, w, local) == (rank, world, rank)
        assert dist.get_backend() == "gloo"
        # slowest rank decides: rank 1 took 3x longer
        ms = 10.0 * (1 + 2 * rank)
        rate, ms_max = bench.replica_rate(1000, ms, world)
        bench.barrier(world)
        # reference arm: rank 0 prints, the others do no work
        args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "1",
                                 "--warmup", "0", "--ref-rows", "2"])
        line = bench.run_reference(args, r, w)
        q.put((rank, rate, ms_max, None if line is None else (line["impl"], line["n_gpus"],
                                                               line["value"] > 0)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_rate_and_reference_arm():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, rate, ms_max, ref = q.get(timeout=240)
        res[rank] = (rate, ms_max, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        rate, ms_max, _ = res[rank]
        assert ms_max == pytest.approx(30.0)
        assert rate == pytest.approx(2 * 1000 / 0.030)
    assert res[0][2] == ("reference", 2, True)
    assert res[1][2] is None
