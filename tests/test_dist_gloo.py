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


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank), OMP_NUM_THREADS="2")
    import torch
    import torch.distributed as dist
    import oracle
    import synth
    import block_sparse_long_branch_b200 as msa
    from block_sparse_long_branch_b200 import shard
    dist.init_process_group("gloo")
    try:
        s = synth.PrefillShape("shard", N=640, H=8, G=4, d=64, d_idx=64, top_k=4, n_needles=4,
                               seed=61)
        inp = synth.make_prefill_inputs(s, device="cpu")
        cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, scale=s.scale)

        def oracle_slice(c, qq, kk, vv, qi, ki):
            r = oracle.prefill(qq, kk, vv, qi, ki, block=c.block_size, top_k=c.top_k,
                               scale=c.softmax_scale)
            assert qq.shape[1] == c.num_heads and kk.shape[1] == c.num_groups
            return torch.from_numpy(r["out"]), torch.from_numpy(r["ids"])

        out, ids = shard.head_sharded_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                              inp["k_idx"], prefill=oracle_slice)
        if rank == 0:
            full = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                                  block=s.block, top_k=s.top_k, scale=s.scale)
            same = (torch.equal(out, torch.from_numpy(full["out"])) and
                    torch.equal(ids, torch.from_numpy(full["ids"])))
            q.put(("ok", same, tuple(out.shape), tuple(ids.shape)))
    except Exception as e:  # report instead of hanging the parent
        q.put(("error", repr(e), None, None))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_head_sharded_prefill_equals_one_rank():
    """Two gloo ranks, two GQA groups each, the oracle standing in for the
    per-rank prefill: the gathered output and ids equal the unsharded oracle."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    status, same, oshape, ishape = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
    assert status == "ok", same
    assert same and oshape == (640, 8, 64) and ishape == (640, 4, 4)
    for p in procs:
        assert p.exitcode == 0


def test_group_range_splits_evenly():
    from block_sparse_long_branch_b200 import shard
    assert [shard.group_range(8, r, 4) for r in range(4)] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    with pytest.raises(ValueError):
        shard.group_range(8, 0, 3)


def _seq_shard_worker(rank, world, port, lens, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank), OMP_NUM_THREADS="2")
    import torch
    import torch.distributed as dist
    import oracle
    import synth
    import block_sparse_long_branch_b200 as msa
    from block_sparse_long_branch_b200 import shard
    dist.init_process_group("gloo")
    try:
        s = synth.DecodeShape("dshard", seq_lens=tuple(lens), H=8, G=2, d=64, d_idx=64,
                              top_k=4, seed=23)
        inp = synth.make_decode_inputs(s, device="cpu")
        cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, scale=s.scale)

        def oracle_shard(c, qq, qi, kc, vc, kic, cu):
            r = oracle.decode(qq, qi, kc, vc, kic, cu.numpy(), block=c.block_size,
                              top_k=c.top_k, scale=c.softmax_scale)
            return (torch.from_numpy(r["out"]).to(torch.bfloat16),
                    torch.from_numpy(r["ids"]))

        cu = inp["cu_seqlens"].tolist()
        out, ids = shard.sequence_sharded_decode(cfg, inp["q"], inp["q_idx"], inp["k_cache"],
                                                 inp["v_cache"], inp["k_idx_cache"], cu,
                                                 decode=oracle_shard)
        mine = shard.sequence_range(cu, rank, world)
        if rank == 0:
            full = oracle.decode(inp["q"], inp["q_idx"], inp["k_cache"], inp["v_cache"],
                                 inp["k_idx_cache"], cu, block=s.block, top_k=s.top_k,
                                 scale=s.scale)
            same = (torch.equal(out, torch.from_numpy(full["out"]).to(torch.bfloat16)) and
                    torch.equal(ids, torch.from_numpy(full["ids"])))
            q.put(("ok", same, tuple(out.shape), mine))
        else:
            q.put(("rank", None, None, mine))
    except Exception as e:  # report instead of hanging the parent
        q.put(("error", repr(e), None, None))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("lens", [[300, 700, 129, 2000, 50], [4000]])
def test_sequence_sharded_decode_equals_one_rank(lens):
    """Two gloo ranks split the batch by cached length (with one sequence, rank 0
    has none); the gathered outputs equal the unsharded oracle's."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seq_shard_worker, args=(r, world, port, lens, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    errors = [g for g in got if g[0] == "error"]
    assert not errors, errors
    main = next(g for g in got if g[0] == "ok")
    assert main[1] and main[2] == (len(lens), 8, 64)
    ranges = sorted(g[3] for g in got)
    assert ranges[0][0] == 0 and ranges[-1][1] == len(lens)
    for p in procs:
        assert p.exitcode == 0


def test_sequence_range_balances_cached_length():
    from block_sparse_long_branch_b200 import shard
    cu = [0]
    for L in [262144] * 16 + [1048576]:
        cu.append(cu[-1] + L)
    assert [shard.sequence_range(cu, r, 2) for r in range(2)] == [(0, 10), (10, 17)]
    parts = [shard.sequence_range(cu, r, 8) for r in range(8)]
    assert parts[0][0] == 0 and parts[-1] == (16, 17)
    assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
    # one sequence: its middle lies in rank 1's half, rank 0 has none
    assert shard.sequence_range([0, 4000], 0, 2) == (0, 0)
    assert shard.sequence_range([0, 4000], 1, 2) == (0, 1)


@pytest.mark.parametrize("world", [1, 3, 4, 6])
def test_decode_shards_cover_the_batch_exactly(world):
    """Every rank's slice, concatenated in rank order, gives back the batch; each
    slice's offsets start at 0 and keep the sequence lengths."""
    import torch
    from block_sparse_long_branch_b200 import shard
    lens = [5, 1, 300, 2, 40, 7]
    cu = [0]
    for L in lens:
        cu.append(cu[-1] + L)
    B, T = len(lens), cu[-1]
    q = torch.arange(B * 3, dtype=torch.float32).reshape(B, 3)
    qi = q + 1000
    kc = torch.arange(T * 2, dtype=torch.float32).reshape(T, 2)
    parts = [shard.shard_decode_inputs(q, qi, kc, kc + 1, kc + 2, cu, r, world)
             for r in range(world)]
    assert torch.equal(torch.cat([p[0] for p in parts]), q)
    assert torch.equal(torch.cat([p[1] for p in parts]), qi)
    assert torch.equal(torch.cat([p[2] for p in parts]), kc)
    assert torch.equal(torch.cat([p[4] for p in parts]), kc + 2)
    got_lens = []
    for p in parts:
        c = p[5].tolist()
        assert c[0] == 0 and len(c) == p[0].shape[0] + 1 and c[-1] == p[2].shape[0]
        got_lens += [b - a for a, b in zip(c, c[1:])]
    assert got_lens == lens
