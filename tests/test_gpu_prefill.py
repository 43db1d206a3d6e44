"""GPU parity: the sm_100a prefill path against the fp64 oracle.

Every kernel is reached through the C ABI (ctypes binding).  Inputs come from
the shared seeded generator; expected values come only from ``oracle/``.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import block_sparse_long_branch_b200 as m
    m.load_library()
    return m


def _cfg(msa, s):
    return msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, block=s.block, scale=s.scale)


def _ref(inp, s, rows=None, partials=False):
    return oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                          block=s.block, top_k=s.top_k, scale=s.scale, rows=rows,
                          partials=partials)


def _check_prefill(msa, s, inp, rows=None, workspace=None):
    cfg = _cfg(msa, s)
    out, ids = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                               ids_out=True, workspace=workspace)
    torch.cuda.synchronize()
    ref = _ref(inp, s, rows=rows)
    rows = ref["rows"]
    g_ids = ids.cpu().numpy()[rows]
    parity.check_id_rows_valid(g_ids, rows, s.block, s.top_k)
    ties = parity.compare_ids(g_ids, ref["ids"], ref["pooled"], rows, s.block, s.top_k)
    ref_out = ref["out"]
    if ties:  # re-run the Main Branch of the oracle on the GPU's selection
        ref_out = oracle.block_attention(oracle.as_bf16_bits(inp["q"])[rows], rows, inp["k"],
                                         inp["v"], g_ids, s.scale, s.block)
    g_out = out.float().cpu().numpy()[rows]
    errs = parity.check_output(g_out, ref_out)
    return out, ids, ties, errs


# ---------------------------------------------------------------- index branch

@pytest.mark.parametrize("name", ["tiny", "tiny_dense"])
def test_index_scores_match_oracle(msa, name):
    s = synth.PREFILL_CONFIGS[name]
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    got = msa.msa_index_scores(cfg, inp["q_idx"], inp["k_idx"]).cpu().numpy()
    rows = np.arange(s.N)
    want = oracle.pooled_scores(inp["q_idx"], rows, inp["k_idx"], s.block, s.nb)
    inv = np.isneginf(want)
    assert np.array_equal(np.isneginf(got), inv)
    assert np.abs(got[~inv] - want[~inv]).max() < 1e-3


def test_index_scores_row_window_ragged(msa):
    s = synth.PrefillShape("w", N=1000, H=8, G=4, d=128, d_idx=128, top_k=4, n_needles=2,
                           seed=31)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    got = msa.msa_index_scores(cfg, inp["q_idx"], inp["k_idx"], row_begin=301,
                               row_count=555).cpu().numpy()
    rows = np.arange(301, 856)
    want = oracle.pooled_scores(oracle.as_bf16_bits(inp["q_idx"])[rows], rows, inp["k_idx"],
                                s.block, s.nb)
    inv = np.isneginf(want)
    assert np.array_equal(np.isneginf(got), inv)
    assert np.abs(got[~inv] - want[~inv]).max() < 1e-3


@pytest.mark.parametrize("name", ["tiny", "tiny_dense"])
def test_select_topk_matches_oracle(msa, name):
    s = synth.PREFILL_CONFIGS[name]
    inp = synth.make_prefill_inputs(s, device="cuda")
    ids = msa.msa_select_topk(_cfg(msa, s), inp["q_idx"], inp["k_idx"]).cpu().numpy()
    rows = np.arange(s.N)
    pooled = oracle.pooled_scores(inp["q_idx"], rows, inp["k_idx"], s.block, s.nb)
    ref = oracle.select_blocks(pooled, rows, s.block, s.top_k)
    parity.check_id_rows_valid(ids, rows, s.block, s.top_k)
    ties = parity.compare_ids(ids, ref, pooled, rows, s.block, s.top_k)
    assert len(ties) <= 4, ties
    for (j, g, t) in inp["needles"]:
        assert j in ids[t, g]


def test_select_ties_go_to_lower_block(msa):
    """Integer-valued index vectors: many exactly equal pooled scores."""
    s = synth.PrefillShape("ties", N=2048, H=4, G=2, d=64, d_idx=64, top_k=5)
    g = torch.Generator().manual_seed(3)
    q_idx = torch.randint(-1, 2, (s.N, s.G, s.d_idx), generator=g).to(torch.bfloat16).cuda()
    k_idx = torch.randint(-1, 2, (s.N, s.d_idx), generator=g).to(torch.bfloat16).cuda()
    ids = msa.msa_select_topk(_cfg(msa, s), q_idx, k_idx).cpu().numpy()
    rows = np.arange(s.N)
    pooled = oracle.pooled_scores(q_idx, rows, k_idx, s.block, s.nb)
    ref = oracle.select_blocks(pooled, rows, s.block, s.top_k)
    np.testing.assert_array_equal(ids, ref)  # integer sums are exact in fp32


# ---------------------------------------------------------------- query lists

@pytest.mark.parametrize("N,G,top_k", [(4096, 2, 16), (1000, 4, 4), (5000, 8, 32), (130, 1, 2)])
def test_block_query_lists_exact(msa, N, G, top_k):
    s = synth.PrefillShape("c", N=N, H=G, G=G, d=64, d_idx=64, top_k=top_k, n_needles=3,
                           seed=N + top_k)
    inp = synth.make_prefill_inputs(s)
    rows = np.arange(N)
    ids = oracle.select_blocks(oracle.pooled_scores(inp["q_idx"], rows, inp["k_idx"], s.block,
                                                    s.nb), rows, s.block, top_k)
    want_ptr, want_ent = oracle.block_query_lists(ids, s.nb)
    row_ptr, entries = msa.msa_build_block_query_lists(_cfg(msa, s),
                                                       torch.from_numpy(ids).cuda())
    row_ptr = row_ptr.cpu().numpy()
    np.testing.assert_array_equal(row_ptr, want_ptr)
    np.testing.assert_array_equal(entries.cpu().numpy()[:row_ptr[-1]], want_ent)


# ---------------------------------------------------------------- whole prefill

def test_prefill_tiny_all_rows(msa):
    s = synth.PREFILL_CONFIGS["tiny"]
    inp = synth.make_prefill_inputs(s, device="cuda")
    _, ids, ties, _ = _check_prefill(msa, s, inp)
    ids = ids.cpu().numpy()
    for (j, g, t) in inp["needles"]:
        assert j in ids[t, g]


def test_prefill_tiny_topk32_equals_dense(msa):
    """k >= number of blocks: the GPU result must equal dense causal GQA."""
    s = synth.PREFILL_CONFIGS["tiny_dense"]
    inp = synth.make_prefill_inputs(s, device="cuda")
    out, ids, ties, _ = _check_prefill(msa, s, inp)
    assert not ties
    q = inp["q"].float().permute(1, 0, 2)[None]
    k = inp["k"].float().repeat_interleave(s.H // s.G, dim=1).permute(1, 0, 2)[None]
    v = inp["v"].float().repeat_interleave(s.H // s.G, dim=1).permute(1, 0, 2)[None]
    dense = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                             scale=s.scale)
    dense = dense[0].permute(1, 0, 2)
    assert (out.float() - dense).abs().max().item() < 1e-2


@pytest.mark.parametrize("N,H,G,d,di,k", [(1000, 16, 2, 128, 128, 16), (1333, 8, 8, 64, 128, 3),
                                         (777, 32, 4, 128, 64, 32), (129, 8, 1, 64, 64, 1),
                                         (1500, 32, 2, 128, 128, 16), (700, 32, 1, 64, 64, 8)])
def test_prefill_ragged_shapes(msa, N, H, G, d, di, k):
    s = synth.PrefillShape("r", N=N, H=H, G=G, d=d, d_idx=di, top_k=k, n_needles=3,
                           seed=N * 7 + H)
    inp = synth.make_prefill_inputs(s, device="cuda")
    _check_prefill(msa, s, inp)


def test_prefill_chunked_equals_one_shot(msa):
    s = synth.PrefillShape("ch", N=3000, H=16, G=4, d=128, d_idx=128, top_k=8, n_needles=4,
                           seed=8)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    out1, ids1 = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                                 ids_out=True)
    small = msa.msa_prefill_min_workspace(cfg, s.N) * 3
    ws = torch.empty(small, dtype=torch.uint8, device="cuda")
    out2, ids2 = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                                 ids_out=True, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(ids1, ids2)
    assert torch.equal(out1, out2)
    assert msa.msa_get_device_error(ws) == 0


def test_prefill_32k_sampled_rows(msa):
    """The 32K workload in the launch configuration the benchmark times."""
    s = synth.PREFILL_CONFIGS["prefill_32k"]
    inp = synth.make_prefill_inputs(s, device="cuda")
    needle_rows = [t for (_, _, t) in inp["needles"]][:16]
    rows = synth.sample_rows(s.N, 48, seed=5, extra=needle_rows)
    ws = torch.empty(msa.msa_workspace_size(_cfg(msa, s), msa.OP_PREFILL, s.N),
                     dtype=torch.uint8, device="cuda")
    out, ids, ties, errs = _check_prefill(msa, s, inp, rows=rows, workspace=ws)
    assert msa.msa_get_device_error(ws) == 0
    ids = ids.cpu().numpy()
    for (j, g, t) in inp["needles"]:
        assert j in ids[t, g]
    # properties that hold at every row: the forced local block and the budget
    parity.check_id_rows_valid(ids, np.arange(s.N), s.block, s.top_k)
    assert torch.isfinite(out.float()).all()


@pytest.mark.slow
def test_prefill_32k_all_rows(msa):
    """The 32K workload checked on every one of its 32,768 query rows (the
    oracle walks the rows in chunks of 4,096; a few minutes of host time)."""
    s = synth.PREFILL_CONFIGS["prefill_32k"]
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    ws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_PREFILL, s.N), dtype=torch.uint8,
                     device="cuda")
    out, ids = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                               ids_out=True, workspace=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    g_ids = ids.cpu().numpy()
    g_out = out.float().cpu().numpy()
    host = {name: inp[name].cpu() for name in ("q", "k", "v", "q_idx", "k_idx")}
    del inp, out, ids, ws
    ties, max_err, err_sum = [], 0.0, 0.0
    for r0 in range(0, s.N, 4096):
        rows = np.arange(r0, min(r0 + 4096, s.N))
        ref = oracle.prefill(host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"],
                             block=s.block, top_k=s.top_k, scale=s.scale, rows=rows)
        parity.check_id_rows_valid(g_ids[rows], rows, s.block, s.top_k)
        t = parity.compare_ids(g_ids[rows], ref["ids"], ref["pooled"], rows, s.block, s.top_k)
        ref_out = ref["out"]
        if t:  # the oracle's Main Branch on the GPU's selection
            ref_out = oracle.block_attention(oracle.as_bf16_bits(host["q"])[rows], rows,
                                             host["k"], host["v"], g_ids[rows], s.scale,
                                             s.block)
        ties += t
        err = np.abs(g_out[rows].astype(np.float64) - ref_out)
        max_err = max(max_err, float(err.max()))
        err_sum += float(err.sum())
    mean_err = err_sum / g_out.size
    assert np.isfinite(g_out).all()
    assert max_err <= parity.OUT_MAX_ABS, max_err
    assert mean_err <= parity.OUT_MEAN_ABS, mean_err
    assert len(ties) <= 64, len(ties)


def _check_sampled_large(msa, s, n_rows, ws_bytes, seed):
    """Prefill of a long workload in the benchmark's launch configuration
    (chunked query axis when the workspace is capped), checked on sampled rows
    against the oracle; only the sampled rows' queries leave the device."""
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    ws = torch.empty(max(ws_bytes, msa.msa_prefill_min_workspace(cfg, s.N)), dtype=torch.uint8,
                     device="cuda")
    out, ids = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                               ids_out=True, workspace=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    needle_rows = [t for (_, _, t) in inp["needles"]][:24]
    rows = synth.sample_rows(s.N, n_rows, seed=seed, extra=needle_rows)
    rows_dev = torch.from_numpy(rows).cuda()
    nb = s.nb
    qi = oracle.as_bf16_bits(inp["q_idx"][rows_dev])
    pooled = oracle.pooled_scores(qi, rows, inp["k_idx"], s.block, nb)
    ref_ids = oracle.select_blocks(pooled, rows, s.block, s.top_k)
    g_ids = ids[rows_dev].cpu().numpy()
    parity.check_id_rows_valid(g_ids, rows, s.block, s.top_k)
    ties = parity.compare_ids(g_ids, ref_ids, pooled, rows, s.block, s.top_k)
    # Main Branch of the oracle on the GPU's selection (equal to the oracle's
    # own except at listed near-ties)
    sel = g_ids if ties else ref_ids
    qr = oracle.as_bf16_bits(inp["q"][rows_dev])
    ref_out = oracle.block_attention(qr, rows, inp["k"], inp["v"], sel, s.scale, s.block)
    parity.check_output(out[rows_dev].float().cpu().numpy(), ref_out)
    # every needle's query selected its block
    ids_np = ids.cpu().numpy()
    for (j, g, t) in inp["needles"]:
        assert j in ids_np[t, g], (j, g, t)
    return len(ties)


@pytest.mark.slow
def test_prefill_128k_sampled_rows(msa):
    """128K tokens, one pass over the query axis, 4096 rows sampled uniformly
    over the positions plus the needles' queries."""
    s = synth.PREFILL_CONFIGS["prefill_128k"]
    n_ties = _check_sampled_large(msa, s, 4096, 96 << 30, seed=7)
    assert n_ties <= 64


@pytest.mark.slow
def test_prefill_1m_sampled_rows_chunked(msa):
    """1M tokens with a 40 GiB workspace: the query axis runs in chunks, as in
    the benchmark; 2048 rows sampled uniformly plus the needles' queries."""
    s = synth.PREFILL_CONFIGS["prefill_1m"]
    cfg = _cfg(msa, s)
    assert msa.msa_prefill_chunk_tokens(cfg, s.N, 40 << 30) < s.N
    n_ties = _check_sampled_large(msa, s, 2048, 40 << 30, seed=8)
    assert n_ties <= 64


def _check_varlen(msa, s, inp, lens, out, ids):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    for b, L in enumerate(lens):
        if L == 0:
            continue
        s0, s1 = int(cu[b]), int(cu[b + 1])
        ref = oracle.prefill(inp["q"][s0:s1], inp["k"][s0:s1], inp["v"][s0:s1],
                             inp["q_idx"][s0:s1], inp["k_idx"][s0:s1], block=s.block,
                             top_k=s.top_k, scale=s.scale)
        rows = np.arange(L)
        g_ids = ids[s0:s1].cpu().numpy()
        parity.check_id_rows_valid(g_ids, rows, s.block, s.top_k)
        ties = parity.compare_ids(g_ids, ref["ids"], ref["pooled"], rows, s.block, s.top_k)
        ref_out = ref["out"]
        if ties:
            ref_out = oracle.block_attention(oracle.as_bf16_bits(inp["q"][s0:s1]), rows,
                                             inp["k"][s0:s1], inp["v"][s0:s1], g_ids, s.scale,
                                             s.block)
        parity.check_output(out[s0:s1].float().cpu().numpy(), ref_out)


def test_prefill_varlen_matches_per_sequence_oracle(msa):
    """Packed sequences of mixed lengths (one empty, one of a single token), run
    as one batch: each must equal its own causal prefill, ids counted within
    the sequence."""
    lens = [700, 0, 4096 + 5, 128, 1, 2049]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    s = synth.PrefillShape("varlen", N=int(cu[-1]), H=16, G=2, d=128, d_idx=64, top_k=8,
                           n_needles=6, seed=41)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    out, ids = msa.msa_prefill_varlen(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                      inp["k_idx"], cu, ids_out=True)
    torch.cuda.synchronize()
    # one pass over the batch: the plan, the five prefill stages, not six sequences
    assert 0 < msa.msa_last_launch_count() < 20
    _check_varlen(msa, s, inp, lens, out, ids)


def test_prefill_varlen_many_short_sequences(msa):
    """96 sequences of 1 to 600 tokens (most end in a partial block, followed
    directly by the next sequence's rows) with the benchmark's head layout."""
    rng = np.random.default_rng(43)
    lens = [int(x) for x in rng.integers(1, 601, 96)]
    lens[5] = 128
    lens[6] = 256
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    s = synth.PrefillShape("varlen_many", N=int(cu[-1]), H=64, G=8, d=128, d_idx=128,
                           top_k=16, n_needles=0, seed=44)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    ws = torch.empty(msa.msa_prefill_varlen_workspace_size(cfg, cu), dtype=torch.uint8,
                     device="cuda")
    out, ids = msa.msa_prefill_varlen(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                      inp["k_idx"], cu, ids_out=True, workspace=ws)
    assert msa.msa_get_device_error(ws) == 0
    assert msa.msa_last_launch_count() < 20
    _check_varlen(msa, s, inp, lens, out, ids)


@pytest.mark.parametrize("B", [1024, 1100])
def test_prefill_varlen_batch_size_limit(msa, B):
    """1024 sequences is the largest batch the one-pass plan takes (its offsets
    travel as a kernel parameter); 1100 run one after another.  Both match the
    oracle on a spread of sequences."""
    rng = np.random.default_rng(B)
    lens = [int(x) for x in rng.integers(1, 5, B)]
    lens[B // 2] = 300
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    s = synth.PrefillShape("varlen_b", N=int(cu[-1]), H=8, G=2, d=64, d_idx=64, top_k=4,
                           seed=45)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    out, ids = msa.msa_prefill_varlen(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                      inp["k_idx"], cu, ids_out=True)
    torch.cuda.synchronize()
    one_pass = msa.msa_last_launch_count() < 20
    assert one_pass == (B <= 1024)
    pick = sorted({0, 1, B // 2, B - 1} | set(int(x) for x in rng.integers(0, B, 8)))
    sub = [lens[b] for b in pick]
    rows = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in pick])
    sub_inp = {n: inp[n][torch.from_numpy(rows).cuda()] for n in ("q", "k", "v", "q_idx",
                                                                    "k_idx")}
    _check_varlen(msa, s, sub_inp, sub, out[torch.from_numpy(rows).cuda()],
                  ids[torch.from_numpy(rows).cuda()])


def test_prefill_varlen_small_workspace_chunks_each_sequence(msa):
    """With the minimum workspace every sequence runs in query chunks; the
    result equals the one-shot call bit for bit."""
    lens = [3000, 5000]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    s = synth.PrefillShape("varlen2", N=int(cu[-1]), H=8, G=2, d=64, d_idx=64, top_k=4, seed=42)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    full = msa.msa_prefill_varlen(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                                  cu)
    ws = torch.empty(msa.msa_prefill_min_workspace(cfg, max(lens)), dtype=torch.uint8,
                     device="cuda")
    assert msa.msa_prefill_chunk_tokens(cfg, max(lens), ws.numel(), ids_returned=False) < max(lens)
    small = msa.msa_prefill_varlen(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                   inp["k_idx"], cu, workspace=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    assert torch.equal(full, small)


def test_head_shards_equal_whole_prefill(msa):
    """The head-sharded plan on one GPU: each rank's group slice computed by
    its own msa_prefill call (one after another here, no collective), the
    slices concatenated along the heads, equal the single call bit for bit."""
    from block_sparse_long_branch_b200 import shard
    s = synth.PrefillShape("shards", N=3000, H=16, G=4, d=128, d_idx=128, top_k=8, n_needles=4,
                           seed=62)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    whole_out, whole_ids = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                           inp["k_idx"], ids_out=True)
    for world in (2, 4):
        outs, idss = [], []
        for rank in range(world):
            g0, g1 = shard.group_range(s.G, rank, world)
            c = msa.config((g1 - g0) * (s.H // s.G), g1 - g0, s.d, s.d_idx, top_k=s.top_k,
                           scale=s.scale)
            o, i = msa.msa_prefill(c, *shard.shard_inputs(inp["q"], inp["k"], inp["v"],
                                                          inp["q_idx"], inp["k_idx"], s.H, s.G,
                                                          rank, world), ids_out=True)
            outs.append(o)
            idss.append(i)
        torch.cuda.synchronize()
        assert torch.equal(torch.cat(idss, dim=1), whole_ids)
        assert torch.equal(torch.cat(outs, dim=1), whole_out)
