"""Pins for the oracle's Index Branch (scoring, block max-pool, forced-local top-k).

Each check compares the oracle with something other than itself: a dense
masked score matrix reduced by a library max, brute-force enumeration of block
subsets, exact invariances, and needles planted by construction.  Passages:
ai-tool-zukan MiniMax MSA guide, sections "2段階構造の中身", "GQAグループ単位の
選択共有とは", "クエリを含むローカルブロックの強制取り込み" and the table in
"ブロック単位選択の数値設計（128トークン×16ブロック=2048）".
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import synth


def _int_bf16(shape, lo, hi, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi, shape, generator=g).to(torch.bfloat16)


def _dense_pooled(q_idx, k_idx, block):
    """Dense [N, G, N] score matrix, causal -inf mask, library amax per block."""
    qi = q_idx.double()
    ki = k_idx.double()
    N = qi.shape[0]
    s = torch.einsum("tgc,sc->tgs", qi, ki)
    causal = torch.arange(N)[None, :] > torch.arange(N)[:, None]
    s = s.masked_fill(causal[:, None, :], float("-inf"))
    nb = (N + block - 1) // block
    pad = nb * block - N
    s = torch.nn.functional.pad(s, (0, pad), value=float("-inf"))
    return s.view(N, s.shape[1], nb, block).amax(dim=-1).numpy()


def _outranks(p, a, b):
    return p[a] > p[b] or (p[a] == p[b] and a < b)


def _brute_force(p, local, top_k):
    others = list(range(local))
    size = min(top_k, local + 1)
    hits = []
    for comb in itertools.combinations(others, size - 1):
        chosen = set(comb)
        if all(_outranks(p, a, b) for a in chosen for b in others if b not in chosen):
            hits.append(sorted(chosen | {local}))
    assert len(hits) == 1, hits
    return hits[0]


@pytest.mark.parametrize("seed", [1, 2, 3])
@pytest.mark.parametrize("N,block,top_k", [(61, 4, 2), (64, 4, 3), (40, 8, 3), (33, 4, 1)])
def test_pooled_matches_dense_masked_max(seed, N, block, top_k):
    G, di = 2, 4
    q_idx = _int_bf16((N, G, di), -3, 4, seed)
    k_idx = _int_bf16((N, di), -3, 4, seed + 100)
    nb = (N + block - 1) // block
    rows = np.arange(N)
    got = oracle.pooled_scores(q_idx, rows, k_idx, block, nb)
    want = _dense_pooled(q_idx, k_idx, block)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("seed", [11, 12, 13, 14])
@pytest.mark.parametrize("N,block,top_k", [(61, 4, 2), (64, 4, 3), (40, 8, 3), (33, 4, 1),
                                           (48, 4, 5)])
def test_selection_equals_brute_force(seed, N, block, top_k):
    """Integer-valued inputs make equal pooled scores common, so ties are exercised."""
    G, di = 2, 3
    q_idx = _int_bf16((N, G, di), -2, 3, seed)
    k_idx = _int_bf16((N, di), -2, 3, seed + 7)
    nb = (N + block - 1) // block
    rows = np.arange(N)
    pooled = _dense_pooled(q_idx, k_idx, block)
    ids = oracle.select_blocks(pooled, rows, block, top_k)
    n_ties = 0
    for t in range(N):
        local = t // block
        for g in range(G):
            want = _brute_force(pooled[t, g], local, top_k)
            got = [int(x) for x in ids[t, g] if x >= 0]
            assert got == want, (t, g, got, want)
            assert all(x == -1 for x in ids[t, g][len(got):])
            n_ties += len(set(pooled[t, g, :local])) < local
    assert n_ties > 0  # the inputs really did contain equal scores


def test_invariants_tiny_config():
    s = synth.PREFILL_CONFIGS["tiny"]
    inp = synth.make_prefill_inputs(s)
    rows = np.arange(s.N)
    pooled = oracle.pooled_scores(inp["q_idx"], rows, inp["k_idx"], s.block, s.nb)
    ids = oracle.select_blocks(pooled, rows, s.block, s.top_k)
    for t in range(0, s.N, 7):
        local = t // s.block
        for g in range(s.G):
            sel = ids[t, g]
            valid = sel[sel >= 0]
            assert local in valid                                  # forced local block
            assert len(valid) == min(s.top_k, local + 1)           # count
            assert np.all(np.diff(valid) > 0)                      # ascending, distinct
            assert valid.max() <= local                            # causal
            assert np.all(sel[len(valid):] == -1)
            keys = sum(min(s.block, t - j * s.block + 1) for j in valid)
            assert keys <= s.top_k * s.block                       # 2,048-token budget
    # the pooled score of a fully invisible block is -inf, of a visible one finite
    assert np.all(np.isneginf(pooled[0, :, 1:]))
    assert np.all(np.isfinite(pooled[-1]))


def test_scaling_k_idx_by_two_keeps_ids():
    s = synth.PREFILL_CONFIGS["tiny"]
    inp = synth.make_prefill_inputs(s)
    rows = np.arange(0, s.N, 3)
    qi = oracle.as_bf16_bits(inp["q_idx"])[rows]
    base = oracle.select_blocks(
        oracle.pooled_scores(qi, rows, inp["k_idx"], s.block, s.nb), rows, s.block, s.top_k)
    k2 = (inp["k_idx"].float() * 2).to(torch.bfloat16)  # exact in bf16
    assert torch.equal(k2.float(), inp["k_idx"].float() * 2)
    scaled = oracle.select_blocks(
        oracle.pooled_scores(qi, rows, k2, s.block, s.nb), rows, s.block, s.top_k)
    np.testing.assert_array_equal(base, scaled)


def test_duplicated_block_lower_id_wins():
    N, G, di, block = 256, 1, 8, 16
    q_idx = _int_bf16((N, G, di), -1, 2, 5)
    k_idx = _int_bf16((N, di), -1, 2, 6)
    a, b = 2, 9
    strong = torch.full((block, di), 4.0).to(torch.bfloat16)
    q_idx[:, 0, :] = torch.ones(di).to(torch.bfloat16)   # every query points along (1,..,1)
    k_idx[a * block:(a + 1) * block] = strong
    k_idx[b * block:(b + 1) * block] = strong
    rows = np.arange((b + 1) * block, N)
    pooled = oracle.pooled_scores(oracle.as_bf16_bits(q_idx)[rows], rows, k_idx, block,
                                  N // block)
    assert np.all(pooled[:, 0, a] == pooled[:, 0, b])
    ids = oracle.select_blocks(pooled, rows, block, 2)  # local + one more
    for i, t in enumerate(rows):
        assert list(ids[i, 0]) == [a, t // block]


def test_groups_select_independently():
    """Changing one group's index query changes only that group's selection."""
    s = synth.PrefillShape("g", N=1024, H=4, G=2, d=16, d_idx=16, block=64, top_k=4)
    inp = synth.make_prefill_inputs(s)
    rows = np.arange(s.N)
    ids0 = oracle.select_blocks(
        oracle.pooled_scores(inp["q_idx"], rows, inp["k_idx"], s.block, s.nb), rows, s.block,
        s.top_k)
    qi = inp["q_idx"].clone()
    qi[:, 1] = -qi[:, 1]
    ids1 = oracle.select_blocks(
        oracle.pooled_scores(qi, rows, inp["k_idx"], s.block, s.nb), rows, s.block, s.top_k)
    np.testing.assert_array_equal(ids0[:, 0], ids1[:, 0])
    assert np.any(ids0[:, 1] != ids1[:, 1])


def test_needles_are_selected():
    s = synth.PREFILL_CONFIGS["tiny"]
    inp = synth.make_prefill_inputs(s)
    assert len(inp["needles"]) == s.n_needles
    rows = np.array(sorted({t for (_, _, t) in inp["needles"]}), dtype=np.int64)
    qi = oracle.as_bf16_bits(inp["q_idx"])[rows]
    ids = oracle.select_blocks(
        oracle.pooled_scores(qi, rows, inp["k_idx"], s.block, s.nb), rows, s.block, s.top_k)
    where = {int(t): i for i, t in enumerate(rows)}
    for (j, g, t) in inp["needles"]:
        assert j in ids[where[t], g]


def test_fewer_visible_blocks_than_k_takes_all():
    s = synth.PREFILL_CONFIGS["tiny"]
    inp = synth.make_prefill_inputs(s)
    rows = np.array([0, 127, 128, 1000, 15 * 128 + 5, 16 * 128], dtype=np.int64)
    qi = oracle.as_bf16_bits(inp["q_idx"])[rows]
    ids = oracle.select_blocks(
        oracle.pooled_scores(qi, rows, inp["k_idx"], s.block, s.nb), rows, s.block, s.top_k)
    for i, t in enumerate(rows):
        local = t // s.block
        if local + 1 <= s.top_k:
            for g in range(s.G):
                assert list(ids[i, g][: local + 1]) == list(range(local + 1))
