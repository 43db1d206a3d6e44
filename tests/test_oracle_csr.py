"""Pins for the oracle's inversion of the selection map into per-block query lists.

The KV-block-outer operator gathers, for each key block, the queries that hit
it (tnkblog MiniMax M3 / MSA post, section "MSA の実装"; CSDN M3 write-up,
section "MiniMax Sparse Attention（MSA）").  The lists are checked against a
Python dictionary grouping followed by a library sort.
"""
import collections

import numpy as np
import pytest

import oracle
import synth


def _by_dict(ids, nb):
    N, G, k = ids.shape
    lists = collections.defaultdict(list)
    for t in range(N):
        for g in range(G):
            for r in range(k):
                j = int(ids[t, g, r])
                if j >= 0:
                    lists[(g, j)].append((t, r))
    return {key: sorted(val) for key, val in lists.items()}


@pytest.mark.parametrize("top_k", [1, 4, 16])
def test_lists_match_dictionary_grouping(top_k):
    s = synth.PrefillShape("c", N=700, H=2, G=2, d=8, d_idx=8, block=32, top_k=top_k,
                           n_needles=3, seed=21)
    inp = synth.make_prefill_inputs(s)
    rows = np.arange(s.N)
    ids = oracle.select_blocks(
        oracle.pooled_scores(inp["q_idx"], rows, inp["k_idx"], s.block, s.nb), rows, s.block,
        top_k)
    row_ptr, entries = oracle.block_query_lists(ids, s.nb)
    want = _by_dict(ids, s.nb)
    assert row_ptr[0] == 0 and row_ptr[-1] == len(entries)
    assert len(entries) == int((ids >= 0).sum())
    for g in range(s.G):
        for j in range(s.nb):
            seg = entries[row_ptr[g * s.nb + j]:row_ptr[g * s.nb + j + 1]]
            got = [(int(e) >> 5, int(e) & 31) for e in seg]
            assert got == want.get((g, j), []), (g, j)
            # the block's own 32 queries always hit it (forced local block)
            own = [t for (t, _) in got if t // s.block == j]
            assert own == list(range(j * s.block, min(s.N, (j + 1) * s.block)))


def test_out_of_range_id_is_rejected():
    ids = np.zeros((4, 1, 2), dtype=np.int32)
    ids[2, 0, 1] = 7
    with pytest.raises(ValueError):
        oracle.block_query_lists(ids, 4)
