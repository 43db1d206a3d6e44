"""GPU parity: one decode step against the fp64 oracle, every query checked."""
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


def _oracle_one(inp, s, b):
    """Oracle for sequence b.  Only the selected key blocks' K/V rows are copied
    to the host: they are stacked in ascending block order, which keeps every
    selected key's visibility (the local block is the last one)."""
    cu = inp["cu_seqlens"].tolist()
    s0, s1 = cu[b], cu[b + 1]
    L = s1 - s0
    nb = (L + s.block - 1) // s.block
    pos = np.array([L - 1], dtype=np.int64)
    qib = oracle.as_bf16_bits(inp["q_idx"][b:b + 1])
    pooled = oracle.pooled_scores(qib, pos, inp["k_idx_cache"][s0:s1], s.block, nb)
    ids = oracle.select_blocks(pooled, pos, s.block, s.top_k)
    used = sorted({int(j) for j in ids[0].ravel() if j >= 0})
    remap = {j: c for c, j in enumerate(used)}
    kc = torch.zeros(len(used) * s.block, s.G, s.d, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for c, j in enumerate(used):
        r0, r1 = s0 + j * s.block, min(s1, s0 + (j + 1) * s.block)
        kc[c * s.block:c * s.block + (r1 - r0)] = inp["k_cache"][r0:r1].cpu()
        vc[c * s.block:c * s.block + (r1 - r0)] = inp["v_cache"][r0:r1].cpu()
    cids = np.vectorize(lambda j: remap[j] if j >= 0 else -1)(ids).astype(np.int32)
    cpos = np.array([(len(used) - 1) * s.block + (L - 1) % s.block], dtype=np.int64)
    out = oracle.block_attention(oracle.as_bf16_bits(inp["q"][b:b + 1]), cpos, kc, vc, cids,
                                 s.scale, s.block)
    return ids[0], pooled[0], out[0], (used, remap, kc, vc, cpos)


def _run(msa, s, inp):
    cu = inp["cu_seqlens"].cuda()
    cfg = _cfg(msa, s)
    total = inp["k_cache"].shape[0]
    ws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_DECODE, total, s.B), dtype=torch.uint8,
                     device="cuda")
    out, ids = msa.msa_decode(cfg, inp["q"], inp["q_idx"], inp["k_cache"], inp["v_cache"],
                              inp["k_idx_cache"], cu, max(s.seq_lens), ids_out=True,
                              workspace=ws)
    assert msa.msa_get_device_error(ws) == 0
    return out.float().cpu().numpy(), ids.cpu().numpy()


def _check(msa, s, inp):
    g_out, g_ids = _run(msa, s, inp)
    n_ties = 0
    for b in range(s.B):
        L = s.seq_lens[b]
        pos = np.array([L - 1])
        ids, pooled, out, (used, remap, kc, vc, cpos) = _oracle_one(inp, s, b)
        parity.check_id_rows_valid(g_ids[b:b + 1], pos, s.block, s.top_k)
        ties = parity.compare_ids(g_ids[b:b + 1], ids[None], pooled[None], pos, s.block, s.top_k)
        if ties:
            n_ties += len(ties)
            # oracle Main Branch on the GPU's blocks (those rows' K/V copied as above)
            gsel = sorted({int(j) for j in g_ids[b].ravel() if j >= 0})
            s0 = int(inp["cu_seqlens"][b])
            kc2 = torch.zeros(len(gsel) * s.block, s.G, s.d, dtype=torch.bfloat16)
            vc2 = torch.zeros_like(kc2)
            for c, j in enumerate(gsel):
                r0, r1 = s0 + j * s.block, min(s0 + L, s0 + (j + 1) * s.block)
                kc2[c * s.block:c * s.block + (r1 - r0)] = inp["k_cache"][r0:r1].cpu()
                vc2[c * s.block:c * s.block + (r1 - r0)] = inp["v_cache"][r0:r1].cpu()
            rm = {j: c for c, j in enumerate(gsel)}
            cids = np.vectorize(lambda j: rm[j] if j >= 0 else -1)(g_ids[b:b + 1]).astype(np.int32)
            cpos2 = np.array([(len(gsel) - 1) * s.block + (L - 1) % s.block])
            out = oracle.block_attention(oracle.as_bf16_bits(inp["q"][b:b + 1]), cpos2, kc2, vc2,
                                         cids, s.scale, s.block)[0]
        parity.check_output(g_out[b], out)
    for (b, j, g) in inp["needles"]:
        assert j in g_ids[b, g], (b, j, g)
    return n_ties


def test_decode_short_sequences(msa):
    """160 sequences of 2 to 5 tokens: softmaxes over a handful of keys, whose
    outputs reach magnitude 2 to 4, where the bf16 output rounding alone takes
    up to 0.0078 of the 1e-2 bound."""
    s = synth.DecodeShape("dshort", seq_lens=(2, 3, 4, 5) * 40, H=64, G=8, d=128, d_idx=128,
                          top_k=16, seed=17)
    inp = synth.make_decode_inputs(s, device="cuda")
    _check(msa, s, inp)


def test_decode_sixteen_heads_per_group(msa):
    """16 query heads per group: the attention's two 8-head tiles."""
    s = synth.DecodeShape("d16", seq_lens=(3, 300, 4097, 2, 128 * 9 + 1, 5000), H=32, G=2,
                          d=128, d_idx=128, top_k=16, needles_per_seq=(0, 1, 2, 0, 1, 2), seed=19)
    inp = synth.make_decode_inputs(s, device="cuda")
    _check(msa, s, inp)


def test_decode_small_mixed_lengths(msa):
    s = synth.DecodeShape("ds", seq_lens=(300, 5000, 128 * 20 + 7, 128, 1, 2049), H=16, G=2,
                          d=128, d_idx=64, top_k=4, needles_per_seq=(1, 2, 2, 0, 0, 1), seed=12)
    inp = synth.make_decode_inputs(s, device="cuda")
    _check(msa, s, inp)


def test_decode_small_d64_topk32(msa):
    s = synth.DecodeShape("ds2", seq_lens=(9000, 4096, 700), H=8, G=8, d=64, d_idx=128, top_k=32,
                          needles_per_seq=(3, 2, 1), seed=13)
    inp = synth.make_decode_inputs(s, device="cuda")
    _check(msa, s, inp)


@pytest.mark.slow
def test_decode_full_config_every_query(msa):
    """16 x 256K + 1 x 1M caches, every one of the 17 queries against the oracle."""
    s = synth.DECODE_CONFIG
    inp = synth.make_decode_inputs(s, device="cuda")
    n_ties = _check(msa, s, inp)
    assert n_ties <= 8


def test_decode_all_scores_tied(msa):
    """Every index key zero: all pooled scores tie at 0, so the lowest block ids win
    (ties go to the lower id), plus the local block."""
    s = synth.DecodeShape("dtie", seq_lens=(128 * 600 + 17, 128 * 40), H=16, G=2, d=64,
                          d_idx=64, top_k=16, seed=14)
    inp = synth.make_decode_inputs(s, device="cuda")
    inp["k_idx_cache"].zero_()
    g_out, g_ids = _run(msa, s, inp)
    for b, L in enumerate(s.seq_lens):
        nb = (L + s.block - 1) // s.block
        want = list(range(min(s.top_k - 1, nb - 1))) + [nb - 1]
        want += [-1] * (s.top_k - len(want))
        for g in range(s.G):
            assert g_ids[b, g].tolist() == want, (b, g)
        ids, pooled, out, _ = _oracle_one(inp, s, b)
        assert (ids == np.asarray(want)[None, :]).all()
        parity.check_output(g_out[b], out)


def test_decode_clustered_high_scores(msa):
    """The high-scoring blocks all fall on the candidates of one warp of the
    selection (block ids j with j mod 256 < 32), so the threshold taken from
    per-warp bests is weak and the exhaustive per-thread-list path decides."""
    s = synth.DecodeShape("dclu", seq_lens=(128 * 2048, 128 * 300), H=16, G=2, d=64, d_idx=128,
                          top_k=16, seed=15)
    inp = synth.make_decode_inputs(s, device="cuda")
    kic = inp["k_idx_cache"]
    cu = inp["cu_seqlens"].tolist()
    for b in range(s.B):
        u = inp["q_idx"][b, 0].double() + inp["q_idx"][b, 1].double()
        nb = (s.seq_lens[b] + s.block - 1) // s.block
        for j in range(nb - 1):
            if j % 256 < 32:
                r0 = cu[b] + j * s.block
                kic[r0:r0 + s.block] = (u * (1.0 + 1e-3 * j)).to(torch.bfloat16)
    _check(msa, s, inp)


def test_decode_selection_long_sequences(msa):
    """Selection over sequences of 2,000 to 3,000 blocks.
    Sequence 0: the best blocks all lie in its last third (ids >= 2048).
    Sequence 1: every score ties, so the lowest ids win.  Sequence 2: 2,050
    blocks, one more than a multiple of 1,024 non-local candidates."""
    s = synth.DecodeShape("dsli", seq_lens=(128 * 3000 + 9, 128 * 2601, 128 * 2050), H=16, G=2,
                          d=64, d_idx=128, top_k=16, seed=16)
    inp = synth.make_decode_inputs(s, device="cuda")
    kic = inp["k_idx_cache"]
    cu = inp["cu_seqlens"].tolist()
    u = inp["q_idx"][0, 0].double() + inp["q_idx"][0, 1].double()
    for j in range(2048, 3000):
        if j % 61 == 3:
            r0 = cu[0] + j * s.block
            kic[r0:r0 + s.block] = (u * (1.0 + 1e-3 * j)).to(torch.bfloat16)
    kic[cu[1]:cu[2]].zero_()
    g_out, g_ids = _run(msa, s, inp)
    nb1 = 2601
    want = list(range(s.top_k - 1)) + [nb1 - 1]
    for g in range(s.G):
        assert g_ids[1, g].tolist() == want, g
    sel0 = {int(j) for j in g_ids[0].ravel() if j >= 0}
    assert all(j >= 2048 for j in sel0), sorted(sel0)
    _check(msa, s, inp)


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_shards_equal_whole_decode(msa, world):
    """The sequence-sharded decode's per-rank calls on one GPU: shards run with
    the library's msa_decode and concatenated in rank order give the whole
    batch's ids exactly, and its outputs up to the order of the split merge."""
    from block_sparse_long_branch_b200 import shard
    s = synth.DecodeShape("dsh", seq_lens=(3000, 129, 70000, 4096, 1, 20000, 640), H=16, G=2,
                          d=128, d_idx=128, top_k=16, seed=29)
    inp = synth.make_decode_inputs(s, device="cuda")
    whole_out, whole_ids = _run(msa, s, inp)
    cu = inp["cu_seqlens"].tolist()
    cfg = _cfg(msa, s)
    outs, ids = [], []
    for r in range(world):
        qq, qi, kc, vc, kic, cu_r = shard.shard_decode_inputs(
            inp["q"], inp["q_idx"], inp["k_cache"], inp["v_cache"], inp["k_idx_cache"], cu, r,
            world)
        if qq.shape[0] == 0:
            continue
        lens = (cu_r[1:] - cu_r[:-1]).tolist()
        o, i = msa.msa_decode(cfg, qq, qi, kc, vc, kic, cu_r.cuda(), max(lens), ids_out=True)
        outs.append(o.float().cpu().numpy())
        ids.append(i.cpu().numpy())
    np.testing.assert_array_equal(np.concatenate(ids), whole_ids)
    np.testing.assert_allclose(np.concatenate(outs), whole_out, atol=2e-3, rtol=0)
