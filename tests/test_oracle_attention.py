"""Pins for the oracle's Main Branch (exact softmax over the selected blocks).

Checks against the library attention routine (torch SDPA, fp64) with causal
and block masks, against closed forms, and against the convex-combination and
log-sum-exp merge identities of softmax.  Passages: ai-tool-zukan MiniMax MSA
guide, sections "Index BranchとMain Branchの役割分担" (exact softmax over the
selected blocks) and "アテンション主計算をコンテキスト長から切り離す仕組み"
(dense GQA is O(N) per query; MSA is O(k B_k)), and "GQAグループ単位の選択共有
とは" (heads of a group share one block set).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


def _sdpa(q_rows, pos, k, v, H, G, scale, allowed=None):
    """torch SDPA in fp64 for query rows at positions ``pos`` over all keys."""
    n = q_rows.shape[0]
    T = k.shape[0]
    qq = q_rows.double().permute(1, 0, 2)[None]                      # [1,H,n,d]
    kk = k.double().repeat_interleave(H // G, dim=1).permute(1, 0, 2)[None]
    vv = v.double().repeat_interleave(H // G, dim=1).permute(1, 0, 2)[None]
    causal = torch.arange(T)[None, :] <= torch.as_tensor(pos)[:, None]   # [n,T]
    mask = causal[None, None].expand(1, H, n, T)
    if allowed is not None:
        mask = mask & allowed[None]
    o = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def _block_mask(ids, pos, T, H, G, block):
    """allowed[h, i, s] = key block of s is selected by row i's group."""
    n = len(pos)
    blk = torch.arange(T) // block
    allowed = torch.zeros(H, n, T, dtype=torch.bool)
    for i in range(n):
        for h in range(H):
            sel = [int(x) for x in ids[i, h // (H // G)] if x >= 0]
            allowed[h, i] = torch.isin(blk, torch.tensor(sel))
    return allowed


def test_dense_equivalence_small():
    """top_k >= number of blocks: MSA must equal dense causal GQA."""
    s = synth.PrefillShape("d", N=300, H=4, G=2, d=16, d_idx=8, block=32, top_k=16)
    inp = synth.make_prefill_inputs(s)
    r = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                       block=s.block, top_k=s.top_k, scale=s.scale)
    want = _sdpa(inp["q"], np.arange(s.N), inp["k"], inp["v"], s.H, s.G, s.scale)
    np.testing.assert_allclose(r["out"], want, rtol=0, atol=1e-12)


def test_dense_equivalence_tiny_config_topk32():
    """The tiny workload with top-k 32 (= all 32 blocks) equals dense causal GQA."""
    s = synth.PREFILL_CONFIGS["tiny_dense"]
    inp = synth.make_prefill_inputs(s)
    rows = synth.sample_rows(s.N, 96, seed=1)
    r = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                       block=s.block, top_k=s.top_k, scale=s.scale, rows=rows)
    want = _sdpa(inp["q"][rows], rows, inp["k"], inp["v"], s.H, s.G, s.scale)
    np.testing.assert_allclose(r["out"], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("top_k", [1, 3, 5])
def test_block_masked_library_attention(top_k):
    s = synth.PrefillShape("m", N=257, H=6, G=3, d=8, d_idx=8, block=16, top_k=top_k,
                           n_needles=4, seed=77)
    inp = synth.make_prefill_inputs(s)
    r = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                       block=s.block, top_k=s.top_k, scale=s.scale)
    pos = np.arange(s.N)
    allowed = _block_mask(r["ids"], pos, s.N, s.H, s.G, s.block)
    want = _sdpa(inp["q"], pos, inp["k"], inp["v"], s.H, s.G, s.scale, allowed)
    np.testing.assert_allclose(r["out"], want, rtol=0, atol=1e-12)


def test_partials_merge_and_single_block_softmax():
    s = synth.PrefillShape("p", N=200, H=4, G=2, d=8, d_idx=8, block=16, top_k=4, seed=5)
    inp = synth.make_prefill_inputs(s)
    r = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                       block=s.block, top_k=s.top_k, scale=s.scale, partials=True)
    lse, o = r["lse"], r["o"]
    L = np.logaddexp.reduce(lse, axis=2)                                  # [n,H]
    w = np.exp(lse - L[..., None])
    merged = np.einsum("nhr,nhrd->nhd", w, o)
    np.testing.assert_allclose(merged, r["out"], rtol=0, atol=1e-12)
    # every partial is the softmax restricted to its one block
    pos = np.arange(s.N)
    for slot in range(s.top_k):
        one = np.where(np.arange(s.top_k)[None, None, :] == slot, r["ids"], -1)
        allowed = _block_mask(one, pos, s.N, s.H, s.G, s.block)
        has = np.array([[r["ids"][i, h // 2, slot] >= 0 for h in range(s.H)]
                        for i in range(s.N)])
        want = _sdpa(inp["q"], pos, inp["k"], inp["v"], s.H, s.G, s.scale, allowed)
        np.testing.assert_allclose(o[:, :, slot][has], want[has], rtol=0, atol=1e-12)
        assert np.all(np.isneginf(lse[:, :, slot][~has]))


def test_constant_values_give_constant_output():
    s = synth.PrefillShape("c", N=256, H=4, G=2, d=8, d_idx=8, block=32, top_k=3, seed=9)
    inp = synth.make_prefill_inputs(s)
    v = torch.empty_like(inp["v"])
    v[:, 0, :] = torch.tensor([1.5, -2.0, 0.25, 3.0, 0.0, -0.5, 8.0, 1.0])
    v[:, 1, :] = -0.75
    r = oracle.prefill(inp["q"], inp["k"], v, inp["q_idx"], inp["k_idx"],
                       block=s.block, top_k=s.top_k, scale=s.scale)
    np.testing.assert_allclose(r["out"][:, :2], np.broadcast_to(v[0, 0].double().numpy(),
                                                                (s.N, 2, s.d)), atol=1e-14)
    np.testing.assert_allclose(r["out"][:, 2:], -0.75, atol=1e-14)


def test_identical_keys_give_running_mean():
    """All keys equal and every block selected: uniform weights, out[t] = mean(v[0..t])."""
    s = synth.PrefillShape("u", N=160, H=2, G=1, d=4, d_idx=4, block=16, top_k=10, seed=3)
    inp = synth.make_prefill_inputs(s)
    k = inp["k"][:1].expand_as(inp["k"]).contiguous()
    r = oracle.prefill(inp["q"], k, inp["v"], inp["q_idx"], inp["k_idx"],
                       block=s.block, top_k=s.top_k, scale=s.scale)
    vv = inp["v"][:, 0].double().numpy()
    running = np.cumsum(vv, axis=0) / np.arange(1, s.N + 1)[:, None]
    for h in range(s.H):
        np.testing.assert_allclose(r["out"][:, h], running, rtol=0, atol=1e-13)


def test_two_key_closed_form():
    """q=(1,0), k0=(0,0), k1=(1,0), scale 1: weights 1 and e at t=1."""
    q = torch.tensor([[[1.0, 0.0]], [[1.0, 0.0]]]).to(torch.bfloat16)   # [2,1,2]
    k = torch.tensor([[[0.0, 0.0]], [[1.0, 0.0]]]).to(torch.bfloat16)
    v = torch.tensor([[[2.0, -1.0]], [[-4.0, 0.5]]]).to(torch.bfloat16)
    ids = np.array([[[0, 1]], [[0, 1]]], dtype=np.int32)
    out = oracle.block_attention(q, np.array([0, 1]), k, v, ids, 1.0, block=1)
    e = math.e
    np.testing.assert_allclose(out[0, 0], [2.0, -1.0], atol=1e-15)
    np.testing.assert_allclose(out[1, 0], [(2.0 - 4.0 * e) / (1 + e), (-1.0 + 0.5 * e) / (1 + e)],
                               atol=1e-15)


def test_output_is_convex_combination_of_selected_values():
    s = synth.PREFILL_CONFIGS["tiny"]
    inp = synth.make_prefill_inputs(s)
    rows = synth.sample_rows(s.N, 40, seed=4)
    r = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                       block=s.block, top_k=s.top_k, scale=s.scale, rows=rows)
    v = inp["v"].double().numpy()
    for i, t in enumerate(rows):
        for h in range(s.H):
            g = h // (s.H // s.G)
            keys = [x for j in r["ids"][i, g] if j >= 0
                    for x in range(j * s.block, min((j + 1) * s.block, t + 1))]
            vals = v[keys, g]
            assert np.all(r["out"][i, h] >= vals.min(axis=0) - 1e-12)
            assert np.all(r["out"][i, h] <= vals.max(axis=0) + 1e-12)
