"""GPU parity: the block-alignment outputs of msa_prefill_block_alignment.

The expected values come from the oracle only: its pooled index scores of
every visible block and its per-slot partial softmax (lse) of the Main Branch
on the same selection, combined by oracle.block_alignment (head-mean
attention mass per slot; KL of that mass from the softmax of the slots'
scores).
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


def _expected(inp, s, ids):
    """Oracle block scores, head-mean block mass and KL for the given selection."""
    rows = np.arange(s.N)
    pooled = oracle.pooled_scores(oracle.as_bf16_bits(inp["q_idx"]), rows, inp["k_idx"], s.block,
                                  s.nb)
    _, lse, _ = oracle.block_attention(oracle.as_bf16_bits(inp["q"]), rows, inp["k"], inp["v"],
                                       ids, s.scale, s.block, partials=True)
    return oracle.block_alignment(pooled, ids, lse)


@pytest.mark.parametrize("d_idx", [128, 64])
def test_block_alignment_matches_oracle(msa, d_idx):
    s = synth.PrefillShape("align", N=4096 + 37, H=8, G=2, d=64, d_idx=d_idx, top_k=8,
                           n_needles=8, seed=51)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, scale=s.scale)
    out, ids, score, mass, kl = msa.msa_prefill_block_alignment(cfg, inp["q"], inp["k"], inp["v"],
                                                                inp["q_idx"], inp["k_idx"])
    torch.cuda.synchronize()
    # the prefill itself is untouched: same kernels, same result as msa_prefill
    ref_out, ref_ids = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                       inp["k_idx"], ids_out=True)
    assert torch.equal(ids, ref_ids)
    assert torch.equal(out, ref_out)
    g_ids = ids.cpu().numpy()
    e_score, e_mass, e_kl = _expected(inp, s, g_ids)
    g_score, g_mass, g_kl = score.cpu().numpy(), mass.cpu().numpy(), kl.cpu().numpy()
    filled = g_ids >= 0
    assert np.all(np.isneginf(g_score[~filled])) and np.all(g_mass[~filled] == 0)
    np.testing.assert_allclose(g_score[filled], e_score[filled], rtol=1e-4, atol=2e-3)
    np.testing.assert_allclose(g_mass, e_mass, atol=2e-3)
    np.testing.assert_allclose(g_mass.sum(axis=2), 1.0, atol=1e-4)
    np.testing.assert_allclose(g_kl, e_kl, rtol=1e-2, atol=1e-2)
