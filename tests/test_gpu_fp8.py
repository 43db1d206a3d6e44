"""GPU parity: the quantised (e4m3) Index Branch against the fp64 oracle.

The quantiser's bytes and scales must equal the oracle's quantiser exactly
(same fp32 division and rounding).  The selection runs on inputs quantised by
the oracle and is compared with the oracle's selection over the dequantised
values: ids equal except near-ties, which are checked to be ties within the
fp32 accumulation error of the tensor cores.
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


@pytest.mark.parametrize("N", [4096 + 37, 1000])
def test_quantizer_equals_oracle(msa, N):
    s = synth.PrefillShape("q8", N=N, H=8, G=4, d=64, d_idx=128, top_k=8, n_needles=4, seed=61)
    inp = synth.make_prefill_inputs(s, device="cuda")
    inp["k_idx"][256:384] = 0  # an all-zero key block
    inp["q_idx"][5] = 0        # all-zero query rows
    q8, k8, ks = msa.msa_quantize_index_fp8(_cfg(msa, s), inp["q_idx"], inp["k_idx"])
    torch.cuda.synchronize()
    e_q8, e_k8, e_ks = oracle.quantize_index_fp8(inp["q_idx"].cpu(), inp["k_idx"].cpu())
    np.testing.assert_array_equal(ks.cpu().numpy(), e_ks)
    np.testing.assert_array_equal(k8.cpu().numpy(), e_k8)
    np.testing.assert_array_equal(q8.cpu().numpy(), e_q8)


def _select_case(msa, s, rows=None):
    inp = synth.make_prefill_inputs(s, device="cpu")
    q8, k8, ks = oracle.quantize_index_fp8(inp["q_idx"], inp["k_idx"])
    cfg = _cfg(msa, s)
    ids = msa.msa_select_topk_fp8(cfg, torch.from_numpy(q8).cuda(), torch.from_numpy(k8).cuda(),
                                  torch.from_numpy(ks).cuda()).cpu().numpy()
    rows = np.arange(s.N) if rows is None else rows
    pooled = oracle.pooled_scores_fp8(q8[rows], rows, k8, ks, s.block, s.nb)
    ref = oracle.select_blocks(pooled, rows, s.block, s.top_k)
    g_ids = ids[rows]
    parity.check_id_rows_valid(g_ids, rows, s.block, s.top_k)
    fin = pooled[np.isfinite(pooled)]
    tol = 1e-5 * float(np.abs(fin).max())  # fp32 sums of exact fp8 products
    ties = parity.compare_ids(g_ids, ref, pooled, rows, s.block, s.top_k, tol=tol)
    return inp, ids, ties


@pytest.mark.parametrize("G,top_k", [(2, 16), (4, 8), (2, 24)])
def test_select_topk_fp8_matches_oracle(msa, G, top_k):
    s = synth.PrefillShape("f8", N=4096 + 77, H=2 * G, G=G, d=64, d_idx=128, top_k=top_k,
                           n_needles=8, seed=62 + G)
    inp, ids, ties = _select_case(msa, s)
    assert len(ties) <= 8, ties
    for (j, g, t) in inp["needles"]:
        assert j in ids[t, g]


@pytest.mark.parametrize("top_k", [5, 20])
def test_select_topk_fp8_ties_go_to_lower_block(msa, top_k):
    """Codes of -1, 0 and 1 with unit scales: integer pooled scores, many exactly
    equal, so every rank decision between equal blocks is the lower-id rule."""
    s = synth.PrefillShape("f8_ties", N=4096 + 5, H=4, G=2, d=64, d_idx=128, top_k=top_k)
    rng = np.random.default_rng(top_k)
    codes = np.array([0xB8, 0x00, 0x38], np.uint8)
    q8 = codes[rng.integers(0, 3, (s.N, s.G, 128))]
    k8 = codes[rng.integers(0, 3, (s.N, 128))]
    ks = np.ones(s.nb, np.float32)
    ids = msa.msa_select_topk_fp8(_cfg(msa, s), torch.from_numpy(q8).cuda(),
                                  torch.from_numpy(k8).cuda(),
                                  torch.from_numpy(ks).cuda()).cpu().numpy()
    rows = np.arange(s.N)
    pooled = oracle.pooled_scores_fp8(q8, rows, k8, ks, s.block, s.nb)
    ref = oracle.select_blocks(pooled, rows, s.block, s.top_k)
    np.testing.assert_array_equal(ids, ref)  # integer sums are exact in fp32


def test_select_topk_fp8_32k_sampled_rows(msa):
    s = synth.PREFILL_CONFIGS["prefill_32k"]
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.integers(0, s.N, 48), [0, 127, 128, s.N - 1]]))
    inp, ids, ties = _select_case(msa, s, rows)
    assert len(ties) <= 4, ties
    for (j, g, t) in inp["needles"]:
        assert j in ids[t, g]


def test_fp8_pipeline_keeps_bf16_selection_mostly(msa):
    """GPU quantiser -> GPU fp8 selection: needles survive, and most rows pick
    the same blocks as the bf16 selection (quantisation moves only near-ties)."""
    s = synth.PREFILL_CONFIGS["prefill_8k"]
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = _cfg(msa, s)
    q8, k8, ks = msa.msa_quantize_index_fp8(cfg, inp["q_idx"], inp["k_idx"])
    ids8 = msa.msa_select_topk_fp8(cfg, q8, k8, ks).cpu().numpy()
    ids16 = msa.msa_select_topk(cfg, inp["q_idx"], inp["k_idx"]).cpu().numpy()
    parity.check_id_rows_valid(ids8, np.arange(s.N), s.block, s.top_k)
    for (j, g, t) in inp["needles"]:
        assert j in ids8[t, g]
    overlap = np.mean([len(set(a) & set(b)) / len(set(b))
                       for a, b in zip(ids8.reshape(-1, s.top_k), ids16.reshape(-1, s.top_k))])
    assert overlap > 0.9, overlap


def test_fp8_rejects_other_index_dims(msa):
    s = synth.PrefillShape("f8_64", N=256, H=4, G=2, d=64, d_idx=64, top_k=4)
    cfg = _cfg(msa, s)
    q8 = torch.zeros((s.N, s.G, 64), dtype=torch.uint8, device="cuda")
    k8 = torch.zeros((s.N, 64), dtype=torch.uint8, device="cuda")
    ks = torch.ones((s.nb,), dtype=torch.float32, device="cuda")
    with pytest.raises(msa.MsaError):
        msa.msa_select_topk_fp8(cfg, q8, k8, ks)
    with pytest.raises(msa.MsaError):
        msa.msa_quantize_index_fp8(cfg, torch.zeros((s.N, s.G, 64), dtype=torch.bfloat16,
                                                    device="cuda"),
                                   torch.zeros((s.N, 64), dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("chunked", [False, True])
def test_prefill_fp8_index_matches_oracle(msa, chunked):
    """Whole prefill on the quantised Index Branch: the selection of the oracle
    on the dequantised index values, then its fp64 Main Branch; in one pass
    and with a workspace small enough to chunk the query axis."""
    s = synth.PrefillShape("pf8", N=4096 + 77, H=8, G=2, d=128, d_idx=128, top_k=16,
                           n_needles=8, seed=64)
    inp = synth.make_prefill_inputs(s, device="cpu")
    q8, k8, ks = oracle.quantize_index_fp8(inp["q_idx"], inp["k_idx"])
    cfg = _cfg(msa, s)
    ws_bytes = msa.msa_workspace_size(cfg, msa.OP_PREFILL, s.N)
    if chunked:
        ws_bytes = msa.msa_prefill_min_workspace(cfg, s.N) + (ws_bytes >> 3)
        assert msa.msa_prefill_chunk_tokens(cfg, s.N, ws_bytes) < s.N
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    dev = {n: inp[n].cuda() for n in ("q", "k", "v")}
    out, ids = msa.msa_prefill_fp8_index(cfg, dev["q"], dev["k"], dev["v"],
                                         torch.from_numpy(q8).cuda(),
                                         torch.from_numpy(k8).cuda(),
                                         torch.from_numpy(ks).cuda(), ids_out=True,
                                         workspace=ws)
    assert msa.msa_get_device_error(ws) == 0
    g_ids = ids.cpu().numpy()
    rows = np.arange(s.N)
    pooled = oracle.pooled_scores_fp8(q8, rows, k8, ks, s.block, s.nb)
    ref_ids = oracle.select_blocks(pooled, rows, s.block, s.top_k)
    parity.check_id_rows_valid(g_ids, rows, s.block, s.top_k)
    fin = pooled[np.isfinite(pooled)]
    ties = parity.compare_ids(g_ids, ref_ids, pooled, rows, s.block, s.top_k,
                              tol=1e-5 * float(np.abs(fin).max()))
    assert len(ties) <= 8, ties
    sel = g_ids if ties else ref_ids
    ref_out = oracle.block_attention(oracle.as_bf16_bits(inp["q"]), rows, inp["k"], inp["v"],
                                     sel, s.scale, s.block)
    parity.check_output(out.float().cpu().numpy(), ref_out)
    for (j, g, t) in inp["needles"]:
        assert j in g_ids[t, g]
