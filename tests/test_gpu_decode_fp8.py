"""GPU parity: the decode step with the quantised (e4m3) Index Branch.

The index-key cache is e4m3 with one fp32 scale per key row, the index query
e4m3 per row (msa_quantize_rows_fp8).  The quantiser's bytes and scales must
equal the oracle's exactly.  The selection is compared with the oracle's over
the dequantised values (ids equal except near-ties within the fp32
accumulation error of the tensor cores), and the attention output with the
fp64 oracle over the selected blocks (bf16 K/V, unchanged by the quantised
index).
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


def _quantize(msa, inp):
    q8, _ = msa.msa_quantize_rows_fp8(inp["q_idx"])
    k8, ks = msa.msa_quantize_rows_fp8(inp["k_idx_cache"])
    return q8, k8, ks


def test_row_quantizer_equals_oracle(msa):
    x = (torch.randn(5000, 128, device="cuda") * 3).to(torch.bfloat16)
    x[17] = 0
    x8, sc = msa.msa_quantize_rows_fp8(x)
    e8, es = oracle.quantize_rows_fp8(x.cpu())
    np.testing.assert_array_equal(sc.cpu().numpy(), es)
    np.testing.assert_array_equal(x8.cpu().numpy(), e8)


def _gather_blocks(inp, s0, L, blocks, s):
    kc = torch.zeros(len(blocks) * s.block, s.G, s.d, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for c, j in enumerate(blocks):
        r0, r1 = s0 + j * s.block, min(s0 + L, s0 + (j + 1) * s.block)
        kc[c * s.block:c * s.block + (r1 - r0)] = inp["k_cache"][r0:r1].cpu()
        vc[c * s.block:c * s.block + (r1 - r0)] = inp["v_cache"][r0:r1].cpu()
    return kc, vc


def _attend(inp, s, b, L, ids_b):
    """Oracle Main Branch of sequence b on the selection ids_b [G, k] (only the
    selected blocks' K/V rows are copied, stacked in ascending block order)."""
    s0 = int(inp["cu_seqlens"][b])
    used = sorted({int(j) for j in ids_b.ravel() if j >= 0})
    kc, vc = _gather_blocks(inp, s0, L, used, s)
    rm = {j: c for c, j in enumerate(used)}
    cids = np.vectorize(lambda j: rm[j] if j >= 0 else -1)(ids_b[None]).astype(np.int32)
    cpos = np.array([(len(used) - 1) * s.block + (L - 1) % s.block])
    return oracle.block_attention(oracle.as_bf16_bits(inp["q"][b:b + 1]), cpos, kc, vc, cids,
                                  s.scale, s.block)[0]


def _check(msa, s, inp):
    q8, k8, ks = _quantize(msa, inp)
    cfg = _cfg(msa, s)
    cu = inp["cu_seqlens"].cuda()
    total = inp["k_cache"].shape[0]
    ws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_DECODE, total, s.B), dtype=torch.uint8,
                     device="cuda")
    out, ids = msa.msa_decode_fp8_index(cfg, inp["q"], q8, inp["k_cache"], inp["v_cache"], k8, ks,
                                        cu, max(s.seq_lens), ids_out=True, workspace=ws)
    assert msa.msa_get_device_error(ws) == 0
    g_out, g_ids = out.float().cpu().numpy(), ids.cpu().numpy()
    q8h, k8h, ksh = q8.cpu().numpy(), k8.cpu().numpy(), ks.cpu().numpy()
    cu_h = inp["cu_seqlens"].tolist()
    n_ties = 0
    for b in range(s.B):
        s0, s1 = cu_h[b], cu_h[b + 1]
        L = s1 - s0
        nb = (L + s.block - 1) // s.block
        pos = np.array([L - 1], dtype=np.int64)
        pooled = oracle.pooled_scores_fp8_rows(q8h[b:b + 1], pos, k8h[s0:s1], ksh[s0:s1], s.block,
                                               nb)
        ref = oracle.select_blocks(pooled, pos, s.block, s.top_k)
        parity.check_id_rows_valid(g_ids[b:b + 1], pos, s.block, s.top_k)
        fin = pooled[np.isfinite(pooled)]
        tol = 1e-5 * float(np.abs(fin).max()) if fin.size else 0.0
        ties = parity.compare_ids(g_ids[b:b + 1], ref, pooled, pos, s.block, s.top_k, tol=tol)
        n_ties += len(ties)
        # the output against the oracle on the GPU's own selection (equal to the
        # oracle's except at listed near-ties)
        parity.check_output(g_out[b], _attend(inp, s, b, L, g_ids[b]))
    for (b, j, g) in inp["needles"]:
        assert j in g_ids[b, g], (b, j, g)
    return n_ties


def test_decode_fp8_small_mixed_lengths(msa):
    s = synth.DecodeShape("f8dec", seq_lens=(3000, 700, 128 * 9 + 5, 4096, 1, 130), H=32, G=4,
                          d=128, d_idx=128, top_k=8, needles_per_seq=(2, 1, 1, 2, 0, 0), seed=81)
    inp = synth.make_decode_inputs(s, device="cuda")
    assert _check(msa, s, inp) <= 2


def test_decode_fp8_full_config_every_query(msa):
    """16 x 256K + 1 x 1M caches, every one of the 17 queries against the oracle."""
    s = synth.DECODE_CONFIG
    inp = synth.make_decode_inputs(s, device="cuda")
    assert _check(msa, s, inp) <= 8


def test_decode_fp8_ties_go_to_lower_block(msa):
    """Codes of -1, 0 and 1 with unit scales: integer pooled scores, many exactly
    equal, so every rank decision between equal blocks is the lower-id rule."""
    s = synth.DecodeShape("f8tie", seq_lens=(5000, 2049), H=16, G=2, d=128, d_idx=128, top_k=12,
                          needles_per_seq=(0, 0), seed=83)
    inp = synth.make_decode_inputs(s, device="cuda")
    rng = np.random.default_rng(5)
    codes = np.array([0xB8, 0x00, 0x38], np.uint8)
    total = inp["k_cache"].shape[0]
    q8 = torch.from_numpy(codes[rng.integers(0, 3, (s.B, s.G, 128))]).cuda()
    k8 = torch.from_numpy(codes[rng.integers(0, 3, (total, 128))]).cuda()
    ks = torch.ones(total, dtype=torch.float32, device="cuda")
    cfg = _cfg(msa, s)
    out, ids = msa.msa_decode_fp8_index(cfg, inp["q"], q8, inp["k_cache"], inp["v_cache"], k8, ks,
                                        inp["cu_seqlens"].cuda(), max(s.seq_lens), ids_out=True)
    g_ids = ids.cpu().numpy()
    cu_h = inp["cu_seqlens"].tolist()
    for b in range(s.B):
        L = cu_h[b + 1] - cu_h[b]
        pos = np.array([L - 1])
        pooled = oracle.pooled_scores_fp8_rows(q8[b:b + 1].cpu().numpy(), pos,
                                               k8[cu_h[b]:cu_h[b + 1]].cpu().numpy(),
                                               np.ones(L, np.float32), s.block,
                                               (L + s.block - 1) // s.block)
        ref = oracle.select_blocks(pooled, pos, s.block, s.top_k)
        np.testing.assert_array_equal(g_ids[b], ref[0])  # integer sums are exact in fp32
