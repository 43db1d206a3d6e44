"""Pins for the oracle's quantised Index Branch (e4m3 index tensors).

The pages report the indexer moving from Q8KV8 to Q8KV4 in a later model
(dot-ai "MiniMax M3.1 Flashとは？428BのMoEモデルがウェイト公開", the passage
on the model card's quantisation) without a number format; the reading pinned
here is e4m3 values with one fp32 scale per index-query row and per 128-key
block of index keys.  The codec is checked against torch's float8_e4m3fn, the
quantiser against its defining properties, and the pooled score of quantised
inputs against a dense masked max and against the bf16 oracle on values both
represent exactly.
"""
import numpy as np
import pytest
import torch

import oracle


def test_decode_all_codes_equals_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    # fixed points of the format: max normal, one, min normal, min subnormal
    np.testing.assert_array_equal(oracle.e4m3_decode(np.array([0x7E, 0x38, 0x08, 0x01, 0x80],
                                                              np.uint8)),
                                  [448.0, 1.0, 2.0 ** -6, 2.0 ** -9, -0.0])


@pytest.mark.parametrize("seed", [0, 1])
def test_encode_equals_torch_round_to_nearest_even(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-10, 7, 100000))).astype(np.float32)
    x = np.clip(x, -448, 448)
    # exact midpoints between neighbouring codes, and both sides of them
    grid = oracle.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, np.float32(0)),
                        np.nextafter(mids, np.float32(1e9))])
    got = oracle.e4m3_encode(x)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, want)
    # a midpoint goes to the code with the even mantissa
    half = oracle.e4m3_encode(mids)
    assert np.all(half & 1 == 0)


def test_encode_saturates():
    big = np.array([448.0, 464.0, 1e6, -1e30, np.float32(3.4e38)], np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(big), [0x7E, 0x7E, 0x7E, 0xFE, 0x7E])


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def test_quantizer_scales_and_roundtrip():
    N, G, di = 300, 2, 128
    q = _bf16((N, G, di), 1, 3.0)
    k = _bf16((N, di), 2, 0.5)
    k[128:256] = 0  # an all-zero key block takes scale 1
    q8, k8, ks = oracle.quantize_index_fp8(q, k)
    assert q8.shape == (N, G, di) and k8.shape == (N, di) and ks.shape == (3,)
    kf = k.double().numpy()
    assert ks[1] == 1.0 and np.all(k8[128:256] == 0)
    for j in (0, 2):
        blk = kf[j * 128:(j + 1) * 128]
        assert ks[j] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448))
        # the largest magnitude of the block lands on +-448
        r, c = np.unravel_index(np.abs(blk).argmax(), blk.shape)
        assert (k8[j * 128 + r, c] & 0x7F) == 0x7E
        deq = oracle.e4m3_decode(k8[j * 128:(j + 1) * 128]) * ks[j]
        # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for normals,
        # absolute <= half the subnormal step otherwise
        err = np.abs(deq - blk)
        bound = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * ks[j]) * (1 + 1e-6)
        assert np.all(err <= bound)
    qd = oracle.e4m3_decode(q8)
    assert np.all(np.abs(qd).max(axis=2) == 448.0)


def _dense_pooled(qv, kv, block):
    N = qv.shape[0]
    s = np.einsum("tgc,sc->tgs", qv, kv)
    causal = np.arange(N)[None, :] > np.arange(N)[:, None]
    s = np.where(causal[:, None, :], -np.inf, s)
    nb = (N + block - 1) // block
    s = np.pad(s, ((0, 0), (0, 0), (0, nb * block - N)), constant_values=-np.inf)
    return s.reshape(N, s.shape[1], nb, block).max(axis=-1)


@pytest.mark.parametrize("N,block", [(70, 8), (64, 16), (33, 4)])
def test_pooled_fp8_equals_dense_masked_max(N, block):
    rng = np.random.default_rng(N)
    G, di = 2, 16
    q8 = rng.integers(0, 256, (N, G, di)).astype(np.uint8)
    k8 = rng.integers(0, 256, (N, di)).astype(np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0x38
    k8[(k8 & 0x7F) == 0x7F] = 0xB8
    nb = (N + block - 1) // block
    ks = np.exp2(rng.integers(-3, 4, nb)).astype(np.float32)
    got = oracle.pooled_scores_fp8(q8, np.arange(N), k8, ks, block, nb)
    kv = oracle.e4m3_decode(k8) * np.repeat(ks.astype(np.float64), block)[:N, None]
    want = _dense_pooled(oracle.e4m3_decode(q8), kv, block)
    # power-of-two scales and 3-bit mantissas: every product and sum is exact
    np.testing.assert_array_equal(got, want)


def test_pooled_fp8_equals_bf16_oracle_on_shared_values():
    """Unit scales: e4m3 values are bf16 values, so both oracles must agree."""
    N, G, di, block = 200, 3, 32, 16
    rng = np.random.default_rng(5)
    q8 = rng.integers(0, 0x7F, (N, G, di)).astype(np.uint8) | (rng.integers(0, 2, (N, G, di)) << 7).astype(np.uint8)
    k8 = rng.integers(0, 0x7F, (N, di)).astype(np.uint8)
    nb = (N + block - 1) // block
    rows = np.arange(N)
    got = oracle.pooled_scores_fp8(q8, rows, k8, np.ones(nb, np.float32), block, nb)
    qb = torch.from_numpy(oracle.e4m3_decode(q8)).to(torch.bfloat16)
    kb = torch.from_numpy(oracle.e4m3_decode(k8)).to(torch.bfloat16)
    assert torch.equal(qb.double(), torch.from_numpy(oracle.e4m3_decode(q8)))
    want = oracle.pooled_scores(qb, rows, kb, block, nb)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=0)


def test_quantised_selection_keeps_planted_block():
    """A key block aligned with the query stays on top after quantisation."""
    N, G, di, block, top_k = 1024, 1, 128, 128, 3
    q = _bf16((N, G, di), 7)
    k = _bf16((N, di), 8, 0.1)
    k[300] = (q[900, 0].float() * 4).to(torch.bfloat16)   # block 2
    q8, k8, ks = oracle.quantize_index_fp8(q, k)
    nb = N // block
    pooled = oracle.pooled_scores_fp8(q8, np.arange(N), k8, ks, block, nb)
    ids = oracle.select_blocks(pooled, np.arange(N), block, top_k)
    assert 2 in ids[900, 0]


def test_row_quantizer_equals_query_rows_of_index_quantizer():
    """Per-row quantisation of the decode tensors follows the same rule as the
    index-query rows of quantize_index_fp8 (pinned above): identical bytes."""
    q_idx = _bf16((300, 4, 128), 21, 2.5)
    k_idx = _bf16((300, 128), 22)
    q_idx[7, 2] = 0
    q8, _, _ = oracle.quantize_index_fp8(q_idx, k_idx)
    r8, rs = oracle.quantize_rows_fp8(q_idx)
    np.testing.assert_array_equal(r8, q8)
    assert rs.shape == (300, 4) and rs[7, 2] == 1.0
    # every non-zero row's largest magnitude lands on code +-448
    dec = oracle.e4m3_decode(r8)
    amax = np.abs(dec).max(axis=2)
    assert np.all((amax == 448.0) | ((rs == 1.0) & (amax == 0)))


def test_row_scaled_pooled_equals_block_scaled_when_scales_agree():
    """With each row's scale equal to its block's, the per-row pooled score is
    the pinned per-block one."""
    N, block = 700, 128
    q8, k8, ks = oracle.quantize_index_fp8(_bf16((N, 2, 128), 31), _bf16((N, 128), 32))
    rows = np.arange(0, N, 7)
    nb = (N + block - 1) // block
    a = oracle.pooled_scores_fp8(q8[rows], rows, k8, ks, block, nb)
    b = oracle.pooled_scores_fp8_rows(q8[rows], rows, k8, np.repeat(ks, block)[:N], block, nb)
    np.testing.assert_array_equal(a, b)


def test_row_scaled_pooled_equals_dense_masked_max():
    """Random codes and power-of-two row scales (every product and sum exact):
    the pooled score equals a dense masked score matrix reduced by a library max."""
    rng = np.random.default_rng(9)
    N, G, block = 300, 2, 32
    q8 = rng.integers(0, 0x7E, (N, G, 128)).astype(np.uint8) & 0xBF
    k8 = rng.integers(0, 0x7E, (N, 128)).astype(np.uint8) & 0xBF
    sc = (2.0 ** rng.integers(-3, 4, N)).astype(np.float32)
    rows = np.arange(N)
    nb = (N + block - 1) // block
    got = oracle.pooled_scores_fp8_rows(q8, rows, k8, sc, block, nb)
    qv = torch.from_numpy(oracle.e4m3_decode(q8))
    kv = torch.from_numpy(oracle.e4m3_decode(k8) * sc[:, None].astype(np.float64))
    dense = torch.einsum("tgc,sc->tgs", qv, kv)
    vis = torch.arange(N)[None, :] <= torch.arange(N)[:, None]
    dense = dense.masked_fill(~vis[:, None, :], -torch.inf)
    want = dense.view(N, G, nb, block).amax(dim=3).numpy() if N % block == 0 else None
    if want is None:
        pad = nb * block - N
        dense = torch.nn.functional.pad(dense, (0, pad), value=-torch.inf)
        want = dense.view(N, G, nb, block).amax(dim=3).numpy()
    np.testing.assert_array_equal(got, want)
