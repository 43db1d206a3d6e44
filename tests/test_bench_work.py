"""bench.py's algorithmic-work counts (the numerators of every roofline
fraction), checked against brute-force counts over small selections."""
import numpy as np
import torch

import bench
import oracle


def test_index_flops_counts_every_non_local_visible_key():
    for N, G, di in [(700, 2, 64), (129, 1, 128), (128, 4, 64), (1, 8, 128)]:
        keys = sum(128 * (t // 128) for t in range(N))  # whole blocks before the local one
        assert bench.index_flops(N, G, di) == 2.0 * di * G * keys
    # the 32K workload: 1.095e12, derived independently by hand
    assert abs(bench.index_flops(32768, 8, 128) - 1.095e12) / 1.095e12 < 1e-3


def test_dense_flops_is_causal_qk_plus_pv():
    N, H, d = 300, 4, 64
    pairs = sum(t + 1 for t in range(N))
    assert bench.dense_flops(N, H, d) == 4.0 * d * H * pairs


def _selection(N, G, k, seed):
    g = torch.Generator().manual_seed(seed)
    q_idx = torch.randn((N, G, 16), generator=g).to(torch.bfloat16)
    k_idx = torch.randn((N, 16), generator=g).to(torch.bfloat16)
    rows = np.arange(N)
    pooled = oracle.pooled_scores(q_idx, rows, k_idx, 128, (N + 127) // 128)
    return oracle.select_blocks(pooled, rows, 128, k)


def test_prefill_work_matches_a_per_slot_count():
    N, G, k, H, d = 1000, 2, 4, 8, 64
    ids = _selection(N, G, k, 1)
    w = bench.prefill_work(ids, H, d)
    HG = H // G
    keys = slots = 0
    for t in range(N):
        for g in range(G):
            for j in ids[t, g]:
                if j >= 0:
                    slots += 1
                    keys += sum(1 for s in range(128 * j, 128 * j + 128) if s <= t)
    assert w["slots"] == slots and w["pairs"] == slots * HG
    assert w["main_flops"] == 4.0 * d * HG * keys          # QK^T and PV per visible key
    assert w["main_bytes"] == slots * HG * (2 * d + 2 * d + 8)
    assert w["merge_bytes"] == slots * HG * (2 * d + 8) + N * H * 2 * d + N * G * k * 4
    assert w["selected_keys"] == keys / (N * G)


def test_decode_work_counts_scan_and_selected_keys():
    lens = [300, 129, 1000]
    G, H, d, di, k = 2, 8, 64, 64, 4
    ids = np.full((len(lens), G, k), -1, np.int32)
    ids[0, 0, :2] = [0, 2]
    ids[0, 1, :3] = [0, 1, 2]
    ids[1, :, :2] = [0, 1]
    ids[2, 0, :] = [1, 3, 5, 7]
    w = bench.decode_work(lens, H, G, d, di, ids)
    scan = sum(128 * ((L + 127) // 128 - 1) for L in lens)  # every non-local block
    assert w["idx_flops"] == 2.0 * di * G * scan
    assert w["idx_bytes"] == scan * di * 2 + len(lens) * G * di * 2
    keys = 0
    for b, L in enumerate(lens):
        for j in ids[b].ravel():
            if j >= 0:
                keys += sum(1 for s in range(128 * j, 128 * j + 128) if s < L)
    assert w["attn_bytes"] == keys * d * 2 * 2
    assert w["attn_flops"] == 4.0 * d * (H // G) * keys


def test_decode_work_e4m3_index_bytes():
    """e4m3 index cache: one byte per index value plus the row's 4-byte scale per
    scanned key, one byte per index-query value; the attention bytes unchanged."""
    lens = [300, 129, 1000]
    G, H, d, di, k = 2, 8, 64, 128, 4
    ids = np.full((len(lens), G, k), -1, np.int32)
    ids[:, :, 0] = 0
    w8 = bench.decode_work(lens, H, G, d, di, ids, fp8_index=True)
    w16 = bench.decode_work(lens, H, G, d, di, ids)
    scan = sum(128 * ((L + 127) // 128 - 1) for L in lens)
    assert w8["idx_bytes"] == scan * (di + 4) + len(lens) * G * di
    assert w8["attn_bytes"] == w16["attn_bytes"]
    assert w8["bytes"] == w8["idx_bytes"] + w8["attn_bytes"]
