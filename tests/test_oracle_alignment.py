"""Pins of oracle.block_alignment (the NEXT-2 block-alignment quantities).

The pages state only that the Index Branch's block-score distribution is
aligned by a KL divergence with the blocks that mattered to the Main Branch's
exact attention (ai-tool-zukan MiniMax MSA guide, section
"非微分的な選択をどう学習させるか（KLダイバージェンス）").  The function follows the
reading in its docstring; these tests fix it against things other than itself:
a hand-worked fixture, a two-slot closed form, KL = 0 on equal distributions,
invariances, and the block mass read off a dense masked softmax computed by a
library routine.
"""
import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _expr(x):
    return eval(x, {"__builtins__": {}}, {"log": math.log, "inf": math.inf})


def test_worked_example():
    with open(os.path.join(GOLDEN, "worked_example_alignment.json"), encoding="utf-8") as f:
        fx = json.load(f)
    ids = np.array(fx["ids"], dtype=np.int32).reshape(1, 1, -1)
    pooled = np.array([_expr(x) for x in fx["pooled"]]).reshape(1, 1, -1)
    lse = np.array([[_expr(x) for x in fx["lse_head0"]],
                    [_expr(x) for x in fx["lse_head1"]]]).reshape(1, 2, -1)
    score, mass, kl = oracle.block_alignment(pooled, ids, lse)
    np.testing.assert_array_equal(np.isneginf(score[0, 0]), [False, False, False, True])
    np.testing.assert_allclose(score[0, 0, :3], [_expr(x) for x in fx["expected_score"][:3]],
                               rtol=0, atol=1e-15)
    np.testing.assert_allclose(mass[0, 0], [_expr(x) for x in fx["expected_mass"]], rtol=0,
                               atol=1e-15)
    assert abs(kl[0, 0] - _expr(fx["expected_kl"])) < 1e-14


def test_two_slots_closed_form():
    """Two filled slots: p = (s(a), 1-s(a)), q = (s(b), 1-s(b)) with the
    logistic s, so KL is the binary relative entropy."""
    rng = np.random.default_rng(3)
    for _ in range(20):
        a, b = rng.normal(size=2) * 3
        pooled = np.array([[[b, 0.0]]])
        lse = np.array([[[a, 0.0]]])  # one head
        ids = np.array([[[0, 1]]], dtype=np.int32)
        _, mass, kl = oracle.block_alignment(pooled, ids, lse)
        pa = 1 / (1 + math.exp(-a))
        qb = 1 / (1 + math.exp(-b))
        want = pa * math.log(pa / qb) + (1 - pa) * math.log((1 - pa) / (1 - qb))
        np.testing.assert_allclose(mass[0, 0], [pa, 1 - pa], rtol=1e-12, atol=1e-15)
        # the closed form itself cancels in 1 - q at large |b|: relative 1e-10
        assert abs(kl[0, 0] - want) < 1e-10 * max(1.0, abs(want))


def test_kl_zero_when_distributions_agree_and_mass_sums_to_one():
    """Every head's lse equal to the scores plus a head constant makes the mass
    the softmax of the scores: KL = 0.  Masses always sum to 1."""
    rng = np.random.default_rng(5)
    n, G, HG, k, nb = 6, 2, 4, 5, 9
    ids = np.stack([np.sort(rng.choice(nb, size=k, replace=False)) for _ in range(n * G)])
    ids = ids.reshape(n, G, k).astype(np.int32)
    pooled = rng.normal(size=(n, G, nb)) * 2
    sc = np.take_along_axis(pooled, ids, axis=2)
    lse = np.repeat(sc, HG, axis=1) + rng.normal(size=(n, G * HG, 1)) * 5
    _, mass, kl = oracle.block_alignment(pooled, ids, lse)
    np.testing.assert_allclose(kl, 0.0, atol=1e-13)
    np.testing.assert_allclose(mass.sum(axis=2), 1.0, atol=1e-14)
    # a different main distribution gives a positive divergence
    lse2 = lse + rng.normal(size=lse.shape)
    _, mass2, kl2 = oracle.block_alignment(pooled, ids, lse2)
    assert (kl2 > 0).all()
    np.testing.assert_allclose(mass2.sum(axis=2), 1.0, atol=1e-14)


def test_shift_invariance_and_unselected_blocks_ignored():
    rng = np.random.default_rng(7)
    n, G, HG, k, nb = 4, 2, 2, 4, 8
    ids = np.stack([np.sort(rng.choice(nb, size=k, replace=False)) for _ in range(n * G)])
    ids = ids.reshape(n, G, k).astype(np.int32)
    ids[0, 0, 3] = -1  # an empty slot
    pooled = rng.normal(size=(n, G, nb))
    lse = rng.normal(size=(n, G * HG, k))
    s0, m0, k0 = oracle.block_alignment(pooled, ids, lse)
    s1, m1, k1 = oracle.block_alignment(pooled + 3.0, ids, lse - 7.0)
    np.testing.assert_allclose(m1, m0, rtol=1e-13)
    np.testing.assert_allclose(k1, k0, atol=1e-13)
    # unselected blocks' scores change nothing
    p2 = pooled.copy()
    mask = np.ones_like(p2, dtype=bool)
    for t in range(n):
        for g in range(G):
            mask[t, g, ids[t, g][ids[t, g] >= 0]] = False
    p2[mask] += 100.0
    s2, m2, k2 = oracle.block_alignment(p2, ids, lse)
    np.testing.assert_array_equal(s2, s0)
    np.testing.assert_array_equal(k2, k0)
    assert m0[0, 0, 3] == 0 and np.isneginf(s0[0, 0, 3])


def test_mass_equals_dense_masked_softmax_per_block():
    """The main-side mass of slot r is the attention weight that the exact
    softmax puts on block r's keys, averaged over the group's heads: read off
    a dense fp64 masked softmax (torch) and compared with the mass from the
    oracle's per-block log-sum-exp partials."""
    gen = torch.Generator().manual_seed(11)
    N, H, G, d, block, k = 40, 4, 2, 8, 4, 3
    q = torch.randn(N, H, d, generator=gen).to(torch.bfloat16)
    kk = torch.randn(N, G, d, generator=gen).to(torch.bfloat16)
    v = torch.randn(N, G, d, generator=gen).to(torch.bfloat16)
    q_idx = torch.randn(N, G, d, generator=gen).to(torch.bfloat16)
    k_idx = torch.randn(N, d, generator=gen).to(torch.bfloat16)
    scale = 0.3
    r = oracle.prefill(q, kk, v, q_idx, k_idx, block=block, top_k=k, scale=scale, partials=True)
    _, mass, _ = oracle.block_alignment(r["pooled"], r["ids"], r["lse"])
    qf, kf = q.double(), kk.double()
    HG = H // G
    for t in range(N):
        for h in range(H):
            g = h // HG
            logits = scale * (kf[:, g, :] @ qf[t, h, :])
            allowed = torch.zeros(N, dtype=torch.bool)
            for j in r["ids"][t, g]:
                if j >= 0:
                    allowed[j * block:(j + 1) * block] = True
            allowed[t + 1:] = False
            p = torch.softmax(logits.masked_fill(~allowed, -math.inf), dim=0)
            for slot, j in enumerate(r["ids"][t, g]):
                if j < 0:
                    continue
                share = float(p[j * block:(j + 1) * block].sum())
                # accumulate the head mean: compare per head via the partial lse
                lse = r["lse"][t, h, r["ids"][t, g] >= 0]
                own = math.exp(r["lse"][t, h, slot] - (lse.max() + math.log(
                    np.exp(lse - lse.max()).sum())))
                assert abs(own - share) < 1e-12, (t, h, slot)
    # and the oracle's mass is the mean of those shares over the group's heads
    for t in range(N):
        for g in range(G):
            for slot, j in enumerate(r["ids"][t, g]):
                if j < 0:
                    assert mass[t, g, slot] == 0
                    continue
                shares = []
                for h in range(g * HG, (g + 1) * HG):
                    logits = scale * (kf[:, g, :] @ qf[t, h, :])
                    allowed = torch.zeros(N, dtype=torch.bool)
                    for jj in r["ids"][t, g]:
                        if jj >= 0:
                            allowed[jj * block:(jj + 1) * block] = True
                    allowed[t + 1:] = False
                    p = torch.softmax(logits.masked_fill(~allowed, -math.inf), dim=0)
                    shares.append(float(p[j * block:(j + 1) * block].sum()))
                assert abs(mass[t, g, slot] - np.mean(shares)) < 1e-12
