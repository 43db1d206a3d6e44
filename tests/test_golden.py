"""Hand-worked examples (tests/golden/*.json) run through the oracle.

The pages print no numeric worked example, so these fixtures are small cases
whose answers were derived by hand from the definitions the fixtures cite.
"""
import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)


def _closed_form(expr):
    return eval(expr, {"__builtins__": {}}, {"e": math.e})  # expressions in e only


def _index_inputs(fx):
    c = fx["config"]
    N, di = c["N"], c["d_idx"]
    q_idx = torch.tensor(fx["q_idx"] * N, dtype=torch.float32).view(N, 1, di)
    k_idx = torch.zeros(N, di)
    k_idx[:, 0] = torch.tensor(fx["k_idx_first_component"])
    return q_idx.to(torch.bfloat16), k_idx.to(torch.bfloat16)


def test_worked_example_selection_and_output():
    fx = _load("worked_example_block2.json")
    c = fx["config"]
    N, block, H, d = c["N"], c["block"], c["H"], c["d"]
    q_idx, k_idx = _index_inputs(fx)
    q = torch.tensor(fx["q_per_head"], dtype=torch.float32)[None].expand(N, H, d)
    k = torch.zeros(N, 1, d)
    k[:, 0, 0] = torch.tensor(fx["k_first_component"], dtype=torch.float32)
    v = torch.tensor(fx["v"], dtype=torch.float32).view(N, 1, d)
    r = oracle.prefill(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16),
                       q_idx, k_idx, block=block, top_k=c["top_k"], scale=c["scale"])
    np.testing.assert_array_equal(r["ids"][:, 0], np.array(fx["expected_ids"]))
    want0 = [_closed_form(x) for x in fx["expected_out_head0_x"]]
    want1 = [_closed_form(x) for x in fx["expected_out_head1_x"]]
    np.testing.assert_allclose(r["out"][:, 0, 0], want0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(r["out"][:, 1, 0], want1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(r["out"][:, :, 1], 1.0, rtol=0, atol=1e-15)


def test_worked_example_tie_goes_to_lower_block():
    fx = _load("worked_example_tie.json")
    c = fx["config"]
    q_idx, k_idx = _index_inputs(fx)
    rows = np.arange(c["N"])
    pooled = oracle.pooled_scores(q_idx, rows, k_idx, c["block"], c["N"] // c["block"])
    ids = oracle.select_blocks(pooled, rows, c["block"], c["top_k"])
    np.testing.assert_array_equal(ids[:, 0], np.array(fx["expected_ids"]))
