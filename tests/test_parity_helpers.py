"""The comparison helpers' own arithmetic: bf16's half-spacing at a value, checked
against torch's bf16 neighbours, and the output bound built from it."""
import numpy as np
import torch

from tests import parity


def test_bf16_half_spacing_equals_torch_neighbour_gap():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-8, 6, 20000))).astype(np.float32)
    b = torch.from_numpy(np.abs(x)).to(torch.bfloat16)
    b = b[(b.float() > 0) & torch.isfinite(b.float())]
    # the next bf16 value above a positive one: its bit pattern plus one
    up = (b.view(torch.int16) + 1).view(torch.bfloat16)
    gap = (up.double() - b.double()).numpy()
    np.testing.assert_array_equal(parity.bf16_half_spacing(b.double().numpy()), gap / 2)


def test_output_bound_is_the_stated_one_below_four():
    ref = np.array([0.1, 1.0, 2.0, 3.999, 4.0, 5.0, 9.0])
    bound = np.maximum(parity.OUT_MAX_ABS, parity.bf16_half_spacing(ref) + parity.OUT_ARITH)
    np.testing.assert_allclose(bound[:4], parity.OUT_MAX_ABS)
    assert np.all(bound[4:] > parity.bf16_half_spacing(ref[4:]))
