"""The seeded input generator: deterministic, right shapes, needles in range."""
import numpy as np
import torch

import synth


def test_prefill_inputs_are_deterministic_and_shaped():
    s = synth.PrefillShape("x", N=512, H=4, G=2, d=16, d_idx=8, block=64, n_needles=3, seed=9)
    a = synth.make_prefill_inputs(s)
    b = synth.make_prefill_inputs(s)
    for key, shape in [("q", (512, 4, 16)), ("k", (512, 2, 16)), ("v", (512, 2, 16)),
                       ("q_idx", (512, 2, 8)), ("k_idx", (512, 8))]:
        assert a[key].shape == shape and a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
    assert a["needles"] == b["needles"] and len(a["needles"]) == 3
    for (j, g, t) in a["needles"]:
        assert 0 <= j <= s.nb - 2 and 0 <= g < s.G and (j + 1) * s.block <= t < s.N
    c = synth.make_prefill_inputs(s, seed=10)
    assert not torch.equal(a["q"], c["q"])


def test_unit_variance():
    s = synth.PrefillShape("x", N=4096, H=8, G=2, d=64, d_idx=64, seed=3)
    a = synth.make_prefill_inputs(s)
    x = a["q"].double()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1) < 0.01


def test_decode_inputs_layout():
    s = synth.DecodeShape("d", seq_lens=(300, 128, 1000), H=4, G=2, d=16, d_idx=8,
                          needles_per_seq=(2, 0, 3), seed=4)
    a = synth.make_decode_inputs(s)
    assert a["cu_seqlens"].tolist() == [0, 300, 428, 1428]
    assert a["k_cache"].shape == (1428, 2, 16) and a["k_idx_cache"].shape == (1428, 8)
    assert a["q"].shape == (3, 4, 16) and a["q_idx"].shape == (3, 2, 8)
    assert len(a["needles"]) == 5


def test_sample_rows_cover_edges():
    rows = synth.sample_rows(32768, 100, seed=1)
    for r in (0, 1, 127, 128, 32767):
        assert r in rows
    assert np.all(np.diff(rows) > 0)
