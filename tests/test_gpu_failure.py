"""Device-side failure detection without a GPU fault.

Every wait in the kernels is bounded: when it runs out, the kernel records a
code in the workspace's error word and returns.  An input value outside the
range a kernel computes in is recorded in the same word.  msa_selftest_wait_timeout
plants such a wait (an mbarrier that nothing arrives on) with a short limit;
the checks below read the code back, and then run real work on the same
context to show that it stayed usable.
"""
import time

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import block_sparse_long_branch_b200 as m
    m.load_library()
    return m


def test_planted_wait_times_out_and_reports(msa):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    msa.msa_selftest_wait_timeout(ws, 5_000_000)  # 5 ms
    code = msa.msa_get_device_error(ws)  # synchronises
    assert code == 0x1FE
    assert time.time() - t0 < 30.0
    # read-and-clear: a second read sees no error
    assert msa.msa_get_device_error(ws) == 0


def test_selftest_rejects_bad_arguments(msa):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for limit in (0, 999, 10 ** 9 + 1):
        with pytest.raises(msa.MsaError):
            msa.msa_selftest_wait_timeout(ws, limit)
    with pytest.raises(msa.MsaError):
        msa.msa_selftest_wait_timeout(ws[1:], 10_000)  # misaligned workspace


def test_context_usable_after_timeout(msa):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    msa.msa_selftest_wait_timeout(ws, 1_000_000)
    assert msa.msa_get_device_error(ws) == 0x1FE
    s = synth.PrefillShape("after", N=640, H=4, G=2, d=64, d_idx=64, top_k=4, seed=31)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, scale=s.scale)
    pws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_PREFILL, s.N), dtype=torch.uint8,
                      device="cuda")
    out, ids = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                               ids_out=True, workspace=pws)
    assert msa.msa_get_device_error(pws) == 0
    assert torch.isfinite(out.float()).all()
    assert (ids[:, :, 0] >= 0).all()


def test_v_beyond_fp16_range_is_computed(msa):
    """The PV product runs in fp16 on V scaled, per key block and group, by a
    power of two: values far beyond the fp16 range are computed like any other,
    with no error recorded.  Block 1 of group 0 is scaled by 300 (|v| up to
    about 1.3e3) and one value of block 2, group 1 is 1e5."""
    import oracle
    from tests import parity
    s = synth.PrefillShape("vrange", N=512, H=8, G=2, d=64, d_idx=64, top_k=4, seed=71)
    inp = synth.make_prefill_inputs(s, device="cuda")
    inp["v"][128:256, 0, :] = (inp["v"][128:256, 0, :].float() * 300.0).to(torch.bfloat16)
    inp["v"][300, 1, 5] = 1.0e5
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, scale=s.scale)
    ws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_PREFILL, s.N), dtype=torch.uint8,
                     device="cuda")
    out = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                          workspace=ws)
    assert msa.msa_get_device_error(ws) == 0
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], block=s.block,
                         top_k=s.top_k, scale=s.scale)
    got = out.float().cpu().numpy().astype(np.float64)
    want = ref["out"]
    assert np.isfinite(got).all()
    # the same weights on |v|: sum_s p_s |v_s|, the size of the terms each
    # output is summed from (the oracle on |V|)
    mag = oracle.prefill(inp["q"], inp["k"], inp["v"].abs(), inp["q_idx"], inp["k_idx"],
                         block=s.block, top_k=s.top_k, scale=s.scale)["out"]
    # outputs summed from ordinary values meet the usual bar; where large values
    # enter, fp16 P and fp16 partials add up to 2^-9 of the terms' size
    err = np.abs(got - want)
    bound = np.maximum(parity.OUT_MAX_ABS, parity.bf16_half_spacing(want) + parity.OUT_ARITH)
    bound = bound + np.where(mag > 4.0, 2.0 ** -9 * mag, 0.0)
    assert (err <= bound).all(), float((err - bound).max())
    assert np.abs(want).max() > 1.0e3  # the large values reached the outputs
    plain = mag <= 4.0
    assert plain.mean() > 0.5 and err[plain].max() <= parity.OUT_MAX_ABS


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_v_not_finite_is_reported(msa, bad):
    """A NaN or infinite V value is recorded as 0x301 in the device error word;
    the prefill completes, rows that cannot see that key are exact as usual,
    and the next read finds the word cleared."""
    import oracle
    from tests import parity
    s = synth.PrefillShape("vbad", N=512, H=8, G=2, d=64, d_idx=64, top_k=4, seed=71)
    inp = synth.make_prefill_inputs(s, device="cuda")
    inp["v"][300, 1, 5] = bad
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, scale=s.scale)
    ws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_PREFILL, s.N), dtype=torch.uint8,
                     device="cuda")
    out = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                          workspace=ws)
    assert msa.msa_get_device_error(ws) == 0x301
    assert msa.msa_get_device_error(ws) == 0
    # rows whose selection cannot reach key 300 (queries before it) are exact as usual
    rows = np.arange(0, 300)
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], block=s.block,
                         top_k=s.top_k, scale=s.scale, rows=rows)
    parity.check_output(out.float().cpu().numpy()[rows], ref["out"])
