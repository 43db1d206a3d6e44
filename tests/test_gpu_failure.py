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


def test_v_beyond_fp16_range_is_reported(msa):
    """The PV product runs in fp16: a V value beyond 65504 is saturated and
    recorded as 0x301 in the device error word; the prefill completes, other
    rows are unaffected and the next read finds the word cleared."""
    import oracle
    import synth
    from tests import parity
    s = synth.PrefillShape("vrange", N=512, H=8, G=2, d=64, d_idx=64, top_k=4, seed=71)
    inp = synth.make_prefill_inputs(s, device="cuda")
    inp["v"][300, 1, 5] = 1.0e5
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
