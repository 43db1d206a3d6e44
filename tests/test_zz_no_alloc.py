"""msa_decode_static: the decode step for callers that cannot allocate.

Some callers cannot call cudaMalloc at the point where they decode (their
device memory is reserved up front by another runtime, or the calling thread
must not enter the allocator).  msa_decode_static keeps its scratch in an array
compiled into the library instead of a caller workspace.  These checks call it
through the C ABI (ctypes, no binding helper) and compare it with msa_decode on
the same inputs, twice in a row, since every call reuses the same array.
This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from tests import parity

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def setup(cuda_device):
    import block_sparse_long_branch_b200 as msa
    lib = msa.load_library()
    s = synth.DecodeShape("static", seq_lens=(3000, 700, 128 * 9 + 5, 4096), H=32, G=4, d=128,
                          d_idx=128, top_k=8, needles_per_seq=(2, 1, 1, 2), seed=21)
    inp = synth.make_decode_inputs(s, device="cuda")
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, block=s.block, scale=s.scale)
    cu = inp["cu_seqlens"].cuda()
    ref_out, ref_ids = msa.msa_decode(cfg, inp["q"], inp["q_idx"], inp["k_cache"],
                                      inp["v_cache"], inp["k_idx_cache"], cu, max(s.seq_lens),
                                      ids_out=True)
    torch.cuda.synchronize()
    return msa, lib, s, inp, cfg, cu, ref_out, ref_ids


def _call_static(lib, s, inp, cfg, cu, out, ids):
    return lib.msa_decode_static(
        ctypes.byref(cfg), _ptr(inp["q"]), _ptr(inp["q_idx"]), _ptr(inp["k_cache"]),
        _ptr(inp["v_cache"]), _ptr(inp["k_idx_cache"]), _ptr(cu), s.B, max(s.seq_lens),
        s.total_len, _ptr(out), _ptr(ids), 1,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_decode_matches_workspace_decode_twice(setup):
    msa, lib, s, inp, cfg, cu, ref_out, ref_ids = setup
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        ids = torch.full_like(ref_ids, -7)
        st = _call_static(lib, s, inp, cfg, cu, out, ids)
        torch.cuda.synchronize()
        assert st == 0, msa.msa_status_string(st)
        assert torch.equal(ids, ref_ids)
        parity.check_output(out.float().cpu().numpy(), ref_out.double().cpu().numpy())


def test_static_decode_rejects_sizes_beyond_its_array(setup):
    msa, lib, s, inp, cfg, cu, ref_out, ref_ids = setup
    # 2^32 cached tokens need about 1 GiB of block scores: far beyond the fixed array
    st = lib.msa_decode_static(ctypes.byref(cfg), _ptr(inp["q"]), _ptr(inp["q_idx"]),
                               _ptr(inp["k_cache"]), _ptr(inp["v_cache"]),
                               _ptr(inp["k_idx_cache"]), _ptr(cu), s.B, max(s.seq_lens), 1 << 32,
                               _ptr(ref_out), None, 0, None)
    assert st == 3  # MSA_ERR_WORKSPACE, nothing launched
    assert np.isfinite(ref_out.float().cpu().numpy()).all()
