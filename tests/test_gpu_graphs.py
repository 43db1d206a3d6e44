"""The library under CUDA graph capture: every call is stream-ordered and
allocation-free, so a prefill and a decode step captured once replay with the
same results as direct calls (new inputs copied into the captured buffers)."""
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


def test_prefill_and_decode_replay_from_a_graph(msa):
    s = synth.PrefillShape("g", N=3000, H=16, G=2, d=128, d_idx=128, top_k=8, n_needles=4,
                           seed=81)
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, scale=s.scale)
    inp = synth.make_prefill_inputs(s, device="cuda")
    ws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_PREFILL, s.N), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((s.N, s.H, s.d), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((s.N, s.G, s.top_k), dtype=torch.int32, device="cuda")

    dc = synth.DecodeShape("gd", seq_lens=(5000, 129, 20000), H=16, G=2, d=128, d_idx=128,
                           top_k=8, seed=82)
    dinp = synth.make_decode_inputs(dc, device="cuda")
    cu = dinp["cu_seqlens"].cuda()
    dws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_DECODE, dinp["k_cache"].shape[0], dc.B),
                      dtype=torch.uint8, device="cuda")
    dout = torch.empty((dc.B, dc.H, dc.d), dtype=torch.bfloat16, device="cuda")
    dids = torch.empty((dc.B, dc.G, dc.top_k), dtype=torch.int32, device="cuda")

    def step(stream):
        msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], out=out,
                        ids_out=ids, workspace=ws, stream=stream)
        msa.msa_decode(cfg, dinp["q"], dinp["q_idx"], dinp["k_cache"], dinp["v_cache"],
                       dinp["k_idx_cache"], cu, max(dc.seq_lens), out=dout, ids_out=dids,
                       workspace=dws, stream=stream)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(side)  # warm-up outside the capture (builds tensor maps, sets attributes)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = (out.clone(), ids.clone(), dout.clone(), dids.clone())

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream())
    # new queries in the captured buffers: the replay must follow them
    out.zero_()
    dout.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager[0]) and torch.equal(ids, eager[1])
    assert torch.equal(dout, eager[2]) and torch.equal(dids, eager[3])
    assert msa.msa_get_device_error(ws) == 0 and msa.msa_get_device_error(dws) == 0

    q_new = synth.make_prefill_inputs(s, device="cuda", seed=s.seed + 9)["q"]
    inp["q"].copy_(q_new)
    graph.replay()
    torch.cuda.synchronize()
    direct = msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"])
    assert torch.equal(out, direct)
    assert not torch.equal(out, eager[0])
    del graph
