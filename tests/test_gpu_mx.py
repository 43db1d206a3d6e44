"""GPU parity of the quantised Main Branch inputs ("Q8KV4", read as MX formats):
the quantiser bit for bit against the oracle's, and msa_prefill_q8kv4 against
the fp64 oracle run on the dequantised tensors."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import block_sparse_long_branch_b200 as m
    m.load_library()
    return m


def _edge_rows(d: int) -> torch.Tensor:
    """Rows whose blocks hit the format's edge cases: all zero, e2m1 and e4m3
    rounding ties, saturation, tiny and huge magnitudes, negative zero."""
    rows = []
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    r = np.zeros(d)
    rows.append(r)
    r = np.resize(np.concatenate([mids, -mids]), d) * 2.0 ** -3
    rows.append(r)                      # e2m1 ties at scale 2^-3
    r = np.resize(np.array([448.0, 464.0, 480.0, 1.0, -0.0, 3.0, 7.0, 9.0]), d)
    rows.append(r)                      # e4m3: saturation and ties in the top binade
    r = np.resize(np.array([2.0 ** -133, 2.0 ** -126, 1e-30, -1e-35]), d)
    rows.append(r)                      # subnormal and tiny blocks
    r = np.resize(np.array([3.0e38, -1.0e38, 1.0, 2.0 ** 100]), d)
    rows.append(r)                      # the top of the bf16 range
    return torch.from_numpy(np.stack(rows).astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_mx_matches_oracle(msa, fmt):
    d = 128
    g = torch.Generator().manual_seed(41 + fmt)
    x = torch.randn((300, d), generator=g) * torch.exp2(torch.randint(-20, 20, (300, 1),
                                                                      generator=g).float())
    x = torch.cat([x.to(torch.bfloat16), _edge_rows(d)]).cuda()
    codes, scales = msa.msa_quantize_mx(x, fmt)
    want_c, want_s = oracle.mx_quantize(x.cpu(), fmt)
    if fmt == msa.MX_E2M1:
        want_c = oracle.pack_e2m1(want_c)
    assert np.array_equal(scales.cpu().numpy(), want_s)
    assert np.array_equal(codes.cpu().numpy(), want_c)


def _quantised_inputs(msa, inp):
    q8, qs = msa.msa_quantize_mx(inp["q"], msa.MX_E4M3)
    k4, ks = msa.msa_quantize_mx(inp["k"], msa.MX_E2M1)
    v4, vs = msa.msa_quantize_mx(inp["v"], msa.MX_E2M1)
    return q8, qs, k4, ks, v4, vs


def _dequantised(codes, scales, fmt):
    c = codes.cpu().numpy()
    if fmt == oracle.MX_E2M1:
        c = oracle.unpack_e2m1(c)
    vals = oracle.mx_dequantize(c, scales.cpu().numpy(), fmt)
    return torch.from_numpy(oracle.f64_to_bf16_bits(vals).view(np.int16)).view(torch.bfloat16)


def _check(msa, s, inp, rows):
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, block=s.block, scale=s.scale)
    q8, qs, k4, ks, v4, vs = _quantised_inputs(msa, inp)
    ws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_PREFILL_Q8KV4, s.N), dtype=torch.uint8,
                     device="cuda")
    out, ids = msa.msa_prefill_q8kv4(cfg, q8, qs, k4, ks, v4, vs, inp["q_idx"], inp["k_idx"],
                                     ids_out=True, workspace=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    if rows is None:
        qd = _dequantised(q8, qs, oracle.MX_E4M3)
    else:  # only the sampled query rows are needed (and dequantised)
        rows = np.asarray(rows)
        idx = torch.from_numpy(rows).cuda()
        qd = torch.zeros((s.N, s.H, s.d), dtype=torch.bfloat16)
        qd[torch.from_numpy(rows)] = _dequantised(q8[idx], qs[idx], oracle.MX_E4M3)
    kd = _dequantised(k4, ks, oracle.MX_E2M1)
    vd = _dequantised(v4, vs, oracle.MX_E2M1)
    ref = oracle.prefill(qd, kd, vd, inp["q_idx"], inp["k_idx"], block=s.block, top_k=s.top_k,
                         scale=s.scale, rows=rows)
    rows = ref["rows"]
    g_ids = ids.cpu().numpy()[rows]
    parity.check_id_rows_valid(g_ids, rows, s.block, s.top_k)
    ties = parity.compare_ids(g_ids, ref["ids"], ref["pooled"], rows, s.block, s.top_k)
    ref_out = ref["out"]
    if ties:
        ref_out = oracle.block_attention(oracle.as_bf16_bits(qd)[rows], rows, kd, vd, g_ids,
                                         s.scale, s.block)
    parity.check_output(out.float().cpu().numpy()[rows], ref_out)
    # the same selection as the bf16 prefill: the index tensors are not quantised
    return out


@pytest.mark.parametrize("rows,d", [(1, 32), (3, 64), (1000, 96)])
def test_quantize_mx_small_shapes(msa, rows, d):
    g = torch.Generator().manual_seed(rows + d)
    x = (torch.randn((rows, d), generator=g) * 5.0).to(torch.bfloat16).cuda()
    for fmt in (msa.MX_E4M3, msa.MX_E2M1):
        codes, scales = msa.msa_quantize_mx(x, fmt)
        want_c, want_s = oracle.mx_quantize(x.cpu(), fmt)
        if fmt == msa.MX_E2M1:
            want_c = oracle.pack_e2m1(want_c)
        assert np.array_equal(scales.cpu().numpy(), want_s)
        assert np.array_equal(codes.cpu().numpy(), want_c)


def test_prefill_q8kv4_chunked_equals_one_shot(msa):
    """A workspace that holds only part of the query axis: the prefill runs in
    query chunks behind the dequantised tensors and gives the same bytes."""
    s = synth.PrefillShape("mxc", N=2000, H=16, G=2, d=128, d_idx=128, top_k=8, n_needles=2,
                           seed=77)
    inp = synth.make_prefill_inputs(s, device="cuda")
    cfg = msa.config(s.H, s.G, s.d, s.d_idx, top_k=s.top_k, block=s.block, scale=s.scale)
    q8, qs, k4, ks, v4, vs = _quantised_inputs(msa, inp)
    full = msa.msa_workspace_size(cfg, msa.OP_PREFILL_Q8KV4, s.N)
    dq = full - msa.msa_workspace_size(cfg, msa.OP_PREFILL, s.N)
    small = msa.msa_prefill_min_workspace(cfg, s.N) + dq + 4096
    outs = []
    for size in (full, small):
        ws = torch.empty(size, dtype=torch.uint8, device="cuda")
        out, ids = msa.msa_prefill_q8kv4(cfg, q8, qs, k4, ks, v4, vs, inp["q_idx"], inp["k_idx"],
                                         ids_out=True, workspace=ws)
        torch.cuda.synchronize()
        assert msa.msa_get_device_error(ws) == 0
        outs.append((out.clone(), ids.clone()))
    assert msa.msa_prefill_chunk_tokens(cfg, s.N, small - dq, ids_returned=True) < s.N
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_prefill_q8kv4_tiny_all_rows(msa):
    s = synth.PREFILL_CONFIGS["tiny"]
    inp = synth.make_prefill_inputs(s, device="cuda")
    _check(msa, s, inp, rows=None)


@pytest.mark.parametrize("N,H,G,d,k", [(1000, 16, 2, 128, 16), (777, 32, 4, 64, 8)])
def test_prefill_q8kv4_ragged(msa, N, H, G, d, k):
    s = synth.PrefillShape("mx", N=N, H=H, G=G, d=d, d_idx=128, top_k=k, n_needles=2,
                           seed=N + 3 * H)
    inp = synth.make_prefill_inputs(s, device="cuda")
    _check(msa, s, inp, rows=None)


def test_prefill_q8kv4_32k_sampled_rows(msa):
    s = synth.PREFILL_CONFIGS["prefill_32k"]
    inp = synth.make_prefill_inputs(s, device="cuda")
    rows = synth.sample_rows(s.N, 48, seed=9)
    out = _check(msa, s, inp, rows=rows)
    assert torch.isfinite(out.float()).all()
