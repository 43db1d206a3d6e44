"""The C-ABI library: it loads, exports every symbol include/msa.h declares, and
its host-side validation and workspace sizing behave as documented.  No call
here reaches a kernel, so no GPU is needed."""
import ctypes
import os
import re

import pytest

import block_sparse_long_branch_b200 as msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "msa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^MSA_API [^(]*?\b(msa_\w+)\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("msa_index_scores", "msa_select_topk", "msa_build_block_query_lists",
              "msa_prefill", "msa_decode", "msa_workspace_size", "msa_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = msa.load_library()
    for n in _declared():
        assert hasattr(lib, n), n
        assert hasattr(msa, n), n  # the binding keeps the C names


def _cfg(**kw):
    base = dict(H=64, G=8, d=128, d_idx=128, top_k=16)
    base.update(kw)
    return msa.config(base["H"], base["G"], base["d"], base["d_idx"], top_k=base["top_k"])


@pytest.mark.parametrize("kw,status", [
    (dict(H=6, G=4), 1),            # H % G
    (dict(d=96), 2),                # head dim
    (dict(d_idx=32), 2),            # index dim
    (dict(top_k=33), 2),            # k > 32
    (dict(top_k=0), 1),
    (dict(H=24, G=8), 2),           # H/G not a power of two
    (dict(H=12, G=3), 2),           # G not a power of two
])
def test_invalid_configs_are_rejected(kw, status):
    with pytest.raises(msa.MsaError) as e:
        msa.msa_workspace_size(_cfg(**kw), msa.OP_PREFILL, 4096)
    assert e.value.status == status


def test_block_size_must_be_128():
    cfg = _cfg()
    cfg.block_size = 64
    with pytest.raises(msa.MsaError) as e:
        msa.msa_workspace_size(cfg, msa.OP_PREFILL, 4096)
    assert e.value.status == 2


def test_token_limits():
    with pytest.raises(msa.MsaError):
        msa.msa_workspace_size(_cfg(), msa.OP_PREFILL, 0)
    with pytest.raises(msa.MsaError):
        msa.msa_workspace_size(_cfg(), msa.OP_PREFILL, 1 << 26)


def test_workspace_sizes_are_consistent():
    cfg = _cfg()
    full = msa.msa_workspace_size(cfg, msa.OP_PREFILL, 32768)
    small = msa.msa_prefill_min_workspace(cfg, 32768)
    assert 0 < small < full
    # partials dominate: rows * G * k * (H/G) * (2d + 4) bytes
    assert full >= 32768 * 8 * 16 * 8 * (2 * 128 + 4)
    assert msa.msa_workspace_size(cfg, msa.OP_SELECT_TOPK, 32768) == 256
    dec = msa.msa_workspace_size(cfg, msa.OP_DECODE, 5242880, 17)
    assert dec > (5242880 // 128) * 8 * 4


def test_null_pointers_rejected_before_any_launch():
    lib = msa.load_library()
    cfg = _cfg()
    st = lib.msa_prefill(ctypes.byref(cfg), None, None, None, None, None, 128, None, None, None,
                         0, None)
    assert st == 1
    st = lib.msa_select_topk(ctypes.byref(cfg), None, None, 128, None, None, 0, None)
    assert st == 1
    st = lib.msa_decode(ctypes.byref(cfg), None, None, None, None, None, None, 1, 1, None, None,
                        None, 0, None)
    assert st == 1


def test_misaligned_pointer_rejected():
    lib = msa.load_library()
    cfg = _cfg()
    p = ctypes.c_void_p(0x1000)
    bad = ctypes.c_void_p(0x1002)
    st = lib.msa_select_topk(ctypes.byref(cfg), bad, p, 128, p, p, 4096, None)
    assert st == 1


def test_missing_workspace_rejected():
    lib = msa.load_library()
    cfg = _cfg()
    p = ctypes.c_void_p(0x1000)
    st = lib.msa_select_topk(ctypes.byref(cfg), p, p, 128, p, None, 0, None)
    assert st == 3
    st = lib.msa_build_block_query_lists(ctypes.byref(cfg), p, 1024, p, p, p, 16, None)
    assert st == 3


def test_status_strings():
    for s in range(8):
        assert msa.msa_status_string(s)
    assert msa.msa_status_string(7) != msa.msa_status_string(99)


def test_selftest_arguments_checked_before_any_launch():
    lib = msa.load_library()
    p = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced: rejected first
    assert lib.msa_selftest_wait_timeout(None, 10_000, None) == 1
    assert lib.msa_selftest_wait_timeout(ctypes.c_void_p((1 << 20) + 4), 10_000, None) == 1
    assert lib.msa_selftest_wait_timeout(p, 999, None) == 1
    assert lib.msa_selftest_wait_timeout(p, 10 ** 9 + 1, None) == 1


def test_varlen_offsets_checked_before_any_launch():
    lib = msa.load_library()
    cfg = _cfg()
    p = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 21)

    def call(cu):
        arr = (ctypes.c_int64 * len(cu))(*cu)
        return lib.msa_prefill_varlen(ctypes.byref(cfg), p, p, p, p, p, arr, len(cu) - 1, p, None,
                                      ws, 1 << 30, None)
    assert call([1, 5]) == 1        # must start at 0
    assert call([0, 5, 3]) == 1     # decreasing offsets
    assert call([0, 0, 0]) == 1     # nothing to do
    assert lib.msa_prefill_varlen(ctypes.byref(cfg), p, p, p, p, p, None, 1, p, None, ws, 1 << 30,
                                  None) == 1


def test_fp8_entry_points_checked_before_any_launch():
    lib = msa.load_library()
    p = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 21)
    cfg = msa.config(8, 2, 128, 128, top_k=16)
    cfg64 = msa.config(8, 2, 128, 64, top_k=16)
    # the key scales are required
    assert lib.msa_prefill_fp8_index(ctypes.byref(cfg), p, p, p, p, p, None, 256, p, None, ws,
                                     1 << 30, None) == 1
    assert lib.msa_select_topk_fp8(ctypes.byref(cfg), p, p, None, 256, p, ws, 1 << 20,
                                   None) == 1
    assert lib.msa_quantize_index_fp8(ctypes.byref(cfg), p, p, 256, p, p, None, None) == 1
    # e4m3 index tensors only with d_idx = 128
    assert lib.msa_prefill_fp8_index(ctypes.byref(cfg64), p, p, p, p, p, p, 256, p, None, ws,
                                     1 << 30, None) == 2
    assert lib.msa_select_topk_fp8(ctypes.byref(cfg64), p, p, p, 256, p, ws, 1 << 20,
                                   None) == 2
    assert lib.msa_quantize_index_fp8(ctypes.byref(cfg64), p, p, 256, p, p, p, None) == 2
    # no tokens
    assert lib.msa_prefill_fp8_index(ctypes.byref(cfg), p, p, p, p, p, p, 0, p, None, ws,
                                     1 << 30, None) == 1


def test_mx_entry_points_checked_before_any_launch():
    lib = msa.load_library()
    p = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 21)
    cfg = msa.config(8, 2, 128, 128, top_k=16)
    # rows of a multiple of 32 values, a known element format, aligned pointers
    assert lib.msa_quantize_mx(p, 4, 48, msa.MX_E4M3, p, p, None) == 1
    assert lib.msa_quantize_mx(p, 4, 64, 7, p, p, None) == 1
    assert lib.msa_quantize_mx(p, -1, 64, msa.MX_E2M1, p, p, None) == 1
    assert lib.msa_quantize_mx(ctypes.c_void_p((1 << 20) + 8), 4, 64, msa.MX_E2M1, p, p,
                               None) == 1
    assert lib.msa_quantize_mx(p, 4, 64, msa.MX_E2M1, p, None, None) == 1
    assert lib.msa_quantize_mx(None, 0, 64, msa.MX_E2M1, None, None, None) == 0  # no rows
    # the three scale arrays are required
    assert lib.msa_prefill_q8kv4(ctypes.byref(cfg), p, p, p, None, p, p, p, p, 256, p, None, ws,
                                 1 << 30, None) == 1
    # the dequantised q, k, v must fit behind the prefill's own workspace
    need = msa.msa_workspace_size(cfg, msa.OP_PREFILL_Q8KV4, 256)
    full = msa.msa_workspace_size(cfg, msa.OP_PREFILL, 256)
    assert need - full == 256 * 8 * 128 * 2 + 2 * 256 * 2 * 128 * 2
    assert lib.msa_prefill_q8kv4(ctypes.byref(cfg), p, p, p, p, p, p, p, p, 256, p, None, ws,
                                 need - full, None) == 3  # MSA_ERR_WORKSPACE


def test_decode_heads_per_group_limit():
    """Decode tiles a group's heads in 8s, at most 16; prefill takes up to 2048/d."""
    lib = msa.load_library()
    cfg32 = msa.config(32, 1, 64, 64, top_k=4)   # 32 heads per group, d = 64
    n = ctypes.c_size_t(0)
    assert lib.msa_workspace_size(ctypes.byref(cfg32), msa.OP_DECODE, 1024, 2, ctypes.byref(n)) == 2
    assert lib.msa_workspace_size(ctypes.byref(cfg32), msa.OP_PREFILL, 1024, 0, ctypes.byref(n)) == 0
    p = ctypes.c_void_p(1 << 20)
    assert lib.msa_decode(ctypes.byref(cfg32), p, p, p, p, p, p, 2, 512, p, None, p, 1 << 30,
                          None) == 2
    cfg16 = msa.config(32, 2, 128, 128, top_k=4)  # 16 heads per group: supported
    assert lib.msa_workspace_size(ctypes.byref(cfg16), msa.OP_DECODE, 1024, 2, ctypes.byref(n)) == 0


def test_binding_offers_every_declared_function():
    """The Python layer has a function of the same name for every C entry point."""
    missing = [name for name in _declared() if not callable(getattr(msa, name, None))]
    assert not missing, missing
    assert set(_declared()) <= set(msa.__all__) | {"msa_last_launch_count"}
