"""B200 (sm_100a) MiniMax Sparse Attention hot path -- Python binding.

Thin ctypes marshalling over ``libmsa_b200.so`` (C ABI in ``include/msa.h``).
PyTorch provides device memory and the current CUDA stream; every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback: if
the library is missing or no CUDA device is present, the calls raise.

Function names mirror the C ABI: ``msa_index_scores``, ``msa_select_topk``,
``msa_build_block_query_lists``, ``msa_prefill``, ``msa_decode``,
``msa_workspace_size``, ``msa_get_device_error``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "MsaConfig", "MsaError", "config", "library_path", "load_library",
    "OP_SELECT_TOPK", "OP_BLOCK_QUERY_LISTS", "OP_PREFILL", "OP_DECODE",
    "msa_workspace_size", "msa_prefill_min_workspace", "msa_prefill_chunk_tokens",
    "msa_index_scores", "msa_select_topk", "msa_quantize_index_fp8", "msa_select_topk_fp8",
    "msa_build_block_query_lists", "msa_prefill", "msa_decode", "msa_get_device_error",
    "msa_status_string", "msa_last_launch_count", "msa_set_phase_events", "msa_decode_static",
    "msa_selftest_wait_timeout", "msa_prefill_varlen", "msa_prefill_block_alignment",
    "msa_prefill_fp8_index", "msa_prefill_varlen_workspace_size", "msa_decode_fp8_index",
    "msa_quantize_rows_fp8", "OP_PREFILL_Q8KV4", "MX_E4M3", "MX_E2M1", "msa_quantize_mx",
    "msa_prefill_q8kv4",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmsa_b200.so")

OP_SELECT_TOPK = 0
OP_BLOCK_QUERY_LISTS = 1
OP_PREFILL = 2
OP_DECODE = 3
OP_PREFILL_Q8KV4 = 4
MX_E4M3, MX_E2M1 = 0, 1

STATUS_NAMES = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED",
                3: "MSA_ERR_WORKSPACE", 4: "MSA_ERR_CUDA", 5: "MSA_ERR_DEVICE_TIMEOUT",
                6: "MSA_ERR_DEVICE_INDEX", 7: "MSA_ERR_DEVICE_RANGE"}


class MsaConfig(ctypes.Structure):
    """Mirror of ``msa_config_t``."""

    _fields_ = [("num_heads", ctypes.c_int32), ("num_groups", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("index_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]

    def __repr__(self):
        return (f"MsaConfig(H={self.num_heads}, G={self.num_groups}, d={self.head_dim}, "
                f"d_idx={self.index_dim}, block={self.block_size}, k={self.top_k}, "
                f"scale={self.softmax_scale:.6g})")


class MsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def config(H: int, G: int, d: int, d_idx: int, top_k: int = 16, block: int = 128,
           scale: Optional[float] = None) -> MsaConfig:
    return MsaConfig(H, G, d, d_idx, block, top_k, 1.0 / math.sqrt(d) if scale is None else scale)


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the in-tree library (built by ``build.py``); raise if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    from . import build as _build
    if not _build.is_current():
        # sources changed since the last build: rebuild in-tree (nvcc, sm_100a)
        _build.build()
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libmsa_b200.so not built ({_LIB_PATH}); run "
                           "block_sparse_long_branch_b200/build.py")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    C = ctypes.POINTER(MsaConfig)
    lib.msa_workspace_size.argtypes = [C, ctypes.c_int, I64, I32, ctypes.POINTER(SZ)]
    lib.msa_prefill_min_workspace.argtypes = [C, I64, ctypes.POINTER(SZ)]
    lib.msa_prefill_chunk_tokens.argtypes = [C, I64, SZ, I32, ctypes.POINTER(I64)]
    lib.msa_index_scores.argtypes = [C, P, P, I64, I64, I64, P, P]
    lib.msa_select_topk.argtypes = [C, P, P, I64, P, P, SZ, P]
    lib.msa_quantize_index_fp8.argtypes = [C, P, P, I64, P, P, P, P]
    lib.msa_select_topk_fp8.argtypes = [C, P, P, P, I64, P, P, SZ, P]
    lib.msa_build_block_query_lists.argtypes = [C, P, I64, P, P, P, SZ, P]
    lib.msa_prefill.argtypes = [C, P, P, P, P, P, I64, P, P, P, SZ, P]
    lib.msa_prefill_varlen.argtypes = [C, P, P, P, P, P, P, I32, P, P, P, SZ, P]
    lib.msa_prefill_varlen_workspace_size.argtypes = [C, P, I32, ctypes.POINTER(SZ)]
    lib.msa_prefill_fp8_index.argtypes = [C, P, P, P, P, P, P, I64, P, P, P, SZ, P]
    lib.msa_prefill_block_alignment.argtypes = [C, P, P, P, P, P, I64, P, P, P, P, P, P, SZ, P]
    lib.msa_decode.argtypes = [C, P, P, P, P, P, P, I32, I64, P, P, P, SZ, P]
    lib.msa_decode_static.argtypes = [C, P, P, P, P, P, P, I32, I64, I64, P, P, I32, P]
    lib.msa_decode_fp8_index.argtypes = [C, P, P, P, P, P, P, P, I32, I64, P, P, P, SZ, P]
    lib.msa_quantize_rows_fp8.argtypes = [P, I64, P, P, P]
    lib.msa_quantize_mx.argtypes = [P, I64, I32, I32, P, P, P]
    lib.msa_prefill_q8kv4.argtypes = [C, P, P, P, P, P, P, P, P, I64, P, P, P, SZ, P]
    lib.msa_get_device_error.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    lib.msa_selftest_wait_timeout.argtypes = [P, ctypes.c_uint64, P]
    lib.msa_status_string.argtypes = [ctypes.c_int]
    lib.msa_status_string.restype = ctypes.c_char_p
    lib.msa_set_phase_events.argtypes = [P, I32]
    lib.msa_set_phase_events.restype = ctypes.c_int
    lib.msa_last_launch_count.argtypes = []
    lib.msa_last_launch_count.restype = I32
    for name in ("msa_workspace_size", "msa_prefill_min_workspace", "msa_prefill_chunk_tokens",
                 "msa_index_scores",
                 "msa_select_topk", "msa_quantize_index_fp8", "msa_select_topk_fp8",
                 "msa_build_block_query_lists", "msa_prefill",
                 "msa_prefill_varlen", "msa_prefill_varlen_workspace_size",
                 "msa_prefill_block_alignment", "msa_prefill_fp8_index",
                 "msa_quantize_mx", "msa_prefill_q8kv4",
                 "msa_decode",
                 "msa_decode_static", "msa_get_device_error", "msa_selftest_wait_timeout"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise MsaError(status, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, dtype, name: str, shape=None) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def msa_status_string(status: int) -> str:
    return load_library().msa_status_string(status).decode()


def msa_last_launch_count() -> int:
    return int(load_library().msa_last_launch_count())


def msa_workspace_size(cfg: MsaConfig, op: int, n_tokens: int, batch: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().msa_workspace_size(ctypes.byref(cfg), op, n_tokens, batch,
                                             ctypes.byref(out)), "msa_workspace_size")
    return int(out.value)


def msa_prefill_min_workspace(cfg: MsaConfig, N: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().msa_prefill_min_workspace(ctypes.byref(cfg), N, ctypes.byref(out)),
           "msa_prefill_min_workspace")
    return int(out.value)


def msa_prefill_chunk_tokens(cfg: MsaConfig, N: int, ws_bytes: int,
                             ids_returned: bool = True) -> int:
    """Query rows per chunk that msa_prefill uses with ``ws_bytes`` of workspace."""
    out = ctypes.c_int64(0)
    _check(load_library().msa_prefill_chunk_tokens(ctypes.byref(cfg), N, ws_bytes,
                                                   1 if ids_returned else 0, ctypes.byref(out)),
           "msa_prefill_chunk_tokens")
    return int(out.value)


def _workspace(ws: Optional[torch.Tensor], nbytes: int, device) -> torch.Tensor:
    if ws is None:
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    if ws.dtype != torch.uint8 or not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 CUDA tensor")
    return ws


def msa_index_scores(cfg: MsaConfig, q_idx: torch.Tensor, k_idx: torch.Tensor,
                     row_begin: int = 0, row_count: Optional[int] = None,
                     scores: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Pooled Index Branch scores [rows, G, nb] (fp32, -inf where invisible)."""
    lib = load_library()
    N = q_idx.shape[0]
    G, di = cfg.num_groups, cfg.index_dim
    nb = (N + cfg.block_size - 1) // cfg.block_size
    row_count = N - row_begin if row_count is None else row_count
    if scores is None:
        scores = torch.empty((row_count, G, nb), dtype=torch.float32, device=q_idx.device)
    st = lib.msa_index_scores(ctypes.byref(cfg), _dev(q_idx, torch.bfloat16, "q_idx", (N, G, di)),
                              _dev(k_idx, torch.bfloat16, "k_idx", (N, di)), N, row_begin,
                              row_count, _dev(scores, torch.float32, "scores", (row_count, G, nb)),
                              _stream(stream))
    _check(st, "msa_index_scores")
    return scores


def msa_select_topk(cfg: MsaConfig, q_idx: torch.Tensor, k_idx: torch.Tensor,
                    ids: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Forced-local top-k block ids [N, G, k] (int32, ascending, -1 padded)."""
    lib = load_library()
    N = q_idx.shape[0]
    G, di, k = cfg.num_groups, cfg.index_dim, cfg.top_k
    if ids is None:
        ids = torch.empty((N, G, k), dtype=torch.int32, device=q_idx.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_SELECT_TOPK, N), q_idx.device)
    st = lib.msa_select_topk(ctypes.byref(cfg), _dev(q_idx, torch.bfloat16, "q_idx", (N, G, di)),
                             _dev(k_idx, torch.bfloat16, "k_idx", (N, di)), N,
                             _dev(ids, torch.int32, "ids", (N, G, k)), _dev(ws, torch.uint8, "ws"),
                             ws.numel(), _stream(stream))
    _check(st, "msa_select_topk")
    return ids


def msa_quantize_index_fp8(cfg: MsaConfig, q_idx: torch.Tensor, k_idx: torch.Tensor,
                           stream=None):
    """(q_idx [N,G,128], k_idx [N,128] bf16) -> (q_idx8, k_idx8 uint8 e4m3 bytes,
    k_scale [ceil(N/128)] float32)."""
    lib = load_library()
    N = q_idx.shape[0]
    G, di = cfg.num_groups, cfg.index_dim
    dev = q_idx.device
    q8 = torch.empty((N, G, di), dtype=torch.uint8, device=dev)
    k8 = torch.empty((N, di), dtype=torch.uint8, device=dev)
    ks = torch.empty(((N + cfg.block_size - 1) // cfg.block_size,), dtype=torch.float32,
                     device=dev)
    st = lib.msa_quantize_index_fp8(ctypes.byref(cfg),
                                    _dev(q_idx, torch.bfloat16, "q_idx", (N, G, di)),
                                    _dev(k_idx, torch.bfloat16, "k_idx", (N, di)), N,
                                    _dev(q8, torch.uint8, "q_idx8"), _dev(k8, torch.uint8, "k_idx8"),
                                    _dev(ks, torch.float32, "k_scale"), _stream(stream))
    _check(st, "msa_quantize_index_fp8")
    return q8, k8, ks


def msa_select_topk_fp8(cfg: MsaConfig, q_idx8: torch.Tensor, k_idx8: torch.Tensor,
                        k_scale: torch.Tensor, ids: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """msa_select_topk on e4m3 index tensors with per-block key scales."""
    lib = load_library()
    N = q_idx8.shape[0]
    G, di, k = cfg.num_groups, cfg.index_dim, cfg.top_k
    nb = (N + cfg.block_size - 1) // cfg.block_size
    if ids is None:
        ids = torch.empty((N, G, k), dtype=torch.int32, device=q_idx8.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_SELECT_TOPK, N), q_idx8.device)
    st = lib.msa_select_topk_fp8(ctypes.byref(cfg), _dev(q_idx8, torch.uint8, "q_idx8", (N, G, di)),
                                 _dev(k_idx8, torch.uint8, "k_idx8", (N, di)),
                                 _dev(k_scale, torch.float32, "k_scale", (nb,)), N,
                                 _dev(ids, torch.int32, "ids", (N, G, k)),
                                 _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_select_topk_fp8")
    return ids


def msa_build_block_query_lists(cfg: MsaConfig, ids: torch.Tensor,
                                workspace: Optional[torch.Tensor] = None,
                                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-(group, block) query lists: (row_ptr [G*nb+1], entries [N*G*k] capacity)."""
    lib = load_library()
    N, G, k = ids.shape
    nb = (N + cfg.block_size - 1) // cfg.block_size
    row_ptr = torch.empty(G * nb + 1, dtype=torch.int32, device=ids.device)
    entries = torch.empty(N * G * k, dtype=torch.int32, device=ids.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_BLOCK_QUERY_LISTS, N), ids.device)
    st = lib.msa_build_block_query_lists(ctypes.byref(cfg), _dev(ids, torch.int32, "ids"), N,
                                         _dev(row_ptr, torch.int32, "row_ptr"),
                                         _dev(entries, torch.int32, "entries"),
                                         _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_build_block_query_lists")
    return row_ptr, entries


def msa_prefill(cfg: MsaConfig, q, k, v, q_idx, k_idx, out: Optional[torch.Tensor] = None,
                ids_out=None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Whole MSA prefill.  ``ids_out``: None, True (allocate) or an int32 tensor.

    Returns ``out`` or ``(out, ids)`` when ids are requested.
    """
    lib = load_library()
    N = q.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    if out is None:
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=q.device)
    if ids_out is True:
        ids_out = torch.empty((N, G, kk), dtype=torch.int32, device=q.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_PREFILL, N), q.device)
    ids_ptr = None if ids_out is None else _dev(ids_out, torch.int32, "ids_out", (N, G, kk))
    st = lib.msa_prefill(ctypes.byref(cfg), _dev(q, torch.bfloat16, "q", (N, H, d)),
                         _dev(k, torch.bfloat16, "k", (N, G, d)),
                         _dev(v, torch.bfloat16, "v", (N, G, d)),
                         _dev(q_idx, torch.bfloat16, "q_idx", (N, G, di)),
                         _dev(k_idx, torch.bfloat16, "k_idx", (N, di)), N,
                         _dev(out, torch.bfloat16, "out", (N, H, d)), ids_ptr,
                         _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_prefill")
    return out if ids_out is None else (out, ids_out)


def msa_prefill_fp8_index(cfg: MsaConfig, q, k, v, q_idx8, k_idx8, k_scale,
                          out: Optional[torch.Tensor] = None, ids_out=None,
                          workspace: Optional[torch.Tensor] = None, stream=None):
    """msa_prefill with the quantised Index Branch (e4m3 index tensors and
    per-block key scales, as msa_quantize_index_fp8 returns them)."""
    lib = load_library()
    N = q.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    nb = (N + cfg.block_size - 1) // cfg.block_size
    if out is None:
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=q.device)
    if ids_out is True:
        ids_out = torch.empty((N, G, kk), dtype=torch.int32, device=q.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_PREFILL, N), q.device)
    ids_ptr = None if ids_out is None else _dev(ids_out, torch.int32, "ids_out", (N, G, kk))
    st = lib.msa_prefill_fp8_index(ctypes.byref(cfg), _dev(q, torch.bfloat16, "q", (N, H, d)),
                                   _dev(k, torch.bfloat16, "k", (N, G, d)),
                                   _dev(v, torch.bfloat16, "v", (N, G, d)),
                                   _dev(q_idx8, torch.uint8, "q_idx8", (N, G, di)),
                                   _dev(k_idx8, torch.uint8, "k_idx8", (N, di)),
                                   _dev(k_scale, torch.float32, "k_scale", (nb,)), N,
                                   _dev(out, torch.bfloat16, "out", (N, H, d)), ids_ptr,
                                   _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_prefill_fp8_index")
    return out if ids_out is None else (out, ids_out)


def msa_prefill_block_alignment(cfg: MsaConfig, q, k, v, q_idx, k_idx,
                                workspace: Optional[torch.Tensor] = None, stream=None):
    """Prefill plus the KL-alignment data (see include/msa.h).

    Returns ``(out, ids, block_score, block_mass, kl)``.
    """
    lib = load_library()
    N = q.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    dev = q.device
    out = torch.empty((N, H, d), dtype=torch.bfloat16, device=dev)
    ids = torch.empty((N, G, kk), dtype=torch.int32, device=dev)
    score = torch.empty((N, G, kk), dtype=torch.float32, device=dev)
    mass = torch.empty((N, G, kk), dtype=torch.float32, device=dev)
    kl = torch.empty((N, G), dtype=torch.float32, device=dev)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_PREFILL, N), dev)
    st = lib.msa_prefill_block_alignment(
        ctypes.byref(cfg), _dev(q, torch.bfloat16, "q", (N, H, d)),
        _dev(k, torch.bfloat16, "k", (N, G, d)), _dev(v, torch.bfloat16, "v", (N, G, d)),
        _dev(q_idx, torch.bfloat16, "q_idx", (N, G, di)), _dev(k_idx, torch.bfloat16, "k_idx", (N, di)),
        N, _dev(out, torch.bfloat16, "out"), _dev(ids, torch.int32, "ids"),
        _dev(score, torch.float32, "block_score"), _dev(mass, torch.float32, "block_mass"),
        _dev(kl, torch.float32, "kl"), _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_prefill_block_alignment")
    return out, ids, score, mass, kl


def msa_prefill_varlen_workspace_size(cfg: MsaConfig, cu_seqlens) -> int:
    """Bytes of workspace with which msa_prefill_varlen runs the batch in one
    pass (or, beyond 1024 sequences, each sequence without chunking)."""
    import numpy as _np
    cu = _np.ascontiguousarray(_np.asarray(
        cu_seqlens.cpu() if isinstance(cu_seqlens, torch.Tensor) else cu_seqlens,
        dtype=_np.int64))
    out = ctypes.c_size_t(0)
    _check(load_library().msa_prefill_varlen_workspace_size(
        ctypes.byref(cfg), cu.ctypes.data_as(ctypes.c_void_p), len(cu) - 1, ctypes.byref(out)),
        "msa_prefill_varlen_workspace_size")
    return int(out.value)


def msa_prefill_varlen(cfg: MsaConfig, q, k, v, q_idx, k_idx, cu_seqlens,
                       out: Optional[torch.Tensor] = None, ids_out=None,
                       workspace: Optional[torch.Tensor] = None, stream=None):
    """Prefill of sequences packed along the token axis (host ``cu_seqlens``,
    any int sequence of B+1 offsets).  Returns ``out`` or ``(out, ids)``.

    Without ``workspace`` one is allocated: the one-pass size when it takes at
    most half of the device's free memory, else the size for the longest
    sequence (the sequences then run one after another)."""
    lib = load_library()
    import numpy as _np
    cu = _np.ascontiguousarray(_np.asarray(
        cu_seqlens.cpu() if isinstance(cu_seqlens, torch.Tensor) else cu_seqlens,
        dtype=_np.int64))
    B = len(cu) - 1
    T = q.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    if B < 1 or int(cu[-1]) != T:
        raise ValueError(f"cu_seqlens must end at the packed length {T}")
    if out is None:
        out = torch.empty((T, H, d), dtype=torch.bfloat16, device=q.device)
    if ids_out is True:
        ids_out = torch.empty((T, G, kk), dtype=torch.int32, device=q.device)
    need = msa_prefill_varlen_workspace_size(cfg, cu)
    if workspace is None:
        # one pass over the batch if it fits comfortably, else one sequence at a time
        free, _ = torch.cuda.mem_get_info(q.device)
        if need > free // 2:
            need = msa_workspace_size(cfg, OP_PREFILL, max(int(_np.max(_np.diff(cu))), 1))
    ws = _workspace(workspace, need, q.device)
    ids_ptr = None if ids_out is None else _dev(ids_out, torch.int32, "ids_out", (T, G, kk))
    st = lib.msa_prefill_varlen(ctypes.byref(cfg), _dev(q, torch.bfloat16, "q", (T, H, d)),
                                _dev(k, torch.bfloat16, "k", (T, G, d)),
                                _dev(v, torch.bfloat16, "v", (T, G, d)),
                                _dev(q_idx, torch.bfloat16, "q_idx", (T, G, di)),
                                _dev(k_idx, torch.bfloat16, "k_idx", (T, di)),
                                cu.ctypes.data_as(ctypes.c_void_p), B,
                                _dev(out, torch.bfloat16, "out", (T, H, d)), ids_ptr,
                                _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_prefill_varlen")
    return out if ids_out is None else (out, ids_out)


def msa_decode(cfg: MsaConfig, q, q_idx, k_cache, v_cache, k_idx_cache, cu_seqlens,
               max_seqlen: int, out: Optional[torch.Tensor] = None, ids_out=None,
               workspace: Optional[torch.Tensor] = None, stream=None):
    """One decode step for B sequences (packed caches, device cu_seqlens int64)."""
    lib = load_library()
    B = q.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    total = k_cache.shape[0]
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device)
    if ids_out is True:
        ids_out = torch.empty((B, G, kk), dtype=torch.int32, device=q.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_DECODE, total, B), q.device)
    ids_ptr = None if ids_out is None else _dev(ids_out, torch.int32, "ids_out", (B, G, kk))
    st = lib.msa_decode(ctypes.byref(cfg), _dev(q, torch.bfloat16, "q", (B, H, d)),
                        _dev(q_idx, torch.bfloat16, "q_idx", (B, G, di)),
                        _dev(k_cache, torch.bfloat16, "k_cache", (total, G, d)),
                        _dev(v_cache, torch.bfloat16, "v_cache", (total, G, d)),
                        _dev(k_idx_cache, torch.bfloat16, "k_idx_cache", (total, di)),
                        _dev(cu_seqlens, torch.int64, "cu_seqlens", (B + 1,)), B, max_seqlen,
                        _dev(out, torch.bfloat16, "out", (B, H, d)), ids_ptr,
                        _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_decode")
    return out if ids_out is None else (out, ids_out)


def msa_quantize_rows_fp8(x: torch.Tensor, stream=None):
    """x [..., 128] bf16 -> (x8 uint8 e4m3 bytes of the same shape, scale [...] float32):
    one scale per row of 128 values."""
    lib = load_library()
    rows = x.numel() // 128
    x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    sc = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    if x.shape[-1] != 128:
        raise MsaError("msa_quantize_rows_fp8: rows of 128 values expected")
    st = lib.msa_quantize_rows_fp8(_dev(x, torch.bfloat16, "x"), rows,
                                   _dev(x8, torch.uint8, "x8"), _dev(sc, torch.float32, "scale"),
                                   _stream(stream))
    _check(st, "msa_quantize_rows_fp8")
    return x8, sc


def msa_quantize_mx(x: torch.Tensor, fmt: int, stream=None):
    """x [..., d] bf16 (d a multiple of 32) -> (codes uint8, scales uint8 [..., d/32]):
    MX_E4M3 codes [..., d], MX_E2M1 codes [..., d/2] (two per byte)."""
    lib = load_library()
    d = x.shape[-1]
    if d % 32 != 0:
        raise MsaError("msa_quantize_mx: rows of a multiple of 32 values expected")
    rows = x.numel() // d
    cw = d if fmt == MX_E4M3 else d // 2
    codes = torch.empty(x.shape[:-1] + (cw,), dtype=torch.uint8, device=x.device)
    scales = torch.empty(x.shape[:-1] + (d // 32,), dtype=torch.uint8, device=x.device)
    st = lib.msa_quantize_mx(_dev(x, torch.bfloat16, "x"), rows, d, fmt,
                             _dev(codes, torch.uint8, "codes"), _dev(scales, torch.uint8, "scales"),
                             _stream(stream))
    _check(st, "msa_quantize_mx")
    return codes, scales


def msa_prefill_q8kv4(cfg: MsaConfig, q8, q_scale, k4, k_scale, v4, v_scale, q_idx, k_idx,
                      out: Optional[torch.Tensor] = None, ids_out=None,
                      workspace: Optional[torch.Tensor] = None, stream=None):
    """msa_prefill on MX inputs (see include/msa.h): q8 [N,H,d] e4m3 with q_scale
    [N,H,d/32]; k4, v4 [N,G,d/2] packed e2m1 with k_scale, v_scale [N,G,d/32]."""
    lib = load_library()
    N = q8.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    if out is None:
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device=q8.device)
    if ids_out is True:
        ids_out = torch.empty((N, G, kk), dtype=torch.int32, device=q8.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_PREFILL_Q8KV4, N), q8.device)
    ids_ptr = None if ids_out is None else _dev(ids_out, torch.int32, "ids_out", (N, G, kk))
    st = lib.msa_prefill_q8kv4(
        ctypes.byref(cfg), _dev(q8, torch.uint8, "q8", (N, H, d)),
        _dev(q_scale, torch.uint8, "q_scale", (N, H, d // 32)),
        _dev(k4, torch.uint8, "k4", (N, G, d // 2)),
        _dev(k_scale, torch.uint8, "k_scale", (N, G, d // 32)),
        _dev(v4, torch.uint8, "v4", (N, G, d // 2)),
        _dev(v_scale, torch.uint8, "v_scale", (N, G, d // 32)),
        _dev(q_idx, torch.bfloat16, "q_idx", (N, G, di)), _dev(k_idx, torch.bfloat16, "k_idx", (N, di)),
        N, _dev(out, torch.bfloat16, "out", (N, H, d)), ids_ptr, _dev(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream))
    _check(st, "msa_prefill_q8kv4")
    return out if ids_out is None else (out, ids_out)


def msa_decode_fp8_index(cfg: MsaConfig, q, q_idx8, k_cache, v_cache, k_idx8_cache, k_idx_scale,
                         cu_seqlens, max_seqlen: int, out: Optional[torch.Tensor] = None,
                         ids_out=None, workspace: Optional[torch.Tensor] = None, stream=None):
    """msa_decode with the e4m3 Index Branch: q_idx8 [B,G,128] and k_idx8_cache
    [sum L,128] e4m3 bytes, k_idx_scale [sum L] float32 (one scale per key row)."""
    lib = load_library()
    B = q.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    total = k_cache.shape[0]
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device)
    if ids_out is True:
        ids_out = torch.empty((B, G, kk), dtype=torch.int32, device=q.device)
    ws = _workspace(workspace, msa_workspace_size(cfg, OP_DECODE, total, B), q.device)
    ids_ptr = None if ids_out is None else _dev(ids_out, torch.int32, "ids_out", (B, G, kk))
    st = lib.msa_decode_fp8_index(
        ctypes.byref(cfg), _dev(q, torch.bfloat16, "q", (B, H, d)),
        _dev(q_idx8, torch.uint8, "q_idx8", (B, G, di)),
        _dev(k_cache, torch.bfloat16, "k_cache", (total, G, d)),
        _dev(v_cache, torch.bfloat16, "v_cache", (total, G, d)),
        _dev(k_idx8_cache, torch.uint8, "k_idx8_cache", (total, di)),
        _dev(k_idx_scale, torch.float32, "k_idx_scale", (total,)),
        _dev(cu_seqlens, torch.int64, "cu_seqlens", (B + 1,)), B, max_seqlen,
        _dev(out, torch.bfloat16, "out", (B, H, d)), ids_ptr,
        _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "msa_decode_fp8_index")
    return out if ids_out is None else (out, ids_out)


def msa_decode_static(cfg: MsaConfig, q, q_idx, k_cache, v_cache, k_idx_cache, cu_seqlens,
                      max_seqlen: int, total_len: int, out: Optional[torch.Tensor] = None,
                      ids_out=None, check_device_error: bool = False, stream=None):
    """msa_decode with the library's fixed scratch array instead of a workspace.

    For callers that cannot allocate device memory: the library allocates
    nothing either.  ``out``/``ids_out`` must then be passed in by the caller.
    """
    lib = load_library()
    B = q.shape[0]
    H, G, d, di, kk = cfg.num_heads, cfg.num_groups, cfg.head_dim, cfg.index_dim, cfg.top_k
    total = k_cache.shape[0]
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device)
    if ids_out is True:
        ids_out = torch.empty((B, G, kk), dtype=torch.int32, device=q.device)
    ids_ptr = None if ids_out is None else _dev(ids_out, torch.int32, "ids_out", (B, G, kk))
    st = lib.msa_decode_static(ctypes.byref(cfg), _dev(q, torch.bfloat16, "q", (B, H, d)),
                               _dev(q_idx, torch.bfloat16, "q_idx", (B, G, di)),
                               _dev(k_cache, torch.bfloat16, "k_cache", (total, G, d)),
                               _dev(v_cache, torch.bfloat16, "v_cache", (total, G, d)),
                               _dev(k_idx_cache, torch.bfloat16, "k_idx_cache", (total, di)),
                               _dev(cu_seqlens, torch.int64, "cu_seqlens", (B + 1,)), B,
                               max_seqlen, total_len, _dev(out, torch.bfloat16, "out", (B, H, d)),
                               ids_ptr, 1 if check_device_error else 0, _stream(stream))
    _check(st, "msa_decode_static")
    return out if ids_out is None else (out, ids_out)


_phase_keep = None


def msa_set_phase_events(events) -> None:
    """Record ``torch.cuda.Event`` objects at kernel phase boundaries (see msa.h);
    ``None`` stops recording."""
    global _phase_keep
    lib = load_library()
    if events is None:
        _check(lib.msa_set_phase_events(None, 0), "msa_set_phase_events")
        _phase_keep = None
        return
    for e in events:  # torch creates the CUDA event lazily, on its first record
        if not e.cuda_event:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _phase_keep = (arr, events)
    _check(lib.msa_set_phase_events(arr, len(events)), "msa_set_phase_events")


def msa_selftest_wait_timeout(workspace: torch.Tensor, limit_ns: int, stream=None) -> None:
    """Launch the planted-timeout self-test (see include/msa.h); read the result
    with msa_get_device_error."""
    _check(load_library().msa_selftest_wait_timeout(_dev(workspace, torch.uint8, "workspace"),
                                                    int(limit_ns), _stream(stream)),
           "msa_selftest_wait_timeout")


def msa_get_device_error(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the workspace's device error word."""
    code = ctypes.c_uint32(0)
    st = load_library().msa_get_device_error(_dev(workspace, torch.uint8, "workspace"),
                                             _stream(stream), ctypes.byref(code))
    if st not in (0, 5, 6, 7):
        _check(st, "msa_get_device_error")
    return int(code.value)
