"""fp64 CPU oracle for the MSA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``block_sparse_long_branch_b200``) never imports it and has no CPU fallback.

The attention arithmetic lives in ``msa_oracle.c`` (plain loops, fp64); this
module marshals numpy arrays through ctypes, and holds in numpy the e4m3
codec and quantiser of the quantised Index Branch (format arithmetic only).
Each wrapper names the passage of the pages it follows; the C file carries the
same citations.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int32
        lib.msa_oracle_pooled_scores.argtypes = [P, P, I64, P, I32, I32, I32, I64, P]
        lib.msa_oracle_pooled_scores.restype = None
        lib.msa_oracle_pooled_scores_f64.argtypes = [P, P, I64, P, I32, I32, I32, I64, P]
        lib.msa_oracle_pooled_scores_f64.restype = None
        lib.msa_oracle_select_blocks.argtypes = [P, P, I64, I32, I64, I32, I32, P]
        lib.msa_oracle_select_blocks.restype = None
        lib.msa_oracle_block_attention.argtypes = [P, P, I64, P, P, I32, I32, I32, I32, I32,
                                                   ctypes.c_double, P, P, P, P]
        lib.msa_oracle_block_attention.restype = None
        lib.msa_oracle_block_query_lists.argtypes = [P, I64, I32, I64, I32, P, P]
        lib.msa_oracle_block_query_lists.restype = I64
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def as_bf16_bits(x) -> np.ndarray:
    """A bf16 torch tensor (or uint16 array) as a contiguous uint16 array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy()
                                .view(np.uint16))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pooled_scores(qi_rows, pos, k_idx, block: int, nb_out: int) -> np.ndarray:
    """Index Branch scoring + per-block max over visible tokens.

    ai-tool-zukan MiniMax MSA guide, section "2段階構造の中身": visible key
    tokens are scored, then max-pooled to the block level.
    qi_rows [n,G,di] bf16, pos [n] int64, k_idx [T,di] bf16 -> [n,G,nb_out] f64.
    """
    lib = _load()
    qi = as_bf16_bits(qi_rows)
    ki = as_bf16_bits(k_idx)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    n, G, di = qi.shape
    assert ki.shape[1] == di and pos.shape == (n,)
    assert n == 0 or ki.shape[0] > int(pos.max())
    out = np.empty((n, G, nb_out), dtype=np.float64)
    lib.msa_oracle_pooled_scores(_ptr(qi), _ptr(pos), n, _ptr(ki), G, di, block, nb_out,
                                 _ptr(out))
    return out


def select_blocks(pooled: np.ndarray, pos, block: int, top_k: int) -> np.ndarray:
    """Forced-local top-k per (query, group), ids ascending and -1 padded.

    ai-tool-zukan MiniMax MSA guide, sections "2段階構造の中身" (top-k per query
    and group, local block always included) and
    "クエリを含むローカルブロックの強制取り込み".
    """
    lib = _load()
    pooled = np.ascontiguousarray(pooled, dtype=np.float64)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    n, G, nb_in = pooled.shape
    assert n == 0 or int(pos.max()) // block < nb_in
    ids = np.empty((n, G, top_k), dtype=np.int32)
    lib.msa_oracle_select_blocks(_ptr(pooled), _ptr(pos), n, G, nb_in, block, top_k,
                                 _ptr(ids))
    return ids


def block_attention(q_rows, pos, k, v, ids: np.ndarray, scale: float, block: int,
                    partials: bool = False):
    """Main Branch: exact softmax over the selected blocks' visible keys.

    ai-tool-zukan MiniMax MSA guide, section "Index BranchとMain Branchの役割分担".
    q_rows [n,H,d], k/v [T,G,d] bf16, ids [n,G,top_k] -> out [n,H,d] f64
    (and, with ``partials``, lse [n,H,top_k] and o [n,H,top_k,d]).
    """
    lib = _load()
    qb = as_bf16_bits(q_rows)
    kb = as_bf16_bits(k)
    vb = as_bf16_bits(v)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n, H, d = qb.shape
    G = kb.shape[1]
    top_k = ids.shape[2]
    assert ids.shape == (n, G, top_k) and kb.shape == vb.shape and kb.shape[2] == d
    assert H % G == 0
    out = np.empty((n, H, d), dtype=np.float64)
    lse = np.empty((n, H, top_k), dtype=np.float64) if partials else None
    po = np.empty((n, H, top_k, d), dtype=np.float64) if partials else None
    lib.msa_oracle_block_attention(_ptr(qb), _ptr(pos), n, _ptr(kb), _ptr(vb), H, G, d, block,
                                   top_k, float(scale), _ptr(ids), _ptr(out), _ptr(lse),
                                   _ptr(po))
    if partials:
        return out, lse, po
    return out


def block_query_lists(ids: np.ndarray, nb: int):
    """Per-(group, key block) lists of (query t, slot r), ascending t.

    tnkblog MiniMax M3 / MSA post, section "MSA の実装": key blocks are the
    outer loop and the queries that hit a block are gathered.
    Returns (row_ptr [G*nb+1] int32, entries [nnz] int32 with (t<<5)|r).
    """
    lib = _load()
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    N, G, top_k = ids.shape
    assert top_k <= 32
    row_ptr = np.empty(G * nb + 1, dtype=np.int32)
    entries = np.empty(N * G * top_k, dtype=np.int32)
    total = lib.msa_oracle_block_query_lists(_ptr(ids), N, G, nb, top_k, _ptr(row_ptr),
                                             _ptr(entries))
    if total < 0:
        raise ValueError("block id out of range")
    return row_ptr, entries[:total].copy()


def block_alignment(pooled: np.ndarray, ids: np.ndarray, lse: np.ndarray):
    """Index-vs-Main alignment of the selected blocks of every (query, group).

    ai-tool-zukan MiniMax MSA guide, section "非微分的な選択をどう学習させるか
    （KLダイバージェンス）" (subsection "選択を学習可能にするKL損失"): the Index
    Branch's distribution of scores over the blocks is brought close, by a KL
    divergence, to the distribution of which blocks really mattered to the Main
    Branch's exact attention.  The pages give no formulas; the reading used:
      index side  q_r = softmax over the filled slots of the pooled raw-dot
                  scores (temperature 1);
      main side   p_r = mean over the group's heads of exp(lse[h, r] - L_h),
                  the share of head h's exact softmax on slot r's keys
                  (L_h = logsumexp_r lse[h, r]);
      KL(p || q) = sum_r p_r (ln p_r - ln q_r), in nats, terms with p_r = 0
                  contributing 0.
    pooled [n,G,nb] (as from pooled_scores), ids [n,G,k] (-1 = empty slot),
    lse [n,H,k] (as from block_attention with partials) ->
    (score [n,G,k] with -inf in empty slots, mass [n,G,k] with 0 there, kl [n,G]).
    """
    pooled = np.asarray(pooled, dtype=np.float64)
    ids = np.asarray(ids)
    lse = np.asarray(lse, dtype=np.float64)
    n, G, k = ids.shape
    H = lse.shape[1]
    assert lse.shape == (n, H, k) and H % G == 0
    HG = H // G
    filled = ids >= 0
    score = np.full((n, G, k), -np.inf)
    mass = np.zeros((n, G, k))
    kl = np.zeros((n, G))
    for t in range(n):
        for g in range(G):
            f = filled[t, g]
            if not f.any():
                continue
            sc = pooled[t, g, ids[t, g, f]]
            score[t, g, f] = sc
            # index side: softmax of the scores over the filled slots
            lq = sc - sc.max()
            lq = lq - np.log(np.exp(lq).sum())
            # main side: each head's softmax mass per slot, averaged over heads
            p = np.zeros(int(f.sum()))
            for h in range(g * HG, (g + 1) * HG):
                lh = lse[t, h, f]
                w = np.exp(lh - lh.max())
                p += w / w.sum()
            p /= HG
            mass[t, g, f] = p
            pos = p > 0
            kl[t, g] = float(np.sum(p[pos] * (np.log(p[pos]) - lq[pos])))
    return score, mass, kl


# ---------------------------------------------------------------------------
# Whole-path helpers (composition of the steps above, nothing more).
# ---------------------------------------------------------------------------

def prefill(q, k, v, q_idx, k_idx, *, block: int, top_k: int, scale: float, rows=None,
            partials: bool = False) -> dict:
    """Index Branch + Main Branch for the query rows ``rows`` (default: all).

    Returns dict(rows, pooled [n,G,nb], ids [n,G,top_k], out [n,H,d] f64, and
    with ``partials`` also lse/o per slot).
    """
    N = q.shape[0]
    nb = (N + block - 1) // block
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    qi = as_bf16_bits(q_idx)[rows]
    pooled = pooled_scores(qi, rows, k_idx, block, nb)
    ids = select_blocks(pooled, rows, block, top_k)
    qr = as_bf16_bits(q)[rows]
    res = dict(rows=rows, pooled=pooled, ids=ids)
    if partials:
        res["out"], res["lse"], res["o"] = block_attention(qr, rows, k, v, ids, scale, block,
                                                          partials=True)
    else:
        res["out"] = block_attention(qr, rows, k, v, ids, scale, block)
    return res


def decode(q, q_idx, k_cache, v_cache, k_idx_cache, cu_seqlens, *, block: int, top_k: int,
           scale: float, seqs=None) -> dict:
    """One decode step: sequence b's query sits at position L_b - 1 of its cache.

    The pages give no separate decode algorithm (zhaixingw M3 review, section
    "这套注意力到底怎么省的", reports decode speed only); the plainest reading is
    the same two branches for the single newest query row.
    Returns dict(ids [B,G,top_k], out [B,H,d], pooled list per sequence).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = len(cu) - 1
    seqs = range(B) if seqs is None else seqs
    qb = as_bf16_bits(q)
    qib = as_bf16_bits(q_idx)
    H, d = qb.shape[1], qb.shape[2]
    G = qib.shape[1]
    ids = np.full((B, G, top_k), -1, dtype=np.int32)
    out = np.full((B, H, d), np.nan)
    pooled = {}
    for b in seqs:
        s0, s1 = int(cu[b]), int(cu[b + 1])
        L = s1 - s0
        pos = np.array([L - 1], dtype=np.int64)
        nb = (L + block - 1) // block
        kb = k_idx_cache[s0:s1]
        p = pooled_scores(qib[b:b + 1], pos, kb, block, nb)
        sel = select_blocks(p, pos, block, top_k)
        o = block_attention(qb[b:b + 1], pos, k_cache[s0:s1], v_cache[s0:s1], sel, scale, block)
        ids[b] = sel[0]
        out[b] = o[0]
        pooled[b] = p[0]
    return dict(ids=ids, out=out, pooled=pooled)


# ---------------------------------------------------------------------------
# Quantised Index Branch (e4m3).  The pages report the indexer and main branch
# moving from Q8KV8 to Q8KV4 in a later model (dot-ai "MiniMax M3.1 Flashとは？
# 428BのMoEモデルがウェイト公開", the passage on the ModelScope model card's
# quantisation) with no number format; the reading used: per index-query row
# and per 128-key block of index keys, s = max|x| / 448 in fp32 (1 when the
# max is 0) and x8 = e4m3(x / s), fp32 division, nearest even, saturating.
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """e4m3 bytes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
    infinities, 0x7F/0xFF are NaN) -> fp64."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    val = np.where((b & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp32 values -> nearest e4m3 byte (ties to even), saturating at +-448."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.where(np.signbit(x), 0x80, 0).astype(np.int64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # quantum of the binade: 2^(e-3) for normals (e >= -6), 2^-9 below
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    q = 2.0 ** (e - 3)
    n = np.rint(a / q)  # round half to even
    v = n * q           # the e4m3 value (may reach the next binade)
    e2 = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    normal = v >= 2.0 ** -6
    ef = np.where(normal, e2 + 7, 0).astype(np.int64)
    mf = np.where(normal, np.rint((v / 2.0 ** e2 - 1.0) * 8.0), np.rint(v / 2.0 ** -9))
    code = (ef << 3) | mf.astype(np.int64)
    code = np.where(v == 0, 0, code)
    return (sign | code).astype(np.uint8)


def _scale(amax: np.ndarray) -> np.ndarray:
    amax = np.asarray(amax, dtype=np.float32)
    return np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)


def quantize_index_fp8(q_idx, k_idx, block: int = 128):
    """(q_idx [N,G,d] bf16, k_idx [N,d] bf16) -> (q8 [N,G,d] u8, k8 [N,d] u8,
    k_scale [ceil(N/block)] f32)."""
    qf = bf16_bits_to_f64(as_bf16_bits(q_idx)).astype(np.float32)
    kf = bf16_bits_to_f64(as_bf16_bits(k_idx)).astype(np.float32)
    sq = _scale(np.abs(qf).max(axis=2))
    q8 = e4m3_encode(qf / sq[:, :, None])
    N = kf.shape[0]
    nb = (N + block - 1) // block
    amax = np.array([np.abs(kf[j * block:(j + 1) * block]).max() for j in range(nb)],
                    dtype=np.float32)
    sk = _scale(amax)
    k8 = e4m3_encode(kf / np.repeat(sk, block)[:N, None])
    return q8, k8, sk


def pooled_scores_fp8(q8_rows, pos, k8, k_scale, block: int, nb_out: int) -> np.ndarray:
    """Pooled scores of the quantised Index Branch: the max over visible keys of
    <e4m3(q8), e4m3(k8) * k_scale[block of the key]> (fp64)."""
    lib = _load()
    qv = np.ascontiguousarray(e4m3_decode(q8_rows), dtype=np.float64)
    kv = e4m3_decode(k8) * np.repeat(np.asarray(k_scale, dtype=np.float64),
                                     block)[:np.asarray(k8).shape[0], None]
    kv = np.ascontiguousarray(kv, dtype=np.float64)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    n, G, di = qv.shape
    assert kv.shape[1] == di and pos.shape == (n,)
    assert n == 0 or kv.shape[0] > int(pos.max())
    out = np.empty((n, G, nb_out), dtype=np.float64)
    lib.msa_oracle_pooled_scores_f64(_ptr(qv), _ptr(pos), n, _ptr(kv), G, di, block, nb_out,
                                     _ptr(out))
    return out


# ---------------------------------------------------------------------------
# Quantised Index Branch over a decode cache: the same e4m3 reading with one
# fp32 scale per index-key row (a cache grows one token at a time, and each
# token is quantised once, when it is appended); the query rows as above.
# ---------------------------------------------------------------------------

def quantize_rows_fp8(x):
    """x [..., d] bf16 -> (x8 [..., d] u8, scale [...] f32): per row of d values,
    s = max|x| / 448 in fp32 (1 when the max is 0), x8 = e4m3(x / s)."""
    xf = bf16_bits_to_f64(as_bf16_bits(x)).astype(np.float32)
    s = _scale(np.abs(xf).max(axis=-1))
    return e4m3_encode(xf / s[..., None]), s


def pooled_scores_fp8_rows(q8_rows, pos, k8, k_row_scale, block: int, nb_out: int) -> np.ndarray:
    """Pooled scores of the quantised Index Branch with per-key-row scales: the
    max over visible keys s of <e4m3(q8), e4m3(k8[s]) * k_row_scale[s]> (fp64)."""
    lib = _load()
    qv = np.ascontiguousarray(e4m3_decode(q8_rows), dtype=np.float64)
    kv = e4m3_decode(k8) * np.asarray(k_row_scale, dtype=np.float64)[:, None]
    kv = np.ascontiguousarray(kv, dtype=np.float64)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    n, G, di = qv.shape
    assert kv.shape[1] == di and pos.shape == (n,)
    assert n == 0 or kv.shape[0] > int(pos.max())
    out = np.empty((n, G, nb_out), dtype=np.float64)
    lib.msa_oracle_pooled_scores_f64(_ptr(qv), _ptr(pos), n, _ptr(kv), G, di, block, nb_out,
                                     _ptr(out))
    return out


# ---------------------------------------------------------------------------
# Quantised Main Branch ("Q8KV4"; dot-ai "MiniMax M3.1 Flashとは？428BのMoEモデル
# がウェイト公開", the passage on the ModelScope model card's quantisation: the
# sparse attention moving from Q8KV8 to Q8KV4).  The pages name no number
# format.  The reading used: the OCP Microscaling (MX) formats, version 1.0 --
# every 32 consecutive values along d share one power-of-two scale 2^X, kept
# as an 8-bit biased exponent (E8M0, X + 127); X = floor(log2(max|x|)) -
# emax_elem (emax_elem = 8 for e4m3, 2 for e2m1), -127 for an all-zero block,
# clamped to [-127, 127]; each element is the nearest value of its format to
# x / 2^X (ties to even), saturating at the format's largest magnitude.  Q is
# MXFP8 (e4m3 elements), K and V are MXFP4 (e2m1 elements).
# ---------------------------------------------------------------------------

MX_BLOCK = 32
MX_E4M3, MX_E2M1 = 0, 1
MX_EMAX = {MX_E4M3: 8, MX_E2M1: 2}
# e2m1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; code & 7 indexes
# the magnitude (0 and 1 are the zero and the subnormal 0.5)
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """e2m1 codes (0..15, one per byte) -> fp64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    return np.where(c & 8, -1.0, 1.0) * E2M1_VALUES[c & 7]


def e2m1_encode(y: np.ndarray) -> np.ndarray:
    """Values -> nearest e2m1 code, ties to the even code, saturating at 6;
    the sign bit is the value's own (so -0 gives code 8)."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), 6.0)
    lo = np.clip(np.searchsorted(E2M1_VALUES, a, side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    vlo, vhi = E2M1_VALUES[lo], E2M1_VALUES[hi]
    mid = (vlo + vhi) / 2.0
    pick = np.where(a < mid, lo, np.where(a > mid, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(hi == lo, lo, pick)
    return (pick | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def mx_block_exponent(amax: np.ndarray, fmt: int) -> np.ndarray:
    """X of each block from its largest magnitude (exact: frexp)."""
    amax = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(np.where(amax > 0, amax, 1.0))  # amax = m 2^e, m in [0.5, 1)
    x = np.where(amax > 0, e - 1 - MX_EMAX[fmt], -127)
    return np.clip(x, -127, 127).astype(np.int64)


def mx_quantize(x, fmt: int):
    """x [..., d] bf16 (d a multiple of 32) -> (codes [..., d] uint8: e4m3
    bytes or e2m1 codes, one per byte; scales [..., d/32] uint8, X + 127)."""
    xf = bf16_bits_to_f64(as_bf16_bits(x))
    d = xf.shape[-1]
    assert d % MX_BLOCK == 0
    blocks = xf.reshape(xf.shape[:-1] + (d // MX_BLOCK, MX_BLOCK))
    X = mx_block_exponent(np.abs(blocks).max(axis=-1), fmt)
    y = blocks / np.exp2(X.astype(np.float64))[..., None]  # exact: a power of two
    codes = e4m3_encode(y.astype(np.float32)) if fmt == MX_E4M3 else e2m1_encode(y)
    return codes.reshape(xf.shape).astype(np.uint8), (X + 127).astype(np.uint8)


def mx_dequantize(codes, scales, fmt: int) -> np.ndarray:
    """(codes [..., d], scales [..., d/32]) -> fp64 values code * 2^(scale - 127)."""
    codes = np.asarray(codes, dtype=np.uint8)
    d = codes.shape[-1]
    v = e4m3_decode(codes) if fmt == MX_E4M3 else e2m1_decode(codes)
    X = np.asarray(scales, dtype=np.uint8).astype(np.int64) - 127
    v = v.reshape(codes.shape[:-1] + (d // MX_BLOCK, MX_BLOCK))
    return (v * np.exp2(X.astype(np.float64))[..., None]).reshape(codes.shape)


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """[..., d] codes -> [..., d/2] bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 values that bf16 represents exactly -> their bf16 bit patterns."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    assert np.array_equal(f.astype(np.float64), np.asarray(x, dtype=np.float64),
                          equal_nan=True), "value not exact in fp32"
    bits = f.view(np.uint32)
    assert not np.any(bits & 0xFFFF), "value not exact in bf16"
    return (bits >> 16).astype(np.uint16)
