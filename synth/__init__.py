"""Seeded synthetic inputs for the MSA hot path.

This module is shared by both sides of every parity check: the fp64 oracle
(``oracle/``) and the CUDA library (``block_sparse_long_branch_b200``).  It
holds none of the method's arithmetic; it only draws tensors and plants
"needle" key blocks so that block selection is not trivial.

Recipe (the shapes are the long-context workloads the pages describe: a 1M
context, 128-token key blocks, 16 selected blocks per (query, GQA group)):

* every tensor is drawn i.i.d. N(0, 1) with ``torch.randn`` from a seeded
  ``torch.Generator`` on the target device, in fp32, then rounded to bf16
  (round-to-nearest-even, ``Tensor.to``);
* needles: for each needle a key block ``j`` (uniform in ``[0, nb-2]``), a
  group ``g`` and a query ``t`` in a later block are drawn from a numpy
  generator seeded independently of the device; every key row ``s`` of block
  ``j`` gets ``k_idx[s] += 3 * u`` with ``u = q_idx[t, g] / |q_idx[t, g]|``
  (fp64, re-rounded to bf16).  The query ``t`` of group ``g`` should then
  select block ``j``.

The softmax scale of every workload is ``1/sqrt(d)`` applied once to the
logits; the tensors themselves are not pre-scaled.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import numpy as np
import torch

__all__ = [
    "PrefillShape",
    "DecodeShape",
    "PREFILL_CONFIGS",
    "DECODE_CONFIG",
    "DECODE_SMALL",
    "make_prefill_inputs",
    "make_decode_inputs",
    "sample_rows",
]

SEED_BASE = 0x4D534100  # "MSA\0": workload i uses SEED_BASE + i


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    """One causal sequence of N tokens."""

    name: str
    N: int
    H: int
    G: int
    d: int
    d_idx: int
    block: int = 128
    top_k: int = 16
    n_needles: int = 0
    seed: int = SEED_BASE

    @property
    def nb(self) -> int:
        return (self.N + self.block - 1) // self.block

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    """B sequences, one new query token each; caches hold the new token."""

    name: str
    seq_lens: Tuple[int, ...]
    H: int
    G: int
    d: int
    d_idx: int
    block: int = 128
    top_k: int = 16
    needles_per_seq: Tuple[int, ...] = ()
    seed: int = SEED_BASE

    @property
    def B(self) -> int:
        return len(self.seq_lens)

    @property
    def total_len(self) -> int:
        return int(sum(self.seq_lens))

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


PREFILL_CONFIGS = {
    "tiny": PrefillShape("tiny", N=4096, H=4, G=2, d=64, d_idx=64, top_k=16,
                         n_needles=8, seed=SEED_BASE + 0),
    "tiny_dense": PrefillShape("tiny_dense", N=4096, H=4, G=2, d=64, d_idx=64,
                               top_k=32, n_needles=8, seed=SEED_BASE + 0),
    "prefill_8k": PrefillShape("prefill_8k", N=8192, H=64, G=8, d=128, d_idx=128, top_k=16,
                               n_needles=16, seed=SEED_BASE + 5),
    "prefill_32k": PrefillShape("prefill_32k", N=32768, H=64, G=8, d=128,
                                d_idx=128, top_k=16, n_needles=64,
                                seed=SEED_BASE + 1),
    "prefill_128k": PrefillShape("prefill_128k", N=131072, H=64, G=8, d=128,
                                 d_idx=128, top_k=16, n_needles=256,
                                 seed=SEED_BASE + 2),
    "prefill_1m": PrefillShape("prefill_1m", N=1 << 20, H=64, G=8, d=128,
                               d_idx=128, top_k=16, n_needles=1024,
                               seed=SEED_BASE + 4),
}

DECODE_CONFIG = DecodeShape(
    "decode_16x256k_1x1m",
    seq_lens=(262144,) * 16 + (1048576,),
    H=64, G=8, d=128, d_idx=128, top_k=16,
    needles_per_seq=(16,) * 16 + (64,),
    seed=SEED_BASE + 3,
)

# Smaller decode case (two 256K caches, 2.2 GB) used to size profiler captures.
DECODE_SMALL = DecodeShape(
    "decode_2x256k",
    seq_lens=(262144,) * 2,
    H=64, G=8, d=128, d_idx=128, top_k=16,
    needles_per_seq=(16,) * 2,
    seed=SEED_BASE + 6,
)

# Elements drawn per randn call: bounds the fp32 temporary on the device.
_CHUNK_ELEMS = 1 << 28


def _randn_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _CHUNK_ELEMS):
        e = min(n, s + _CHUNK_ELEMS)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device,
                                dtype=torch.float32).to(torch.bfloat16)
    return out


def _plant(k_idx: torch.Tensor, rows: slice, q_vec: torch.Tensor) -> None:
    """k_idx[rows] += 3 * q_vec / |q_vec| (fp64, re-rounded to bf16)."""
    u = q_vec.double()
    u = u / u.norm()
    blk = k_idx[rows].double() + 3.0 * u
    k_idx[rows] = blk.to(torch.bfloat16)


def make_prefill_inputs(shape: PrefillShape, device="cpu",
                        seed: Optional[int] = None) -> dict:
    """Draw q [N,H,d], k/v [N,G,d], q_idx [N,G,d_idx], k_idx [N,d_idx] (bf16).

    Returns a dict with the tensors and ``needles``: a list of
    ``(block j, group g, query t)`` triples.
    """
    seed = shape.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    N, H, G, d, di = shape.N, shape.H, shape.G, shape.d, shape.d_idx
    q = _randn_bf16((N, H, d), gen, device)
    k = _randn_bf16((N, G, d), gen, device)
    v = _randn_bf16((N, G, d), gen, device)
    q_idx = _randn_bf16((N, G, di), gen, device)
    k_idx = _randn_bf16((N, di), gen, device)
    needles: List[Tuple[int, int, int]] = []
    nb = shape.nb
    if shape.n_needles and nb >= 2:
        rng = np.random.default_rng(seed ^ 0x5EED)
        for _ in range(shape.n_needles):
            j = int(rng.integers(0, nb - 1))
            g = int(rng.integers(0, G))
            t = int(rng.integers(shape.block * (j + 1), N))
            _plant(k_idx, slice(j * shape.block, min(N, (j + 1) * shape.block)),
                   q_idx[t, g])
            needles.append((j, g, t))
    return dict(q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx, needles=needles,
                shape=shape)


def make_decode_inputs(shape: DecodeShape, device="cpu",
                       seed: Optional[int] = None) -> dict:
    """Draw one decode step: q [B,H,d], q_idx [B,G,d_idx] and packed caches.

    Caches: k/v [sum L, G, d], k_idx [sum L, d_idx]; sequence b owns rows
    ``cu_seqlens[b] .. cu_seqlens[b+1]-1`` and its new query sits at position
    ``L_b - 1`` (its key/value rows are already in the cache).
    """
    seed = shape.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, H, G, d, di = shape.B, shape.H, shape.G, shape.d, shape.d_idx
    L = shape.total_len
    cu = np.zeros(B + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(shape.seq_lens, dtype=np.int64))
    q = _randn_bf16((B, H, d), gen, device)
    q_idx = _randn_bf16((B, G, di), gen, device)
    k_cache = _randn_bf16((L, G, d), gen, device)
    v_cache = _randn_bf16((L, G, d), gen, device)
    k_idx_cache = _randn_bf16((L, di), gen, device)
    needles: List[Tuple[int, int, int]] = []  # (sequence b, block j, group g)
    rng = np.random.default_rng(seed ^ 0x5EED)
    for b in range(B):
        nb_b = (shape.seq_lens[b] + shape.block - 1) // shape.block
        n_b = shape.needles_per_seq[b] if shape.needles_per_seq else 0
        if nb_b < 2:
            continue
        for _ in range(n_b):
            j = int(rng.integers(0, nb_b - 1))
            g = int(rng.integers(0, G))
            r0 = int(cu[b]) + j * shape.block
            _plant(k_idx_cache, slice(r0, r0 + shape.block), q_idx[b, g])
            needles.append((b, j, g))
    return dict(q=q, q_idx=q_idx, k_cache=k_cache, v_cache=v_cache,
                k_idx_cache=k_idx_cache, cu_seqlens=torch.from_numpy(cu),
                needles=needles, shape=shape)


def sample_rows(N: int, count: int, seed: int, extra=()) -> np.ndarray:
    """Query positions spread uniformly over [0, N) plus ``extra`` rows.

    Always includes the first and last position and the first/last token of
    the first and last key block, so the degenerate early rows and the ragged
    end are covered.
    """
    rng = np.random.default_rng(seed ^ 0xA11)
    base = np.linspace(0, N - 1, num=min(count, N)).round().astype(np.int64)
    jitter = rng.integers(-3, 4, size=base.shape)
    rows = np.clip(base + jitter, 0, N - 1)
    fixed = [0, 1, min(N - 1, 127), min(N - 1, 128), N - 1]
    rows = np.unique(np.concatenate([rows, np.asarray(fixed, np.int64),
                                     np.asarray(list(extra), np.int64)]))
    return rows
