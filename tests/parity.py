"""Comparison helpers shared by the GPU parity tests (no method arithmetic here)."""
from __future__ import annotations

import numpy as np

# Acceptance bars: selected ids bit-exact except near-ties within 1e-3 (raw
# dot-product units) of the boundary score; bf16 outputs within 1e-2 max-abs
# and 2e-3 mean-abs of the fp64 oracle.  An output of magnitude 4 or more is
# beyond that bound by its own bf16 rounding (half a spacing there is 2^-6 >
# 1e-2, even for the correctly rounded exact value): such an output may be off
# by its bf16 half-spacing plus the arithmetic budget the bound leaves at
# magnitudes 2 to 4 (1e-2 - 2^-7).
NEAR_TIE = 1e-3
OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 2e-3


def bf16_half_spacing(x):
    """Half the distance between neighbouring bf16 values at |x| (normal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 8)


OUT_ARITH = OUT_MAX_ABS - 2.0 ** -7


def check_id_rows_valid(ids: np.ndarray, rows: np.ndarray, block: int, top_k: int):
    """Structure every selection must have, whatever the scores."""
    for i, t in enumerate(rows):
        local = int(t) // block
        for g in range(ids.shape[1]):
            sel = ids[i, g]
            valid = sel[sel >= 0]
            assert len(valid) == min(top_k, local + 1), (t, g, sel)
            assert np.all(sel[len(valid):] == -1), (t, g, sel)
            assert np.all(np.diff(valid) > 0), (t, g, sel)
            assert valid[-1] == local, (t, g, sel)


def compare_ids(gpu_ids: np.ndarray, ref_ids: np.ndarray, ref_pooled: np.ndarray,
                rows: np.ndarray, block: int, top_k: int, tol: float = NEAR_TIE):
    """Assert equality except near-ties; return the list of (t, g) near-tie rows."""
    ties = []
    for i, t in enumerate(rows):
        local = int(t) // block
        for g in range(gpu_ids.shape[1]):
            a = set(int(x) for x in gpu_ids[i, g] if x >= 0)
            b = set(int(x) for x in ref_ids[i, g] if x >= 0)
            if a == b:
                continue
            cand = ref_pooled[i, g, :local]
            order = np.sort(cand)[::-1]
            boundary = order[top_k - 2] if local >= top_k - 1 else order[-1]
            for j in a ^ b:
                assert j != local, (t, g, a, b)
                assert abs(cand[j] - boundary) <= tol, (t, g, j, cand[j], boundary)
            ties.append((int(t), g))
    return ties


def check_output(gpu_out: np.ndarray, ref_out: np.ndarray, max_abs: float = OUT_MAX_ABS,
                 mean_abs: float = OUT_MEAN_ABS):
    err = np.abs(gpu_out.astype(np.float64) - ref_out)
    assert np.isfinite(gpu_out).all()
    bound = np.maximum(max_abs, bf16_half_spacing(ref_out) + OUT_ARITH)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), (f"max abs err {err.max():.3g}; worst over its bound: "
                                  f"{err[worst]:.3g} at |ref| {abs(ref_out[worst]):.3g}")
    assert err.mean() <= mean_abs, f"mean abs err {err.mean():.3g}"
    return float(err.max()), float(err.mean())
