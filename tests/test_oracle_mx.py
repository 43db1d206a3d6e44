"""Pins of the oracle's MX codec and quantiser (the reading of the pages'
Q8KV4: OCP Microscaling v1.0, e4m3 and e2m1 elements, one E8M0 scale per 32
values), checked against the format definitions and by brute force."""
import numpy as np
import pytest
import torch

import oracle


def _e2m1_from_fields(c: int) -> float:
    """The element format's own definition: 1 sign bit, 2 exponent bits with
    bias 1, 1 mantissa bit; exponent field 0 is subnormal (0.m x 2^0)."""
    s, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -mag if s else mag


def test_e2m1_decode_matches_bit_fields():
    got = oracle.e2m1_decode(np.arange(16))
    want = np.array([_e2m1_from_fields(c) for c in range(16)])
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.arange(16) >= 8)


def test_e2m1_encode_is_nearest_by_brute_force():
    rng = np.random.default_rng(3)
    y = np.concatenate([rng.uniform(-7.5, 7.5, 20000), rng.uniform(-1, 1, 5000)])
    codes = oracle.e2m1_encode(y)
    vals = oracle.e2m1_decode(codes)
    table = np.array([_e2m1_from_fields(c) for c in range(16)])
    best = np.abs(y[:, None] - table[None, :]).min(axis=1)
    clipped = np.clip(y, -6.0, 6.0)
    assert np.all(np.abs(clipped - vals) <= best + 1e-12)
    assert np.all(np.abs(vals) <= 6.0)


@pytest.mark.parametrize("lo,hi", [(0.0, 0.5), (0.5, 1.0), (1.0, 1.5), (1.5, 2.0),
                                   (2.0, 3.0), (3.0, 4.0), (4.0, 6.0)])
def test_e2m1_ties_go_to_the_even_code(lo, hi):
    mid = (lo + hi) / 2.0
    c = int(oracle.e2m1_encode(np.array([mid]))[0])
    assert c % 2 == 0 and oracle.e2m1_decode(np.array([c]))[0] in (lo, hi)
    # just off the midpoint, the nearer value wins
    eps = (hi - lo) * 1e-6
    assert oracle.e2m1_decode(oracle.e2m1_encode(np.array([mid - eps])))[0] == lo
    assert oracle.e2m1_decode(oracle.e2m1_encode(np.array([mid + eps])))[0] == hi
    # the same for negative values, with the sign bit set
    cn = int(oracle.e2m1_encode(np.array([-mid]))[0])
    assert cn == c | 8


@pytest.mark.parametrize("fmt,amax,X", [
    (oracle.MX_E2M1, 6.0, 0), (oracle.MX_E2M1, 4.0, 0), (oracle.MX_E2M1, 3.999, -1),
    (oracle.MX_E2M1, 1.0, -2), (oracle.MX_E2M1, 0.75, -3),
    (oracle.MX_E4M3, 448.0, 0), (oracle.MX_E4M3, 256.0, 0), (oracle.MX_E4M3, 255.0, -1),
    (oracle.MX_E4M3, 1.0, -8), (oracle.MX_E4M3, 2.0 ** -130, -138 + 0),
    (oracle.MX_E2M1, 0.0, -127), (oracle.MX_E4M3, 0.0, -127),
])
def test_block_exponent_is_floor_log2_minus_emax(fmt, amax, X):
    # X = floor(log2(amax)) - emax_elem, clamped to the E8M0 range [-127, 127]
    got = int(oracle.mx_block_exponent(np.array([amax]), fmt)[0])
    assert got == max(-127, X)


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", [oracle.MX_E4M3, oracle.MX_E2M1])
def test_representable_blocks_round_trip_exactly(fmt):
    rng = np.random.default_rng(5 + fmt)
    if fmt == oracle.MX_E2M1:
        table = np.array([_e2m1_from_fields(c) for c in range(16)])
    else:
        table = oracle.e4m3_decode(np.arange(256))
        table = table[np.isfinite(table)]
    rows = []
    for X in (-20, -3, 0, 5, 40):
        v = rng.choice(table, size=32)
        v[0] = table.max()  # pins the block's scale to 2^X
        rows.append(v * 2.0 ** X)
    x = np.stack(rows)
    codes, scales = oracle.mx_quantize(_bf16(x), fmt)
    assert np.array_equal(scales[:, 0].astype(np.int64) - 127, [-20, -3, 0, 5, 40])
    assert np.array_equal(oracle.mx_dequantize(codes, scales, fmt), x)


@pytest.mark.parametrize("fmt", [oracle.MX_E4M3, oracle.MX_E2M1])
def test_quantisation_error_is_within_half_a_step(fmt):
    rng = np.random.default_rng(11 + fmt)
    x = (rng.standard_normal((64, 128)) * np.exp2(rng.integers(-6, 6, (64, 1)))).astype(np.float32)
    xb = _bf16(x)
    xf = oracle.bf16_bits_to_f64(oracle.as_bf16_bits(xb))
    codes, scales = oracle.mx_quantize(xb, fmt)
    deq = oracle.mx_dequantize(codes, scales, fmt)
    X = np.repeat(scales.astype(np.int64) - 127, 32, axis=-1).astype(np.float64)
    y = xf / np.exp2(X)  # the scaled value the element format rounds
    err = np.abs(deq / np.exp2(X) - y)
    if fmt == oracle.MX_E2M1:
        # step of the bracketing pair: 0.5 below 2, 1 in [2, 4), 2 in [4, 6]
        step = np.where(np.abs(y) < 2, 0.5, np.where(np.abs(y) < 4, 1.0, 2.0))
        sat = np.maximum(np.abs(y) - 6.0, 0.0)
    else:
        e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6)))
        step = 2.0 ** (e - 3)
        sat = np.maximum(np.abs(y) - 448.0, 0.0)
    assert np.all(err <= step / 2 + sat + 1e-12)
    # the block maximum's scaled value stays below 2^(emax + 1)
    assert np.all(np.abs(y).reshape(64, 4, 32).max(axis=-1) < 2.0 ** (oracle.MX_EMAX[fmt] + 1))


def test_dequantised_values_are_exact_in_bf16():
    # an element has at most 4 significant bits and the scale is a power of two,
    # so the product is a bf16 value (8 significant bits) while it stays normal;
    # rows span block magnitudes from 2^-100 to 2^100
    rng = np.random.default_rng(17)
    mag = np.exp2(np.linspace(-100, 100, 16))[:, None]
    x = _bf16(rng.standard_normal((16, 128)) * 3.0 * mag)
    for fmt in (oracle.MX_E4M3, oracle.MX_E2M1):
        codes, scales = oracle.mx_quantize(x, fmt)
        deq = oracle.mx_dequantize(codes, scales, fmt)
        back = oracle.bf16_bits_to_f64(oracle.f64_to_bf16_bits(deq))
        assert np.array_equal(back, deq)
        assert np.count_nonzero(deq) > deq.size // 2


def test_e2m1_packing_puts_even_elements_in_the_low_nibble():
    codes = np.arange(16, dtype=np.uint8)[None, :]
    packed = oracle.pack_e2m1(codes)
    assert packed.tolist() == [[0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]]
    assert np.array_equal(oracle.unpack_e2m1(packed), codes)
