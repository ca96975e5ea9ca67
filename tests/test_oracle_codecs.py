"""Pins for the oracle's number formats (bf16 rounding, FP8 e4m3 codec).

The FP8 payload is the "FP8 activations (1 byte)" of "Expert parallelism
and all-to-all", section "Traffic math".  The pages do not define the
format; the oracle follows the OCP 8-bit floating point E4M3 encoding
(bias 7, no infinities, S.1111.111 = NaN, max 448).  These tests pin it
against (a) values the OCP definition fixes, (b) an exhaustive round trip,
(c) brute-force nearest-value search, and (d) torch's own conversions.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _all_finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_e4m3_decode_fixed_points():
    c = torch.tensor([0x00, 0x01, 0x07, 0x08, 0x38, 0x40, 0x7E, 0xFE, 0x80, 0xB8],
                     dtype=torch.uint8)
    v = oracle.e4m3_decode(c).tolist()
    assert v[0] == 0.0 and not math.copysign(1.0, v[0]) < 0
    assert v[1] == 2.0 ** -9          # smallest subnormal
    assert v[2] == 7 * 2.0 ** -9      # largest subnormal
    assert v[3] == 2.0 ** -6          # smallest normal
    assert v[4] == 1.0
    assert v[5] == 2.0
    assert v[6] == 448.0              # largest finite
    assert v[7] == -448.0
    assert v[8] == 0.0 and math.copysign(1.0, v[8]) < 0
    assert v[9] == -1.0
    nan = oracle.e4m3_decode(torch.tensor([0x7F, 0xFF], dtype=torch.uint8))
    assert torch.isnan(nan).all()


def test_e4m3_exhaustive_round_trip():
    codes = torch.tensor(_all_finite_codes(), dtype=torch.uint8)
    vals = oracle.e4m3_decode(codes).to(torch.float32)
    back = oracle.e4m3_encode(vals)
    assert torch.equal(back, codes)


def _brute_force_e4m3(v: float) -> int:
    """Nearest finite e4m3 code, ties to the even code, saturating."""
    if v > 448.0:
        v = 448.0
    if v < -448.0:
        v = -448.0
    best, best_d = None, None
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        s = -1.0 if c & 0x80 else 1.0
        E, m = (c >> 3) & 15, c & 7
        val = s * (m * 2.0 ** -9 if E == 0 else (1 + m / 8) * 2.0 ** (E - 7))
        if (val == 0.0) and ((c & 0x80) != 0) != (math.copysign(1.0, v) < 0):
            continue  # zero keeps the sign of the input
        d = abs(val - v)
        if best is None or d < best_d or (d == best_d and (c & 1) == 0 and (best & 1) == 1):
            best, best_d = c, d
    return best


def test_e4m3_encode_matches_brute_force():
    rng = np.random.default_rng(1)
    vals = list(rng.normal(0, 50, 400).astype(np.float32))
    vals += list((rng.random(200) * 2 ** -7).astype(np.float32))  # subnormal range
    # exact midpoints between neighbouring codes (ties)
    codes = sorted(_all_finite_codes(), key=lambda c: float(oracle.e4m3_decode(
        torch.tensor([c], dtype=torch.uint8))[0]))
    dec = oracle.e4m3_decode(torch.tensor(codes, dtype=torch.uint8)).tolist()
    mids = [np.float32((a + b) / 2) for a, b in zip(dec, dec[1:]) if a != b]
    vals += mids + [np.float32(x) for x in (449.0, 463.9, 464.0, 1000.0, -1e9, 0.0, -0.0)]
    v = torch.tensor(np.array(vals, dtype=np.float32))
    got = oracle.e4m3_encode(v).tolist()
    want = [_brute_force_e4m3(float(x)) for x in vals]
    assert got == want


def test_e4m3_matches_torch_in_range():
    rng = np.random.default_rng(2)
    v = torch.tensor(np.clip(rng.normal(0, 100, 20000), -448, 448).astype(np.float32))
    ours = oracle.e4m3_encode(v)
    lib = v.to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(ours, lib)


def test_bf16_round_matches_torch_on_floats():
    rng = np.random.default_rng(3)
    f = rng.normal(0, 1, 20000).astype(np.float32)
    # append exact ties: a bf16 value plus half its ulp
    base = torch.tensor(f[:1000]).to(torch.bfloat16).to(torch.float32).numpy()
    ulp = np.abs(base) * 2.0 ** -7
    ties = (base + np.sign(base) * ulp / 2).astype(np.float32)
    f = np.concatenate([f, ties, np.array([1e-40, -3e-39, 3e38], np.float32)])
    ours = oracle.bf16_round(torch.tensor(f, dtype=torch.float64))
    lib = torch.tensor(f).to(torch.bfloat16)
    assert torch.equal(ours.view(torch.int16), lib.view(torch.int16))


def test_bf16_round_ties_to_even_from_double():
    v = torch.tensor([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40, -2.5,
                      2.0 ** 128, 0.0], dtype=torch.float64)
    out = oracle.bf16_round(v).to(torch.float64).tolist()
    assert out[0] == 1.0                       # tie, even mantissa stays
    assert out[1] == 1 + 2.0 ** -6             # tie, odd mantissa rounds up
    assert out[2] == 1 + 2.0 ** -7             # just above the tie rounds up
    assert out[3] == -2.5
    assert math.isinf(out[4])
    assert out[5] == 0.0
