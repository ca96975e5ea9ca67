"""Pins of the oracle's FP8 combine payload: per-128 block e4m3 quantisation
of y (scale = amax / 448, codes e4m3(y * (1 / scale))) and the combine that
dequantises it.

Source: "Expert parallelism and all-to-all", "Traffic math": 1-byte
activations both ways (dispatch and combine).
"""
import torch

import oracle


def _dequant(q, sc):
    """torch's own e4m3 decode times the block scale, as an fp32 product."""
    return q.float() * sc.repeat_interleave(128, dim=1)


def test_codes_equal_torch_e4m3_of_the_scaled_values():
    g = torch.Generator().manual_seed(21)
    v = torch.randn(64, 512, generator=g) * torch.logspace(-3, 3, 64).unsqueeze(1)
    q, sc = oracle.quantize_rows_e4m3(v)
    amax = v.abs().view(64, 4, 128).amax(dim=2)
    assert torch.equal(sc, amax / 448.0)                    # fp32 IEEE division
    recip = 1.0 / sc                                        # one IEEE division per block
    scaled = v * recip.repeat_interleave(128, dim=1)        # every |value| <= 448 (+ rounding)
    ref = scaled.clamp(-448, 448).to(torch.float8_e4m3fn)   # torch: round to nearest even
    assert torch.equal(q.view(torch.uint8), ref.view(torch.uint8))


def test_block_maximum_and_zero_blocks():
    v = torch.zeros(2, 256)
    v[0, :128] = torch.linspace(-3.0, 7.0, 128)
    v[0, 5] = -448.0 * 4                                    # amax = 448 * 2^2
    q, sc = oracle.quantize_rows_e4m3(v)
    assert float(sc[0, 0]) == 4.0 and q.view(torch.uint8)[0, 5].item() == 0xFE   # -448
    assert float(sc[0, 1]) == 1.0 and float(sc[1, 0]) == 1.0                      # zero blocks
    assert bool((q.view(torch.uint8)[1] == 0).all())


def test_quantisation_error_is_within_half_a_code_step():
    g = torch.Generator().manual_seed(22)
    v = torch.randn(32, 384, generator=g)
    q, sc = oracle.quantize_rows_e4m3(v)
    s = sc.repeat_interleave(128, dim=1)
    err = (_dequant(q, sc) - v).abs() / s
    mag = (v / s).abs()
    # e4m3 spacing: 2^(e-3) for normal values of exponent e, 2^-9 below 2^-6
    e = torch.floor(torch.log2(mag.clamp(min=2.0 ** -6)))
    step = torch.where(mag >= 2.0 ** -6, 2.0 ** (e - 3), torch.full_like(mag, 2.0 ** -9))
    assert bool((err <= step / 2 * (1 + 1e-6)).all())


def test_combine_of_identity_experts_returns_the_dequantised_rows():
    """y = x for every pick and weights 1/2, 1/2: out is exactly the fp32
    product decode(q) * scale of x's row."""
    g = torch.Generator().manual_seed(23)
    T, k, H = 40, 2, 256
    x = torch.randn(T, H, generator=g)
    q, sc = oracle.quantize_rows_e4m3(x)
    sop = torch.arange(T * k, dtype=torch.int32) // k      # both picks read the token's row
    w = torch.full((T, k), 0.5)
    out = oracle.combine_e4m3(q, sc, sop, w)
    assert torch.equal(out, _dequant(q, sc).double())


def test_combine_equals_the_plain_combine_of_the_dequantised_rows():
    g = torch.Generator().manual_seed(24)
    T, k, H, S = 30, 3, 128, 100
    y = torch.randn(S, H, generator=g) * 3
    q, sc = oracle.quantize_rows_e4m3(y)
    sop = torch.randint(-1, S, (T * k,), generator=g, dtype=torch.int32)   # -1: dropped
    w = torch.rand(T, k, generator=g)
    out = oracle.combine_e4m3(q, sc, sop, w)
    ref = oracle.combine(_dequant(q, sc), sop, w)
    assert torch.equal(out, ref)
