"""Pins of the INT4 re-encoding oracle (oracle/int4_oracle.py) to facts that do
not come from the oracle itself: exact arithmetic, the definition of
round-to-nearest-even, a hand-computed nibble layout, brute-force nearest
levels and error bounds."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O


def _layer(rows, cols, seed):
    g = np.random.default_rng(seed)
    W = (g.standard_t(4, size=(rows, cols)) * 0.02 / np.sqrt(2)).astype(np.float32)
    return W, O.quantize(W)


def test_dequantized_values_are_exact_in_fp64():
    """Reading I3: w_hat = (n16 / 128) * sum_j c[k_j] H[j][i] is exactly
    representable in fp64, so every fp64 evaluation order gives the same value
    (checked against exact rational arithmetic)."""
    _, q = _layer(3, 256, 5)
    w_hat = O.dequantize(q["packed"], q["norms"], 256)
    c32, _, _ = O.codebook_fp32()
    codes = O.unpack_codes(q["packed"])
    H = O.sylvester_hadamard()
    rng = np.random.default_rng(0)
    for _ in range(40):
        o, b, i = rng.integers(3), rng.integers(2), rng.integers(128)
        n = Fraction(float(q["norms"][o, b]))
        s = sum(Fraction(float(c32[codes[o, b, j]])) * int(H[j, i]) for j in range(128))
        assert Fraction(float(w_hat[o, 128 * b + i])) == n * s / 128


def test_bf16_rounding_is_direct_nearest_even():
    """Reading I2: bf16 = round to nearest even of the fp64 value itself."""
    assert O.bf16_rne_bits([1.0, -2.0, 0.0])[0] == 0x3F80
    assert O.bf16_rne_bits([-2.0])[0] == 0xC000
    assert O.bf16_rne_bits([1.0 + 2.0 ** -8])[0] == 0x3F80          # tie -> even (down)
    assert O.bf16_rne_bits([1.0 + 3 * 2.0 ** -8])[0] == 0x3F82      # tie -> even (up)
    # just above a tie: direct rounding goes up; fp64 -> fp32 -> bf16 would
    # first drop the 2^-30 and then round the tie down to 0x3F80
    assert O.bf16_rne_bits([1.0 + 2.0 ** -8 + 2.0 ** -30])[0] == 0x3F81
    assert O.bf16_rne_bits([2.0 ** -130])[0] == 0x0000
    assert O.bf16_rne_bits([-(2.0 ** -130)])[0] == 0x8000
    # fp32-representable values: equal to torch's float32 -> bfloat16 (RNE)
    x = (np.random.default_rng(1).standard_normal(20000) * 0.03).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(O.bf16_rne_bits(x.astype(np.float64)), want)
    # and back: bits -> value is exact
    assert np.array_equal(O.bf16_bits_to_f64(want), torch.from_numpy(x).to(torch.bfloat16).double().numpy())


def test_int4_nibble_layout_hand_computed():
    """Reading I5: element 2k in the low nibble of byte k."""
    q = np.concatenate([np.arange(16), np.arange(15, -1, -1)] * 4).astype(np.uint8)
    b = O.pack_int4(q)
    assert b.shape == (64,)
    assert list(b[:8]) == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]
    assert list(b[8:16]) == [0xEF, 0xCD, 0xAB, 0x89, 0x67, 0x45, 0x23, 0x01]
    assert np.array_equal(O.unpack_int4(b), q)
    with pytest.raises(ValueError):
        O.pack_int4(np.full(128, 16))


def test_int4_codes_are_the_nearest_level():
    """Each code is the nearest of the 16 levels z + k s (brute force), except
    at an exact half-way point, where round-half-to-even decides."""
    _, q = _layer(16, 1024, 7)
    r = O.requantize_int4(q["packed"], q["norms"], 1024)
    w = r["w_hat"]
    s = O.bf16_bits_to_f64(r["scale"])[..., None]
    z = O.bf16_bits_to_f64(r["zero"])[..., None]
    levels = z[..., None] + np.arange(16) * s[..., None]        # [O][NB][1][16]
    d = np.abs(w[..., None] - levels)
    best = d.argmin(axis=-1)
    tie = np.sort(d, axis=-1)[..., 1] == d.min(axis=-1)
    assert np.all((best == r["codes"]) | tie)
    assert np.all(s > 0)


def test_int4_error_bound_and_range_ends():
    """|w - (z + q s)| <= s / 2 plus the bf16 rounding of z and s (clamping);
    the group's minimum maps to 0 and its maximum to 15 when the range is not
    tiny against the values."""
    _, q = _layer(32, 512, 9)
    r = O.requantize_int4(q["packed"], q["norms"], 512)
    w = r["w_hat"]
    lo, hi = w.min(-1), w.max(-1)
    s = O.bf16_bits_to_f64(r["scale"])
    z = O.bf16_bits_to_f64(r["zero"])
    back = O.dequantize_int4(r["q4"], r["scale"], r["zero"]).reshape(w.shape)
    slack = 0.5 * s + np.abs(lo - z) + 15 * np.abs((hi - lo) / 15 - s) + 1e-15
    assert np.all(np.abs(back - w) <= slack[..., None])
    wide = (hi - lo) > 0.2 * np.maximum(np.abs(lo), np.abs(hi))
    codes = r["codes"]
    amin, amax = w.argmin(-1), w.argmax(-1)
    cmin = np.take_along_axis(codes, amin[..., None], -1)[..., 0]
    cmax = np.take_along_axis(codes, amax[..., None], -1)[..., 0]
    assert wide.mean() > 0.9
    assert np.all(cmin[wide] == 0) and np.all(cmax[wide] == 15)


def test_int4_constant_group_and_zero_block():
    """A constant group has s = 0: every code is 0 and the group decodes to
    bf16(value).  A zero HLWQ block (norm 0) decodes to exact zeros."""
    enc = O.int4_encode_groups(np.full((2, 128), 0.3))
    assert np.all(enc["q"] == 0) and np.all(enc["scale"] == 0)
    assert np.all(O.bf16_bits_to_f64(enc["zero"]) == O.bf16_bits_to_f64(O.bf16_rne_bits([0.3]))[0])
    W = np.zeros((2, 256), np.float32)
    W[1, 128:] = np.linspace(-0.05, 0.05, 128, dtype=np.float32)
    q = O.quantize(W)
    r = O.requantize_int4(q["packed"], q["norms"], 256)
    back = O.dequantize_int4(r["q4"], r["scale"], r["zero"])
    assert np.all(back[0] == 0.0) and np.all(back[1, :128] == 0.0)
    # the zero block's minimum is a signed zero: stored as +0 (reading I2)
    assert np.all(r["zero"][0] == 0x0000) and np.all(r["scale"][0] == 0x0000)


def test_int4_only_for_aligned_rows():
    """Reading I4: rows whose length is not a multiple of 128 stay in the
    dequantized form."""
    W = np.zeros((2, 704), np.float32)
    q = O.quantize(W)
    with pytest.raises(ValueError):
        O.requantize_int4(q["packed"], q["norms"], 704)


def test_int4_keeps_the_weights():
    """On Gaussian weights the re-encoding error follows the uniform-noise model
    of a 16-level quantizer: total squared error within 15 % of
    sum over groups of 128 s^2 / 12, and cosine to the HLWQ weights ~0.995."""
    g = np.random.default_rng(11)
    W = (g.standard_normal((64, 1024)) * 0.02).astype(np.float32)
    q = O.quantize(W)
    r = O.requantize_int4(q["packed"], q["norms"], 1024)
    a = r["w_hat"].reshape(64, -1)
    b = O.dequantize_int4(r["q4"], r["scale"], r["zero"])
    err = float(((a - b) ** 2).sum())
    model = float((128 * O.bf16_bits_to_f64(r["scale"]) ** 2 / 12).sum())
    assert abs(err / model - 1) < 0.15, err / model
    assert float((a * b).sum() / np.linalg.norm(a) / np.linalg.norm(b)) > 0.994


def test_int4_hand_computed_group():
    """w = -0.3 + 0.1 k for k = 0..15 (eight copies each): lo = -0.3, hi = 1.2,
    s = bf16(1.5 / 15) = 0x3DCD (0.10009765625), z = bf16(-0.3) = 0xBE9A
    (-0.30078125, mantissa round(0.2 * 128) = 26), and the code of -0.3 + 0.1 k
    is k (e.g. k = 15: 1.50078125 / 0.10009765625 = 14.993 -> 15)."""
    k = np.repeat(np.arange(16), 8)
    enc = O.int4_encode_groups((-0.3 + 0.1 * k)[None, :])
    assert int(enc["scale"][0]) == 0x3DCD
    assert int(enc["zero"][0]) == 0xBE9A
    assert np.array_equal(enc["q"][0], k.astype(np.uint8))
