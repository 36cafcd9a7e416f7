"""Pins for the oracle's Hadamard, nearest-centroid, pack, quantize and
dequantize steps (Method steps [1]-[5] of the "Qwen3.6-35B-A3B -- HLWQ Q5" model
card; rotation and 0.625 B/weight from the "Qwopus3.6-27B-v2 . HLWQ Q5"
Methodology notes; cos_sim > 0.996 from the "Gemma-4-26B-A4B-it-HLWQ-Q5" card,
section "Method: HLWQ")."""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- Hadamard
def test_hadamard_is_sylvester_kron():
    h2 = np.array([[1, 1], [1, -1]], dtype=np.int64)
    h = np.array([[1]], dtype=np.int64)
    for _ in range(7):
        h = np.kron(h2, h)
    assert np.array_equal(O.sylvester_hadamard(128).astype(np.int64), h)


def test_hadamard_orthogonal_symmetric():
    h = O.sylvester_hadamard(128).astype(np.int64)
    assert np.array_equal(h @ h.T, 128 * np.eye(128, dtype=np.int64))
    assert np.array_equal(h, h.T)
    assert np.all(h[0] == 1) and np.all(h[:, 0] == 1)


# ---------------------------------------------------------------- nearest centroid
def test_nearest_centroid_equals_midpoint_count():
    """Brute-force argmin (ties low) == number of exact midpoints strictly below y,
    on random values, on every midpoint, and one fp64 ulp either side of the
    non-zero midpoints (next to 0 the fp64 distances themselves round to a tie,
    so the probes there are +-1e-15)."""
    c32, mid64, _ = O.codebook_fp32()
    y = synth.uniform(200_000, -5.0, 5.0, seed=7)
    nz = mid64[mid64 != 0]
    probes = np.concatenate([y, mid64, np.nextafter(nz, np.inf), np.nextafter(nz, -np.inf),
                             [0.0, -0.0, 1e-15, -1e-15, 50.0, -50.0]])
    count = (probes[:, None] > mid64[None, :]).sum(axis=1)
    assert np.array_equal(O.nearest_centroid(probes, c32), count)


def test_tie_goes_low():
    c32, mid64, _ = O.codebook_fp32()
    assert O.nearest_centroid(np.array([0.0]), c32)[0] == 15
    for k in range(31):
        assert O.nearest_centroid(np.array([mid64[k]]), c32)[0] == k


# ---------------------------------------------------------------- pack
def _golden_pack():
    rows = []
    with open(os.path.join(GOLDEN, "pack_5bit_lsb_first.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split(";")
            rows.append(([int(v) for v in a.split()], bytes(int(v, 16) for v in b.split())))
    return rows


def test_pack_golden_bytes():
    rows = _golden_pack()
    assert len(rows) >= 5
    for codes, want in rows:
        block = np.zeros(128, dtype=np.uint8)
        block[:8] = codes
        got = O.pack_codes(block)
        assert got.shape == (80,)
        assert bytes(got[:5]) == want
        assert not got[5:].any()
        # the same group in the last slot of the block lands in the last 5 bytes
        block2 = np.zeros(128, dtype=np.uint8)
        block2[120:] = codes
        assert bytes(O.pack_codes(block2)[75:]) == want


def test_pack_round_trip_every_slot_value():
    for slot in range(128):
        for v in range(32):
            codes = np.zeros(128, dtype=np.uint8)
            codes[slot] = v
            assert np.array_equal(O.unpack_codes(O.pack_codes(codes)), codes)


def test_pack_round_trip_random_groups():
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 32, size=(1 << 15, 128), dtype=np.uint8)  # 2^22 random groups of 8
    packed = O.pack_codes(codes)
    assert packed.shape == (1 << 15, 80)
    assert packed.nbytes / codes.size == 0.625
    assert np.array_equal(O.unpack_codes(packed), codes)
    for v in range(32):
        assert np.array_equal(O.unpack_codes(O.pack_codes(np.full(128, v, np.uint8))), np.full(128, v))


# ---------------------------------------------------------------- fp16 norm rounding
def _fp16_rne_exact(x: float) -> float:
    """Exact rational round-to-nearest-even to fp16 (normal range)."""
    fx = Fraction(x)
    e = fx.numerator.bit_length() - fx.denominator.bit_length()
    while Fraction(2) ** e > fx:
        e -= 1
    while Fraction(2) ** (e + 1) <= fx:
        e += 1
    ulp = Fraction(2) ** (e - 10)
    q, r = divmod(fx, ulp)
    if r * 2 > ulp or (r * 2 == ulp and q % 2 == 1):
        q += 1
    return float(q * ulp)


def test_numpy_fp16_conversion_is_rne_from_fp64():
    vals = []
    for h in np.arange(0x1000, 0x7b00, 37, dtype=np.uint16):
        a = float(h.view(np.float16))
        b = float(np.uint16(h + 1).view(np.float16))
        m = (a + b) / 2
        vals += [m, np.nextafter(m, np.inf), np.nextafter(m, -np.inf), a]
    for v in vals:
        assert float(np.float16(v)) == _fp16_rne_exact(v), v


# ---------------------------------------------------------------- whole quantizer
@pytest.fixture(scope="module")
def gauss_q():
    w = synth.gaussian_with_outliers(64, 512, seed=0)
    return w, O.quantize(w, return_rotated=True)


def test_rotated_norm_is_sqrt128(gauss_q):
    _, q = gauss_q
    ss = (q["y"] ** 2).sum(axis=-1)
    assert np.allclose(ss, 128.0, rtol=0, atol=1e-9)


def test_rotated_mse_matches_lloyd(gauss_q):
    w = synth.student_t((256, 1024), dtype=torch.float32, df4_seed=5)
    q = O.quantize(w, return_rotated=True)
    c32, _, _ = O.codebook_fp32()
    err = (q["y"] - c32.astype(np.float64)[q["codes"]]) ** 2
    d = O.lloyd_max_gaussian(32)["mse"]
    assert abs(err.mean() - d) / d < 0.05


def test_cosine_above_0996():
    for w in (synth.gaussian_with_outliers(256, 512, seed=0),
              synth.student_t((256, 640), dtype=torch.bfloat16, df4_seed=3)):
        q = O.quantize(w)
        w_hat = O.dequantize(q["packed"], q["norms"], w.shape[1])
        assert O.cosine_similarity(w_hat, w) > 0.996


def test_sizes_and_dtypes():
    w = synth.student_t((16, 704), dtype=torch.bfloat16, df4_seed=1)   # 5.5 blocks
    q = O.quantize(w)
    assert q["packed"].shape == (16, 6, 80) and q["packed"].dtype == np.uint8
    assert q["norms"].shape == (16, 6) and q["norms"].dtype == np.float16
    assert O.dequantize(q["packed"], q["norms"], 704).shape == (16, 704)


def test_tail_padding_does_not_change_norm():
    w = synth.student_t((8, 704), dtype=torch.float32, df4_seed=2)
    q = O.quantize(w)
    tail = w[:, 640:].double().numpy()
    want = np.sqrt((tail ** 2).sum(axis=1)).astype(np.float16)
    assert np.array_equal(q["norms"][:, 5], want)


def test_zero_block():
    w = torch.zeros(2, 256)
    w[1, 128:] = 0.03
    q = O.quantize(w)
    assert np.all(q["codes"][0] == 15) and np.all(q["norms"][0] == 0)
    assert np.all(q["codes"][1, 0] == 15)
    assert np.all(O.dequantize(q["packed"], q["norms"], 256)[0] == 0)


def test_spike_block():
    """w = a e_i -> y_j = sign(a) H[i][j]: every entry is +-1."""
    for i in (0, 5, 127):
        w = torch.zeros(1, 128)
        w[0, i] = -0.7
        q = O.quantize(w, return_rotated=True)
        h = O.sylvester_hadamard(128)[i].astype(np.float64)
        assert np.allclose(q["y"][0, 0], -h, atol=1e-15)
        c32, _, _ = O.codebook_fp32()
        nearest_plus_one = int(np.argmin(np.abs(c32.astype(np.float64) - 1.0)))
        assert np.all(q["codes"][0, 0] == np.where(h > 0, 31 - nearest_plus_one, nearest_plus_one))


def test_constant_block():
    """w = a * ones -> y = sqrt(128) e_0: code 31 at j=0, ties (y=0) -> 15 elsewhere."""
    q = O.quantize(torch.full((1, 128), 0.01), return_rotated=True)
    assert q["y"][0, 0, 0] == pytest.approx(np.sqrt(128.0), abs=1e-12)
    assert q["codes"][0, 0, 0] == 31 and np.all(q["codes"][0, 0, 1:] == 15)


def test_dequant_requantize_fixed_point():
    w = synth.student_t((32, 256), dtype=torch.float32, df4_seed=9)
    q = O.quantize(w)
    w_hat = O.dequantize(q["packed"], q["norms"], 256)
    q2 = O.quantize(w_hat)
    assert np.array_equal(q2["codes"], q["codes"])


def test_power_of_two_scaling():
    w = synth.student_t((32, 384), dtype=torch.float32, df4_seed=4)
    q = O.quantize(w)
    for k in (-3, 4):
        qk = O.quantize(w * 2.0 ** k)
        assert np.array_equal(qk["codes"], q["codes"])
        assert np.array_equal(qk["norms"].astype(np.float64), q["norms"].astype(np.float64) * 2.0 ** k)


def test_quantize_is_deterministic():
    w = synth.student_t((8, 256), df4_seed=6)
    a, b = O.quantize(w), O.quantize(w)
    assert np.array_equal(a["packed"], b["packed"]) and np.array_equal(a["norms"], b["norms"])


def test_relative_reconstruction_error_is_lloyd_mse():
    """H/sqrt(128) is orthonormal, so ||w_hat - w||^2 / ||w||^2 equals the mean
    squared quantization error in the rotated domain (per unit variance) up to
    the fp16 norm rounding: about D_32.  Catches a wrong dequantization scale,
    which the (scale-free) cosine check cannot."""
    w = synth.student_t((256, 1024), dtype=torch.float32, df4_seed=12)
    q = O.quantize(w)
    w_hat = O.dequantize(q["packed"], q["norms"], 1024)
    wd = w.double().numpy()
    rel = ((w_hat - wd) ** 2).sum() / (wd ** 2).sum()
    d = O.lloyd_max_gaussian(32)["mse"]
    assert abs(rel - d) / d < 0.05


def test_exact_ties_resolve_low():
    """Constant blocks: 127 rotated values are exactly 0 (a tie between codes 15
    and 16 under the symmetric codebook) and must all take code 15."""
    for v in (0.01, -0.02, 0.3):
        q = O.quantize(torch.full((2, 256), v), return_rotated=True)
        assert np.all(q["y"][..., 1:] == 0.0)
        assert np.all(q["codes"][..., 1:] == 15)
