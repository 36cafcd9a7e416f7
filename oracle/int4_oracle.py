"""HLWQ Q5 -> INT4 re-encoder, CPU oracle -- TEST INFRASTRUCTURE, not part of
the product (the same rules as hlwq_oracle apply: only tests/, the smoke check
and bench.py's CPU legs use it; it shares no code with the CUDA library).

What it computes ("Qwopus3.6-27B-v2 . HLWQ Q5" model card, section "Pipeline":
HLWQ Q5 -> dequantize per-Linear -> INT4 weight-only quantization with groups
of 128 on the 128-aligned Linears; "Architecture": non-128-aligned shapes stay
in the dequantized form; "Why HLWQ INT4 is Better" on the same card: the
rotated-and-cleaned weights are re-encoded to INT4):

  1. w_hat = the HLWQ dequantization of the row (hlwq_oracle.dequantize);
  2. per row and group g of 128 consecutive inputs (the HLWQ block b = g):
       lo = min w_hat, hi = max w_hat over the group,
       s  = bf16(( hi - lo ) / 15),  z = bf16(lo + 0),
       q  = clamp(rint((w_hat - z) / s), 0, 15)   (q = 0 everywhere if s = 0),
     dequantized as z + q * s;
  3. store q two per byte, element 2k in the low nibble of byte k (64 bytes per
     group), s and z as bfloat16 bit patterns.

Readings where the pages are silent (each pinned in tests/test_oracle_int4.py):
  I1  The INT4 format is asymmetric min-max round-to-nearest with 16 levels per
      group of 128 (the plainest reading of "INT4, group size 128"); the format
      of the library the pages name is not reproduced.
  I2  Scale and zero are stored as bfloat16, rounded to nearest even directly
      from the fp64 value; values below the bfloat16 normal range round to a
      signed zero.  A zero minimum is stored as +0 (z = bf16(min + 0.0): the
      minimum of a zero block may be -0 or +0).  The codes are chosen against
      the stored (rounded) s and z.
  I3  Every step is evaluated in fp64.  w_hat is exact in fp64 (sums of 128
      fp32 centroids times +-1, times an fp16 norm / 128), so the decisions are
      reproducible bit for bit by any implementation that evaluates the same
      fp64 operations (min, max, subtract, divide, round half to even).
  I4  Only rows whose length is a multiple of 128 are re-encoded (the pages keep
      the others in the dequantized form).
  I5  Nibble order: element 2k in bits 0-3, element 2k+1 in bits 4-7 of byte k
      (LSB first, as the 5-bit pack of the Q5 codes).
"""

from __future__ import annotations

import numpy as np

from .hlwq_oracle import BLOCK, dequantize

INT4_LEVELS = 16
INT4_GROUP_BYTES = BLOCK // 2  # 64


def bf16_rne_bits(x) -> np.ndarray:
    """bfloat16 bit patterns of fp64 values, rounded to nearest even directly
    from fp64 (no intermediate fp32); magnitudes below 2^-126 give a signed
    zero; finite values only."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.uint16)
    flat = x.reshape(-1)
    res = out.reshape(-1)
    for i, v in enumerate(flat):
        v = float(v)
        sign = 0x8000 if np.signbit(v) else 0
        a = abs(v)
        if a < 2.0 ** -126:
            res[i] = sign
            continue
        m, e = np.frexp(a)            # a = m * 2^e, m in [0.5, 1)
        sig = float(np.rint(m * 256.0))   # 8 significant bits, ties to even
        if sig == 256.0:
            sig, e = 128.0, e + 1
        exp8 = e - 1 + 127           # a = (sig / 128) * 2^(e - 1)
        if exp8 >= 255:
            raise ValueError("value beyond the bfloat16 range")
        res[i] = sign | (exp8 << 7) | (int(sig) - 128)
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def pack_int4(q) -> np.ndarray:
    """[..., 128] codes 0..15 -> [..., 64] bytes, element 2k in the low nibble."""
    q = np.asarray(q, dtype=np.uint8)
    if np.any(q > 15):
        raise ValueError("INT4 codes are 0..15")
    return (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 15
    out[..., 1::2] = b >> 4
    return out


def int4_encode_groups(w) -> dict:
    """Step 2 on fp64 values w [..., 128] (one group per last-axis row)."""
    w = np.asarray(w, dtype=np.float64)
    lo = w.min(axis=-1)
    hi = w.max(axis=-1)
    s_bits = bf16_rne_bits((hi - lo) / 15.0)
    z_bits = bf16_rne_bits(lo + 0.0)  # -0 -> +0 (reading I2)
    s = bf16_bits_to_f64(s_bits)[..., None]
    z = bf16_bits_to_f64(z_bits)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.clip(np.rint((w - z) / s), 0, 15)
    q = np.where(s > 0.0, q, 0.0).astype(np.uint8)
    return {"q": q, "scale": s_bits, "zero": z_bits}


def requantize_int4(packed, norms, in_features: int) -> dict:
    """HLWQ Q5 (packed [O][NB][80], norms fp16 [O][NB]) of a 128-aligned matrix
    -> INT4: q4 uint8 [O][NB][64], scale / zero bf16 bits uint16 [O][NB], plus
    the codes [O][NB][128] and w_hat [O][NB][128] for the tests."""
    if in_features % BLOCK:
        raise ValueError("the INT4 re-encoding covers 128-aligned rows only")
    w_hat = dequantize(packed, norms, in_features)
    O = w_hat.shape[0]
    g = w_hat.reshape(O, in_features // BLOCK, BLOCK)
    enc = int4_encode_groups(g)
    return {"q4": pack_int4(enc["q"]), "scale": enc["scale"], "zero": enc["zero"], "codes": enc["q"],
            "w_hat": g}


def dequantize_int4(q4, scale_bits, zero_bits) -> np.ndarray:
    """z + q * s per group, fp64, [O][NB * 128]."""
    q = unpack_int4(q4).astype(np.float64)
    s = bf16_bits_to_f64(scale_bits)[..., None]
    z = bf16_bits_to_f64(zero_bits)[..., None]
    w = z + q * s
    return w.reshape(w.shape[0], -1)
