"""TQ3 (the scalar case of HIGGS) weight quantizer, CPU oracle -- TEST
INFRASTRUCTURE, not part of the product (the same rules as hlwq_oracle apply:
only tests/, the smoke check and bench.py's CPU legs use it; it shares no code
with the CUDA library).

What it computes ("Qwen3.6-35B-A3B-TQ3-native" model card, "What TQ3 actually
does": a Walsh-Hadamard rotation of every group of 128 weights made of two
random sign vectors and an in-place FWHT, an 8-entry Lloyd-Max codebook for a
unit Gaussian, and a shape-gain norm per group equal to the original norm over
the reconstruction norm; "Files": uint8 packed codes and float32 norms per
weight; the quantizer state is bits = 3, group_size = 128 and a seed):

  per row and group g of 128 inputs (the tail group zero-padded):
    n      = ||g||_2 (fp64);
    y      = s2 * (H128 (s1 * g)) / n       (y = 0 if n = 0)
    code_j = nearest of the 8 fp32 Lloyd-Max centroids of N(0,1) (ties low);
    r      = sqrt(||c[code]||^2 / 128)       the norm of the reconstructed unit vector
    gamma  = n / r, stored as float32        (0 for a zero group)
    pack 3 bits per code, LSB first: 48 bytes per group;
  dequantized group  w_hat = gamma * s1 * (H128 (s2 * c[code])) / 128,
  so that ||w_hat|| = n up to the float32 rounding of gamma;
  the matmul is Y = X @ W_hat^T.

Readings where the pages are silent (pinned in tests/test_oracle_tq3.py):
  T1  The rotation is: multiply by the first sign vector, FWHT (the +-1
      Sylvester H128 in natural order), multiply by the second; it acts on the
      unit-norm group, so the entries of y have unit variance and meet the N(0,1)
      codebook (as readings R1, R2 of the Q5 method).
  T2  One pair of sign vectors (s1, s2), each 128 values of +-1, serves every
      group of every matrix (the stored state is one seed).  The generator that
      turns the seed into signs is not given, so the signs are an input here.
  T3  The codebook is the 8-level Lloyd-Max quantizer of N(0,1) (reading R7),
      nearest centroid with ties to the lower index (a zero group: code 3).
  T4  "Reconstruction norm" is the norm of the reconstructed unit vector,
      ||c[code]|| / sqrt(128); gamma = n / that is what dequantization
      multiplies by.  ||c[code]||^2 is evaluated as sum_l m_l * c_l^2 over the
      8 levels in ascending order (m_l = how many codes equal l), in fp64.
  T5  Pack: code j of a group at bits [3j, 3j + 3) of its 48 bytes, LSB first
      (as reading R6 with 3 bits); layout [rows][NB][48], norms [rows][NB].
  T6  Rows whose length is not a multiple of 128 are zero-padded to the next
      group, as in step [1] of the Q5 method; dequantization drops the pad.
"""

from __future__ import annotations

import numpy as np

from .hlwq_oracle import BLOCK, _as_f64, codebook_fp32, n_blocks, nearest_centroid, pack_codes, sylvester_hadamard, \
    unpack_codes

TQ3_BITS = 3
TQ3_LEVELS = 8
TQ3_GROUP_BYTES = BLOCK * TQ3_BITS // 8   # 48

_H = sylvester_hadamard(BLOCK).astype(np.float64)


def _signs(s) -> np.ndarray:
    s = np.asarray(s)
    if s.shape != (BLOCK,) or not np.all(np.abs(s) == 1):
        raise ValueError("a sign vector is 128 values of +-1")
    return s.astype(np.float64)


def tq3_rotate(G, s1, s2) -> np.ndarray:
    """Reading T1 on raw groups: s2 * (H128 (s1 * g)) for each row g of G."""
    return ((np.asarray(G, np.float64) * _signs(s1)) @ _H) * _signs(s2)


def tq3_unrotate(Y, s1, s2) -> np.ndarray:
    """The inverse of tq3_rotate: s1 * (H128 (s2 * y)) / 128 (H128 H128 = 128 I)."""
    return ((np.asarray(Y, np.float64) * _signs(s2)) @ _H) * _signs(s1) / BLOCK


def _groups(W) -> np.ndarray:
    w = _as_f64(W)
    if w.ndim != 2:
        raise ValueError("W must be [rows][in]")
    rows, in_f = w.shape
    nb = n_blocks(in_f)
    pad = np.zeros((rows, nb * BLOCK), np.float64)
    pad[:, :in_f] = w
    return pad.reshape(rows, nb, BLOCK)


def reconstruction_sq(codes) -> np.ndarray:
    """||c[code]||^2 per group, as reading T4: sum over the levels l = 0..7 in
    order of (count of code l) * c_l^2, in fp64."""
    c32, _, _ = codebook_fp32(TQ3_LEVELS)
    codes = np.asarray(codes)
    acc = np.zeros(codes.shape[:-1], np.float64)
    for level in range(TQ3_LEVELS):
        cnt = (codes == level).sum(axis=-1).astype(np.float64)
        cl = np.float64(c32[level])
        acc = acc + cnt * (cl * cl)
    return acc


def tq3_quantize(W, s1, s2) -> dict:
    """W [rows][in] (bf16 / fp32 values, widened exactly) -> packed uint8
    [rows][NB][48], norms float32 [rows][NB] (gamma), codes uint8 [rows][NB][128],
    y float64 [rows][NB][128], n float64 [rows][NB] (the original norms)."""
    g = _groups(W)
    n = np.sqrt(np.sum(g * g, axis=-1))
    safe = np.where(n > 0.0, n, 1.0)
    y = np.where((n > 0.0)[..., None], tq3_rotate(g, s1, s2) / safe[..., None], 0.0)
    c32, _, _ = codebook_fp32(TQ3_LEVELS)
    codes = nearest_centroid(y, c32)
    r = np.sqrt(reconstruction_sq(codes) / BLOCK)
    gamma = np.where(n > 0.0, n / r, 0.0)
    return {"packed": pack_codes(codes, bits=TQ3_BITS), "norms": gamma.astype(np.float32), "codes": codes, "y": y,
            "n": n}


def tq3_dequantize(packed, norms, in_features: int, s1, s2) -> np.ndarray:
    """W_hat [rows][in] in fp64 (the pad dropped)."""
    codes = unpack_codes(np.asarray(packed), bits=TQ3_BITS)
    c32, _, _ = codebook_fp32(TQ3_LEVELS)
    vals = c32.astype(np.float64)[codes]
    w = tq3_unrotate(vals, s1, s2) * np.asarray(norms, np.float64)[..., None]
    rows = w.shape[0]
    return w.reshape(rows, -1)[:, :in_features]


def tq3_matmul(packed, norms, in_features: int, s1, s2, X) -> np.ndarray:
    """Y [M][rows] = X @ W_hat^T in fp64 (X widened exactly)."""
    x = _as_f64(X)
    if x.ndim == 1:
        x = x[None, :]
    return x @ tq3_dequantize(packed, norms, in_features, s1, s2).T
