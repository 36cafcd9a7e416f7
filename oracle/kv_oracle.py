"""HLWQ Q3 KV-cache quantizer, CPU oracle -- TEST INFRASTRUCTURE, not part of
the product (the same rules as hlwq_oracle apply: only tests/, the smoke check
and bench.py's CPU legs use it; it shares no code with the CUDA library).

What it computes ("Qwopus3.6-27B-v2 . HLWQ Q5" model card, "Methodology
notes", KV-cache bullet: per-head Hadamard 256x256 rotation, 8-centroid (Q3)
Lloyd-Max quantization, bit-packed at 3 bits per scalar, a 128-token residual
buffer of recent tokens kept unquantized; "Architecture": head_dim = 256;
"Gemma-4-26B-A4B-it-HLWQ-Q5", usage: kv_cache_nbits=3):

  per key or value vector x of one head (256 values, bf16):
    n = ||x||_2 (fp64), stored as fp16;
    y = (x / n) @ H256 (+-1 Sylvester), evaluated as (x @ H256) / n; y = 0 if n = 0;
    code_j = nearest of the 8 fp32 Lloyd-Max centroids of N(0,1) (ties low);
    pack 3 bits per code, LSB first: 96 bytes per vector;
  dequantized x_hat = n16 * (c[code] @ H256) / 256;
  attention scores against a query q: s = q . x_hat.

Readings where the pages are silent (pinned in tests/test_oracle_kv.py):
  K1  "Hadamard 256x256" is applied as for the weights (readings R1, R2): the
      +-1 Sylvester matrix in natural order on the unit-norm vector, so the
      rotated entries have unit variance, matching the N(0,1) codebook.
  K2  One norm per (token, head) vector, stored as fp16 (round to nearest
      even), as the weight norms (reading R3).
  K3  The codebook is the 8-level Lloyd-Max quantizer of N(0,1) built as the
      32-level one (reading R7); midpoints between the fp32 centroids; ties to
      the lower index (a zero vector gets code 3 everywhere).
  K4  Pack: code j at bits [3j, 3j + 3) of the vector's little-endian 768-bit
      field, i.e. 8 codes per 3 bytes, LSB first (as reading R6 with 3 bits).
  K5  The 128-token residual buffer of recent tokens kept without
      quantization: the cache of one head is the encoded tokens followed by the window of the
      most recent min(128, total) tokens, kept exactly as given (bf16).  A
      token is encoded when it leaves the window, oldest first
      (kv_window_append), and attention scores cover every cached token in
      order: decoded keys for the encoded ones, the exact keys for the window
      (kv_scores_window).
"""

from __future__ import annotations

import numpy as np

from .hlwq_oracle import _as_f64, codebook_fp32, nearest_centroid, pack_codes, sylvester_hadamard, unpack_codes

HEAD_DIM = 256
KV_BITS = 3
KV_LEVELS = 8
KV_BYTES = HEAD_DIM * KV_BITS // 8   # 96
RESIDUAL_TOKENS = 128

_H256 = sylvester_hadamard(HEAD_DIM).astype(np.float64)


def kv_quantize(X) -> dict:
    """X [N][256] (bf16 / fp32 values widened exactly) -> packed uint8 [N][96],
    norms float16 [N], codes uint8 [N][256], y float64 [N][256]."""
    x = _as_f64(X)
    if x.ndim != 2 or x.shape[1] != HEAD_DIM:
        raise ValueError("X must be [N][256]")
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0.0, n, 1.0)
    y = np.where((n > 0.0)[:, None], (x @ _H256) / safe[:, None], 0.0)
    c32, _, _ = codebook_fp32(KV_LEVELS)
    codes = nearest_centroid(y, c32)
    return {"packed": pack_codes(codes, bits=KV_BITS), "norms": n.astype(np.float16), "codes": codes, "y": y}


def kv_dequantize(packed, norms) -> np.ndarray:
    """x_hat [N][256] in fp64."""
    codes = unpack_codes(np.asarray(packed), bits=KV_BITS)
    c32, _, _ = codebook_fp32(KV_LEVELS)
    vals = c32.astype(np.float64)[codes]
    return (vals @ _H256) / HEAD_DIM * np.asarray(norms).astype(np.float64)[:, None]


def kv_scores(Q, packed, norms) -> np.ndarray:
    """scores [M][N] = Q @ x_hat^T in fp64 (Q widened exactly)."""
    q = _as_f64(Q)
    if q.ndim == 1:
        q = q[None, :]
    return q @ kv_dequantize(packed, norms).T


def kv_window_append(packed, norms, window, x_new, capacity: int = RESIDUAL_TOKENS):
    """The cache after appending the tokens x_new [t][256] (reading K5).

    The window's tokens (oldest first) are followed by the new ones; all but
    the `capacity` most recent leave the window in order and are encoded with
    kv_quantize and appended to (packed, norms).  Returns (packed uint8 [n][96],
    norms float16 [n], window float64 [w][256], w <= capacity)."""
    if capacity < 1:
        raise ValueError("capacity must be >= 1")
    win = _as_f64(window).reshape(-1, HEAD_DIM)
    new = _as_f64(x_new).reshape(-1, HEAD_DIM)
    tokens = np.concatenate([win, new], axis=0)
    leave = max(0, tokens.shape[0] - capacity)
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1, KV_BYTES)
    norms = np.asarray(norms, dtype=np.float16).reshape(-1)
    if leave:
        q = kv_quantize(tokens[:leave])
        packed = np.concatenate([packed, q["packed"]], axis=0)
        norms = np.concatenate([norms, q["norms"]])
    return packed, norms, tokens[leave:]


def kv_scores_window(Q, packed, norms, window) -> np.ndarray:
    """scores [M][n + w] against every cached token in order: the n encoded
    keys (kv_scores) followed by the w window keys, exact (q . k in fp64)."""
    q = _as_f64(Q)
    if q.ndim == 1:
        q = q[None, :]
    win = _as_f64(window).reshape(-1, HEAD_DIM)
    enc = kv_scores(q, packed, norms) if np.asarray(packed).shape[0] else np.zeros((q.shape[0], 0))
    return np.concatenate([enc, q @ win.T], axis=1)
