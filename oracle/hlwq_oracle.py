"""HLWQ Q5 CPU oracle -- TEST INFRASTRUCTURE, not part of the product.

A plain, slow, fp64 restatement of what Hadamard-Lloyd Weight Quantization (Q5)
computes, written from the model cards that describe it:

  * "Qwen3.6-35B-A3B -- HLWQ Q5" model card, section "Method": the five-step
    diagram (block reshape -> per-block L2 normalise, norms saved -> Walsh-Hadamard
    rotation "blocks @ H128 x sqrt(128)" -> Lloyd-Max 5-bit quantization with 32
    centroids for N(0,1) -> 5-bit pack, 8 codes into 5 bytes), and the stored
    tensors __packed / __norms / __meta;
  * "Qwopus3.6-27B-v2 . HLWQ Q5" model card, "Methodology notes", weight
    quantization bullet: rotation by a 128x128 Walsh-Hadamard matrix scaled by
    sqrt(128), nearest of 32 Lloyd-Max centroids computed for a unit Gaussian,
    0.625 byte per weight; "Pipeline": the per-Linear dequantisation;
    "Architecture": non-128-aligned Linears exist;
  * "Gemma-4-26B-A4B-it-HLWQ-Q5", "Technical Details": experts quantized
    independently, fp16 norms;
  * "Qwen3.6-35B-A3B -- HLWQ Q5", tables "Architecture" and metrics: 8 routed +
    1 shared expert per token.

Who may use this module: only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference leg.  The product path (the CUDA library and its Python
binding) never imports it, and it imports nothing from the product: the two
share no code.  Its only inputs are arrays (numpy or CPU torch tensors).

Readings taken where the pages are silent (each also pinned by a test):
  R1  "H128 x sqrt(128)" is the orthonormal Hadamard times sqrt(128), i.e. the
      +-1 Sylvester matrix H[i][j] = (-1)^popcount(i & j).  A unit-norm block
      then has entries of unit variance, matching the N(0,1) codebook.
  R2  Natural (Sylvester) row order; row vector times H (H is symmetric).
  R3  Normalise by the exact norm; store it as fp16 (round to nearest even);
      dequantise with the stored fp16 value.
  R4  A zero block has y = 0, which is equidistant from the two centre
      centroids; ties go to the lower index (code 15); its stored norm is 0.
  R5  Tail block zero-padded to 128 before the norm; padded positions are
      encoded and stored, and dropped on dequantisation.
  R6  Pack: code j of a block sits at bits [5j, 5j+5) of the block's 640-bit
      little-endian field, i.e. 8 consecutive codes per 40-bit group, LSB first;
      each block is 80 bytes; blocks in row order.
  R7  Lloyd iteration starts at the Gaussian quantiles (k+1/2)/L and is
      symmetrised every step; the fp32 codebook is the fp64 fixed point rounded
      to nearest; decision midpoints are taken between the fp32 centroids.
  R8  MoE: softmax over the k selected router logits; ties in selection go to
      the lower expert id; gate rows [0, F), up rows [F, 2F); h = SiLU(g) * u;
      the shared expert is added with weight 1.

Parity: pinned as listed in tests/test_oracle_*.py.  Beyond those pins parity is
unpinned: the pages print no worked example or golden output.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 128          # block width (Method step [1])
BITS = 5             # bits per code (Method step [5])
LEVELS = 32          # centroids (Method step [4])
GROUP = 8            # codes per 40-bit group (Method step [5]: 8 codes -> 5 bytes)
BLOCK_BYTES = BLOCK * BITS // 8   # 80


# --------------------------------------------------------------------------
# Standard normal helpers (pdf, upper tail, cell probability) in fp64.
# --------------------------------------------------------------------------

def _pdf(x: float) -> float:
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _upper_tail(x: float) -> float:
    """P(Z > x) for Z ~ N(0,1), via erfc (accurate in the far tail)."""
    if x == math.inf:
        return 0.0
    if x == -math.inf:
        return 1.0
    return 0.5 * math.erfc(x / math.sqrt(2.0))


def _cell_probability(a: float, b: float) -> float:
    """P(a < Z <= b), written so that no difference of two values near 1 occurs."""
    if a >= 0.0:
        return _upper_tail(a) - _upper_tail(b)
    if b <= 0.0:
        return _upper_tail(-b) - _upper_tail(-a)
    return 1.0 - _upper_tail(-a) - _upper_tail(b)


def _gaussian_quantile(p: float) -> float:
    """Inverse CDF by bisection on the upper tail (slow, obviously monotone)."""
    lo, hi = -40.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 1.0 - _upper_tail(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# --------------------------------------------------------------------------
# Step [4]: Lloyd-Max codebook for N(0,1).
# --------------------------------------------------------------------------

def quantizer_mse(centroids, thresholds=None) -> float:
    """E[(Z - q(Z))^2] for Z ~ N(0,1) and the scalar quantizer with the given
    centroids and decision thresholds (midpoints when thresholds is None).

    Closed-form cell integrals: over (a, b], int phi = P, int z phi = phi(a) -
    phi(b), int z^2 phi = P + a phi(a) - b phi(b).  Valid for any codebook, not
    only at the Lloyd fixed point.
    """
    c = [float(v) for v in centroids]
    L = len(c)
    if thresholds is None:
        thresholds = [0.5 * (c[k] + c[k + 1]) for k in range(L - 1)]
    t = [-math.inf] + [float(v) for v in thresholds] + [math.inf]
    d = 0.0
    for k in range(L):
        a, b = t[k], t[k + 1]
        p = _cell_probability(a, b)
        m1 = _pdf(a) - _pdf(b)
        m2 = p + (0.0 if math.isinf(a) else a * _pdf(a)) - (0.0 if math.isinf(b) else b * _pdf(b))
        d += m2 - 2.0 * c[k] * m1 + c[k] * c[k] * p
    return d


def lloyd_max_gaussian(levels: int = LEVELS, tol: float = 1e-15, max_iter: int = 200000):
    """Lloyd's algorithm on the N(0,1) density (Method step [4]; "optimal MSE for
    Gaussian values").  Alternates the two optimality conditions:
      thresholds t_k = (c_{k-1} + c_k) / 2              (nearest-neighbour cells)
      centroids  c_k = E[Z | t_k < Z <= t_{k+1}]
                     = (phi(t_k) - phi(t_{k+1})) / P(t_k < Z <= t_{k+1})
    starting from the quantiles (k + 1/2)/L, symmetrising c_k = -c_{L-1-k} each
    step (reading R7).  Stops when no centroid moves by more than tol, or when
    the step stops shrinking (fp64 noise floor).

    Returns dict(centroids, thresholds, mse, iterations) in fp64.
    """
    if levels < 2:
        raise ValueError("levels must be >= 2")
    L = levels
    c = [_gaussian_quantile((k + 0.5) / L) for k in range(L)]
    c = [0.5 * (c[k] - c[L - 1 - k]) for k in range(L)]
    best_step = math.inf
    stall = 0
    it = 0
    for it in range(1, max_iter + 1):
        t = [-math.inf] + [0.5 * (c[k - 1] + c[k]) for k in range(1, L)] + [math.inf]
        new = [(_pdf(t[k]) - _pdf(t[k + 1])) / _cell_probability(t[k], t[k + 1]) for k in range(L)]
        new = [0.5 * (new[k] - new[L - 1 - k]) for k in range(L)]
        step = max(abs(a - b) for a, b in zip(c, new))
        c = new
        if step <= tol:
            break
        if step < best_step:
            best_step, stall = step, 0
        else:
            stall += 1
            if stall > 50:
                break
    else:
        raise RuntimeError("Lloyd iteration did not converge")
    t = [0.5 * (c[k] + c[k + 1]) for k in range(L - 1)]
    return {
        "centroids": np.array(c, dtype=np.float64),
        "thresholds": np.array(t, dtype=np.float64),
        "mse": quantizer_mse(c, t),
        "iterations": it,
    }


_CODEBOOK_CACHE: dict = {}


def codebook_fp32(levels: int = LEVELS):
    """The stored codebook: fp32 centroids (fp64 fixed point rounded to nearest)
    and the decision midpoints between consecutive fp32 centroids.

    Returns (c32 float32[L], mid64 float64[L-1], b32 float32[L-1]) where mid64 is
    exact ((a + b)/2 of two fp32 values is exact in fp64) and b32 = fp32(mid64).
    """
    if levels not in _CODEBOOK_CACHE:
        c64 = lloyd_max_gaussian(levels)["centroids"]
        c32 = c64.astype(np.float32)
        mid64 = (c32[:-1].astype(np.float64) + c32[1:].astype(np.float64)) * 0.5
        _CODEBOOK_CACHE[levels] = (c32, mid64, mid64.astype(np.float32))
    c32, mid64, b32 = _CODEBOOK_CACHE[levels]
    return c32.copy(), mid64.copy(), b32.copy()


# --------------------------------------------------------------------------
# Step [3]: Walsh-Hadamard rotation.
# --------------------------------------------------------------------------

def sylvester_hadamard(n: int = BLOCK) -> np.ndarray:
    """H[i][j] = (-1)^popcount(i & j), the +-1 Sylvester matrix (readings R1, R2)."""
    if n <= 0 or n & (n - 1):
        raise ValueError("n must be a power of two")
    h = np.empty((n, n), dtype=np.int8)
    for i in range(n):
        for j in range(n):
            h[i, j] = -1 if bin(i & j).count("1") % 2 else 1
    return h


_H64 = sylvester_hadamard(BLOCK).astype(np.float64)


# --------------------------------------------------------------------------
# Steps [4]-[5]: nearest centroid, 5-bit pack.
# --------------------------------------------------------------------------

def nearest_centroid(y: np.ndarray, centroids: np.ndarray, chunk: int = 1 << 20) -> np.ndarray:
    """code = argmin_k |y - c_k| in fp64 over every centroid (brute force); on an
    exact tie the lower index wins (np.argmin returns the first minimum)."""
    y = np.asarray(y, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    flat = y.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    for s in range(0, flat.size, chunk):
        d = np.abs(flat[s:s + chunk, None] - c[None, :])
        out[s:s + chunk] = np.argmin(d, axis=1)
    return out.reshape(y.shape)


def pack_codes(codes: np.ndarray, bits: int = BITS) -> np.ndarray:
    """[..., 128] codes -> [..., 128*bits/8] bytes (reading R6): code j occupies
    bits [bits*j, bits*j + bits) of a little-endian bit string, LSB first."""
    codes = np.asarray(codes)
    if codes.shape[-1] % 8:
        raise ValueError("last dim must be a multiple of 8")
    lead = codes.shape[:-1]
    n = codes.shape[-1]
    g = codes.reshape(-1, n // 8, 8).astype(np.uint64)
    v = np.zeros(g.shape[:2], dtype=np.uint64)
    for j in range(8):
        v |= g[:, :, j] << np.uint64(bits * j)
    out = np.empty(g.shape[:2] + (bits,), dtype=np.uint8)
    for byte in range(bits):
        out[:, :, byte] = ((v >> np.uint64(8 * byte)) & np.uint64(0xFF)).astype(np.uint8)
    return out.reshape(lead + (n * bits // 8,))


def unpack_codes(packed: np.ndarray, bits: int = BITS) -> np.ndarray:
    """Inverse of pack_codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    nbytes = packed.shape[-1]
    if nbytes % bits:
        raise ValueError("last dim must be a multiple of the bit width")
    lead = packed.shape[:-1]
    b = packed.reshape(-1, nbytes // bits, bits).astype(np.uint64)
    v = np.zeros(b.shape[:2], dtype=np.uint64)
    for byte in range(bits):
        v |= b[:, :, byte] << np.uint64(8 * byte)
    mask = np.uint64((1 << bits) - 1)
    out = np.empty(b.shape[:2] + (8,), dtype=np.uint8)
    for j in range(8):
        out[:, :, j] = ((v >> np.uint64(bits * j)) & mask).astype(np.uint8)
    return out.reshape(lead + (nbytes // bits * 8,))


# --------------------------------------------------------------------------
# The whole quantizer, dequantizer and the matmuls.
# --------------------------------------------------------------------------

def _as_f64(a) -> np.ndarray:
    """Widen fp32 / bf16 / fp16 input exactly to fp64 (torch tensors accepted)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


def n_blocks(in_features: int) -> int:
    return (in_features + BLOCK - 1) // BLOCK


def quantize(W, levels: int = LEVELS, return_rotated: bool = False):
    """HLWQ Q5 encoding of one weight matrix W (out x in), Method steps [1]-[5].

    [1] view W as (out, n_blocks, 128), zero-padding the tail (reading R5);
    [2] n = ||block||_2 in fp64, stored as fp16 (reading R3);
    [3] y = (block / n) @ H (+-1 Sylvester, reading R1), evaluated as
        (block @ H) / n; y = 0 for n = 0;
    [4] code = nearest fp32 centroid (ties to the lower index);
    [5] pack 8 codes per 5 bytes (reading R6).

    Returns dict(packed uint8 [out][NB][80], norms float16 [out][NB],
    codes uint8 [out][NB][128], and y float64 [out][NB][128] if asked).
    """
    w = _as_f64(W)
    if w.ndim != 2:
        raise ValueError("W must be 2-D (out x in)")
    O, I = w.shape
    nb = n_blocks(I)
    wp = np.zeros((O, nb * BLOCK), dtype=np.float64)
    wp[:, :I] = w
    blocks = wp.reshape(O, nb, BLOCK)
    n = np.sqrt(np.sum(blocks * blocks, axis=-1))
    safe = np.where(n > 0.0, n, 1.0)
    # (block / n) @ H evaluated as (block @ H) / n: the +-1 sum of fp32/bf16
    # values is exact in fp64, so an exact tie (e.g. y = 0 on a constant block)
    # stays a tie and is resolved by the tie rule, not by rounding noise.
    y = np.where((n > 0.0)[..., None], (blocks @ _H64) / safe[..., None], 0.0)
    c32, _, _ = codebook_fp32(levels)
    codes = nearest_centroid(y, c32)
    out = {
        "packed": pack_codes(codes) if levels == LEVELS else None,
        "norms": n.astype(np.float16),
        "codes": codes,
    }
    if return_rotated:
        out["y"] = y
    return out


def dequantize(packed, norms, in_features: int, levels: int = LEVELS) -> np.ndarray:
    """w_hat[o][128b + i] = n16[o][b] * (1/128) * sum_j c[k_obj] * H[j][i], for
    i < in_features (pad dropped).  H @ H = 128 I, so this inverts step [3] for a
    codebook-exact block ("Pipeline": dequantize per-Linear)."""
    codes = unpack_codes(np.asarray(packed))
    c32, _, _ = codebook_fp32(levels)
    vals = c32.astype(np.float64)[codes]
    n16 = np.asarray(norms).astype(np.float64)
    blocks = (vals @ _H64) / 128.0 * n16[..., None]
    O = blocks.shape[0]
    return blocks.reshape(O, -1)[:, :in_features]


def matmul(packed, norms, in_features: int, X) -> np.ndarray:
    """Y[m][o] = sum_i X[m][i] * w_hat[o][i] in fp64, X widened exactly."""
    x = _as_f64(X)
    if x.ndim == 1:
        x = x[None, :]
    w_hat = dequantize(packed, norms, in_features)
    return x @ w_hat.T


def rotate_activation(X, in_features: int) -> np.ndarray:
    """x_tilde = x_b @ H per 128-block, zero-padded: the activation seen from the
    rotated domain (used only to cross-check matmul's algebra)."""
    x = _as_f64(X)
    if x.ndim == 1:
        x = x[None, :]
    M = x.shape[0]
    nb = n_blocks(in_features)
    xp = np.zeros((M, nb * BLOCK))
    xp[:, :in_features] = x
    return (xp.reshape(M, nb, BLOCK) @ _H64).reshape(M, -1)


def matmul_rotated_domain(packed, norms, in_features: int, X) -> np.ndarray:
    """Y[m][o] = sum_b (n16[o][b]/128) sum_j c[k_obj] x_tilde[m][128b + j]: the
    same product evaluated without inverse-rotating any weight."""
    codes = unpack_codes(np.asarray(packed))
    c32, _, _ = codebook_fp32()
    vals = c32.astype(np.float64)[codes]               # [O][NB][128]
    n16 = np.asarray(norms).astype(np.float64)          # [O][NB]
    xt = rotate_activation(X, in_features)              # [M][NB*128]
    M = xt.shape[0]
    O, nb, _ = vals.shape
    xt = xt.reshape(M, nb, BLOCK)
    per_block = np.einsum("obj,mbj->mob", vals, xt)     # [M][O][NB]
    return np.einsum("mob,ob->mo", per_block, n16 / 128.0)


def cosine_similarity(a, b) -> float:
    a = _as_f64(a).reshape(-1)
    b = _as_f64(b).reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


# --------------------------------------------------------------------------
# Routed MoE (8 routed + 1 shared expert per token; reading R8).
# --------------------------------------------------------------------------

def router_topk(logits, k: int):
    """Select the k largest logits per token (ties: lower expert id first) and
    weight them by a softmax over the selected logits, in fp64.

    Returns (ids int64 [T][k] in selection order, weights float64 [T][k])."""
    lg = _as_f64(logits)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("k must be in [1, E]")
    ids = np.empty((T, k), dtype=np.int64)
    wts = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-lg[t, e], e))[:k]
        sel = np.array([lg[t, e] for e in order])
        ex = np.exp(sel - sel.max())
        ids[t] = order
        wts[t] = ex / ex.sum()
    return ids, wts


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def moe_forward(experts_gu, experts_dn, hidden: int, inter: int, topk: int,
                logits, X, shared_gu=None, shared_dn=None):
    """out_t = sum_{e in topk(t)} p_te * Wd_e @ (SiLU(g) * u) + shared expert.

    experts_gu[e] / experts_dn[e] are (packed, norms) pairs of the gate_up matrix
    (2F x H) and the down matrix (H x F); shared_* likewise or None.  Only the
    experts a token selects are dequantized.  Everything stays fp64 (the
    intermediate h is not rounded).

    Returns (out float64 [T][H], ids, weights)."""
    x = _as_f64(X)
    ids, wts = router_topk(logits, topk)
    T = x.shape[0]
    out = np.zeros((T, hidden), dtype=np.float64)
    cache: dict = {}

    def expert_mlp(key, gu, dn, xt):
        if key not in cache:
            cache[key] = (dequantize(gu[0], gu[1], hidden), dequantize(dn[0], dn[1], inter))
        wgu, wdn = cache[key]
        gu_out = wgu @ xt
        h = silu(gu_out[:inter]) * gu_out[inter:]
        return wdn @ h

    for t in range(T):
        for s in range(topk):
            e = int(ids[t, s])
            out[t] += wts[t, s] * expert_mlp(e, experts_gu[e], experts_dn[e], x[t])
        if shared_gu is not None:
            out[t] += expert_mlp("shared", shared_gu, shared_dn, x[t])
    return out, ids, wts
