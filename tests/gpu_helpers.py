"""Helpers shared by the GPU parity tests (test-side only)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

CODE_FLIP_BAND = 1e-5      # flips allowed only this close to a decision midpoint
CODE_FLIP_RATE = 1e-6      # ... and at most this fraction of all codes
NORM_BAND = 2.0 ** -20     # norm bits may differ only this close (relative) to a binary16 rounding midpoint
DEQ_REL = 1e-5             # dequantized weights, relative L2
MATMUL_REL = 2e-3          # GEMV / GEMM / MoE outputs, relative L2 against fp64


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def half_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    return np.asarray(u16, dtype=np.uint16).view(np.float16).astype(np.float64)


def norm_near_fp16_midpoint(n64: np.ndarray) -> np.ndarray:
    """True where the exact norm lies within NORM_BAND (relative) of a binary16 rounding midpoint."""
    n64 = np.asarray(n64, dtype=np.float64)
    h = n64.astype(np.float16)
    hv = h.astype(np.float64)
    up = np.nextafter(h, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(h, np.float16(-np.inf)).astype(np.float64)
    mid = np.minimum(np.abs(n64 - (hv + up) / 2), np.abs(n64 - (hv + dn) / 2))
    return mid <= NORM_BAND * np.abs(n64)


def check_quantized(gpu_packed: torch.Tensor, gpu_norms: torch.Tensor, W, q=None, rows_idx=None):
    """Compares the GPU encoding with the oracle's.  Codes: bit-exact except flips
    where the oracle's rotated value is within CODE_FLIP_BAND of a midpoint (at
    most CODE_FLIP_RATE of all codes, at least allowing none on tiny inputs).
    Norms: bit-exact except within NORM_BAND of a binary16 midpoint.
    Returns a dict of counts."""
    if q is None:
        q = O.quantize(W, return_rotated=True)
    gp = gpu_packed.cpu().numpy()
    gn = gpu_norms.cpu().numpy()
    if rows_idx is not None:
        gp, gn = gp[rows_idx], gn[rows_idx]
    gcodes = O.unpack_codes(gp)
    mism = gcodes != q["codes"]
    _, mid64, _ = O.codebook_fp32()
    nflip = int(mism.sum())
    if nflip:
        y = q["y"][mism]
        dist = np.min(np.abs(y[:, None] - mid64[None, :]), axis=1)
        assert np.all(dist < CODE_FLIP_BAND), f"code flips away from a midpoint: max dist {dist.max()}"
        assert nflip <= CODE_FLIP_RATE * mism.size, f"{nflip} flips of {mism.size}"
    onorm = q["norms"].view(np.uint16)
    nbad = gn != onorm
    nnorm = int(nbad.sum())
    if nnorm:
        w = O._as_f64(W)
        nb = onorm.shape[1]
        wp = np.zeros((w.shape[0], nb * 128))
        wp[:, : w.shape[1]] = w
        n64 = np.sqrt((wp.reshape(w.shape[0], nb, 128) ** 2).sum(-1))
        assert np.all(norm_near_fp16_midpoint(n64[nbad])), "norm mismatch away from a binary16 midpoint"
    if nflip == 0 and nnorm == 0:
        assert np.array_equal(gp, q["packed"]), "codes equal but bytes differ"
    return {"flips": nflip, "norm_mismatch": nnorm, "codes": mism.size}


def to_dev(arr, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def oracle_to_dev(q):
    """(packed uint8, norms uint16) device tensors from an oracle encoding."""
    return to_dev(q["packed"]), to_dev(q["norms"].view(np.uint16))
