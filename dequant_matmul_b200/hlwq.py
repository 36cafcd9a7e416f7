"""Thin ctypes binding of libhlwq (include/hlwq.h).

Argument marshalling only: every step of the quantizer and of the matmuls runs
in the library's CUDA kernels.  Tensors must be CUDA tensors; the call is
enqueued on torch's current stream.  If the shared library is missing or cannot
be loaded the import fails loudly -- there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhlwq.so")

HLWQ_OK, HLWQ_EINVAL, HLWQ_EALIGN, HLWQ_EUNSUPPORTED, HLWQ_ECUDA, HLWQ_EWORKSPACE = 0, -1, -2, -3, -4, -5
HLWQ_ESCRATCH = -6
NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024 + 64 * 1024
HLWQ_F32, HLWQ_BF16, HLWQ_F16 = 0, 1, 2
HLWQ_OP_GEMM, HLWQ_OP_MOE, HLWQ_OP_TQ3_GEMM = 1, 2, 3
HLWQ_FLAG_WEIGHTS_STATIC = 1
HLWQ_FLAG_MOE_GROUPED = 2
DEVERR_CODEBOOK, DEVERR_TIMEOUT, DEVERR_CODE_RANGE = 0x1, 0x2, 0x4
BLOCK, BLOCK_BYTES, LEVELS = 128, 80, 32

# (name, restype, argtypes) for every symbol include/hlwq.h declares.
_P, _I, _I64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
SIGNATURES = {
    "hlwq_lloyd_codebook": (_I, [_I, _P, _P, _P]),
    "hlwq_quantize": (_I, [_P, _I, _I64, _I64, _P, _P, _P, _P]),
    "hlwq_dequantize": (_I, [_P, _P, _P, _I64, _I64, _P, _I, _P]),
    "hlwq_codes_unpack": (_I, [_P, _I64, _P, _P]),
    "hlwq_codes_pack": (_I, [_P, _I64, _P, _P]),
    "hlwq_tq3_quantize": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "hlwq_tq3_dequantize": (_I, [_P, _P, _P, _P, _I64, _I64, _P, _I, _P]),
    "hlwq_tq3_gemv": (_I, [_P, _P, _P, _P, _I64, _I64, _P, _P, _I, _P]),
    "hlwq_tq3_gemm": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _I64, _I, _P, _SZ, _P]),
    "hlwq_requantize_int4": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _P, _P]),
    "hlwq_kv_quantize": (_I, [_P, _I64, _I64, _P, _P, _P, _P]),
    "hlwq_kv_dequantize": (_I, [_P, _P, _P, _I64, _P, _I, _P]),
    "hlwq_kv_scores": (_I, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _I64, _P]),
    "hlwq_kv_window_append": (_I, [_P, _I64, _I64, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "hlwq_kv_scores_window": (_I, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _I64, _I64, _P, _I64, _P]),
    "hlwq_gemv": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _I, _P]),
    "hlwq_gemv_ex": (_I, [_P, _P, _P, _I64, _I64, _P, _P, _I, ctypes.c_uint, _P]),
    "hlwq_gemm": (_I, [_P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _I64, _I, _P, _SZ, _P]),
    "hlwq_moe_gemv": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P, _P, _I,
                           _P, _P, _P, _SZ, _P]),
    "hlwq_moe_gemv_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P, _P, _I,
                              _P, _P, _P, _SZ, ctypes.c_uint, _P]),
    "hlwq_gemm_noalloc": (_I, [_P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _I64, _I, _P]),
    "hlwq_workspace_bytes": (_SZ, [_I, _I64, _I64, _I64, _I64, _I64]),
    "hlwq_device_error": (_I, [_P]),
    "hlwq_fault_inject": (_I, [ctypes.c_uint, ctypes.c_ulonglong]),
    "hlwq_status_string": (ctypes.c_char_p, [_I]),
    "hlwq_version": (_I, []),
}


class HLWQError(RuntimeError):
    pass


# Failure-detection test build (hlwq_fault_inject is live there); never used by
# the functions below unless a test swaps it in as `lib`.
FAULT_LIB_PATH = os.path.join(_PKG, "libhlwq_fault.so")


def load_library(path: str):
    """Loads a build of the library and declares the header's signatures."""
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not built ({path}); run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load_library(LIB_PATH)


def _check(status: int, what: str):
    if status != HLWQ_OK:
        raise HLWQError(f"{what}: {lib.hlwq_status_string(status).decode()} ({status})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(dt) -> int:
    if dt == torch.float32:
        return HLWQ_F32
    if dt == torch.bfloat16:
        return HLWQ_BF16
    raise HLWQError(f"unsupported dtype {dt}")


def _cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise HLWQError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise HLWQError(f"{name} must be contiguous")


def _cuda_rows(t: torch.Tensor, name: str):
    """A CUDA matrix whose rows are contiguous (any row pitch)."""
    if not t.is_cuda:
        raise HLWQError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or t.stride(1) != 1:
        raise HLWQError(f"{name} must be a matrix with contiguous rows")


def n_blocks(in_features: int) -> int:
    return (in_features + BLOCK - 1) // BLOCK


# ------------------------------------------------------------------ host calls
def lloyd_codebook(levels: int = LEVELS):
    """Returns (centroids float32[L], midpoints float32[L-1], mse) on the host."""
    c = (ctypes.c_float * levels)()
    m = (ctypes.c_float * max(levels - 1, 1))()
    mse = ctypes.c_double()
    _check(lib.hlwq_lloyd_codebook(levels, ctypes.cast(c, _P), ctypes.cast(m, _P), ctypes.byref(mse)),
           "hlwq_lloyd_codebook")
    return (torch.tensor(list(c), dtype=torch.float32), torch.tensor(list(m)[: levels - 1], dtype=torch.float32),
            mse.value)


def codebook(device="cuda") -> torch.Tensor:
    return lloyd_codebook(LEVELS)[0].to(device)


def kv_codebook(device="cuda") -> torch.Tensor:
    """The 8 Lloyd-Max centroids of the Q3 KV-cache encoding."""
    return lloyd_codebook(8)[0].to(device)


def workspace_bytes(op: int, a: int, b: int, c: int, E: int = 1, topk: int = 0) -> int:
    return int(lib.hlwq_workspace_bytes(op, a, b, c, E, topk))


def device_error() -> int:
    bits = ctypes.c_uint32()
    _check(lib.hlwq_device_error(ctypes.byref(bits)), "hlwq_device_error")
    return bits.value


# ------------------------------------------------------------------ device calls
def quantize(W: torch.Tensor, cb: torch.Tensor, packed=None, norms=None, stream=None):
    """W: [..., in] fp32/bf16 CUDA tensor (leading dims are stacked rows).
    Returns (packed uint8 [..., NB, 80], norms uint16 [..., NB] binary16 bits)."""
    _cuda(W, "W")
    in_f = W.shape[-1]
    rows = W.numel() // in_f
    nb = n_blocks(in_f)
    lead = tuple(W.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + (nb, BLOCK_BYTES), dtype=torch.uint8, device=W.device)
    if norms is None:
        norms = torch.empty(lead + (nb,), dtype=torch.uint16, device=W.device)
    _check(lib.hlwq_quantize(_ptr(W), _dtype_code(W.dtype), rows, in_f, _ptr(cb), _ptr(packed), _ptr(norms),
                             _stream(stream)), "hlwq_quantize")
    return packed, norms


def dequantize(packed, norms, cb, in_features: int, out_dtype=torch.float32, out=None, stream=None):
    _cuda(packed, "packed")
    nb = packed.shape[-2]
    lead = tuple(packed.shape[:-2])
    rows = packed.numel() // (nb * BLOCK_BYTES)
    if out is None:
        out = torch.empty(lead + (in_features,), dtype=out_dtype, device=packed.device)
    _check(lib.hlwq_dequantize(_ptr(packed), _ptr(norms), _ptr(cb), rows, in_features, _ptr(out),
                               _dtype_code(out.dtype), _stream(stream)), "hlwq_dequantize")
    return out


def codes_unpack(packed, codes=None, stream=None):
    """packed uint8 [..., NB, 80] -> codes uint8 [..., NB, 128], one code per byte."""
    _cuda(packed, "packed")
    if packed.shape[-1] != BLOCK_BYTES:
        raise HLWQError("packed must end in 80-byte blocks")
    nblocks = packed.numel() // BLOCK_BYTES
    if codes is None:
        codes = torch.empty(tuple(packed.shape[:-1]) + (BLOCK,), dtype=torch.uint8, device=packed.device)
    _check(lib.hlwq_codes_unpack(_ptr(packed), nblocks, _ptr(codes), _stream(stream)), "hlwq_codes_unpack")
    return codes


def codes_pack(codes, packed=None, stream=None):
    """codes uint8 [..., NB, 128] (0..31) -> packed uint8 [..., NB, 80]."""
    _cuda(codes, "codes")
    if codes.shape[-1] != BLOCK:
        raise HLWQError("codes must end in blocks of 128")
    nblocks = codes.numel() // BLOCK
    if packed is None:
        packed = torch.empty(tuple(codes.shape[:-1]) + (BLOCK_BYTES,), dtype=torch.uint8, device=codes.device)
    _check(lib.hlwq_codes_pack(_ptr(codes), nblocks, _ptr(packed), _stream(stream)), "hlwq_codes_pack")
    return packed


def tq3_quantize(W: torch.Tensor, signs: torch.Tensor, cb8, packed=None, norms=None, stream=None):
    """W bf16 [..., in] (leading dims are stacked rows), signs int8 [2][128]
    (+-1; row 0 before the FWHT, row 1 after) -> (packed uint8 [..., NB, 48],
    norms float32 [..., NB]: the shape-gain norms)."""
    _cuda(W, "W")
    _cuda(signs, "signs")
    if W.dtype != torch.bfloat16 or signs.dtype != torch.int8 or signs.numel() != 2 * BLOCK:
        raise HLWQError("tq3_quantize takes bf16 weights and int8 signs [2][128]")
    in_f = W.shape[-1]
    rows = W.numel() // in_f
    nb = n_blocks(in_f)
    lead = tuple(W.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + (nb, 48), dtype=torch.uint8, device=W.device)
    if norms is None:
        norms = torch.empty(lead + (nb,), dtype=torch.float32, device=W.device)
    _check(lib.hlwq_tq3_quantize(_ptr(W), rows, in_f, _ptr(signs), _ptr(cb8), _ptr(packed), _ptr(norms),
                                 _stream(stream)), "hlwq_tq3_quantize")
    return packed, norms


def tq3_dequantize(packed, norms, signs, cb8, in_features: int, out_dtype=torch.float32, out=None, stream=None):
    """-> W_hat [..., in] (the pad dropped)."""
    _cuda(packed, "packed")
    nb = packed.shape[-2]
    lead = tuple(packed.shape[:-2])
    rows = packed.numel() // (nb * 48)
    if out is None:
        out = torch.empty(lead + (in_features,), dtype=out_dtype, device=packed.device)
    _check(lib.hlwq_tq3_dequantize(_ptr(packed), _ptr(norms), _ptr(signs), _ptr(cb8), rows, in_features, _ptr(out),
                                   _dtype_code(out.dtype), _stream(stream)), "hlwq_tq3_dequantize")
    return out


def tq3_gemv(packed, norms, signs, cb8, x: torch.Tensor, out_dtype=torch.float32, y=None, stream=None):
    """x bf16 [in] -> y [out] = W_hat @ x (fp32 accumulation)."""
    _cuda(x, "x")
    out_f = packed.shape[0]
    if y is None:
        y = torch.empty(out_f, dtype=out_dtype, device=x.device)
    _check(lib.hlwq_tq3_gemv(_ptr(packed), _ptr(norms), _ptr(signs), _ptr(cb8), out_f, x.shape[-1], _ptr(x), _ptr(y),
                             _dtype_code(y.dtype), _stream(stream)), "hlwq_tq3_gemv")
    return y


def tq3_gemm(packed, norms, signs, cb8, X: torch.Tensor, out_dtype=torch.float32, Y=None, workspace=None,
             stream=None):
    """X bf16 [M][in] (row pitch X.stride(0)) -> Y [M][out] = X @ W_hat^T."""
    _cuda_rows(X, "X")
    out_f = packed.shape[0]
    M, in_f = X.shape
    if Y is None:
        Y = torch.empty(M, out_f, dtype=out_dtype, device=X.device)
    _cuda_rows(Y, "Y")
    need = workspace_bytes(HLWQ_OP_TQ3_GEMM, out_f, in_f, M)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.hlwq_tq3_gemm(_ptr(packed), _ptr(norms), _ptr(signs), _ptr(cb8), out_f, in_f, M, _ptr(X), X.stride(0),
                             _ptr(Y), Y.stride(0), _dtype_code(Y.dtype), _ptr(workspace), ws_bytes, _stream(stream)),
           "hlwq_tq3_gemm")
    return Y


def requantize_int4(packed, norms, cb, in_features: int, q4=None, scale=None, zero=None, stream=None):
    """Q5 -> INT4 (groups of 128): returns (q4 uint8 [..., NB, 64], scale and
    zero as bfloat16 bit patterns, uint16 [..., NB])."""
    _cuda(packed, "packed")
    nb = packed.shape[-2]
    lead = tuple(packed.shape[:-2])
    rows = packed.numel() // (nb * BLOCK_BYTES)
    if q4 is None:
        q4 = torch.empty(lead + (nb, 64), dtype=torch.uint8, device=packed.device)
    if scale is None:
        scale = torch.empty(lead + (nb,), dtype=torch.uint16, device=packed.device)
    if zero is None:
        zero = torch.empty(lead + (nb,), dtype=torch.uint16, device=packed.device)
    _check(lib.hlwq_requantize_int4(_ptr(packed), _ptr(norms), _ptr(cb), rows, in_features, _ptr(q4), _ptr(scale),
                                    _ptr(zero), _stream(stream)), "hlwq_requantize_int4")
    return q4, scale, zero


def kv_quantize(X: torch.Tensor, cb8, packed=None, norms=None, stream=None):
    """X bf16 [N][256] (row pitch X.stride(0)) -> (packed uint8 [N][96], norms fp16 bits uint16 [N])."""
    _cuda_rows(X, "X")
    N = X.shape[0]
    if packed is None:
        packed = torch.empty(N, 96, dtype=torch.uint8, device=X.device)
    if norms is None:
        norms = torch.empty(N, dtype=torch.uint16, device=X.device)
    _check(lib.hlwq_kv_quantize(_ptr(X), N, X.stride(0), _ptr(cb8), _ptr(packed), _ptr(norms), _stream(stream)),
           "hlwq_kv_quantize")
    return packed, norms


def kv_dequantize(packed, norms, cb8, out_dtype=torch.float32, out=None, stream=None):
    N = packed.shape[0]
    if out is None:
        out = torch.empty(N, 256, dtype=out_dtype, device=packed.device)
    _check(lib.hlwq_kv_dequantize(_ptr(packed), _ptr(norms), _ptr(cb8), N, _ptr(out), _dtype_code(out.dtype),
                                  _stream(stream)), "hlwq_kv_dequantize")
    return out


def kv_scores(Q: torch.Tensor, packed, norms, cb8, S=None, stream=None):
    """Q bf16 [M][256] (M <= 64, row pitch Q.stride(0)) against N encoded vectors -> S fp32 [M][N]."""
    _cuda_rows(Q, "Q")
    M, N = Q.shape[0], packed.shape[0]
    if S is None:
        S = torch.empty(M, N, dtype=torch.float32, device=Q.device)
    _check(lib.hlwq_kv_scores(_ptr(Q), M, Q.stride(0), _ptr(packed), _ptr(norms), _ptr(cb8), N, _ptr(S), S.stride(0),
                              _stream(stream)), "hlwq_kv_scores")
    return S


class KVWindowCache:
    """One head's Q3 KV cache with its residual window (hlwq_kv_window_append /
    hlwq_kv_scores_window): `capacity` encoded rows preallocated, a bf16 ring
    of R slots for the most recent tokens.  Bookkeeping only; the device work
    is the library's."""

    def __init__(self, capacity: int, R: int = 128, device="cuda", cb8=None):
        self.packed = torch.zeros(capacity, 96, dtype=torch.uint8, device=device)
        self.norms = torch.zeros(capacity, dtype=torch.uint16, device=device)
        self.window = torch.zeros(R, 256, dtype=torch.bfloat16, device=device)
        self.R, self.n_enc, self.n_total = R, 0, 0
        self.cb8 = cb8 if cb8 is not None else kv_codebook(device)

    def append(self, X: torch.Tensor, stream=None):
        """X bf16 [t][256] (row pitch X.stride(0))."""
        _cuda_rows(X, "X")
        t = X.shape[0]
        if self.n_total + t - self.R > self.packed.shape[0]:
            raise HLWQError("KVWindowCache: capacity of encoded rows exceeded")
        out = ctypes.c_int64()
        _check(lib.hlwq_kv_window_append(_ptr(X), t, X.stride(0), _ptr(self.window), self.R, self.n_enc,
                                         self.n_total, _ptr(self.cb8), _ptr(self.packed), _ptr(self.norms),
                                         ctypes.byref(out), _stream(stream)), "hlwq_kv_window_append")
        self.n_enc, self.n_total = out.value, self.n_total + t

    def scores(self, Q: torch.Tensor, S=None, stream=None):
        """Q bf16 [M][256] (M <= 64) -> S fp32 [M][n_total] over every cached token."""
        _cuda_rows(Q, "Q")
        M = Q.shape[0]
        if S is None:
            S = torch.empty(M, self.n_total, dtype=torch.float32, device=Q.device)
        _check(lib.hlwq_kv_scores_window(_ptr(Q), M, Q.stride(0), _ptr(self.packed), _ptr(self.norms), _ptr(self.cb8),
                                         self.n_enc, _ptr(self.window), self.R, self.n_total, _ptr(S), S.stride(0),
                                         _stream(stream)), "hlwq_kv_scores_window")
        return S


def gemv(packed, norms, cb, x: torch.Tensor, out_dtype=torch.float32, y=None, stream=None, flags: int = 0):
    """x: bf16 [in].  Returns y [out].  flags != 0 calls hlwq_gemv_ex (e.g.
    HLWQ_FLAG_WEIGHTS_STATIC: the weights are not written by earlier work still
    running on the stream, so the kernel's set-up may overlap it)."""
    _cuda(x, "x")
    out_f = packed.shape[0]
    if y is None:
        y = torch.empty(out_f, dtype=out_dtype, device=x.device)
    if flags:
        _check(lib.hlwq_gemv_ex(_ptr(packed), _ptr(norms), _ptr(cb), out_f, x.shape[-1], _ptr(x), _ptr(y),
                                _dtype_code(y.dtype), flags, _stream(stream)), "hlwq_gemv_ex")
    else:
        _check(lib.hlwq_gemv(_ptr(packed), _ptr(norms), _ptr(cb), out_f, x.shape[-1], _ptr(x), _ptr(y),
                             _dtype_code(y.dtype), _stream(stream)), "hlwq_gemv")
    return y


def gemm(packed, norms, cb, X: torch.Tensor, out_dtype=torch.bfloat16, Y=None, workspace=None, stream=None):
    """X: bf16 [M][in] (row pitch X.stride(0)).  Returns Y [M][out]."""
    _cuda(X, "X")
    out_f = packed.shape[0]
    M, in_f = X.shape
    if Y is None:
        Y = torch.empty(M, out_f, dtype=out_dtype, device=X.device)
    need = workspace_bytes(HLWQ_OP_GEMM, out_f, in_f, M)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.hlwq_gemm(_ptr(packed), _ptr(norms), _ptr(cb), out_f, in_f, M, _ptr(X), X.stride(0), _ptr(Y),
                         Y.stride(0), _dtype_code(Y.dtype), _ptr(workspace), ws_bytes, _stream(stream)), "hlwq_gemm")
    return Y


def moe_gemv(gu, dn, cb, logits, X, topk: int, shared=None, out_dtype=torch.float32, Y=None, ids=None,
             weights=None, workspace=None, stream=None, flags: int = 0):
    """gu = (packed [E][2F][NBh][80], norms [E][2F][NBh]); dn = (packed [E][H][NBf][80], norms [E][H][NBf]);
    shared = ((packed, norms) of gate_up, (packed, norms) of down) or None.
    logits fp32 [T][E], X bf16 [T][H].  Returns (Y, ids, weights)."""
    E, two_f = gu[0].shape[0], gu[0].shape[1]
    F = two_f // 2
    H = dn[0].shape[1]
    T = X.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty(T, H, dtype=out_dtype, device=dev)
    if ids is None:
        ids = torch.empty(T, topk, dtype=torch.int32, device=dev)
    if weights is None:
        weights = torch.empty(T, topk, dtype=torch.float32, device=dev)
    need = workspace_bytes(HLWQ_OP_MOE, H, F, T, E, topk)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    sg = shared[0] if shared is not None else (None, None)
    sd = shared[1] if shared is not None else (None, None)
    if flags:
        _check(lib.hlwq_moe_gemv_ex(_ptr(gu[0]), _ptr(gu[1]), _ptr(dn[0]), _ptr(dn[1]), _ptr(sg[0]), _ptr(sg[1]),
                                    _ptr(sd[0]), _ptr(sd[1]), _ptr(cb), E, H, F, topk, T, _ptr(logits), _ptr(X),
                                    _ptr(Y), _dtype_code(Y.dtype), _ptr(ids), _ptr(weights), _ptr(workspace),
                                    workspace.numel(), flags, _stream(stream)), "hlwq_moe_gemv_ex")
    else:
        _check(lib.hlwq_moe_gemv(_ptr(gu[0]), _ptr(gu[1]), _ptr(dn[0]), _ptr(dn[1]), _ptr(sg[0]), _ptr(sg[1]),
                                 _ptr(sd[0]), _ptr(sd[1]), _ptr(cb), E, H, F, topk, T, _ptr(logits), _ptr(X),
                                 _ptr(Y), _dtype_code(Y.dtype), _ptr(ids), _ptr(weights), _ptr(workspace),
                                 workspace.numel(), _stream(stream)), "hlwq_moe_gemv")
    return Y, ids, weights


def gemm_noalloc(packed, norms, cb, X: torch.Tensor, out_dtype=torch.bfloat16, Y=None, stream=None):
    """hlwq_gemm_noalloc: the GEMM with the library's static scratch (no workspace)."""
    _cuda(X, "X")
    out_f = packed.shape[0]
    M, in_f = X.shape
    if Y is None:
        Y = torch.empty(M, out_f, dtype=out_dtype, device=X.device)
    _check(lib.hlwq_gemm_noalloc(_ptr(packed), _ptr(norms), _ptr(cb), out_f, in_f, M, _ptr(X), X.stride(0),
                                 _ptr(Y), Y.stride(0), _dtype_code(Y.dtype), _stream(stream)), "hlwq_gemm_noalloc")
    return Y
