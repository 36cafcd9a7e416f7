"""CPU checks of the C ABI: the library loads, exports every symbol the header
declares, the host codebook builder agrees bit-for-bit with the oracle, and
argument validation rejects bad calls before anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import build
    build.build()
    from dequant_matmul_b200 import hlwq
    return hlwq


def header_symbols():
    text = open(os.path.join(ROOT, "include", "hlwq.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(hlwq_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(hl):
    syms = header_symbols()
    assert len(syms) >= 9
    for s in syms:
        assert hasattr(hl.lib, s), s
        assert s in hl.SIGNATURES, s


@pytest.mark.parametrize("levels", [2, 4, 8, 16, 32])
def test_host_codebook_equals_oracle(hl, levels):
    c, m, mse = hl.lloyd_codebook(levels)
    c32, mid64, b32 = O.codebook_fp32(levels)
    assert np.array_equal(c.numpy(), c32)
    assert np.array_equal(m.numpy(), b32)
    assert mse == pytest.approx(O.lloyd_max_gaussian(levels)["mse"], rel=1e-9)


def test_codebook_rejects_bad_levels(hl):
    buf = (ctypes.c_float * 64)()
    for bad in (0, 1, 3, 64):
        assert hl.lib.hlwq_lloyd_codebook(bad, ctypes.cast(buf, ctypes.c_void_p), None, None) == hl.HLWQ_EINVAL
    assert hl.lib.hlwq_lloyd_codebook(32, None, None, None) == hl.HLWQ_EINVAL


def test_validation_before_launch(hl):
    L = hl.lib
    p = ctypes.c_void_p(256)        # fake, 16-byte aligned, never dereferenced
    odd = ctypes.c_void_p(257)
    assert L.hlwq_quantize(None, hl.HLWQ_BF16, 4, 128, p, p, p, None) == hl.HLWQ_EINVAL
    assert L.hlwq_quantize(p, hl.HLWQ_BF16, 0, 128, p, p, p, None) == hl.HLWQ_EINVAL
    assert L.hlwq_quantize(p, hl.HLWQ_F16, 4, 128, p, p, p, None) == hl.HLWQ_EUNSUPPORTED
    assert L.hlwq_quantize(p, hl.HLWQ_BF16, 4, 128, p, odd, p, None) == hl.HLWQ_EALIGN
    assert L.hlwq_dequantize(p, p, p, 4, -1, p, hl.HLWQ_F32, None) == hl.HLWQ_EINVAL
    assert L.hlwq_gemv(p, p, p, 4, 128, p, p, 7, None) == hl.HLWQ_EUNSUPPORTED
    assert L.hlwq_requantize_int4(p, p, p, 4, 128, None, p, p, None) == hl.HLWQ_EINVAL
    assert L.hlwq_requantize_int4(p, p, p, 4, 704, p, p, p, None) == hl.HLWQ_EUNSUPPORTED  # not 128-aligned
    assert L.hlwq_requantize_int4(p, p, p, 4, 128, ctypes.c_void_p(264), p, p, None) == hl.HLWQ_EALIGN
    assert L.hlwq_tq3_quantize(p, 4, 128, None, p, p, p, None) == hl.HLWQ_EINVAL      # no signs
    assert L.hlwq_tq3_quantize(p, 4, 128, p, p, ctypes.c_void_p(258), p, None) == hl.HLWQ_EALIGN
    assert L.hlwq_tq3_dequantize(p, p, p, p, 4, 128, p, hl.HLWQ_F16, None) == hl.HLWQ_EUNSUPPORTED
    assert L.hlwq_tq3_dequantize(p, p, p, p, 0, 128, p, hl.HLWQ_F32, None) == hl.HLWQ_EINVAL
    assert L.hlwq_tq3_gemv(p, p, p, p, 4, 128, odd, p, hl.HLWQ_F32, None) == hl.HLWQ_EALIGN
    assert L.hlwq_tq3_gemv(p, p, p, p, 4, 0, p, p, hl.HLWQ_F32, None) == hl.HLWQ_EINVAL
    assert L.hlwq_tq3_gemv(p, p, p, p, 4, 128, p, p, 9, None) == hl.HLWQ_EUNSUPPORTED
    assert L.hlwq_codes_unpack(p, 0, p, None) == hl.HLWQ_EINVAL
    assert L.hlwq_codes_pack(None, 4, p, None) == hl.HLWQ_EINVAL
    assert L.hlwq_codes_pack(p, 4, ctypes.c_void_p(264), None) == hl.HLWQ_EALIGN
    assert L.hlwq_codes_unpack(ctypes.c_void_p(260), 4, p, None) == hl.HLWQ_EALIGN
    assert L.hlwq_kv_quantize(p, 4, 128, p, p, p, None) == hl.HLWQ_EINVAL             # ldx < 256
    assert L.hlwq_kv_dequantize(p, p, p, 4, p, hl.HLWQ_F16, None) == hl.HLWQ_EUNSUPPORTED
    assert L.hlwq_kv_scores(p, 65, 256, p, p, p, 4, p, 4, None) == hl.HLWQ_EUNSUPPORTED  # > 64 queries
    assert L.hlwq_kv_scores(p, 2, 256, odd, p, p, 4, p, 4, None) == hl.HLWQ_EALIGN
    assert L.hlwq_gemm(p, p, p, 4, 128, 2, p, 64, p, 4, hl.HLWQ_BF16, None, 0, None) == hl.HLWQ_EINVAL  # ldx < in
    ws = hl.workspace_bytes(hl.HLWQ_OP_MOE, 2048, 512, 8, 256, 8)
    assert ws > 0
    args = [p, p, p, p, None, None, None, None, p, 256, 2048, 512, 8, 8, p, p, p, hl.HLWQ_F32, None, None]
    assert L.hlwq_moe_gemv(*args, p, ws - 1, None) == hl.HLWQ_EWORKSPACE
    bad_topk = list(args)
    bad_topk[12] = 300
    assert L.hlwq_moe_gemv(*bad_topk, p, ws, None) == hl.HLWQ_EINVAL
    half_shared = list(args)
    half_shared[4] = p
    assert L.hlwq_moe_gemv(*half_shared, p, ws, None) == hl.HLWQ_EINVAL
    assert hl.lib.hlwq_status_string(-5).decode().startswith("workspace")
    assert hl.lib.hlwq_version() >= 100


def test_workspace_sizes(hl):
    assert hl.workspace_bytes(hl.HLWQ_OP_GEMM, 4096, 4096, 1) == 0
    a = hl.workspace_bytes(hl.HLWQ_OP_MOE, 2048, 512, 1, 256, 8)
    b = hl.workspace_bytes(hl.HLWQ_OP_MOE, 2048, 512, 64, 256, 8)
    assert 0 < a < b


def test_gemm_workspace_only_on_the_tensor_core_path(hl):
    # rows of at most 8192 inputs take the tensor cores from M = 5 (workspace);
    # longer rows run on the CUDA-core path at every M and need none
    assert hl.workspace_bytes(hl.HLWQ_OP_GEMM, 256, 8192, 64) > 0
    assert hl.workspace_bytes(hl.HLWQ_OP_GEMM, 256, 8193, 64) == 0
    assert hl.workspace_bytes(hl.HLWQ_OP_GEMM, 256, 65536, 512) == 0
    assert hl.workspace_bytes(hl.HLWQ_OP_GEMM, 256, 8192, 4) == 0


def test_tq3_gemm_validation_and_workspace(hl):
    L = hl.lib
    p = ctypes.c_void_p(256)        # fake, 16-byte aligned, never dereferenced
    p8 = ctypes.c_void_p(264)       # 8-byte aligned only
    p2 = ctypes.c_void_p(258)       # 2-byte aligned only

    def call(packed=p, norms=p, signs=p, cb=p, out=256, in_f=512, M=16, X=p, ldx=512, Y=p, ldy=256,
             dt=hl.HLWQ_F32, ws=None, ws_bytes=0):
        return L.hlwq_tq3_gemm(packed, norms, signs, cb, out, in_f, M, X, ldx, Y, ldy, dt, ws, ws_bytes, None)

    assert call(packed=None) == hl.HLWQ_EINVAL
    assert call(signs=None) == hl.HLWQ_EINVAL
    assert call(M=0) == hl.HLWQ_EINVAL
    assert call(ldx=511) == hl.HLWQ_EINVAL
    assert call(ldy=255) == hl.HLWQ_EINVAL
    assert call(in_f=(1 << 20) + 1, ldx=(1 << 20) + 1) == hl.HLWQ_EINVAL
    assert call(dt=hl.HLWQ_F16) == hl.HLWQ_EUNSUPPORTED
    assert call(packed=p8) == hl.HLWQ_EALIGN          # 48-byte groups are copied by TMA boxes
    assert call(norms=p2) == hl.HLWQ_EALIGN
    assert call(Y=p2) == hl.HLWQ_EALIGN               # fp32 output
    assert call() == hl.HLWQ_EWORKSPACE               # M >= 2: the tensor-core path needs its workspace
    need = hl.workspace_bytes(hl.HLWQ_OP_TQ3_GEMM, 256, 512, 16)
    assert need > 0
    assert call(ws=p, ws_bytes=need - 1) == hl.HLWQ_EWORKSPACE   # two row tiles: no K split, need = minimum
    assert call(ws=p8, ws_bytes=need) == hl.HLWQ_EALIGN
    # no workspace for one token or for rows longer than 8192 (the GEMV per token)
    assert hl.workspace_bytes(hl.HLWQ_OP_TQ3_GEMM, 256, 512, 1) == 0
    assert hl.workspace_bytes(hl.HLWQ_OP_TQ3_GEMM, 256, 8193, 64) == 0
    assert hl.workspace_bytes(hl.HLWQ_OP_TQ3_GEMM, 256, 8192, 2) > 0


def test_moe_grouped_path_row_limit(hl):
    """The grouped path takes H and F up to 16384; asked for with longer rows
    it returns HLWQ_EUNSUPPORTED before launching anything."""
    L = hl.lib
    p = ctypes.c_void_p(256)
    E, H, F, topk, T = 8, 16512, 256, 2, 4
    need = hl.workspace_bytes(hl.HLWQ_OP_MOE, H, F, T, E, topk)
    args = [p] * 4 + [None] * 4 + [p, E, H, F, topk, T, p, p, p, hl.HLWQ_F32, None, None, p, need]
    assert L.hlwq_moe_gemv_ex(*args, hl.HLWQ_FLAG_MOE_GROUPED, None) == hl.HLWQ_EUNSUPPORTED


def test_noalloc_validates_arguments_before_sizing_its_scratch(hl):
    L = hl.lib
    p = ctypes.c_void_p(256)
    F32 = hl.HLWQ_F32
    # out-of-range sizes are argument errors, not scratch errors
    assert L.hlwq_gemm_noalloc(p, p, p, 128, 1 << 21, 64, p, 1 << 21, p, 128, F32, None) == hl.HLWQ_EINVAL
    assert L.hlwq_gemm_noalloc(p, p, p, 128, 512, (1 << 20) + 1, p, 512, p, 128, F32, None) == hl.HLWQ_EINVAL
    assert L.hlwq_gemm_noalloc(p, p, p, 128, 512, 64, p, 256, p, 128, F32, None) == hl.HLWQ_EINVAL  # ldx < in
    assert L.hlwq_gemm_noalloc(p, p, p, 128, 512, 64, p, 512, p, 64, F32, None) == hl.HLWQ_EINVAL   # ldy < out
    assert L.hlwq_gemm_noalloc(None, p, p, 128, 512, 64, p, 512, p, 128, F32, None) == hl.HLWQ_EINVAL
    assert L.hlwq_gemm_noalloc(p, p, p, 128, 512, 64, p, 512, p, 128, 7, None) == hl.HLWQ_EUNSUPPORTED
    assert L.hlwq_gemm_noalloc(p, p, p, 128, 512, 64, ctypes.c_void_p(257), 512, p, 128, F32,
                               None) == hl.HLWQ_EALIGN
    # a tensor-core request above the static scratch (512 x 64 blocks x 256 B)
    assert hl.workspace_bytes(hl.HLWQ_OP_GEMM, 128, 8192, 512) > hl.NOALLOC_SCRATCH_BYTES
    assert L.hlwq_gemm_noalloc(p, p, p, 128, 8192, 512, p, 8192, p, 128, F32, None) == hl.HLWQ_ESCRATCH


def test_kv_window_validation(hl):
    L = hl.lib
    p = ctypes.c_void_p(256)
    out = ctypes.c_int64()
    # more tokens in the window than its R slots
    assert L.hlwq_kv_window_append(p, 1, 256, p, 128, 0, 129, p, p, p, ctypes.byref(out), None) == hl.HLWQ_EINVAL
    assert L.hlwq_kv_window_append(p, 1, 256, p, 128, 5, 4, p, p, p, None, None) == hl.HLWQ_EINVAL    # n_enc > n_total
    assert L.hlwq_kv_window_append(p, 1, 128, p, 128, 0, 0, p, p, p, None, None) == hl.HLWQ_EINVAL    # ldx < 256
    assert L.hlwq_kv_window_append(None, 1, 256, p, 128, 0, 0, p, p, p, None, None) == hl.HLWQ_EINVAL # no x
    assert L.hlwq_kv_window_append(p, 1, 256, ctypes.c_void_p(264), 128, 0, 0, p, p, p, None,
                                   None) == hl.HLWQ_EALIGN                                         # window 8-byte
    assert L.hlwq_kv_window_append(p, 1, 256, p, 0, 0, 0, p, p, p, None, None) == hl.HLWQ_EINVAL      # R = 0
    assert L.hlwq_kv_scores_window(p, 2, 256, p, p, p, 10, p, 128, 9, p, 16, None) == hl.HLWQ_EINVAL  # n_enc > n_total
    assert L.hlwq_kv_scores_window(p, 2, 256, p, p, p, 0, p, 128, 200, p, 256, None) == hl.HLWQ_EINVAL  # > R in window
    assert L.hlwq_kv_scores_window(p, 2, 256, p, p, p, 10, None, 128, 20, p, 20, None) == hl.HLWQ_EINVAL  # no window
    assert L.hlwq_kv_scores_window(p, 2, 256, p, p, p, 10, p, 128, 20, p, 19, None) == hl.HLWQ_EINVAL  # lds < n_total
    assert L.hlwq_kv_scores_window(p, 65, 256, p, p, p, 10, p, 128, 20, p, 20, None) == hl.HLWQ_EUNSUPPORTED
