"""hlwq_gemm_noalloc: the GEMM entry point for callers that cannot allocate
device memory (its scratch is a static device array owned by the library).

Collected last on purpose: it must pass both in a fresh process and after every
other test has run on the same device."""
import ctypes

import pytest
import torch

from dequant_matmul_b200 import synth
from gpu_helpers import MATMUL_REL, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


def test_noalloc_matches_gemm_on_consecutive_calls(hl):
    cb = hl.codebook("cuda")
    W = synth.student_t((1024, 5120), df4_seed=77).cuda()
    p, n = hl.quantize(W, cb)
    # two calls in a row with different inputs: the shared scratch keeps the
    # first call's contents, which must not leak into the second result
    for M, seed in ((64, 1), (200, 2), (5, 3)):
        X = synth.activations(M, 5120, seed=seed).cuda()
        got = hl.gemm_noalloc(p, n, cb, X, out_dtype=torch.float32)
        want = hl.gemm(p, n, cb, X, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert rel_l2(got.double().cpu().numpy(), want.double().cpu().numpy()) <= MATMUL_REL, M
    assert hl.device_error() == 0


def test_noalloc_rejects_requests_beyond_the_scratch(hl):
    # stays on the tensor-core path (64 blocks per row) but needs 8 MiB of scratch
    need = hl.workspace_bytes(hl.HLWQ_OP_GEMM, 128, 8192, 512)
    assert need > hl.NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(256)
    st = hl.lib.hlwq_gemm_noalloc(p, p, p, 128, 8192, 512, p, 8192, p, 128, hl.HLWQ_F32, None)
    assert st == hl.HLWQ_ESCRATCH
    assert hl.lib.hlwq_status_string(st).decode().startswith("request exceeds")


def test_noalloc_serves_long_rows_without_scratch(hl):
    # rows longer than the tensor-core tile's 8192 inputs run on the CUDA-core
    # path, which needs no scratch, so any M is served
    cb = hl.codebook("cuda")
    W = synth.student_t((256, 8320), df4_seed=78).cuda()
    p, n = hl.quantize(W, cb)
    assert hl.workspace_bytes(hl.HLWQ_OP_GEMM, 256, 8320, 64) == 0
    X = synth.activations(64, 8320, seed=4).cuda()
    got = hl.gemm_noalloc(p, n, cb, X, out_dtype=torch.float32)
    want = hl.gemm(p, n, cb, X, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rel_l2(got.double().cpu().numpy(), want.double().cpu().numpy()) <= MATMUL_REL
    assert hl.device_error() == 0
