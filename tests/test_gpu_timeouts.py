"""Failure detection without a GPU fault.

The failure-detection build of the library (libhlwq_fault.so) can tell the TMA
producers of the TMA-fed kernels to issue no copies.  Every consumer's bounded
mbarrier wait then runs out with nothing in flight; the kernel raises
HLWQ_DEVERR_TIMEOUT, frees its tensor memory and returns.  The tests check the
reported status and that the next normal call on the same context is still
correct (a kernel that kept its tensor memory would leave the next tensor-core
launch without columns).  Nothing here faults, traps or hangs a GPU: the waits
are bounded (5 ms here) and no copy is ever issued."""
import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth
from gpu_helpers import MATMUL_REL, oracle_to_dev, rel_l2

pytestmark = pytest.mark.gpu

WAIT_NS = 5_000_000          # 5 ms per bounded wait while injecting
PRODUCT_WAIT_NS = 2_000_000_000


@pytest.fixture(scope="module")
def fl():
    """The binding with its library swapped for the failure-detection build."""
    from dequant_matmul_b200 import hlwq
    prod = hlwq.lib
    hlwq.lib = hlwq.load_library(hlwq.FAULT_LIB_PATH)
    try:
        yield hlwq
    finally:
        hlwq.lib.hlwq_fault_inject(0, PRODUCT_WAIT_NS)
        hlwq.lib = prod


@pytest.fixture(scope="module")
def layer():
    W = synth.student_t((1024, 5120), df4_seed=41)
    q = O.quantize(W)
    return q, oracle_to_dev(q)


def _inject(fl, on: bool):
    assert fl.lib.hlwq_fault_inject(1 if on else 0, WAIT_NS if on else PRODUCT_WAIT_NS) == fl.HLWQ_OK


def test_product_library_has_no_fault_hook():
    from dequant_matmul_b200 import hlwq
    prod = hlwq.load_library(hlwq.LIB_PATH)
    assert prod.hlwq_fault_inject(1, WAIT_NS) == hlwq.HLWQ_EUNSUPPORTED


def test_fault_hook_validates_the_wait_limit(fl):
    assert fl.lib.hlwq_fault_inject(1, 0) == fl.HLWQ_EINVAL
    assert fl.lib.hlwq_fault_inject(1, 3 * PRODUCT_WAIT_NS) == fl.HLWQ_EINVAL


@pytest.mark.parametrize("M", [1, 3, 64])
def test_wait_runs_out_then_next_call_is_correct(fl, layer, M):
    """M = 1: single-token GEMV; M = 3: few-token kernel; M = 64: tensor-core
    GEMM (tensor memory allocated, then freed on the error path)."""
    q, (p, n) = layer
    cb = fl.codebook("cuda")
    X = synth.activations(M, 5120, seed=50 + M)
    Xd = X.cuda()
    assert fl.device_error() == 0
    _inject(fl, True)
    fl.gemm(p, n, cb, Xd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fl.device_error() & fl.DEVERR_TIMEOUT
    _inject(fl, False)
    want = O.matmul(q["packed"], q["norms"], 5120, X)
    for _ in range(2):   # twice: tensor memory must be free on every SM
        Y = fl.gemm(p, n, cb, Xd, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert rel_l2(Y.double().cpu().numpy(), want) <= MATMUL_REL
    assert fl.device_error() == 0


def test_fused_moe_wait_runs_out_then_next_call_is_correct(fl):
    E, H, F, k, T = 8, 256, 128, 2, 2
    qg = [O.quantize(synth.student_t((2 * F, H), df4_seed=60 + e)) for e in range(E)]
    qd = [O.quantize(synth.student_t((H, F), df4_seed=70 + e)) for e in range(E)]
    gu = (torch.from_numpy(np.stack([q["packed"] for q in qg])).cuda(),
          torch.from_numpy(np.stack([q["norms"].view(np.uint16) for q in qg])).cuda())
    dn = (torch.from_numpy(np.stack([q["packed"] for q in qd])).cuda(),
          torch.from_numpy(np.stack([q["norms"].view(np.uint16) for q in qd])).cuda())
    cb = fl.codebook("cuda")
    logits = synth.router_logits(T, E, seed=61)
    X = synth.activations(T, H, seed=62)
    _inject(fl, True)
    fl.moe_gemv(gu, dn, cb, logits.cuda(), X.cuda(), k)
    torch.cuda.synchronize()
    assert fl.device_error() & fl.DEVERR_TIMEOUT
    _inject(fl, False)
    Y, _, _ = fl.moe_gemv(gu, dn, cb, logits.cuda(), X.cuda(), k)
    torch.cuda.synchronize()
    want, _, _ = O.moe_forward([(q["packed"], q["norms"]) for q in qg], [(q["packed"], q["norms"]) for q in qd],
                               H, F, k, logits, X)
    assert rel_l2(Y.double().cpu().numpy(), want) <= MATMUL_REL
    assert fl.device_error() == 0
