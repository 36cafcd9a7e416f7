"""Device-side errors are reported, not trapped.  A codebook that is not
strictly ascending is only visible on the device: every call that reads the
codebook (quantize, the decode GEMV, the multi-token and tensor-core GEMMs,
both MoE paths) must still complete, raise HLWQ_DEVERR_CODEBOOK in the device
error word, and leave the context usable.  hlwq_device_error reads and clears
the word.  A descending codebook keeps every index in range (codes count the
midpoints below a value; decode tables are plain lookups), so these calls
cannot fault."""
import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth
from gpu_helpers import MATMUL_REL, oracle_to_dev, rel_l2

pytestmark = pytest.mark.gpu

DEVERR_CODEBOOK = 0x1  # include/hlwq.h


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


def _moe_weights(E, H, F):
    nbh, nbf = O.n_blocks(H), O.n_blocks(F)
    gu_p = np.zeros((E, 2 * F, nbh, 80), np.uint8)
    gu_n = np.zeros((E, 2 * F, nbh), np.uint16)
    dn_p = np.zeros((E, H, nbf, 80), np.uint8)
    dn_n = np.zeros((E, H, nbf), np.uint16)
    for e in range(E):
        qg = O.quantize(synth.student_t((2 * F, H), df4_seed=40 + 2 * e))
        qd = O.quantize(synth.student_t((H, F), df4_seed=41 + 2 * e))
        gu_p[e], gu_n[e] = qg["packed"], qg["norms"].view(np.uint16)
        dn_p[e], dn_n[e] = qd["packed"], qd["norms"].view(np.uint16)
    gu = (torch.from_numpy(gu_p).cuda(), torch.from_numpy(gu_n).cuda())
    dn = (torch.from_numpy(dn_p).cuda(), torch.from_numpy(dn_n).cuda())
    return gu, dn


def test_descending_codebook_raises_the_error_word_and_context_survives(hl):
    cb = hl.codebook("cuda")
    torch.cuda.synchronize()
    assert hl.device_error() == 0
    in_f, out_f = 640, 256
    W = synth.student_t((out_f, in_f), df4_seed=3)
    q = O.quantize(W)
    p, n = oracle_to_dev(q)
    X16 = synth.activations(16, in_f, seed=4).cuda()
    E, H, F = 8, 256, 128
    gu, dn = _moe_weights(E, H, F)
    calls = {
        "quantize": lambda c: hl.quantize(W.cuda(), c),
        "gemv": lambda c: hl.gemv(p, n, c, X16[0]),
        "gemm_m4": lambda c: hl.gemm(p, n, c, X16[:4], out_dtype=torch.float32),
        "gemm_m16": lambda c: hl.gemm(p, n, c, X16, out_dtype=torch.float32),
        "moe_t1": lambda c: hl.moe_gemv(gu, dn, c, synth.router_logits(1, E, seed=5).cuda(),
                                        synth.activations(1, H, seed=6).cuda(), 2),
        "moe_t64": lambda c: hl.moe_gemv(gu, dn, c, synth.router_logits(64, E, seed=7).cuda(),
                                         synth.activations(64, H, seed=8).cuda(), 2),
    }
    bad_books = {
        "descending": torch.flip(cb, dims=[0]).contiguous(),
        "two_equal": torch.cat([cb[:16], cb[15:16], cb[17:]]).contiguous(),
    }
    for bname, bad in bad_books.items():
        assert bad.numel() == 32
        for name, call in calls.items():
            call(cb)  # a correct call first: no error
            torch.cuda.synchronize()
            assert hl.device_error() == 0, (bname, name)
            call(bad)
            torch.cuda.synchronize()
            assert hl.device_error() & DEVERR_CODEBOOK, (bname, name)
            assert hl.device_error() == 0, (bname, name)  # read-and-clear
    # the context is intact and the results are right again
    for M in (1, 4, 16):
        Y = hl.gemm(p, n, cb, X16[:M], out_dtype=torch.float32) if M > 1 else hl.gemv(p, n, cb, X16[0])[None]
        torch.cuda.synchronize()
        want = O.matmul(q["packed"], q["norms"], in_f, X16[:M].cpu())
        assert rel_l2(Y.double().cpu().numpy(), want) <= MATMUL_REL, M
    assert hl.device_error() == 0
