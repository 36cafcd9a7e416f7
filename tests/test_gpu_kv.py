"""GPU parity of the Q3 KV-cache encoding against the oracle: codes and norms
bit-exact (the quantizer decides in fp64 like the oracle), decoded vectors and
attention scores within fp32 rounding of the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth
from gpu_helpers import rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


@pytest.fixture(scope="module")
def cb8(hl):
    return hl.kv_codebook("cuda")


def _keys(n, seed):
    X = synth.activations(n, 256, seed=seed).float()
    X[:, :3] *= 30.0          # a few large channels, as keys have
    X[0] = 0.0                # a zero vector
    return X.to(torch.bfloat16)


@pytest.mark.parametrize("n,ld", [(1, 256), (5, 256), (1000, 256), (77, 264), (33, 260)])
def test_kv_quantize_bit_exact(hl, cb8, n, ld):
    X = _keys(n, seed=n + ld)
    buf = torch.zeros(n, ld, dtype=torch.bfloat16)
    buf[:, :256] = X
    Xd = buf.cuda()[:, :256]
    p, nr = hl.kv_quantize(Xd, cb8)
    torch.cuda.synchronize()
    want = O.kv_quantize(X)
    got_codes = O.unpack_codes(p.cpu().numpy(), bits=3)
    bad = got_codes != want["codes"]
    if bad.any():
        _, mid, _ = O.codebook_fp32(8)
        assert np.all(np.min(np.abs(want["y"][bad][:, None] - mid[None, :]), axis=1) < 1e-12)
    assert np.array_equal(nr.cpu().numpy(), want["norms"].view(np.uint16))
    assert hl.device_error() == 0


def test_kv_dequantize(hl, cb8):
    X = _keys(513, seed=3)
    want_q = O.kv_quantize(X)
    p = torch.from_numpy(want_q["packed"]).cuda()
    nr = torch.from_numpy(want_q["norms"].view(np.uint16)).cuda()
    want = O.kv_dequantize(want_q["packed"], want_q["norms"])
    out = hl.kv_dequantize(p, nr, cb8)
    out16 = hl.kv_dequantize(p, nr, cb8, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert rel_l2(out.cpu().numpy(), want) <= 1e-5
    w16 = torch.from_numpy(want).float().to(torch.bfloat16).float().numpy()
    g16 = out16.float().cpu().numpy()
    # within one bf16 ulp, plus the fp32 rounding of the decode relative to the
    # vector's RMS (n / 16) for entries near zero
    rms = want_q["norms"].astype(np.float64)[:, None] / 16.0
    assert np.all(np.abs(g16 - w16) <= 2.0 ** -7 * np.abs(w16) + 1e-5 * rms)


@pytest.mark.parametrize("m,n", [(1, 1), (6, 300), (64, 4097)])
def test_kv_scores(hl, cb8, m, n):
    K = _keys(n, seed=7 + n)
    Q = synth.activations(m, 256, seed=11 + m)
    kq = O.kv_quantize(K)
    p = torch.from_numpy(kq["packed"]).cuda()
    nr = torch.from_numpy(kq["norms"].view(np.uint16)).cuda()
    S = hl.kv_scores(Q.cuda(), p, nr, cb8)
    torch.cuda.synchronize()
    want = O.kv_scores(Q, kq["packed"], kq["norms"])
    assert S.shape == (m, n)
    assert rel_l2(S.cpu().numpy(), want) <= 1e-5


def test_kv_scores_limits(hl, cb8):
    Q = synth.activations(65, 256, seed=1).cuda()
    p = torch.zeros(4, 96, dtype=torch.uint8, device="cuda")
    nr = torch.zeros(4, dtype=torch.uint16, device="cuda")
    with pytest.raises(hl.HLWQError):
        hl.kv_scores(Q, p, nr, cb8)


def test_kv_codebook_error_word(hl, cb8):
    X = _keys(8, seed=1).cuda()
    hl.device_error()
    hl.kv_quantize(X, torch.flip(cb8, dims=[0]).contiguous())
    torch.cuda.synchronize()
    assert hl.device_error() & 0x1
    assert hl.device_error() == 0
