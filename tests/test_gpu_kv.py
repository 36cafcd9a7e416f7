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


# --------------------------------------------------------------------------
# Residual window: appends encode the tokens that leave the window, oldest
# first, bit-exact with the oracle; scores cover encoded and exact keys.
# --------------------------------------------------------------------------

def _window_state_matches(cache, Xall, n_total, R):
    """Encoded rows and window slots against the oracle's state after the
    same tokens."""
    n_enc = max(0, n_total - R)
    assert cache.n_enc == n_enc and cache.n_total == n_total
    if n_enc:
        want = O.kv_quantize(Xall[:n_enc])
        assert np.array_equal(cache.packed[:n_enc].cpu().numpy(), want["packed"])
        assert np.array_equal(cache.norms[:n_enc].cpu().numpy(), want["norms"].view(np.uint16))
    win = cache.window.cpu()
    for i in range(n_enc, n_total):
        assert torch.equal(win[i % R], Xall[i]), i


@pytest.mark.parametrize("R,chunks", [(128, [1, 3, 200, 1, 128, 50, 7]), (5, [2, 2, 9, 1, 1, 13]),
                                      (128, [300])])
def test_kv_window_append_matches_the_oracle(hl, cb8, R, chunks):
    Xall = _keys(sum(chunks), seed=R + len(chunks))
    cache = hl.KVWindowCache(capacity=sum(chunks), R=R, cb8=cb8)
    n = 0
    for c in chunks:
        cache.append(Xall[n:n + c].cuda())
        n += c
        torch.cuda.synchronize()
        _window_state_matches(cache, Xall, n, R)
    assert hl.device_error() == 0


@pytest.mark.parametrize("R,n_tokens,m", [(128, 1000, 6), (128, 100, 3), (7, 40, 64), (128, 128, 1)])
def test_kv_scores_window_one_launch(hl, cb8, R, n_tokens, m):
    Xall = _keys(n_tokens, seed=n_tokens + m)
    Q = synth.activations(m, 256, seed=19 + m)
    cache = hl.KVWindowCache(capacity=n_tokens, R=R, cb8=cb8)
    cache.append(Xall.cuda())
    S = cache.scores(Q.cuda())
    torch.cuda.synchronize()
    p, nrm, w = O.kv_window_append(np.zeros((0, 96), np.uint8), np.zeros(0, np.float16), np.zeros((0, 256)),
                                   Xall, capacity=R)
    want = O.kv_scores_window(Q, p, nrm, w)
    got = S.cpu().numpy()
    assert got.shape == want.shape == (m, n_tokens)
    ne = cache.n_enc
    if ne:
        assert rel_l2(got[:, :ne], want[:, :ne]) <= 1e-5
    # exact keys: fp32 rotation and dot against the fp64 dot of the bf16 values
    assert rel_l2(got[:, ne:], want[:, ne:]) <= 1e-6


def test_kv_scores_window_edges(hl, cb8):
    """A cache with no window tokens (window may be NULL) equals hlwq_kv_scores;
    a cache with no encoded tokens scores only exact keys."""
    K = _keys(300, seed=23)
    Q = synth.activations(4, 256, seed=24).cuda()
    kq = O.kv_quantize(K)
    p = torch.from_numpy(kq["packed"]).cuda()
    nr = torch.from_numpy(kq["norms"].view(np.uint16)).cuda()
    S0 = hl.kv_scores(Q, p, nr, cb8)
    S1 = torch.empty(4, 300, dtype=torch.float32, device="cuda")
    st = hl.lib.hlwq_kv_scores_window(hl._ptr(Q), 4, 256, hl._ptr(p), hl._ptr(nr), hl._ptr(cb8), 300, None, 128, 300,
                                      hl._ptr(S1), 300, None)
    assert st == hl.HLWQ_OK
    win = K[:100].cuda()
    S2 = torch.empty(4, 100, dtype=torch.float32, device="cuda")
    st = hl.lib.hlwq_kv_scores_window(hl._ptr(Q), 4, 256, None, None, hl._ptr(cb8), 0, hl._ptr(win), 128, 100,
                                      hl._ptr(S2), 100, None)
    assert st == hl.HLWQ_OK
    torch.cuda.synchronize()
    assert torch.equal(S0, S1)
    want = Q.cpu().double().numpy() @ K[:100].double().numpy().T
    assert rel_l2(S2.cpu().numpy(), want) <= 1e-6
