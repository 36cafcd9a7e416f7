"""GPU parity of the TQ3 path ("Qwen3.6-35B-A3B-TQ3-native", "What TQ3 actually
does") against the oracle: packed codes and fp32 shape-gain norms bit-exact
(every decision and the norm are evaluated in fp64 on both sides, the norm's
sum of squares in the same level order); dequantized weights within 1e-5
relative L2 (fp32 arithmetic); GEMV within 2e-3 relative L2 (the matmul bar),
also checked at 1e-4, what fp32 accumulation gives."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import tq3_oracle as T
from dequant_matmul_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


@pytest.fixture(scope="module")
def cb8(hl):
    return hl.kv_codebook("cuda")


@pytest.fixture(scope="module")
def signs():
    return synth.sign_vectors(42)


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _quant(hl, cb8, signs, W):
    p, n = hl.tq3_quantize(W.cuda(), signs.cuda(), cb8)
    torch.cuda.synchronize()
    s = signs.numpy()
    want = T.tq3_quantize(W, s[0], s[1])
    return p, n, want


SHAPES = [(256, 512), (300, 704), (37, 128), (1, 5120), (129, 300), (64, 9316)]


@pytest.mark.parametrize("shape", SHAPES)
def test_tq3_quantize_bit_exact(hl, cb8, signs, shape):
    W = synth.student_t(shape, df4_seed=shape[0] * 7 + shape[1])
    p, n, want = _quant(hl, cb8, signs, W)
    assert np.array_equal(p.cpu().numpy(), want["packed"])
    assert np.array_equal(n.cpu().numpy().view(np.uint32), want["norms"].view(np.uint32))
    assert hl.device_error() == 0


def test_tq3_zero_rows_groups_and_outliers(hl, cb8, signs):
    """The 256 x 512 layer with 0.1 % outliers at 20 sigma, one zero row and one
    zero group (code 3, gamma 0, decoded zeros)."""
    W = synth.gaussian_with_outliers(256, 512, seed=0).to(torch.bfloat16)
    W[3] = 0
    W[7, 128:256] = 0
    p, n, want = _quant(hl, cb8, signs, W)
    assert np.array_equal(p.cpu().numpy(), want["packed"])
    assert np.array_equal(n.cpu().numpy().view(np.uint32), want["norms"].view(np.uint32))
    assert np.all(want["codes"][3] == 3) and want["norms"][7, 1] == 0


@pytest.mark.parametrize("shape", [(256, 512), (300, 704), (65, 300)])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_tq3_dequantize(hl, cb8, signs, shape, dt):
    W = synth.student_t(shape, df4_seed=shape[1] + 1)
    p, n, want = _quant(hl, cb8, signs, W)
    s = signs.numpy()
    ref = T.tq3_dequantize(want["packed"], want["norms"], shape[1], s[0], s[1])
    got = hl.tq3_dequantize(p, n, signs.cuda(), cb8, shape[1], out_dtype=dt)
    torch.cuda.synchronize()
    g = got.double().cpu().numpy()
    assert g.shape == ref.shape
    if dt == torch.float32:
        assert rel(g, ref) <= 1e-5
    else:
        assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(ref).max())


@pytest.mark.parametrize("shape", [(256, 512), (300, 704), (1000, 2048), (512, 5120), (64, 9316), (8, 128),
                                   (3, 1000)])
def test_tq3_gemv(hl, cb8, signs, shape):
    """Slices of 1024 inputs: one CTA (in <= 1024), clusters of 2, 5 and 8 CTAs,
    and 10 slices taken in turn by a cluster of 8; ragged tails."""
    W = synth.student_t(shape, df4_seed=shape[0] + 3 * shape[1])
    p, n, want = _quant(hl, cb8, signs, W)
    x = synth.activations(1, shape[1], seed=shape[1])[0]
    s = signs.numpy()
    ref = T.tq3_matmul(want["packed"], want["norms"], shape[1], s[0], s[1], x)[0]
    y = hl.tq3_gemv(p, n, signs.cuda(), cb8, x.cuda())
    yb = hl.tq3_gemv(p, n, signs.cuda(), cb8, x.cuda(), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    e = rel(y.cpu().numpy(), ref)
    assert e <= 2e-3 and e <= 1e-4, e
    assert rel(yb.double().cpu().numpy(), ref) <= 4e-3


def test_tq3_gemv_many_rows_sampled(hl, cb8, signs):
    """700,003 rows of 200 inputs (the per-cluster row range is covered in
    several passes of 4096 rows); random codes and norms, checked on sampled
    rows against the oracle on those rows."""
    g = np.random.default_rng(21)
    O_, I_ = 700_003, 200
    packed = g.integers(0, 256, size=(O_, 2, 48), dtype=np.uint8)
    norms = g.uniform(0.05, 0.5, size=(O_, 2)).astype(np.float32)
    x = synth.activations(1, I_, seed=22)[0]
    y = hl.tq3_gemv(torch.from_numpy(packed).cuda(), torch.from_numpy(norms).cuda(), signs.cuda(), cb8, x.cuda())
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, 600), np.arange(O_ - 600, O_), g.integers(0, O_, 2000),
                                     np.arange(4090, 4100), np.arange(4096 * 5 - 5, 4096 * 5 + 5)]))
    s = signs.numpy()
    ref = T.tq3_matmul(packed[rows], norms[rows], I_, s[0], s[1], x)[0]
    assert rel(y.cpu().numpy()[rows], ref) <= 1e-4


def test_tq3_full_size_sampled(hl, cb8, signs):
    """The 27648 x 5120 layer quantized on the GPU; 48 sampled rows quantized by
    the oracle must match bit for bit, and the GEMV's outputs for those rows
    must match the oracle's matmul of its own codes."""
    O_, I_ = 27648, 5120
    W = synth.student_t_device((O_, I_), seed=77)
    p, n = hl.tq3_quantize(W, signs.cuda(), cb8)
    x = synth.activations(1, I_, seed=78)[0]
    y = hl.tq3_gemv(p, n, signs.cuda(), cb8, x.cuda())
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 1, O_ - 1], np.random.default_rng(79).integers(0, O_, 45)]))
    Ws = W[torch.from_numpy(rows).cuda()].cpu()
    s = signs.numpy()
    want = T.tq3_quantize(Ws, s[0], s[1])
    assert np.array_equal(p[torch.from_numpy(rows).cuda()].cpu().numpy(), want["packed"])
    assert np.array_equal(n[torch.from_numpy(rows).cuda()].cpu().numpy().view(np.uint32), want["norms"].view(np.uint32))
    ref = T.tq3_matmul(want["packed"], want["norms"], I_, s[0], s[1], x)[0]
    assert rel(y.cpu().numpy()[rows], ref) <= 1e-4


def test_tq3_bad_codebook_sets_the_error_bit(hl, signs):
    bad = torch.tensor([0.0, -1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0], device="cuda")
    W = synth.student_t((8, 256), df4_seed=1).cuda()
    assert hl.device_error() == 0
    p, n = hl.tq3_quantize(W, signs.cuda(), bad)
    hl.tq3_gemv(p, n, signs.cuda(), bad, synth.activations(1, 256, seed=2)[0].cuda())
    assert hl.device_error() & hl.DEVERR_CODEBOOK


# TQ3 small-M GEMM: the tensor-core kernel from M = 2 (in <= 8192), the GEMV
# once per token for M = 1 and for longer rows.
TQ3_GEMM_CASES = [
    (256, 512, 2),      # two tokens, one 16-token tile
    (300, 704, 5),      # ragged rows (300 = 2 x 128 + 44) and inputs (704 = 5.5 groups)
    (129, 300, 37),     # one row past a tile, 3 groups with a zero-padded tail, tokens past a 16-multiple
    (1000, 2048, 16),
    (512, 5120, 64),
    (200, 8192, 300),   # the longest rows the tensor-core path takes; two token tiles of 256
    (64, 9316, 3),      # rows longer than 8192: one GEMV per token
    (96, 640, 1),       # M = 1: the GEMV
]


@pytest.mark.parametrize("O_,I_,M", TQ3_GEMM_CASES)
def test_tq3_gemm(hl, cb8, signs, O_, I_, M):
    W = synth.student_t((O_, I_), df4_seed=5 * O_ + I_ + M)
    p, n, want = _quant(hl, cb8, signs, W)
    X = synth.activations(M, I_, seed=O_ + M)
    s = signs.numpy()
    ref = T.tq3_matmul(want["packed"], want["norms"], I_, s[0], s[1], X)
    Y = hl.tq3_gemm(p, n, signs.cuda(), cb8, X.cuda())
    Yb = hl.tq3_gemm(p, n, signs.cuda(), cb8, X.cuda(), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    e = rel(Y.cpu().numpy(), ref)
    assert e <= 2e-3, e
    assert rel(Yb.double().cpu().numpy(), ref) <= 4e-3
    assert hl.device_error() == 0


def test_tq3_gemm_strided_operands(hl, cb8, signs):
    """X and Y inside wider buffers (ldx > in, ldy > out): the columns past
    out are left untouched."""
    O_, I_, M = 384, 1000, 24
    W = synth.student_t((O_, I_), df4_seed=9)
    p, n, want = _quant(hl, cb8, signs, W)
    Xw = torch.zeros(M, I_ + 24, dtype=torch.bfloat16)
    Xw[:, :I_] = synth.activations(M, I_, seed=10)
    Yw = torch.full((M, O_ + 8), 7.0, dtype=torch.float32, device="cuda")
    hl.tq3_gemm(p, n, signs.cuda(), cb8, Xw.cuda()[:, :I_], Y=Yw[:, :O_])
    torch.cuda.synchronize()
    s = signs.numpy()
    ref = T.tq3_matmul(want["packed"], want["norms"], I_, s[0], s[1], Xw[:, :I_])
    assert rel(Yw[:, :O_].cpu().numpy(), ref) <= 2e-3
    assert torch.all(Yw[:, O_:] == 7.0)


def test_tq3_gemm_k_split_and_minimum_workspace(hl, cb8, signs):
    """160 row tiles on 148 SMs: the last 12 tiles are split in K (full
    workspace); with only the minimum workspace nothing is split.  Both match
    the oracle on sampled rows."""
    O_, I_, M = 160 * 128, 1000, 24
    W = synth.student_t_device((O_, I_), seed=91)
    p, n = hl.tq3_quantize(W, signs.cuda(), cb8)
    X = synth.activations(M, I_, seed=92)
    Xd = X.cuda()
    Y = hl.tq3_gemm(p, n, signs.cuda(), cb8, Xd)
    ws_min = (M * 8 * 128 * 2 + 255) // 256 * 256 + M * 4 + 256
    assert hl.workspace_bytes(hl.HLWQ_OP_TQ3_GEMM, O_, I_, M) > ws_min
    Y2 = hl.tq3_gemm(p, n, signs.cuda(), cb8, Xd, workspace=torch.empty(ws_min, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(O_ - 12 * 128 - 8, O_ - 12 * 128 + 8),
                                     np.arange(O_ - 64, O_), np.random.default_rng(93).integers(0, O_, 64)]))
    ri = torch.from_numpy(rows).cuda()
    s = signs.numpy()
    ref = T.tq3_matmul(p[ri].cpu().numpy(), n[ri].cpu().numpy(), I_, s[0], s[1], X)
    assert rel(Y.cpu().numpy()[:, rows], ref) <= 2e-3
    assert rel(Y2.cpu().numpy()[:, rows], ref) <= 2e-3


def test_tq3_gemm_full_size_sampled(hl, cb8, signs):
    """27648 x 5120 at M = 64 (216 row tiles: 148 whole tiles and 68 split in
    K over the second wave) and M = 16; outputs of sampled rows against the
    oracle's matmul of the GPU's own codes (those codes are pinned bit-exact
    by test_tq3_full_size_sampled)."""
    O_, I_ = 27648, 5120
    W = synth.student_t_device((O_, I_), seed=81)
    p, n = hl.tq3_quantize(W, signs.cuda(), cb8)
    del W
    rows = np.unique(np.concatenate([[0, 1, 127, 128, O_ - 129, O_ - 1],
                                     np.random.default_rng(82).integers(0, O_, 58)]))
    ri = torch.from_numpy(rows).cuda()
    ps, ns = p[ri].cpu().numpy(), n[ri].cpu().numpy()
    s = signs.numpy()
    for M in (16, 64):
        X = synth.activations(M, I_, seed=83 + M)
        Y = hl.tq3_gemm(p, n, signs.cuda(), cb8, X.cuda())
        torch.cuda.synchronize()
        ref = T.tq3_matmul(ps, ns, I_, s[0], s[1], X)
        assert rel(Y.cpu().numpy()[:, rows], ref) <= 2e-3
    assert hl.device_error() == 0
