"""GPU parity: quantizer and dequantizer against the oracle (element by element)."""
import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth
from gpu_helpers import DEQ_REL, check_quantized, oracle_to_dev, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


@pytest.fixture(scope="module")
def cb(hl):
    return hl.codebook("cuda")


def test_quantize_fp32_outliers_256x512(hl, cb):
    """Single Linear out=256, in=512, fp32 N(0, 0.02^2) + 0.1% outliers at 20 sigma."""
    W = synth.gaussian_with_outliers(256, 512, seed=0)
    p, n = hl.quantize(W.cuda(), cb)
    torch.cuda.synchronize()
    r = check_quantized(p, n, W)
    assert r["codes"] == 256 * 4 * 128
    assert hl.device_error() == 0


@pytest.mark.parametrize("shape", [(64, 704), (33, 129), (5, 127), (3, 1), (7, 1000), (130, 2816)])
def test_quantize_bf16_ragged(hl, cb, shape):
    W = synth.student_t(shape, df4_seed=shape[0] + shape[1])
    p, n = hl.quantize(W.cuda(), cb)
    torch.cuda.synchronize()
    check_quantized(p, n, W)


def test_quantize_misaligned_source(hl, cb):
    """W starting 2 bytes past a 16-byte boundary takes the scalar load path."""
    W = synth.student_t((40, 513), df4_seed=3)
    base = torch.zeros(40 * 513 + 8, dtype=torch.bfloat16, device="cuda")
    view = base[1:1 + 40 * 513].view(40, 513)
    view.copy_(W.cuda())
    p, n = hl.quantize(view, cb)
    torch.cuda.synchronize()
    check_quantized(p, n, W)


def test_quantize_degenerate_blocks(hl, cb):
    """Zero block, single spike, constant block (127 values exactly on the
    centre midpoint -> ties to code 15), tiny and huge scales."""
    W = torch.zeros(8, 256, dtype=torch.float32)
    W[1, 3] = -0.7                         # spike: every y = +-1
    W[2, :128] = 0.01                      # constant: y = sqrt(128) e_0
    W[3] = synth.student_t((1, 256), dtype=torch.float32, df4_seed=4)[0] * 1e-30
    W[4] = synth.student_t((1, 256), dtype=torch.float32, df4_seed=5)[0] * 1e30
    W[5, 128:] = synth.student_t((1, 128), dtype=torch.float32, df4_seed=6)[0]
    W[6] = -0.02
    W[7, 255] = 3.0
    p, n = hl.quantize(W.cuda(), cb)
    torch.cuda.synchronize()
    check_quantized(p, n, W)
    assert hl.device_error() == 0


def test_quantize_dense_5120_full(hl, cb):
    """Dense decode layer 5120 x 5120, bf16 Student-t(4) std 0.02: every code and norm."""
    W = synth.student_t((5120, 5120), df4_seed=0)
    p, n = hl.quantize(W.cuda(), cb)
    torch.cuda.synchronize()
    r = check_quantized(p, n, W)
    assert r["codes"] == 5120 * 40 * 128


def test_quantize_experts_stacked(hl, cb):
    """Experts are independent: a stacked [E][O][I] call equals per-expert calls."""
    W = synth.student_t((4, 96, 704), df4_seed=7).cuda()
    p, n = hl.quantize(W, cb)
    for e in range(4):
        pe, ne = hl.quantize(W[e].contiguous(), cb)
        assert torch.equal(pe, p[e]) and torch.equal(ne, n[e])


@pytest.mark.parametrize("shape", [(256, 512), (48, 704), (9, 130)])
@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16])
def test_dequantize(hl, cb, shape, odt):
    W = synth.student_t(shape, df4_seed=11)
    q = O.quantize(W)
    p, n = oracle_to_dev(q)
    got = hl.dequantize(p, n, cb, shape[1], out_dtype=odt)
    torch.cuda.synchronize()
    want = O.dequantize(q["packed"], q["norms"], shape[1])
    g = got.double().cpu().numpy()
    if odt == torch.float32:
        assert rel_l2(g, want) <= DEQ_REL
        # per-block bound: |error| <= 1e-5 * n / sqrt(128)
        nb = q["norms"].shape[1]
        pad = np.zeros((shape[0], nb * 128))
        pad[:, : shape[1]] = np.abs(g - want)
        bound = 1e-5 * q["norms"].astype(np.float64) / np.sqrt(128.0)
        assert np.all(pad.reshape(shape[0], nb, 128).max(-1) <= bound + 1e-30)
    else:
        # bf16 output: exactly the bf16 rounding of the fp32 result (within one bf16 ulp of fp64)
        assert rel_l2(g, want) <= 4e-3


def test_quantize_codebook_with_midpoints_beyond_the_table(hl, cb):
    """A strictly ascending codebook whose outer decision midpoints lie beyond
    +-3 (the Lloyd-Max centroids times 1.6, outermost midpoint ~4): rotated
    values beyond the quantizer's bucket table go to its exact path, so the
    codes still equal brute-force nearest-centroid codes of the oracle's
    rotated values (decisions within 1e-5 of a midpoint excepted)."""
    wide = (cb * 1.6).contiguous()
    c = wide.cpu().double().numpy()
    mids = 0.5 * (c[1:] + c[:-1])
    assert mids.max() > 3.5 and mids.min() < -3.5
    W = synth.gaussian_with_outliers(256, 1024, seed=7)
    p, n = hl.quantize(W.cuda(), wide)
    torch.cuda.synchronize()
    assert hl.device_error() == 0
    q = O.quantize(W, return_rotated=True)
    y = q["y"]
    assert (np.abs(y) > 3.5).sum() > 50  # the case is exercised
    want = O.nearest_centroid(y, c)
    got = O.unpack_codes(p.cpu().numpy()).reshape(want.shape)
    bad = got != want
    if bad.any():
        near = np.min(np.abs(y[bad][:, None] - mids[None, :]), axis=1)
        assert np.all(near < 1e-5), (int(bad.sum()), float(near.max()))
