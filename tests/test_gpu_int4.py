"""GPU parity of the Q5 -> INT4 re-encoder against the oracle: codes, scales
and zeros bit-exact (every decision is taken in fp64 on both sides on values
that are exact in fp64)."""
import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth
from gpu_helpers import oracle_to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


@pytest.fixture(scope="module")
def cb(hl):
    return hl.codebook("cuda")


def _check(hl, cb, q, in_f, rows=None):
    p, n = oracle_to_dev(q)
    q4, s, z = hl.requantize_int4(p, n, cb, in_f)
    torch.cuda.synchronize()
    want = O.requantize_int4(q["packed"], q["norms"], in_f)
    assert np.array_equal(q4.cpu().numpy(), want["q4"])
    assert np.array_equal(s.cpu().numpy(), want["scale"])
    assert np.array_equal(z.cpu().numpy(), want["zero"])
    return want


@pytest.mark.parametrize("shape", [(256, 512), (300, 1024), (37, 128), (1, 5120), (4099, 256)])
def test_int4_shapes_bit_exact(hl, cb, shape):
    W = synth.student_t(shape, df4_seed=shape[0] + shape[1])
    _check(hl, cb, O.quantize(W), shape[1])
    assert hl.device_error() == 0


def test_int4_outliers_zero_and_constant_blocks(hl, cb):
    """The 256 x 512 fp32 layer with 0.1 % outliers at 20 sigma, with one all-zero
    row and one row of equal weights per block (s = 0 after the Q5 round trip
    only for the zero row: a constant block rotates to one non-zero value)."""
    W = synth.gaussian_with_outliers(256, 512, seed=0).numpy().copy()
    W[3] = 0.0
    W[5] = 0.01
    want = _check(hl, cb, O.quantize(W), 512)
    assert np.all(want["scale"][3] == 0) and np.all(want["q4"][3] == 0)


def test_int4_stacked_experts(hl, cb):
    """[E][rows][NB][80] inputs (the expert layers of the MoE configs)."""
    W = synth.student_t((4, 96, 512), df4_seed=3)
    q = O.quantize(W.reshape(-1, 512))
    p, n = oracle_to_dev(q)
    q4, s, z = hl.requantize_int4(p.view(4, 96, 4, 80), n.view(4, 96, 4), cb, 512)
    torch.cuda.synchronize()
    want = O.requantize_int4(q["packed"], q["norms"], 512)
    assert q4.shape == (4, 96, 4, 64)
    assert np.array_equal(q4.cpu().numpy().reshape(-1, 4, 64), want["q4"])
    assert np.array_equal(s.cpu().numpy().reshape(-1, 4), want["scale"])
    assert np.array_equal(z.cpu().numpy().reshape(-1, 4), want["zero"])


def test_int4_full_27648x5120_sampled_rows(hl, cb):
    """The 27648 x 5120 layer, Q5-encoded on the device; the oracle re-encodes
    the device's codes of 256 sampled rows."""
    W = synth.student_t_device((27648, 5120), seed=21)
    p, n = hl.quantize(W, cb)
    del W
    q4, s, z = hl.requantize_int4(p, n, cb, 5120)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(2).choice(27648, 256, replace=False))
    ri = torch.as_tensor(rows, device="cuda")
    pk = p[ri].cpu().numpy()
    nm = n.view(torch.int16)[ri].cpu().numpy().view(np.float16)   # (no uint16 indexing on the device)
    want = O.requantize_int4(pk, nm, 5120)
    assert np.array_equal(q4[ri].cpu().numpy(), want["q4"])
    assert np.array_equal(s.view(torch.int16)[ri].cpu().numpy().view(np.uint16), want["scale"])
    assert np.array_equal(z.view(torch.int16)[ri].cpu().numpy().view(np.uint16), want["zero"])
    assert hl.device_error() == 0


def test_int4_rejects_unaligned_rows(hl, cb):
    W = synth.student_t((8, 704), df4_seed=1)
    p, n = oracle_to_dev(O.quantize(W))
    with pytest.raises(hl.HLWQError):
        hl.requantize_int4(p, n, cb, 704)
