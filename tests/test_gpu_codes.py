"""GPU parity of the one-code-per-byte layout ("Gemma-4-26B-A4B-it-HLWQ-Q5",
Technical Details: int8 codes) against the oracle's 5-bit pack and unpack
(Method step [5], pinned by hand-computed bytes in test_oracle_quantizer.py):
bit-exact in both directions, ragged block counts, the range check."""
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


@pytest.mark.parametrize("nblocks", [1, 3, 7, 8, 9, 64, 65, 1027, 148 * 64 * 8 + 5])
def test_pack_and_unpack_random_codes(hl, nblocks):
    g = np.random.default_rng(nblocks)
    codes = g.integers(0, 32, size=(nblocks, 128), dtype=np.uint8)
    want = O.pack_codes(codes, bits=5)
    dc = torch.from_numpy(codes).cuda()
    packed = hl.codes_pack(dc)
    assert np.array_equal(packed.cpu().numpy(), want)
    back = hl.codes_unpack(torch.from_numpy(want).cuda())
    assert np.array_equal(back.cpu().numpy(), codes)
    assert hl.device_error() == 0


def test_unpack_of_quantized_layer(hl):
    """The codes of a quantized 300 x 704 layer (ragged tail block), as the
    oracle's quantizer wrote them; [rows][NB][80] <-> [rows][NB][128]."""
    W = synth.student_t((300, 704), df4_seed=11)
    q = O.quantize(W)
    p, _ = oracle_to_dev(q)
    codes = hl.codes_unpack(p.view(300, 6, 80))
    assert codes.shape == (300, 6, 128)
    assert np.array_equal(codes.cpu().numpy().reshape(300, 6, 128),
                          O.unpack_codes(q["packed"], bits=5).reshape(300, 6, 128))
    assert torch.equal(hl.codes_pack(codes).view(-1), p.view(-1))


def test_every_code_at_every_position(hl):
    """All 32 codes at all 128 positions: block v holds code (v + j) % 32 at j."""
    j = np.arange(128)
    codes = np.stack([(v + j) % 32 for v in range(32)]).astype(np.uint8)
    packed = hl.codes_pack(torch.from_numpy(codes).cuda()).cpu().numpy()
    assert np.array_equal(packed, O.pack_codes(codes, bits=5))


def test_code_above_31_sets_the_range_bit(hl):
    """A code above 31 keeps its low five bits and raises the device error bit;
    the bit is cleared by the read."""
    g = np.random.default_rng(5)
    codes = g.integers(0, 32, size=(20, 128), dtype=np.uint8)
    bad = codes.copy()
    bad[13, 77] = 0xE5
    assert hl.device_error() == 0
    packed = hl.codes_pack(torch.from_numpy(bad).cuda())
    assert hl.device_error() == hl.DEVERR_CODE_RANGE
    fixed = codes.copy()
    fixed[13, 77] = 0xE5 & 31
    assert np.array_equal(packed.cpu().numpy(), O.pack_codes(fixed, bits=5))
    assert hl.device_error() == 0
