"""GPU parity: fused dequant GEMV / small-M GEMM against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import oracle as O_
from dequant_matmul_b200 import synth
from gpu_helpers import MATMUL_REL, oracle_to_dev, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


@pytest.fixture(scope="module")
def cb(hl):
    return hl.codebook("cuda")


def _layer(shape, seed):
    W = synth.student_t(shape, df4_seed=seed)
    return W, O.quantize(W)


def test_gemv_256x512_fp32_outliers(hl, cb):
    W = synth.gaussian_with_outliers(256, 512, seed=0)
    q = O.quantize(W)
    p, n = oracle_to_dev(q)
    x = synth.activations(1, 512, seed=1)
    y = hl.gemv(p, n, cb, x[0].cuda())
    torch.cuda.synchronize()
    want = O.matmul(q["packed"], q["norms"], 512, x)[0]
    assert rel_l2(y.cpu().numpy(), want) <= MATMUL_REL


@pytest.mark.parametrize("shape", [(5120, 5120), (300, 704), (37, 1000), (1, 128), (4099, 256)])
def test_gemv_shapes(hl, cb, shape):
    W, q = _layer(shape, seed=shape[0])
    p, n = oracle_to_dev(q)
    x = synth.activations(1, shape[1], seed=2)
    for odt in (torch.float32, torch.bfloat16):
        y = hl.gemv(p, n, cb, x[0].cuda(), out_dtype=odt)
        torch.cuda.synchronize()
        want = O.matmul(q["packed"], q["norms"], shape[1], x)[0]
        tol = MATMUL_REL if odt == torch.float32 else MATMUL_REL
        assert rel_l2(y.double().cpu().numpy(), want) <= tol, odt


def test_gemv_activation_scale_extremes(hl, cb):
    """Activations far from unit scale (the rotated activation is rescaled by a
    power of two before it is stored in binary16)."""
    W, q = _layer((128, 512), seed=9)
    p, n = oracle_to_dev(q)
    for s in (1e-20, 1e3, 3e4):
        x = (synth.activations(1, 512, seed=3, dtype=torch.float32) * s).to(torch.bfloat16)
        y = hl.gemv(p, n, cb, x[0].cuda())
        torch.cuda.synchronize()
        want = O.matmul(q["packed"], q["norms"], 512, x)[0]
        assert rel_l2(y.cpu().numpy(), want) <= MATMUL_REL, s


def test_gemv_ex_weights_static_chain(hl, cb):
    """hlwq_gemv_ex with HLWQ_FLAG_WEIGHTS_STATIC on a chain of square layers in
    which every GEMV reads the bf16 output of the kernel before it (the decode
    pattern; each launch's set-up overlaps the previous kernel), with a torch
    kernel producing the input of every other layer.  Bit-identical to plain
    launches, and each layer matches the oracle on the input it was given."""
    D = 2048
    layers = [_layer((D, D), seed=40 + l) for l in range(4)]
    devs = [oracle_to_dev(q) for _, q in layers]
    x0 = synth.activations(1, D, seed=41)[0].cuda()
    outs = {}
    for flags in (0, hl.HLWQ_FLAG_WEIGHTS_STATIC):
        x, ins, ys = x0.clone(), [], []
        for l, (p, n) in enumerate(devs):
            if l % 2:
                x = (x.float() * 1.0).to(torch.bfloat16)   # a torch kernel writes this layer's input
            ins.append(x)
            x = hl.gemv(p, n, cb, x, out_dtype=torch.bfloat16, flags=flags)
            ys.append(x)
        torch.cuda.synchronize()
        outs[flags] = (ins, ys)
    for a, b in zip(outs[0][1], outs[hl.HLWQ_FLAG_WEIGHTS_STATIC][1]):
        assert torch.equal(a, b)
    for (W, q), xin, y in zip(layers, *outs[hl.HLWQ_FLAG_WEIGHTS_STATIC]):
        want = O.matmul(q["packed"], q["norms"], D, xin.cpu()[None])[0]
        assert rel_l2(y.double().cpu().numpy(), want) <= MATMUL_REL


@pytest.mark.parametrize("flags", [0, 1])
def test_gemv_caller_codebook_replaces_the_expected_one(hl, cb, flags):
    """The single-token GEMV builds its table from the Lloyd-Max centroids it
    expects and rebuilds it when the caller's codebook differs.  With every
    centroid doubled (exact in binary16 and fp32) each product and each fp32
    partial sum doubles exactly, so y must be exactly 2 y; a codebook scaled
    by 1.6 must give 1.6 y within the matmul tolerance."""
    W, q = _layer((1024, 5120), seed=31)
    p, n = oracle_to_dev(q)
    x = synth.activations(1, 5120, seed=32)[0].cuda()
    y1 = hl.gemv(p, n, cb, x, flags=flags)
    y2 = hl.gemv(p, n, (cb * 2).contiguous(), x, flags=flags)
    y3 = hl.gemv(p, n, (cb * 1.6).contiguous(), x, flags=flags)
    y4 = hl.gemv(p, n, cb, x, flags=flags)   # back to the expected codebook
    torch.cuda.synchronize()
    assert torch.equal(y2, 2 * y1)
    assert torch.equal(y4, y1)
    want = O.matmul(q["packed"], q["norms"], 5120, x.cpu()[None])[0]
    assert rel_l2(y3.double().cpu().numpy(), 1.6 * want) <= MATMUL_REL
    assert hl.device_error() == 0


@pytest.mark.parametrize("M", [1, 3, 16])
def test_accumulation_with_one_dominant_rotated_value_per_block(hl, cb, M):
    """Each 128-block of x is 4 H[j] plus noise of std 0.1 (kept by bf16), so
    its rotated block is one value 512 beside values ~500x smaller, and a few
    rows have norms 1000x the others; y (fp32 and bf16 out) must stay within
    the matmul tolerance (every product is added to an fp32 accumulator)."""
    O_, I = 512, 2048
    W = synth.student_t((O_, I), df4_seed=33).double()
    W[::37] *= 1000.0
    W = W.to(torch.bfloat16)
    q = O.quantize(W)
    p, n = oracle_to_dev(q)
    H = O.sylvester_hadamard(128).astype(np.float64)
    g = np.random.default_rng(34)
    X = np.empty((M, I))
    for m in range(M):
        for b in range(I // 128):
            j = int(g.integers(0, 128))
            X[m, 128 * b:128 * (b + 1)] = 4.0 * H[j] + 0.1 * g.standard_normal(128)
    Xb = torch.from_numpy(X).to(torch.bfloat16)
    want = O.matmul(q["packed"], q["norms"], I, Xb)
    for odt in (torch.float32, torch.bfloat16):
        Y = hl.gemm(p, n, cb, Xb.cuda(), out_dtype=odt)
        torch.cuda.synchronize()
        err = rel_l2(Y.double().cpu().numpy(), want)
        print(f"[margin] dominant rotated value, M={M}, {odt}: rel L2 {err:.2e} (bar {MATMUL_REL})")
        assert err <= MATMUL_REL, (odt, err)


def test_gemv_ex_rejects_unknown_flags(hl, cb):
    W, q = _layer((64, 256), seed=3)
    p, n = oracle_to_dev(q)
    x = synth.activations(1, 256, seed=3)[0].cuda()
    y = torch.empty(64, device="cuda")
    st = hl.lib.hlwq_gemv_ex(p.data_ptr(), n.data_ptr(), cb.data_ptr(), 64, 256, x.data_ptr(), y.data_ptr(),
                             hl.HLWQ_F32, 0x2, torch.cuda.current_stream().cuda_stream)
    assert st == hl.HLWQ_EINVAL


def _sampled_gemv(hl, cb, Od, I, seed, rows):
    W = synth.student_t_device((Od, I), seed=seed)
    p, n = hl.quantize(W, cb)
    x = synth.activations(1, I, seed=seed + 1)
    y = hl.gemv(p, n, cb, x[0].cuda())
    torch.cuda.synchronize()
    q = O.quantize(W[torch.as_tensor(rows, device=W.device)].cpu())
    del W, p, n
    want = O.matmul(q["packed"], q["norms"], I, x)[0]
    return rel_l2(y.cpu().numpy()[rows], want)


def test_gemv_long_rows_several_passes(hl, cb):
    """in = 27648 (216 blocks): the rotated activation takes most of shared
    memory, so the code ring is one slot deep and a CTA covers its 44 rows in
    two passes of 36 and 8 (rows sampled for the oracle: the first CTAs' pass
    boundaries, the last rows and random rows)."""
    Od, I = 6000, 27648
    rows = np.unique(np.concatenate([np.arange(0, 48), np.arange(80, 92), np.arange(Od - 16, Od),
                                     np.random.default_rng(1).choice(Od, 24, replace=False)]))
    assert _sampled_gemv(hl, cb, Od, I, 12, rows) <= MATMUL_REL


def test_gemv_rows_too_long_for_the_ring(hl, cb):
    """in = 32768 (256 blocks): no code ring fits beside the table and the
    activation; the CUDA-core decode kernel takes the call."""
    Od, I = 600, 32768
    rows = np.unique(np.concatenate([np.arange(0, 16), np.arange(Od - 8, Od),
                                     np.random.default_rng(2).choice(Od, 24, replace=False)]))
    assert _sampled_gemv(hl, cb, Od, I, 14, rows) <= MATMUL_REL


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 9, 15, 16, 17, 64])
def test_gemm_small_m(hl, cb, M):
    W, q = _layer((1024, 5120), seed=21)
    p, n = oracle_to_dev(q)
    X = synth.activations(M, 5120, seed=M)
    Y = hl.gemm(p, n, cb, X.cuda(), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    want = O.matmul(q["packed"], q["norms"], 5120, X)
    assert rel_l2(Y.double().cpu().numpy(), want) <= MATMUL_REL


@pytest.mark.parametrize("M", [3, 6])
def test_gemm_ragged_fp32_out_and_pitch(hl, cb, M):
    """Row pitches larger than the rows (X: 720 > 704, Y: 208 > 200) on the
    multi-token CUDA-core path (M = 3) and the tensor-core path (M = 6, with
    the workspace hlwq_workspace_bytes reports); the pitch padding of Y stays
    untouched."""
    W, q = _layer((200, 704), seed=5)
    p, n = oracle_to_dev(q)
    X = synth.activations(M, 720, seed=6)[:, :704]        # row pitch 720 > in
    Xd = X.cuda()
    Y = torch.full((M, 208), 7.0, device="cuda")          # row pitch 208 > out
    need = hl.workspace_bytes(hl.HLWQ_OP_GEMM, 200, 704, M)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    st = hl.lib.hlwq_gemm(p.data_ptr(), n.data_ptr(), cb.data_ptr(), 200, 704, M, Xd.data_ptr(), Xd.stride(0),
                          Y.data_ptr(), 208, hl.HLWQ_F32, ws.data_ptr() if need else None, need,
                          torch.cuda.current_stream().cuda_stream)
    assert st == hl.HLWQ_OK
    torch.cuda.synchronize()
    want = O.matmul(q["packed"], q["norms"], 704, X)
    assert rel_l2(Y[:, :200].cpu().numpy(), want) <= MATMUL_REL
    assert torch.all(Y[:, 200:] == 7.0)


def test_gemm_m1_equals_gemv(hl, cb):
    W, q = _layer((512, 1024), seed=8)
    p, n = oracle_to_dev(q)
    x = synth.activations(1, 1024, seed=4).cuda()
    a = hl.gemv(p, n, cb, x[0])
    b = hl.gemm(p, n, cb, x, out_dtype=torch.float32)[0]
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_gemv_full_27648x5120_sampled_rows(hl, cb):
    """The 27648 x 5120 layer at full size (GPU-quantized); rows sampled for the
    oracle, which encodes them itself from the same synthetic weights."""
    W = synth.student_t((27648, 5120), df4_seed=0)
    p, n = hl.quantize(W.cuda(), cb)
    X = synth.activations(4, 5120, seed=11)
    Y1 = hl.gemv(p, n, cb, X[0].cuda())
    Y4 = hl.gemm(p, n, cb, X.cuda(), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(27648, 384, replace=False))
    q = O.quantize(W[rows])
    want = O.matmul(q["packed"], q["norms"], 5120, X)
    assert rel_l2(Y1.cpu().numpy()[rows], want[0]) <= MATMUL_REL
    assert rel_l2(Y4.double().cpu().numpy()[:, rows], want) <= MATMUL_REL


@pytest.mark.parametrize("O,I,M", [(200, 704, 16), (384, 1024, 17), (256, 5120, 256), (130, 256, 48),
                                   (1024, 5120, 200), (128, 128, 300)])
def test_gemm_tensor_core_shapes(hl, cb, O, I, M):
    """M >= 5 runs on the tcgen05 path: partial 128-row tile, ragged K (704 =
    5.5 blocks), M not a multiple of 16, M = 256, and M > 256 (two token tiles)."""
    W, q = _layer((O, I), seed=O + I + M)
    p, n = oracle_to_dev(q)
    X = synth.activations(M, I, seed=M + 1)
    for odt in (torch.bfloat16, torch.float32):
        Y = hl.gemm(p, n, cb, X.cuda(), out_dtype=odt)
        torch.cuda.synchronize()
        want = O_.matmul(q["packed"], q["norms"], I, X)
        assert rel_l2(Y.double().cpu().numpy(), want) <= MATMUL_REL, odt
    assert hl.device_error() == 0


def test_gemm_full_27648x5120_m64_m256_sampled(hl, cb):
    """The 27648 x 5120 layer at M = 64 and 256 (tensor-core path), rows sampled
    for the oracle."""
    W = synth.student_t((27648, 5120), df4_seed=0)
    p, n = hl.quantize(W.cuda(), cb)
    rows = np.sort(np.random.default_rng(1).choice(27648, 256, replace=False))
    q = O_.quantize(W[rows])
    for M in (64, 256):
        X = synth.activations(M, 5120, seed=20 + M)
        Y = hl.gemm(p, n, cb, X.cuda(), out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        want = O_.matmul(q["packed"], q["norms"], 5120, X)
        assert rel_l2(Y.double().cpu().numpy()[:, rows], want) <= MATMUL_REL, M
    assert hl.device_error() == 0


def test_gemm_long_rows_m256(hl, cb):
    """in = 8192 at M = 256 (token tile narrowed to fit shared memory) and
    in = 8320 (longer than the tile-norm staging: CUDA-core path)."""
    for I in (8192, 8320):
        W, q = _layer((256, I), seed=I)
        p, n = oracle_to_dev(q)
        X = synth.activations(256 if I == 8192 else 20, I, seed=I + 1)
        Y = hl.gemm(p, n, cb, X.cuda(), out_dtype=torch.float32)
        torch.cuda.synchronize()
        want = O_.matmul(q["packed"], q["norms"], I, X)
        assert rel_l2(Y.double().cpu().numpy(), want) <= MATMUL_REL, I


def test_gemm_k_split_of_the_last_wave(hl, cb):
    """168 row tiles on a 148-SM part: the 20 tiles after the first wave run as
    two K halves each (fp32 partials, added in a fixed order by the half that
    finishes second).  Rows sampled in whole and split tiles against the
    oracle; repeated calls are bit-identical; the same call with the smallest
    accepted workspace (no split) agrees within the tolerance."""
    Od = 168 * 128
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rng = np.random.default_rng(5)
    for I, M in ((1024, 16), (704, 80)):
        W = synth.student_t_device((Od, I), seed=I + M)
        p, n = hl.quantize(W, cb)
        rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(sms * 128 - 8, sms * 128 + 8),
                                         np.arange(Od - 16, Od), rng.choice(Od, 64, replace=False)]))
        q = O_.quantize(W[torch.as_tensor(rows, device=W.device)].cpu())
        del W
        X = synth.activations(M, I, seed=M + 2)
        Xc = X.cuda()
        full = hl.workspace_bytes(hl.HLWQ_OP_GEMM, Od, I, M)
        small = 2 * M * 128 * ((I + 127) // 128) + 4 * M + 512
        if sms == 148:
            assert full > small  # the split's partials are part of the reported size
        ws = torch.empty(full, dtype=torch.uint8, device="cuda")
        Y1 = hl.gemm(p, n, cb, Xc, out_dtype=torch.float32, workspace=ws)
        Y2 = hl.gemm(p, n, cb, Xc, out_dtype=torch.float32, workspace=ws)
        Y3 = hl.gemm(p, n, cb, Xc, out_dtype=torch.float32,
                     workspace=torch.empty(small, dtype=torch.uint8, device="cuda"))
        torch.cuda.synchronize()
        assert torch.equal(Y1, Y2)
        want = O_.matmul(q["packed"], q["norms"], I, X)
        for Y in (Y1, Y3):
            assert rel_l2(Y.double().cpu().numpy()[:, rows], want) <= MATMUL_REL, (I, M)
        assert (Y1 - Y3).abs().max().item() <= 1e-3 * Y3.abs().max().item()
    assert hl.device_error() == 0
