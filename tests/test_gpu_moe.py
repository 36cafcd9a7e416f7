"""GPU parity: routed MoE layer (top-k + softmax, SiLU-gated experts, shared
expert) against the oracle's fp64 forward pass."""
import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth
from gpu_helpers import MATMUL_REL, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hl():
    from dequant_matmul_b200 import hlwq
    return hlwq


@pytest.fixture(scope="module")
def cb(hl):
    return hl.codebook("cuda")


def expert_weights(E, H, F, seed):
    gu = [synth.student_t((2 * F, H), df4_seed=seed + 2 * e) for e in range(E)]
    dn = [synth.student_t((H, F), df4_seed=seed + 2 * e + 1) for e in range(E)]
    return gu, dn


def run_case(hl, cb, E, H, F, T, topk, shared, seed, odt=torch.float32, used_only=False, flags=0, logits=None):
    """Oracle-quantized experts on both sides (only the experts the oracle's
    router picks are encoded when used_only; the others stay zero on the GPU)."""
    if logits is None:
        logits = synth.router_logits(T, E, seed=seed)
    X = synth.activations(T, H, seed=seed + 1)
    ids_ref, _ = O.router_topk(logits, topk)
    need = set(ids_ref.reshape(-1).tolist()) if used_only else set(range(E))
    nbh, nbf = O.n_blocks(H), O.n_blocks(F)
    gu_p = np.zeros((E, 2 * F, nbh, 80), np.uint8)
    gu_n = np.zeros((E, 2 * F, nbh), np.uint16)
    dn_p = np.zeros((E, H, nbf, 80), np.uint8)
    dn_n = np.zeros((E, H, nbf), np.uint16)
    gu_o, dn_o = [None] * E, [None] * E
    for e in sorted(need):
        qg = O.quantize(synth.student_t((2 * F, H), df4_seed=seed + 10 + 2 * e))
        qd = O.quantize(synth.student_t((H, F), df4_seed=seed + 11 + 2 * e))
        gu_p[e], gu_n[e] = qg["packed"], qg["norms"].view(np.uint16)
        dn_p[e], dn_n[e] = qd["packed"], qd["norms"].view(np.uint16)
        gu_o[e] = (qg["packed"], qg["norms"])
        dn_o[e] = (qd["packed"], qd["norms"])
    sh = sh_o = None
    sg_o = sd_o = None
    if shared:
        qg = O.quantize(synth.student_t((2 * F, H), df4_seed=seed + 7))
        qd = O.quantize(synth.student_t((H, F), df4_seed=seed + 8))
        sg_o, sd_o = (qg["packed"], qg["norms"]), (qd["packed"], qd["norms"])
        sh = ((torch.from_numpy(qg["packed"]).cuda(), torch.from_numpy(qg["norms"].view(np.uint16)).cuda()),
              (torch.from_numpy(qd["packed"]).cuda(), torch.from_numpy(qd["norms"].view(np.uint16)).cuda()))
    gu = (torch.from_numpy(gu_p).cuda(), torch.from_numpy(gu_n).cuda())
    dn = (torch.from_numpy(dn_p).cuda(), torch.from_numpy(dn_n).cuda())
    Y, ids, w = hl.moe_gemv(gu, dn, cb, logits.cuda(), X.cuda(), topk, shared=sh, out_dtype=odt, flags=flags)
    torch.cuda.synchronize()
    want, ids_o, w_o = O.moe_forward(gu_o, dn_o, H, F, topk, logits, X, sg_o, sd_o)
    assert np.array_equal(ids.cpu().numpy(), ids_o)
    assert np.allclose(w.cpu().numpy(), w_o, rtol=1e-5, atol=1e-7)
    err = rel_l2(Y.double().cpu().numpy(), want)
    assert err <= MATMUL_REL, err
    return err


@pytest.mark.parametrize("T,topk,shared", [(1, 8, True), (5, 2, False), (17, 8, True), (3, 1, False)])
def test_moe_small(hl, cb, T, topk, shared):
    run_case(hl, cb, E=16, H=256, F=128, T=T, topk=topk, shared=shared, seed=100 + T)


# ----------------------------------------------------------------------------
# The grouped path (tensor cores, each active expert read once for all its
# tokens): selected with HLWQ_FLAG_MOE_GROUPED, and taken by default once
# 4 T topk >= 3 E or when the fused path's shared memory does not fit.
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T,topk,shared", [(1, 8, True), (5, 2, False), (17, 8, True), (64, 8, True)])
def test_moe_grouped_path(hl, cb, T, topk, shared):
    run_case(hl, cb, E=16, H=256, F=128, T=T, topk=topk, shared=shared, seed=600 + T, flags=hl.HLWQ_FLAG_MOE_GROUPED)


def test_moe_grouped_path_ragged_and_bf16(hl, cb):
    run_case(hl, cb, E=8, H=320, F=176, T=6, topk=3, shared=True, seed=607, flags=hl.HLWQ_FLAG_MOE_GROUPED)
    run_case(hl, cb, E=8, H=256, F=128, T=4, topk=2, shared=False, seed=608, odt=torch.bfloat16,
             flags=hl.HLWQ_FLAG_MOE_GROUPED)


def test_moe_grouped_path_full_shapes_t1(hl, cb):
    run_case(hl, cb, E=256, H=2048, F=512, T=1, topk=8, shared=True, seed=610, used_only=True,
             flags=hl.HLWQ_FLAG_MOE_GROUPED)
    run_case(hl, cb, E=128, H=2816, F=704, T=1, topk=8, shared=False, seed=611, used_only=True,
             flags=hl.HLWQ_FLAG_MOE_GROUPED)


def test_moe_many_tokens_default_falls_back_to_grouped(hl, cb):
    """T = 400 tokens x (8 + 1) slots: the fused path's per-pair partial sums
    no longer fit in shared memory, so the default call runs the grouped path;
    its result must equal the one the flag selects, and the oracle's."""
    err = run_case(hl, cb, E=32, H=256, F=128, T=400, topk=8, shared=True, seed=612)
    err_g = run_case(hl, cb, E=32, H=256, F=128, T=400, topk=8, shared=True, seed=612,
                     flags=hl.HLWQ_FLAG_MOE_GROUPED)
    assert err == err_g   # the same kernels ran


def test_moe_grouped_path_one_expert_set_for_every_token(hl, cb):
    """Every token routes to the same top-3 experts (one logit row repeated):
    those experts get T = 300 assignments each, more than one 256-token tile,
    and the other 13 experts none."""
    row = synth.router_logits(1, 16, seed=613)
    logits = row.repeat(300, 1)
    run_case(hl, cb, E=16, H=256, F=128, T=300, topk=3, shared=True, seed=613, logits=logits,
             flags=hl.HLWQ_FLAG_MOE_GROUPED)


def test_moe_grouped_path_rows_past_8192(hl, cb):
    """H = 8320 (65 blocks): the grouped GEMMs stage tile norms of more than 64
    blocks (up to 128, H and F <= 16384)."""
    run_case(hl, cb, E=4, H=8320, F=256, T=3, topk=2, shared=True, seed=614, used_only=True,
             flags=hl.HLWQ_FLAG_MOE_GROUPED)


def test_moe_ex_rejects_unknown_flags(hl, cb):
    p = torch.zeros(16, dtype=torch.uint8, device="cuda")
    args = [hl._ptr(p)] * 4 + [None] * 4 + [hl._ptr(cb), 2, 128, 128, 1, 1, hl._ptr(p), hl._ptr(p), hl._ptr(p),
                                             hl.HLWQ_F32, None, None, hl._ptr(p), 1 << 20]
    assert hl.lib.hlwq_moe_gemv_ex(*args, 4, None) == hl.HLWQ_EINVAL


def test_moe_ragged_intermediate(hl, cb):
    """F = 176 (1.375 blocks) and H = 320 (2.5 blocks): zero-padded tails on both matrices."""
    run_case(hl, cb, E=8, H=320, F=176, T=6, topk=3, shared=True, seed=7)


def test_moe_bf16_out(hl, cb):
    run_case(hl, cb, E=8, H=256, F=128, T=4, topk=2, shared=False, seed=8, odt=torch.bfloat16)


def test_moe_256_experts_full_shape_t1(hl, cb):
    """256 experts + shared, hidden 2048, intermediate 512, T = 1 (9 experts used)."""
    run_case(hl, cb, E=256, H=2048, F=512, T=1, topk=8, shared=True, seed=300, used_only=True)


def test_moe_128_experts_ragged_full_shape_t1(hl, cb):
    """128 experts, hidden 2816, intermediate 704 (tail block zero-padded), T = 1."""
    run_case(hl, cb, E=128, H=2816, F=704, T=1, topk=8, shared=False, seed=400, used_only=True)


def test_moe_full_t64_sampled_tokens(hl, cb):
    """Full 257-expert layer at T = 64 quantized on the GPU; the oracle encodes
    and evaluates the experts of two sampled tokens itself."""
    E, H, F, T, k = 256, 2048, 512, 64, 8
    seed = 500
    logits = synth.router_logits(T, E, seed=seed)
    X = synth.activations(T, H, seed=seed + 1)
    gu_w = torch.empty(E, 2 * F, H, dtype=torch.bfloat16, device="cuda")
    dn_w = torch.empty(E, H, F, dtype=torch.bfloat16, device="cuda")
    for e in range(E):
        gu_w[e] = synth.student_t((2 * F, H), df4_seed=seed + 10 + 2 * e).cuda()
        dn_w[e] = synth.student_t((H, F), df4_seed=seed + 11 + 2 * e).cuda()
    gu = hl.quantize(gu_w, cb)
    dn = hl.quantize(dn_w, cb)
    sg_w = synth.student_t((2 * F, H), df4_seed=seed + 7)
    sd_w = synth.student_t((H, F), df4_seed=seed + 8)
    sh = (hl.quantize(sg_w.cuda(), cb), hl.quantize(sd_w.cuda(), cb))
    Y, ids, w = hl.moe_gemv(gu, dn, cb, logits.cuda(), X.cuda(), k, shared=sh)
    torch.cuda.synchronize()
    ids_o, w_o = O.router_topk(logits, k)
    assert np.array_equal(ids.cpu().numpy(), ids_o)
    for t in (0, 41):
        sel = ids_o[t]
        gu_o = {int(e): (lambda q: (q["packed"], q["norms"]))(O.quantize(gu_w[int(e)].cpu())) for e in sel}
        dn_o = {int(e): (lambda q: (q["packed"], q["norms"]))(O.quantize(dn_w[int(e)].cpu())) for e in sel}
        qsg, qsd = O.quantize(sg_w), O.quantize(sd_w)
        want, _, _ = O.moe_forward(gu_o, dn_o, H, F, k, logits[t:t + 1], X[t:t + 1],
                                   (qsg["packed"], qsg["norms"]), (qsd["packed"], qsd["norms"]))
        assert rel_l2(Y[t].cpu().numpy(), want[0]) <= MATMUL_REL


def test_moe_128_experts_full_t16_sampled_tokens(hl, cb):
    """The 128-expert layer (hidden 2816, intermediate 704, no shared expert)
    at T = 16: the gate_up kernel's partial sums need two waves of CTAs and the
    down kernel takes the 128 pairs in groups.  The oracle encodes and
    evaluates the experts of three sampled tokens itself."""
    E, H, F, T, k = 128, 2816, 704, 16, 8
    seed = 600
    logits = synth.router_logits(T, E, seed=seed)
    X = synth.activations(T, H, seed=seed + 1)
    gu_w = torch.empty(E, 2 * F, H, dtype=torch.bfloat16, device="cuda")
    dn_w = torch.empty(E, H, F, dtype=torch.bfloat16, device="cuda")
    for e in range(E):
        gu_w[e] = synth.student_t((2 * F, H), df4_seed=seed + 10 + 2 * e).cuda()
        dn_w[e] = synth.student_t((H, F), df4_seed=seed + 11 + 2 * e).cuda()
    gu = hl.quantize(gu_w, cb)
    dn = hl.quantize(dn_w, cb)
    for odt in (torch.float32, torch.bfloat16):
        Y, ids, w = hl.moe_gemv(gu, dn, cb, logits.cuda(), X.cuda(), k, out_dtype=odt)
        torch.cuda.synchronize()
        ids_o, w_o = O.router_topk(logits, k)
        assert np.array_equal(ids.cpu().numpy(), ids_o)
        assert np.allclose(w.cpu().numpy(), w_o, rtol=1e-5, atol=1e-7)
        for t in (0, 7, 15):
            sel = ids_o[t]
            gu_o = {int(e): (lambda q: (q["packed"], q["norms"]))(O.quantize(gu_w[int(e)].cpu())) for e in sel}
            dn_o = {int(e): (lambda q: (q["packed"], q["norms"]))(O.quantize(dn_w[int(e)].cpu())) for e in sel}
            want, _, _ = O.moe_forward(gu_o, dn_o, H, F, k, logits[t:t + 1], X[t:t + 1], None, None)
            assert rel_l2(Y[t].double().cpu().numpy(), want[0]) <= MATMUL_REL, (odt, t)
