"""Pins for the oracle's dequant-matmul and routed-MoE arithmetic."""
import numpy as np
import pytest
import torch

import oracle as O
from dequant_matmul_b200 import synth


@pytest.fixture(scope="module")
def layer():
    w = synth.student_t((48, 704), dtype=torch.bfloat16, df4_seed=8)
    q = O.quantize(w)
    return w, q


def test_rotated_domain_agrees(layer):
    """Dequantize-then-dot and rotate-the-activation-once are the same algebra
    (H symmetric, H H = 128 I); they must agree to fp64 rounding."""
    _, q = layer
    x = synth.activations(3, 704, seed=4)
    a = O.matmul(q["packed"], q["norms"], 704, x)
    b = O.matmul_rotated_domain(q["packed"], q["norms"], 704, x)
    assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


def test_one_hot_activation_reads_a_column(layer):
    _, q = layer
    w_hat = O.dequantize(q["packed"], q["norms"], 704)
    for i in (0, 127, 128, 703):
        x = np.zeros((1, 704))
        x[0, i] = 1.0
        assert np.array_equal(O.matmul(q["packed"], q["norms"], 704, x)[0], w_hat[:, i])


def test_rotate_activation_pads_with_zero():
    x = np.zeros((1, 704))
    x[0, 640] = 2.0          # first element of the half block
    xt = O.rotate_activation(x, 704)
    assert xt.shape == (1, 768)
    assert np.allclose(xt[0, 640:], 2.0) and not xt[0, :640].any()


def test_router_ties_and_softmax():
    lg = np.array([[0.5, 2.0, 2.0, -1.0, 2.0, 0.0]])
    ids, w = O.router_topk(lg, 3)
    assert list(ids[0]) == [1, 2, 4]
    assert np.allclose(w[0], 1 / 3)
    ids, w = O.router_topk(lg, 4)
    assert list(ids[0]) == [1, 2, 4, 0]
    e = np.exp([2.0, 2.0, 2.0, 0.5])
    assert np.allclose(w[0], e / e.sum(), rtol=1e-15)


def test_router_weights_sum_to_one():
    lg = synth.router_logits(16, 128, seed=3)
    ids, w = O.router_topk(lg, 8)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-15)
    assert all(len(set(r)) == 8 for r in ids)
    top = np.sort(lg.numpy(), axis=1)[:, ::-1][:, :8]
    assert np.array_equal(np.take_along_axis(lg.numpy(), ids, axis=1), top)


def test_silu_closed_form():
    z = np.array([0.0, 1.0, -1.0, 30.0])
    assert np.allclose(O.silu(z), [0.0, 1 / (1 + np.exp(-1)), -1 / (1 + np.e), 30.0])


def test_moe_topk1_one_hot_is_dense_mlp():
    """One expert with weight 1 (k = 1): out = Wd (SiLU(Wg x) * (Wu x))."""
    H, F, E = 256, 128, 4
    gus = [O.quantize(synth.student_t((2 * F, H), df4_seed=10 + e)) for e in range(E)]
    dns = [O.quantize(synth.student_t((H, F), df4_seed=20 + e)) for e in range(E)]
    gu = [(q["packed"], q["norms"]) for q in gus]
    dn = [(q["packed"], q["norms"]) for q in dns]
    x = synth.activations(2, H, seed=5)
    logits = np.full((2, E), -5.0)
    logits[0, 2] = 3.0
    logits[1, 0] = 3.0
    out, ids, w = O.moe_forward(gu, dn, H, F, 1, logits, x)
    for t, e in ((0, 2), (1, 0)):
        wg = O.dequantize(*gu[e], H)
        wd = O.dequantize(*dn[e], F)
        xt = x[t].double().numpy()
        h = O.silu(wg[:F] @ xt) * (wg[F:] @ xt)
        assert np.allclose(out[t], wd @ h, rtol=1e-13, atol=1e-15)
        assert w[t, 0] == 1.0


def test_moe_shared_expert_adds_with_weight_one():
    H, F, E = 128, 128, 3
    mk = lambda shape, s: (lambda q: (q["packed"], q["norms"]))(O.quantize(synth.student_t(shape, df4_seed=s)))
    gu = [mk((2 * F, H), 30 + e) for e in range(E)]
    dn = [mk((H, F), 40 + e) for e in range(E)]
    sg, sd = mk((2 * F, H), 50), mk((H, F), 51)
    x = synth.activations(1, H, seed=6)
    lg = synth.router_logits(1, E, seed=7)
    a, _, _ = O.moe_forward(gu, dn, H, F, 2, lg, x)
    b, _, _ = O.moe_forward(gu, dn, H, F, 2, lg, x, sg, sd)
    shared_only, _, _ = O.moe_forward([sg], [sd], H, F, 1, np.zeros((1, 1)), x)
    assert np.allclose(b - a, shared_only, rtol=1e-12, atol=1e-15)
