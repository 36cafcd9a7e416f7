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


# --------------------------------------------------------------------------
# The routing-weighted combine for k >= 2 ("Qwen3.6-35B-A3B -- HLWQ Q5",
# Architecture table: 8 routed + 1 shared expert per token).  The weights are
# fixed in closed form by the logits, and each expert's MLP is rebuilt here
# from the dequantized matrices with SiLU written out, so a combine that drops
# a weight, takes it from the wrong slot or normalises over all E fails.
# --------------------------------------------------------------------------

H_C, F_C, E_C = 128, 128, 5


@pytest.fixture(scope="module")
def experts():
    mk = lambda shape, s: (lambda q: (q["packed"], q["norms"]))(O.quantize(synth.student_t(shape, df4_seed=s)))
    gu = [mk((2 * F_C, H_C), 60 + e) for e in range(E_C)]
    dn = [mk((H_C, F_C), 70 + e) for e in range(E_C)]
    x = synth.activations(1, H_C, seed=9)
    return gu, dn, x


def _mlp(gu, dn, xt):
    wg = O.dequantize(gu[0], gu[1], H_C)
    wd = O.dequantize(dn[0], dn[1], F_C)
    g, u = wg[:F_C] @ xt, wg[F_C:] @ xt
    return wd @ ((g / (1.0 + np.exp(-g))) * u)


def _logits(sel, offsets):
    """Experts `sel` get logits 1.5 - offsets (the others -4): softmax over the
    selected ones is proportional to exp(-offsets)."""
    lg = np.full((1, E_C), -4.0)
    for e, d in zip(sel, offsets):
        lg[0, e] = 1.5 - d
    return lg


def _combine_matches_closed_form(forward, experts) -> bool:
    gu, dn, x = experts
    xt = x[0].double().numpy()
    cases = [  # (selected experts in selection order, logit offsets, closed-form weights)
        ((3, 1), (0.0, np.log(3.0)), (3 / 4, 1 / 4)),
        ((0, 4, 2), (0.0, np.log(2.0), np.log(4.0)), (4 / 7, 2 / 7, 1 / 7)),
    ]
    for sel, offs, p in cases:
        out = forward(gu, dn, H_C, F_C, len(sel), _logits(sel, offs), x)[0][0]
        want = sum(pi * _mlp(gu[e], dn[e], xt) for e, pi in zip(sel, p))
        if not np.allclose(out, want, rtol=1e-12, atol=1e-14):
            return False
    return True


def test_moe_combine_weights_in_closed_form(experts):
    """k = 2 with logits (a, a - ln 3) gives p = (3/4, 1/4); k = 3 with
    (a, a - ln 2, a - ln 4) gives (4/7, 2/7, 1/7)."""
    assert _combine_matches_closed_form(O.moe_forward, experts)


def test_moe_combine_is_linear_in_the_weights(experts):
    """Moving one selected logit changes the output by exactly
    delta_p * (MLP_first - MLP_second) for k = 2."""
    gu, dn, x = experts
    xt = x[0].double().numpy()
    m1, m2 = _mlp(gu[1], dn[1], xt), _mlp(gu[3], dn[3], xt)
    a, _, wa = O.moe_forward(gu, dn, H_C, F_C, 2, _logits((1, 3), (0.0, 1.0)), x)
    b, _, wb = O.moe_forward(gu, dn, H_C, F_C, 2, _logits((1, 3), (0.0, 0.25)), x)
    pa, pb = 1 / (1 + np.exp(-1.0)), 1 / (1 + np.exp(-0.25))
    assert wa[0, 0] == pytest.approx(pa, rel=1e-15) and wb[0, 0] == pytest.approx(pb, rel=1e-15)
    assert np.allclose(b[0] - a[0], (pb - pa) * (m1 - m2), rtol=1e-11, atol=1e-14)


def test_moe_combine_planted_mistakes_fail_the_pin(experts, monkeypatch):
    """A router whose weights are dropped (all 1), normalised over all E, or
    handed to the wrong slots; and a combine that takes every slot's weight
    from slot 0: each fails the closed-form pin."""
    from oracle import hlwq_oracle as HO
    good = HO.router_topk

    def ones(lg, k):
        ids, w = good(lg, k)
        return ids, np.ones_like(w)

    def over_all(lg, k):
        ids, _ = good(lg, k)
        z = np.exp(lg - lg.max(axis=1, keepdims=True))
        z /= z.sum(axis=1, keepdims=True)
        return ids, np.take_along_axis(z, ids, axis=1)

    def reversed_slots(lg, k):
        ids, w = good(lg, k)
        return ids, w[:, ::-1].copy()

    for bad in (ones, over_all, reversed_slots):
        monkeypatch.setattr(HO, "router_topk", bad)
        assert not _combine_matches_closed_form(O.moe_forward, experts), bad.__name__
    monkeypatch.setattr(HO, "router_topk", good)
    assert _combine_matches_closed_form(O.moe_forward, experts)

    def slot0_weight(gu, dn, hidden, inter, k, logits, X):
        ids, w = O.router_topk(logits, k)
        xt = X[0].double().numpy()
        out = sum(w[0, 0] * _mlp(gu[int(e)], dn[int(e)], xt) for e in ids[0])
        return out[None], ids, w
    assert not _combine_matches_closed_form(slot0_weight, experts)
