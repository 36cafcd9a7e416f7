"""Pins of the TQ3 oracle (oracle/tq3_oracle.py) to facts that do not come from
the oracle itself: scipy's Sylvester Hadamard matrix, the roles of the two sign
vectors (invariances of the method), a hand-computed 3-bit pack, brute-force
nearest centroids, the shape-gain identity ||w_hat|| = ||w||, the moments of
the sphere marginal behind the error, and planted mistakes that each fail a pin."""
import numpy as np
from scipy.linalg import hadamard

import oracle as O
from oracle import tq3_oracle as T
from dequant_matmul_b200 import synth

S = synth.sign_vectors(42).numpy()
S1, S2 = S[0].astype(np.int64), S[1].astype(np.int64)


def _rotation_matches_scipy(rotate) -> bool:
    g = np.random.default_rng(0).standard_normal((5, 128))
    Hs = hadamard(128).astype(np.float64)        # Sylvester construction, natural order
    want = np.stack([S2 * (Hs @ (S1 * v)) for v in g])
    return np.allclose(rotate(g, S1, S2), want, rtol=0, atol=1e-12)


def _norm_is_kept(quantize, dequantize) -> bool:
    W = synth.student_t((40, 512), df4_seed=8)
    q = quantize(W, S1, S2)
    wh = dequantize(q["packed"], q["norms"], 512, S1, S2).reshape(40, 4, 128)
    w = W.double().numpy().reshape(40, 4, 128)
    return np.allclose(np.linalg.norm(wh, axis=-1), np.linalg.norm(w, axis=-1), rtol=2e-7, atol=0)


def test_rotation_is_scipy_hadamard_with_the_signs_and_inverts():
    assert _rotation_matches_scipy(T.tq3_rotate)
    g = np.random.default_rng(1).standard_normal((7, 128))
    assert np.allclose(T.tq3_unrotate(T.tq3_rotate(g, S1, S2), S1, S2), g, rtol=0, atol=1e-12)
    # an orthogonal map up to sqrt(128): norms scale by sqrt(128)
    assert np.allclose(np.linalg.norm(T.tq3_rotate(g, S1, S2), axis=1), np.sqrt(128) * np.linalg.norm(g, axis=1))


def test_sign_vector_roles():
    """Reading T1: s1 acts on the weights before the FWHT, s2 on the rotated
    values.  Flipping s1_i and negating w_i changes nothing; flipping s2_j
    mirrors code j (c[7-k] = -c[k]) and leaves the others and gamma (to an ulp)."""
    W = synth.student_t((30, 256), df4_seed=9).double().numpy()
    q = T.tq3_quantize(W, S1, S2)
    s1f = S1.copy()
    s1f[17] = -s1f[17]
    W2 = W.copy()
    W2[:, 17] = -W2[:, 17]
    W2[:, 128 + 17] = -W2[:, 128 + 17]
    q2 = T.tq3_quantize(W2, s1f, S2)
    assert np.array_equal(q2["codes"], q["codes"]) and np.array_equal(q2["norms"], q["norms"])
    s2f = S2.copy()
    s2f[40] = -s2f[40]
    q3 = T.tq3_quantize(W, S1, s2f)
    want = q["codes"].copy()
    want[..., 40] = 7 - want[..., 40]
    assert np.array_equal(q3["codes"], want)
    assert np.all(np.abs(q3["norms"] - q["norms"]) <= np.spacing(q["norms"]))


def test_three_bit_pack_hand_computed():
    """Reading T5: codes 0..7 -> 0x88, 0xC6, 0xFA (v = sum j 8^j = 0xFAC688); 48 bytes per group."""
    codes = np.tile(np.arange(8, dtype=np.uint8), 16)
    b = O.pack_codes(codes, bits=3)
    assert b.shape == (48,) and list(b[:3]) == [0x88, 0xC6, 0xFA] and list(b[3:6]) == [0x88, 0xC6, 0xFA]


def test_codes_are_nearest_and_gamma_is_norm_over_reconstruction_norm():
    W = synth.student_t((50, 384), df4_seed=10)
    q = T.tq3_quantize(W, S1, S2)
    c32, mid, _ = O.codebook_fp32(8)
    c = c32.astype(np.float64)
    assert np.array_equal(q["codes"], np.abs(q["y"][..., None] - c).argmin(-1))
    # y has unit variance per entry: ||y||^2 = 128
    assert np.allclose((q["y"] ** 2).sum(-1), 128.0, rtol=0, atol=1e-9)
    n = np.linalg.norm(W.double().numpy().reshape(50, 3, 128), axis=-1)
    r = np.linalg.norm(c[q["codes"]], axis=-1) / np.sqrt(128.0)
    assert np.all(np.abs(q["norms"] - (n / r)) <= np.spacing(q["norms"]))


def test_shape_gain_keeps_the_group_norm():
    """Reading T4: ||w_hat|| = ||w|| per group (float32 rounding of gamma)."""
    assert _norm_is_kept(T.tq3_quantize, T.tq3_dequantize)


def _sphere_moments(n=128):
    """D = E[(y - Q(y))^2], A = E[y Q(y)], B = E[Q(y)^2] for y = sqrt(n) u_1, u
    uniform on the unit sphere of R^n (density proportional to
    (1 - y^2/n)^((n-3)/2)), by numerical integration over the decision cells."""
    from scipy import integrate, special
    c32, mid, _ = O.codebook_fp32(8)
    c = c32.astype(np.float64)
    logc = special.gammaln(n / 2) - special.gammaln((n - 1) / 2) - 0.5 * np.log(np.pi * n)
    f = lambda y: np.exp(logc + (n - 3) / 2 * np.log1p(-y * y / n))  # noqa: E731
    edges = np.concatenate([[-np.sqrt(n)], mid, [np.sqrt(n)]])
    out = []
    for g in (lambda y, k: (y - c[k]) ** 2, lambda y, k: y * c[k], lambda y, k: c[k] ** 2):
        out.append(sum(integrate.quad(lambda y: g(y, k) * f(y), edges[k], edges[k + 1], epsabs=1e-14,
                                      epsrel=1e-12)[0] for k in range(8)))
    return out


def test_error_and_cosine_match_the_sphere_marginal():
    """For iid Gaussian rows, g / ||g|| is uniform on the sphere and so is its
    rotation: each y_j has the sphere marginal.  The mean squared code error,
    the cosine sqrt-law A / sqrt(B) and the shape-gain error 2 - 2 A / sqrt(B)
    follow from its moments (the N(0,1) values D_8 = 0.03455 are the n -> inf
    limit).  The raw-norm reconstruction n * u_hat has the same error to ~1 %,
    so the shape-gain gain is small for a Lloyd-Max codebook."""
    D, A, B = _sphere_moments()
    assert 0.0335 < D < 0.0345 and abs(A - B) < 2e-3
    W = synth.activations(400, 1024, seed=3, dtype=__import__("torch").float32)
    q = T.tq3_quantize(W, S1, S2)
    c32, _, _ = O.codebook_fp32(8)
    e = ((q["y"] - c32.astype(np.float64)[q["codes"]]) ** 2).mean(-1).reshape(-1)
    assert abs(e.mean() - D) < 4 * e.std() / np.sqrt(e.size)
    w = W.double().numpy().reshape(400, 8, 128)
    wh = T.tq3_dequantize(q["packed"], q["norms"], 1024, S1, S2).reshape(400, 8, 128)
    n = np.linalg.norm(w, axis=-1)
    cos = ((wh * w).sum(-1) / (np.linalg.norm(wh, axis=-1) * n)).mean()
    assert abs(cos - A / np.sqrt(B)) < 1e-3
    err_gain = (np.linalg.norm(wh - w, axis=-1) ** 2 / n ** 2).mean()
    assert abs(err_gain / (2 - 2 * A / np.sqrt(B)) - 1) < 0.05
    assert abs(err_gain / e.mean() - 1) < 0.03


def test_zero_groups_and_ragged_tail():
    """A zero group: y = 0, code 3 everywhere, gamma 0, decoded zeros.  A row of
    300 values is padded with zeros to 384 (reading T6)."""
    W = synth.student_t((3, 300), df4_seed=13).double().numpy()
    W[1] = 0.0
    q = T.tq3_quantize(W, S1, S2)
    assert np.all(q["codes"][1] == 3) and np.all(q["norms"][1] == 0)
    assert q["packed"].shape == (3, 3, 48)
    wh = T.tq3_dequantize(q["packed"], q["norms"], 300, S1, S2)
    assert wh.shape == (3, 300) and np.all(wh[1] == 0)
    qp = T.tq3_quantize(np.pad(W, ((0, 0), (0, 84))), S1, S2)
    assert np.array_equal(qp["packed"], q["packed"]) and np.array_equal(qp["norms"], q["norms"])


def test_matmul_in_the_rotated_domain():
    """x . w_hat = sum_b gamma_b / 128 * sum_j c[k_j] (s2 * H (s1 * x_b))_j, with
    scipy's Hadamard matrix."""
    W = synth.student_t((20, 256), df4_seed=14)
    X = synth.activations(3, 256, seed=15)
    q = T.tq3_quantize(W, S1, S2)
    Y = T.tq3_matmul(q["packed"], q["norms"], 256, S1, S2, X)
    Hs = hadamard(128).astype(np.float64)
    x = X.double().numpy().reshape(3, 2, 128)
    xt = np.einsum("ij,mbj->mbi", Hs, x * S1) * S2
    c32, _, _ = O.codebook_fp32(8)
    vals = c32.astype(np.float64)[q["codes"]]
    alt = np.einsum("mbj,obj,ob->mo", xt, vals, q["norms"].astype(np.float64)) / 128
    assert np.allclose(Y, alt, rtol=1e-12, atol=1e-12)


def test_planted_mistakes_fail_a_pin():
    """Sign vectors swapped, or applied on the wrong side of the FWHT; the raw
    norm stored instead of the shape-gain one."""
    assert not _rotation_matches_scipy(lambda g, a, b: T.tq3_rotate(g, b, a))
    assert not _rotation_matches_scipy(lambda g, a, b: (np.asarray(g) @ hadamard(128)) * a * b)

    def raw_norm(W, a, b):
        q = T.tq3_quantize(W, a, b)
        return dict(q, norms=q["n"].astype(np.float32))
    assert not _norm_is_kept(raw_norm, T.tq3_dequantize)
