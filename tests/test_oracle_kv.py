"""Pins of the Q3 KV-cache oracle (oracle/kv_oracle.py) to facts that do not
come from the oracle itself: the Hadamard identity, a hand-computed 3-bit
pack, brute-force nearest centroids, norms and rotation identities, the
Lloyd-Max distortion D_8 and the rotated-domain form of the scores."""
import numpy as np

import oracle as O


def test_h256_is_a_scaled_orthogonal_symmetric_matrix():
    H = O.sylvester_hadamard(256).astype(np.int64)
    assert np.array_equal(H, H.T)
    assert np.array_equal(H @ H.T, 256 * np.eye(256, dtype=np.int64))
    assert H[1, 1] == -1 and H[3, 5] == -1 and H[3, 4] == 1   # (-1)^popcount(i & j)


def test_three_bit_pack_hand_computed():
    """Reading K4: codes 0..7 of one group -> v = sum j * 8^j = 0xFAC688 ->
    little-endian bytes 0x88, 0xC6, 0xFA; 96 bytes per vector."""
    codes = np.tile(np.arange(8, dtype=np.uint8), 32)
    b = O.pack_codes(codes, bits=3)
    assert b.shape == (96,)
    assert list(b[:3]) == [0x88, 0xC6, 0xFA]
    assert np.array_equal(O.unpack_codes(b, bits=3), codes)
    rnd = np.random.default_rng(0).integers(0, 8, size=(50, 256)).astype(np.uint8)
    assert np.array_equal(O.unpack_codes(O.pack_codes(rnd, bits=3), bits=3), rnd)


def test_rotated_vectors_have_norm_16_and_codes_are_nearest():
    """||y||^2 = 256 for a non-zero vector (H H^T = 256 I); every code is the
    brute-force nearest of the 8 centroids (threshold rule on the midpoints,
    ties low), also for values 1e-12 around each midpoint (closer than that the
    fp64 distances themselves round to a tie)."""
    g = np.random.default_rng(1)
    X = (g.standard_normal((40, 256)) * 0.7).astype(np.float32)
    r = O.kv_quantize(X)
    assert np.allclose((r["y"] ** 2).sum(1), 256.0, rtol=0, atol=1e-9)
    c32, mid, _ = O.codebook_fp32(8)
    c = c32.astype(np.float64)
    assert np.array_equal(r["codes"], np.abs(r["y"][..., None] - c).argmin(-1))
    eps = 1e-12 * np.maximum(1.0, np.abs(mid))
    probe = np.concatenate([mid, mid - eps, mid + eps])
    rule = (probe[:, None] > mid[None, :]).sum(1)
    assert np.array_equal(O.nearest_centroid(probe, c32), rule)


def test_zero_vector_and_scale_invariance():
    """Reading K3: a zero vector has y = 0, equidistant from c[3] and c[4]:
    code 3 everywhere, norm 0, decodes to zeros.  Scaling x by 2^k leaves the
    codes unchanged and scales the stored norm exactly."""
    X = np.zeros((2, 256), np.float32)
    X[1] = np.linspace(-1, 1, 256, dtype=np.float32)
    r = O.kv_quantize(X)
    assert np.all(r["codes"][0] == 3) and r["norms"][0] == 0
    assert np.all(O.kv_dequantize(r["packed"], r["norms"])[0] == 0.0)
    r8 = O.kv_quantize(X * 8.0)
    assert np.array_equal(r8["codes"], r["codes"])
    assert np.array_equal(r8["norms"].astype(np.float64), 8.0 * r["norms"].astype(np.float64))


def test_distortion_matches_the_lloyd_max_value():
    """On Gaussian vectors the rotated entries are (nearly) N(0,1), so the mean
    squared error of the code values equals D_8 = 0.03455 within 3 standard
    errors, and the decoded vectors keep cosine ~ sqrt(1 - D_8)."""
    g = np.random.default_rng(2)
    X = g.standard_normal((400, 256)).astype(np.float32)
    r = O.kv_quantize(X)
    c32, _, _ = O.codebook_fp32(8)
    err = (r["y"] - c32.astype(np.float64)[r["codes"]]) ** 2
    D8 = O.lloyd_max_gaussian(8)["mse"]
    assert abs(D8 - 0.03455) < 5e-5
    se = err.std() / np.sqrt(err.size)
    assert abs(err.mean() - D8) < 3 * se + 1e-4
    xh = O.kv_dequantize(r["packed"], r["norms"])
    cos = (X * xh).sum(1) / np.linalg.norm(X, axis=1) / np.linalg.norm(xh, axis=1)
    assert abs(cos.mean() - np.sqrt(1 - D8)) < 2e-3


def test_scores_in_the_rotated_domain():
    """q . x_hat = (n16 / 256) sum_j c[k_j] (q H)_j: the dot with the decoded
    vectors equals the rotated-domain form (to rounding)."""
    g = np.random.default_rng(3)
    K = g.standard_normal((30, 256)).astype(np.float32)
    Q = g.standard_normal((4, 256)).astype(np.float32)
    r = O.kv_quantize(K)
    s = O.kv_scores(Q, r["packed"], r["norms"])
    c32, _, _ = O.codebook_fp32(8)
    H = O.sylvester_hadamard(256).astype(np.float64)
    qt = Q.astype(np.float64) @ H
    alt = (qt @ c32.astype(np.float64)[r["codes"]].T) * (r["norms"].astype(np.float64) / 256.0)[None, :]
    assert np.allclose(s, alt, rtol=1e-12, atol=1e-12)
    assert s.shape == (4, 30)


# --------------------------------------------------------------------------
# The 128-token residual window (reading K5; "Qwopus3.6-27B-v2 . HLWQ Q5",
# Methodology notes, KV-cache bullet).
# --------------------------------------------------------------------------

def _tokens(n, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal((n, 256)).astype(np.float32)


def _append_all(tokens, chunks, capacity=O.RESIDUAL_TOKENS, append=None):
    append = append or O.kv_window_append
    p = np.zeros((0, 96), np.uint8)
    n = np.zeros((0,), np.float16)
    w = np.zeros((0, 256))
    i = 0
    for c in chunks:
        p, n, w = append(p, n, w, tokens[i:i + c], capacity)
        i += c
    return p, n, w


def _window_is_the_recent_tokens(append) -> bool:
    """After appending N tokens in any batching, the encoded part is
    kv_quantize of tokens [0, N - 128) and the window holds tokens
    [N - 128, N) exactly, oldest first."""
    X = _tokens(400, 5)
    for chunks in ([400], [1] * 130 + [270], [5, 200, 1, 128, 66], [127, 1, 1, 271]):
        p, n, w = _append_all(X, chunks, append=append)
        want = O.kv_quantize(X[:400 - 128])
        if not (np.array_equal(p, want["packed"]) and np.array_equal(n.view(np.uint16), want["norms"].view(np.uint16))
                and np.array_equal(w, X[400 - 128:].astype(np.float64))):
            return False
    return True


def test_window_keeps_the_128_most_recent_tokens():
    assert O.RESIDUAL_TOKENS == 128
    assert _window_is_the_recent_tokens(O.kv_window_append)


def test_window_encodes_nothing_until_it_is_full():
    X = _tokens(128, 6)
    p, n, w = _append_all(X, [100, 28])
    assert p.shape == (0, 96) and n.shape == (0,)
    assert np.array_equal(w, X.astype(np.float64))
    p, n, w = _append_all(X[:1], [1], capacity=1)
    assert p.shape == (0, 96) and w.shape == (1, 256)


def test_window_scores_with_an_empty_window_are_the_encoded_scores():
    X = _tokens(300, 7)
    Q = _tokens(3, 8)
    r = O.kv_quantize(X)
    s = O.kv_scores_window(Q, r["packed"], r["norms"], np.zeros((0, 256)))
    assert np.array_equal(s, O.kv_scores(Q, r["packed"], r["norms"]))


def test_window_scores_of_exact_keys_equal_integer_dot_products():
    """With small-integer keys and queries every product and sum is an integer,
    computed here in Python integers: the window part is the exact dot."""
    g = np.random.default_rng(9)
    K = g.integers(-8, 9, size=(128, 256))
    Q = g.integers(-8, 9, size=(2, 256))
    s = O.kv_scores_window(Q.astype(np.float32), np.zeros((0, 96), np.uint8), np.zeros(0, np.float16),
                           K.astype(np.float32))
    want = [[sum(int(a) * int(b) for a, b in zip(q, k)) for k in K] for q in Q]
    assert np.array_equal(s, np.array(want, dtype=np.float64))


def test_window_scores_cover_every_cached_token_in_order():
    X = _tokens(200, 10)
    Q = _tokens(2, 11)
    p, n, w = _append_all(X, [3, 197])
    s = O.kv_scores_window(Q, p, n, w)
    assert s.shape == (2, 200)
    assert np.array_equal(s[:, :72], O.kv_scores(Q, p, n))
    assert np.allclose(s[:, 72:], Q.astype(np.float64) @ X[72:].astype(np.float64).T, rtol=0, atol=1e-9)


def test_window_planted_mistakes_fail_the_pin():
    """Evicting the newest tokens instead of the oldest, or keeping one token
    too many, fails the recent-tokens pin."""
    def newest_first(p, n, w, x, cap):
        t = np.concatenate([np.asarray(w, np.float64).reshape(-1, 256), np.asarray(x, np.float64).reshape(-1, 256)])
        leave = max(0, t.shape[0] - cap)
        if leave:
            q = O.kv_quantize(t[t.shape[0] - leave:])
            p, n = np.concatenate([p, q["packed"]]), np.concatenate([n, q["norms"]])
        return p, n, t[:t.shape[0] - leave]

    def one_too_many(p, n, w, x, cap):
        return O.kv_window_append(p, n, w, x, cap + 1)

    assert not _window_is_the_recent_tokens(newest_first)
    assert not _window_is_the_recent_tokens(one_too_many)
