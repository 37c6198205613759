"""Pins for the oracle's decoupled RoPE: closed-form 2x2 rotations, the
textbook frequency schedule, orthogonality and relative-position dependence
(the properties the pages rely on in '2. The RoPE Non-Commutativity
Challenge')."""
import numpy as np

from oracle import mla_oracle as O


def rotation_closed_form(x, p, base):
    """Pair (i, i + d/2) rotated by angle p * base**(-2i/d), written out."""
    d = len(x)
    out = np.empty(d)
    for i in range(d // 2):
        th = p * base ** (-2.0 * i / d)
        a, b = x[i], x[i + d // 2]
        out[i] = np.cos(th) * a - np.sin(th) * b
        out[i + d // 2] = np.sin(th) * a + np.cos(th) * b
    return out


def test_rope_matches_closed_form_rotations():
    rng = np.random.default_rng(0)
    for d, base in [(2, 10000.0), (4, 10000.0), (16, 10000.0), (64, 10000.0), (64, 500.0)]:
        for p in [0, 1, 7, 4096, 131071]:
            x = rng.standard_normal(d)
            # the two spell the angle differently in fp64: allow a few ulps of the angle
            np.testing.assert_allclose(O.apply_rope(x, p, base), rotation_closed_form(x, p, base),
                                       rtol=0, atol=1e-13 + 4e-16 * p * np.abs(x).max())


def test_rope_d2_is_plane_rotation():
    # d=2: the only frequency is 1, so position p rotates by p radians
    np.testing.assert_allclose(O.apply_rope(np.array([1.0, 0.0]), 3), [np.cos(3), np.sin(3)], atol=1e-15)


def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((10, 64))
    np.testing.assert_array_equal(O.apply_rope(x, 0), x)
    pos = rng.integers(0, 200000, 10)
    y = O.apply_rope(x, pos)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n, delta in [(10, 3, 100), (5000, 4999, 77), (131000, 0, 33)]:
        a = O.apply_rope(q, m) @ O.apply_rope(k, n)
        b = O.apply_rope(q, m + delta) @ O.apply_rope(k, n + delta)
        assert abs(a - b) < 1e-9 * (abs(a) + 1)


def test_rotation_does_not_commute_with_up_projection():
    # R_s W != W R_s for a generic W: the reason RoPE is kept off the latent
    rng = np.random.default_rng(3)
    W = rng.standard_normal((64, 64))
    R = np.stack([O.apply_rope(e, 17) for e in np.eye(64)], axis=1)  # column j = R e_j
    assert np.abs(R @ W - W @ R).max() > 1e-2
