"""Pins for the oracle's append: exact integer arithmetic at position 0 and the
closed-form rotation of k^R at other positions."""
import numpy as np

from oracle import mla_oracle as O
from tests.test_oracle_rope import rotation_closed_form


def test_append_exact_integer_case():
    rng = np.random.default_rng(0)
    d, d_c, d_r = 96, 16, 8
    h = rng.integers(-4, 5, size=(3, d))
    W_dkv = rng.integers(-1, 2, size=(d_c, d))
    W_kr = rng.integers(-1, 2, size=(d_r, d))
    c, kr = O.append_latent(h, W_dkv, W_kr, pos=np.zeros(3, dtype=int))
    for n in range(3):
        for j in range(d_c):
            assert c[n, j] == sum(int(W_dkv[j, k]) * int(h[n, k]) for k in range(d))
        for j in range(d_r):
            assert kr[n, j] == sum(int(W_kr[j, k]) * int(h[n, k]) for k in range(d))


def test_append_rotates_kr_at_its_position():
    rng = np.random.default_rng(1)
    d, d_c, d_r = 32, 8, 16
    h = rng.standard_normal((4, d))
    W_dkv, W_kr = rng.standard_normal((d_c, d)), rng.standard_normal((d_r, d))
    pos = np.array([0, 3, 64, 100000])
    c, kr = O.append_latent(h, W_dkv, W_kr, pos)
    for n in range(4):
        np.testing.assert_allclose(c[n], W_dkv @ h[n], rtol=1e-13)
        np.testing.assert_allclose(kr[n], rotation_closed_form(W_kr @ h[n], pos[n], 10000.0), atol=1e-12)


def test_encode_rows_formats():
    rng = np.random.default_rng(2)
    c, kr = rng.standard_normal((5, 256)), rng.standard_normal((5, 64))
    r = O.encode_cache_rows(c, kr, "bf16")
    assert np.abs(r["c"] - c).max() <= 2.0 ** -8 * np.abs(c).max()
    r = O.encode_cache_rows(c, kr, "f32")
    np.testing.assert_array_equal(r["c"], c.astype(np.float32))
    r = O.encode_cache_rows(c, kr, "fp8")
    cc, kk = O.decode_cache_rows(r)
    assert np.abs(cc - c).max() <= 2.0 ** -4 * np.abs(c).max()
    np.testing.assert_array_equal(kk, O.to_bf16(kr))


def test_paged_slot():
    pt = np.array([[5, 2, 9], [0, 7, 1]])
    assert O.paged_slot(pt, 0, 0, 64) == (5, 0)
    assert O.paged_slot(pt, 0, 63, 64) == (5, 63)
    assert O.paged_slot(pt, 0, 64, 64) == (2, 0)
    assert O.paged_slot(pt, 1, 150, 64) == (1, 22)
