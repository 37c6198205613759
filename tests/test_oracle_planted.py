"""Planted mistakes: each plausible error in the oracle makes at least one of
its pins fail. The errors tried are a dropped term, a wrong sign or pairing,
an off-by-one position, a swapped operand, a wrong scale and a wrong
rounding. Each mistake is planted in the oracle, on the CPU, only for the
duration of one test (monkeypatch). The mutated functions below copy the
oracle's steps with exactly one change; they are not pins themselves."""
import numpy as np
import pytest

from oracle import mla_oracle as O
from tests import test_oracle_append as TA
from tests import test_oracle_decode as TD
from tests import test_oracle_formats as TF
from tests import test_oracle_rope as TR

PINS = [
    ("absorbed=explicit T1", lambda: TD.test_absorbed_equals_explicit(1, 37)),
    ("absorbed=explicit T2", lambda: TD.test_absorbed_equals_explicit(2, 65)),
    ("absorbed=explicit T3", lambda: TD.test_absorbed_equals_explicit(3, 40)),
    ("textbook sdpa T1", lambda: TD.test_textbook_reduction_matches_torch_sdpa(1)),
    ("textbook sdpa T2", lambda: TD.test_textbook_reduction_matches_torch_sdpa(2)),
    ("single key", TD.test_single_key_returns_its_value),
    ("two keys", TD.test_two_keys_logistic_weights),
    ("equal latents", TD.test_equal_latents_give_their_value_for_any_query),
    ("zero query", TD.test_zero_query_gives_mean_value),
    ("query at own position", TD.test_query_rotated_at_its_own_position),
    ("causal", TD.test_causal_between_new_tokens),
    ("merge", TD.test_merge_of_split_softmax_equals_full),
    ("rope closed form", TR.test_rope_matches_closed_form_rotations),
    ("rope d2", TR.test_rope_d2_is_plane_rotation),
    ("rope identity/norm", TR.test_rope_identity_at_zero_and_norm_preserving),
    ("rope relative", TR.test_rope_scores_depend_on_relative_position_only),
    ("append integer", TA.test_append_exact_integer_case),
    ("append rotation", TA.test_append_rotates_kr_at_its_position),
    ("bf16 cast", TF.test_bf16_matches_torch_cast),
    ("bf16 ties", TF.test_bf16_ties_to_even),
    ("e4m3 cast", TF.test_e4m3_encode_matches_torch_cast),
    ("fp8 tiles", TF.test_fp8_tile_quantiser_properties),
]


def failing_pins():
    failed = []
    with np.errstate(all="ignore"):
        for name, pin in PINS:
            try:
                pin()
            except Exception:  # an assertion, or a crash the mistake causes
                failed.append(name)
    return failed


# --- planted variants --------------------------------------------------------

def rope_wrong_sign(x, pos, base=10000.0):
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    cos, sin = O.rope_cos_sin(pos, x.shape[-1], base)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos + x2 * sin, x2 * cos - x1 * sin], axis=-1)


def rope_interleaved_pairs(x, pos, base=10000.0):
    x = np.asarray(x, dtype=np.float64)
    cos, sin = O.rope_cos_sin(pos, x.shape[-1], base)
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, cos.shape[:-1] + (x.shape[-1],)))
    out[..., 0::2] = x1 * cos - x2 * sin
    out[..., 1::2] = x2 * cos + x1 * sin
    return out


def rope_freq_over_d(pos, d_rope, base=10000.0):
    half = d_rope // 2
    inv_freq = np.exp(-np.log(base) * np.arange(half, dtype=np.float64) / d_rope)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    return np.cos(ang), np.sin(ang)


def decode_planted(mistake):
    """The explicit decode with one planted mistake."""
    def decode(q_nope, q_rope, C, KR, W_uk, W_uv, seq_len, scale, base=10000.0, heads=None):
        q_nope = np.asarray(q_nope, np.float64)
        q_rope = np.asarray(q_rope, np.float64)
        C = np.asarray(C, np.float64)[:seq_len]
        KR = np.asarray(KR, np.float64)[:seq_len]
        T = q_nope.shape[0]
        heads = range(q_nope.shape[1]) if heads is None else heads
        pos = O.query_positions(seq_len, T)
        o = np.zeros((T, len(heads), np.asarray(W_uv).shape[1]))
        lse = np.zeros((T, len(heads)))
        for hi, h in enumerate(heads):
            K_c = C @ np.asarray(W_uk[h], np.float64).T
            V = C @ np.asarray((W_uk if mistake == "values-from-W_uk" else W_uv)[h], np.float64).T
            for t in range(T):
                p = int(pos[t])
                qr = q_rope[t, h] if mistake == "query-unrotated" else O.apply_rope(q_rope[t, h], p, base)
                if mistake == "rope-score-dropped":
                    q, K = q_nope[t, h], K_c[:p + 1]
                else:
                    q = np.concatenate([q_nope[t, h], qr])
                    K = np.concatenate([K_c[:p + 1], KR[:p + 1]], axis=1)
                if mistake == "no-causal-limit":
                    K = np.concatenate([K_c, KR], axis=1)
                s = scale * (2.0 if mistake == "scale-doubled" else 1.0)
                a = s * (K @ q)
                m = a.max()
                e = np.exp(a - m)
                l = e.sum()
                o[t, hi] = (e / l) @ V[:len(a)]
                lse[t, hi] = np.log(l) if mistake == "lse-without-max" else m + np.log(l)
        return o, lse
    return decode


def merge_unnormalised(us, lses):
    lses = np.asarray(lses, np.float64)
    u = np.einsum("k...,k...d->...d", np.exp(lses), np.asarray(us, np.float64))
    return u, np.log(np.exp(lses).sum(axis=0))


def append_without_rope(h, W_dkv, W_kr, pos, base=10000.0):
    h = np.asarray(h, dtype=np.float64)
    return h @ np.asarray(W_dkv, np.float64).T, h @ np.asarray(W_kr, np.float64).T


def bf16_truncating(x):
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp = np.ldexp(1.0, np.maximum(e, -125) - 8)
    return np.where(x == 0, x, np.trunc(x / ulp) * ulp)


def fp8_scale_240(c):
    c = np.asarray(c, np.float64)
    tiles = c.reshape(*c.shape[:-1], -1, 128)
    amax = np.abs(tiles).max(axis=-1)
    scales = O.to_f32(np.where(amax > 0, amax / 240.0, 1.0))
    codes = O.e4m3_encode(tiles / scales[..., None]).reshape(c.shape)
    return codes, scales


PLANTED = [
    ("rope: rotation sign", "apply_rope", rope_wrong_sign),
    ("rope: interleaved pairs", "apply_rope", rope_interleaved_pairs),
    ("rope: frequency exponent over d", "rope_cos_sin", rope_freq_over_d),
    ("query position one late", "query_positions", lambda S, T: S - T + np.arange(T) + 1),
    ("query position one early", "query_positions", lambda S, T: S - T + np.arange(T) - 1),
    ("decode: rope score dropped", "decode_explicit", decode_planted("rope-score-dropped")),
    ("decode: query not rotated", "decode_explicit", decode_planted("query-unrotated")),
    ("decode: no causal limit", "decode_explicit", decode_planted("no-causal-limit")),
    ("decode: scale doubled", "decode_explicit", decode_planted("scale-doubled")),
    ("decode: lse without max", "decode_explicit", decode_planted("lse-without-max")),
    ("decode: values through W_uk", "decode_explicit", decode_planted("values-from-W_uk")),
    ("merge: weights not normalised", "merge_partials", merge_unnormalised),
    ("append: k^R not rotated", "append_latent", append_without_rope),
    ("bf16: truncation", "to_bf16", bf16_truncating),
    ("fp8: e4m3fnuz scale 240", "fp8_quantise_latent", fp8_scale_240),
]


def test_pins_pass_on_the_oracle_as_written():
    assert failing_pins() == []


@pytest.mark.parametrize("name,attr,planted", PLANTED, ids=[p[0] for p in PLANTED])
def test_planted_mistake_fails_a_pin(monkeypatch, name, attr, planted):
    monkeypatch.setattr(O, attr, planted)
    assert failing_pins(), f"no pin catches: {name}"
