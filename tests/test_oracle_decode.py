"""Pins for the oracle's decode: the absorbed and explicit forms agree (the
associativity identity of '3. Decoupled RoPE and Matrix Absorption'), the
textbook single-head reduction equals torch's scaled_dot_product_attention,
and closed-form special cases hold."""
import numpy as np
import pytest
import torch

from oracle import mla_oracle as O


def rand_problem(rng, n_h=3, d_c=24, d_r=8, d_nope=10, d_v=7, S=37, T=1):
    return dict(
        q_nope=rng.standard_normal((T, n_h, d_nope)),
        q_rope=rng.standard_normal((T, n_h, d_r)),
        C=rng.standard_normal((S, d_c)),
        KR=rng.standard_normal((S, d_r)),
        W_uk=rng.standard_normal((n_h, d_nope, d_c)) / np.sqrt(d_c),
        W_uv=rng.standard_normal((n_h, d_v, d_c)) / np.sqrt(d_c),
        seq_len=S, scale=1 / np.sqrt(d_nope + d_r))


@pytest.mark.parametrize("T,S", [(1, 1), (1, 2), (1, 37), (2, 2), (2, 65), (3, 40)])
def test_absorbed_equals_explicit(T, S):
    P = rand_problem(np.random.default_rng(T * 100 + S), S=S, T=T)
    o1, l1 = O.decode_explicit(**P)
    o2, l2, _ = O.decode_absorbed(**P)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, l1, rtol=1e-12, atol=1e-13)


def closed_form_rotate(x, p, base=10000.0):
    d = len(x)
    out = np.empty(d)
    for i in range(d // 2):
        th = p * base ** (-2.0 * i / d)
        out[i] = np.cos(th) * x[i] - np.sin(th) * x[i + d // 2]
        out[i + d // 2] = np.sin(th) * x[i] + np.cos(th) * x[i + d // 2]
    return out


@pytest.mark.parametrize("fmt", ["bf16", "f16"])
def test_query_rounding_option_matches_sdpa_on_a_rounded_query(fmt):
    """decode_absorbed(q_round=...) is the attention of the query rounded to
    that format: in the textbook reduction (n_h = 1, W_uk = W_uv = I) it equals
    torch's attention on a query cast to the format by torch itself."""
    rng = np.random.default_rng(31)
    d_c, d_r, S, T = 16, 8, 40, 2
    P = rand_problem(rng, n_h=1, d_c=d_c, d_r=d_r, d_nope=d_c, d_v=d_c, S=S, T=T)
    P["q_nope"] = P["q_nope"] * 7.0  # wide logits, so that the rounding shows
    P["W_uk"] = np.eye(d_c)[None]
    P["W_uv"] = np.eye(d_c)[None]
    rnd = O.to_bf16 if fmt == "bf16" else O.to_f16
    tdt = torch.bfloat16 if fmt == "bf16" else torch.float16
    o, _, _ = O.decode_absorbed(**P, q_round=rnd)
    o_exact, _, _ = O.decode_absorbed(**P)
    pos = S - T + np.arange(T)
    Q = np.stack([np.concatenate([P["q_nope"][t, 0], closed_form_rotate(P["q_rope"][t, 0], pos[t])])
                  for t in range(T)])
    Q = torch.from_numpy(Q.astype(np.float32)).to(tdt).to(torch.float64)
    K = np.concatenate([P["C"], P["KR"]], axis=1)
    mask = np.arange(S)[None, :] <= pos[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q[None], torch.from_numpy(K)[None], torch.from_numpy(P["C"])[None],
        attn_mask=torch.from_numpy(mask)[None])[0].numpy()
    np.testing.assert_allclose(o[:, 0], ref, rtol=1e-12, atol=1e-13)
    assert np.abs(o - o_exact).max() > 0  # the option does round


@pytest.mark.parametrize("T", [1, 2])
def test_textbook_reduction_matches_torch_sdpa(T):
    """n_h = 1, d_nope = d_c, W_uk = W_uv = I: MLA is single-head attention with
    keys [c_s ; k^R_s], values c_s and query [q ; R_p q^R]."""
    rng = np.random.default_rng(7 + T)
    d_c, d_r, S = 16, 8, 50
    P = rand_problem(rng, n_h=1, d_c=d_c, d_r=d_r, d_nope=d_c, d_v=d_c, S=S, T=T)
    P["W_uk"] = np.eye(d_c)[None]
    P["W_uv"] = np.eye(d_c)[None]
    o, lse = O.decode_explicit(**P)
    pos = S - T + np.arange(T)
    Q = np.stack([np.concatenate([P["q_nope"][t, 0], closed_form_rotate(P["q_rope"][t, 0], pos[t])])
                  for t in range(T)])
    K = np.concatenate([P["C"], P["KR"]], axis=1)
    mask = np.arange(S)[None, :] <= pos[:, None]  # key s visible to query t iff s <= L + t
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(P["C"])[None],
        attn_mask=torch.from_numpy(mask)[None])[0].numpy()  # default scale 1/sqrt(d_c + d_r)
    np.testing.assert_allclose(o[:, 0], ref, rtol=1e-12, atol=1e-13)


def test_single_key_returns_its_value():
    P = rand_problem(np.random.default_rng(3), S=1)
    o, lse = O.decode_explicit(**P)
    for h in range(3):
        np.testing.assert_allclose(o[0, h], P["W_uv"][h] @ P["C"][0], rtol=1e-13)
        score = P["scale"] * (P["q_nope"][0, h] @ (P["W_uk"][h] @ P["C"][0])
                              + P["q_rope"][0, h] @ P["KR"][0])  # position 0: no rotation
        assert abs(lse[0, h] - score) < 1e-12


def test_two_keys_logistic_weights():
    P = rand_problem(np.random.default_rng(4), n_h=1, S=2)
    o, lse = O.decode_explicit(**P)
    q, qr = P["q_nope"][0, 0], P["q_rope"][0, 0]
    a = [P["scale"] * (q @ (P["W_uk"][0] @ P["C"][s]) + closed_form_rotate(qr, 1) @ P["KR"][s]) for s in (0, 1)]
    w0 = 1 / (1 + np.exp(a[1] - a[0]))
    expect = w0 * (P["W_uv"][0] @ P["C"][0]) + (1 - w0) * (P["W_uv"][0] @ P["C"][1])
    np.testing.assert_allclose(o[0, 0], expect, rtol=1e-12)
    assert abs(lse[0, 0] - np.logaddexp(a[0], a[1])) < 1e-12


def test_equal_latents_give_their_value_for_any_query():
    P = rand_problem(np.random.default_rng(5), S=30)
    P["C"][:] = P["C"][0]
    o, _ = O.decode_explicit(**P)
    for h in range(3):
        np.testing.assert_allclose(o[0, h], P["W_uv"][h] @ P["C"][0], rtol=1e-12)


def test_zero_query_gives_mean_value():
    P = rand_problem(np.random.default_rng(6), S=30)
    P["q_nope"][:] = 0
    P["q_rope"][:] = 0
    o, lse = O.decode_explicit(**P)
    for h in range(3):
        np.testing.assert_allclose(o[0, h], P["W_uv"][h] @ P["C"].mean(0), rtol=1e-12)
    np.testing.assert_allclose(lse, np.log(30.0), rtol=1e-14)


def test_query_rotated_at_its_own_position():
    """Content scores off, k^R_s = R_s k0 and q^R = k0: the RoPE score peaks at
    relative distance 0, i.e. at the newest key (the query's own position)."""
    d_c, S, d_r = 64, 50, 64
    rng = np.random.default_rng(8)
    k0 = rng.standard_normal(d_r)
    P = dict(q_nope=np.zeros((1, 1, 4)), q_rope=k0[None, None] * 3, C=np.eye(S, d_c),
             KR=np.stack([O.apply_rope(k0, s) for s in range(S)]),
             W_uk=np.zeros((1, 4, d_c)), W_uv=np.eye(d_c)[None], seq_len=S,
             scale=1 / np.sqrt(4 + d_r))
    o, _ = O.decode_explicit(**P)
    weights = o[0, 0, :S]  # c_s = e_s, W_uv = I: the output is the weight vector
    assert int(np.argmax(weights)) == S - 1
    np.testing.assert_allclose(weights.sum(), 1.0, rtol=1e-13)


def test_causal_between_new_tokens():
    P = rand_problem(np.random.default_rng(9), S=20, T=2)
    o1, l1 = O.decode_explicit(**P)
    P2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in P.items()}
    P2["C"][-1] += 5.0
    P2["KR"][-1] -= 3.0
    o2, l2 = O.decode_explicit(**P2)
    np.testing.assert_array_equal(o1[0], o2[0])  # query 0 does not see the last key
    assert np.abs(o1[1] - o2[1]).max() > 1e-3


def test_merge_of_split_softmax_equals_full():
    rng = np.random.default_rng(10)
    a = rng.standard_normal((4, 90)) * 3  # 4 rows of scores over 90 keys
    X = rng.standard_normal((90, 6))

    def part(idx):
        m = a[:, idx].max(1, keepdims=True)
        e = np.exp(a[:, idx] - m)
        return (e / e.sum(1, keepdims=True)) @ X[idx], (m + np.log(e.sum(1, keepdims=True)))[:, 0]

    full_u, full_l = part(np.arange(90))
    for cuts in [[45], [1, 89], [10, 20, 30, 80]]:
        pieces = np.split(np.arange(90), cuts)
        us, ls = zip(*[part(p) for p in pieces])
        u, l = O.merge_partials(np.stack(us), np.stack(ls))
        np.testing.assert_allclose(u, full_u, rtol=1e-12)
        np.testing.assert_allclose(l, full_l, rtol=1e-13)
