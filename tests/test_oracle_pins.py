"""Pins of the fp64 oracle against facts fixed by the pages and by the mathematics.

Each test checks the oracle against something other than itself:
  * hand-derived worked examples under tests/golden/ (each cites its passage);
  * closed forms (a two-token softmax is a logistic; a one-token frame attends
    to itself; orthonormal keys make the delta rule write V' exactly);
  * invariants (row sums, permutation equivariance, shift invariance, linearity,
    decay over many frames).
A plausible slip in the oracle (dropped 1/sqrt(d), softmax over the wrong axis,
a transposed phi or state, beta instead of beta/T, a product instead of a mean
of the gates, decaying S before the residual, a missing key normalisation) fails
at least one of them; test_planted_mistakes_are_caught shows it.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import arl2_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _commit_from_fixture(g, commit=orc.frame_commit):
    T, d = g["T"], g["d"]
    k = np.array(g["K"], float).reshape(1, T, 1, d)
    v = np.array(g["V"], float).reshape(1, T, 1, d)
    Wk = np.array(g["Wk"], float).reshape(1, d, d)
    Wv = np.array(g["Wv"], float).reshape(1, d, d)
    S = np.array(g["S_prev"], float).reshape(1, 1, d, d)
    a = np.array(g["alpha"], float).reshape(1, 1, T)
    b = np.array(g["beta"], float).reshape(1, 1, T)
    return commit(k, v, a, b, Wk, Wv, S)[0, 0]


# ---------------------------------------------------------------- golden examples
@pytest.mark.parametrize("name", ["commit_normalised_keys.json", "commit_general.json"])
def test_commit_golden(name):
    g = _golden(name)
    np.testing.assert_allclose(_commit_from_fixture(g), np.array(g["S_next"]), rtol=0, atol=1e-14)


def test_query_readout_golden():
    g = _golden("query_readout.json")
    q = np.array(g["q"], float).reshape(1, 1, 1, 2)
    k = np.array(g["k"], float).reshape(1, 1, 1, 2)
    v = np.array(g["v"], float).reshape(1, 1, 1, 2)
    Wq = np.array(g["Wq"], float).reshape(1, 2, 2)
    S = np.array(g["S"], float).reshape(1, 1, 2, 2)
    o, o_intra, o_inter = orc.frame_query(q, k, v, Wq, S)
    np.testing.assert_allclose(o_inter.ravel(), g["O_inter"], atol=1e-14)
    np.testing.assert_allclose(o.ravel(), g["O"], atol=1e-14)


def test_two_token_attention_golden():
    g = _golden("attention_two_tokens.json")
    q = np.array(g["q"], float).reshape(1, 2, 1, 4)
    k = np.array(g["k"], float).reshape(1, 2, 1, 4)
    v = np.array(g["v"], float).reshape(1, 2, 1, 4)
    np.testing.assert_allclose(orc.intra_attention(q, k, v)[0, :, 0, :], np.array(g["O"]), atol=1e-15)


# ---------------------------------------------------------------- intra-frame attention
def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_softmax_rows_sum_to_one():
    Q, K = _rand((37, 16), 1), _rand((53, 16), 2) * 3
    P = orc.attention_matrix(Q, K)
    assert P.shape == (37, 53)
    assert np.all(P > 0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-15)


def test_single_token_frame_returns_v():
    q, k, v = _rand((2, 1, 3, 8), 3), _rand((2, 1, 3, 8), 4), _rand((2, 1, 3, 8), 5)
    np.testing.assert_allclose(orc.intra_attention(q, k, v), v, atol=1e-15)


def test_equal_keys_give_column_mean_of_v():
    q, v = _rand((1, 9, 2, 8), 6), _rand((1, 9, 2, 8), 7)
    k = np.broadcast_to(_rand((1, 1, 2, 8), 8), (1, 9, 2, 8))
    out = orc.intra_attention(q, k, v)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=1, keepdims=True), out.shape), atol=1e-14)


def test_token_permutation_is_equivariant():
    q, k, v = _rand((1, 11, 2, 8), 9), _rand((1, 11, 2, 8), 10), _rand((1, 11, 2, 8), 11)
    perm = np.random.default_rng(12).permutation(11)
    base = orc.intra_attention(q, k, v)
    out = orc.intra_attention(q[:, perm], k[:, perm], v[:, perm])
    np.testing.assert_allclose(out, base[:, perm], atol=1e-13)


def test_key_shift_invariance():
    # Adding one vector w to every key shifts each score row by q.w, which softmax removes.
    q, k, v = _rand((1, 13, 1, 8), 13), _rand((1, 13, 1, 8), 14), _rand((1, 13, 1, 8), 15)
    w = _rand((1, 1, 1, 8), 16) * 5
    np.testing.assert_allclose(orc.intra_attention(q, k + w, v), orc.intra_attention(q, k, v), atol=1e-12)


def test_dominant_key_selects_its_value():
    T, d = 6, 8
    q = np.zeros((1, T, 1, d)); q[..., 0] = 1.0
    k = np.zeros((1, T, 1, d)); k[0, 4, 0, 0] = 2000.0  # score 2000/sqrt(8) above the rest
    v = _rand((1, T, 1, d), 17)
    np.testing.assert_allclose(orc.intra_attention(q, k, v)[0, :, 0], np.broadcast_to(v[0, 4, 0], (T, d)), atol=1e-12)


def test_rows_subset_matches_full():
    q, k, v = _rand((2, 20, 3, 8), 18), _rand((2, 20, 3, 8), 19), _rand((2, 20, 3, 8), 20)
    rows = [0, 7, 19]
    np.testing.assert_allclose(orc.intra_attention(q, k, v, rows), orc.intra_attention(q, k, v)[:, rows], atol=1e-15)


# ---------------------------------------------------------------- readout
def test_readout_identity_maps_return_q():
    q = _rand((1, 5, 2, 4), 21)
    Wq = np.broadcast_to(np.eye(4), (2, 4, 4))
    S = np.broadcast_to(np.eye(4), (1, 2, 4, 4))
    np.testing.assert_allclose(orc.readout(q, Wq, S), q, atol=1e-15)


def test_readout_is_linear_in_state():
    q, Wq, S = _rand((1, 7, 2, 4), 22), _rand((2, 4, 4), 23), _rand((1, 2, 4, 4), 24)
    np.testing.assert_allclose(orc.readout(q, Wq, -2.5 * S), -2.5 * orc.readout(q, Wq, S), atol=1e-13)


def test_heads_are_independent():
    B, T, H, d = 2, 6, 3, 4
    q, k, v = _rand((B, T, H, d), 25), _rand((B, T, H, d), 26), _rand((B, T, H, d), 27)
    Wq, S = _rand((H, d, d), 28), _rand((B, H, d, d), 29)
    perm = np.array([2, 0, 1])
    base = orc.frame_query(q, k, v, Wq, S)[0]
    out = orc.frame_query(q[:, :, perm], k[:, :, perm], v[:, :, perm], Wq[perm], S[:, perm])[0]
    np.testing.assert_allclose(out, base[:, :, perm], atol=1e-13)


# ---------------------------------------------------------------- commit
def _commit_inputs(B=1, T=8, H=2, d=4, seed=30):
    r = np.random.default_rng(seed)
    k, v = r.standard_normal((B, T, H, d)), r.standard_normal((B, T, H, d))
    Wk, Wv = r.standard_normal((H, d, d)) / 2, r.standard_normal((H, d, d)) / 2
    S = r.standard_normal((B, H, d, d))
    a = 1 / (1 + np.exp(-r.normal(2, 0.5, (B, H, T))))
    b = 1 / (1 + np.exp(-r.standard_normal((B, H, T))))
    return k, v, a, b, Wk, Wv, S


def test_alpha_one_beta_zero_keeps_state():
    k, v, a, b, Wk, Wv, S = _commit_inputs()
    np.testing.assert_array_equal(orc.frame_commit(k, v, np.ones_like(a), np.zeros_like(b), Wk, Wv, S), S)


def test_zero_state_zero_gate_is_weighted_outer_product():
    # With S_{N-1}=0, alpha=0, phi_k = phi_v = I and unit keys: S_N = K^T diag(beta/T) V.
    B, T, H, d = 1, 7, 1, 4
    r = np.random.default_rng(31)
    k = r.standard_normal((B, T, H, d)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, d))
    beta = r.uniform(0.1, 1, (B, H, T))
    I = np.eye(d)[None]
    S = orc.frame_commit(k, v, np.zeros((B, H, T)), beta, I, I, np.zeros((B, H, d, d)))
    outer = sum(beta[0, 0, t] / T * np.outer(k[0, t, 0], v[0, t, 0]) for t in range(T))
    np.testing.assert_allclose(S[0, 0], outer, atol=1e-14)


@pytest.mark.parametrize("abar", [1.0, 0.6])
def test_single_unit_key_writes_value(abar):
    # T=1, unit key, beta/T = 1: K'S_N = abar K'S + (V' - K'S) = V' - (1 - abar) K'S.
    d = 4
    r = np.random.default_rng(32)
    k = r.standard_normal((1, 1, 1, d)); k /= np.linalg.norm(k)
    v = r.standard_normal((1, 1, 1, d))
    S0 = r.standard_normal((1, 1, d, d))
    I = np.eye(d)[None]
    S1 = orc.frame_commit(k, v, np.full((1, 1, 1), abar), np.ones((1, 1, 1)), I, I, S0)
    kS0 = k[0, 0, 0] @ S0[0, 0]
    np.testing.assert_allclose(k[0, 0, 0] @ S1[0, 0], v[0, 0, 0] - (1 - abar) * kS0, atol=1e-14)


def test_orthonormal_keys_store_values_and_recommit_is_idempotent():
    # K' = I (T = d one-hot keys), beta = T, alpha = 1: S_N = V'; committing the same frame again keeps it.
    d = 5
    r = np.random.default_rng(33)
    k = np.eye(d).reshape(1, d, 1, d) * r.uniform(0.5, 3, (1, d, 1, 1))  # positive scales vanish in K'
    v = r.standard_normal((1, d, 1, d))
    Wv = r.standard_normal((1, d, d))
    S0 = r.standard_normal((1, 1, d, d))
    ones, beta = np.ones((1, 1, d)), np.full((1, 1, d), float(d))
    S1 = orc.frame_commit(k, v, ones, beta, np.eye(d)[None], Wv, S0)
    np.testing.assert_allclose(S1[0, 0], v[0, :, 0] @ Wv[0], atol=1e-13)
    S2 = orc.frame_commit(k, v, ones, beta, np.eye(d)[None], Wv, S1)
    np.testing.assert_allclose(S2, S1, atol=1e-13)


def test_pure_decay_over_many_frames():
    k, v, a, b, Wk, Wv, S0 = _commit_inputs(seed=34)
    c = 0.97
    S = S0
    for n in range(1, 241):
        S = orc.frame_commit(k, v, np.full_like(a, c), np.zeros_like(b), Wk, Wv, S)
        if n in (1, 60, 240):
            np.testing.assert_allclose(S, c ** n * S0, rtol=1e-12, atol=0)


def test_commit_ignores_token_order():
    k, v, a, b, Wk, Wv, S = _commit_inputs(T=9, seed=35)
    perm = np.random.default_rng(36).permutation(9)
    S1 = orc.frame_commit(k, v, a, b, Wk, Wv, S)
    S2 = orc.frame_commit(k[:, perm], v[:, perm], a[..., perm], b[..., perm], Wk, Wv, S)
    np.testing.assert_allclose(S2, S1, atol=1e-13)


def test_zero_key_contributes_nothing():
    k, v, a, b, Wk, Wv, S = _commit_inputs(T=4, seed=37)
    k2 = k.copy(); k2[:, 2] = 0.0
    out = orc.frame_commit(k2, v, a, b, Wk, Wv, S)
    assert np.all(np.isfinite(out))
    keep = [0, 1, 3]
    # Removing the zero-key token changes only abar (its alpha) and T (the beta/T rate).
    a3, b3 = a[..., keep], b[..., keep] * 3 / 4
    abar_ratio = a.mean(axis=-1) / a3.mean(axis=-1)
    ref = orc.frame_commit(k2[:, keep], v[:, keep], a3 * abar_ratio[..., None], b3, Wk, Wv, S)
    np.testing.assert_allclose(out, ref, atol=1e-13)


def test_normalised_keys_have_unit_norm():
    x = _rand((2, 5, 3, 8), 38) * 7
    n = np.linalg.norm(orc.l2_normalize_rows(x), axis=-1)
    np.testing.assert_allclose(n, 1.0, atol=1e-15)
    unit = np.zeros(4); unit[1] = 1.0
    np.testing.assert_array_equal(orc.l2_normalize_rows(unit), unit)


# ---------------------------------------------------------------- the frame schedule
def test_layer_frame_level_access_and_clean_pass_update():
    B, T, H, d = 1, 6, 2, 4
    r = np.random.default_rng(39)
    Wq, Wk, Wv = (r.standard_normal((H, d, d)) for _ in range(3))
    layer = oracle.Layer(Wq, Wk, Wv, B)
    q, k, v = (r.standard_normal((B, T, H, d)) for _ in range(3))
    a, b = r.uniform(0.5, 1, (B, H, T)), r.uniform(0, 1, (B, H, T))
    # Frame 1 reads S_0 = 0: the output is the intra branch alone; queries never write S.
    np.testing.assert_allclose(layer.query(q, k, v), orc.intra_attention(q, k, v), atol=1e-15)
    layer.query(q, k, v)
    np.testing.assert_array_equal(layer.S, 0.0)
    S1 = layer.commit(k, v, a, b)
    assert layer.frame == 1 and np.any(S1 != 0)
    # Frame 2 reads S_1 for every token.
    np.testing.assert_allclose(layer.query(q, k, v), orc.frame_query(q, k, v, Wq, S1)[0], atol=1e-15)
    layer.reset()
    np.testing.assert_array_equal(layer.S, 0.0)


def test_kv_cache_baseline_reduces_to_intra_attention_for_one_frame():
    q, k, v = _rand((1, 8, 2, 4), 40), _rand((1, 8, 2, 4), 41), _rand((1, 8, 2, 4), 42)
    cache_k = np.concatenate([k, _rand((1, 16, 2, 4), 43)], axis=1)
    cache_v = np.concatenate([v, _rand((1, 16, 2, 4), 44)], axis=1)
    np.testing.assert_allclose(orc.kv_cache_attention(q, cache_k, cache_v, 8), orc.intra_attention(q, k, v), atol=1e-15)


# ---------------------------------------------------------------- the pins catch plausible slips
def _mutants():
    """Oracle commits with one planted mistake each (test-only copies; the oracle is untouched)."""
    fm, norm = orc.feature_map, orc.l2_normalize_rows

    def make(transpose_w=False, no_norm=False, beta_plain=False, prod_alpha=False,
             decayed_residual=False, transposed_update=False, plus_residual=False):
        def commit(k, v, alpha, beta, Wk, Wv, S):
            Wk2 = np.swapaxes(Wk, 1, 2) if transpose_w else Wk
            kp = fm(k, Wk2) if no_norm else norm(fm(k, Wk2))
            vp = fm(v, Wv)
            B, T, H, _ = kp.shape
            out = np.empty_like(S)
            for bb in range(B):
                for h in range(H):
                    K, V, S0 = kp[bb, :, h], vp[bb, :, h], S[bb, h]
                    abar = alpha[bb, h].prod() if prod_alpha else alpha[bb, h].mean()
                    rate = beta[bb, h] if beta_plain else beta[bb, h] / T
                    base = abar * S0 if decayed_residual else S0
                    res = V + K @ base if plus_residual else V - K @ base
                    U = K.T @ (rate[:, None] * res)
                    out[bb, h] = abar * S0 + (U.T if transposed_update else U)
            return out
        return commit

    names = ["transpose_w", "no_norm", "beta_plain", "prod_alpha", "decayed_residual",
             "transposed_update", "plus_residual"]
    return {n: make(**{n: True}) for n in names}


@pytest.mark.parametrize("mistake", sorted(_mutants()))
def test_planted_mistakes_are_caught(mistake):
    bad = _mutants()[mistake]
    g = _golden("commit_general.json")
    caught = not np.allclose(_commit_from_fixture(g, bad), np.array(g["S_next"]), atol=1e-12)
    g0 = _golden("commit_normalised_keys.json")
    caught |= not np.allclose(_commit_from_fixture(g0, bad), np.array(g0["S_next"]), atol=1e-12)
    assert caught, f"planted mistake {mistake!r} passed both commit fixtures"


# ---------------------------------------------------------------- gate producer
def _gates_fixture():
    g = _golden("gates_from_hidden.json")
    x = np.array(g["x"], float)[None]
    return g, x, np.array(g["Wa"], float), np.array(g["ba"], float), np.array(g["Wb"], float), np.array(g["bb"], float)


def test_gates_golden():
    g, x, Wa, ba, Wb, bb = _gates_fixture()
    a, b = orc.gates_from_hidden(x, Wa, ba, Wb, bb)
    np.testing.assert_allclose(a[0], np.array(g["alpha"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(b[0], np.array(g["beta"]), rtol=0, atol=1e-15)


def test_gates_of_a_zero_hidden_state_are_the_bias_sigmoid():
    rng = np.random.default_rng(3)
    H, D = 3, 8
    Wa, Wb = rng.standard_normal((H, D)), rng.standard_normal((H, D))
    ba, bb = rng.standard_normal(H), rng.standard_normal(H)
    a, b = orc.gates_from_hidden(np.zeros((2, 5, D)), Wa, ba, Wb, bb)
    for h in range(H):
        assert np.all(a[:, h] == 1.0 / (1.0 + np.exp(-ba[h])))
        assert np.all(b[:, h] == 1.0 / (1.0 + np.exp(-bb[h])))


def test_gate_logits_are_affine_in_the_hidden_state():
    # logit(alpha(x1 + x2)) = logit(alpha(x1)) + logit(alpha(x2)) - ba, per head and token.
    rng = np.random.default_rng(4)
    B, T, D, H = 2, 6, 16, 3
    x1, x2 = rng.standard_normal((B, T, D)) * 0.3, rng.standard_normal((B, T, D)) * 0.3
    Wa, Wb = rng.standard_normal((H, D)) * 0.5, rng.standard_normal((H, D)) * 0.5
    ba, bb = rng.standard_normal(H), rng.standard_normal(H)
    logit = lambda p: np.log(p) - np.log1p(-p)
    a1, b1 = orc.gates_from_hidden(x1, Wa, ba, Wb, bb)
    a2, b2 = orc.gates_from_hidden(x2, Wa, ba, Wb, bb)
    a12, b12 = orc.gates_from_hidden(x1 + x2, Wa, ba, Wb, bb)
    np.testing.assert_allclose(logit(a12), logit(a1) + logit(a2) - ba[None, :, None], atol=1e-12)
    np.testing.assert_allclose(logit(b12), logit(b1) + logit(b2) - bb[None, :, None], atol=1e-12)


def test_gated_commit_is_the_commit_with_produced_gates():
    rng = np.random.default_rng(5)
    B, T, H, d = 1, 9, 2, 4
    D = H * d
    x = rng.standard_normal((B, T, D))
    k, v = rng.standard_normal((B, T, H, d)), rng.standard_normal((B, T, H, d))
    Wa, Wb = rng.standard_normal((H, D)), rng.standard_normal((H, D))
    ba, bb = rng.standard_normal(H), rng.standard_normal(H)
    Wk, Wv = rng.standard_normal((H, d, d)), rng.standard_normal((H, d, d))
    S = rng.standard_normal((B, H, d, d))
    # The same commit with hand-computed gates (a loop over tokens, not the oracle's matmul).
    a = np.empty((B, H, T))
    b = np.empty((B, H, T))
    for h in range(H):
        for t in range(T):
            a[0, h, t] = 1.0 / (1.0 + np.exp(-(sum(x[0, t, j] * Wa[h, j] for j in range(D)) + ba[h])))
            b[0, h, t] = 1.0 / (1.0 + np.exp(-(sum(x[0, t, j] * Wb[h, j] for j in range(D)) + bb[h])))
    np.testing.assert_allclose(orc.frame_commit_gated(x, k, v, Wa, ba, Wb, bb, Wk, Wv, S),
                               orc.frame_commit(k, v, a, b, Wk, Wv, S), atol=1e-12)


def test_planted_gate_mistakes_are_caught():
    g, x, Wa, ba, Wb, bb = _gates_fixture()
    sig = lambda z: 1.0 / (1.0 + np.exp(-z))
    mistakes = {
        "no bias": lambda: (sig(x[0] @ Wa.T).T, sig(x[0] @ Wb.T).T),
        "gates swapped": lambda: (sig(x[0] @ Wb.T + bb).T, sig(x[0] @ Wa.T + ba).T),
        "weights transposed": lambda: (sig(x[0] @ Wa + ba).T, sig(x[0] @ Wb + bb).T),
        "tanh for sigmoid": lambda: (np.tanh(x[0] @ Wa.T + ba).T, np.tanh(x[0] @ Wb.T + bb).T),
        "minus sign": lambda: (sig(-(x[0] @ Wa.T) + ba).T, sig(-(x[0] @ Wb.T) + bb).T),
    }
    for name, wrong in mistakes.items():
        a, b = wrong()
        ok = np.allclose(a, g["alpha"], atol=1e-12) and np.allclose(b, g["beta"], atol=1e-12)
        assert not ok, f"the gate fixture does not catch: {name}"


# ---- Token-level access (reading R15) ------------------------------------------------------

def _token_fixture():
    g = _golden("token_scan_two_tokens.json")
    q, k, v = (np.array(g[n], float)[None, :, None, :] for n in ("q", "k", "v"))
    a = np.array(g["alpha"], float)[None, None, :]
    b = np.array(g["beta"], float)[None, None, :]
    S0 = np.array(g["S0"], float)[None, None]
    I = np.eye(2)[None]
    return g, q, k, v, a, b, I, S0


def test_token_scan_golden():
    g, q, k, v, a, b, I, S0 = _token_fixture()
    o, S = orc.token_level_scan(q, k, v, a, b, I, I, I, S0)
    np.testing.assert_allclose(o[0, :, 0], np.array(g["o_inter"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], np.array(g["S_end"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(orc.frame_commit_token(k, v, a, b, I, I, S0)[0, 0], np.array(g["S_end"]), atol=1e-14)


def test_token_scan_of_one_token_is_the_frame_level_layer():
    # T = 1: the frame's mean gate is the token's gate and beta/T = beta, so token-level and
    # frame-level access agree, for the readout and the commit.
    rng = np.random.default_rng(21)
    B, H, d = 2, 3, 4
    q, k, v = (rng.standard_normal((B, 1, H, d)) for _ in range(3))
    Wq, Wk, Wv = (rng.standard_normal((H, d, d)) for _ in range(3))
    S = rng.standard_normal((B, H, d, d))
    a, b = rng.uniform(0.1, 0.9, (B, H, 1)), rng.uniform(0.1, 0.9, (B, H, 1))
    o, S_end = orc.token_level_scan(q, k, v, a, b, Wq, Wk, Wv, S)
    np.testing.assert_allclose(o, orc.readout(q, Wq, S), atol=1e-12)
    np.testing.assert_allclose(S_end, orc.frame_commit(k, v, a, b, Wk, Wv, S), atol=1e-12)


def test_token_scan_is_a_sequence_of_one_token_frames():
    # Token-level access over T tokens = T frame-level commits of one-token frames, each token
    # reading the state its predecessors left.
    rng = np.random.default_rng(22)
    B, T, H, d = 1, 7, 2, 4
    q, k, v = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    Wq, Wk, Wv = (rng.standard_normal((H, d, d)) / 2 for _ in range(3))
    S = rng.standard_normal((B, H, d, d))
    a, b = rng.uniform(0.5, 1.0, (B, H, T)), rng.uniform(0.0, 1.0, (B, H, T))
    o, S_end = orc.token_level_scan(q, k, v, a, b, Wq, Wk, Wv, S)
    St = S
    for t in range(T):
        np.testing.assert_allclose(o[:, t:t + 1], orc.readout(q[:, t:t + 1], Wq, St), atol=1e-12)
        St = orc.frame_commit(k[:, t:t + 1], v[:, t:t + 1], a[:, :, t:t + 1], b[:, :, t:t + 1], Wk, Wv, St)
    np.testing.assert_allclose(S_end, St, atol=1e-12)


def test_token_scan_closed_forms():
    rng = np.random.default_rng(23)
    B, T, H, d = 1, 6, 2, 6
    q, k, v = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    I = np.stack([np.eye(d)] * H)
    S = rng.standard_normal((B, H, d, d))
    # alpha = 1, beta = 0: nothing moves; every token reads S.
    o, S_end = orc.token_level_scan(q, k, v, np.ones((B, H, T)), np.zeros((B, H, T)), I, I, I, S)
    np.testing.assert_array_equal(S_end, S)
    np.testing.assert_allclose(o, orc.readout(q, I, S), atol=1e-12)
    # beta = 0: pure decay, token t reads (prod of the gates before it) S.
    a = rng.uniform(0.3, 0.99, (B, H, T))
    o, S_end = orc.token_level_scan(q, k, v, a, np.zeros((B, H, T)), I, I, I, S)
    for h in range(H):
        np.testing.assert_allclose(S_end[0, h], np.prod(a[0, h]) * S[0, h], atol=1e-12)
        for t in range(T):
            np.testing.assert_allclose(o[0, t, h], np.prod(a[0, h, :t]) * (q[0, t, h] @ S[0, h]), atol=1e-12)
    # Orthonormal keys and alpha = 1: the tokens' updates do not interact, so
    # S_end = S + sum_t beta_t k_t^T (v_t - k_t S).
    Qm = np.linalg.qr(rng.standard_normal((d, d)))[0]
    k_on = np.broadcast_to(Qm[:T][None, :, None, :], (B, T, H, d)).copy()
    b = rng.uniform(0.1, 1.0, (B, H, T))
    _, S_end = orc.token_level_scan(None, k_on, v, np.ones((B, H, T)), b, None, I, I, S)
    for h in range(H):
        want = S[0, h] + sum(b[0, h, t] * np.outer(k_on[0, t, h], v[0, t, h] - k_on[0, t, h] @ S[0, h])
                             for t in range(T))
        np.testing.assert_allclose(S_end[0, h], want, atol=1e-12)


def test_token_query_adds_the_scan_readout_to_intra_attention():
    rng = np.random.default_rng(24)
    B, T, H, d = 1, 5, 2, 4
    q, k, v = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    W = [rng.standard_normal((H, d, d)) for _ in range(3)]
    S = rng.standard_normal((B, H, d, d))
    a, b = rng.uniform(0.5, 1.0, (B, H, T)), rng.uniform(0.0, 1.0, (B, H, T))
    o_inter, _ = orc.token_level_scan(q, k, v, a, b, *W, S)
    np.testing.assert_allclose(orc.frame_query_token(q, k, v, a, b, *W, S),
                               orc.intra_attention(q, k, v) + o_inter, atol=1e-12)


def test_planted_token_scan_mistakes_are_caught():
    # Test-local copies of the scan, each with one plausible slip; the golden fixture must
    # reject every one of them.
    g, q, k, v, a, b, I, S0 = _token_fixture()
    qv, kv, vv = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    al, be = a[0, 0], b[0, 0]

    def scan(after=False, beta_over_T=False, decayed=False, reverse=False, no_norm=False, mean_alpha=False):
        S = S0[0, 0].copy()
        T = len(al)
        order = range(T - 1, -1, -1) if reverse else range(T)
        o = np.zeros((T, 2))
        for t in order:
            kt = kv[t] if no_norm else kv[t] / np.linalg.norm(kv[t])
            at = al.mean() if mean_alpha else al[t]
            bt = be[t] / T if beta_over_T else be[t]
            res = vv[t] - kt @ (at * S if decayed else S)
            S_next = at * S + bt * np.outer(kt, res)
            o[t] = qv[t] @ (S_next if after else S)
            S = S_next
        return o, S

    ok_o, ok_S = scan()
    np.testing.assert_allclose(ok_o, np.array(g["o_inter"]), atol=1e-14)
    np.testing.assert_allclose(ok_S, np.array(g["S_end"]), atol=1e-14)
    for slip in ("after", "beta_over_T", "decayed", "reverse", "no_norm", "mean_alpha"):
        o, S = scan(**{slip: True})
        caught = (not np.allclose(o, np.array(g["o_inter"]), atol=1e-9) or
                  not np.allclose(S, np.array(g["S_end"]), atol=1e-9))
        assert caught, slip
