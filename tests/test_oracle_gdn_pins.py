"""Pins of the oracle's GatedDeltaNet decode step against facts outside it.

The Flash-MoE pages (lilting.ch article, section "GatedDeltaNet
acceleration") give the shape of the recurrence (64 heads, a 128x128 state per
head) and the BLAS calls it is built from (scal, gemv, ger), not a formula.
The oracle reads it as the gated delta rule.  These tests hold that reading
and the oracle's code to things that do not come from the oracle:

* the closed matrix form of the gated delta rule, S' = alpha S (I - beta k k^T)
  + beta v k^T (Yang, Kautz and Hatamizadeh, "Gated Delta Networks: Improving
  Mamba2 with Delta Rule", ICLR 2025), evaluated with numpy matrix products
  rather than the oracle's scal/gemv/ger sequence;
* a 2x2 example worked by hand;
* exact special cases: no write (beta = 0), full forgetting (alpha = 0), and
  the delta rule's defining property that a full-strength write at a unit key
  makes the state recall exactly the written value at that key;
* an associative-memory closed form for orthonormal keys;
* invariants: heads are independent, and the update never grows the state
  when nothing is written.

A dropped term, a wrong sign, alpha applied after the recall instead of
before it, or a transposed state breaks at least one of them.
"""
import numpy as np
import pytest

import oracle
import synth


def closed_form(S, q, k, v, alpha, beta):
    """S' and o from the matrix form of the gated delta rule, per head."""
    S, q, k, v = (np.asarray(a, dtype=np.float64) for a in (S, q, k, v))
    alpha, beta = np.asarray(alpha, dtype=np.float64), np.asarray(beta, dtype=np.float64)
    nh, dv, dk = S.shape
    S2 = np.empty_like(S)
    o = np.empty((nh, dv))
    for h in range(nh):
        kk = k[h][:, None]
        P = np.eye(dk) - beta[h] * (kk @ kk.T)
        S2[h] = alpha[h] * (S[h] @ P) + beta[h] * np.outer(v[h], k[h])
        o[h] = S2[h] @ q[h]
    return S2, o


def random_case(seed, nh, dk, dv):
    S = synth.host_gdn_state(seed, 0, nh, dk, dv)
    t = synth.host_gdn_token(seed, 0, 0, nh, dk, dv)
    return S, t


@pytest.mark.parametrize("nh,dk,dv", [(1, 2, 2), (3, 5, 7), (4, 16, 8), (2, 128, 128)])
def test_matches_the_closed_matrix_form(nh, dk, dv):
    S, t = random_case(11, nh, dk, dv)
    S1, o1 = oracle.gdn_step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    S2, o2 = closed_form(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    assert np.allclose(S1, S2, rtol=0, atol=1e-13 * max(1.0, np.abs(S2).max()))
    assert np.allclose(o1, o2, rtol=0, atol=1e-12 * max(1.0, np.abs(o2).max()))


def test_worked_2x2_example():
    # S = [[1,2],[3,4]], k = e1, q = e2, v = (5,6), alpha = beta = 1/2, by hand:
    #   alpha S = [[.5,1],[1.5,2]]; recall at k = (.5,1.5); correction
    #   beta (v - recall) = (2.25, 2.25) written along e1:
    #   S' = [[2.75,1],[3.75,2]]; o = S' e2 = (1, 2).
    S = np.array([[[1.0, 2.0], [3.0, 4.0]]])
    S1, o = oracle.gdn_step(S, [[0.0, 1.0]], [[1.0, 0.0]], [[5.0, 6.0]], [0.5], [0.5])
    assert np.array_equal(S1[0], np.array([[2.75, 1.0], [3.75, 2.0]]))
    assert np.array_equal(o[0], np.array([1.0, 2.0]))
    assert np.array_equal(S[0], np.array([[1.0, 2.0], [3.0, 4.0]]))  # input untouched


def test_no_write_only_decays():
    S, t = random_case(12, 3, 32, 16)
    beta0 = np.zeros(3)
    S1, o = oracle.gdn_step(S, t["q"], t["k"], t["v"], t["alpha"], beta0)
    for h in range(3):
        assert np.array_equal(S1[h], t["alpha"][h].astype(np.float64) * S[h].astype(np.float64))
        assert np.allclose(o[h], S1[h] @ t["q"][h].astype(np.float64), rtol=1e-14, atol=1e-15)


def test_full_forgetting_leaves_the_outer_product():
    S, t = random_case(13, 2, 24, 20)
    S1, o = oracle.gdn_step(S, t["q"], t["k"], t["v"], np.zeros(2), t["beta"])
    for h in range(2):
        expect = t["beta"][h].astype(np.float64) * np.outer(t["v"][h].astype(np.float64),
                                                            t["k"][h].astype(np.float64))
        assert np.array_equal(S1[h], expect)
        # o = beta v (k . q)
        kq = float(np.dot(t["k"][h].astype(np.float64), t["q"][h].astype(np.float64)))
        assert np.allclose(o[h], t["beta"][h] * t["v"][h].astype(np.float64) * kq, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("alpha", [1.0, 0.93])
def test_full_write_recalls_the_value_at_its_key(alpha):
    # beta = 1 and |k| = 1: S' k = alpha S k + (v - alpha S k) = v, whatever S
    # was; reading with q = k returns v.
    nh, dk, dv = 4, 64, 48
    S, t = random_case(14, nh, dk, dv)
    k = t["k"].astype(np.float64)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    S1, o = oracle.gdn_step(S, k, k, t["v"], np.full(nh, alpha), np.ones(nh))
    for h in range(nh):
        assert np.allclose(S1[h] @ k[h], t["v"][h], rtol=0, atol=1e-13)
        assert np.allclose(o[h], t["v"][h], rtol=0, atol=1e-13)


def test_orthonormal_keys_make_an_exact_associative_memory():
    # from a zero state, full-strength writes (alpha = beta = 1) at orthonormal
    # keys k_1..k_n leave S = sum_j v_j k_j^T, so S k_j = v_j for every j
    rng = np.random.default_rng(5)
    dk, dv, n = 16, 9, 6
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Q[:, :n].T
    vals = rng.standard_normal((n, dv))
    S = np.zeros((1, dv, dk))
    for j in range(n):
        S, _ = oracle.gdn_step(S, keys[j:j + 1], keys[j:j + 1], vals[j:j + 1], [1.0], [1.0])
    assert np.allclose(S[0], vals.T @ keys, atol=1e-13)
    for j in range(n):
        assert np.allclose(S[0] @ keys[j], vals[j], atol=1e-13)


def test_heads_are_independent():
    S, t = random_case(15, 5, 12, 10)
    perm = np.array([3, 0, 4, 1, 2])
    S1, o1 = oracle.gdn_step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    S2, o2 = oracle.gdn_step(S[perm], t["q"][perm], t["k"][perm], t["v"][perm], t["alpha"][perm],
                             t["beta"][perm])
    assert np.array_equal(S2, S1[perm]) and np.array_equal(o2, o1[perm])


def test_no_write_never_grows_the_state():
    # v = 0, |k| = 1, beta in [0, 1], |alpha| <= 1: S' = alpha S (I - beta k k^T)
    # and I - beta k k^T has spectral norm 1, so every row's norm can only shrink
    S, t = random_case(16, 3, 40, 30)
    k = t["k"].astype(np.float64)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    S1, _ = oracle.gdn_step(S, t["q"], k, np.zeros((3, 30)), t["alpha"], t["beta"])
    rows0 = np.linalg.norm(S.astype(np.float64), axis=2)
    rows1 = np.linalg.norm(S1, axis=2)
    assert np.all(rows1 <= rows0 * (1 + 1e-14))
    # and the component along k shrinks by the factor alpha (1 - beta)
    for h in range(3):
        along0 = S[h].astype(np.float64) @ k[h]
        along1 = S1[h] @ k[h]
        assert np.allclose(along1, t["alpha"][h] * (1 - t["beta"][h]) * along0, rtol=1e-12, atol=1e-15)


def test_recurrence_over_tokens_matches_the_unrolled_closed_form():
    # three tokens through the oracle equal three applications of the matrix form
    nh, dk, dv = 2, 8, 6
    S = synth.host_gdn_state(17, 0, nh, dk, dv).astype(np.float64)
    Sa, Sb = S.copy(), S.copy()
    for tok in range(3):
        t = synth.host_gdn_token(17, 0, tok, nh, dk, dv)
        Sa, oa = oracle.gdn_step(Sa, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
        Sb, ob = closed_form(Sb, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
        assert np.allclose(oa, ob, atol=1e-13)
    assert np.allclose(Sa, Sb, atol=1e-13)


def test_generator_draws_unit_keys_and_bounded_gates():
    t = synth.host_gdn_token(3, 2, 9, 64, 128, 128)
    for name in ("q", "k"):
        n = np.linalg.norm(t[name].astype(np.float64), axis=1)
        assert np.all(np.abs(n - 1) < 1e-6)
    assert np.all((t["alpha"] >= 0.9) & (t["alpha"] <= 1.0))
    assert np.all((t["beta"] >= 0.0) & (t["beta"] <= 1.0))
    assert t["v"].dtype == np.float32 and t["v"].shape == (64, 128)
