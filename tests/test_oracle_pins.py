"""The fp64 oracle pinned to what the pages and the mathematics fix.

None of these tests compares the oracle with itself: every expected value is
either the target's own distribution (lossless-ness), a closed form, a
library routine on a special case (scipy softmax, numpy argmax decoding),
brute-force enumeration, or a hand-worked fixture under ``tests/golden/``.
"""
import json
import os

import numpy as np
import pytest
from scipy import special

import oracle
import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- lossless, exact

@pytest.mark.parametrize("V,gamma,K,seed,kind,T", [
    (3, 2, 3, 1, "probs", 1.0),
    (3, 2, 3, 11, "logits", 1.0),
    (4, 3, 2, 21, "probs", 0.6),
    (3, 2, 3, 31, "logits", 0.7),
    (2, 4, 3, 41, "probs", 1.3),
    (4, 1, 2, 51, "logits", 2.0),
])
def test_chain_bruteforce_lossless(V, gamma, K, seed, kind, T):
    r = pins.chain_bruteforce(V=V, gamma=gamma, K=K, seed=seed, draft_kind=kind, T=T)
    assert r["ok"], r


@pytest.mark.parametrize("parents,V,K,seed,T,zeros", [
    ((-1, 0, 0, 1, 1, 2, 3), 3, 3, 5, 1.0, False),
    ((-1, 0, 0, 1, 1, 2, 3), 3, 3, 8, 0.8, True),
    ((-1, 0, 1, 2), 4, 2, 15, 1.0, False),            # chain-shaped tree
    ((-1, 0, 0, 0, 1, 1, 2), 4, 2, 25, 1.5, False),   # wide root
    ((-1,), 3, 2, 35, 1.0, False),                     # root only: plain sampling
])
def test_tree_bruteforce_lossless(parents, V, K, seed, T, zeros):
    r = pins.tree_bruteforce(V=V, K=K, seed=seed, parents=parents, T=T, draft_probs_zero=zeros)
    assert r["ok"], r


@pytest.mark.parametrize("parents,V,K,seed,T", [
    ((-1, 0, 0, 0, 1, 1), 3, 3, 5, 1.0),
    ((-1, 0, 0, 1, 2, 2), 3, 2, 7, 0.7),
    ((-1, 0, 0, 0, 1, 1), 4, 2, 3, 1.0),              # three siblings, V=4: second residuals matter
    ((-1, 0, 1, 2), 4, 2, 9, 1.3),                     # chain-shaped tree
    ((-1,), 3, 2, 35, 1.0),                            # root only: plain sampling
])
def test_tree_mss_bruteforce_lossless(parents, V, K, seed, T):
    """Multi-step speculative sampling with the children drawn from q keeps the
    target distribution exactly ([origins] "SpecInfer", MSS bullet)."""
    r = pins.tree_mss_bruteforce(V=V, K=K, seed=seed, parents=parents, T=T)
    assert r["ok"], r


# ----------------------------------------------------------------------------- top-k / top-p

def test_filter_properties():
    """The oracle's top-k / top-p filter satisfies the defining properties on
    random rows with ties, signed zeros and -inf entries."""
    r = pins.filter_properties(trials=600)
    assert r["ok"], r


def test_filter_special_cases():
    l = np.array([0.5, 2.0, -1.0, 1.5, 2.0, 0.0], np.float32)
    base = special.softmax(l.astype(np.float64) / float(np.float32(0.8)))   # T is taken as its f32 value
    p, m = oracle.filter_row(l, 0.8, 0, 1.0)
    np.testing.assert_allclose(p, base, rtol=0, atol=1e-15)          # both off: the softmax
    p, m = oracle.filter_row(l, 0.8, len(l) + 5, 1.0)
    np.testing.assert_allclose(p, base, rtol=0, atol=1e-15)          # top_k >= V: off
    p, m = oracle.filter_row(l, 0.8, 1, 1.0)
    np.testing.assert_allclose(p, [0, 0.5, 0, 0, 0.5, 0], atol=1e-15)   # top-1 keeps both tied maxima
    p, m = oracle.filter_row(l, 0.8, 0, 1e-6)
    np.testing.assert_allclose(p, [0, 0.5, 0, 0, 0.5, 0], atol=1e-15)   # tiny top_p: the top group
    p, m = oracle.filter_row(l, 0.8, 3, 1.0)                          # 2, 2, 1.5
    want = np.where(l >= 1.5, base, 0)
    np.testing.assert_allclose(p, want / want.sum(), atol=1e-15)
    assert oracle.filter_row(l, 0.8, -1, 1.0) is None
    assert oracle.filter_row(l, 0.8, 0, 0.0) is None
    assert oracle.filter_row(l, 0.8, 0, 1.5) is None


def test_chain_filter_off_is_plain_chain():
    """top_k = 0 and top_p = 1 for every sequence: the filtered chain equals the
    plain chain bit for bit."""
    rng = np.random.default_rng(31)
    B, gamma, V = 40, 3, 50
    t = rng.normal(0, 2, (B, gamma + 1, V)).astype(np.float32)
    d = rng.normal(0, 2, (B, gamma, V)).astype(np.float32)
    x = rng.integers(0, V, (B, gamma)).astype(np.int32)
    T = np.full(B, 0.9, np.float32)
    c = rng.random((B, gamma)).astype(np.float32)
    u = rng.random(B).astype(np.float32)
    a = oracle.chain(t, d, False, x, T, c, u)
    b = oracle.chain(t, d, False, x, T, c, u, top_k=np.zeros(B, np.int32), top_p=np.ones(B, np.float32))
    for key in ("tokens", "num_accepted", "px", "qx", "S"):
        np.testing.assert_array_equal(a[key], b[key])


@pytest.mark.parametrize("kw", [
    dict(),
    dict(draft_kind="probs", seed=2, top_k=2, top_p=0.9, tol=1e-7),   # filtered q rounded to f32
    dict(V=4, gamma=2, seed=5, T=0.7, top_k=0, top_p=0.61),
    dict(V=5, gamma=1, seed=6, top_k=2, top_p=1.0),
    dict(V=3, gamma=3, K=3, seed=8, top_k=2, top_p=0.77),
])
def test_chain_filtered_bruteforce_lossless(kw):
    """The rules keep the (filtered) target distribution exactly."""
    r = pins.chain_filtered_bruteforce(**kw)
    assert r["ok"], r


# ----------------------------------------------------------------------------- closed form

@pytest.mark.parametrize("seed,kind", [(2, "probs"), (3, "logits"), (12, "probs")])
def test_closed_form_exact(seed, kind):
    r = pins.chain_closed_form_exact(seed=seed, draft_kind=kind)
    assert r["ok"], r


@pytest.mark.parametrize("seed,kind", [(9, "probs"), (10, "logits")])
def test_closed_form_positional(seed, kind):
    r = pins.chain_closed_form_positional(seed=seed, draft_kind=kind)
    assert r["ok"], r


def test_closed_form_monte_carlo():
    r = pins.chain_closed_form_mc(rounds=1_000_000)
    assert r["ok"], r


# ----------------------------------------------------------------------------- chi-square

@pytest.mark.parametrize("seed,kind,T", [(3, "probs", 1.0), (13, "logits", 1.0), (23, "logits", 0.6)])
def test_chain_chisquare(seed, kind, T):
    r = pins.chain_chisquare(rounds=1_000_000, seed=seed, draft_kind=kind, T=T)
    assert r["ok"], r


@pytest.mark.parametrize("seed", [6, 16])
def test_tree_chisquare(seed):
    r = pins.tree_chisquare(rounds=1_000_000, seed=seed)
    assert r["ok"], r


@pytest.mark.parametrize("seed", [16, 17])
def test_tree_mss_chisquare(seed):
    r = pins.tree_mss_chisquare(rounds=1_000_000, seed=seed)
    assert r["ok"], r


# ----------------------------------------------------------------------------- greedy

def test_greedy_equals_argmax_decoding():
    r = pins.greedy_equivalence(steps=10_000)
    assert r["ok"], r


def test_greedy_chain_tree_is_prefix_match():
    """On a chain-shaped tree the greedy walk keeps the longest prefix of drafts
    equal to the running argmax (Blockwise verify) and appends the argmax after it."""
    rng = np.random.default_rng(0)
    for _ in range(200):
        V, N = int(rng.integers(2, 9)), int(rng.integers(1, 8))
        vals = rng.integers(0, 3, (N, V)).astype(np.float32)
        bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
        am = vals.argmax(axis=1)
        tokens = np.zeros(N, np.int32)
        for n in range(1, N):
            tokens[n] = am[n - 1] if rng.random() < 0.7 else rng.integers(V)
        parents = np.arange(-1, N - 1, dtype=np.int32)
        res = oracle.tree_greedy(bits[None], tokens[None], parents[None], max(N - 1, 0))
        k = 0
        while k + 1 < N and tokens[k + 1] == am[k]:
            k += 1
        assert res["num_accepted"][0] == k
        assert list(res["tokens"][0, :k + 1]) == list(tokens[1:k + 1]) + [am[k]]
        assert list(res["accept_index"][0, :k + 1]) == list(range(k + 1))


# ----------------------------------------------------------------------------- special cases

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [0.6, 1.0, 2.5])
def test_softmax_is_scipy_softmax(dtype, T):
    rng = np.random.default_rng(1)
    x = (rng.normal(0, 3, 257)).astype(np.float32)
    x[5] = -np.inf
    if dtype == "bf16":
        row = (x.view(np.uint32) >> 16).astype(np.uint16)
        xv = (row.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    else:
        row, xv = x, x.astype(np.float64)
    p = oracle.softmax_row(row, T)
    want = special.softmax(xv / np.float64(np.float32(T)))
    np.testing.assert_allclose(p, want, rtol=1e-13, atol=0)
    assert p[5] == 0.0


def test_softmax_rejects_bad_rows():
    assert oracle.softmax_row(np.array([0.0, np.nan], np.float32), 1.0) is None
    assert oracle.softmax_row(np.array([0.0, np.inf], np.float32), 1.0) is None
    assert oracle.softmax_row(np.array([-np.inf, -np.inf], np.float32), 1.0) is None


def test_inverse_cdf_cells():
    w = np.array([0.0, 1.0, 0.0, 3.0, 0.0])
    assert oracle.inverse_cdf(w, 0.0)[0] == 1
    assert oracle.inverse_cdf(w, 0.2499999)[0] == 1
    assert oracle.inverse_cdf(w, 0.25)[0] == 3          # boundary belongs to the next cell
    assert oracle.inverse_cdf(w, 1 - 2 ** -24)[0] == 3
    j, S, m = oracle.inverse_cdf(w, 0.125)
    assert (j, S) == (1, 4.0) and m == pytest.approx(0.125)
    assert oracle.inverse_cdf(np.zeros(4), 0.5)[0] == -1


def test_golden_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_v3.json")))
    p, q = np.array(g["p"]), np.array(g["q"])
    tl = np.log(p).astype(np.float32)
    # accept probability of every token = measure of coins that accept it
    for x in range(3):
        a = g["accept_prob"][x]
        for u, want in [(a - 1e-6, 1), (min(a + 1e-6, 1 - 2 ** -24), 0 if a < 1 else 1)]:
            r = oracle.chain(tl[None, None].repeat(2, 1), q.astype(np.float32)[None, None], True,
                             np.array([[x]]), np.ones(1), np.array([[u]]), np.array([0.5]))
            assert r["num_accepted"][0] == want, (x, u)
            assert r["px"][0, 0] == pytest.approx(p[x], rel=1e-6)
            assert r["qx"][0, 0] == pytest.approx(q[x], rel=1e-12)
            if want == 0:
                # the residual puts all mass on token 0
                assert r["tokens"][0, 0] == int(np.argmax(g["residual"]))
                assert r["S"][0] == pytest.approx(g["residual_weights"][0], rel=1e-6)
    # exact output distribution and E[tau] by enumeration for gamma = 1..3
    model = pins.ToyModel(3, 0, "probs", iid=True)
    model._p[()] = (tl, p)
    model._q[()] = (q.astype(np.float32), q)
    for gamma in (1, 2, 3):
        cases = pins._chain_cases(model, (), gamma)
        res = pins._run_chain_cases(model, cases)
        w = np.array([c["weight"] for c in cases])
        e_tau = float((w * (res["num_accepted"] + 1.0)).sum())
        assert e_tau == pytest.approx(g["expected_tokens_per_round"][str(gamma)], abs=1e-12)
        first = np.zeros(3)
        for i in range(len(cases)):
            first[res["tokens"][i, 0]] += w[i]
        np.testing.assert_allclose(first, g["emit_prob_first_token"], atol=1e-12)
    # tree: root with children tokens 0, 1
    tokens = np.array([[0, 0, 1]], np.int32)
    parents = np.array([[-1, 0, 0]], np.int32)
    rows = np.stack([tl, tl, tl])[None]
    for lo, hi, what in g["tree_coin_cells"]:
        u = (lo + hi) / 2
        r = oracle.tree_sample(rows, tokens, parents, np.ones(1), np.array([[u, 0.5, 0.5]]),
                               np.array([0.5]), 1)
        if "reject" in what:
            assert r["num_accepted"][0] == 0
            assert r["tokens"][0, 0] == int(np.argmax(g["tree_final_after_rejecting_0_and_1"]))
        else:
            assert r["num_accepted"][0] == 1 and r["tokens"][0, 0] == int(what.split()[-1])


def test_invariant_q_equals_p_accepts_all():
    rng = np.random.default_rng(2)
    B, gamma, V = 64, 5, 50
    t = rng.normal(0, 3, (B, gamma + 1, V)).astype(np.float32)
    x = rng.integers(0, V, (B, gamma)).astype(np.int32)
    u = (rng.integers(0, 1 << 24, (B, gamma)) * 2.0 ** -24).astype(np.float32)
    r = oracle.chain(t, t[:, :gamma].copy(), False, x, np.full(B, 0.7), u, u[:, 0].copy())
    assert (r["num_accepted"] == gamma).all()
    assert (r["tokens"][:, :gamma] == x).all()


def test_invariant_onehot_accepts_and_is_deterministic():
    V, gamma = 7, 3
    t = np.full((1, gamma + 1, V), -np.inf, np.float32)
    x = np.array([[2, 5, 1]], np.int32)
    for i in range(gamma):
        t[0, i, x[0, i]] = 0.0
    t[0, gamma, 4] = 0.0
    q = np.zeros((1, gamma, V), np.float32)
    for i in range(gamma):
        q[0, i, x[0, i]] = 1.0
    r = oracle.chain(t, q, True, x, np.ones(1), np.full((1, gamma), 1 - 2 ** -24), np.array([0.9]))
    assert r["num_accepted"][0] == gamma
    assert list(r["tokens"][0]) == [2, 5, 1, 4]


def test_invariant_tau_at_least_one():
    rng = np.random.default_rng(3)
    B, gamma, V = 500, 4, 30
    t = rng.normal(0, 3, (B, gamma + 1, V)).astype(np.float32)
    d = rng.normal(0, 3, (B, gamma, V)).astype(np.float32)
    x = rng.integers(0, V, (B, gamma)).astype(np.int32)
    u = rng.random((B, gamma)).astype(np.float32)
    r = oracle.chain(t, d, False, x, np.ones(B), u, rng.random(B).astype(np.float32))
    k = r["num_accepted"]
    assert (k >= 0).all()
    for b in range(B):
        assert (r["tokens"][b, :k[b]] == x[b, :k[b]]).all()
        assert 0 <= r["tokens"][b, k[b]] < V
        assert (r["tokens"][b, k[b] + 1:] == -1).all()


def test_cross_identity_tree_chain_onehot():
    """Target-only tree on a chain-shaped tree == chain verify with one-hot draft
    probabilities: both accept iff coin <= p(x), both draw the residual from p
    with x removed, both draw the bonus from p at the end."""
    rng = np.random.default_rng(4)
    for trial in range(300):
        V = int(rng.integers(2, 40))
        gamma = int(rng.integers(1, 7))
        T = float(rng.choice([0.5, 1.0, 1.7]))
        t = (rng.normal(0, 2, (1, gamma + 1, V))).astype(np.float32)
        x = rng.integers(0, V, (1, gamma)).astype(np.int32)
        q = np.zeros((1, gamma, V), np.float32)
        q[0, np.arange(gamma), x[0]] = 1.0
        coins = (rng.integers(0, 1 << 24, (1, gamma)) * 2.0 ** -24).astype(np.float32)
        # make acceptance likely enough to reach the bonus now and then
        coins *= np.float32(rng.choice([1.0, 0.01]))
        fu = rng.random(1).astype(np.float32)
        rc = oracle.chain(t, q, True, x, np.array([T]), coins, fu)
        tokens = np.concatenate([[0], x[0]]).astype(np.int32)[None]
        parents = np.arange(-1, gamma, dtype=np.int32)[None]
        tc = np.concatenate([coins[0], [0.5]]).astype(np.float32)[None]
        rt = oracle.tree_sample(t, tokens, parents, np.array([T]), tc, fu, gamma)
        assert rc["num_accepted"][0] == rt["num_accepted"][0], trial
        k = rc["num_accepted"][0]
        assert list(rc["tokens"][0, :k + 1]) == list(rt["tokens"][0, :k + 1]), trial


def test_cross_identity_mss_chain_tree_equals_chain():
    """Multi-step speculative sampling on a chain-shaped tree is chain verify with
    draft probabilities: one child per node, so the rejection of that child is
    rule 2 (draw from norm(max(0, p - q))) and reaching the leaf is rule 3."""
    rng = np.random.default_rng(14)
    for trial in range(300):
        V = int(rng.integers(2, 40))
        gamma = int(rng.integers(1, 7))
        T = float(rng.choice([0.5, 1.0, 1.7]))
        t = rng.normal(0, 2, (1, gamma + 1, V)).astype(np.float32)
        q = special.softmax(rng.normal(0, 2, (1, gamma, V)), axis=-1).astype(np.float32)
        x = np.array([[rng.choice(V, p=q[0, i] / q[0, i].sum()) for i in range(gamma)]], np.int32)
        coins = (rng.integers(0, 1 << 24, (1, gamma)) * 2.0 ** -24).astype(np.float32)
        fu = rng.random(1).astype(np.float32)
        rc = oracle.chain(t, q, True, x, np.array([T]), coins, fu)
        tokens = np.concatenate([[0], x[0]]).astype(np.int32)[None]
        parents = np.arange(-1, gamma, dtype=np.int32)[None]
        tc = np.concatenate([[0.5], coins[0]]).astype(np.float32)[None]     # coin of child n = coins[n-1]
        qt = np.concatenate([q, np.full((1, 1, V), 1.0 / V, np.float32)], axis=1)
        rt = oracle.tree_mss(t, tokens, parents, np.array([T]), tc, fu, gamma, qt)
        if min(rc["dmargin"][0], rt["dmargin"][0], rc["cmargin"][0], rt["cmargin"][0]) < 1e-9:
            continue
        assert rc["num_accepted"][0] == rt["num_accepted"][0], trial
        k = rc["num_accepted"][0]
        assert list(rc["tokens"][0, :k + 1]) == list(rt["tokens"][0, :k + 1]), trial
        if k < gamma:
            assert abs(rc["S"][0] - rt["S"][0]) <= 1e-12 * max(1.0, rc["S"][0]), trial


def test_mss_invalid_inputs_and_diagnostics():
    rng = np.random.default_rng(15)
    V, N = 12, 4
    t = rng.normal(0, 1, (4, N, V)).astype(np.float32)
    q = special.softmax(rng.normal(0, 1, (4, N, V)), axis=-1).astype(np.float32)
    tok = np.array([[0, 3, 5, 7]] * 4, np.int32)
    par = np.array([[-1, 0, 0, 1]] * 4, np.int32)
    T = np.array([1.0, np.nan, 1.0, 1.0], np.float32)
    par[2, 2] = 3                                          # parent after child
    q[3, 0, 3] = -0.5                                      # a drafted token's q(x) < 0
    coins = np.full((4, N), 0.999, np.float32)             # reject every child
    r = oracle.tree_mss(t, tok, par, T, coins, np.full(4, 0.5, np.float32), 2, q)
    assert list(r["num_accepted"]) == [0, -1, -1, -1]
    assert (r["tokens"][1:] == -1).all() and np.isnan(r["ptest"][1:]).all()
    # sequence 0: both root children tested (p(x) recorded), node 3 never tested
    p0 = special.softmax(t[0, 0].astype(np.float64))
    assert abs(r["ptest"][0, 1] - p0[3]) < 1e-12
    p1 = np.maximum(0, p0 - q[0, 0].astype(np.float64))
    p1 /= p1.sum()
    assert abs(r["ptest"][0, 2] - p1[5]) < 1e-12
    assert np.isnan(r["ptest"][0, 3]) and np.isnan(r["ptest"][0, 0])


def test_thresholds_literal():
    """threshold_single = 0 accepts the first child at every level (p >= 0);
    a tiny threshold_acc accepts the first child with positive probability."""
    rng = np.random.default_rng(5)
    V = 9
    parents = np.array([[-1, 0, 0, 1, 1, 3]], np.int32)
    tokens = np.array([[0, 3, 4, 1, 2, 7]], np.int32)
    t = rng.normal(0, 2, (1, 6, V)).astype(np.float32)
    coins = np.full((1, 6), 0.999, np.float32)
    r = oracle.tree_sample(t, tokens, parents, np.ones(1), coins, np.array([0.3]), 3,
                           threshold_single=0.0)
    assert list(r["accept_index"][0, :4]) == [0, 1, 3, 5]
    r = oracle.tree_sample(t, tokens, parents, np.ones(1), coins, np.array([0.3]), 3,
                           threshold_acc=1e-30)
    assert list(r["accept_index"][0, :4]) == [0, 1, 3, 5]
    r = oracle.tree_sample(t, tokens, parents, np.ones(1), coins, np.array([0.3]), 3)
    assert r["num_accepted"][0] == 0                      # coin 0.999 rejects both children


def test_invalid_inputs_mark_sequence():
    V, gamma = 10, 2
    rng = np.random.default_rng(6)
    t = rng.normal(0, 1, (4, gamma + 1, V)).astype(np.float32)
    d = rng.normal(0, 1, (4, gamma, V)).astype(np.float32)
    x = np.array([[1, 2], [1, V], [1, 2], [1, 2]], np.int32)
    T = np.array([1.0, 1.0, 0.0, 1.0], np.float32)
    t[3, 2, 4] = np.nan                                   # NaN in a row after the drafts
    r = oracle.chain(t, d, False, x, T, np.full((4, gamma), 0.5, np.float32), np.full(4, 0.5, np.float32))
    assert list(r["num_accepted"][1:]) == [-1, -1, -1]
    assert (r["tokens"][1:] == -1).all()
    assert r["num_accepted"][0] >= 0
    # malformed trees
    tt = rng.normal(0, 1, (3, 3, V)).astype(np.float32)
    tok = np.array([[0, 1, 2]] * 3, np.int32)
    par = np.array([[-1, 0, 0], [-1, 2, 0], [0, 0, 0]], np.int32)
    g = oracle.tree_greedy(tt, tok, par, 2)
    assert list(g["num_accepted"]) [1:] == [-1, -1] and g["num_accepted"][0] >= 0
    g = oracle.tree_greedy(tt, tok, np.array([[-1, 0, 1]] * 3, np.int32), 1)   # too deep
    assert (g["num_accepted"] == -1).all()


# ----------------------------------------------------------------------------- filtered tree sampling

def test_tree_filter_off_is_plain_tree():
    """Target-only tree sampling with both filters off (top_k 0, top_p 1) is the
    unfiltered walk bit for bit, with and without draft probabilities."""
    rng = np.random.default_rng(21)
    B, V = 6, 40
    parents = np.array([[-1, 0, 0, 1, 1, 2, 4, 4]] * B, np.int32)
    N = parents.shape[1]
    tokens = rng.integers(0, V, (B, N)).astype(np.int32)
    t = rng.normal(0, 2, (B, N, V)).astype(np.float32)
    coins = pins._uniform24(rng, (B, N))
    fu = pins._uniform24(rng, (B,))
    T = np.full(B, 0.8, np.float32)
    for dp in (None, rng.dirichlet(np.ones(V), (B, N)).astype(np.float32)):
        a = oracle.tree_sample(t, tokens, parents, T, coins, fu, 3, draft_probs=dp)
        b = oracle.tree_sample(t, tokens, parents, T, coins, fu, 3, draft_probs=dp,
                               top_k=np.zeros(B, np.int32), top_p=np.ones(B, np.float32))
        for key in ("accept_index", "tokens", "num_accepted", "pchild", "S"):
            np.testing.assert_array_equal(a[key], b[key])


@pytest.mark.parametrize("kw", [
    dict(top_k=2, top_p=None),
    dict(top_k=None, top_p=0.7),
    dict(top_k=3, top_p=0.8, V=4, K=2, seed=3, parents=(-1, 0, 0, 1, 2)),
    dict(top_k=2, top_p=0.9, T=0.7, seed=8, draft_probs_zero=True),
])
def test_tree_filtered_bruteforce_lossless(kw):
    """Filtered target-only tree rounds emit the filtered target's
    autoregressive distribution exactly ([origins] "In SGLang": the walk keeps
    whatever target distribution it is given; the filters follow the
    threshold-form definition written separately in the harness)."""
    r = pins.tree_bruteforce(**kw)
    assert r["ok"], (kw, r)


def test_tree_topk1_sampling_is_greedy():
    """top_k = 1 on rows without ties makes every filtered row one-hot at its
    argmax: a child is accepted iff it carries its parent's argmax, and the last
    token is the argmax, which is greedy tree verification."""
    rng = np.random.default_rng(22)
    B, V = 40, 12
    parents = np.array([[-1, 0, 0, 0, 1, 1, 2, 3, 5, 5]] * B, np.int32)
    N = parents.shape[1]
    t = rng.normal(0, 2, (B, N, V)).astype(np.float32)             # continuous: no ties
    am = t.argmax(axis=2)
    tokens = rng.integers(0, V, (B, N)).astype(np.int32)
    hit = rng.random((B, N)) < 0.6                                   # many children match their parent's argmax
    for n in range(1, N):
        tokens[hit[:, n], n] = am[hit[:, n], parents[0, n]]
    g = oracle.tree_greedy(t, tokens, parents, 3)
    s = oracle.tree_sample(t, tokens, parents, np.full(B, 0.9, np.float32), pins._uniform24(rng, (B, N)),
                           pins._uniform24(rng, (B,)), 3, top_k=np.ones(B, np.int32))
    np.testing.assert_array_equal(s["num_accepted"], g["num_accepted"])
    np.testing.assert_array_equal(s["accept_index"], g["accept_index"])
    np.testing.assert_array_equal(s["tokens"], g["tokens"])


def test_tree_margin_of_two_condition_acceptance():
    """A child is accepted when coin <= prob_acc/theta_acc or p >= theta_single.
    An acceptance flips only if every condition that holds can flip: p = 1 exactly
    at theta_single = 1 with a coin far below 1 is not a near-tie; a rejection
    with the coin just above prob_acc is."""
    V = 6
    parents = np.array([[-1, 0]], np.int32)
    t = np.full((1, 2, V), -np.inf, np.float32)
    t[0, 0, 3] = 0.0                                      # the root row keeps one token: p = 1 exactly
    t[0, 1, :] = 0.0
    tokens = np.array([[0, 3]], np.int32)
    r = oracle.tree_sample(t, tokens, parents, np.ones(1, np.float32), np.array([[0.25, 0.5]], np.float32),
                           np.array([0.5], np.float32), 1)
    assert r["num_accepted"][0] == 1 and r["pchild"][0, 1] == 1.0
    assert r["dmargin"][0] >= 0.5                         # the coin settles it: 1 - 0.25
    t2 = np.zeros((1, 2, V), np.float32)                  # uniform root row: p = 1/6 for every token
    c = np.float32(1.0 / 6.0) + np.float32(2 ** -24)
    r2 = oracle.tree_sample(t2, tokens, parents, np.ones(1, np.float32), np.array([[c, 0.5]], np.float32),
                            np.array([0.5], np.float32), 1)
    assert r2["num_accepted"][0] == 0                     # coin just above prob_acc: rejected
    assert r2["dmargin"][0] < 1e-6                        # and flagged as a near-tie


# ----------------------------------------------------------------------------- the pins bite

MUTATIONS = {
    1: ("p and q swapped in the ratio", lambda: pins.chain_bruteforce()),
    2: ("max(0, .) dropped from the residual", lambda: pins.chain_bruteforce()),
    3: ("residual taken as max(0, q - p)", lambda: pins.chain_bruteforce()),
    4: ("every position uses coin 0", lambda: pins.chain_bruteforce()),
    5: ("inverse CDF off by one cell", lambda: pins.chain_bruteforce()),
    6: ("bonus drawn from p_{gamma-1}", lambda: pins.chain_bruteforce()),
    7: ("argmax ties go to the last index", lambda: pins.greedy_equivalence(steps=3000)),
    8: ("tree walk reuses the root's coin", lambda: pins.tree_bruteforce()),
    9: ("prob_acc not accumulated", lambda: pins.tree_bruteforce()),
    10: ("rejected children not removed", lambda: pins.tree_bruteforce()),
    11: ("logits multiplied by T", lambda: pins.chain_bruteforce(T=0.6)),
    12: ("draft logits without T", lambda: pins.chain_bruteforce(draft_kind="logits", seed=11, T=0.7)),
    13: ("MSS: p not replaced by the residual after a rejection", lambda: pins.tree_mss_bruteforce()),
    14: ("MSS: every residual taken from the node's first p",
         lambda: pins.tree_mss_bruteforce(V=4, K=2, seed=3, parents=(-1, 0, 0, 0, 1, 1))),
    15: ("MSS: children tested with their parent's coin", lambda: pins.tree_mss_bruteforce()),
    16: ("top-k keeps one group too few", lambda: pins.filter_properties()),
    17: ("top-p drops the group that reaches top_p", lambda: pins.filter_properties()),
    18: ("draft logits left unfiltered", lambda: pins.chain_filtered_bruteforce()),
    19: ("tree rows left unfiltered", lambda: pins.tree_bruteforce(V=4, K=2, seed=3, top_k=2, top_p=0.8,
                                                                    parents=(-1, 0, 0, 1, 2))),
}


@pytest.mark.parametrize("m", sorted(MUTATIONS))
def test_planted_mistake_is_caught(m):
    what, check = MUTATIONS[m]
    oracle.set_mutation(m)
    try:
        r = check()
    finally:
        oracle.set_mutation(0)
    assert not r["ok"], f"pin missed planted mistake {m}: {what}"
