"""Pins for the oracle: each test checks it against something other than itself.

- page-printed numbers (tests/golden/page_numbers.json, each with its source),
- closed forms (binomial counts, hockey-stick sum, multinomial theorem, the
  page's total-cost formulas),
- brute force over the full tensor power (tiny d),
- exact integer identities,
- special cases with a textbook answer (P = 1 running mean, P = 2 linear
  attention written as prefix sums, d_K = 1),
- the softmax limit as P grows, within the Taylor remainder bound.

A plausible slip in the oracle (a dropped term, a wrong sign, an index or
coefficient error, a transposed operand, an off-by-one in the causal range)
fails at least one of these.
"""
import itertools
import json
import math
import os
from collections import Counter
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- basis ----

@pytest.mark.parametrize("d", [1, 2, 3, 5, 8, 13, 16])
@pytest.mark.parametrize("P", [1, 2, 3, 4, 5])
def test_basis_sizes_are_binomials(oracle_mod, d, P):
    deg, M, C, off = oracle_mod.basis(d, P)
    for p in range(P):
        assert off[p + 1] - off[p] == math.comb(d + p - 1, p)
    # hockey stick: sum_{p<P} binom(d+p-1, p) = binom(d+P-1, P-1)
    assert off[P] == math.comb(d + P - 1, P - 1) == len(deg)
    assert np.all(deg[off[0]:off[1]] == 0)


def test_config_feature_counts(oracle_mod, golden):
    g = golden["config_feature_counts"]
    for d, F in g["values"].items():
        assert oracle_mod.num_features(int(d), g["P"]) == F


def test_quoted_basis_and_reduction(oracle_mod, golden):
    full = golden["full_tensor_monomials_d64_p4"]
    assert full["d_K"] ** full["p"] == full["value"]
    q = golden["minimal_basis_quoted_d64"]
    assert oracle_mod.num_features(q["d_K"], q["P"]) == q["value"]
    assert full["value"] / q["value"] > golden["reduction_factor_lower_bound"]["value"]


@pytest.mark.parametrize("d,p", [(1, 3), (2, 2), (2, 4), (3, 3), (4, 3), (5, 2), (5, 4)])
def test_basis_matches_brute_force(oracle_mod, d, p):
    """Sort every one of the d^p full index tuples and count: this is the
    symmetric reduction done by brute force.  The distinct sorted tuples in
    lexicographic order are M_p and their counts are C_p."""
    deg, M, C, off = oracle_mod.basis(d, p + 1)
    counts = Counter(tuple(sorted(t)) for t in itertools.product(range(d), repeat=p))
    want = sorted(counts)
    got = [tuple(int(i) for i in M[r, :p]) for r in range(off[p], off[p + 1])]
    assert got == want
    assert [int(C[r]) for r in range(off[p], off[p + 1])] == [counts[t] for t in want]
    # unused slots are padded
    if p < M.shape[1]:
        assert np.all(M[off[p]:off[p + 1], p:] == -1)


@pytest.mark.parametrize("d", [1, 2, 4, 7, 16, 64])
def test_multiplicities_sum_to_full_count(oracle_mod, d):
    """Multinomial theorem: the multiplicities of degree p add up to d^p."""
    deg, M, C, off = oracle_mod.basis(d, 4)
    for p in range(4):
        assert int(C[off[p]:off[p + 1]].sum()) == d ** p


def test_worked_example_d2_p2(oracle_mod, golden):
    g = golden["worked_example_d2_p2"]
    deg, M, C, off = oracle_mod.basis(g["d_K"], g["p"] + 1)
    p = g["p"]
    rows = [list(map(int, M[r, :p])) for r in range(off[p], off[p + 1])]
    assert rows == g["tuples"]
    assert list(map(int, C[off[p]:off[p + 1]])) == g["multiplicities"]
    assert sum(g["multiplicities"]) == g["full_terms"]


# --------------------------------------------------------- feature map ----

@pytest.mark.parametrize("d", [1, 2, 3, 5, 8])
def test_feature_identity_exact_on_integers(oracle_mod, d):
    """<phi_p(q), phi_p(k)>_C == (q.k)^p exactly: small integer vectors keep
    every float64 product exact, and the check itself runs in Python ints."""
    rng = np.random.default_rng(100 + d)
    P = 5
    deg, M, C, off = oracle_mod.basis(d, P)
    for _ in range(20):
        q = rng.integers(-3, 4, size=d).astype(np.float64)
        k = rng.integers(-3, 4, size=d).astype(np.float64)
        fq = oracle_mod.features(d, P, q)
        fk = oracle_mod.features(d, P, k)
        dot = int(sum(int(a) * int(b) for a, b in zip(q, k)))
        for p in range(P):
            s = sum(int(C[r]) * int(fq[r]) * int(fk[r]) for r in range(off[p], off[p + 1]))
            assert s == dot ** p


@pytest.mark.parametrize("d", [4, 16, 64])
def test_feature_identity_floats(oracle_mod, d):
    rng = np.random.default_rng(7)
    P = 4
    deg, M, C, off = oracle_mod.basis(d, P)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    fq, fk = oracle_mod.features(d, P, q), oracle_mod.features(d, P, k)
    dot = float(q @ k)
    for p in range(P):
        s = float(np.sum(C[off[p]:off[p + 1]] * fq[off[p]:off[p + 1]] * fk[off[p]:off[p + 1]]))
        assert s == pytest.approx(dot ** p, rel=1e-12, abs=1e-12)


def test_features_d1_are_powers(oracle_mod):
    x = 1.7
    f = oracle_mod.features(1, 6, np.array([x]))
    assert np.allclose(f, [x ** p for p in range(6)], rtol=1e-15)
    _, _, C, _ = oracle_mod.basis(1, 6)
    assert np.all(C == 1)


# ------------------------------------------------------------ attention ----

def _inputs(rng, T, dK, dV, scale=1.0):
    return (rng.standard_normal((T, dK)) * scale, rng.standard_normal((T, dK)) * scale,
            rng.standard_normal((T, dV)))


@pytest.mark.parametrize("dK,dV,P,T", [(1, 1, 4, 40), (2, 3, 1, 30), (2, 2, 2, 50), (4, 4, 3, 64),
                                        (8, 8, 4, 64), (3, 5, 5, 33), (8, 4, 4, 17)])
def test_recurrence_equals_direct(oracle_mod, dK, dV, P, T):
    """The state recurrence (update, then normalised readout) equals causal
    attention with the truncated Taylor kernel written out pairwise."""
    rng = np.random.default_rng(dK * 100 + P)
    q, k, v = _inputs(rng, T, dK, dV)
    y, den, S, Z = oracle_mod.scan(q, k, v, P)
    y2, den2, kappa = oracle_mod.direct(q, k, v, P)
    np.testing.assert_allclose(y, y2, rtol=1e-10, atol=1e-10 * np.abs(y2).max())
    np.testing.assert_allclose(den, den2, rtol=1e-10)
    assert np.all(kappa >= 1.0 - 1e-12)


def test_direct_pairwise_weights_by_hand(oracle_mod):
    """Two tokens, numbers small enough to do by hand."""
    q = np.array([[1.0, 0.0], [0.0, 2.0]])
    k = np.array([[2.0, 0.0], [1.0, 1.0]])
    v = np.array([[1.0], [3.0]])
    c = 2.0
    # w_00 = T(1*2/2 = 1) ; w_10 = T(0/2 = 0) = 1 ; w_11 = T(2/2 = 1)
    T3 = lambda x: 1 + x + x * x / 2
    y, den, _ = oracle_mod.direct(q, k, v, P=3, c=c)
    assert y[0, 0] == pytest.approx(1.0)
    assert den[0] == pytest.approx(T3(1.0))
    assert den[1] == pytest.approx(1.0 + T3(1.0))
    assert y[1, 0] == pytest.approx((1.0 * 1 + 3.0 * T3(1.0)) / (1 + T3(1.0)))
    ys, dens, _, _ = oracle_mod.scan(q, k, v, P=3, c=c)
    np.testing.assert_allclose(ys, y, rtol=1e-14)


@pytest.mark.parametrize("dK,dV,P,T", [(2, 3, 4, 40), (8, 8, 4, 64), (3, 5, 2, 33)])
def test_direct_at_selected_tokens(oracle_mod, dK, dV, P, T):
    """direct_at (outputs at chosen tokens only) equals the full direct table at
    those tokens, in any order and with repeats, and the P = 1 running mean at
    selected tokens; an index outside [0, T) is rejected."""
    rng = np.random.default_rng(dK * 10 + P)
    q, k, v = _inputs(rng, T, dK, dV)
    y, den, kappa = oracle_mod.direct(q, k, v, P)
    ts = [T - 1, 0, T // 2, T // 2, 1]
    ya, dena, kappaa = oracle_mod.direct_at(q, k, v, P, ts)
    np.testing.assert_array_equal(ya, y[ts])
    np.testing.assert_array_equal(dena, den[ts])
    np.testing.assert_array_equal(kappaa, kappa[ts])
    y1, _, _ = oracle_mod.direct_at(q, k, v, 1, ts)
    want = (np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None])[ts]
    np.testing.assert_allclose(y1, want, rtol=1e-12)
    with pytest.raises(RuntimeError):
        oracle_mod.direct_at(q, k, v, P, [T])


def test_P1_is_running_mean(oracle_mod):
    rng = np.random.default_rng(1)
    q, k, v = _inputs(rng, 50, 4, 3)
    y, den, _, _ = oracle_mod.scan(q, k, v, P=1)
    want = np.cumsum(v, axis=0) / np.arange(1, 51)[:, None]
    np.testing.assert_allclose(y, want, rtol=1e-12)
    np.testing.assert_allclose(den, np.arange(1, 51), rtol=0)


def test_P2_is_linear_attention(oracle_mod):
    """P = 2: kernel 1 + q.k/c, i.e. linear attention with feature [1, x/sqrt(c)],
    computed here from prefix sums of k and k v^T."""
    rng = np.random.default_rng(2)
    T, dK, dV = 60, 5, 4
    q, k, v = _inputs(rng, T, dK, dV)
    c = math.sqrt(dK)
    ks = np.cumsum(k, axis=0)                                  # [T, dK]
    kv = np.cumsum(k[:, :, None] * v[:, None, :], axis=0)      # [T, dK, dV]
    vs = np.cumsum(v, axis=0)
    num = vs + np.einsum("ti,tij->tj", q, kv) / c
    den = np.arange(1, T + 1) + np.einsum("ti,ti->t", q, ks) / c
    y, d2, _, _ = oracle_mod.scan(q, k, v, P=2)
    np.testing.assert_allclose(y, num / den[:, None], rtol=1e-11)
    np.testing.assert_allclose(d2, den, rtol=1e-12)


def test_dK1_kernel_is_truncated_exp(oracle_mod):
    """d_K = 1: w = sum_{p<P} (q k / c)^p / p!, evaluated with math.factorial."""
    rng = np.random.default_rng(3)
    T, P, c = 20, 6, 1.3
    q, k, v = rng.standard_normal((T, 1)), rng.standard_normal((T, 1)), rng.standard_normal((T, 2))
    y, den, _, _ = oracle_mod.scan(q, k, v, P=P, c=c)
    for t in range(T):
        w = np.array([sum((q[t, 0] * k[s, 0] / c) ** p / math.factorial(p) for p in range(P))
                      for s in range(t + 1)])
        assert den[t] == pytest.approx(w.sum(), rel=1e-12)
        np.testing.assert_allclose(y[t], (w[:, None] * v[:t + 1]).sum(0) / w.sum(), rtol=1e-11)


def test_affine_equivariance_in_v(oracle_mod):
    rng = np.random.default_rng(4)
    q, k, v = _inputs(rng, 40, 4, 3)
    y, _, _, _ = oracle_mod.scan(q, k, v, P=4)
    a, b = -2.5, np.array([0.5, -1.0, 3.0])
    y2, _, _, _ = oracle_mod.scan(q, k, a * v + b, P=4)
    np.testing.assert_allclose(y2, a * y + b, rtol=1e-11, atol=1e-11)


def test_causality(oracle_mod):
    """Changing token s leaves every output before s unchanged."""
    rng = np.random.default_rng(5)
    q, k, v = _inputs(rng, 30, 4, 4)
    y, _, _, _ = oracle_mod.scan(q, k, v, P=4)
    k2, v2 = k.copy(), v.copy()
    k2[20] += 1.0
    v2[20] -= 2.0
    y2, _, _, _ = oracle_mod.scan(q, k2, v2, P=4)
    np.testing.assert_array_equal(y[:20], y2[:20])
    assert np.abs(y[20:] - y2[20:]).max() > 1e-3


def test_state_equals_full_tensor_power(oracle_mod):
    """S_p[r] equals entry r of sum_t k_t^{(x)p} v_t^T built with outer products,
    read at the tuple's index and at every permutation of it (the symmetric
    tensor), and Z_p likewise.  Pins the update rule and the state layout."""
    rng = np.random.default_rng(6)
    T, d, dV, P = 12, 3, 2, 4
    q, k, v = _inputs(rng, T, d, dV)
    _, _, S, Z = oracle_mod.scan(q, k, v, P)
    deg, M, C, off = oracle_mod.basis(d, P)
    for p in range(P):
        full = np.zeros((d,) * p + (dV,))
        for t in range(T):
            kp = np.array(1.0)
            for _ in range(p):
                kp = np.multiply.outer(kp, k[t])
            full += np.multiply.outer(kp, v[t])
        fullz = full[..., 0] * 0
        for t in range(T):
            kp = np.array(1.0)
            for _ in range(p):
                kp = np.multiply.outer(kp, k[t])
            fullz = fullz + kp
        for r in range(off[p], off[p + 1]):
            tup = tuple(int(i) for i in M[r, :p])
            for perm in set(itertools.permutations(tup)):
                np.testing.assert_allclose(S[r], full[perm], rtol=1e-12, atol=1e-12)
                assert Z[r] == pytest.approx(float(fullz[perm]) if p else float(fullz), rel=1e-12)


def test_scan_continues_from_state(oracle_mod):
    """Decode steps (T = 1 calls) after a prefix equal one scan over all tokens."""
    rng = np.random.default_rng(8)
    q, k, v = _inputs(rng, 25, 4, 4)
    y, den, S, Z = oracle_mod.scan(q, k, v, P=4)
    y1, _, S1, Z1 = oracle_mod.scan(q[:20], k[:20], v[:20], P=4)
    outs = []
    for t in range(20, 25):
        yt, _, S1, Z1 = oracle_mod.scan(q[t:t + 1], k[t:t + 1], v[t:t + 1], P=4, S=S1, Z=Z1)
        outs.append(yt[0])
    np.testing.assert_allclose(np.vstack([y1] + [o[None] for o in outs]), y, rtol=1e-12)
    np.testing.assert_allclose(S1, S, rtol=1e-12)
    np.testing.assert_allclose(Z1, Z, rtol=1e-12)


@pytest.mark.parametrize("d", [1, 2, 4])
def test_softmax_limit(oracle_mod, d):
    """As P grows the truncated kernel tends to exp: the error against exact
    causal softmax attention stays inside the Taylor remainder bound and falls
    to ~0.  With |x| <= X for x = q.k/c, each weight has relative error at most
    r = e^{2X} X^P / P!, so |y - y_softmax| <= 2 r max|v| / (1 - r)."""
    rng = np.random.default_rng(9 + d)
    T, dV = 40, 3
    c = math.sqrt(d)
    a = math.sqrt(2.0 * c / d)          # keeps |q.k/c| <= 2
    q = rng.uniform(-a, a, (T, d))
    k = rng.uniform(-a, a, (T, d))
    v = rng.standard_normal((T, dV))
    X = np.abs(q @ k.T / c).max()
    assert X <= 2.0 + 1e-12
    ys = oracle_mod.softmax(q, k, v)
    errs = {}
    for P in [1, 2, 4, 6, 8, 10, 12, 16]:
        y, _, _ = oracle_mod.direct(q, k, v, P)
        err = np.abs(y - ys).max()
        r = math.exp(2 * X) * X ** P / math.factorial(P)
        if r < 1:
            assert err <= 2 * r * np.abs(v).max() / (1 - r) + 1e-13
        errs[P] = err
    assert errs[16] < 1e-6
    assert errs[16] < errs[8] < errs[4]


def test_softmax_oracle_against_numpy():
    """The softmax routine itself, against numpy's exp on a small case."""
    import oracle
    rng = np.random.default_rng(10)
    q, k, v = rng.standard_normal((6, 3)), rng.standard_normal((6, 3)), rng.standard_normal((6, 2))
    ys = oracle.softmax(q, k, v, c=1.5)
    for t in range(6):
        s = q[t] @ k[:t + 1].T / 1.5
        w = np.exp(s - s.max())
        np.testing.assert_allclose(ys[t], w @ v[:t + 1] / w.sum(), rtol=1e-13)


# ---------------------------------------------------------------- costs ----

@pytest.mark.parametrize("dK,dV,P", [(8, 8, 4), (16, 16, 4), (32, 32, 4), (64, 64, 4), (5, 7, 3),
                                      (128, 128, 4), (3, 2, 6)])
def test_costs_match_page_closed_forms(oracle_mod, dK, dV, P):
    """Term-by-term sums (counted on the enumerated basis) equal the page's
    closed forms: state (d_V+1) binom(d_K+P-1,P-1) and FLOPs/token
    (4 d_V + 2(P d_K + 1)/(d_K + 1) + 2) binom(d_K+P-1,P-1) (exact rationals)."""
    st, fl = oracle_mod.costs(dK, dV, P)
    F = math.comb(dK + P - 1, P - 1)
    assert st == (dV + 1) * F
    closed = (4 * dV + Fraction(2 * (P * dK + 1), dK + 1) + 2) * F
    assert closed.denominator == 1 and fl == closed.numerator


def test_costs_page_values(oracle_mod, golden):
    g = golden["state_values_d64_P4"]
    st, fl = oracle_mod.costs(g["d_K"], g["d_V"], g["P"])
    assert st == g["value"]
    assert abs(st * 2 / 1e6 - 6.2) < 0.05            # "about 6.2 MB at float16"
    assert fl == golden["flops_per_token_d64_P4"]["formula_value"]
    g = golden["state_values_d128_P4"]
    st, fl = oracle_mod.costs(g["d_K"], g["d_V"], g["P"])
    assert st == g["value"]
    assert abs(st * 4 / 2 ** 20 - 180) < 1.0          # "about 180 MB in float32"
    assert fl == golden["flops_per_token_d128_P4"]["formula_value"]
    kv = golden["kv_cache_1M_tokens_d64"]
    assert 1000000 * (64 + 64) == kv["value"] and kv["value"] * 2 == kv["bytes_fp16"]


def test_fourth_term_coefficient(golden):
    g = golden["fourth_term_coefficient_d64"]
    c = math.sqrt(g["d_K"])
    alpha = Fraction(1, math.factorial(g["p"])) / Fraction(int(c)) ** g["p"]
    assert alpha == Fraction(1, g["value_inverse"])


# ------------------------------------------------------------- gradient ----
# The gradient of L = sum(dy * y) (the pages define no backward pass; the
# oracle states the exact chain rule).  Pinned against central differences of
# the forward oracle (itself pinned above), the P = 1 closed form, and two
# identities that hold for any P.

def _loss(oracle_mod, q, k, v, dy, P):
    y, _, _ = oracle_mod.direct(q, k, v, P)
    return float((y * dy).sum())


@pytest.mark.parametrize("dK,dV,P,T", [(3, 2, 4, 6), (2, 3, 2, 5), (4, 1, 5, 5), (1, 2, 3, 7)])
def test_grad_matches_central_differences(oracle_mod, dK, dV, P, T):
    rng = np.random.default_rng(40 + P)
    q, k, v = _inputs(rng, T, dK, dV)
    dy = rng.standard_normal((T, dV))
    dq, dk, dv = oracle_mod.direct_grad(q, k, v, dy, P)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            lp = _loss(oracle_mod, **{**args, name: xp}, dy=dy, P=P)
            lm = _loss(oracle_mod, **{**args, name: xm}, dy=dy, P=P)
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-7 * max(1.0, np.abs(fd).max()),
                                   err_msg=f"d{name}")


def test_grad_P1_is_running_mean_gradient(oracle_mod):
    """P = 1: y_t is the mean of v_0..v_t, so dv_s = sum_{t>=s} dy_t / (t+1) and
    q, k receive no gradient."""
    rng = np.random.default_rng(41)
    T = 25
    q, k, v = _inputs(rng, T, 3, 4)
    dy = rng.standard_normal((T, 4))
    dq, dk, dv = oracle_mod.direct_grad(q, k, v, dy, P=1)
    scaled = dy / np.arange(1, T + 1)[:, None]
    want = np.cumsum(scaled[::-1], axis=0)[::-1]
    np.testing.assert_allclose(dv, want, rtol=1e-12)
    assert np.all(dq == 0) and np.all(dk == 0)


@pytest.mark.parametrize("P", [2, 3, 4, 6])
def test_grad_identities(oracle_mod, P):
    """(1) Shifting every v by b shifts every y by b, so sum_s dv_s = sum_t dy_t.
    (2) y depends on q and k only through q_t . k_s, so
        sum_t q_t . dq_t = sum_s k_s . dk_s (both are sum x_ts dL/dx_ts)."""
    rng = np.random.default_rng(42 + P)
    T, dK, dV = 40, 5, 3
    q, k, v = _inputs(rng, T, dK, dV, scale=0.7)
    dy = rng.standard_normal((T, dV))
    dq, dk, dv = oracle_mod.direct_grad(q, k, v, dy, P)
    np.testing.assert_allclose(dv.sum(0), dy.sum(0), rtol=1e-10, atol=1e-10)
    a, b = float((q * dq).sum()), float((k * dk).sum())
    assert a == pytest.approx(b, rel=1e-10, abs=1e-10)
    assert abs(a) > 1e-3   # not trivially zero


def test_grad_is_causal(oracle_mod):
    """dy on tokens before s gives token s's keys and values no gradient."""
    rng = np.random.default_rng(43)
    T = 20
    q, k, v = _inputs(rng, T, 3, 3)
    dy = np.zeros((T, 3))
    dy[:8] = rng.standard_normal((8, 3))
    dq, dk, dv = oracle_mod.direct_grad(q, k, v, dy, P=4)
    assert np.all(dk[8:] == 0) and np.all(dv[8:] == 0) and np.all(dq[8:] == 0)
    assert np.abs(dk[:8]).max() > 0 and np.abs(dv[:8]).max() > 0
