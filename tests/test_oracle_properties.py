"""Property tests of the oracle over generated cases (CPU only, hypothesis).

Each property is fixed by the mathematics rather than by the oracle's own formulas:
- routing: the top-K set is the unique K-subset whose members all precede all non-members in
  (value desc, index asc), found by enumeration; the real count obeys the threshold reading;
- gates: a softmax over the selected non-null logits (sum 1, invariant to a common shift);
- statistics: counts add up to T K, P sums to 1;
- backward: the analytic gradient equals central finite differences of the forward objective
  on random small layers (entries sampled).
"""
import itertools

import numpy as np
import pytest
from hypothesis import HealthCheck, assume, given, settings
from hypothesis import strategies as st

from oracle import moe_null_oracle as o


def _enumerate_topk(v, K):
    P = len(v)

    def before(i, j):
        return v[i] > v[j] or (v[i] == v[j] and i < j)

    hits = [S for S in itertools.combinations(range(P), K)
            if all(before(i, j) for i in S for j in range(P) if j not in S)]
    assert len(hits) == 1
    return sorted(hits[0], key=lambda i: (-v[i], i))


@st.composite
def pools(draw):
    N = draw(st.integers(1, 5))
    M = draw(st.integers(0, 4))
    C = draw(st.integers(0, 2))
    V = draw(st.integers(0, 2))
    K = draw(st.integers(1, min(4, N + M + C + V)))
    T = draw(st.integers(1, 6))
    # half-integer logits in a small range: exact ties among reals, nulls and MoE++ experts
    vals = draw(st.lists(st.integers(-3, 3), min_size=T * (N + 1 + C + V), max_size=T * (N + 1 + C + V)))
    s = np.array(vals, dtype=np.float64).reshape(T, N + 1 + C + V) / 2.0
    return s, N, M, C, V, K


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(pools())
def test_routing_properties(case):
    s, N, M, C, V, K = case
    T = s.shape[0]
    r = o.route_pp(s, N, M, C, V, K)
    v = r["v"]
    for t in range(T):
        assert r["idx"][t].tolist() == _enumerate_topk(list(v[t]), K)
    if C + V == 0:
        np.testing.assert_array_equal(r["n_real"], o.threshold_real_count(s, M, K))
    # gates: softmax over the selected non-null slots
    g = r["gates"]
    nonnull = (r["idx"] < N) | (r["idx"] >= N + M)
    for t in range(T):
        if nonnull[t].any():
            assert abs(g[t].sum() - 1.0) < 1e-12
            sel = v[t, r["idx"][t][nonnull[t]]]
            e = np.exp(sel - sel.max())
            np.testing.assert_allclose(g[t][nonnull[t]], e / e.sum(), rtol=1e-13)
        assert np.all(g[t][~nonnull[t]] == 0.0)
    # shift invariance of routing and gates
    r2 = o.route_pp(s + 1.25, N, M, C, V, K)
    np.testing.assert_array_equal(r2["idx"], r["idx"])
    np.testing.assert_allclose(r2["gates"], g, rtol=1e-12, atol=1e-15)
    # statistics
    counts, f, P, L_bal, L_z = o.aux_stats(r["idx"], r["p"], r["lse"], N, M)
    assert counts.sum() == T * K
    assert abs(P.sum() - 1.0) < 1e-12


@st.composite
def layers(draw):
    N = draw(st.integers(1, 4))
    M = draw(st.integers(0, 3))
    K = draw(st.integers(1, min(3, N + M)))
    T = draw(st.integers(1, 5))
    d = draw(st.integers(2, 5))
    F = draw(st.integers(1, 4))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return N, M, K, T, d, F, seed


@settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(layers())
def test_backward_matches_finite_differences(case):
    N, M, K, T, d, F, seed = case
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((N + 1, d))
    bias = rng.standard_normal(N + 1)
    experts = (rng.standard_normal((N, F, d)), rng.standard_normal((N, F, d)), rng.standard_normal((N, d, F)))
    shared = (rng.standard_normal((F, d)), rng.standard_normal((F, d)), rng.standard_normal((d, F)))
    dy = rng.standard_normal((T, d))
    alpha, beta = 0.8, 0.3
    s = o.router_logits(x, w_r, bias)
    v = o.expanded_pool(s, M)
    # keep cases whose routing cannot flip within the difference step (a gap of 1e-3 between
    # the K-th and (K+1)-th pool values of every token)
    srt = -np.sort(-v, axis=1)
    assume(v.shape[1] == K or np.min(srt[:, K - 1] - srt[:, K]) >= 1e-3)
    g = o.layer_backward(x, s, w_r, N, M, K, experts, shared, dy, alpha, beta)
    eps = 1e-6

    def obj(**over):
        a = dict(x=x, w_r=w_r, bias=bias, experts=experts)
        a.update(over)
        return o.layer_objective(a["x"], a["w_r"], a["bias"], None, N, M, K, a["experts"], shared, dy, alpha, beta)

    def check(name, arr, grad, build):
        flat = rng.choice(arr.size, size=min(6, arr.size), replace=False)
        for i in flat:
            e = np.unravel_index(i, arr.shape)
            ap, am = arr.copy(), arr.copy()
            ap[e] += eps
            am[e] -= eps
            fd = (obj(**build(ap)) - obj(**build(am))) / (2 * eps)
            assert abs(fd - grad[e]) <= 1e-5 * max(1.0, abs(fd)), (name, e, fd, grad[e])

    check("x", x, g["dx"], lambda a: {"x": a})
    check("w_r", w_r, g["dW_r"], lambda a: {"w_r": a})
    check("bias", bias, g["dbias"], lambda a: {"bias": a})
    check("w_down", experts[2], g["dW_down"], lambda a: {"experts": (experts[0], experts[1], a)})
    check("w_gate", experts[0], g["dW_gate"], lambda a: {"experts": (a, experts[1], experts[2])})
