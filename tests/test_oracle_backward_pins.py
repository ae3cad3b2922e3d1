"""Pins of the oracle's backward pass (CPU only).

The backward functions are checked against central finite differences of the scalar
objective L = <y, dy> + alpha L_bal + beta L_z, computed by the (separately pinned)
forward functions alone. The routing and the load fractions are piecewise constant, so
each case first checks that no top-K choice flips inside the difference step. Large loss
weights make the load-balance and Z-loss terms as visible as the expert terms, so a
dropped term, a wrong sign or a transposed product in any part fails here.
"""
import numpy as np
import pytest

from oracle import moe_null_oracle as o

EPS = 1e-5


def _case(T, d, N, M, K, F, Fs, C=0, V=0, seed=0):
    rng = np.random.default_rng(seed)
    rows = N + 1 + C + V
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((rows, d)) / np.sqrt(d)
    bias = 0.3 * rng.standard_normal(rows)
    # per-token null offsets: strongly negative (all real), strongly positive (all null
    # while copies last) and moderate ones (mixed)
    tnb = rng.choice([-6.0, 6.0, 0.0, 0.3, -0.3], size=T)
    experts = (rng.standard_normal((N, F, d)) / np.sqrt(d), rng.standard_normal((N, F, d)) / np.sqrt(d),
               rng.standard_normal((N, d, F)) / np.sqrt(F))
    shared = (rng.standard_normal((Fs, d)) / np.sqrt(d), rng.standard_normal((Fs, d)) / np.sqrt(d),
              rng.standard_normal((d, Fs)) / np.sqrt(Fs))
    cv = rng.standard_normal((V, d))
    dy = rng.standard_normal((T, d))
    return dict(x=x, w_r=w_r, bias=bias, tnb=tnb, experts=experts, shared=shared, cv=cv, dy=dy,
                N=N, M=M, K=K, C=C, V=V)


def _objective(c, alpha, beta, **over):
    a = dict(c)
    a.update(over)
    return o.layer_objective(a["x"], a["w_r"], a["bias"], a["tnb"], a["N"], a["M"], a["K"],
                             a["experts"], a["shared"], a["dy"], alpha, beta, C=a["C"], V=a["V"],
                             const_vectors=a["cv"])


def _routing(c, **over):
    a = dict(c)
    a.update(over)
    null_col = a["N"] if (a["C"] + a["V"]) else None
    s = o.router_logits(a["x"], a["w_r"], a["bias"], a["tnb"], null_col=null_col)
    return o.route_pp(s, a["N"], a["M"], a["C"], a["V"], a["K"])["idx"]


def _fd(c, alpha, beta, name, getter, setter, entries):
    """Central differences of the objective with respect to the given entries."""
    idx0 = _routing(c)
    out = []
    for e in entries:
        vals = []
        for sgn in (1.0, -1.0):
            arr = getter(c).copy()
            arr[e] += sgn * EPS
            over = setter(c, arr)
            assert np.array_equal(_routing(c, **over), idx0), f"routing flipped at {name}{e}"
            vals.append(_objective(c, alpha, beta, **over))
        out.append((vals[0] - vals[1]) / (2 * EPS))
    return np.array(out)


def _backward(c, alpha, beta):
    null_col = c["N"] if (c["C"] + c["V"]) else None
    s = o.router_logits(c["x"], c["w_r"], c["bias"], c["tnb"], null_col=null_col)
    return o.layer_backward(c["x"], s, c["w_r"], c["N"], c["M"], c["K"], c["experts"], c["shared"],
                            c["dy"], alpha, beta, C=c["C"], V=c["V"], const_vectors=c["cv"])


def _sample(shape, n, rng):
    flat = rng.choice(int(np.prod(shape)), size=min(n, int(np.prod(shape))), replace=False)
    return [tuple(np.unravel_index(i, shape)) for i in flat]


def _check_all(c, alpha, beta, seed=1):
    rng = np.random.default_rng(seed)
    g = _backward(c, alpha, beta)
    checks = [
        ("x", lambda c: c["x"], lambda c, a: {"x": a}, g["dx"]),
        ("w_r", lambda c: c["w_r"], lambda c, a: {"w_r": a}, g["dW_r"]),
        ("bias", lambda c: c["bias"], lambda c, a: {"bias": a}, g["dbias"]),
        ("tnb", lambda c: c["tnb"], lambda c, a: {"tnb": a}, g["dtnb"]),
    ]
    for j, key in enumerate(("dW_gate", "dW_up", "dW_down")):
        checks.append((key, lambda c, j=j: c["experts"][j],
                       lambda c, a, j=j: {"experts": tuple(a if i == j else c["experts"][i]
                                                           for i in range(3))}, g[key]))
    for j, key in enumerate(("dWs_gate", "dWs_up", "dWs_down")):
        checks.append((key, lambda c, j=j: c["shared"][j],
                       lambda c, a, j=j: {"shared": tuple(a if i == j else c["shared"][i]
                                                          for i in range(3))}, g[key]))
    if c["V"]:
        checks.append(("cv", lambda c: c["cv"], lambda c, a: {"cv": a}, g["dconst"]))
    for name, getter, setter, analytic in checks:
        entries = _sample(getter(c).shape, 40, rng)
        fd = _fd(c, alpha, beta, name, getter, setter, entries)
        an = np.array([analytic[e] for e in entries])
        np.testing.assert_allclose(an, fd, rtol=1e-6, atol=1e-8, err_msg=name)
    return g


def test_backward_matches_finite_differences_null_pool():
    c = _case(T=14, d=8, N=4, M=3, K=3, F=6, Fs=5, seed=11)
    g = _check_all(c, alpha=0.7, beta=0.4)
    n_real = (g["idx"] < c["N"]).sum(axis=1)
    # the case exercises tokens with no real expert, all real experts and a mix
    assert n_real.min() == 0 and n_real.max() == c["K"] and ((n_real > 0) & (n_real < c["K"])).any()


def test_backward_matches_finite_differences_no_null():
    # M = 0: plain top-K with renormalised gates; every slot is real
    c = _case(T=10, d=6, N=5, M=0, K=2, F=4, Fs=3, seed=12)
    _check_all(c, alpha=0.5, beta=0.5)


def test_backward_matches_finite_differences_moepp_pool():
    c = _case(T=16, d=6, N=4, M=2, K=3, F=4, Fs=3, C=1, V=2, seed=13)
    g = _check_all(c, alpha=0.6, beta=0.3)
    P = c["N"] + c["M"]
    assert (g["idx"] >= P).any(), "the case must select copy or constant experts"


def test_loss_weights_separate_cleanly():
    # each loss term alone: zero dy and one weight at a time still matches differences
    c = _case(T=12, d=6, N=4, M=3, K=2, F=4, Fs=3, seed=14)
    c["dy"] = np.zeros_like(c["dy"])
    for alpha, beta in ((1.0, 0.0), (0.0, 1.0)):
        _check_all(c, alpha, beta, seed=2)


def test_logit_gradient_invariants():
    """Closed forms: adding a constant to every router logit of a token changes neither
    the gates nor P, and moves lse by that constant. So the gate and load-balance parts
    of ds sum to 0 over a token's logit columns (null column counted once, it already
    holds the M copies' sum), and the Z-loss part sums to 2 lse_t / T."""
    c = _case(T=20, d=8, N=6, M=4, K=3, F=4, Fs=3, seed=15)
    s = o.router_logits(c["x"], c["w_r"], c["bias"], c["tnb"])
    T = c["x"].shape[0]
    only_gate = o.layer_backward(c["x"], s, c["w_r"], 6, 4, 3, c["experts"], c["shared"], c["dy"], 0.0, 0.0)
    np.testing.assert_allclose(only_gate["ds"].sum(axis=1), 0.0, atol=1e-12)
    no_dy = np.zeros_like(c["dy"])
    bal = o.layer_backward(c["x"], s, c["w_r"], 6, 4, 3, c["experts"], c["shared"], no_dy, 1.0, 0.0)
    np.testing.assert_allclose(bal["ds"].sum(axis=1), 0.0, atol=1e-12)
    z = o.layer_backward(c["x"], s, c["w_r"], 6, 4, 3, c["experts"], c["shared"], no_dy, 0.0, 1.0)
    lse = o.pool_logsumexp(o.expanded_pool(s, 4))
    np.testing.assert_allclose(z["ds"].sum(axis=1), 2.0 * lse / T, rtol=1e-12)
    # with no upstream gradient and no loss, nothing moves
    zero = o.layer_backward(c["x"], s, c["w_r"], 6, 4, 3, c["experts"], c["shared"], no_dy, 0.0, 0.0)
    for k in ("dx", "ds", "dW_r", "dW_gate", "dW_down", "dWs_up"):
        assert not np.any(zero[k])


def test_gate_gradient_of_single_real_expert_is_zero():
    """A token with exactly one real expert has gate 1 whatever its logit: the gate part of
    its logit gradient vanishes, while dg (the expert output's projection on dy) does not."""
    c = _case(T=8, d=6, N=4, M=6, K=4, F=4, Fs=3, seed=16)
    s = o.router_logits(c["x"], c["w_r"], c["bias"], c["tnb"])
    # make every token select exactly one real expert: its best real beats the null
    # logit, all others fall below it
    best = s[:, :4].argmax(axis=1)
    for t in range(8):
        s[t, 4] = s[t, best[t]] - 1e-3
        s[t, :4] = np.where(np.arange(4) == best[t], s[t, :4], s[t, 4] - 1.0)
    g = o.layer_backward(c["x"], s, c["w_r"], 4, 6, 4, c["experts"], c["shared"], c["dy"], 0.0, 0.0)
    assert ((g["idx"] < 4).sum(axis=1) == 1).all()
    np.testing.assert_allclose(g["ds"], 0.0, atol=1e-15)
    assert np.abs(g["dg"][:, 0]).min() > 0


def test_aux_backward_of_a_shard_equals_the_rows_of_the_whole_batch():
    """Data parallel: with the whole batch's slot counts and token total, the loss-term
    gradient of one shard's tokens equals those tokens' rows of the whole-batch gradient
    (f and both means are whole-batch quantities; each token's row depends on no other
    token's logits)."""
    rng = np.random.default_rng(21)
    T, N, M, K = 40, 6, 5, 3
    s = rng.standard_normal((T, N + 1))
    v = o.expanded_pool(s, M)
    lse = o.pool_logsumexp(v)
    p = o.pool_probs(v, lse)
    idx = o.topk_pool(v, K)
    whole = o.aux_backward(idx, p, lse, N, 0.7, 0.3)
    counts = np.bincount(idx.reshape(-1), minlength=N + M)
    for rows in (np.arange(0, 17), np.arange(17, 40)):
        part = o.aux_backward(idx[rows], p[rows], lse[rows], N, 0.7, 0.3, counts=counts, t_total=T)
        np.testing.assert_allclose(part, whole[rows], rtol=1e-13, atol=1e-16)
    # and a shard's own statistics give something else
    own = o.aux_backward(idx[:17], p[:17], lse[:17], N, 0.7, 0.3)
    assert not np.allclose(own, whole[:17])


def test_shard_gradients_sum_to_the_whole_batch_gradient():
    """Data parallel: each shard's weight gradients, taken with the whole batch's slot counts
    and token total, add up to the whole batch's weight gradients (the objective is a sum over
    tokens of <y_t, dy_t> plus losses built from whole-batch means)."""
    c = _case(T=18, d=6, N=4, M=3, K=2, F=4, Fs=3, seed=17)
    s = o.router_logits(c["x"], c["w_r"], c["bias"], c["tnb"])
    whole = o.layer_backward(c["x"], s, c["w_r"], 4, 3, 2, c["experts"], c["shared"], c["dy"], 0.7, 0.4)
    counts = np.bincount(whole["idx"].reshape(-1), minlength=7)
    acc = None
    for rows in (np.arange(0, 7), np.arange(7, 18)):
        part = o.layer_backward(c["x"][rows], s[rows], c["w_r"], 4, 3, 2, c["experts"], c["shared"], c["dy"][rows],
                                0.7, 0.4, counts=counts, t_total=18)
        np.testing.assert_allclose(part["dx"], whole["dx"][rows], rtol=1e-12, atol=1e-14)
        acc = part if acc is None else {k: acc[k] + part[k] for k in ("dW_r", "dbias", "dW_gate", "dW_up", "dW_down",
                                                                      "dWs_gate", "dWs_up", "dWs_down")}
    for k in ("dW_r", "dbias", "dW_gate", "dW_up", "dW_down", "dWs_gate", "dWs_up", "dWs_down"):
        np.testing.assert_allclose(acc[k], whole[k], rtol=1e-12, atol=1e-14, err_msg=k)


def test_gate_gradient_two_selected_experts_closed_form():
    """Worked example: a token whose two selected slots are real with logits s1, s2 has gates
    g1 = 1/(1+e^{s2-s1}), g2 = 1 - g1, so dL/ds1 = -dL/ds2 = g1 g2 (dg1 - dg2); the other
    logits get nothing from the gates."""
    s1, s2, dg1, dg2 = 0.7, -0.4, 1.3, -0.6
    v = np.array([[s1, s2, -3.0, -2.5, -2.5]])  # 3 reals, then 2 copies of a null logit -2.5
    idx = np.array([[0, 1]])
    gates = o.renormalised_gates(np.array([[s1, s2, -3.0, -2.5]]), idx, 3)
    g1 = 1.0 / (1.0 + np.exp(s2 - s1))
    np.testing.assert_allclose(gates[0], [g1, 1 - g1], rtol=1e-15)
    dv = o.gate_backward(v, idx, gates, np.array([[dg1, dg2]]), 3, 2)
    expect = g1 * (1 - g1) * (dg1 - dg2)
    np.testing.assert_allclose(dv[0], [expect, -expect, 0.0, 0.0, 0.0], rtol=1e-14, atol=1e-16)
