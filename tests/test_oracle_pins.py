"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test below ties one oracle function to what the pages or plain
mathematics fix: a hand-worked example, brute-force enumeration, closed forms,
a reduction to a textbook routine (torch.topk / softmax / silu, scipy
logsumexp), and invariants stated on the pages. A plausible slip in the
oracle (a dropped null copy, reversed tie rule, gates taken from the pool
softmax, a wrong multiplier in L_bal, a transposed weight) fails at least one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ev(expr):
    return float(eval(expr, {"__builtins__": {}}, {"log": math.log, "exp": math.exp}))


# --- hand-worked example ---------------------------------------------------------------

def test_worked_example_routing_and_dispatch():
    g = json.load(open(os.path.join(GOLDEN, "route_worked_example.json")))
    N, M, K = g["N"], g["M"], g["K"]
    s = np.array([[_ev(v) for v in row] for row in g["logits"]])
    r = O.route(s, M, K)
    ex = g["expected"]
    assert r["idx"].tolist() == ex["topk_idx"]
    assert r["n_real"].tolist() == ex["n_real"]
    np.testing.assert_allclose(r["gates"], [[_ev(v) for v in row] for row in ex["gates"]], rtol=0, atol=1e-15)
    np.testing.assert_allclose(r["lse"], [_ev(v) for v in ex["lse"]], rtol=1e-15)
    counts_ext, f, P, L_bal, L_z = O.aux_stats(r["idx"], r["p"], r["lse"], N, M)
    assert counts_ext.tolist() == ex["counts_ext"]
    counts, offsets, perm, slot_row = O.dispatch(r["idx"], N)
    assert counts.tolist() == ex["counts"]
    assert offsets.tolist() == ex["offsets"]
    assert perm.tolist() == ex["perm_tok"]
    assert slot_row.tolist() == ex["slot_row"]
    # L_bal and L_z from the hand values, written out term by term.
    lse = np.array([_ev(v) for v in ex["lse"]])
    pool = np.concatenate([s[:, :N], np.repeat(s[:, N:], M, axis=1)], axis=1)
    P_hand = (np.exp(pool - lse[:, None])).mean(axis=0)
    f_hand = np.array(ex["counts_ext"]) / 4.0
    assert L_bal == pytest.approx(N * float((f_hand * P_hand).sum()), rel=1e-14)
    assert L_z == pytest.approx(float((lse ** 2).mean()), rel=1e-14)


# --- brute force -----------------------------------------------------------------------

def _brute_topk(v, K):
    """Unique K-subset whose members all precede all non-members in (value desc,
    index asc); returned in rank order. Pure enumeration, no sort of the pool."""
    P = len(v)

    def before(i, j):
        return v[i] > v[j] or (v[i] == v[j] and i < j)

    hits = []
    for S in itertools.combinations(range(P), K):
        rest = [j for j in range(P) if j not in S]
        if all(before(i, j) for i in S for j in rest):
            hits.append(S)
    assert len(hits) == 1
    S = list(hits[0])
    ranked = []
    while S:  # selection by repeated "beats all others"
        best = [i for i in S if all(before(i, j) for j in S if j != i)][0]
        ranked.append(best)
        S.remove(best)
    return ranked


@pytest.mark.parametrize("N,M", [(1, 1), (2, 0), (3, 2), (4, 3), (5, 1), (5, 3)])
def test_topk_matches_bruteforce_with_ties(N, M):
    rng = np.random.default_rng(100 + 10 * N + M)
    T = 48
    # quantised logits make exact ties among reals and with the null logit
    s = rng.integers(-2, 3, size=(T, N + 1)).astype(np.float64) / 2.0
    for K in range(1, min(4, N + M) + 1):
        v = O.expanded_pool(s, M)
        idx = O.topk_pool(v, K)
        r = O.threshold_real_count(s, M, K)
        for t in range(T):
            bt = _brute_topk(list(v[t]), K)
            assert idx[t].tolist() == bt, (t, K, v[t])
            assert int(r[t]) == sum(1 for i in bt if i < N)


def test_null_copies_fill_in_index_order():
    # all copies tie with each other; they must appear as N, N+1, ... in rank order
    N, M, K = 4, 5, 7
    s = np.array([[3.0, -9.0, 2.0, -8.0, 0.0]])
    idx = O.topk_pool(O.expanded_pool(s, M), K)[0].tolist()
    assert idx == [0, 2, 4, 5, 6, 7, 8]
    # when copies run out the lower reals follow
    idx = O.topk_pool(O.expanded_pool(s, 2), 6)[0].tolist()
    assert idx == [0, 2, 4, 5, 3, 1]


def test_real_equal_to_null_beats_every_copy():
    s = np.array([[0.25, 1.0, 0.25]])  # real 0 ties the null logit
    idx = O.topk_pool(O.expanded_pool(s, 3), 3)[0].tolist()
    assert idx == [1, 0, 2]


# --- M = 0 reduces to plain top-K MoE --------------------------------------------------

def _torch_expert(x, wg, wu, wd):
    return (torch.nn.functional.silu(x @ wg.T) * (x @ wu.T)) @ wd.T


def test_m0_is_plain_topk_moe():
    rng = np.random.default_rng(7)
    T, d, N, F, K = 40, 24, 6, 16, 3
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((N + 1, d)) / math.sqrt(d)
    s = O.router_logits(x, wr)
    r = O.route(s, 0, K)
    tx = torch.from_numpy(x)
    ts = torch.from_numpy(s[:, :N])
    vals, ind = torch.topk(ts, K, dim=1, sorted=True)
    assert r["idx"].tolist() == ind.tolist()
    np.testing.assert_allclose(r["gates"], torch.softmax(vals, dim=1).numpy(), rtol=1e-13, atol=1e-15)
    # the layer output equals a textbook top-K MoE built from torch ops
    wg = rng.standard_normal((N, F, d)) / math.sqrt(d)
    wu = rng.standard_normal((N, F, d)) / math.sqrt(d)
    wd = rng.standard_normal((N, d, F)) / math.sqrt(F)
    sg, su, sd = (rng.standard_normal((F, d)) / math.sqrt(d), rng.standard_normal((F, d)) / math.sqrt(d),
                  rng.standard_normal((d, F)) / math.sqrt(F))
    y = O.layer_output(x, r["idx"], r["gates"], N, (wg, wu, wd), (sg, su, sd))
    T_ = lambda a: torch.from_numpy(a)
    ref = _torch_expert(tx, T_(sg), T_(su), T_(sd))
    w = torch.softmax(vals, dim=1)
    for t in range(T):
        for k in range(K):
            e = int(ind[t, k])
            ref[t] += w[t, k] * _torch_expert(tx[t:t + 1], T_(wg[e]), T_(wu[e]), T_(wd[e]))[0]
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)
    # and the pool probabilities are the textbook router softmax
    np.testing.assert_allclose(r["p"], scipy.special.softmax(s[:, :N], axis=1), rtol=1e-13)


# --- renormalisation -------------------------------------------------------------------

def test_gates_are_softmax_over_selected_reals_and_match_masked_topk():
    rng = np.random.default_rng(11)
    T, N, M, K = 200, 8, 8, 4
    s = rng.standard_normal((T, N + 1)) * 1.5
    r = O.route(s, M, K)
    v = r["v"]
    for t in range(T):
        sel = [k for k in range(K) if r["idx"][t, k] < N]
        if not sel:
            assert np.all(r["gates"][t] == 0)
            continue
        ref = scipy.special.softmax(s[t, r["idx"][t, sel]])
        np.testing.assert_allclose(r["gates"][t, sel], ref, rtol=1e-13)
        assert np.all(r["gates"][t, [k for k in range(K) if k not in sel]] == 0)
        # masked-top-K form (MoE++ gating page): softmax over the K pool values,
        # zero the zero-compute slots, divide by the remaining sum
        gk = scipy.special.softmax(v[t, r["idx"][t]])
        gk[r["idx"][t] >= N] = 0.0
        gk /= gk.sum()
        np.testing.assert_allclose(r["gates"][t], gk, rtol=1e-12, atol=1e-15)
        assert r["gates"][t].sum() == pytest.approx(1.0, abs=1e-14)


def test_gates_differ_from_unrenormalised_pool_softmax():
    # guards against taking gates straight from the pool softmax
    s = np.array([[1.0, 0.0, -1.0, 0.5]])
    r = O.route(s, 2, 3)
    assert r["gates"][0].sum() == pytest.approx(1.0)
    assert not np.allclose(r["gates"][0][:2], r["p"][0][r["idx"][0][:2]])


# --- K^4_0.5 reproduces K^2_1.0 (solution-space preservation) --------------------------

def test_k4_half_reproduces_k2_dense():
    rng = np.random.default_rng(5)
    T, d, N, F = 64, 32, 8, 16
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((N + 1, d)) / math.sqrt(d)
    base = O.router_logits(x, wr)
    srt = -np.sort(-base[:, :N], axis=1)
    # null logit placed strictly between the 2nd and 3rd largest real logit
    off = 0.5 * (srt[:, 1] + srt[:, 2]) - base[:, N]
    s4 = O.router_logits(x, wr, tok_null_bias=off)
    r4 = O.route(s4, 64, 4)
    r2 = O.route(s4, 0, 2)
    assert np.all(r4["n_real"] == 2)
    assert r4["idx"][:, :2].tolist() == r2["idx"].tolist()
    assert np.all(r4["idx"][:, 2:] >= N)
    np.testing.assert_allclose(r4["gates"][:, :2], r2["gates"], rtol=0, atol=1e-15)
    ex = (rng.standard_normal((N, F, d)) / math.sqrt(d), rng.standard_normal((N, F, d)) / math.sqrt(d),
          rng.standard_normal((N, d, F)) / math.sqrt(F))
    sh = (rng.standard_normal((F, d)) / math.sqrt(d), rng.standard_normal((F, d)) / math.sqrt(d),
          rng.standard_normal((d, F)) / math.sqrt(F))
    y4 = O.layer_output(x, r4["idx"], r4["gates"], N, ex, sh)
    y2 = O.layer_output(x, r2["idx"], r2["gates"], N, ex, sh)
    np.testing.assert_allclose(y4, y2, rtol=0, atol=1e-12)


# --- invariants ------------------------------------------------------------------------

@pytest.mark.parametrize("N,M,K", [(8, 8, 4), (16, 48, 8), (8, 0, 2), (6, 2, 5)])
def test_invariants(N, M, K):
    rng = np.random.default_rng(N * 100 + M + K)
    T = 300
    s = rng.standard_normal((T, N + 1))
    s[:, N] += rng.normal(0.0, 1.0)
    r = O.route(s, M, K)
    counts_ext, f, P, L_bal, L_z = O.aux_stats(r["idx"], r["p"], r["lse"], N, M)
    assert counts_ext.sum() == T * K
    assert f.sum() == pytest.approx(K, abs=1e-12)
    assert P.sum() == pytest.approx(1.0, abs=1e-12)
    counts, offsets, perm, slot_row = O.dispatch(r["idx"], N)
    assert offsets[-1] == r["n_real"].sum() == counts.sum()
    assert np.array_equal(counts, counts_ext[:N])
    assert np.all(r["n_real"] == O.threshold_real_count(s, M, K))
    if M:
        stair = counts_ext[N:]
        assert np.all(np.diff(stair) <= 0)
        nulls = K - r["n_real"]
        assert np.array_equal(stair, [(nulls > j).sum() for j in range(M)])
        # L_bal does not depend on which copies the nulls occupy
        idx2 = r["idx"].copy()
        for t in range(T):
            c = int(nulls[t])
            if c:
                idx2[t, idx2[t] >= N] = N + rng.choice(M, size=c, replace=False)
        _, _, _, L_bal2, _ = O.aux_stats(idx2, r["p"], r["lse"], N, M)
        assert L_bal2 == pytest.approx(L_bal, rel=1e-13)
    # the shard sums reduce to the whole
    a = O.aux_partial_sums(r["idx"][:100], r["p"][:100], r["lse"][:100], N, M)
    b = O.aux_partial_sums(r["idx"][100:], r["p"][100:], r["lse"][100:], N, M)
    f2, P2, Lb2, Lz2 = O.aux_finalize(a[0] + b[0], a[1] + b[1], a[2] + b[2], a[3] + b[3], N)
    assert Lb2 == pytest.approx(L_bal, rel=1e-13) and Lz2 == pytest.approx(L_z, rel=1e-13)
    np.testing.assert_allclose(P2, P, rtol=1e-13)


def test_token_without_real_expert_gets_only_shared_expert():
    rng = np.random.default_rng(3)
    T, d, N, F, M, K = 10, 16, 4, 8, 4, 3
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((N + 1, d))
    s = O.router_logits(x, wr, bias=np.r_[np.zeros(N), 1e3])
    r = O.route(s, M, K)
    assert np.all(r["n_real"] == 0) and np.all(r["gates"] == 0)
    ex = tuple(rng.standard_normal(sh) for sh in [(N, F, d), (N, F, d), (N, d, F)])
    sh = tuple(rng.standard_normal(q) for q in [(F, d), (F, d), (d, F)])
    y = O.layer_output(x, r["idx"], r["gates"], N, ex, sh)
    np.testing.assert_array_equal(y, O.swiglu(x, *sh))


# --- closed forms ----------------------------------------------------------------------

@pytest.mark.parametrize("N,M,K", [(8, 8, 4), (64, 192, 8), (64, 0, 2)])
def test_closed_form_equal_logits(N, M, K):
    c = 0.37
    s = np.full((5, N + 1), c)
    r = O.route(s, M, K)
    np.testing.assert_allclose(r["lse"], c + math.log(N + M), rtol=1e-15)
    np.testing.assert_allclose(r["p"], 1.0 / (N + M), rtol=1e-13)
    assert r["idx"].tolist() == [list(range(K))] * 5
    np.testing.assert_allclose(r["gates"], 1.0 / K, rtol=1e-14)
    _, _, P, L_bal, L_z = O.aux_stats(r["idx"], r["p"], r["lse"], N, M)
    assert L_bal == pytest.approx(N * K / (N + M), rel=1e-13)
    assert L_z == pytest.approx((c + math.log(N + M)) ** 2, rel=1e-14)


def test_lse_and_probs_match_scipy_on_materialised_pool():
    rng = np.random.default_rng(21)
    s = rng.standard_normal((50, 9)) * 3
    for M in (0, 1, 7):
        v = np.concatenate([s[:, :8]] + ([np.repeat(s[:, 8:], M, axis=1)] if M else []), axis=1)
        assert np.array_equal(O.expanded_pool(s, M), v)
        np.testing.assert_allclose(O.pool_logsumexp(v), scipy.special.logsumexp(v, axis=1), rtol=1e-14)
        lse = O.pool_logsumexp(v)
        np.testing.assert_allclose(O.pool_probs(v, lse), scipy.special.softmax(v, axis=1), rtol=1e-13)


def test_lbal_multiplier_and_normalisation():
    # one token, N=2, M=1, K=1: picks real 0 with p0; L_bal = N * (1 * p0)
    s = np.array([[2.0, 0.0, 1.0]])
    r = O.route(s, 1, 1)
    _, f, P, L_bal, _ = O.aux_stats(r["idx"], r["p"], r["lse"], 2, 1)
    p0 = math.exp(2.0) / (math.exp(2.0) + 1.0 + math.exp(1.0))
    assert f.tolist() == [1.0, 0.0, 0.0]
    assert L_bal == pytest.approx(2 * p0, rel=1e-15)


# --- dispatch and experts ------------------------------------------------------------------

def test_dispatch_matches_explicit_loops():
    rng = np.random.default_rng(9)
    T, N, M, K = 70, 6, 3, 4
    s = rng.integers(-2, 3, size=(T, N + 1)).astype(float)
    idx = O.route(s, M, K)["idx"]
    counts, offsets, perm, slot_row = O.dispatch(idx, N)
    rows, want_slot = [], -np.ones((T, K), dtype=int)
    for e in range(N):
        for t in range(T):
            for k in range(K):
                if idx[t, k] == e:
                    want_slot[t, k] = len(rows)
                    rows.append(t)
    assert perm.tolist() == rows
    assert np.array_equal(slot_row, want_slot)
    assert counts.tolist() == [int((idx == e).sum()) for e in range(N)]
    assert offsets.tolist() == [0] + np.cumsum(counts).tolist()


def test_swiglu_matches_torch():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((9, 12))
    wg, wu, wd = rng.standard_normal((5, 12)), rng.standard_normal((5, 12)), rng.standard_normal((12, 5))
    ref = _torch_expert(torch.from_numpy(z), torch.from_numpy(wg), torch.from_numpy(wu), torch.from_numpy(wd))
    np.testing.assert_allclose(O.swiglu(z, wg, wu, wd), ref.numpy(), rtol=1e-13, atol=1e-13)
    # gate and up are not interchangeable (silu is applied to the gate only)
    assert not np.allclose(O.swiglu(z, wu, wg, wd), ref.numpy())


def test_router_logits_bias_and_null_offset():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 5))
    w = rng.standard_normal((4, 5))
    b = np.array([0.1, 0.2, 0.3, 0.4])
    o = np.array([1.0, 2.0, 3.0])
    s = O.router_logits(x, w, b, o)
    ref = torch.from_numpy(x) @ torch.from_numpy(w).T + torch.from_numpy(b)
    ref[:, 3] += torch.from_numpy(o)
    np.testing.assert_allclose(s, ref.numpy(), rtol=1e-14)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(12)
    a = rng.standard_normal(10000) * 10
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16_round_f64(a.astype(np.float32)), ref)


# --- MoE++ copy and constant experts next to the null expert ----------------------------

def _pp_case(seed, T, d, N, M, C, V, F=16, Fs=12):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    experts = (rng.standard_normal((N, F, d)) / math.sqrt(d), rng.standard_normal((N, F, d)) / math.sqrt(d),
               rng.standard_normal((N, d, F)) / math.sqrt(F))
    shared = (rng.standard_normal((Fs, d)) / math.sqrt(d), rng.standard_normal((Fs, d)) / math.sqrt(d),
              rng.standard_normal((d, Fs)) / math.sqrt(Fs))
    cv = rng.standard_normal((V, d))
    return rng, x, experts, shared, cv


def test_pp_without_copy_or_constant_experts_is_the_null_only_layer():
    rng, x, ex, sh, cv = _pp_case(401, 40, 8, 5, 3, 0, 0)
    s = rng.standard_normal((40, 6))
    for K in (1, 3, 5):
        a, b = O.route(s, 3, K), O.route_pp(s, 5, 3, 0, 0, K)
        for k in ("v", "idx", "n_real"):
            np.testing.assert_array_equal(a[k], b[k])
        for k in ("lse", "p", "gates"):  # same values, NumPy may sum them in another order
            np.testing.assert_allclose(a[k], b[k], rtol=1e-14, atol=1e-300)
        np.testing.assert_allclose(O.layer_output(x, a["idx"], a["gates"], 5, ex, sh),
                                   O.layer_output_pp(x, b["idx"], b["gates"], 5, 3, 0, 0, ex, sh, cv),
                                   rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("N,M,C,V", [(2, 1, 1, 1), (3, 2, 2, 0), (2, 0, 1, 2), (1, 2, 1, 1)])
def test_pp_topk_matches_bruteforce_with_ties(N, M, C, V):
    """Quantised logits tie null copies with copy/constant experts and with reals:
    the pool order (reals, null copies, copy, constant) decides them."""
    rng = np.random.default_rng(500 + N + 10 * M + 100 * C + 1000 * V)
    T = 40
    s = rng.integers(-2, 3, size=(T, N + 1 + C + V)).astype(np.float64) / 2.0
    kind, col = O.pool_kinds(N, M, C, V)
    assert kind.tolist() == [0] * N + [1] * M + [2] * C + [3] * V
    for K in range(1, min(4, N + M + C + V) + 1):
        v = O.expanded_pool_pp(s, N, M, C, V)
        for t in range(T):
            assert [v[t, i] for i in range(v.shape[1])] == [s[t, c] for c in col]
        idx = O.topk_pool(v, K)
        for t in range(T):
            assert idx[t].tolist() == _brute_topk(list(v[t]), K), (t, K, v[t])


def test_pp_gates_match_the_masked_topk_procedure():
    """[MPP] Gating: softmax over the K selected logits, zero the zero expert's
    weight, divide by the remaining sum. The direct softmax over the selected
    non-null slots must give the same gates."""
    N, M, C, V, K = 4, 3, 2, 2, 5
    rng = np.random.default_rng(601)
    s = rng.standard_normal((200, N + 1 + C + V))
    s[:, N] += 0.8  # plenty of null slots
    r = O.route_pp(s, N, M, C, V, K)
    sel = np.take_along_axis(r["v"], r["idx"], axis=1)
    g = scipy.special.softmax(sel, axis=1)
    g[(r["idx"] >= N) & (r["idx"] < N + M)] = 0.0
    tot = g.sum(axis=1, keepdims=True)
    g = np.divide(g, tot, out=np.zeros_like(g), where=tot > 0)
    np.testing.assert_allclose(r["gates"], g, rtol=1e-12, atol=1e-15)


def test_pp_copy_and_constant_outputs():
    """A token whose slots are all copy experts gets E_shared(x) + x; all on
    constant expert j (with K = 1), E_shared(x) + c_j; all null, E_shared(x)."""
    N, M, C, V, K = 3, 2, 2, 2, 2
    rng, x, ex, sh, cv = _pp_case(602, 6, 8, N, M, C, V)
    s = np.full((6, N + 1 + C + V), -50.0)
    s[0, N + 1] = s[0, N + 2] = 3.0  # token 0: both copy experts
    s[1, N + 3] = 4.0                # token 1: constant expert 0 (K = 1 below)
    s[2, N] = 5.0                    # token 2: null copies only
    s[3, N + 4] = 2.0                # token 3: constant 1 and one copy
    s[3, N + 1] = 1.0
    ys = O.swiglu(x, *sh)
    r = O.route_pp(s, N, M, C, V, K)
    y = O.layer_output_pp(x, r["idx"], r["gates"], N, M, C, V, ex, sh, cv)
    np.testing.assert_allclose(y[0], ys[0] + x[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y[2], ys[2], rtol=1e-12, atol=1e-12)
    g3 = scipy.special.softmax([2.0, 1.0])
    np.testing.assert_allclose(y[3], ys[3] + g3[0] * cv[1] + g3[1] * x[3], rtol=1e-12, atol=1e-12)
    r1 = O.route_pp(s, N, M, C, V, 1)
    y1 = O.layer_output_pp(x, r1["idx"], r1["gates"], N, M, C, V, ex, sh, cv)
    np.testing.assert_allclose(y1[1], ys[1] + cv[0], rtol=1e-12, atol=1e-12)


def test_pp_copy_expert_mixes_input_and_dense_output():
    """Review page, 为什么用零专家而非复制专家: with copy experts the MoE output is
    (1 - rho) x + rho y_dense. With r reals and c copies selected on equal logits,
    the real gates sum to rho = r/(r+c) and y_dense is the reals' mean output."""
    N, M, C, V, K = 4, 0, 3, 0, 5
    rng, x, ex, sh, cv = _pp_case(603, 5, 8, N, M, C, V)
    s = np.full((5, N + 1 + C + V), -30.0)
    s[:, [0, 2]] = 1.0          # r = 2 reals
    s[:, N + 1:N + 1 + C] = 1.0  # c = 3 copies
    r = O.route_pp(s, N, M, C, V, K)
    y = O.layer_output_pp(x, r["idx"], r["gates"], N, M, C, V, ex, sh, cv) - O.swiglu(x, *sh)
    rho = 2 / 5
    y_dense = (O.swiglu(x, ex[0][0], ex[1][0], ex[2][0]) + O.swiglu(x, ex[0][2], ex[1][2], ex[2][2])) / 2
    np.testing.assert_allclose(y, (1 - rho) * x + rho * y_dense, rtol=1e-12, atol=1e-12)


def test_pp_aux_invariants():
    N, M, C, V, K, T = 6, 4, 2, 3, 4, 300
    rng = np.random.default_rng(604)
    s = rng.standard_normal((T, N + 1 + C + V))
    r = O.route_pp(s, N, M, C, V, K)
    counts, f, P, L_bal, L_z = O.aux_stats(r["idx"], r["p"], r["lse"], N, M)
    assert counts.shape == (N + M + C + V,) and counts.sum() == T * K
    assert abs(P.sum() - 1.0) < 1e-12 and abs(f.sum() - K) < 1e-12
    # null copies still fill in index order; copy/constant counts are plain counts
    assert np.all(np.diff(counts[N:N + M]) <= 0)
    for j in range(C + V):
        assert counts[N + M + j] == int((r["idx"] == N + M + j).sum())
    np.testing.assert_allclose(L_z, np.mean(scipy.special.logsumexp(r["v"], axis=1) ** 2), rtol=1e-12)
