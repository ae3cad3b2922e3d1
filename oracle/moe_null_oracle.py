"""CPU oracle: forward and backward pass of a token-choice MoE layer with zero-compute
null experts.

TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this module. The CUDA library never calls it, and it
shares no code with the CUDA library: it is a plain, slow, float64 NumPy
restatement of what the pages define, so that a reader can check it against
them line by line.

Sources (cited by page title and section):

[KR]  "Improving MoE Compute Efficiency by Composing Weight and Data Sparsity"
      (Kilian et al.), paper-review page, section 三 技术架构 (architecture):
      核心公式 / Token-Choice MoE (layer equation), Null Expert 机制 (null expert,
      M copies of the null logit before top-K, renormalisation over the selected
      real experts), 阈值解释 (threshold reading), 负载均衡损失 (L_bal),
      Z-Loss (L_z), 关键特性 / 解决方案空间保持 (K^4_0.5 reproduces K^2_1.0),
      实现 (argsort moves null indices >= N to the end, truncate, grouped matmul).
[SS]  same paper, sciencestack page: Figure 3 caption (rho = real / all
      selected experts), Figure 4/5 captions (compute intensity = fraction of
      top-K slots filled by real experts).
[T44] "【Transformer 与注意力机制】44｜MoE：稀疏激活的万亿模型路径", section 三
      (router softmax(W_g x), top-k then renormalise over the k), section 4.2
      (aux loss alpha*E*sum f_i P_i), section 4.3 (router z-loss).
[MPP] MoE++ explainer page, section "Gating 机制与残差门控": topk over all
      logits, softmax over the k, zero the zero-compute experts' weights,
      divide by the remaining sum; section "核心创新：三种零计算专家": the zero
      expert outputs nothing, the copy expert returns its input, the constant
      expert replaces it with a learned vector (one per expert, hidden size).

Readings where the pages are silent (each is listed in the design notes):
* pool = N real slots followed by M null copies (indices N..N+M-1); with M = 0
  there is no null slot at all;
* top-K order is (logit descending, pool index ascending); a real logit equal
  to the null logit therefore precedes every copy, and copies fill in index
  order;
* gates are a softmax over the selected real logits; a token with no real
  expert gets only the shared expert;
* the shared expert is ungated; every expert is SwiGLU W_d(silu(W_g z) * W_u z);
* f_i = count_i / T, so sum_i f_i = K; P_i = mean_t p_{t,i} over the pool;
* rows within an expert's segment are in ascending token order (stable argsort).

Parity status: every forward function below is pinned by the CPU tests in
tests/test_oracle_pins.py (brute force, closed forms, textbook reductions,
library routines); every backward function by tests/test_oracle_backward_pins.py
(central finite differences of the forward objective, shift-invariance closed
forms); none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "router_logits", "expanded_pool", "pool_logsumexp", "pool_probs", "topk_pool",
    "threshold_real_count", "renormalised_gates", "dispatch", "swiglu",
    "layer_output", "aux_stats", "aux_partial_sums", "aux_finalize", "route",
    "bf16_round_f64", "expanded_pool_pp", "pool_kinds", "renormalised_gates_pp",
    "layer_output_pp", "route_pp", "swiglu_backward", "gate_backward", "aux_backward",
    "pool_grad_to_logits", "router_backward", "layer_backward", "layer_objective",
]


def router_logits(x, w_router, bias=None, tok_null_bias=None, null_col=None):
    """Router logits s[t, j], j = 0..N (N real experts, then the null logit).

    [KR] 三/Null Expert 机制: the router is widened to N+1 logits, the last one
    belonging to the null expert. [T44] 三: the router is a linear map of the
    token's hidden state. ``bias`` [N+1] is added to every logit; the optional
    per-token ``tok_null_bias`` [T] is added to the null logit only (column
    ``null_col``, by default the last; with MoE++ experts the null logit is
    column N and the copy and constant experts' logits follow it).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_router, dtype=np.float64)
    s = x @ w.T
    if bias is not None:
        s = s + np.asarray(bias, dtype=np.float64)[None, :]
    if tok_null_bias is not None:
        s[:, -1 if null_col is None else null_col] += np.asarray(tok_null_bias, dtype=np.float64)
    return s


def expanded_pool(s, M):
    """The expanded logit vector [s_0..s_{N-1}, s_N repeated M times].

    [KR] 三/Null Expert 机制: the null logit is copied M times before top-K.
    Returns v [T, N+M].
    """
    s = np.asarray(s, dtype=np.float64)
    N = s.shape[1] - 1
    real = s[:, :N]
    if M == 0:
        return real.copy()
    null = np.repeat(s[:, N:N + 1], M, axis=1)
    return np.concatenate([real, null], axis=1)


def pool_logsumexp(v):
    """lse_t = log sum_i exp(v_{t,i}) over the whole pool ([KR] 三/Z-Loss)."""
    v = np.asarray(v, dtype=np.float64)
    m = v.max(axis=1)
    return m + np.log(np.exp(v - m[:, None]).sum(axis=1))


def pool_probs(v, lse):
    """p_{t,i} = exp(v_{t,i} - lse_t): the routing softmax over the pool."""
    return np.exp(np.asarray(v, dtype=np.float64) - np.asarray(lse)[:, None])


def topk_pool(v, K):
    """Top-K pool indices per token, in rank order (value desc, index asc).

    A stable sort of the pool: primary key the value (descending), secondary
    key the pool index (ascending). Returns int64 [T, K].
    """
    v = np.asarray(v, dtype=np.float64)
    T, P = v.shape
    if K > P:
        raise ValueError("K exceeds the pool size N+M")
    index = np.broadcast_to(np.arange(P), v.shape)
    order = np.lexsort((index, -v), axis=-1)
    return order[:, :K].astype(np.int64)


def threshold_real_count(s, M, K):
    """Number of real experts a token selects, from the threshold reading.

    [KR] 三/阈值解释: a token keeps exactly the real experts whose logit beats
    the null logit, the remaining slots going to null copies. With a = #{i < N :
    s_i >= s_null} (ties go to the real expert, whose index is lower), the
    token takes min(K, a) reals first, then up to M null copies, then, only if
    the copies run out, further reals: r = min(K,a) + max(0, K - min(K,a) - M).
    """
    s = np.asarray(s, dtype=np.float64)
    N = s.shape[1] - 1
    a = (s[:, :N] >= s[:, N:N + 1]).sum(axis=1)
    first = np.minimum(K, a)
    return first + np.maximum(0, K - first - M)


def renormalised_gates(s, idx, N):
    """Gate of each selected slot: softmax over the token's selected real logits.

    [KR] 三/Null Expert 机制: routing weights are renormalised over the selected
    real experts only, so null routing does not change the output's magnitude.
    Null slots get weight 0; a token with no real expert gets all zeros.
    Returns float64 [T, K].
    """
    s = np.asarray(s, dtype=np.float64)
    idx = np.asarray(idx)
    T, K = idx.shape
    g = np.zeros((T, K), dtype=np.float64)
    for t in range(T):
        sel = [k for k in range(K) if idx[t, k] < N]
        if not sel:
            continue
        vals = np.array([s[t, idx[t, k]] for k in sel])
        e = np.exp(vals - vals.max())
        g[t, sel] = e / e.sum()
    return g


def dispatch(idx, N):
    """Expert-contiguous list of the real (token, expert) slots.

    [KR] 三/实现: an argsort moves null indices (>= N) to the end and the
    sorted list is truncated before the grouped matmul. The sort here is a
    stable one on (expert, token), so rows inside an expert's segment are in
    ascending token order. Returns counts [N], offsets [N+1], perm_tok [R]
    (token of each row) and slot_row [T, K] (row of each slot, -1 for nulls).
    """
    idx = np.asarray(idx)
    T, K = idx.shape
    tok = np.repeat(np.arange(T), K)
    kk = np.tile(np.arange(K), T)
    e = idx.reshape(-1)
    real = e < N
    tok_r, k_r, e_r = tok[real], kk[real], e[real]
    order = np.lexsort((tok_r, e_r))
    counts = np.bincount(e_r, minlength=N).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    perm_tok = tok_r[order].astype(np.int64)
    slot_row = np.full((T, K), -1, dtype=np.int64)
    slot_row[tok_r[order], k_r[order]] = np.arange(order.size)
    return counts, offsets, perm_tok, slot_row


def bf16_round_f64(a):
    """Round to the nearest bf16 value (ties to even), returned as float64."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def swiglu(z, w_gate, w_up, w_down, round_h=False):
    """One SwiGLU expert E(z) = (silu(z W_g^T) * (z W_u^T)) W_d^T in float64.

    silu(a) = a * sigmoid(a). w_gate, w_up: [F, d]; w_down: [d, F].
    ``round_h`` rounds the hidden activation to bf16 (the CUDA path stores it
    in bf16 between its two matmuls).
    """
    z = np.asarray(z, dtype=np.float64)
    a = z @ np.asarray(w_gate, dtype=np.float64).T
    b = z @ np.asarray(w_up, dtype=np.float64).T
    h = a / (1.0 + np.exp(-a)) * b
    if round_h:
        h = bf16_round_f64(h)
    return h @ np.asarray(w_down, dtype=np.float64).T


def layer_output(x, idx, gates, N, experts, shared, tokens=None, round_h=False):
    """y_t = E_shared(x_t) + sum over the selected real experts of g_i E_i(x_t).

    [KR] 三/核心公式 (Token-Choice MoE): y = E_shared(x) + sum_{i in top-K}
    g_i(x) E_i(x); null experts output zero ([KR] 三/Null Expert 机制), so only
    real slots contribute. ``experts`` = (w_gate [N,F,d], w_up [N,F,d],
    w_down [N,d,F]); ``shared`` = (ws_gate, ws_up, ws_down). ``tokens`` limits
    the computation to a subset of token indices (rows of the result follow
    that order).
    """
    x = np.asarray(x, dtype=np.float64)
    idx = np.asarray(idx)
    gates = np.asarray(gates, dtype=np.float64)
    if tokens is None:
        tokens = np.arange(x.shape[0])
    tokens = np.asarray(tokens)
    xt = x[tokens]
    y = swiglu(xt, *shared, round_h=round_h)
    wg, wu, wd = experts
    sub_idx = idx[tokens]
    sub_g = gates[tokens]
    for e in range(N):
        rows, ks = np.nonzero(sub_idx == e)
        if rows.size == 0:
            continue
        ye = swiglu(xt[rows], wg[e], wu[e], wd[e], round_h=round_h)
        y[rows] += sub_g[rows, ks][:, None] * ye
    return y


def aux_stats(idx, p, lse, N, M):
    """Load-balance and Z-loss statistics over the expanded pool.

    [KR] 三/负载均衡损失: L_bal = N * sum_{i=1}^{N+M} f_i P_i, f_i the fraction
    of tokens routed to slot i (count_i / T), P_i the mean routing probability.
    [KR] 三/Z-Loss: L_z = (1/T) sum_t (log sum_{i=1}^{N+M} exp s_i)^2.
    Returns counts_ext [N+M], f, P, L_bal, L_z.
    """
    idx = np.asarray(idx)
    T = idx.shape[0]
    pool = np.asarray(p).shape[1]  # N + M (+ MoE++ copy and constant experts)
    counts_ext = np.bincount(idx.reshape(-1), minlength=pool)[:pool].astype(np.int64)
    f = counts_ext / float(T)
    P = np.asarray(p, dtype=np.float64).mean(axis=0)
    L_bal = N * float(np.sum(f * P))
    L_z = float(np.mean(np.asarray(lse, dtype=np.float64) ** 2))
    return counts_ext, f, P, L_bal, L_z


def aux_partial_sums(idx, p, lse, N, M):
    """Additive statistics of a token shard, for data-parallel reduction.

    Returns (counts_ext [N+M] int64, sum_t p [N+M] float64, sum_t lse^2, T).
    Summing these over shards and calling :func:`aux_finalize` equals
    :func:`aux_stats` on the concatenated tokens, because f_i and P_i are means
    over all tokens ([KR] 三/负载均衡损失).
    """
    idx = np.asarray(idx)
    pool = np.asarray(p).shape[1]
    counts_ext = np.bincount(idx.reshape(-1), minlength=pool)[:pool].astype(np.int64)
    psum = np.asarray(p, dtype=np.float64).sum(axis=0)
    lsq = float(np.sum(np.asarray(lse, dtype=np.float64) ** 2))
    return counts_ext, psum, lsq, int(idx.shape[0])


def aux_finalize(counts_ext, psum, lsq, T, N):
    """L_bal and L_z from summed statistics (see :func:`aux_partial_sums`)."""
    f = np.asarray(counts_ext, dtype=np.float64) / float(T)
    P = np.asarray(psum, dtype=np.float64) / float(T)
    return f, P, N * float(np.sum(f * P)), float(lsq) / float(T)


def route(s, M, K):
    """All routing outputs from logits s [T, N+1] (float64 or the GPU's fp32).

    Returns a dict with the pool v, lse, p, top-K indices, per-token real count
    ("compute intensity" numerator, [SS] Figure 4/5 captions) and gates.
    """
    s = np.asarray(s, dtype=np.float64)
    N = s.shape[1] - 1
    v = expanded_pool(s, M)
    lse = pool_logsumexp(v)
    p = pool_probs(v, lse)
    idx = topk_pool(v, K)
    n_real = (idx < N).sum(axis=1)
    gates = renormalised_gates(s, idx, N)
    return dict(v=v, lse=lse, p=p, idx=idx, n_real=n_real, gates=gates)


# ---------------------------------------------------------------------------------------
# MoE++ zero-computation experts next to the null expert ([MPP] 核心创新).
#
# Router rows: N real experts, the null logit (column N), C copy experts, V constant
# experts (columns N+1 .. N+C+V). Pool (what top-K ranks): the N reals, the M null
# copies, then the copy and the constant experts (pool indices N+M .. N+M+C+V-1), so
# on equal logits a null copy precedes a copy or constant expert. Gates: softmax over
# the selected slots that are not null copies ([MPP] zeroes only the zero expert's
# weight before renormalising). Outputs: a copy expert returns x, constant expert j
# the vector c_j, a null copy nothing. With C = V = 0 every function below equals its
# null-only counterpart above.


def pool_kinds(N, M, C, V):
    """Kind of each pool slot (0 real, 1 null copy, 2 copy, 3 constant) and the
    router column its logit comes from. Returns two int64 arrays [N+M+C+V]."""
    kind = np.concatenate([np.zeros(N), np.ones(M), np.full(C, 2), np.full(V, 3)]).astype(np.int64)
    col = np.concatenate([np.arange(N), np.full(M, N), N + 1 + np.arange(C + V)]).astype(np.int64)
    return kind, col


def expanded_pool_pp(s, N, M, C, V):
    """The MoE++ pool [s_0..s_{N-1}, s_N x M, s_{N+1}..s_{N+C+V}] from logits [T, N+1+C+V]."""
    s = np.asarray(s, dtype=np.float64)
    _, col = pool_kinds(N, M, C, V)
    return s[:, col]


def renormalised_gates_pp(v, idx, N, M):
    """Gates over the pool: softmax of the selected slots that are not null copies
    (pool index < N or >= N+M); null copies get 0; all 0 if every slot is null."""
    v = np.asarray(v, dtype=np.float64)
    idx = np.asarray(idx)
    T, K = idx.shape
    g = np.zeros((T, K), dtype=np.float64)
    for t in range(T):
        sel = [k for k in range(K) if idx[t, k] < N or idx[t, k] >= N + M]
        if not sel:
            continue
        vals = np.array([v[t, idx[t, k]] for k in sel])
        e = np.exp(vals - vals.max())
        g[t, sel] = e / e.sum()
    return g


def layer_output_pp(x, idx, gates, N, M, C, V, experts, shared, const_vectors, tokens=None,
                    round_h=False):
    """y_t = E_shared(x_t) + sum of g E_i(x_t) over selected reals + g x_t over
    selected copy experts + g c_j over selected constant experts j ([KR] 三/核心公式
    with the [MPP] experts' outputs). ``const_vectors`` [V, d]."""
    x = np.asarray(x, dtype=np.float64)
    idx = np.asarray(idx)
    gates = np.asarray(gates, dtype=np.float64)
    if tokens is None:
        tokens = np.arange(x.shape[0])
    tokens = np.asarray(tokens)
    y = layer_output(x, idx, gates, N, experts, shared, tokens=tokens, round_h=round_h)
    xt = x[tokens]
    sub_idx = idx[tokens]
    sub_g = np.where((sub_idx >= N + M) & (sub_idx < N + M + C), gates[tokens], 0.0)
    y += sub_g.sum(axis=1)[:, None] * xt
    cv = np.asarray(const_vectors, dtype=np.float64).reshape(V, -1) if V else None
    for j in range(V):
        rows, ks = np.nonzero(sub_idx == N + M + C + j)
        if rows.size:
            np.add.at(y, rows, gates[tokens][rows, ks][:, None] * cv[j][None, :])
    return y


def route_pp(s, N, M, C, V, K):
    """All routing outputs of the MoE++ pool from logits s [T, N+1+C+V]."""
    v = expanded_pool_pp(s, N, M, C, V)
    lse = pool_logsumexp(v)
    p = pool_probs(v, lse)
    idx = topk_pool(v, K)
    n_real = (idx < N).sum(axis=1)
    gates = renormalised_gates_pp(v, idx, N, M)
    return dict(v=v, lse=lse, p=p, idx=idx, n_real=n_real, gates=gates)


# ---------------------------------------------------------------------------------------
# Backward pass of the layer.
#
# The objective differentiated is  L = <y, dy> + alpha * L_bal + beta * L_z, with dy the
# upstream gradient of the layer output ([KR] 四 实验结果/训练配置 trains with the load-balance
# and Z losses added at fixed weights, 2e-2 and 1e-3; here the weights are arguments). The
# routing choice (top-K indices) and the load fractions f_i = count_i / T are piecewise
# constant in the logits, so they carry no gradient: the gradient reaches the logits
# through the renormalised gates, through P_i (the pool softmax) in L_bal, and through
# lse in L_z. Every product below is the chain rule written out for one of those terms.


def swiglu_backward(z, w_gate, w_up, w_down, dout):
    """Gradients of E(z) = (silu(z W_g^T) * (z W_u^T)) W_d^T for an upstream dE.

    With a = z W_g^T, b = z W_u^T, sigma = 1/(1+e^{-a}), h = a sigma b:
      dW_d = dE^T h, dh = dE W_d, db = dh * a sigma,
      da = dh * b * sigma (1 + a (1 - sigma))   (derivative of a sigma(a)),
      dW_g = da^T z, dW_u = db^T z, dz = da W_g + db W_u.
    Returns dz [R, d], dW_g [F, d], dW_u [F, d], dW_d [d, F].
    """
    z = np.asarray(z, dtype=np.float64)
    wg = np.asarray(w_gate, dtype=np.float64)
    wu = np.asarray(w_up, dtype=np.float64)
    wd = np.asarray(w_down, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    a = z @ wg.T
    b = z @ wu.T
    sig = 1.0 / (1.0 + np.exp(-a))
    h = a * sig * b
    dwd = dout.T @ h
    dh = dout @ wd
    db = dh * a * sig
    da = dh * b * sig * (1.0 + a * (1.0 - sig))
    return da @ wg + db @ wu, da.T @ z, db.T @ z, dwd


def gate_backward(v, idx, gates, dg, N, M):
    """Pool-logit gradient of the renormalised gates, from dL/dg [T, K].

    The gates of a token are a softmax over the logits of its selected slots that are
    not null copies ([KR] 三/Null Expert 机制; [MPP] for copy and constant experts), so
    for a selected slot i: dL/dv_i = g_i (dL/dg_i - sum_j g_j dL/dg_j). Other slots get 0.
    Returns float64 [T, P].
    """
    v = np.asarray(v, dtype=np.float64)
    idx = np.asarray(idx)
    g = np.asarray(gates, dtype=np.float64)
    dg = np.asarray(dg, dtype=np.float64)
    T, K = idx.shape
    dv = np.zeros(v.shape, dtype=np.float64)
    for t in range(T):
        sel = [k for k in range(K) if idx[t, k] < N or idx[t, k] >= N + M]
        if not sel:
            continue
        mean = sum(g[t, k] * dg[t, k] for k in sel)
        for k in sel:
            dv[t, idx[t, k]] += g[t, k] * (dg[t, k] - mean)
    return dv


def aux_backward(idx, p, lse, N, alpha, beta, counts=None, t_total=None):
    """Pool-logit gradient of alpha * L_bal + beta * L_z.

    [KR] 三/负载均衡损失 and 三/Z-Loss. With f fixed and P_i = mean_t p_{t,i},
    dL_bal/dv_{t,j} = (N/T) p_{t,j} (f_j - sum_i f_i p_{t,i}); with
    L_z = mean_t lse_t^2, dL_z/dv_{t,j} = (2/T) lse_t p_{t,j}. Returns [T, P] for the
    rows given. For one shard of a data-parallel batch, ``counts`` (slot counts over
    the whole batch) and ``t_total`` (its token count) replace this shard's own:
    f and both means run over the whole batch.
    """
    idx = np.asarray(idx)
    p = np.asarray(p, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    T, P = p.shape
    if counts is None:
        counts = np.bincount(idx.reshape(-1), minlength=P)[:P]
    if t_total is not None:
        T = int(t_total)
    f = np.asarray(counts, dtype=np.float64) / float(T)
    fp = (p * f[None, :]).sum(axis=1)
    d_bal = (N / T) * p * (f[None, :] - fp[:, None])
    d_z = (2.0 / T) * lse[:, None] * p
    return alpha * d_bal + beta * d_z


def pool_grad_to_logits(dv, N, M, C=0, V=0):
    """Fold a pool gradient [T, N+M+C+V] onto the router's logit columns [T, N+1+C+V]:
    the M null copies all read column N, so their gradients add up there."""
    dv = np.asarray(dv, dtype=np.float64)
    _, col = pool_kinds(N, M, C, V)
    ds = np.zeros((dv.shape[0], N + 1 + C + V), dtype=np.float64)
    for i, c in enumerate(col):
        ds[:, c] += dv[:, i]
    return ds


def router_backward(x, w_router, ds):
    """Gradients of the router's linear map s = x W_r^T + bias (+ per-token null offset).

    Returns dx [T, d] = ds W_r, dW_r [rows, d] = ds^T x, dbias [rows] = sum_t ds and the
    per-token null-offset gradient ds[:, N] is the caller's (column N of ds).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_router, dtype=np.float64)
    ds = np.asarray(ds, dtype=np.float64)
    return ds @ w, ds.T @ x, ds.sum(axis=0)


def layer_backward(x, s, w_router, N, M, K, experts, shared, dy, alpha, beta,
                   C=0, V=0, const_vectors=None, counts=None, t_total=None):
    """All gradients of L = <y, dy> + alpha L_bal + beta L_z for one layer.

    ``s`` are the forward logits [T, N+1+C+V] (the routing is taken from them, so a
    parity test passes the logits the GPU computed). For one shard of a data-parallel
    batch, ``counts`` and ``t_total`` are the whole batch's slot counts and token count
    (see :func:`aux_backward`). Returns a dict with dx [T, d],
    dg [T, K] (gradient of each slot's gate), ds [T, N+1+C+V] (logit gradient),
    dW_r, dbias, dtnb [T] (null-offset gradient), dW_gate/dW_up [N, F, d],
    dW_down [N, d, F], the shared expert's (dWs_gate, dWs_up, dWs_down) and
    dconst [V, d].
    """
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    T, d = x.shape
    r = route_pp(s, N, M, C, V, K)
    idx, gates = r["idx"], r["gates"]
    wg, wu, wd = (np.asarray(w, dtype=np.float64) for w in experts)
    dx, dwsg, dwsu, dwsd = swiglu_backward(x, *shared, dy)
    dwg = np.zeros_like(wg)
    dwu = np.zeros_like(wu)
    dwd = np.zeros_like(wd)
    dg = np.zeros((T, K), dtype=np.float64)
    for e in range(N):
        rows, ks = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        z = x[rows]
        ye = swiglu(z, wg[e], wu[e], wd[e])
        dg[rows, ks] = (dy[rows] * ye).sum(axis=1)
        dz, dwg[e], dwu[e], dwd[e] = swiglu_backward(z, wg[e], wu[e], wd[e],
                                                     gates[rows, ks][:, None] * dy[rows])
        np.add.at(dx, rows, dz)
    cv = np.asarray(const_vectors, dtype=np.float64).reshape(V, d) if V else np.zeros((0, d))
    dconst = np.zeros((V, d), dtype=np.float64)
    for j in range(C + V):
        rows, ks = np.nonzero(idx == N + M + j)
        if rows.size == 0:
            continue
        if j < C:  # copy expert: output x_t
            dg[rows, ks] = (dy[rows] * x[rows]).sum(axis=1)
            np.add.at(dx, rows, gates[rows, ks][:, None] * dy[rows])
        else:      # constant expert: output c_j
            dg[rows, ks] = dy[rows] @ cv[j - C]
            dconst[j - C] = (gates[rows, ks][:, None] * dy[rows]).sum(axis=0)
    dv = gate_backward(r["v"], idx, gates, dg, N, M) + aux_backward(idx, r["p"], r["lse"], N,
                                                                   alpha, beta, counts, t_total)
    ds = pool_grad_to_logits(dv, N, M, C, V)
    dx_r, dw_r, dbias = router_backward(x, w_router, ds)
    return dict(dx=dx + dx_r, dg=dg, ds=ds, dW_r=dw_r, dbias=dbias, dtnb=ds[:, N].copy(),
                dW_gate=dwg, dW_up=dwu, dW_down=dwd, dWs_gate=dwsg, dWs_up=dwsu,
                dWs_down=dwsd, dconst=dconst, idx=idx, gates=gates)


def layer_objective(x, w_router, bias, tok_null_bias, N, M, K, experts, shared, dy, alpha,
                    beta, C=0, V=0, const_vectors=None):
    """The scalar L = <y, dy> + alpha L_bal + beta L_z that :func:`layer_backward`
    differentiates, computed by the forward functions alone (for finite differences)."""
    null_col = N if (C + V) else None
    s = router_logits(x, w_router, bias, tok_null_bias, null_col=null_col)
    r = route_pp(s, N, M, C, V, K)
    y = layer_output_pp(x, r["idx"], r["gates"], N, M, C, V, experts, shared,
                        const_vectors if V else np.zeros((0, np.asarray(x).shape[1])))
    _, _, _, L_bal, L_z = aux_stats(r["idx"], r["p"], r["lse"], N, M)
    return float(np.sum(y * np.asarray(dy, dtype=np.float64))) + alpha * L_bal + beta * L_z
