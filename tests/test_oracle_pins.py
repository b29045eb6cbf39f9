"""Pins for the float64 oracle: each test checks the oracle against something
other than itself -- values the pages print, closed forms, invariants, or an
independent algorithm (the explicit O(N^2) masked form) on small inputs.

Sources (page title, section):
  [A] "What Is Linear Attention?" (xutianle.me)
  [B] "Efficient attention variants" (bailixisu.com)
  [C] "LLM inference optimisation (3): Linear Attention" (wangyu.me)
  [D] "Transformers Are RNNs" notes (myhz0606.com)
"""
import numpy as np
import pytest

import oracle


def phi_np(x):
    # ELU(x)+1 written as on [B] §10: max(x,0) + exp(min(x,0)).
    return np.maximum(x, 0) + np.exp(np.minimum(x, 0))


def dense_masked(q, k, v, gamma=1.0, eps=0.0, S0=None, z0=None, apply_phi=True):
    """Explicit causal form for one chain ([B] §10 'dense_kernel_attention';
    [D] multiplicative lower-triangular mask; decay as the weight gamma^(i-j)
    from unrolling [A] §5.1), plus the contribution of a start state, which
    after i+1 writes carries the factor gamma^(i+1)."""
    fq = phi_np(q) if apply_phi else q
    fk = phi_np(k) if apply_phi else k
    N = q.shape[0]
    idx = np.arange(N)
    Gam = np.where(idx[:, None] >= idx[None, :], gamma ** (idx[:, None] - idx[None, :]).clip(min=0), 0.0)
    A = (fq @ fk.T) * Gam
    num = A @ v
    den = A.sum(axis=-1)
    if S0 is not None:
        w = gamma ** (idx + 1.0)
        num = num + w[:, None] * (fq @ S0)
        den = den + w * (fq @ z0)
    return num / (den[:, None] + eps)


def test_hand_example(golden):
    """[B] §5.1: phi(k) = [1,0],[0,1],[1,1]; v = [1,0],[0,2],[3,1];
    phi(q3) = [1,2] -> similarities 1,2,3, weights 1/6,2/6,3/6, o3 = [10/6, 7/6]."""
    rows = golden("hand_example.txt")
    tok = [r for r in rows if r[0] in ("1", "2", "3")]
    fk = np.array([[float(r[1]), float(r[2])] for r in tok])
    v = np.array([[float(r[3]), float(r[4])] for r in tok])
    fq3 = np.array([float(x) for x in next(r for r in rows if r[0] == "q3")[1:]])
    o3_page = np.array([float(x) for x in next(r for r in rows if r[0] == "o3")[1:]])
    sims_page = np.array([float(x) for x in next(r for r in rows if r[0] == "sim")[1:]])
    w_page = np.array([float(x) for x in next(r for r in rows if r[0] == "weights")[1:]])
    q = np.stack([fq3, fq3, fq3])  # only the third output is checked
    o, S, z = oracle.kernelized(q[None, None], fk[None, None], v[None, None], eps=0.0, apply_phi=False)
    np.testing.assert_allclose(o[0, 0, 2], o3_page, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(fk @ fq3, sims_page)
    np.testing.assert_allclose(sims_page / sims_page.sum(), w_page, atol=1e-16)
    # the state path and the explicit weighted sum agree on the same example
    np.testing.assert_allclose(w_page @ v, o3_page, atol=1e-15)


def _page_program_inputs(golden):
    kv = {r[0]: r[1] for r in golden("numpy_program.txt")}
    rng = np.random.default_rng(int(kv["seed"]))
    N, d, dv = int(kv["N"]), int(kv["d"]), int(kv["dv"])
    q = rng.normal(size=(N, d))
    k = rng.normal(size=(N, d))
    v = rng.normal(size=(N, dv))
    return kv, q, k, v


def test_page_program_causal_equivalence(golden):
    """[B] §10: explicit causal kernel form == recurrence at rtol=atol=1e-12 on the
    page's own inputs; the page reports a max abs difference of 4.44e-16."""
    kv, q, k, v = _page_program_inputs(golden)
    o, _, _ = oracle.kernelized(q[None, None], k[None, None], v[None, None], eps=0.0)
    dense = dense_masked(q, k, v)
    np.testing.assert_allclose(o[0, 0], dense, rtol=float(kv["rtol"]), atol=float(kv["atol"]))
    err = np.max(np.abs(o[0, 0] - dense))
    assert err <= 20 * float(kv["reported_max_abs_err"])  # rounding order differs from the page's loop


def test_page_program_no_future_leakage(golden):
    """[B] §10 and §11: change only tokens 8.. (k += 5, v -= 7); the first eight
    outputs must not change (bit for bit: the recurrence has not seen them)."""
    kv, q, k, v = _page_program_inputs(golden)
    t0 = int(kv["perturb_from"])
    k2, v2 = k.copy(), v.copy()
    k2[t0:] += float(kv["k_shift"])
    v2[t0:] += float(kv["v_shift"])
    o1, _, _ = oracle.kernelized(q[None, None], k[None, None], v[None, None], eps=1e-6)
    o2, _, _ = oracle.kernelized(q[None, None], k2[None, None], v2[None, None], eps=1e-6)
    np.testing.assert_array_equal(o1[0, 0, :t0], o2[0, 0, :t0])
    assert not np.allclose(o1[0, 0, t0:], o2[0, 0, t0:])


@pytest.mark.parametrize("B,H,N,d,dv", [(1, 1, 17, 4, 3), (2, 3, 40, 8, 5), (1, 2, 64, 16, 16)])
def test_final_state_closed_form(B, H, N, d, dv):
    """[A] §2 / [C] 'linear_prefill': over the whole sequence the state is
    S = phi(K)^T V and z = sum_j phi(k_j); the last causal output therefore
    equals the non-causal reassociated output phi(q_N)^T S / phi(q_N)^T z
    ([B] §10 reassociation check)."""
    rng = np.random.default_rng(7)
    q = rng.normal(size=(B, H, N, d))
    k = rng.normal(size=(B, H, N, d))
    v = rng.normal(size=(B, H, N, dv))
    o, S, z = oracle.kernelized(q, k, v, eps=0.0)
    fq, fk = phi_np(q), phi_np(k)
    S_ref = np.einsum("bhnd,bhne->bhde", fk, v)
    z_ref = fk.sum(axis=2)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, z_ref, rtol=1e-12, atol=1e-12)
    last = np.einsum("bhd,bhde->bhe", fq[:, :, -1], S_ref) / np.einsum("bhd,bhd->bh", fq[:, :, -1], z_ref)[..., None]
    np.testing.assert_allclose(o[:, :, -1], last, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("eps", [0.0, 1e-6, 0.5])
def test_decay_dense_form_with_start_state(eps):
    """Per-head gamma ([A] §5.1, [B] §7.1): the recurrence equals the explicit
    form with weights gamma^(i-j) under the causal mask, plus a start state
    decayed gamma^(i+1); the normaliser is decayed alike and eps is added to
    the denominator ([D])."""
    rng = np.random.default_rng(11)
    B, H, N, d, dv = 2, 3, 33, 6, 5
    q = rng.normal(size=(B, H, N, d))
    k = rng.normal(size=(B, H, N, d))
    v = rng.normal(size=(B, H, N, dv))
    gamma = np.array([0.5, 0.9, 1.0])
    S0 = rng.normal(size=(B, H, d, dv))
    z0 = np.abs(rng.normal(size=(B, H, d))) + 1.0
    o, S, z = oracle.kernelized(q, k, v, gamma, S0, z0, eps=eps)
    for b in range(B):
        for h in range(H):
            ref = dense_masked(q[b, h], k[b, h], v[b, h], gamma[h], eps, S0[b, h], z0[b, h])
            np.testing.assert_allclose(o[b, h], ref, rtol=1e-11, atol=1e-12)
            w = gamma[h] ** (N - 1 - np.arange(N))
            S_ref = gamma[h] ** N * S0[b, h] + (phi_np(k[b, h]) * w[:, None]).T @ v[b, h]
            np.testing.assert_allclose(S[b, h], S_ref, rtol=1e-12, atol=1e-12)


def test_decay_example_point_99():
    """[B] §7.1: with gamma = 0.99 a record 100 steps old carries the factor
    0.99^100, about 0.366.  One write of e1 (v = 1), then 100 writes of a zero
    key: the state entry is 0.99^100."""
    N = 101
    k = np.zeros((N, 1)); k[0, 0] = 1.0
    v = np.zeros((N, 1)); v[0, 0] = 1.0
    q = np.ones((N, 1))
    _, S, z = oracle.kernelized(q[None, None], k[None, None], v[None, None], np.array([0.99]), eps=0.0, apply_phi=False)
    assert abs(S[0, 0, 0, 0] - 0.99 ** 100) < 1e-15
    assert round(S[0, 0, 0, 0], 3) == 0.366
    assert abs(z[0, 0, 0] - 0.99 ** 100) < 1e-15


def test_delta_example_two_then_five():
    """[B] §7.3: the same unit key written with 2 then 5.  Additive state reads
    7 unnormalised and 3.5 normalised; the delta rule with beta = 1 reads 5."""
    k = np.array([[1.0, 0.0], [1.0, 0.0]])
    v = np.array([[2.0], [5.0]])
    q = k.copy()
    o, S, z = oracle.kernelized(q[None, None], k[None, None], v[None, None], eps=0.0, apply_phi=False)
    assert S[0, 0, 0, 0] == 7.0
    assert o[0, 0, 1, 0] == 3.5
    ones = np.ones((1, 1, 2))
    od, Sd = oracle.gated_delta(q[None, None], k[None, None], v[None, None], ones, ones)
    assert od[0, 0, 1, 0] == 5.0
    # the orthogonal direction is untouched
    assert Sd[0, 0, 1, 0] == 0.0


def test_gated_delta_equals_product_of_transitions():
    """[B] §7.4: merging decay and delta gives
    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T; applying
    those d x d transition matrices explicitly must reproduce the oracle's
    error-on-decayed-state form, outputs o_t = S_t^T q_t included."""
    rng = np.random.default_rng(5)
    B, H, N, d, dv = 1, 2, 24, 5, 3
    q = rng.normal(size=(B, H, N, d))
    k = rng.normal(size=(B, H, N, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(B, H, N, dv))
    alpha = rng.uniform(0.5, 1.0, size=(B, H, N))
    g = rng.uniform(0.0, 1.0, size=(B, H, N))
    S0 = rng.normal(size=(B, H, d, dv))
    o, S = oracle.gated_delta(q, k, v, alpha, g, S0)
    for h in range(H):
        St = S0[0, h].copy()
        for t in range(N):
            kt = k[0, h, t][:, None]
            A = alpha[0, h, t] * (np.eye(d) - g[0, h, t] * kt @ kt.T)
            St = A @ St + g[0, h, t] * kt @ v[0, h, t][None, :]
            np.testing.assert_allclose(o[0, h, t], St.T @ q[0, h, t], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[0, h], St, rtol=1e-12, atol=1e-12)


def test_delta_overwrites_unit_key():
    """[A] §5.2, [C] delta rule: with a unit key and full write strength the
    state's read-back on that key becomes exactly the new value; for g < 1 it
    is the blend (1-g) alpha S_{t-1}^T k_t + g v_t."""
    rng = np.random.default_rng(9)
    N, d, dv = 64, 16, 8
    k = rng.normal(size=(1, 1, N, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(1, 1, N, dv))
    alpha = rng.uniform(0.8, 1.0, size=(1, 1, N))
    o, _ = oracle.gated_delta(k, k, v, alpha, np.ones((1, 1, N)))
    np.testing.assert_allclose(o, v, rtol=1e-12, atol=1e-12)
    g = rng.uniform(0.1, 0.9, size=(1, 1, N))
    q = rng.normal(size=(1, 1, N, d))
    # previous-state read-backs from a run of the prefix
    o_prev_state = np.zeros((N, dv))
    for t in range(1, N):
        _, Sp = oracle.gated_delta(q[:, :, :t], k[:, :, :t], v[:, :, :t], alpha[:, :, :t], g[:, :, :t])
        o_prev_state[t] = Sp[0, 0].T @ k[0, 0, t]
    for t in range(N):
        _, St = oracle.gated_delta(q[:, :, :t + 1], k[:, :, :t + 1], v[:, :, :t + 1], alpha[:, :, :t + 1], g[:, :, :t + 1])
        expect = (1 - g[0, 0, t]) * alpha[0, 0, t] * o_prev_state[t] + g[0, 0, t] * v[0, 0, t]
        np.testing.assert_allclose(St[0, 0].T @ k[0, 0, t], expect, rtol=1e-11, atol=1e-12)


def test_delta_is_gradient_step():
    """[B] §7.3: the delta update (alpha = 1) is one gradient-descent step of
    size beta on L(S) = 1/2 ||S^T k - v||^2; the gradient is taken here by
    central finite differences, independent of any closed form."""
    rng = np.random.default_rng(3)
    d, dv = 4, 3
    S0 = rng.normal(size=(d, dv))
    k = rng.normal(size=d); k /= np.linalg.norm(k)
    v = rng.normal(size=dv)
    beta = 0.37

    def loss(S):
        r = S.T @ k - v
        return 0.5 * float(r @ r)

    grad = np.zeros_like(S0)
    h = 1e-6
    for i in range(d):
        for j in range(dv):
            E = np.zeros_like(S0); E[i, j] = h
            grad[i, j] = (loss(S0 + E) - loss(S0 - E)) / (2 * h)
    _, S1 = oracle.gated_delta(np.zeros((1, 1, 1, d)), k[None, None, None], v[None, None, None],
                               np.ones((1, 1, 1)), np.full((1, 1, 1), beta), S0[None, None])
    np.testing.assert_allclose(S1[0, 0], S0 - beta * grad, rtol=1e-7, atol=1e-8)


def test_decode_step_is_one_recurrence_step():
    """A decode step reads the state after writing the new token
    ([A] §4 order; [B] §5 'write, then read').  Checked against the explicit
    formula o = phi(q)^T (S + phi(k) v^T) / (phi(q)^T (z + phi(k)) + eps)."""
    rng = np.random.default_rng(13)
    Bs, H, d, dv = 3, 2, 8, 6
    S = 0.1 * rng.normal(size=(Bs, H, d, dv))
    z = np.abs(rng.normal(size=(Bs, H, d))) + 1.0
    q = rng.normal(size=(Bs, H, d)); k = rng.normal(size=(Bs, H, d)); v = rng.normal(size=(Bs, H, dv))
    o, S1, z1 = oracle.decode_step(q, k, v, S, z, eps=1e-6)
    fq, fk = phi_np(q), phi_np(k)
    S_ref = S + fk[..., :, None] * v[..., None, :]
    z_ref = z + fk
    o_ref = np.einsum("shd,shde->she", fq, S_ref) / (np.einsum("shd,shd->sh", fq, z_ref)[..., None] + 1e-6)
    np.testing.assert_allclose(S1, S_ref, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(z1, z_ref, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-13)


def test_chained_prefill_equals_prefill_then_decode():
    """State resume: prefill of N tokens == prefill of N-1 tokens continued by
    one decode step from the returned state (the state is the whole cache,
    [A] §6)."""
    rng = np.random.default_rng(17)
    B, H, N, d, dv = 2, 2, 20, 6, 4
    q = rng.normal(size=(B, H, N, d)); k = rng.normal(size=(B, H, N, d)); v = rng.normal(size=(B, H, N, dv))
    o, S, z = oracle.kernelized(q, k, v)
    o1, S1, z1 = oracle.kernelized(q[:, :, :-1], k[:, :, :-1], v[:, :, :-1])
    od, Sd, zd = oracle.decode_step(q[:, :, -1], k[:, :, -1], v[:, :, -1], S1, z1)
    np.testing.assert_allclose(od, o[:, :, -1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sd, S, rtol=1e-12, atol=1e-13)


def test_phi_is_elu_plus_one():
    """[B] §4 / [C] feature(): phi(x) = ELU(x) + 1 with alpha = 1; checked on
    one token with a single unit value against torch's elu."""
    import torch
    x = np.linspace(-30, 30, 241)
    ref = (torch.nn.functional.elu(torch.tensor(x, dtype=torch.float64)) + 1.0).numpy()
    # o_0 = phi(q_0)^T phi(k_0) v / (phi(q_0)^T phi(k_0)) is v; use S instead:
    # with q irrelevant, S = phi(k_0) v^T, so S[:, 0] = phi(x) for v = 1.
    k = x[None, None, None, :]
    _, S, z = oracle.kernelized(np.zeros_like(k), k, np.ones((1, 1, 1, 1)), eps=0.0)
    # torch forms elu as expm1(x) (+1 here), which is exact only in absolute
    # terms for very negative x; exp(x) itself is the reference there.
    np.testing.assert_allclose(S[0, 0, :, 0], ref, rtol=1e-15, atol=4e-16)
    np.testing.assert_allclose(z[0, 0], ref, rtol=1e-15, atol=4e-16)
    neg = x < 0
    np.testing.assert_allclose(S[0, 0, neg, 0], np.exp(x[neg]), rtol=1e-15)


# ---------------------------------------------------------------------------
# Short causal convolution with conv cache ([A] §5.4: x'_t = Conv(x_{t-w:t});
# a "conv cache" keeps the recent tokens' window for decoding).

@pytest.mark.parametrize("W", [1, 2, 4, 5])
def test_conv_equals_numpy_convolve(W):
    # With zero history, output channel c of a chain is the full linear
    # convolution of the channel with its filter, truncated to N (numpy's
    # convolve reverses the kernel, so the filter is passed reversed: the last
    # weight meets the current token).
    rng = np.random.default_rng(7)
    x = rng.standard_normal((2, 3, 37, 6))
    w = rng.standard_normal((3, 6, W))
    y, _ = oracle.causal_conv(x, w)
    for b in range(2):
        for h in range(3):
            for c in range(6):
                ref = np.convolve(x[b, h, :, c], w[h, c, ::-1])[:37]
                np.testing.assert_allclose(y[b, h, :, c], ref, rtol=0, atol=1e-12)


def test_conv_impulse_response():
    # A unit impulse at token t0 of one channel answers with the filter
    # reversed: y_{t0+j} = w[W-1-j] for j < W, and nothing before t0 (causality).
    W, N, t0 = 4, 12, 5
    x = np.zeros((1, 1, N, 2))
    x[0, 0, t0, 1] = 1.0
    w = np.array([[[0.0, 0.0, 0.0, 0.0], [0.5, -1.5, 2.0, 3.0]]])
    y, _ = oracle.causal_conv(x, w)
    expect = np.zeros(N)
    for j in range(W):
        expect[t0 + j] = w[0, 1, W - 1 - j]
    np.testing.assert_array_equal(y[0, 0, :, 1], expect)
    np.testing.assert_array_equal(y[0, 0, :, 0], np.zeros(N))


@pytest.mark.parametrize("n1", [0, 1, 2, 9, 30])
def test_conv_cache_continues_the_sequence(n1):
    # Splitting a sequence anywhere and carrying the cache gives the same outputs
    # and the same final cache as one pass, bit for bit (the same products in the
    # same order); the cache is the last W-1 inputs of the history-extended sequence.
    rng = np.random.default_rng(8)
    W, N = 4, 30
    x = rng.standard_normal((2, 2, N, 5))
    w = rng.standard_normal((2, 5, W))
    c0 = rng.standard_normal((2, 2, W - 1, 5))
    y, c = oracle.causal_conv(x, w, c0)
    ya, ca = oracle.causal_conv(x[:, :, :n1], w, c0)
    yb, cb = oracle.causal_conv(x[:, :, n1:], w, ca)
    np.testing.assert_array_equal(np.concatenate([ya, yb], axis=2), y)
    np.testing.assert_array_equal(cb, c)
    xh = np.concatenate([c0, x], axis=2)
    np.testing.assert_array_equal(c, xh[:, :, -(W - 1):])
    # decoding token by token is the same again
    cc = c0
    for t in range(N):
        yt, cc = oracle.causal_conv(x[:, :, t:t + 1], w, cc)
        np.testing.assert_array_equal(yt[:, :, 0], y[:, :, t])


def test_conv_short_sequence_keeps_old_cache_rows():
    # N < W-1: the new cache still holds W-1-N of the old cache rows, shifted.
    rng = np.random.default_rng(9)
    W = 5
    x = rng.standard_normal((1, 1, 2, 3))
    w = rng.standard_normal((1, 3, W))
    c0 = rng.standard_normal((1, 1, W - 1, 3))
    _, c = oracle.causal_conv(x, w, c0)
    np.testing.assert_array_equal(c[0, 0, :2], c0[0, 0, 2:])
    np.testing.assert_array_equal(c[0, 0, 2:], x[0, 0])


def test_conv_width_one_is_a_channel_scale():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((2, 2, 7, 4))
    w = rng.standard_normal((2, 4, 1))
    y, _ = oracle.causal_conv(x, w)
    np.testing.assert_allclose(y, x * w[None, :, None, :, 0], rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# GLA, per-key-channel gate ([B] §7.2): each entry of alpha_t scales the
# matching row (key channel) of the state, broadcast along the value dimension.

def gla_dense(q, k, v, alpha, S0=None):
    """Unrolled form for one chain: row i of S_t is
    prod_{m<=t} a_m[i] S0[i] + sum_{j<=t} (prod_{j<m<=t} a_m[i]) k_j[i] v_j,
    so o_t = sum_j (q_t * decay_{t,j}) . k_j v_j + (q_t * prod_{m<=t} a_m) S0,
    with the per-channel decay products taken as exp of log-cumsum differences."""
    N, d = q.shape
    L = np.cumsum(np.log(alpha), axis=0)                    # L_t[i] = sum_{m<=t} log a_m[i]
    o = np.zeros((N, v.shape[1]))
    for t in range(N):
        dec = np.exp(L[t][None, :] - L[: t + 1])            # [j, i] = prod_{j<m<=t} a_m[i]
        w = (dec * k[: t + 1]) @ q[t]                       # sum_i q_t[i] dec[j,i] k_j[i]
        o[t] = w @ v[: t + 1]
        if S0 is not None:
            o[t] += (q[t] * np.exp(L[t])) @ S0
    S = (np.exp(L[-1][None, :] - L) * k).T @ v
    if S0 is not None:
        S += np.exp(L[-1])[:, None] * S0
    return o, S


def _gla_inputs(rng, B, H, N, d, dv):
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, H, N, d)) / np.sqrt(d)
    v = rng.standard_normal((B, H, N, dv))
    alpha = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, N, d)) - 2.0))   # in (0, 1)
    return q, k, v, alpha


@pytest.mark.parametrize("with_S0", [False, True])
def test_gla_equals_unrolled_form(with_S0):
    rng = np.random.default_rng(11)
    q, k, v, alpha = _gla_inputs(rng, 2, 2, 23, 5, 3)
    S0 = rng.standard_normal((2, 2, 5, 3)) if with_S0 else None
    o, S = oracle.gla(q, k, v, alpha, S0)
    for b in range(2):
        for h in range(2):
            od, Sd = gla_dense(q[b, h], k[b, h], v[b, h], alpha[b, h], None if S0 is None else S0[b, h])
            np.testing.assert_allclose(o[b, h], od, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(S[b, h], Sd, rtol=1e-10, atol=1e-12)


def test_gla_without_forgetting_is_a_running_sum():
    # alpha = 1: S_t = S0 + sum_{j<=t} k_j v_j^T and o_t = S_t^T q_t.
    rng = np.random.default_rng(12)
    q, k, v, _ = _gla_inputs(rng, 1, 1, 17, 4, 6)
    S0 = rng.standard_normal((1, 1, 4, 6))
    o, S = oracle.gla(q, k, v, np.ones_like(q), S0)
    run = S0[0, 0] + np.cumsum(k[0, 0][:, :, None] * v[0, 0][:, None, :], axis=0)
    np.testing.assert_allclose(o[0, 0], np.einsum("ti,tij->tj", q[0, 0], run), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], run[-1], rtol=1e-12, atol=1e-12)


def test_gla_closed_gate_resets_only_its_channel():
    # a zero gate entry at token t erases key channel i of the state and
    # nothing else: afterwards row i holds exactly k_t[i] v_t, the other rows
    # are those of the run with that entry set to one.
    rng = np.random.default_rng(13)
    q, k, v, alpha = _gla_inputs(rng, 1, 1, 9, 4, 3)
    t, i = 5, 2
    a0 = alpha.copy(); a0[0, 0, t, i] = 0.0
    a1 = alpha.copy(); a1[0, 0, t, i] = 1.0
    _, S0 = oracle.gla(q[:, :, : t + 1], k[:, :, : t + 1], v[:, :, : t + 1], a0[:, :, : t + 1])
    _, S1 = oracle.gla(q[:, :, : t + 1], k[:, :, : t + 1], v[:, :, : t + 1], a1[:, :, : t + 1])
    np.testing.assert_array_equal(S0[0, 0, i], k[0, 0, t, i] * v[0, 0, t])
    rows = [r for r in range(4) if r != i]
    np.testing.assert_array_equal(S0[0, 0, rows], S1[0, 0, rows])


def test_gla_constant_gate_is_the_scalar_decay_form():
    # alpha_t = gamma in every channel: the [B] §7.1 decay recurrence without
    # a normaliser, o_t = sum_{j<=t} gamma^(t-j) (q_t . k_j) v_j.
    rng = np.random.default_rng(14)
    q, k, v, _ = _gla_inputs(rng, 1, 1, 20, 4, 3)
    gamma = 0.9
    o, _ = oracle.gla(q, k, v, np.full_like(q, gamma))
    idx = np.arange(20)
    Gam = np.where(idx[:, None] >= idx[None, :], gamma ** (idx[:, None] - idx[None, :]).clip(min=0), 0.0)
    ref = ((q[0, 0] @ k[0, 0].T) * Gam) @ v[0, 0]
    np.testing.assert_allclose(o[0, 0], ref, rtol=1e-11, atol=1e-12)


def test_empty_sequence_returns_the_start_state():
    """A chain of no tokens has no update to apply: every mode returns its
    start state unchanged (zero without one), which is what a zero-length
    sequence of a padded batch must report."""
    rng = np.random.default_rng(23)
    B, H, d, dv = 2, 3, 4, 5
    e = lambda *s: np.zeros(s)
    S0 = rng.normal(size=(B, H, d, dv))
    z0 = rng.uniform(1, 2, size=(B, H, d))
    gam = np.array([0.9, 0.95, 1.0])
    o, S, z = oracle.kernelized(e(B, H, 0, d), e(B, H, 0, d), e(B, H, 0, dv), gam, S0, z0)
    assert o.shape == (B, H, 0, dv)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_array_equal(z, z0)
    o, S, z = oracle.kernelized(e(B, H, 0, d), e(B, H, 0, d), e(B, H, 0, dv))
    assert not S.any() and not z.any()
    _, S = oracle.gated_delta(e(B, H, 0, d), e(B, H, 0, d), e(B, H, 0, dv), e(B, H, 0), e(B, H, 0), S0)
    np.testing.assert_array_equal(S, S0)
    _, S = oracle.gla(e(B, H, 0, d), e(B, H, 0, d), e(B, H, 0, dv), e(B, H, 0, d), S0)
    np.testing.assert_array_equal(S, S0)
