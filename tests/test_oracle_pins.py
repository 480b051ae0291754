"""Pins for the fp64 oracle, independent of the oracle's own code.

Each test checks the token-by-token oracle (and the chunkwise fp64
re-derivation) against something the recurrence fixes by itself: hand-expanded
closed forms, special cases that reduce to simpler known forms, invariants,
brute-force whole-sequence matrices and central finite differences.  The
recurrence is S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T with
a_t = exp(g_t) and o_t = scale * S_t q_t; the state is stored transposed
(K x V).  Packed documents reset the state (jax-linear-attention 0.1.0, "How it
works"), and one long call equals chained halves with the state carried over
(same page, "Highlights").
"""
import numpy as np
import pytest

import oracle
from oracle import chunked

RNG = np.random.default_rng(1234)


def rand_unit(L, K, V, rng=RNG, gate=0.3, unit_keys=True):
    q = rng.standard_normal((L, K))
    k = rng.standard_normal((L, K))
    if unit_keys:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, V))
    g = -np.log1p(np.exp(rng.standard_normal(L))) * gate
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    return q, k, v, g, beta


def fwd1(q, k, v, g, beta, h0=None, scale=1.0):
    """Oracle forward for one unit given as (L, D) arrays."""
    o, hT = oracle.gdn_fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                           g[None, :, None], beta[None, :, None],
                           h0=None if h0 is None else h0[None, None], scale=scale)
    return o[0, :, 0], hT[0, 0]


def bwd1(q, k, v, g, beta, do, h0=None, dhT=None, scale=1.0):
    r = oracle.gdn_bwd(q[None, :, None], k[None, :, None], v[None, :, None],
                       g[None, :, None], beta[None, :, None], do[None, :, None],
                       h0=None if h0 is None else h0[None, None],
                       dhT=None if dhT is None else dhT[None, None], scale=scale)
    dq, dk, dv, dg, db, dh0 = r
    return dq[0, :, 0], dk[0, :, 0], dv[0, :, 0], dg[0, :, 0], db[0, :, 0], dh0[0, 0]


def test_two_tokens_closed_form_zero_state():
    K, V, s = 3, 2, 0.7
    q, k, v, g, beta = rand_unit(2, K, V, unit_keys=False)
    o, _ = fwd1(q, k, v, g, beta, scale=s)
    a2 = np.exp(g[1])
    o1 = s * beta[0] * (k[0] @ q[0]) * v[0]
    o2 = s * (a2 * beta[0] * (k[0] @ q[1] - beta[1] * (k[0] @ k[1]) * (k[1] @ q[1])) * v[0]
              + beta[1] * (k[1] @ q[1]) * v[1])
    np.testing.assert_allclose(o[0], o1, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(o[1], o2, rtol=1e-13, atol=1e-14)


def test_one_token_closed_form_with_state_orientation():
    # K != V pins the orientation of h0 (stored K x V, S_0 = h0^T).
    K, V, s = 4, 3, 1.3
    q, k, v, g, beta = rand_unit(1, K, V, unit_keys=False)
    h0 = RNG.standard_normal((K, V))
    o, hT = fwd1(q, k, v, g, beta, h0=h0, scale=s)
    S0 = h0.T
    a, b = np.exp(g[0]), beta[0]
    S1 = a * (S0 - b * np.outer(S0 @ k[0], k[0])) + b * np.outer(v[0], k[0])
    np.testing.assert_allclose(o[0], s * (a * (S0 @ q[0] - b * (S0 @ k[0]) * (k[0] @ q[0]))
                                           + b * v[0] * (k[0] @ q[0])), rtol=1e-13)
    np.testing.assert_allclose(hT, S1.T, rtol=1e-13, atol=1e-15)


def test_zero_write_strength():
    L, K, V = 37, 5, 6
    q, k, v, g, beta = rand_unit(L, K, V)
    beta[:] = 0
    o, hT = fwd1(q, k, v, g, beta)
    assert np.all(o == 0) and np.all(hT == 0)
    h0 = RNG.standard_normal((K, V))
    o, hT = fwd1(q, k, v, g, beta, h0=h0, scale=0.5)
    G = np.cumsum(g)
    np.testing.assert_allclose(hT, np.exp(G[-1]) * h0, rtol=1e-13)
    np.testing.assert_allclose(o, 0.5 * np.exp(G)[:, None] * (q @ h0), rtol=1e-12)
    g[:] = 0  # no decay, no write: the state never changes
    o, hT = fwd1(q, k, v, g, beta, h0=h0)
    np.testing.assert_array_equal(hT, h0)
    np.testing.assert_allclose(o, q @ h0, rtol=1e-13, atol=1e-15)


def test_exact_store_unit_strength():
    # beta = 1 with unit keys: after each step S_t k_t = v_t (the delta rule stores exactly).
    L, K, V = 29, 8, 5
    q, k, v, g, beta = rand_unit(L, K, V)
    beta[:] = 1.0
    o, _ = fwd1(k.copy(), k, v, g, beta, h0=RNG.standard_normal((K, V)))
    np.testing.assert_allclose(o, v, rtol=1e-11, atol=1e-12)


def test_orthogonal_keys_reduce_to_gated_linear_attention():
    L = K = 9
    V = 4
    q, _, v, g, beta = rand_unit(L, K, V)
    k = np.eye(K)[:L]
    o, _ = fwd1(q, k, v, g, beta, scale=0.9)
    G = np.cumsum(g)
    ref = np.zeros((L, V))
    for t in range(L):
        for j in range(t + 1):
            ref[t] += np.exp(G[t] - G[j]) * beta[j] * (k[j] @ q[t]) * v[j]
    np.testing.assert_allclose(o, 0.9 * ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("L,K,V", [(23, 6, 7), (70, 256, 128)])
def test_whole_sequence_matrix_form(L, K, V):
    # h0 = 0: U = (I + strict_lower(diag(b) K K^T * Gam))^-1 diag(b) V ; O = lower(Q K^T * Gam) U
    q, k, v, g, beta = rand_unit(L, K, V)
    o, _ = fwd1(q, k, v, g, beta, scale=0.8)
    G = np.cumsum(g)
    Gam = np.zeros((L, L))
    for i in range(L):
        for j in range(i + 1):
            Gam[i, j] = np.exp(G[i] - G[j])
    Lm = np.tril(np.diag(beta) @ k @ k.T * Gam, -1)
    U = np.linalg.inv(np.eye(L) + Lm) @ np.diag(beta) @ v
    O = np.tril(0.8 * q @ k.T * Gam) @ U
    np.testing.assert_allclose(o, O, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("C", [1, 7, 16, 64, 150])
def test_chunked_rederivation_matches_tokens(C):
    L, K, V = 150, 8, 6
    q, k, v, g, beta = rand_unit(L, K, V)
    h0 = RNG.standard_normal((K, V)) * 0.5
    do = RNG.standard_normal((L, V))
    dhT = RNG.standard_normal((K, V)) * 0.3
    o, hT = fwd1(q, k, v, g, beta, h0=h0, scale=0.6)
    oc, hc = chunked.fwd_unit(q, k, v, g, beta, h0, 0.6, C)
    np.testing.assert_allclose(oc, o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(hc, hT, rtol=1e-10, atol=1e-12)
    ref = bwd1(q, k, v, g, beta, do, h0=h0, dhT=dhT, scale=0.6)
    got = chunked.bwd_unit(q, k, v, g, beta, do, h0, dhT, 0.6, C)
    for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-11, err_msg=name)


def test_packed_equals_independent_and_reset_gate():
    lens = [13, 1, 0, 40, 7]
    T, H, K, V = sum(lens), 2, 5, 4
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, T, H, K)); k = rng.standard_normal((1, T, H, K))
    v = rng.standard_normal((1, T, H, V)); g = -rng.random((1, T, H)) * 0.3
    beta = rng.random((1, T, H))
    h0 = rng.standard_normal((len(lens), H, K, V))
    cu = np.cumsum([0] + lens)
    o, hT = oracle.gdn_fwd(q, k, v, g, beta, cu_seqlens=cu, h0=h0, scale=0.7)
    for n in range(len(lens)):
        t0, t1 = cu[n], cu[n + 1]
        on, hn = oracle.gdn_fwd(q[:, t0:t1], k[:, t0:t1], v[:, t0:t1], g[:, t0:t1],
                                beta[:, t0:t1], h0=h0[n:n + 1], scale=0.7)
        np.testing.assert_array_equal(o[:, t0:t1], on)
        np.testing.assert_array_equal(hT[n], hn[0])
    assert np.array_equal(hT[2], h0[2])  # empty document: state passes through
    # A dense row whose log-decay is -1e4 at each document start (exp underflows
    # to exactly 0) equals the packed row with zero initial states.
    o_p, _ = oracle.gdn_fwd(q, k, v, g, beta, cu_seqlens=cu, h0=None)
    g2 = g.copy()
    for n in range(1, len(lens)):
        if lens[n]:
            g2[0, cu[n]] = -1e4
    o_d, _ = oracle.gdn_fwd(q, k, v, g2, beta)
    np.testing.assert_array_equal(o_p, o_d)


def test_chained_halves():
    T, H, K, V = 96, 2, 6, 5
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, T, H, K)); k = rng.standard_normal((2, T, H, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((2, T, H, V)); g = -rng.random((2, T, H)) * 0.1
    beta = rng.random((2, T, H)); h0 = rng.standard_normal((2, H, K, V))
    o, hT = oracle.gdn_fwd(q, k, v, g, beta, h0=h0)
    m = 40
    oa, ha = oracle.gdn_fwd(q[:, :m], k[:, :m], v[:, :m], g[:, :m], beta[:, :m], h0=h0)
    ob, hb = oracle.gdn_fwd(q[:, m:], k[:, m:], v[:, m:], g[:, m:], beta[:, m:], h0=ha)
    np.testing.assert_allclose(np.concatenate([oa, ob], 1), o, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(hb, hT, rtol=1e-13, atol=1e-15)


def test_linearity():
    L, K, V = 31, 5, 4
    q, k, v, g, beta = rand_unit(L, K, V)
    v2 = RNG.standard_normal((L, V))
    h1, h2 = RNG.standard_normal((K, V)), RNG.standard_normal((K, V))
    a, b = 0.37, -1.9
    o1, s1 = fwd1(q, k, v, g, beta, h0=h1)
    o2, s2 = fwd1(q, k, v2, g, beta, h0=h2)
    o3, s3 = fwd1(q, k, a * v + b * v2, g, beta, h0=a * h1 + b * h2)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s3, a * s1 + b * s2, rtol=1e-11, atol=1e-12)
    q2 = RNG.standard_normal((L, K))
    oq, _ = fwd1(a * q + b * q2, k, v, g, beta, h0=h1, scale=0.125)
    oq1, _ = fwd1(q, k, v, g, beta, h0=h1, scale=0.125)
    oq2, _ = fwd1(q2, k, v, g, beta, h0=h1, scale=0.125)
    np.testing.assert_allclose(oq, a * oq1 + b * oq2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(oq1, 0.125 * o1, rtol=1e-12, atol=1e-14)


def _loss_packed(x, cu, do, dhT, scale):
    o, hT = oracle.gdn_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=cu, h0=x["h0"],
                           scale=scale)
    return float(np.sum(o * do) + np.sum(hT * dhT))


def test_backward_directional_derivatives_head_dim_256():
    """At head dim 256 (two packed documents): for a random direction per input,
    the central difference of the loss sum(o . do) + sum(hT . dhT) along it equals
    the oracle's gradient dotted with it."""
    rng = np.random.default_rng(12)
    lens = [40, 31]
    T, H, K, V = sum(lens), 1, 256, 256
    cu = np.cumsum([0] + lens)
    x = dict(q=rng.standard_normal((1, T, H, K)) / 16, k=rng.standard_normal((1, T, H, K)) / 16,
             v=rng.standard_normal((1, T, H, V)), g=-rng.random((1, T, H)) * 0.5,
             beta=rng.random((1, T, H)), h0=rng.standard_normal((2, H, K, V)) * 0.1)
    do = rng.standard_normal((1, T, H, V))
    dhT = rng.standard_normal((2, H, K, V)) * 0.1
    s = 0.7
    dq, dk, dv, dg, db, dh0 = oracle.gdn_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], do,
                                             cu_seqlens=cu, h0=x["h0"], dhT=dhT, scale=s)
    grads = dict(q=dq, k=dk, v=dv, g=dg, beta=db, h0=dh0)
    eps = 1e-5
    for name, gr in grads.items():
        d = rng.standard_normal(x[name].shape)
        xp = {kk: vv.copy() for kk, vv in x.items()}
        xm = {kk: vv.copy() for kk, vv in x.items()}
        xp[name] += eps * d
        xm[name] -= eps * d
        fd = (_loss_packed(xp, cu, do, dhT, s) - _loss_packed(xm, cu, do, dhT, s)) / (2 * eps)
        an = float(np.sum(gr * d))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_finite_differences_and_euler():
    rng = np.random.default_rng(11)
    lens = [12, 9]
    T, H, K, V = sum(lens), 1, 4, 3
    cu = np.cumsum([0] + lens)
    x = dict(q=rng.standard_normal((1, T, H, K)), k=rng.standard_normal((1, T, H, K)) * 0.5,
             v=rng.standard_normal((1, T, H, V)), g=-rng.random((1, T, H)) * 0.5,
             beta=rng.random((1, T, H)), h0=rng.standard_normal((2, H, K, V)) * 0.5)
    do = rng.standard_normal((1, T, H, V))
    dhT = rng.standard_normal((2, H, K, V)) * 0.5
    s = 0.8
    dq, dk, dv, dg, db, dh0 = oracle.gdn_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], do,
                                             cu_seqlens=cu, h0=x["h0"], dhT=dhT, scale=s)
    grads = dict(q=dq, k=dk, v=dv, g=dg, beta=db, h0=dh0)
    eps = 1e-6
    for name, gr in grads.items():
        fd = np.zeros_like(gr)
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (_loss_packed(xp, cu, do, dhT, s) - _loss_packed(xm, cu, do, dhT, s)) / (2 * eps)
        err = np.max(np.abs(fd - gr)) / np.max(np.abs(gr))
        assert err < 1e-7, (name, err)
    o, hT = oracle.gdn_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=cu, h0=x["h0"],
                           scale=s)
    lhs = np.sum(do * o)
    np.testing.assert_allclose(np.sum(dq * x["q"]), lhs, rtol=1e-11)
    np.testing.assert_allclose(np.sum(dv * x["v"]) + np.sum(dh0 * x["h0"]),
                               lhs + np.sum(dhT * hT), rtol=1e-11)


def test_sampled_units_match_full_run():
    rng = np.random.default_rng(5)
    B, T, H, K, V = 2, 33, 3, 4, 5
    q = rng.standard_normal((B, T, H, K)); k = rng.standard_normal((B, T, H, K))
    v = rng.standard_normal((B, T, H, V)); g = -rng.random((B, T, H)); beta = rng.random((B, T, H))
    o, hT = oracle.gdn_fwd(q, k, v, g, beta)
    os_, hs = oracle.gdn_fwd(q, k, v, g, beta, units=[(1, 2), (0, 0)])
    np.testing.assert_array_equal(os_[1, :, 2], o[1, :, 2])
    np.testing.assert_array_equal(hs[0, 0], hT[0, 0])
    assert np.isnan(os_[0, :, 1]).all()


# ---- optional q/k L2 normalisation inside the layer (jax-linear-attention 0.1.0,
# "Quick start": use_qk_l2norm=True; the pages give no formula: x / |x| per token
# and head is the reading taken)
def _l2(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_l2norm_is_identity_on_unit_rows():
    rng = np.random.default_rng(21)
    B, T, H, K, V = 1, 30, 2, 5, 4
    q, k = _l2(rng.standard_normal((B, T, H, K))), _l2(rng.standard_normal((B, T, H, K)))
    v = rng.standard_normal((B, T, H, V)); g = -rng.random((B, T, H)) * 0.3
    beta = rng.random((B, T, H)); h0 = rng.standard_normal((B, H, K, V))
    o0, h0T = oracle.gdn_fwd(q, k, v, g, beta, h0=h0)
    o1, h1T = oracle.gdn_fwd(q, k, v, g, beta, h0=h0, qk_l2norm=True)
    np.testing.assert_allclose(o1, o0, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h1T, h0T, rtol=1e-12, atol=1e-13)


def test_l2norm_scale_invariance_and_zero_rows():
    rng = np.random.default_rng(22)
    B, T, H, K, V = 1, 25, 1, 6, 3
    q, k = rng.standard_normal((B, T, H, K)), rng.standard_normal((B, T, H, K))
    v = rng.standard_normal((B, T, H, V)); g = -rng.random((B, T, H)) * 0.3
    beta = rng.random((B, T, H)); do = rng.standard_normal((B, T, H, V))
    c = np.exp(rng.standard_normal((B, T, H, 1)))  # positive per-row factors
    o, _ = oracle.gdn_fwd(q, k, v, g, beta, qk_l2norm=True)
    oc, _ = oracle.gdn_fwd(q * c, k * c[::-1], v, g, beta, qk_l2norm=True)
    np.testing.assert_allclose(oc, o, rtol=1e-11, atol=1e-12)
    dq, dk, *_ = oracle.gdn_bwd(q, k, v, g, beta, do, qk_l2norm=True)
    dqc, dkc, *_ = oracle.gdn_bwd(q * c, k * c[::-1], v, g, beta, do, qk_l2norm=True)
    np.testing.assert_allclose(dqc * c, dq, rtol=1e-10, atol=1e-12)   # d/d(cx) = (1/c) d/dx
    np.testing.assert_allclose(dkc * c[::-1], dk, rtol=1e-10, atol=1e-12)
    # a zero query row reads nothing; a zero key row writes nothing
    q0, k0 = q.copy(), k.copy()
    q0[0, 7] = 0.0
    k0[0, 3] = 0.0
    oz, _ = oracle.gdn_fwd(q0, k0, v, g, beta, qk_l2norm=True)
    assert np.all(oz[0, 7] == 0.0)
    dqz, dkz, *_ = oracle.gdn_bwd(q0, k0, v, g, beta, do, qk_l2norm=True)
    assert np.all(dqz[0, 7] == 0.0) and np.all(dkz[0, 3] == 0.0)
    # a zero key row acts as a zero write strength (only the decay remains)
    b0 = beta.copy()
    b0[0, 3] = 0.0
    ref, _ = oracle.gdn_fwd(q0, k, v, g, b0, qk_l2norm=True)
    np.testing.assert_allclose(oz, ref, rtol=1e-12, atol=1e-14)


def test_l2norm_backward_finite_differences():
    rng = np.random.default_rng(23)
    lens = [11, 8]
    T, H, K, V = sum(lens), 1, 4, 3
    cu = np.cumsum([0] + lens)
    x = dict(q=rng.standard_normal((1, T, H, K)), k=rng.standard_normal((1, T, H, K)),
             v=rng.standard_normal((1, T, H, V)), g=-rng.random((1, T, H)) * 0.5,
             beta=rng.random((1, T, H)), h0=rng.standard_normal((2, H, K, V)) * 0.5)
    do = rng.standard_normal((1, T, H, V)); dhT = rng.standard_normal((2, H, K, V)) * 0.5

    def loss(y):
        o, hT = oracle.gdn_fwd(y["q"], y["k"], y["v"], y["g"], y["beta"], cu_seqlens=cu,
                               h0=y["h0"], scale=0.7, qk_l2norm=True)
        return float(np.sum(o * do) + np.sum(hT * dhT))

    dq, dk, dv, dg, db, dh0 = oracle.gdn_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], do,
                                             cu_seqlens=cu, h0=x["h0"], dhT=dhT, scale=0.7,
                                             qk_l2norm=True)
    eps = 1e-6
    for name, gr in dict(q=dq, k=dk, v=dv, g=dg, beta=db, h0=dh0).items():
        fd = np.zeros_like(gr)
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (loss(xp) - loss(xm)) / (2 * eps)
        err = np.max(np.abs(fd - gr)) / np.max(np.abs(gr))
        assert err < 1e-7, (name, err)
    # rows of dq and dk are orthogonal to their q and k rows (scale invariance)
    np.testing.assert_allclose(np.sum(dq * x["q"], axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose(np.sum(dk * x["k"], axis=-1), 0.0, atol=1e-12)
