"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Every test here runs on the CPU. The recurrence under test is the gated delta
rule S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
o_t = scale S_t q_t (state S in R^{V x K}, returned as h = S^T), with the
argument list of chunk_gated_delta_rule in the FlashQLA write-up (page 1,
"高级 API 示例"); the gradients are those of chunk_gated_delta_rule_bwd
(page 1, "底层 API"). The pins are chosen so that a dropped term, a wrong sign
or index, or a transposed operand in the oracle fails at least one of them:

* brute-force dense unrolling (ordered products of the per-token transition
  matrices) on tiny inputs with K != V, random h0, unnormalised k;
* hand-worked examples: three tokens forward (tests/golden/worked_example_k2v2.json)
  and two tokens with every gradient (tests/golden/worked_example_grad_k1v1.json);
* closed forms: constant-input scalar recurrence (geometric series), beta=0
  pure decay of h0, g=0 and beta=0 constant state, a reset when exp(g)
  underflows to 0, beta=1 with unit-norm k giving S_t k_t = v_t;
* linearity in (v, h0); varlen and batch rows equal separate calls; GQA equals
  explicitly repeated q/k heads;
* gradients: scalar closed forms, beta=0 closed forms, central finite
  differences of every input, random-direction adjoint identities;
* the dense unrolling and the adjoint identity again over randomly drawn shapes
  (hypothesis): batch or packed sequences with empty ones, T = 0, group sizes
  1-3, any K, V in 1..5.
"""
import json
import math
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_problem(rng, B=1, T=9, Hq=1, Hv=2, K=3, V=4, h0=True, normalise=False):
    q = rng.standard_normal((B, T, Hq, K))
    k = rng.standard_normal((B, T, Hq, K))
    if normalise:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    else:
        k *= 0.6
    v = rng.standard_normal((B, T, Hv, V))
    g = -np.log1p(np.exp(rng.standard_normal((B, T, Hv))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv))))
    H0 = rng.standard_normal((B, Hv, K, V)) * 0.5 if h0 else None
    return q, k, v, g, beta, H0


def unrolled_seq(q, k, v, g, beta, scale, S0):
    """Dense unrolling of one (sequence, head): q,k [T,K], v [T,V], S0 [V,K].

    S_t = S_0 F_1 ... F_t + sum_s beta_s v_s k_s^T F_{s+1} ... F_t with
    F_j = exp(g_j) (I - beta_j k_j k_j^T); every S_t is rebuilt from scratch.
    """
    T, K = k.shape
    F = [math.exp(g[j]) * (np.eye(K) - beta[j] * np.outer(k[j], k[j])) for j in range(T)]

    def prod(a, b):  # F_a ... F_{b-1} (identity when a >= b)
        P = np.eye(K)
        for j in range(a, b):
            P = P @ F[j]
        return P

    o = np.zeros((T, v.shape[1]))
    S = S0
    for t in range(T):
        S = S0 @ prod(0, t + 1)
        for s in range(t + 1):
            S = S + beta[s] * np.outer(v[s], k[s]) @ prod(s + 1, t + 1)
        o[t] = scale * S @ q[t]
    return o, S


def unrolled(q, k, v, g, beta, scale, h0=None, cu=None):
    B, T, Hq, K = q.shape
    Hv, V = v.shape[2:]
    G = Hv // Hq
    if cu is None:
        seqs = [(b, 0, T) for b in range(B)]
    else:
        seqs = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    o = np.zeros((B, T, Hv, V))
    fin = np.zeros((len(seqs), Hv, K, V))
    for n, (b, s0, s1) in enumerate(seqs):
        for h in range(Hv):
            S0 = h0[n, h].T if h0 is not None else np.zeros((V, K))
            if s1 == s0:
                fin[n, h] = S0.T
                continue
            oo, S = unrolled_seq(q[b, s0:s1, h // G], k[b, s0:s1, h // G], v[b, s0:s1, h],
                                 g[b, s0:s1, h], beta[b, s0:s1, h], scale, S0)
            o[b, s0:s1, h] = oo
            fin[n, h] = S.T
    return o, fin


# ------------------------------------------------------------------ forward


@pytest.mark.parametrize("B,Hq,Hv,K,V", [(1, 1, 1, 3, 4), (2, 1, 2, 4, 3), (1, 2, 4, 2, 5)])
def test_fwd_matches_dense_unrolling(oracle_mod, B, Hq, Hv, K, V):
    rng = np.random.default_rng(1)
    q, k, v, g, beta, h0 = rand_problem(rng, B=B, T=11, Hq=Hq, Hv=Hv, K=K, V=V)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 0.7, h0=h0)
    o_ref, fin_ref = unrolled(q, k, v, g, beta, 0.7, h0=h0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fin, fin_ref, rtol=1e-11, atol=1e-12)


def test_fwd_varlen_matches_dense_unrolling(oracle_mod):
    rng = np.random.default_rng(2)
    q, k, v, g, beta, _ = rand_problem(rng, B=1, T=13, Hq=1, Hv=2, K=3, V=2)
    cu = np.array([0, 4, 4, 9, 13], dtype=np.int32)  # includes an empty sequence
    h0 = rng.standard_normal((4, 2, 3, 2))
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 0.5, h0=h0, cu_seqlens=cu)
    o_ref, fin_ref = unrolled(q, k, v, g, beta, 0.5, h0=h0, cu=cu)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fin, fin_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(fin[1], h0[1])  # empty sequence: final = h0


def test_worked_example(oracle_mod):
    with open(os.path.join(HERE, "golden", "worked_example_k2v2.json")) as f:
        ex = json.load(f)
    inp, exp_ = ex["inputs"], ex["expected"]
    q = np.array(inp["q"])[None, :, None, :]
    k = np.array(inp["k"])[None, :, None, :]
    v = np.array(inp["v"])[None, :, None, :]
    g = np.log(np.array(inp["decay"]))[None, :, None]
    beta = np.array(inp["beta"])[None, :, None]
    o, fin = oracle_mod.fwd(q, k, v, g, beta, inp["scale"])
    np.testing.assert_allclose(o[0, :, 0], exp_["o"], atol=ex["tolerance"])
    np.testing.assert_allclose(fin[0, 0], exp_["final_state"], atol=ex["tolerance"])


def test_scalar_constant_inputs_geometric_series(oracle_mod):
    # K=V=1 with constant inputs: s_t = c s_{t-1} + d, c = e^g (1 - b k^2), d = b v k,
    # so s_t = c^t s_0 + d (1 - c^t) / (1 - c) and o_t = scale s_t q.
    T, gg, b, kk, vv, qq, s0, scale = 40, -0.3, 0.7, 0.9, 1.7, -1.3, 0.4, 0.8
    c, d = math.exp(gg) * (1 - b * kk * kk), b * vv * kk
    q = np.full((1, T, 1, 1), qq)
    k = np.full((1, T, 1, 1), kk)
    v = np.full((1, T, 1, 1), vv)
    g = np.full((1, T, 1), gg)
    beta = np.full((1, T, 1), b)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, scale, h0=np.full((1, 1, 1, 1), s0))
    t = np.arange(1, T + 1)
    s = c ** t * s0 + d * (1 - c ** t) / (1 - c)
    np.testing.assert_allclose(o[0, :, 0, 0], scale * s * qq, rtol=1e-12)
    np.testing.assert_allclose(fin[0, 0, 0, 0], s[-1], rtol=1e-12)


def test_beta_zero_is_pure_decay(oracle_mod):
    rng = np.random.default_rng(3)
    q, k, v, g, beta, h0 = rand_problem(rng, B=2, T=10, Hq=2, Hv=2, K=3, V=4)
    beta[:] = 0.0
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 0.9, h0=h0)
    gam = np.cumsum(g, axis=1)  # [B,T,Hv]
    # o_t = scale e^{gamma_t} S_0 q_t with S_0 = h0^T  ->  o[b,t,h,i] = scale e^gam sum_j h0[b,h,j,i] q[b,t,h,j]
    o_ref = 0.9 * np.exp(gam)[..., None] * np.einsum("bhji,bthj->bthi", h0, q)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(fin, np.exp(gam[:, -1])[..., None, None] * h0, rtol=1e-12)


def test_g_zero_beta_zero_constant_state(oracle_mod):
    rng = np.random.default_rng(4)
    q, k, v, g, beta, h0 = rand_problem(rng, B=1, T=8, Hq=1, Hv=1, K=4, V=3)
    g[:] = 0.0
    beta[:] = 0.0
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 1.0, h0=h0)
    np.testing.assert_array_equal(fin, h0)
    np.testing.assert_allclose(o[0, :, 0], q[0, :, 0] @ h0[0, 0], rtol=1e-13)


def test_underflowing_decay_resets_state(oracle_mod):
    # exp(-800) == 0.0 in fp64: the state at t is exactly beta_t v_t k_t^T.
    rng = np.random.default_rng(5)
    q, k, v, g, beta, h0 = rand_problem(rng, B=1, T=6, Hq=1, Hv=1, K=3, V=2)
    g[0, 5, 0] = -800.0
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 1.0, h0=h0)
    S5 = beta[0, 5, 0] * np.outer(v[0, 5, 0], k[0, 5, 0])
    np.testing.assert_allclose(fin[0, 0], S5.T, rtol=1e-14)
    np.testing.assert_allclose(o[0, 5, 0], S5 @ q[0, 5, 0], rtol=1e-14)


def test_beta_one_unit_key_recalls_value(oracle_mod):
    # beta=1, ||k||=1: S_t k_t = v_t. With q_t = k_t the readout is scale * v_t.
    rng = np.random.default_rng(6)
    q, k, v, g, beta, h0 = rand_problem(rng, B=1, T=12, Hq=1, Hv=2, K=5, V=3, normalise=True)
    beta[:] = 1.0
    o, _ = oracle_mod.fwd(k, k, v, g, beta, 0.6, h0=h0)
    np.testing.assert_allclose(o, 0.6 * v, rtol=1e-12, atol=1e-13)


def test_linear_in_v_and_h0(oracle_mod):
    rng = np.random.default_rng(7)
    q, k, v1, g, beta, h1 = rand_problem(rng, B=1, T=9, Hq=1, Hv=2, K=3, V=4)
    v2 = rng.standard_normal(v1.shape)
    h2 = rng.standard_normal(h1.shape)
    a, b = 0.3, -1.7
    o1, f1 = oracle_mod.fwd(q, k, v1, g, beta, 1.0, h0=h1)
    o2, f2 = oracle_mod.fwd(q, k, v2, g, beta, 1.0, h0=h2)
    o3, f3 = oracle_mod.fwd(q, k, a * v1 + b * v2, g, beta, 1.0, h0=a * h1 + b * h2)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(f3, a * f1 + b * f2, rtol=1e-11, atol=1e-12)


def test_batch_rows_and_varlen_equal_separate_calls(oracle_mod):
    rng = np.random.default_rng(8)
    q, k, v, g, beta, h0 = rand_problem(rng, B=3, T=7, Hq=1, Hv=2, K=3, V=2)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 1.0, h0=h0)
    flat = lambda x: x.reshape((1, -1) + x.shape[2:])
    cu = np.array([0, 7, 14, 21], dtype=np.int32)
    o2, fin2 = oracle_mod.fwd(flat(q), flat(k), flat(v), flat(g), flat(beta), 1.0, h0=h0,
                              cu_seqlens=cu)
    np.testing.assert_array_equal(flat(o), o2)
    np.testing.assert_array_equal(fin, fin2)
    for b in range(3):
        ob, fb = oracle_mod.fwd(q[b:b + 1], k[b:b + 1], v[b:b + 1], g[b:b + 1], beta[b:b + 1],
                                1.0, h0=h0[b:b + 1])
        np.testing.assert_array_equal(ob, o[b:b + 1])
        np.testing.assert_array_equal(fb, fin[b:b + 1])


def test_gqa_equals_repeated_heads(oracle_mod):
    rng = np.random.default_rng(9)
    q, k, v, g, beta, h0 = rand_problem(rng, B=1, T=8, Hq=2, Hv=6, K=3, V=2)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 1.0, h0=h0)
    rep = lambda x: np.repeat(x, 3, axis=2)  # head h uses qk head h // 3
    o2, fin2 = oracle_mod.fwd(rep(q), rep(k), v, g, beta, 1.0, h0=h0)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(fin, fin2)
    do = rng.standard_normal(o.shape)
    g1 = oracle_mod.bwd(q, k, v, g, beta, 1.0, do, h0=h0)
    g2 = oracle_mod.bwd(rep(q), rep(k), v, g, beta, 1.0, do, h0=h0)
    np.testing.assert_allclose(g1["dq"], g2["dq"].reshape(1, 8, 2, 3, 3).sum(3), rtol=1e-12)
    np.testing.assert_allclose(g1["dk"], g2["dk"].reshape(1, 8, 2, 3, 3).sum(3), rtol=1e-12)
    for key in ("dv", "dg", "dbeta", "dh0"):
        np.testing.assert_array_equal(g1[key], g2[key])


def test_thread_count_does_not_change_results(oracle_mod):
    rng = np.random.default_rng(10)
    q, k, v, g, beta, h0 = rand_problem(rng, B=2, T=70, Hq=2, Hv=4, K=4, V=3)
    do = rng.standard_normal(v.shape)
    a = oracle_mod.fwd(q, k, v, g, beta, 1.0, h0=h0, nthreads=1)
    b = oracle_mod.fwd(q, k, v, g, beta, 1.0, h0=h0, nthreads=5)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    ga = oracle_mod.bwd(q, k, v, g, beta, 1.0, do, h0=h0, nthreads=1)
    gb = oracle_mod.bwd(q, k, v, g, beta, 1.0, do, h0=h0, nthreads=3)
    for key in ga:
        np.testing.assert_array_equal(ga[key], gb[key])


def test_invalid_arguments_rejected(oracle_mod):
    rng = np.random.default_rng(11)
    q, k, v, g, beta, _ = rand_problem(rng, B=1, T=6, Hq=2, Hv=3, K=2, V=2, h0=False)
    with pytest.raises(ValueError):
        oracle_mod.fwd(q, k, v, g, beta, 1.0)  # Hv % Hq != 0
    q, k, v, g, beta, _ = rand_problem(rng, B=1, T=6, Hq=1, Hv=1, K=2, V=2, h0=False)
    with pytest.raises(ValueError):
        oracle_mod.fwd(q, k, v, g, beta, 1.0, cu_seqlens=np.array([0, 4, 3, 6], np.int32))
    with pytest.raises(ValueError):
        oracle_mod.fwd(q, k, v, g, beta, 1.0, cu_seqlens=np.array([0, 5], np.int32))


# ----------------------------------------------------------------- backward


def loss(oracle_mod, x, scale, d_o, dht, cu=None):
    o, fin = oracle_mod.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], scale, h0=x["h0"],
                            cu_seqlens=cu)
    return float(np.sum(o * d_o) + np.sum(fin * dht))


def test_scalar_single_token_gradients_closed_form(oracle_mod):
    # K=V=1, T=1: S_1 = a s0 (1 - b k^2) + b v k, o = scale S_1 q, L = do*o + dht*S_1.
    s0, gg, b, kk, vv, qq, scale, do, dht = 0.8, -0.4, 0.35, 1.3, -0.9, 0.7, 0.6, 1.1, -0.5
    a = math.exp(gg)
    S1 = a * s0 * (1 - b * kk * kk) + b * vv * kk
    dS = scale * do * qq + dht
    r = oracle_mod.bwd(np.full((1, 1, 1, 1), qq), np.full((1, 1, 1, 1), kk),
                       np.full((1, 1, 1, 1), vv), np.full((1, 1, 1), gg), np.full((1, 1, 1), b),
                       scale, np.full((1, 1, 1, 1), do), dht=np.full((1, 1, 1, 1), dht),
                       h0=np.full((1, 1, 1, 1), s0))
    exp_ = dict(dq=scale * S1 * do, dv=dS * b * kk, dbeta=dS * kk * (vv - a * s0 * kk),
                dk=dS * (b * vv - 2 * a * s0 * b * kk), dg=dS * a * s0 * (1 - b * kk * kk),
                dh0=dS * a * (1 - b * kk * kk))
    for key, val in exp_.items():
        np.testing.assert_allclose(r[key].ravel()[0], val, rtol=1e-13, err_msg=key)


def test_beta_zero_gradients_closed_form(oracle_mod):
    # beta=0: o_t = scale e^{gam_t} S_0 q_t, S_T = e^{gam_T} S_0. Hence
    # dg_j = sum_{t>=j} <do_t, o_t> + <dht, h_T>,
    # dq_t = scale e^{gam_t} S_0^T do_t, dh0 = sum_t scale e^{gam_t} q_t do_t^T + e^{gam_T} dht,
    # dv = 0, dk = 0 (the keys only enter multiplied by beta).
    rng = np.random.default_rng(12)
    q, k, v, g, beta, h0 = rand_problem(rng, B=1, T=9, Hq=1, Hv=1, K=3, V=4)
    beta[:] = 0.0
    d_o = rng.standard_normal(v.shape)
    dht = rng.standard_normal(h0.shape)
    r = oracle_mod.bwd(q, k, v, g, beta, 0.8, d_o, dht=dht, h0=h0)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 0.8, h0=h0)
    per_t = np.sum(o * d_o, axis=-1)[0, :, 0]
    dg_ref = np.cumsum(per_t[::-1])[::-1] + np.sum(fin * dht)
    np.testing.assert_allclose(r["dg"][0, :, 0], dg_ref, rtol=1e-11)
    gam = np.cumsum(g[0, :, 0])
    H = h0[0, 0]  # [K,V], S_0 = H^T
    dq_ref = 0.8 * np.exp(gam)[:, None] * (d_o[0, :, 0] @ H.T)
    np.testing.assert_allclose(r["dq"][0, :, 0], dq_ref, rtol=1e-11)
    dh0_ref = 0.8 * np.einsum("t,tj,ti->ji", np.exp(gam), q[0, :, 0], d_o[0, :, 0]) \
        + np.exp(gam[-1]) * dht[0, 0]
    np.testing.assert_allclose(r["dh0"][0, 0], dh0_ref, rtol=1e-11)
    np.testing.assert_array_equal(r["dv"], 0.0)
    np.testing.assert_array_equal(r["dk"], 0.0)


def test_worked_gradient_example(oracle_mod):
    # two tokens with K = V = 1, gradients derived by hand (tests/golden)
    ex = json.load(open(os.path.join(HERE, "golden", "worked_example_grad_k1v1.json")))
    x, e = ex["inputs"], ex["expected"]
    col = lambda a: np.array(a, dtype=np.float64).reshape(1, -1, 1, 1)  # noqa: E731
    g = np.log(np.array(x["decay"])).reshape(1, -1, 1)
    beta = np.array(x["beta"]).reshape(1, -1, 1)
    h0 = np.full((1, 1, 1, 1), x["h0"])
    o, fin = oracle_mod.fwd(col(x["q"]), col(x["k"]), col(x["v"]), g, beta, x["scale"], h0=h0)
    np.testing.assert_allclose(o.ravel(), e["o"], rtol=0, atol=ex["tolerance"])
    np.testing.assert_allclose(fin.ravel(), [e["final_state"]], rtol=0, atol=ex["tolerance"])
    r = oracle_mod.bwd(col(x["q"]), col(x["k"]), col(x["v"]), g, beta, x["scale"], col(x["do"]),
                       dht=np.full((1, 1, 1, 1), x["dht"]), h0=h0)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        np.testing.assert_allclose(r[name].ravel(), np.ravel(e[name]), rtol=0, atol=ex["tolerance"],
                                   err_msg=name)


@pytest.mark.parametrize("varlen", [False, True])
def test_gradients_match_finite_differences(oracle_mod, varlen):
    rng = np.random.default_rng(13)
    T = 7
    q, k, v, g, beta, h0 = rand_problem(rng, B=1, T=T, Hq=1, Hv=2, K=3, V=2)
    cu = None
    if varlen:
        cu = np.array([0, 3, 3, 7], dtype=np.int32)
        h0 = rng.standard_normal((3, 2, 3, 2))
    x = dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 0.7, h0=h0, cu_seqlens=cu)
    d_o = rng.standard_normal(o.shape)
    dht = rng.standard_normal(fin.shape)
    r = oracle_mod.bwd(q, k, v, g, beta, 0.7, d_o, dht=dht, h0=h0, cu_seqlens=cu)
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")
    eps = 1e-6
    for name, gname in names.items():
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            xp = {n: a.copy() for n, a in x.items()}
            xp[name][idx] += eps
            lp = loss(oracle_mod, xp, 0.7, d_o, dht, cu)
            xp[name][idx] -= 2 * eps
            lm = loss(oracle_mod, xp, 0.7, d_o, dht, cu)
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(r[gname], fd, rtol=1e-6, atol=1e-8, err_msg=gname)


def test_gradients_adjoint_identity_random_direction(oracle_mod):
    # <grad L, dx> equals the directional derivative of L along dx, for every input at once.
    rng = np.random.default_rng(14)
    q, k, v, g, beta, h0 = rand_problem(rng, B=2, T=150, Hq=2, Hv=4, K=6, V=5, normalise=True)
    x = dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 0.4, h0=h0)
    d_o = rng.standard_normal(o.shape)
    dht = rng.standard_normal(fin.shape)
    r = oracle_mod.bwd(q, k, v, g, beta, 0.4, d_o, dht=dht, h0=h0)
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")
    for name, gname in names.items():
        dx = rng.standard_normal(x[name].shape)
        eps = 1e-6
        xp = {n: a.copy() for n, a in x.items()}
        xp[name] = x[name] + eps * dx
        lp = loss(oracle_mod, xp, 0.4, d_o, dht)
        xp[name] = x[name] - eps * dx
        lm = loss(oracle_mod, xp, 0.4, d_o, dht)
        fd = (lp - lm) / (2 * eps)
        an = float(np.sum(r[gname] * dx))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


# ------------------------------------------------------------------ random shapes

from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@st.composite
def shapes(draw):
    Hq = draw(st.integers(1, 2))
    G = draw(st.integers(1, 3))
    K, V = draw(st.integers(1, 5)), draw(st.integers(1, 5))
    varlen = draw(st.booleans())
    if varlen:
        lens = draw(st.lists(st.integers(0, 6), min_size=1, max_size=4))
        return dict(B=1, T=sum(lens), Hq=Hq, Hv=Hq * G, K=K, V=V,
                    cu=np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
    return dict(B=draw(st.integers(1, 2)), T=draw(st.integers(0, 9)), Hq=Hq, Hv=Hq * G, K=K, V=V, cu=None)


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(shapes(), st.integers(0, 2**31 - 1), st.floats(0.1, 2.0))
def test_fwd_matches_dense_unrolling_random_shapes(oracle_mod, s, seed, scale):
    # any batch / packing, group size, K != V, empty sequences and T = 0 included
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, _ = rand_problem(rng, B=s["B"], T=s["T"], Hq=s["Hq"], Hv=s["Hv"], K=s["K"],
                                       V=s["V"], h0=False)
    N = s["B"] if s["cu"] is None else len(s["cu"]) - 1
    h0 = rng.standard_normal((N, s["Hv"], s["K"], s["V"])) * 0.5
    o, fin = oracle_mod.fwd(q, k, v, g, beta, scale, h0=h0, cu_seqlens=s["cu"])
    o_ref, fin_ref = unrolled(q, k, v, g, beta, scale, h0=h0, cu=s["cu"])
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(fin, fin_ref, rtol=1e-10, atol=1e-11)


@settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(shapes(), st.integers(0, 2**31 - 1))
def test_gradients_adjoint_identity_random_shapes(oracle_mod, s, seed):
    # <grad L, dx> equals the central difference of L along a random dx, for every input
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, _ = rand_problem(rng, B=s["B"], T=s["T"], Hq=s["Hq"], Hv=s["Hv"], K=s["K"],
                                       V=s["V"], h0=False)
    N = s["B"] if s["cu"] is None else len(s["cu"]) - 1
    h0 = rng.standard_normal((N, s["Hv"], s["K"], s["V"])) * 0.5
    x = dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)
    o, fin = oracle_mod.fwd(q, k, v, g, beta, 0.6, h0=h0, cu_seqlens=s["cu"])
    d_o, dht = rng.standard_normal(o.shape), rng.standard_normal(fin.shape)
    r = oracle_mod.bwd(q, k, v, g, beta, 0.6, d_o, dht=dht, h0=h0, cu_seqlens=s["cu"])
    for name, gname in dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0").items():
        assert r[gname].shape == x[name].shape, gname
        dx = rng.standard_normal(x[name].shape)
        eps = 1e-6
        lp = loss(oracle_mod, {**x, name: x[name] + eps * dx}, 0.6, d_o, dht, s["cu"])
        lm = loss(oracle_mod, {**x, name: x[name] - eps * dx}, 0.6, d_o, dht, s["cu"])
        fd = (lp - lm) / (2 * eps)
        an = float(np.sum(r[gname] * dx))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
