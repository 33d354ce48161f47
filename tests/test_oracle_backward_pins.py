"""Pins of the backward oracle against things other than its own formulas: central
finite differences of the (separately pinned) forward oracle, the closed forms of
uniform attention, conservation identities of the softmax, and grouped heads
against replicated K/V heads."""

import numpy as np
import pytest

from oracle import attention_backward, attention_head, attention_head_backward

RNG = np.random.default_rng(20261202)


def loss(q, k, v, do, scale, causal):
    """L = sum(O * dO) with O from the forward oracle: dL/dX is the backward of X for dO."""
    O, _ = attention_head(q, k, v, scale, causal, nq=q.shape[0])
    return float(np.sum(O * do))


@pytest.mark.parametrize("nq,nk,causal", [(7, 9, False), (7, 9, True), (9, 7, True), (6, 6, True), (1, 5, False)])
def test_gradients_match_finite_differences(nq, nk, causal):
    d, scale, h = 5, 0.37, 1e-5
    q, k, v, do = (RNG.standard_normal(s) for s in ((nq, d), (nk, d), (nk, d), (nq, d)))
    dq, dk, dv = attention_head_backward(q, k, v, do, scale, causal)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = loss(args["q"], args["k"], args["v"], do, scale, causal)
            args[name] = xm
            lm = loss(args["q"], args["k"], args["v"], do, scale, causal)
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=f"d{name}")


def test_rows_without_visible_keys_have_zero_gradient():
    # causal, Nq > Nk, bottom-right aligned: the first Nq - Nk rows see nothing
    nq, nk, d = 9, 4, 3
    q, k, v, do = (RNG.standard_normal(s) for s in ((nq, d), (nk, d), (nk, d), (nq, d)))
    dq, dk, dv = attention_head_backward(q, k, v, do, 0.5, True)
    assert np.all(dq[: nq - nk] == 0)
    # and those rows do not reach dK/dV: dropping them changes nothing
    dq2, dk2, dv2 = attention_head_backward(q[nq - nk:], k, v, do[nq - nk:], 0.5, True)
    np.testing.assert_allclose(dk, dk2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, dv2, rtol=0, atol=1e-12)


def test_uniform_attention_closed_forms():
    # Q = 0 gives uniform P = 1/Nk (no mask): dV_j = mean_i... = (1/Nk) sum_i dO_i,
    # dQ_i = (scale/Nk) sum_j (dO_i . (v_j - vbar)) k_j, dK = 0
    nq, nk, d, scale = 5, 8, 4, 0.7
    q = np.zeros((nq, d))
    k, v, do = RNG.standard_normal((nk, d)), RNG.standard_normal((nk, d)), RNG.standard_normal((nq, d))
    dq, dk, dv = attention_head_backward(q, k, v, do, scale, False)
    vbar = v.mean(axis=0)
    for j in range(nk):
        np.testing.assert_allclose(dv[j], do.sum(axis=0) / nk, rtol=1e-12, atol=1e-12)
    for i in range(nq):
        expect = sum(float(do[i] @ (v[j] - vbar)) * k[j] for j in range(nk)) * scale / nk
        np.testing.assert_allclose(dq[i], expect, rtol=1e-10, atol=1e-12)
    assert np.all(np.abs(dk) < 1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_conservation(causal):
    # sum_j P_ij = 1 makes sum_j dS_ij = 0, hence sum_j dK_j = 0; and sum_j dV_j = sum_i dO_i
    nq = nk = 12
    d = 6
    q, k, v, do = (RNG.standard_normal(s) for s in ((nq, d), (nk, d), (nk, d), (nq, d)))
    dq, dk, dv = attention_head_backward(q, k, v, do, 0.4, causal)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), rtol=1e-12, atol=1e-12)


def test_grouped_heads_equal_replicated_heads():
    B, Hq, Hkv, N, d = 1, 4, 2, 10, 4
    q = RNG.standard_normal((B, Hq, N, d))
    do = RNG.standard_normal((B, Hq, N, d))
    k, v = RNG.standard_normal((B, Hkv, N, d)), RNG.standard_normal((B, Hkv, N, d))
    dq, dk, dv = attention_backward(q, k, v, do, 0.5, True)
    rep_k, rep_v = np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1)
    dq_r, dk_r, dv_r = attention_backward(q, rep_k, rep_v, do, 0.5, True)
    np.testing.assert_allclose(dq, dq_r, rtol=1e-12, atol=1e-12)
    for kv in range(Hkv):
        np.testing.assert_allclose(dk[:, kv], dk_r[:, 2 * kv] + dk_r[:, 2 * kv + 1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dv[:, kv], dv_r[:, 2 * kv] + dv_r[:, 2 * kv + 1], rtol=1e-12, atol=1e-12)
