"""Pins for the fp64 oracle: facts the pages and the mathematics fix.

The pages print no numerical attention example, so the oracle is pinned by
(a) brute force on tiny inputs written as scalar loops with a different
softmax formulation, (b) a library routine (torch's fp64 SDPA), (c) closed
forms (uniform scores, a single key, two keys, causal row 0, a dominant key)
and (d) invariants (softmax rows sum to one, key permutation, GQA equals MHA
with replicated K/V heads, a common key offset, linearity in V), plus the
paging reading (decode equals the last causal row; page placement does not
matter).  Each case is chosen so that a plausible slip in the oracle (a
transposed product, a dropped scale, a wrong mask alignment, a wrong GQA head
map, a missing max shift) fails at least one of them.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention, attention_head, attention_rows, decode_paged, gather_pages
from attn_fwd_05_b200 import synth

RNG = np.random.default_rng(1234)


def randn(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------- brute force

def brute_head(q, k, v, scale, causal):
    """Scalar loops; softmax_j written as 1 / sum_k exp(s_k - s_j) (no max shift)."""
    nq, nk = len(q), len(k)
    O, L = [], []
    for i in range(nq):
        vis = [j for j in range(nk) if (not causal) or j <= i + (nk - nq)]
        if not vis:
            O.append([0.0] * len(v[0]))
            L.append(-math.inf)
            continue
        s = {j: scale * math.fsum(q[i][t] * k[j][t] for t in range(len(q[i]))) for j in vis}
        w = {j: 1.0 / math.fsum(math.exp(s[kk] - s[j]) for kk in vis) for j in vis}
        O.append([math.fsum(w[j] * v[j][c] for j in vis) for c in range(len(v[0]))])
        s0 = s[vis[0]]
        L.append(s0 + math.log(math.fsum(math.exp(s[j] - s0) for j in vis)))
    return np.array(O), np.array(L)


@pytest.mark.parametrize("nq,nk,causal", [(5, 7, False), (5, 7, True), (7, 5, True), (6, 6, True),
                                          (1, 9, False), (4, 1, False)])
def test_brute_force_tiny(nq, nk, causal):
    B, Hq, Hkv, d = 1, 4, 2, 5
    q, k, v = randn(B, Hq, nq, d), randn(B, Hkv, nk, d), randn(B, Hkv, nk, 3)
    scale = 0.7
    O, L = attention(q, k, v, scale, causal, threads=1)
    for h in range(Hq):
        bo, bl = brute_head(q[0, h].tolist(), k[0, h // 2].tolist(), v[0, h // 2].tolist(),
                            scale, causal)
        np.testing.assert_allclose(O[0, h], bo, rtol=0, atol=1e-13)
        np.testing.assert_array_equal(np.isinf(L[0, h]), np.isinf(bl))
        fin = np.isfinite(bl)
        np.testing.assert_allclose(L[0, h][fin], bl[fin], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("Hq,Hkv,N,d,causal", [(4, 4, 33, 16, False), (8, 2, 40, 8, True),
                                               (6, 1, 17, 32, True)])
def test_matches_torch_sdpa_fp64(Hq, Hkv, N, d, causal):
    B = 2
    q, k, v = randn(B, Hq, N, d), randn(B, Hkv, N, d), randn(B, Hkv, N, d)
    scale = 1 / math.sqrt(d)
    O, L = attention(q, k, v, scale, causal, threads=2)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=(Hq != Hkv)).numpy()
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    # LSE against a library logsumexp of the same scores
    G = Hq // Hkv
    kr = np.repeat(k, G, axis=1)
    S = scale * np.einsum("bhqd,bhkd->bhqk", q, kr)
    if causal:
        S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
    ref_lse = torch.logsumexp(torch.from_numpy(S), dim=-1).numpy()
    np.testing.assert_allclose(L, ref_lse, rtol=0, atol=1e-12)


def test_causal_bottom_right_alignment_against_explicit_mask():
    # Nq < Nk: query i sees keys j <= i + (Nk - Nq)  (the reading for a triangular mask)
    B, H, nq, nk, d = 1, 2, 5, 9, 4
    q, k, v = randn(B, H, nq, d), randn(B, H, nk, d), randn(B, H, nk, d)
    mask = torch.zeros(nq, nk, dtype=torch.bool)
    for i in range(nq):
        for j in range(nk):
            mask[i, j] = j <= i + (nk - nq)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x) for x in (q, k, v)), attn_mask=mask, scale=0.5).numpy()
    O, _ = attention(q, k, v, 0.5, True, threads=1)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_give_mean_of_v(causal):
    B, H, N, d = 1, 2, 37, 8
    q = np.zeros((B, H, N, d))
    k, v = randn(B, H, N, d), randn(B, H, N, d)
    O, L = attention(q, k, v, 0.3, causal, threads=1)
    for i in range(N):
        n = i + 1 if causal else N
        np.testing.assert_allclose(O[0, :, i], v[0, :, :n].mean(axis=1), atol=1e-13)
        np.testing.assert_allclose(L[0, :, i], math.log(n), atol=1e-13)


def test_equal_keys_give_mean_of_v():
    B, H, N, d = 1, 1, 20, 6
    q = randn(B, H, N, d)
    k = np.repeat(randn(1, 1, 1, d), N, axis=2)
    v = randn(B, H, N, d)
    O, L = attention(q, k, v, 0.4, False, threads=1)
    np.testing.assert_allclose(O[0, 0], np.broadcast_to(v[0, 0].mean(0), (N, d)), atol=1e-13)
    np.testing.assert_allclose(L[0, 0], 0.4 * q[0, 0] @ k[0, 0, 0] + math.log(N), atol=1e-12)


def test_single_key_returns_its_value():
    B, H, nq, d = 2, 3, 6, 5
    q, k, v = randn(B, H, nq, d), randn(B, H, 1, d), randn(B, H, 1, d)
    O, L = attention(q, k, v, 0.9, False, threads=1)
    np.testing.assert_allclose(O, np.broadcast_to(v, O.shape), atol=1e-14)
    np.testing.assert_allclose(L, 0.9 * np.einsum("bhqd,bhd->bhq", q, k[:, :, 0]), atol=1e-13)


def test_two_keys_closed_form():
    q, k, v = randn(1, 1, 4, 3), randn(1, 1, 2, 3), randn(1, 1, 2, 2)
    scale = 1.3
    O, L = attention(q, k, v, scale, False, threads=1)
    s0 = scale * q[0, 0] @ k[0, 0, 0]
    s1 = scale * q[0, 0] @ k[0, 0, 1]
    w0 = 1.0 / (1.0 + np.exp(s1 - s0))          # logistic function of the score gap
    ref = w0[:, None] * v[0, 0, 0] + (1 - w0)[:, None] * v[0, 0, 1]
    np.testing.assert_allclose(O[0, 0], ref, atol=1e-14)
    np.testing.assert_allclose(L[0, 0], np.logaddexp(s0, s1), atol=1e-13)


def test_causal_row_zero():
    q, k, v = randn(2, 2, 9, 7), randn(2, 2, 9, 7), randn(2, 2, 9, 7)
    O, L = attention(q, k, v, 0.25, True, threads=1)
    np.testing.assert_allclose(O[:, :, 0], v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(L[:, :, 0], 0.25 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]),
                               atol=1e-14)


def test_dominant_key_selects_its_value():
    N, d = 64, 16
    q = randn(1, 1, N, d)
    k = randn(1, 1, N, d) * 0.1
    v = randn(1, 1, N, d)
    jstar = 41
    # row i's query lines up with key jstar much more than with any other key
    k[0, 0, jstar] = 0.0
    q[0, 0, :, 0] = 100.0
    k[0, 0, jstar, 0] = 1.0
    O, _ = attention(q, k, v, 1.0, False, threads=1)
    np.testing.assert_allclose(O[0, 0], np.broadcast_to(v[0, 0, jstar], (N, d)), atol=1e-12)


def test_fully_masked_rows_are_zero_with_minus_inf_lse():
    # Nq > Nk with a bottom-right causal mask: the first Nq - Nk rows see no key
    q, k, v = randn(1, 1, 8, 4), randn(1, 1, 3, 4), randn(1, 1, 3, 4)
    O, L = attention(q, k, v, 1.0, True, threads=1)
    assert np.all(O[0, 0, :5] == 0.0) and np.all(np.isneginf(L[0, 0, :5]))
    assert np.all(np.isfinite(L[0, 0, 5:]))
    np.testing.assert_allclose(O[0, 0, 5], v[0, 0, 0], atol=1e-15)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_sum_to_one(causal):
    q, k, v = randn(30, 8), randn(45, 8), randn(45, 8)
    _, _, P = attention_head(q, k, v, 0.6, causal, rows=np.arange(30), nq=30, want_p=True)
    assert np.all(P >= 0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-12)
    if causal:
        vis = np.arange(45)[None, :] <= np.arange(30)[:, None] + 15
        assert np.all(P[~vis] == 0.0)


def test_key_permutation_invariance():
    q, k, v = randn(1, 2, 12, 6), randn(1, 2, 20, 6), randn(1, 2, 20, 6)
    perm = RNG.permutation(20)
    O1, L1 = attention(q, k, v, 0.5, False, threads=1)
    O2, L2 = attention(q, k[:, :, perm], v[:, :, perm], 0.5, False, threads=1)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(L1, L2, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_replicated_mha(causal):
    B, Hq, Hkv, N, d = 2, 8, 2, 15, 4
    q, k, v = randn(B, Hq, N, d), randn(B, Hkv, N, d), randn(B, Hkv, N, d)
    O1, L1 = attention(q, k, v, 0.5, causal, threads=1)
    G = Hq // Hkv
    O2, L2 = attention(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), 0.5, causal, threads=1)
    np.testing.assert_allclose(O1, O2, atol=1e-14)
    np.testing.assert_allclose(L1, L2, atol=1e-14)
    # contiguous groups (G = 4): query head 3 uses K/V head 0, query head 4 uses K/V head 1
    O_h3, _ = attention(q[:, 3:4], k[:, 0:1], v[:, 0:1], 0.5, causal, threads=1)
    O_h4, _ = attention(q[:, 4:5], k[:, 1:2], v[:, 1:2], 0.5, causal, threads=1)
    np.testing.assert_allclose(O1[:, 3:4], O_h3, atol=1e-14)
    np.testing.assert_allclose(O1[:, 4:5], O_h4, atol=1e-14)


def test_common_key_offset_shifts_only_lse():
    q, k, v = randn(1, 1, 10, 5), randn(1, 1, 14, 5), randn(1, 1, 14, 5)
    u = randn(5)
    O1, L1 = attention(q, k, v, 0.8, True, threads=1)
    O2, L2 = attention(q, k + u, v, 0.8, True, threads=1)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(L2 - L1, 0.8 * (q @ u), atol=1e-12)


def test_linear_in_v():
    q, k = randn(1, 1, 9, 4), randn(1, 1, 11, 4)
    v1, v2 = randn(1, 1, 11, 4), randn(1, 1, 11, 4)
    O1, _ = attention(q, k, v1, 0.5, True, threads=1)
    O2, _ = attention(q, k, v2, 0.5, True, threads=1)
    O3, _ = attention(q, k, 2 * v1 - 3 * v2, 0.5, True, threads=1)
    np.testing.assert_allclose(O3, 2 * O1 - 3 * O2, atol=1e-13)


def test_rows_entry_matches_full():
    q, k, v = randn(1, 4, 50, 8), randn(1, 2, 50, 8), randn(1, 2, 50, 8)
    O, L = attention(q, k, v, 0.35, True, row_block=7, threads=1)
    rows = np.array([0, 3, 17, 49])
    o, lse = attention_rows(q, k, v, 0.35, True, 0, 3, rows)
    np.testing.assert_allclose(o, O[0, 3, rows], atol=1e-14)
    np.testing.assert_allclose(lse, L[0, 3, rows], atol=1e-14)


# ---------------------------------------------------------------- paging

def _paged_case(lens, page_size=4, Hq=4, Hkv=2, d=6, seed=7):
    shape = synth.DecodeShape(S=len(lens), Hq=Hq, Hkv=Hkv, d=d, page_size=page_size,
                              len_lo=1, len_hi=max(lens))
    return synth.decode_inputs(shape, seed, seq_lens=np.array(lens))


def test_gather_pages_token_order():
    page_size, Hkv, d = 4, 2, 3
    lens = [10, 3]
    kv = _paged_case(lens, page_size=page_size, Hkv=Hkv, d=d)
    pool = np.zeros((kv.num_pages, Hkv, page_size, d))
    table = kv.block_table.numpy()
    for s, n in enumerate(lens):
        for t in range(n):                      # token t of sequence s lives in entry t // page_size
            pool[table[s, t // page_size], :, t % page_size, 0] = 1000 * s + t
    for s, n in enumerate(lens):
        seq = gather_pages(pool, table[s], n, page_size)
        assert seq.shape == (Hkv, n, d)
        np.testing.assert_array_equal(seq[0, :, 0], 1000 * s + np.arange(n))
    with pytest.raises(IndexError):
        bad = table[0].copy()
        bad[1] = kv.num_pages
        gather_pages(pool, bad, 10, page_size)


def test_decode_equals_last_causal_row_of_prefill():
    lens = [13, 1, 8]
    kv = _paged_case(lens)
    O, L = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, kv.page_size, 0.45)
    kp, vp = kv.k_pool.double().numpy(), kv.v_pool.double().numpy()
    for s, n in enumerate(lens):
        K = gather_pages(kp, kv.block_table[s].numpy(), n, kv.page_size)[None]
        V = gather_pages(vp, kv.block_table[s].numpy(), n, kv.page_size)[None]
        # a causal prefill over the same n tokens whose last query is this token's query
        qq = np.zeros((1, 4, n, 6))
        qq[0, :, -1] = kv.q[s].double().numpy()
        Op, Lp = attention(qq, K, V, 0.45, True, threads=1)
        np.testing.assert_allclose(O[s], Op[0, :, -1], atol=1e-13)
        np.testing.assert_allclose(L[s], Lp[0, :, -1], atol=1e-13)


def test_decode_invariant_to_page_placement():
    lens = [9, 16, 5]
    kv = _paged_case(lens)
    O1, L1 = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, kv.page_size, 0.5)
    perm = RNG.permutation(kv.num_pages)          # move physical page p to slot perm[p]
    k2 = torch.empty_like(kv.k_pool)
    v2 = torch.empty_like(kv.v_pool)
    k2[torch.from_numpy(perm)] = kv.k_pool
    v2[torch.from_numpy(perm)] = kv.v_pool
    t = kv.block_table.numpy().copy()
    t[t >= 0] = perm[t[t >= 0]]
    O2, L2 = decode_paged(kv.q, k2, v2, torch.from_numpy(t), kv.seq_lens, kv.page_size, 0.5)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_decode_empty_sequence():
    kv = _paged_case([0, 5])
    O, L = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, kv.page_size, 0.5)
    assert np.all(O[0] == 0) and np.all(np.isneginf(L[0])) and np.all(np.isfinite(L[1]))


# ---------------------------------------------------------------- a planted slip is caught

def test_a_transposed_product_would_be_caught():
    """Sanity of the pins themselves: an oracle that forgot the max shift's sign
    or swapped Q and K fails the brute-force comparison."""
    q, k, v = randn(3, 4), randn(5, 4), randn(5, 2)
    bo, _ = brute_head(q.tolist(), k.tolist(), v.tolist(), 0.5, False)
    S = 0.5 * (k @ q.T).T[:, ::-1]  # wrong key order, as a swapped operand would give
    P = np.exp(S - S.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    assert np.abs(P @ v - bo).max() > 1e-3


# ---------------------------------------------------------------- sliding window and block-sparse masks

def _explicit_mask(nq, nk, causal, window=None, block=None):
    m = torch.zeros(nq, nk, dtype=torch.bool)
    for i in range(nq):
        for j in range(nk):
            ok = True
            if causal or window is not None:
                ok = j <= i + (nk - nq)
            if window is not None:
                ok = ok and j > i + (nk - nq) - window
            if block is not None:
                ok = ok and bool(block[i // 128][j // 128])
            m[i, j] = ok
    return m


@pytest.mark.parametrize("nq,nk,w", [(40, 40, 7), (30, 50, 12), (50, 30, 5), (20, 20, 1), (33, 33, 100)])
def test_window_matches_sdpa_with_explicit_mask(nq, nk, w):
    q, k, v = randn(1, 2, nq, 8), randn(1, 2, nk, 8), randn(1, 2, nk, 8)
    mask = _explicit_mask(nq, nk, True, window=w)
    O, L = attention(q, k, v, 0.4, True, window=w, threads=1)
    rows_alive = mask.any(dim=1).numpy()
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x) for x in (q, k, v)), attn_mask=mask, scale=0.4).numpy()
    np.testing.assert_allclose(O[..., rows_alive, :], ref[..., rows_alive, :], atol=1e-12)
    assert np.all(O[..., ~rows_alive, :] == 0) and np.all(np.isneginf(L[..., ~rows_alive]))


def test_window_of_one_returns_own_value_and_wide_window_is_causal():
    q, k, v = randn(1, 1, 20, 6), randn(1, 1, 20, 6), randn(1, 1, 20, 6)
    O, L = attention(q, k, v, 0.5, True, window=1, threads=1)
    np.testing.assert_allclose(O[0, 0], v[0, 0], atol=1e-15)
    np.testing.assert_allclose(L[0, 0], 0.5 * np.einsum("id,id->i", q[0, 0], k[0, 0]), atol=1e-13)
    Ow, Lw = attention(q, k, v, 0.5, True, window=20, threads=1)
    Oc, Lc = attention(q, k, v, 0.5, True, threads=1)
    np.testing.assert_array_equal(Ow, Oc)
    np.testing.assert_array_equal(Lw, Lc)


@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_matches_sdpa_with_explicit_mask(causal):
    nq, nk = 300, 400
    bm = (np.random.default_rng(5).random(((nq + 127) // 128, (nk + 127) // 128)) > 0.4).astype(np.uint8)
    bm[0, 0] = 1
    q, k, v = randn(1, 2, nq, 8), randn(1, 2, nk, 8), randn(1, 2, nk, 8)
    mask = _explicit_mask(nq, nk, causal, block=bm)
    O, L = attention(q, k, v, 0.3, causal, block_mask=bm, threads=1)
    alive = mask.any(dim=1).numpy()
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x) for x in (q, k, v)), attn_mask=mask, scale=0.3).numpy()
    np.testing.assert_allclose(O[..., alive, :], ref[..., alive, :], atol=1e-12)
    assert np.all(O[..., ~alive, :] == 0) and np.all(np.isneginf(L[..., ~alive]))


def test_full_block_mask_is_no_mask():
    q, k, v = randn(1, 1, 200, 4), randn(1, 1, 300, 4), randn(1, 1, 300, 4)
    O1, L1 = attention(q, k, v, 0.3, False, block_mask=np.ones((2, 3), np.uint8), threads=1)
    O2, L2 = attention(q, k, v, 0.3, False, threads=1)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)
