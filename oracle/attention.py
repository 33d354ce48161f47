"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code, table or helper with the CUDA
library; the only thing the two sides have in common is the seeded input
generator that hands both of them the same bf16 tensors.

Sources (web pages, cited by title and section):

[FA-glossary]  polydesk.ai glossary, "FlashAttention", section
               "Le goulot d'étranglement de l'attention standard": the formula
               Attention(Q,K,V) = softmax(Q K^T / sqrt(d)) V and the naive
               implementation that writes the N x N matrix S, re-reads it for
               the softmax and again for the product with V.
[85pct-VRAM]   patricehuetz.fr, "Flash Attention : pourquoi ton GPU utilise 85%
               de VRAM", section "L'attention classique en 3 étapes": the same
               formula as three materialised steps, S = Q K^T of shape
               [batch, n_heads, seq_len, seq_len], P = softmax(S / sqrt(d)),
               O = P V of shape [batch, n_heads, seq_len, head_dim].
[FA-PA]        ranksignal.fr, "FlashAttention et PagedAttention : à quoi
               servent-elles ?", sections "FlashAttention : calculer sur le plan
               de travail" (the formula, with sqrt(d_k)), "Le cache KV, ce
               locataire qui grossit" (past keys/values are kept and the new
               token attends to them) and "PagedAttention : ranger par pages"
               (the KV cache stored in fixed-size pages found through a table).
[Variantes]    analyticslegends.ai, "Variantes d'attention", glossary entries
               GQA / MQA / MHA: H_q query heads share H_kv < H_q groups of K/V.
[FA-glossary §vs] "FlashAttention vs attention standard": the tiled method
               returns the same result as this one up to floating-point rounding,
               which is what makes a plain materialising implementation the
               right reference.

Readings where the pages are silent (each one is listed in the design notes):

* scale is passed explicitly; every workload uses 1/sqrt(d) (d_k = d_v = d).
* causal: key j is visible to query i iff j <= i + (Nk - Nq), i.e. the mask is
  aligned to the bottom-right corner; the pages only say a triangular mask is
  supported.  With Nq == Nk this is the usual j <= i.
* a query row with no visible key returns O = 0 and LSE = -inf.
* sliding window of w tokens (ranksignal.fr, "Trois idées reçues à écarter": attend
  only to the last w tokens; polydesk.ai glossary, "FlashAttention et attention
  block-sparse": a sliding window is one of the block patterns): key j is visible to
  query i iff i' - w < j <= i' with i' = i + (Nk - Nq), the same bottom-right alignment
  as the causal mask.
* block-sparse mask (same glossary section: a mask over blocks of tokens says which
  blocks attend to each other): blocks of 128 queries by 128 keys; block_mask[bq][bk]
  nonzero means the queries of block bq see the keys of block bk; one mask for every
  batch and head; optionally intersected with the causal mask.
* LSE is the natural log of sum_j exp(scale * q.k_j) over visible keys.
* GQA: query head h uses K/V head h // (Hq / Hkv) (contiguous groups).
* paging: row s of the block table lists the pool pages of sequence s in
  token order; entry i holds tokens [i*page_size, (i+1)*page_size); the last
  page may be partly used; entries past ceil(len/page_size) are ignored; the
  pool is laid out [num_pages, Hkv, page_size, d].  The decode query attends to
  all seq_len cached tokens, its own included, with no mask.

Precision: inputs are bf16 values widened exactly to float64; every step runs
in float64.  Nothing here is blocked, fused or reordered: each query row's
scores are materialised in full, then its probabilities, then its output.
Rows are processed in groups only to bound memory; rows are independent, so
grouping does not change any value.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

try:  # numpy's BLAS threads would oversubscribe the per-head thread pool
    from threadpoolctl import threadpool_limits
except Exception:  # pragma: no cover - threadpoolctl is optional
    threadpool_limits = None


def as_f64(x) -> np.ndarray:
    """Widen a bf16/fp32 torch tensor or numpy array to float64 (exact for bf16)."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def causal_visible(rows: np.ndarray, nq: int, nk: int) -> np.ndarray:
    """Boolean [len(rows), nk]: key j is visible to query i iff j <= i + (nk - nq)."""
    i = np.asarray(rows)[:, None]
    j = np.arange(nk)[None, :]
    return j <= i + (nk - nq)


MASK_BLOCK = 128  # block size of the block-sparse reading


def visible_mask(rows: np.ndarray, nq: int, nk: int, causal: bool, window: int | None = None,
                 block_mask=None) -> np.ndarray | None:
    """Boolean [len(rows), nk] of visible keys, or None when every key is visible.

    causal: j <= i + (nk - nq).  window: additionally j > i + (nk - nq) - window.
    block_mask: [ceil(nq/128), ceil(nk/128)], nonzero = the block pair attends.
    """
    rows = np.asarray(rows)
    vis = None
    if causal or window is not None:
        vis = causal_visible(rows, nq, nk)
    if window is not None:
        j = np.arange(nk)[None, :]
        vis = vis & (j > rows[:, None] + (nk - nq) - window)
    if block_mask is not None:
        bm = np.asarray(block_mask) != 0
        blk = bm[(rows // MASK_BLOCK)[:, None], (np.arange(nk) // MASK_BLOCK)[None, :]]
        vis = blk if vis is None else (vis & blk)
    return vis


def attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, causal: bool,
                   rows: np.ndarray | None = None, nq: int | None = None,
                   want_p: bool = False, window: int | None = None, block_mask=None):
    """One head: the three materialised steps of [85pct-VRAM] "L'attention classique en 3 étapes".

    q: [R, d] query rows (absolute row indices ``rows`` among ``nq`` queries),
    k: [Nk, d], v: [Nk, dv], all float64.
    Returns O [R, dv], LSE [R] and, if asked, P [R, Nk].
    """
    R = q.shape[0]
    nk = k.shape[0]
    if rows is None:
        rows = np.arange(R)
    if nq is None:
        nq = R
    # step 1: scores S = scale * Q K^T  ([FA-glossary] formula; [FA-PA] uses sqrt(d_k))
    S = scale * (q @ k.T)
    vis = visible_mask(rows, nq, nk, causal, window, block_mask)
    if vis is not None:
        S = np.where(vis, S, -np.inf)
    # step 2: P = softmax(S) along each row, with the row maximum taken out first
    rowmax = S.max(axis=1) if nk > 0 else np.full(R, -np.inf)
    alive = np.isfinite(rowmax)              # rows with at least one visible key
    shift = np.where(alive, rowmax, 0.0)
    E = np.exp(S - shift[:, None])           # exp(-inf) = 0 for masked keys
    rowsum = E.sum(axis=1)
    P = np.zeros_like(E)
    P[alive] = E[alive] / rowsum[alive, None]
    # step 3: O = P V
    O = P @ v
    with np.errstate(divide="ignore"):
        LSE = np.where(alive, shift + np.log(np.where(alive, rowsum, 1.0)), -np.inf)
    if want_p:
        return O, LSE, P
    return O, LSE


def _head_job(args):
    q, k, v, scale, causal, row_block, window, block_mask = args
    nq = q.shape[0]
    O = np.empty((nq, v.shape[1]))
    L = np.empty(nq)
    for r0 in range(0, nq, row_block):
        rows = np.arange(r0, min(nq, r0 + row_block))
        O[rows], L[rows] = attention_head(q[rows], k, v, scale, causal, rows=rows, nq=nq, window=window,
                                          block_mask=block_mask)
    return O, L


def kv_head_of(hq: int, Hq: int, Hkv: int) -> int:
    """GQA head mapping ([Variantes] glossary, GQA): contiguous groups of Hq/Hkv query heads."""
    return hq // (Hq // Hkv)


def attention(q, k, v, scale: float, causal: bool, row_block: int = 512,
              threads: int | None = None, window: int | None = None, block_mask=None):
    """Full attention. q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] (bf16 tensors or arrays).

    Returns O [B,Hq,Nq,d] and LSE [B,Hq,Nq] as float64 arrays.  Heads run on a
    thread pool; each head is the plain routine above.  ``window`` and ``block_mask``
    add the sliding-window and block-sparse masks described in the module notes.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, Hq, Nq, _ = q.shape
    Hkv = k.shape[1]
    assert Hq % Hkv == 0, "Hq must be a multiple of Hkv"
    if block_mask is not None and hasattr(block_mask, "cpu"):
        block_mask = block_mask.cpu().numpy()
    jobs = [(q[b, h], k[b, kv_head_of(h, Hq, Hkv)], v[b, kv_head_of(h, Hq, Hkv)],
             scale, causal, row_block, window, block_mask) for b in range(B) for h in range(Hq)]
    threads = threads or os.cpu_count() or 1
    if threads > 1 and len(jobs) > 1:
        ctx = threadpool_limits(1) if threadpool_limits is not None else _nullctx()
        with ctx, ThreadPoolExecutor(max_workers=threads) as ex:
            res = list(ex.map(_head_job, jobs))
    else:
        res = [_head_job(j) for j in jobs]
    O = np.stack([r[0] for r in res]).reshape(B, Hq, Nq, v.shape[-1])
    L = np.stack([r[1] for r in res]).reshape(B, Hq, Nq)
    return O, L


def attention_rows(q, k, v, scale: float, causal: bool, b: int, hq: int, rows, window=None, block_mask=None):
    """Selected query rows of one (batch, head), computed one by one from the full K/V.

    Used to check sampled outputs of full-size runs.  Same arithmetic as
    ``attention``; rows are independent.
    """
    rows = np.asarray(rows)
    Hq, Nq = q.shape[1], q.shape[2]
    Hkv = k.shape[1]
    kv = kv_head_of(hq, Hq, Hkv)
    qr = as_f64(q[b, hq][rows])
    kk = as_f64(k[b, kv])
    vv = as_f64(v[b, kv])
    return attention_head(qr, kk, vv, scale, causal, rows=rows, nq=Nq, window=window, block_mask=block_mask)


class _nullctx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


# ----------------------------------------------------------------------------
# Paged-KV decode ([FA-PA] "Le cache KV, ce locataire qui grossit" and
# "PagedAttention : ranger par pages plutôt que d'un seul tenant")
# ----------------------------------------------------------------------------

def _pages_f64(pool, ids: np.ndarray) -> np.ndarray:
    """pool[ids] widened to float64; only the selected pages are converted."""
    if hasattr(pool, "detach"):
        import torch
        return as_f64(pool[torch.as_tensor(ids, dtype=torch.long)])
    return np.asarray(pool)[ids].astype(np.float64)


def gather_pages(pool, table_row, seq_len: int, page_size: int) -> np.ndarray:
    """Rebuild one sequence's contiguous cache [Hkv, seq_len, d] (float64) from its pages.

    pool: [num_pages, Hkv, page_size, d]; entry i of the table row holds tokens
    [i*page_size, (i+1)*page_size).  Raises on a page id outside the pool.
    """
    npages = (seq_len + page_size - 1) // page_size
    ids = np.asarray(table_row[:npages], dtype=np.int64)
    if npages and (ids.min() < 0 or ids.max() >= pool.shape[0]):
        raise IndexError("block table entry outside the page pool")
    pages = _pages_f64(pool, ids)                       # [npages, Hkv, page_size, d]
    Hkv, d = pool.shape[1], pool.shape[3]
    seq = pages.transpose(1, 0, 2, 3).reshape(Hkv, npages * page_size, d)
    return seq[:, :seq_len]


def decode_paged(q, k_pool, v_pool, block_table, seq_lens, page_size: int, scale: float,
                 seqs=None):
    """One decode step: each sequence's single query token attends to its whole cache.

    q [S,Hq,d]; pools [num_pages,Hkv,page_size,d]; block_table [S,max_pages];
    seq_lens [S].  Returns O [S,Hq,d], LSE [S,Hq] in float64 (only for ``seqs``
    if given, in that order).
    """
    qf = as_f64(q)
    table = np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table)
    lens = np.asarray(seq_lens.cpu() if hasattr(seq_lens, "cpu") else seq_lens)
    S, Hq, d = qf.shape
    Hkv = k_pool.shape[1]
    seqs = range(S) if seqs is None else list(seqs)
    O = np.zeros((len(seqs), Hq, d))
    L = np.full((len(seqs), Hq), -np.inf)
    for n, s in enumerate(seqs):
        ln = int(lens[s])
        if ln <= 0:
            continue
        K = gather_pages(k_pool, table[s], ln, page_size)
        V = gather_pages(v_pool, table[s], ln, page_size)
        for h in range(Hq):
            kv = kv_head_of(h, Hq, Hkv)
            o, l = attention_head(qf[s, h][None], K[kv], V[kv], scale, causal=False)
            O[n, h], L[n, h] = o[0], l[0]
    return O, L
