"""fp64 CPU oracle for the gradients of exact attention (the backward pass).

TEST INFRASTRUCTURE ONLY, like the rest of this package: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may call it, and it
shares no code with the CUDA library.

What it computes.  The forward pass of ``attention.py`` is three materialised steps
(patricehuetz.fr, "Flash Attention : pourquoi ton GPU utilise 85% de VRAM", section
"L'attention classique en 3 étapes"): S = scale Q K^T with the mask applied,
P = softmax(S) row by row, O = P V.  The pages name the backward pass only through
how the tiled method runs it: the score matrix is never stored by the forward pass
and is recomputed block by block during the backward pass (same page, section "Ce
que fait Flash Attention", the second of its two ideas); the polydesk.ai glossary
"FlashAttention", section on FlashAttention-4, names shared-memory traffic as the
backward pass's bottleneck on Blackwell.  The pages give no formulas for it, so
this oracle is the plain definition: the gradient of the three steps by the chain
rule, for an upstream gradient dO of O,

    dV    = P^T dO
    dP    = dO V^T
    dS_ij = P_ij (dP_ij - Delta_i),   Delta_i = sum_j P_ij dP_ij = dO_i . O_i
    dQ    = scale dS K
    dK    = scale dS^T Q

(the softmax Jacobian diag(p) - p p^T applied row by row), with masked entries of
P equal to 0 and rows without a visible key giving zero gradients.  With grouped
heads (Hq/Hkv query heads per K/V head, contiguous groups) dK and dV of a K/V head
are the sums over its query heads.  Every step runs in float64 on the exactly
widened bf16 inputs; nothing is blocked, fused or reordered.

Pins (tests/test_oracle_backward_pins.py): central finite differences of the pinned
forward oracle, the closed forms of uniform attention, sum_j dK_j = 0 and
sum_j dV_j = sum_i dO_i, grouped heads against replicated K/V heads, and the
causal last key.
"""

from __future__ import annotations

import numpy as np

from .attention import as_f64, kv_head_of, visible_mask


def attention_head_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray, scale: float,
                            causal: bool, want_parts: bool = False):
    """One head.  q, do: [Nq, d]; k, v: [Nk, d]; float64.  Returns dq, dk, dv
    (and, if asked, the materialised P, dS and Delta)."""
    nq, nk = q.shape[0], k.shape[0]
    # forward recomputation: S, P (the three steps of the forward oracle)
    S = scale * (q @ k.T)
    vis = visible_mask(np.arange(nq), nq, nk, causal)
    if vis is not None:
        S = np.where(vis, S, -np.inf)
    rowmax = S.max(axis=1) if nk > 0 else np.full(nq, -np.inf)
    alive = np.isfinite(rowmax)
    E = np.exp(S - np.where(alive, rowmax, 0.0)[:, None])
    P = np.zeros_like(E)
    P[alive] = E[alive] / E[alive].sum(axis=1, keepdims=True)
    O = P @ v
    # chain rule through O = P V, then through the row softmax, then through S = scale Q K^T
    dv = P.T @ do
    dP = do @ v.T
    delta = np.sum(do * O, axis=1)
    dS = P * (dP - delta[:, None])
    dq = scale * (dS @ k)
    dk = scale * (dS.T @ q)
    if want_parts:
        return dq, dk, dv, P, dS, delta
    return dq, dk, dv


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Gradients of attention.  q, do: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] (bf16
    tensors or arrays).  Returns dq [B, Hq, Nq, d], dk and dv [B, Hkv, Nk, d] as float64."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    assert Hq % Hkv == 0, "Hq must be a multiple of Hkv"
    dq = np.zeros_like(q)
    dk = np.zeros((B, Hkv, Nk, d))
    dv = np.zeros((B, Hkv, Nk, v.shape[-1]))
    for b in range(B):
        for h in range(Hq):
            kv = kv_head_of(h, Hq, Hkv)
            g_q, g_k, g_v = attention_head_backward(q[b, h], k[b, kv], v[b, kv], do[b, h], scale, causal)
            dq[b, h] = g_q
            dk[b, kv] += g_k
            dv[b, kv] += g_v
    return dq, dk, dv
