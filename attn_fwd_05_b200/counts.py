"""Work and byte counts used to turn measured times into roofline figures.

These are bookkeeping for the benchmark, not part of the attention arithmetic.

* Prefill FLOPs: two contractions (Q K^T and P V), each 2*Nq*Nk*d multiply-adds
  per head, so 4*B*Hq*Nq*Nk*d; a causal mask counts half of that.
* Decode bytes: every cached key and value of every sequence is read once,
  seq_len * Hkv * d elements for K and the same for V.
* The KV-cache size grows as layers * H_kv * d_head * seq_len * batch
  ("Variantes d'attention", glossary entry "KV cache"); the factor 2 is K and V.
* The score matrix of the naive method is batch * heads * N * N elements
  ("Flash Attention : pourquoi ton GPU utilise 85% de VRAM", section
  "L'attention classique en 3 étapes").
"""

from __future__ import annotations

from typing import Iterable


def prefill_flops(B: int, Hq: int, Nq: int, Nk: int, d: int, causal: bool) -> float:
    dense = 4.0 * B * Hq * Nq * Nk * d
    return dense / 2.0 if causal else dense


def prefill_min_bytes(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int,
                      elem: int = 2, out_elem: int = 2, lse: bool = True) -> int:
    """Compulsory HBM traffic: read Q, K, V once, write O (and the fp32 LSE) once."""
    q = B * Hq * Nq * d * elem
    kv = 2 * B * Hkv * Nk * d * elem
    o = B * Hq * Nq * d * out_elem
    lse_b = B * Hq * Nq * 4 if lse else 0
    return q + kv + o + lse_b


def decode_kv_bytes(seq_lens: Iterable[int], Hkv: int, d: int, elem: int = 2) -> int:
    """K and V bytes a decode step must read: sum_s len_s * Hkv * d * 2 tensors."""
    return int(sum(int(n) for n in seq_lens)) * Hkv * d * 2 * elem


def decode_flops(seq_lens: Iterable[int], Hq: int, d: int) -> float:
    return 4.0 * float(sum(int(n) for n in seq_lens)) * Hq * d


def kv_cache_bytes(layers: int, Hkv: int, d_head: int, tokens: int, batch: int,
                   elem: int = 2) -> int:
    """Size of a KV cache: 2 (K and V) * layers * Hkv * d_head * tokens * batch * elem."""
    return 2 * layers * Hkv * d_head * tokens * batch * elem


def score_matrix_bytes(batch: int, heads: int, n: int, elem: int = 2) -> int:
    """One materialised [batch, heads, n, n] score (or probability) matrix."""
    return batch * heads * n * n * elem


def output_bytes(batch: int, heads: int, n: int, d: int, elem: int = 2) -> int:
    return batch * heads * n * d * elem
