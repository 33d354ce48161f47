"""Seeded synthetic inputs for the attention workloads.

This module draws random numbers and lays them out; it performs none of the
attention arithmetic.  Both the CUDA path (through the tests and the benchmark)
and the fp64 oracle receive the tensors produced here, so that the two sides
see bit-identical bf16 inputs.

Recipe (the pages fix only the shapes and distributions, see the workload
table): every tensor comes from its own numpy PCG64 stream keyed by
``(seed, stream_id, chunk)``; values are standard normals drawn in float32,
multiplied by the stated standard deviation and rounded to bf16 with
round-to-nearest-even.  Chunks are fixed at 2**24 elements so the result does
not depend on how many threads generate it.
"""

from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

_CHUNK = 1 << 24

# stream ids: one independent generator per tensor
_Q, _K, _V, _LENS, _PERM, _MASK, _DO = 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class PrefillShape:
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    qk_std: float = 1.0
    v_std: float = 1.0


@dataclass(frozen=True)
class DecodeShape:
    S: int  # number of sequences, one query token each
    Hq: int
    Hkv: int
    d: int
    page_size: int
    len_lo: int  # sequence lengths are uniform integers in [len_lo, len_hi]
    len_hi: int


# The five synthetic workloads, in the order the method's benchmark lists them.
WORKLOADS: dict[str, PrefillShape | DecodeShape] = {
    "tiny_mha_d64": PrefillShape(B=1, Hq=2, Hkv=2, Nq=128, Nk=128, d=64, causal=False),
    "gqa_causal_2k": PrefillShape(B=4, Hq=32, Hkv=8, Nq=2048, Nk=2048, d=128, causal=True),
    "gqa_causal_16k": PrefillShape(B=1, Hq=64, Hkv=8, Nq=16384, Nk=16384, d=128, causal=True),
    "peaked_mha_d256": PrefillShape(B=2, Hq=16, Hkv=16, Nq=4096, Nk=4096, d=256, causal=False,
                                    qk_std=3.0),
    "paged_decode_gqa": DecodeShape(S=64, Hq=64, Hkv=8, d=128, page_size=16,
                                    len_lo=512, len_hi=32768),
}

WORKLOAD_ORDER = list(WORKLOADS)


def workload_seed(name: str) -> int:
    """Fixed seed per workload: 0x5EED0000 plus its position in the table."""
    return 0x5EED0000 + WORKLOAD_ORDER.index(name)


def _fill_chunk(out_f32: np.ndarray, seed: int, stream: int, chunk: int, std: float) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, chunk])))
    rng.standard_normal(out=out_f32, dtype=np.float32)
    if std != 1.0:
        out_f32 *= np.float32(std)
    return out_f32


def normal_bf16(shape: tuple[int, ...], seed: int, stream: int, std: float = 1.0,
                threads: int | None = None) -> torch.Tensor:
    """i.i.d. N(0, std^2) rounded to bf16 (RNE), as a contiguous CPU tensor."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(n, dtype=torch.bfloat16)
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def work(c: int) -> None:
        lo = c * _CHUNK
        hi = min(n, lo + _CHUNK)
        buf = np.empty(hi - lo, dtype=np.float32)
        _fill_chunk(buf, seed, stream, c, std)
        out[lo:hi] = torch.from_numpy(buf).to(torch.bfloat16)

    if nchunks <= 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(max_workers=threads or min(16, nchunks)) as ex:
            list(ex.map(work, range(nchunks)))
    return out.view(shape)


def prefill_inputs(shape: PrefillShape, seed: int):
    """q [B,Hq,Nq,d], k and v [B,Hkv,Nk,d], bf16, contiguous, on the CPU."""
    s = shape
    q = normal_bf16((s.B, s.Hq, s.Nq, s.d), seed, _Q, s.qk_std)
    k = normal_bf16((s.B, s.Hkv, s.Nk, s.d), seed, _K, s.qk_std)
    v = normal_bf16((s.B, s.Hkv, s.Nk, s.d), seed, _V, s.v_std)
    return q, k, v


@dataclass
class PagedKV:
    q: torch.Tensor            # [S, Hq, d] bf16
    k_pool: torch.Tensor       # [num_pages, Hkv, page_size, d] bf16
    v_pool: torch.Tensor       # [num_pages, Hkv, page_size, d] bf16
    block_table: torch.Tensor  # [S, max_pages_per_seq] int32, -1 past each sequence's pages
    seq_lens: torch.Tensor     # [S] int32
    page_size: int

    @property
    def num_pages(self) -> int:
        return self.k_pool.shape[0]

    @property
    def max_pages_per_seq(self) -> int:
        return self.block_table.shape[1]


def page_layout(seq_lens: np.ndarray, page_size: int, max_pages_per_seq: int, seed: int):
    """Deal a seeded random permutation of all pool pages out to the sequences in order.

    Sequence s owns ceil(len_s / page_size) pages; entry i of its row holds the
    pool page that stores its tokens [i*page_size, (i+1)*page_size).
    Returns (block_table int32 [S, max_pages_per_seq], num_pages).
    """
    npages = [(int(n) + page_size - 1) // page_size for n in seq_lens]
    total = int(sum(npages))
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _PERM, 0])))
    perm = rng.permutation(total).astype(np.int32)
    table = np.full((len(seq_lens), max_pages_per_seq), -1, dtype=np.int32)
    pos = 0
    for s, n in enumerate(npages):
        table[s, :n] = perm[pos:pos + n]
        pos += n
    return table, total


def decode_inputs(shape: DecodeShape, seed: int, seq_lens: np.ndarray | None = None,
                  max_pages_per_seq: int | None = None) -> PagedKV:
    """Paged-KV decode batch: one query token per sequence, K/V in a shared page pool."""
    s = shape
    if seq_lens is None:
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _LENS, 0])))
        seq_lens = rng.integers(s.len_lo, s.len_hi + 1, size=s.S)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    if max_pages_per_seq is None:
        max_pages_per_seq = max(1, (max(s.len_hi, int(seq_lens.max(initial=0))) + s.page_size - 1)
                                // s.page_size)
    table, total = page_layout(seq_lens, s.page_size, max_pages_per_seq, seed)
    q = normal_bf16((len(seq_lens), s.Hq, s.d), seed, _Q)
    pool_pages = max(total, 1)
    k_pool = normal_bf16((pool_pages, s.Hkv, s.page_size, s.d), seed, _K)
    v_pool = normal_bf16((pool_pages, s.Hkv, s.page_size, s.d), seed, _V)
    return PagedKV(q=q, k_pool=k_pool, v_pool=v_pool,
                   block_table=torch.from_numpy(table),
                   seq_lens=torch.from_numpy(seq_lens.copy()), page_size=s.page_size)


def upstream_grad(shape: PrefillShape, seed: int) -> torch.Tensor:
    """Seeded upstream gradient dO [B, Hq, Nq, d] for the backward pass: bf16 N(0, 1)."""
    return normal_bf16((shape.B, shape.Hq, shape.Nq, shape.d), seed, _DO)


def block_mask(Nq: int, Nk: int, density: float, seed: int, block: int = 128) -> torch.Tensor:
    """Seeded block-sparse map: uint8 [ceil(Nq/block), ceil(Nk/block)], each entry 1
    with probability ``density`` (independently), else 0."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _MASK, 0])))
    shape = ((Nq + block - 1) // block, (Nk + block - 1) // block)
    return torch.from_numpy((rng.random(shape) < density).astype(np.uint8))


def default_scale(d: int) -> float:
    """The softmax temperature every workload uses: 1/sqrt(d)."""
    return 1.0 / math.sqrt(d)
