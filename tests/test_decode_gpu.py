"""GPU parity of the paged-KV decode (split-K pass + log-sum-exp merge) against the
fp64 oracle, plus the paging invariants and the bad-page error path."""

import math

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth
from oracle import decode_paged
from parity import compare_lse, compare_o, run_prefill

pytestmark = pytest.mark.gpu


def make(lens, Hq=8, Hkv=2, d=128, page_size=16, seed=21, max_pages=None):
    shape = synth.DecodeShape(S=len(lens), Hq=Hq, Hkv=Hkv, d=d, page_size=page_size, len_lo=1,
                              len_hi=max(max(lens), 1))
    return synth.decode_inputs(shape, seed, seq_lens=np.array(lens), max_pages_per_seq=max_pages)


def run_decode(kv, scale, table=None, k_pool=None, v_pool=None):
    dev = torch.device("cuda:0")
    S, Hq, d = kv.q.shape
    Hkv = kv.k_pool.shape[1]
    o = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((S, Hq), dtype=torch.float32, device=dev)
    table = kv.block_table if table is None else table
    nbytes = ab.attn_decode_paged_workspace_size(S, Hq, Hkv, d, table.shape[1], kv.page_size)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ab.attn_decode_paged(kv.q.to(dev), (kv.k_pool if k_pool is None else k_pool).to(dev),
                         (kv.v_pool if v_pool is None else v_pool).to(dev), table.to(dev),
                         kv.seq_lens.to(dev), kv.page_size, o, lse, scale, ws)
    status = ab.attn_get_device_status()
    return o.double().cpu().numpy(), lse.double().cpu().numpy(), status


CASES = [
    # lens, Hq, Hkv, d, page_size
    ([1, 15, 16, 17, 1500], 8, 2, 128, 16),        # tails, one exact page, two chunks
    ([3000, 1024, 1025, 2048], 8, 1, 128, 16),     # chunk edges, MQA with 8 query heads
    ([700, 33, 64], 4, 4, 64, 32),                 # d=64, 32-token pages, MHA
    ([513, 130], 4, 2, 256, 64),                   # d=256, 64-token pages
    ([900, 77], 32, 2, 128, 16),                   # 16 query heads per KV head: one full head group
    ([1300, 5], 40, 2, 128, 16),                   # 20 per KV head: head groups of 16 and 4 rows
    ([2100, 600], 64, 1, 128, 16),                 # 64 per KV head (MQA): four head groups
    ([2500], 3, 1, 128, 16),                       # odd group
]


@pytest.mark.parametrize("lens,Hq,Hkv,d,ps", CASES)
def test_decode_matches_oracle(lens, Hq, Hkv, d, ps, cuda_device):
    kv = make(lens, Hq, Hkv, d, ps)
    scale = 1.0 / math.sqrt(d)
    ref_o, ref_l = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, ps, scale)
    o, lse, status = run_decode(kv, scale)
    assert status == 0, ab.attn_status_string(status)
    compare_o(o, ref_o, bf16_out=True)
    compare_lse(lse, ref_l)


def test_more_sequences_than_the_plan_sorts(cuda_device):
    # beyond 2048 sequences the plan keeps the shorter last chunks in sequence order
    rng = np.random.default_rng(77)
    lens = [int(x) for x in rng.integers(0, 200, 2100)]
    for i in range(0, 2100, 50):  # some sequences with a full 2048-token chunk, one exactly
        lens[i] = 2048 + (0 if i == 0 else int(rng.integers(1, 400)))
    kv = make(lens, Hq=4, Hkv=1, d=64, page_size=16, seed=78)
    scale = 1.0 / math.sqrt(64)
    ref_o, ref_l = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, 16, scale)
    o, lse, status = run_decode(kv, scale)
    assert status == 0, ab.attn_status_string(status)
    compare_o(o, ref_o, bf16_out=True)
    compare_lse(lse, ref_l)


def test_zero_length_sequence(cuda_device):
    kv = make([0, 40, 0], Hq=4, Hkv=2)
    o, lse, status = run_decode(kv, 0.1)
    assert status == 0
    assert np.all(o[0] == 0) and np.all(o[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2])) and np.all(np.isfinite(lse[1]))


def test_decode_equals_last_row_of_causal_prefill(cuda_device):
    # GPU decode against GPU prefill over the same tokens laid out contiguously
    lens = [777, 1300]
    kv = make(lens, Hq=8, Hkv=2, d=128)
    o, lse, status = run_decode(kv, 0.09)
    assert status == 0
    kp, vp = kv.k_pool, kv.v_pool
    for s, n in enumerate(lens):
        pages = kv.block_table[s, : (n + 15) // 16].long()
        K = kp[pages].permute(1, 0, 2, 3).reshape(2, -1, 128)[:, :n][None].contiguous()
        V = vp[pages].permute(1, 0, 2, 3).reshape(2, -1, 128)[:, :n][None].contiguous()
        Q = torch.zeros(1, 8, n, 128, dtype=torch.bfloat16)
        Q[0, :, -1] = kv.q[s]
        po, pl = run_prefill(Q, K, V, True, 0.09, out_dtype=torch.bfloat16)
        np.testing.assert_allclose(o[s], po[0, :, -1], atol=8e-3)
        np.testing.assert_allclose(lse[s], pl[0, :, -1], atol=1e-3)


def test_page_placement_does_not_matter(cuda_device):
    kv = make([600, 1111, 45], Hq=8, Hkv=2)
    o1, l1, _ = run_decode(kv, 0.09)
    perm = torch.randperm(kv.num_pages, generator=torch.Generator().manual_seed(3))
    k2 = torch.empty_like(kv.k_pool)
    v2 = torch.empty_like(kv.v_pool)
    k2[perm] = kv.k_pool
    v2[perm] = kv.v_pool
    t = kv.block_table.clone()
    used = t >= 0
    t[used] = perm[t[used].long()].int()
    o2, l2, status = run_decode(kv, 0.09, table=t, k_pool=k2, v_pool=v2)
    assert status == 0
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_bad_page_is_reported_not_read(cuda_device):
    kv = make([100, 50], Hq=4, Hkv=2)
    t = kv.block_table.clone()
    t[0, 2] = kv.num_pages + 5       # in use: tokens 32..47 of sequence 0
    t[1, 0] = -7
    o, lse, status = run_decode(kv, 0.1, table=t)
    assert status == 6  # ATTN_ERR_BAD_PAGE
    assert ab.attn_get_device_status() == 0


def test_unused_table_entries_are_ignored(cuda_device):
    kv = make([40], Hq=4, Hkv=2, max_pages=8)
    t = kv.block_table.clone()
    t[0, 3:] = 123456                 # past ceil(40/16) = 3 pages: never read
    ref_o, ref_l = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, 16, 0.1)
    o, lse, status = run_decode(kv, 0.1, table=t)
    assert status == 0
    compare_o(o, ref_o, bf16_out=True)
    compare_lse(lse, ref_l)


@pytest.mark.slow
def test_full_size_decode_sampled(cuda_device):
    name = "paged_decode_gqa"
    s = synth.WORKLOADS[name]
    kv = synth.decode_inputs(s, synth.workload_seed(name))
    scale = synth.default_scale(s.d)
    o, lse, status = run_decode(kv, scale)
    assert status == 0
    seqs = [0, 1, int(np.argmax(kv.seq_lens.numpy())), int(np.argmin(kv.seq_lens.numpy())), 63]
    ref_o, ref_l = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, s.page_size, scale,
                                seqs=seqs)
    compare_o(o[seqs], ref_o, bf16_out=True)
    compare_lse(lse[seqs], ref_l)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
