"""attn_decode_paged_noalloc: the decode entry point for callers that cannot allocate
device memory (a plugin inside a host application that owns the device memory pool,
a serving loop that must not call cudaMalloc on the request path).  It uses the
library's static scratch instead of a caller workspace, and must return what the
regular entry point returns.  Kept in a file collected last, so that a run stopping at
its first failure has already run every other test."""

import ctypes
import math

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import binding, synth
from parity import LSE_MAX, O_MAX, O_MEAN

pytestmark = pytest.mark.gpu


def _inputs(lens, Hq, Hkv, d, page_size, seed, max_pages):
    shape = synth.DecodeShape(S=len(lens), Hq=Hq, Hkv=Hkv, d=d, page_size=page_size, len_lo=1,
                              len_hi=max(lens))
    return synth.decode_inputs(shape, seed, seq_lens=np.array(lens), max_pages_per_seq=max_pages)


def _both(kv, scale):
    dev = torch.device("cuda:0")
    S, Hq, d = kv.q.shape
    Hkv = kv.k_pool.shape[1]
    args = [t.to(dev) for t in (kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens)]
    o_ref = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=dev)
    l_ref = torch.empty((S, Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(ab.attn_decode_paged_workspace_size(S, Hq, Hkv, d, kv.max_pages_per_seq, kv.page_size),
                     dtype=torch.uint8, device=dev)
    ab.attn_decode_paged(*args, kv.page_size, o_ref, l_ref, scale, ws)
    o = torch.full((S, Hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((S, Hq), float("nan"), dtype=torch.float32, device=dev)
    ab.attn_decode_paged_noalloc(*args, kv.page_size, o, lse, scale)
    assert ab.attn_get_device_status() == 0
    return (o.double().cpu().numpy(), lse.double().cpu().numpy(),
            o_ref.double().cpu().numpy(), l_ref.double().cpu().numpy())


def _close(o, lse, o_ref, l_ref):
    err = np.abs(o - o_ref)
    assert np.all(np.isfinite(o))
    assert err.max() <= O_MAX and err.mean() <= O_MEAN
    assert np.array_equal(np.isneginf(lse), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    assert np.abs(lse[fin] - l_ref[fin]).max(initial=0.0) <= LSE_MAX


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(cuda_device):
    # first call: long sequences fill many partial slots of the static scratch
    kv1 = _inputs([3000, 1500, 700, 2100], Hq=16, Hkv=2, d=128, page_size=16, seed=91, max_pages=256)
    _close(*_both(kv1, 1.0 / math.sqrt(128)))
    # second call: other sizes, fewer chunks; the first call's leftovers must not leak in
    kv2 = _inputs([130, 0, 1100], Hq=8, Hkv=8, d=64, page_size=32, seed=92, max_pages=64)
    o, lse, o_ref, l_ref = _both(kv2, 0.125)
    _close(o, lse, o_ref, l_ref)
    assert np.all(o[1] == 0) and np.all(np.isneginf(lse[1]))


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    lib = binding.load_library()
    limit = lib.attn_decode_paged_noalloc_max_scratch()
    assert limit == 32 << 20
    # 128 sequences x 64 query heads x d=128 with up to 2048 pages of 16 tokens needs ~68 MB
    need = lib.attn_decode_paged_workspace_size(128, 64, 8, 128, 2048, 16)
    assert need > limit
    fake = 0x10000
    st = lib.attn_decode_paged_noalloc(fake, fake, fake, fake, fake, 16, fake, None, 128, 64, 8, 128, 1000, 2048,
                                       ctypes.c_float(0.1), None)
    assert st == 8 and lib.attn_status_string(st) == b"ATTN_ERR_TOO_LARGE"


def _near_limit_pages(lib, S, Hq, Hkv, d, page_size, limit):
    """Largest max_pages_per_seq, in whole 2048-token work chunks, whose workspace fits."""
    step = 2048 // page_size
    pages = step
    while lib.attn_decode_paged_workspace_size(S, Hq, Hkv, d, pages + step, page_size) <= limit:
        pages += step
    return pages


def test_noalloc_near_its_limit_matches_workspace_entry(cuda_device):
    # a call whose scratch layout ends just under the static array's end: the last
    # sequence uses every page it may, so its partials sit at the far end of the array
    lib = binding.load_library()
    limit = lib.attn_decode_paged_noalloc_max_scratch()
    S, Hq, Hkv, d, ps = 2, 64, 1, 128, 16
    pages = _near_limit_pages(lib, S, Hq, Hkv, d, ps, limit)
    need = lib.attn_decode_paged_workspace_size(S, Hq, Hkv, d, pages, ps)
    assert limit - 2 * (1 << 20) < need <= limit
    kv = _inputs([1000, pages * ps], Hq=Hq, Hkv=Hkv, d=d, page_size=ps, seed=93, max_pages=pages)
    _close(*_both(kv, 1.0 / math.sqrt(d)))
    # one more work chunk per sequence needs more than the array holds: rejected, nothing launched
    over = pages + 2048 // ps
    assert lib.attn_decode_paged_workspace_size(S, Hq, Hkv, d, over, ps) > limit
    dev = torch.device("cuda:0")
    table = torch.zeros((S, over), dtype=torch.int32, device=dev)
    o = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=dev)
    with pytest.raises(ab.AttnError) as e:
        ab.attn_decode_paged_noalloc(kv.q.to(dev), kv.k_pool.to(dev), kv.v_pool.to(dev), table,
                                     kv.seq_lens.to(dev), ps, o, None, 0.1)
    assert e.value.status == 8  # ATTN_ERR_TOO_LARGE
    assert ab.attn_get_device_status() == 0
