"""The real kernels' timeout path, without a GPU fault.

A debug entry point leaves one K/V tile fill out in one CTA (the producer neither arms
the stage's barrier nor issues the copy), so the consumer's bounded wait for that tile
runs out.  Checked: the call ends, the device status word reports
ATTN_ERR_DEVICE_TIMEOUT, and the next ordinary call on the same context is correct,
which shows that the aborting CTAs drained their copies and MMAs, freed tensor memory
and left nothing behind.  Nothing here traps, asserts or touches a bad address.
"""

import math
import time

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth
from oracle import attention, decode_paged
from parity import compare_lse, compare_o, run_prefill

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # ATTN_ERR_DEVICE_TIMEOUT
LIMIT_NS = 10_000_000  # 10 ms per wait


def prefill_case(B, Hq, Hkv, N, d, causal, seed):
    shape = synth.PrefillShape(B=B, Hq=Hq, Hkv=Hkv, Nq=N, Nk=N, d=d, causal=causal)
    return synth.prefill_inputs(shape, seed)


def stalled_prefill(q, k, v, causal, scale, cta, fill):
    dev = torch.device("cuda:0")
    B, Hq, N, d = q.shape
    o = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    t0 = time.perf_counter()
    ab.attn_debug_fwd_stall(q.to(dev), k.to(dev), v.to(dev), o, lse, causal, scale, cta, fill, LIMIT_NS)
    status = ab.attn_get_device_status()
    return status, time.perf_counter() - t0


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,cta,fill", [
    (1, 1, 1, 256, 128, False, 0, 2),    # one CTA: V of the first block is missing
    (1, 1, 1, 256, 128, False, 0, 0),    # the very first fill
    (1, 8, 2, 2048, 128, True, 5, 3),    # one CTA of 64 stalls; the others see the latched status
    (2, 16, 4, 4096, 64, True, 100, 40), # d = 64, persistent CTAs that walk several units
])
def test_prefill_wait_runs_out_then_device_is_usable(B, Hq, Hkv, N, d, causal, cta, fill, cuda_device):
    assert ab.attn_get_device_status() == 0
    q, k, v = prefill_case(B, Hq, Hkv, N, d, causal, seed=300 + N + d)
    scale = 1.0 / math.sqrt(d)
    status, secs = stalled_prefill(q, k, v, causal, scale, cta, fill)
    assert status == TIMEOUT, ab.attn_status_string(status)
    assert secs < 5.0
    assert ab.attn_get_device_status() == 0  # the read cleared it
    # the same context, an ordinary call: correct results, no latched fault
    o, lse = run_prefill(q, k, v, causal, scale)
    ref_o, ref_l = attention(q, k, v, scale, causal)
    compare_o(o, ref_o, bf16_out=False)
    compare_lse(lse, ref_l)


def test_prefill_stall_past_the_last_fill_changes_nothing(cuda_device):
    q, k, v = prefill_case(1, 4, 2, 300, 128, True, seed=31)
    scale = 1.0 / math.sqrt(128)
    dev = torch.device("cuda:0")
    o = torch.empty((1, 4, 300, 128), dtype=torch.float32, device=dev)
    lse = torch.empty((1, 4, 300), dtype=torch.float32, device=dev)
    ab.attn_debug_fwd_stall(q.to(dev), k.to(dev), v.to(dev), o, lse, True, scale, 0, 1 << 30, LIMIT_NS)
    assert ab.attn_get_device_status() == 0
    o2, l2 = run_prefill(q, k, v, True, scale)
    assert np.array_equal(o.double().cpu().numpy(), o2)
    assert np.array_equal(lse.double().cpu().numpy(), l2)


def run_decode(kv, scale, stall=None):
    dev = torch.device("cuda:0")
    S, Hq, d = kv.q.shape
    Hkv = kv.k_pool.shape[1]
    o = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((S, Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(ab.attn_decode_paged_workspace_size(S, Hq, Hkv, d, kv.block_table.shape[1], kv.page_size),
                     dtype=torch.uint8, device=dev)
    args = (kv.q.to(dev), kv.k_pool.to(dev), kv.v_pool.to(dev), kv.block_table.to(dev), kv.seq_lens.to(dev),
            kv.page_size, o, lse, scale, ws)
    if stall is None:
        ab.attn_decode_paged(*args)
    else:
        ab.attn_debug_decode_stall(*args, stall[0], stall[1], LIMIT_NS)
    status = ab.attn_get_device_status()
    return o.double().cpu().numpy(), lse.double().cpu().numpy(), status


@pytest.mark.parametrize("lens,cta,piece", [([3000, 1500], 0, 5), ([5000, 800, 4100, 2049], 3, 0),
                                            ([9000] * 8, 17, 64)])
def test_decode_wait_runs_out_then_device_is_usable(lens, cta, piece, cuda_device):
    assert ab.attn_get_device_status() == 0
    shape = synth.DecodeShape(S=len(lens), Hq=8, Hkv=2, d=128, page_size=16, len_lo=1, len_hi=max(lens))
    kv = synth.decode_inputs(shape, 61, seq_lens=np.array(lens))
    scale = 1.0 / math.sqrt(128)
    _, _, status = run_decode(kv, scale, stall=(cta, piece))
    assert status == TIMEOUT, ab.attn_status_string(status)
    o, lse, status = run_decode(kv, scale)
    assert status == 0, ab.attn_status_string(status)
    ref_o, ref_l = decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, 16, scale)
    compare_o(o, ref_o, bf16_out=True)
    compare_lse(lse, ref_l)


def test_stall_arguments_are_checked(cuda_device):
    q, k, v = prefill_case(1, 2, 2, 128, 256, False, seed=3)
    dev = torch.device("cuda:0")
    o = torch.empty((1, 2, 128, 256), dtype=torch.float32, device=dev)
    with pytest.raises(ab.AttnError):  # d = 256 has no stall switch
        ab.attn_debug_fwd_stall(q.to(dev), k.to(dev), v.to(dev), o, None, False, 0.1, 0, 0, LIMIT_NS)
    q, k, v = prefill_case(1, 2, 2, 128, 128, False, seed=3)
    o = torch.empty((1, 2, 128, 128), dtype=torch.float32, device=dev)
    for cta, fill, lim in ((-1, 0, LIMIT_NS), (0, -1, LIMIT_NS), (0, 0, 0), (0, 0, 20_000_000_000)):
        with pytest.raises(ab.AttnError):
            ab.attn_debug_fwd_stall(q.to(dev), k.to(dev), v.to(dev), o, None, False, 0.1, cta, fill, lim)
    assert ab.attn_get_device_status() == 0


def bwd_inputs(B, Hq, Hkv, N, d, causal, seed):
    dev = torch.device("cuda:0")
    shape = synth.PrefillShape(B=B, Hq=Hq, Hkv=Hkv, Nq=N, Nk=N, d=d, causal=causal)
    q, k, v = (t.to(dev) for t in synth.prefill_inputs(shape, seed))
    do = synth.upstream_grad(shape, seed).to(dev)
    o = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    ab.attn_fwd(q, k, v, o, lse, causal, 1.0 / math.sqrt(d))
    return q, k, v, o, do, lse


def bwd_outputs(q, k):
    return (torch.empty(q.shape, dtype=torch.float32, device=q.device),
            torch.empty(k.shape, dtype=torch.float32, device=k.device),
            torch.empty(k.shape, dtype=torch.float32, device=k.device))


def same_gradients(a, b):
    # dK and dV are summed in tensor memory in a fixed order: bit for bit; dQ is summed by
    # additions in L2 in an order that varies: a few fp32 roundings apart
    assert (a[0] - b[0]).abs().max().item() <= 1e-5 * b[0].abs().max().item()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,cta,step", [
    (1, 4, 2, 512, 128, True, 0, 0),      # the first Q tile of CTA 0
    (1, 4, 2, 512, 128, True, 3, 2),      # a later step of another CTA
    (2, 8, 2, 2048, 64, True, 40, 5),     # d = 64, one CTA of 64 stalls
])
def test_backward_wait_runs_out_then_device_is_usable(B, Hq, Hkv, N, d, causal, cta, step, cuda_device):
    assert ab.attn_get_device_status() == 0
    q, k, v, o, do, lse = bwd_inputs(B, Hq, Hkv, N, d, causal, seed=500 + N + d)
    scale = 1.0 / math.sqrt(d)
    ref = bwd_outputs(q, k)
    ab.attn_bwd(q, k, v, o, do, lse, *ref, causal, scale)
    assert ab.attn_get_device_status() == 0
    got = bwd_outputs(q, k)
    t0 = time.perf_counter()
    ab.attn_debug_bwd_stall(q, k, v, o, do, lse, *got, causal, scale, cta, step, LIMIT_NS)
    status = ab.attn_get_device_status()
    assert status == TIMEOUT, ab.attn_status_string(status)
    assert time.perf_counter() - t0 < 5.0
    assert ab.attn_get_device_status() == 0
    # the same context, an ordinary call: the same gradients as before the stall
    for t in got:
        t.fill_(float("nan"))
    ab.attn_bwd(q, k, v, o, do, lse, *got, causal, scale)
    assert ab.attn_get_device_status() == 0
    same_gradients(got, ref)


def test_backward_stall_past_the_last_step_changes_nothing(cuda_device):
    q, k, v, o, do, lse = bwd_inputs(1, 4, 2, 300, 128, True, seed=41)
    scale = 1.0 / math.sqrt(128)
    ref = bwd_outputs(q, k)
    ab.attn_bwd(q, k, v, o, do, lse, *ref, True, scale)
    got = bwd_outputs(q, k)
    ab.attn_debug_bwd_stall(q, k, v, o, do, lse, *got, True, scale, 0, 1 << 30, LIMIT_NS)
    assert ab.attn_get_device_status() == 0
    same_gradients(got, ref)


def test_backward_stall_rejects_bad_arguments(cuda_device):
    q, k, v, o, do, lse = bwd_inputs(1, 2, 2, 128, 64, False, seed=42)
    out = bwd_outputs(q, k)
    for cta, step, limit in ((-1, 0, LIMIT_NS), (0, -1, LIMIT_NS), (0, 0, 0), (0, 0, 20_000_000_000)):
        with pytest.raises(ab.AttnError) as e:
            ab.attn_debug_bwd_stall(q, k, v, o, do, lse, *out, False, 0.125, cta, step, limit)
        assert e.value.status == 1  # ATTN_ERR_INVALID_ARG
    assert ab.attn_get_device_status() == 0
