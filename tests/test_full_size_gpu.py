"""Every output element of the full-size workloads against the fp64 oracle, and launches
whose persistent CTAs each walk several work units.

The tiled method returns the same result as the materialising one up to floating-point
rounding (polydesk.ai glossary "FlashAttention", section "FlashAttention vs attention
standard"), so nothing here is sampled: each test compares the whole O and LSE of one
launch with the oracle, element by element, within the bounds of tests/parity.py.

Launch configurations are those of the benchmark: bf16 O through ``attn_fwd`` (the
timed call) and fp32 O through ``attn_fwd_ex`` (the parity entry), both on the full
workload in one launch.
"""

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth
from oracle import attention, attention_head, block_quantize, decode_paged, dequantize, kv_head_of
from parity import compare_lse, compare_o

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

_ORACLE_CACHE = {}


def _prefill_oracle(key, q, k, v, scale, causal):
    if key not in _ORACLE_CACHE:
        _ORACLE_CACHE.clear()  # one workload's reference at a time: they are large
        _ORACLE_CACHE[key] = attention(q, k, v, scale, causal)
    return _ORACLE_CACHE[key]


def _launch(q, k, v, causal, scale, out_dtype):
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    B, Hq, Nq, d = q.shape
    o = torch.empty((B, Hq, Nq, d), dtype=out_dtype, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    if out_dtype == torch.bfloat16:
        ab.attn_fwd(qd, kd, vd, o, lse, causal, scale)
    else:
        ab.attn_fwd_ex(qd, kd, vd, o, lse, causal, scale)
    status = ab.attn_get_device_status()
    assert status == 0, ab.attn_status_string(status)
    return o, lse


def _check_heads(o, lse, ref_o, ref_l, bf16_out, heads=None):
    """Compare whole heads (all of them, or the listed (b, h) pairs) element by element."""
    if heads is None:
        got_o = o.double().cpu().numpy()
        got_l = lse.double().cpu().numpy()
        compare_o(got_o, ref_o, bf16_out=bf16_out)
        compare_lse(got_l, ref_l)
        return
    for n, (b, h) in enumerate(heads):
        compare_o(o[b, h].double().cpu().numpy(), ref_o[n], bf16_out=bf16_out)
        compare_lse(lse[b, h].double().cpu().numpy(), ref_l[n])


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("name", ["tiny_mha_d64", "gqa_causal_2k", "peaked_mha_d256"])
def test_workload_every_element(name, out, cuda_device):
    s = synth.WORKLOADS[name]
    q, k, v = synth.prefill_inputs(s, synth.workload_seed(name))
    scale = synth.default_scale(s.d)
    ref_o, ref_l = _prefill_oracle(name, q, k, v, scale, s.causal)
    o, lse = _launch(q, k, v, s.causal, scale, torch.float32 if out == "f32" else torch.bfloat16)
    _check_heads(o, lse, ref_o, ref_l, bf16_out=(out == "bf16"))


# Long-context workload: one launch over all 64 heads; eight whole heads (every one of their
# 16384 rows) are compared.  Heads 0/1 and 18/19 are the two tiles of one work unit each;
# 45, 46, 62 and 63 fall in four other units and three other KV groups.
C3_HEADS = [(0, 0), (0, 1), (0, 18), (0, 19), (0, 45), (0, 46), (0, 62), (0, 63)]


@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_long_context_eight_whole_heads(out, cuda_device):
    name = "gqa_causal_16k"
    s = synth.WORKLOADS[name]
    q, k, v = synth.prefill_inputs(s, synth.workload_seed(name))
    scale = synth.default_scale(s.d)
    key = (name, "heads")
    if key not in _ORACLE_CACHE:
        _ORACLE_CACHE.clear()
        G = s.Hq // s.Hkv
        qs = torch.stack([q[b, h] for b, h in C3_HEADS])[None]
        ks = torch.stack([k[b, h // G] for b, h in C3_HEADS])[None]
        vs = torch.stack([v[b, h // G] for b, h in C3_HEADS])[None]
        ro, rl = attention(qs, ks, vs, scale, s.causal)
        _ORACLE_CACHE[key] = (ro[0], rl[0])
    ref_o, ref_l = _ORACLE_CACHE[key]
    o, lse = _launch(q, k, v, s.causal, scale, torch.float32 if out == "f32" else torch.bfloat16)
    _check_heads(o, lse, ref_o, ref_l, bf16_out=(out == "bf16"), heads=C3_HEADS)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


# The two-tile kernel is persistent: one CTA per SM walks work units in a snake order and
# its barriers count phases across units, reloading Q per unit.  These launches give every
# CTA several units (units >= 4 x 148 CTAs), in each of the unit layouts.
MULTI_UNIT = [
    # B, Hq, Hkv, N, d, causal     units (what it exercises)
    (2, 32, 8, 4096, 128, True),   # 1024: paired heads, causal, longest first
    (2, 24, 8, 4096, 128, True),   # 768: odd group, q-tile pairs of one head
    (2, 16, 4, 4096, 64, True),    # 512: d = 64 (eight-stage ring)
    (1, 16, 2, 8192, 128, False),  # 512: non-causal order
    (3, 8, 2, 3000, 128, True),    # 288: ragged, the last q-tile of every head is partial
    (2, 16, 4, 8300, 64, True),    # 1040: 65 q-tiles, levels taken in bands of 16, a short last band
]


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", MULTI_UNIT)
def test_persistent_walk_every_element(B, Hq, Hkv, N, d, causal, out, cuda_device):
    shape = synth.PrefillShape(B=B, Hq=Hq, Hkv=Hkv, Nq=N, Nk=N, d=d, causal=causal)
    q, k, v = synth.prefill_inputs(shape, 4242 + N + Hq + d)
    scale = 1.0 / math.sqrt(d)
    ref_o, ref_l = _prefill_oracle(("multi", B, Hq, Hkv, N, d, causal), q, k, v, scale, causal)
    o, lse = _launch(q, k, v, causal, scale, torch.float32 if out == "f32" else torch.bfloat16)
    _check_heads(o, lse, ref_o, ref_l, bf16_out=(out == "bf16"))


def test_decode_workload_every_sequence(cuda_device):
    """All 64 sequences of the decode workload, in the benchmark's launch (one call)."""
    name = "paged_decode_gqa"
    s = synth.WORKLOADS[name]
    kv = synth.decode_inputs(s, synth.workload_seed(name))
    scale = synth.default_scale(s.d)
    dev = torch.device("cuda:0")
    o = torch.empty((s.S, s.Hq, s.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((s.S, s.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(ab.attn_decode_paged_workspace_size(s.S, s.Hq, s.Hkv, s.d, kv.max_pages_per_seq, s.page_size),
                     dtype=torch.uint8, device=dev)
    ab.attn_decode_paged(kv.q.to(dev), kv.k_pool.to(dev), kv.v_pool.to(dev), kv.block_table.to(dev),
                         kv.seq_lens.to(dev), s.page_size, o, lse, scale, ws)
    status = ab.attn_get_device_status()
    assert status == 0, ab.attn_status_string(status)
    got_o = o.double().cpu().numpy()
    got_l = lse.double().cpu().numpy()
    del ws, o, lse

    # the oracle one sequence at a time, sequences spread over host threads
    def one(n):
        return decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, s.page_size, scale, seqs=[n])

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        refs = list(ex.map(one, range(s.S)))
    ref_o = np.concatenate([r[0] for r in refs])
    ref_l = np.concatenate([r[1] for r in refs])
    compare_o(got_o, ref_o, bf16_out=True)
    compare_lse(got_l, ref_l)


def test_fp8_workload_every_element(cuda_device):
    """FP8 forward on the 2K workload (quantized as the FP8 benchmark does), every element
    against the exact attention of the dequantized inputs, within the derived bound of
    tests/test_fp8_gpu.py."""
    name = "gqa_causal_2k"
    s = synth.WORKLOADS[name]
    q, k, v = synth.prefill_inputs(s, synth.workload_seed(name))
    q8, qs = block_quantize(q, 128)
    k8, ks = block_quantize(k, 128)
    v8, vs = block_quantize(v, s.Nk)
    del q, k, v
    dev = torch.device("cuda:0")
    o = torch.empty((s.B, s.Hq, s.Nq, s.d), dtype=torch.float32, device=dev)
    lse = torch.empty((s.B, s.Hq, s.Nq), dtype=torch.float32, device=dev)
    t = [torch.from_numpy(np.ascontiguousarray(x)).to(dev) for x in (q8, qs, k8, ks, v8, vs[..., 0])]
    scale = synth.default_scale(s.d)
    ab.attn_fwd_fp8(*t, o, lse, s.causal, scale)
    status = ab.attn_get_device_status()
    assert status == 0, ab.attn_status_string(status)
    got_o = o.double().cpu().numpy()
    got_l = lse.double().cpu().numpy()
    qd, kd = dequantize(q8, qs), dequantize(k8, ks)
    vd = dequantize(v8, vs, block=s.Nk)

    def head(bh):
        b, h = bh
        kv = kv_head_of(h, s.Hq, s.Hkv)
        ref_o, ref_l, P = attention_head(qd[b, h], kd[b, kv], vd[b, kv], scale, s.causal, want_p=True)
        bound = (2.0 ** -4 * P + 2.0 ** -18 * (P > 0)) @ np.abs(vd[b, kv]) + 1e-5
        excess = float((np.abs(got_o[b, h] - ref_o) - bound).max())
        lerr = float(np.abs(got_l[b, h] - ref_l).max())
        return excess, lerr

    try:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(1)
    except Exception:  # pragma: no cover
        ctx = None
    try:
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            res = list(ex.map(head, [(b, h) for b in range(s.B) for h in range(s.Hq)]))
    finally:
        if ctx is not None:
            ctx.unregister()
    worst = max(r[0] for r in res)
    assert worst <= 0.0, f"max excess over the FP8 bound {worst:.3e}"
    assert max(r[1] for r in res) <= 1e-3
