"""GPU parity of the FP8 path: the block quantizer bit for bit against the oracle's, and
FP8 attention against the exact attention of the dequantized inputs.

Tolerance of FP8 attention, derived from the arithmetic: the fp8 products and their
fp32 sums are exact to ~1e-7 relative, so the kernel's error is that of rounding each
probability (times 256) to e4m3 before P V: relative 2^-4 for normal values, absolute
2^-10 / 256 = 2^-18 for subnormal ones, while O is normalised by the fp32 sum of the
unrounded probabilities.  Element by element:
    |O err| <= sum_j (2^-4 P_j + 2^-18) |v_j|  (+ 1e-5)
and the log-sum-exp within 1e-3 (it does not see the rounding).
"""

import math

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth
from oracle import attention_head, block_quantize, dequantize, kv_head_of

pytestmark = pytest.mark.gpu


def bf16(shape, seed, std=1.0):
    return synth.normal_bf16(shape, seed, 11, std=std)


@pytest.mark.parametrize("planes,N,block", [(6, 300, 128), (4, 256, 128), (3, 333, 333), (2, 129, 129), (2, 100, 128)])
def test_quantizer_matches_oracle_bit_for_bit(planes, N, block, cuda_device):
    x = bf16((planes, N, 128), seed=N + block)
    x[0, : min(N, 128)] = 0                      # an all-zero block: scale 1, codes 0
    x[1, 5, :8] = torch.tensor([1e-30, -1e-30, 3e4, -3e4, 0.0, -0.0, 1e-3, -1e-3], dtype=torch.bfloat16)
    codes, scales = ab.attn_quantize_fp8(x.cuda(), block)
    ref_codes, ref_scales = block_quantize(x, block)
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_scales)
    got = codes.cpu().numpy()
    diff = np.flatnonzero(got != ref_codes)
    assert diff.size == 0, (f"{diff.size} codes differ, first at {diff[:4]}: "
                            f"{got.ravel()[diff[:4]]} vs {ref_codes.ravel()[diff[:4]]}")


def quantized_inputs(B, Hq, Hkv, Nq, Nk, seed):
    shape = synth.PrefillShape(B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=128, causal=True)
    q, k, v = synth.prefill_inputs(shape, seed)
    q8, qs = block_quantize(q, 128)
    k8, ks = block_quantize(k, 128)
    v8, vs = block_quantize(v, Nk)
    return (q8, qs, k8, ks, v8, vs[..., 0])


def run_fp8(inp, causal, scale, out_dtype=torch.float32):
    dev = torch.device("cuda:0")
    q8, qs, k8, ks, v8, vs = (torch.from_numpy(np.ascontiguousarray(t)).to(dev) for t in inp)
    B, Hq, Nq, d = q8.shape
    o = torch.empty((B, Hq, Nq, d), dtype=out_dtype, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    ab.attn_fwd_fp8(q8, qs, k8, ks, v8, vs, o, lse, causal, scale)
    st = ab.attn_get_device_status()
    assert st == 0, ab.attn_status_string(st)
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


CASES = [
    # B, Hq, Hkv, Nq, Nk, causal
    (1, 4, 2, 256, 256, True),
    (1, 2, 2, 333, 333, False),
    (2, 4, 1, 200, 500, True),    # Nq < Nk
    (1, 2, 2, 300, 100, True),    # Nq > Nk: rows without visible keys
    (1, 8, 2, 640, 640, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,causal", CASES)
def test_fp8_attention_matches_dequantized_reference(B, Hq, Hkv, Nq, Nk, causal, cuda_device):
    inp = quantized_inputs(B, Hq, Hkv, Nq, Nk, seed=500 + Nq + Nk)
    scale = 1.0 / math.sqrt(128)
    o, lse = run_fp8(inp, causal, scale)
    q8, qs, k8, ks, v8, vs = inp
    q, k = dequantize(q8, qs), dequantize(k8, ks)
    v = dequantize(v8, vs[..., None], block=Nk)
    for b in range(B):
        for h in range(Hq):
            kv = kv_head_of(h, Hq, Hkv)
            ref_o, ref_l, P = attention_head(q[b, h], k[b, kv], v[b, kv], scale, causal, nq=Nq, want_p=True)
            bound = (2.0 ** -4 * P + 2.0 ** -18 * (P > 0)) @ np.abs(v[b, kv]) + 1e-5
            err = np.abs(o[b, h] - ref_o)
            assert np.all(err <= bound), f"head {b},{h}: max excess {(err - bound).max():.3e}"
            inf = np.isneginf(ref_l)
            assert np.array_equal(np.isneginf(lse[b, h]), inf)
            assert np.all(np.abs(lse[b, h][~inf] - ref_l[~inf]) <= 1e-3)


def test_fp8_end_to_end_with_gpu_quantizer(cuda_device):
    # quantize on the GPU, attend in FP8: the same codes the oracle makes, so the same reference
    shape = synth.PrefillShape(B=1, Hq=4, Hkv=2, Nq=384, Nk=384, d=128, causal=True)
    q, k, v = synth.prefill_inputs(shape, 77)
    dev = torch.device("cuda:0")
    q8, qs = ab.attn_quantize_fp8(q.to(dev), 128)
    k8, ks = ab.attn_quantize_fp8(k.to(dev), 128)
    v8, vs = ab.attn_quantize_fp8(v.to(dev), 384)
    o = torch.empty((1, 4, 384, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 4, 384), dtype=torch.float32, device=dev)
    ab.attn_fwd_fp8(q8, qs, k8, ks, v8, vs[..., 0].contiguous(), o, lse, True, 1 / math.sqrt(128))
    assert ab.attn_get_device_status() == 0
    ref = quantized_inputs(1, 4, 2, 384, 384, 77)
    np.testing.assert_array_equal(q8.cpu().numpy(), ref[0])
    o2, _ = run_fp8(ref, True, 1 / math.sqrt(128))
    # bf16 output of the same kernel: within half a bf16 unit of the fp32 output
    assert np.all(np.abs(o.double().cpu().numpy() - o2) <= np.abs(o2) * 2.0 ** -8 + 1e-6)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,causal", [(1, 3, 1, 333, 333, True), (1, 2, 2, 33, 200, False),
                                                   (2, 4, 2, 1, 129, True)])
def test_fp8_bf16_store_equals_rounded_fp32_output(B, Hq, Hkv, Nq, Nk, causal, cuda_device):
    # bf16 O leaves through staged tensor stores, fp32 O through direct stores
    inp = quantized_inputs(B, Hq, Hkv, Nq, Nk, seed=900 + Nq)
    scale = 1.0 / math.sqrt(128)
    o32, l32 = run_fp8(inp, causal, scale)
    o16, l16 = run_fp8(inp, causal, scale, out_dtype=torch.bfloat16)
    rounded = torch.from_numpy(o32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(o16, rounded)
    assert np.array_equal(l16, l32)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["gqa_causal_2k", "gqa_causal_16k"])
def test_fp8_full_size_sampled(name, cuda_device):
    # the FP8 bench's launch on the whole workload (quantized on the GPU, bf16 O); sampled
    # rows against the exact attention of the dequantized inputs, within the bound above
    # plus half a bf16 unit for the output's own rounding
    s = synth.WORKLOADS[name]
    q, k, v = synth.prefill_inputs(s, synth.workload_seed(name))
    dev = torch.device("cuda:0")
    q8, qs = ab.attn_quantize_fp8(q.to(dev), 128)
    k8, ks = ab.attn_quantize_fp8(k.to(dev), 128)
    v8, vs = ab.attn_quantize_fp8(v.to(dev), s.Nk)
    del q, k, v
    o = torch.empty((s.B, s.Hq, s.Nq, s.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((s.B, s.Hq, s.Nq), dtype=torch.float32, device=dev)
    scale = synth.default_scale(s.d)
    ab.attn_fwd_fp8(q8, qs, k8, ks, v8, vs[..., 0].contiguous(), o, lse, s.causal, scale)
    assert ab.attn_get_device_status() == 0
    rng = np.random.default_rng(41)
    for trial in range(4):
        b, h = int(rng.integers(s.B)), int(rng.integers(s.Hq))
        kv = kv_head_of(h, s.Hq, s.Hkv)
        rows = np.sort(rng.choice(s.Nq, 6, replace=False))
        rows[0] = 0 if trial == 0 else rows[0]
        rows[-1] = s.Nq - 1 if trial == 1 else rows[-1]
        qd = dequantize(q8[b, h].cpu().numpy(), qs[b, h].cpu().numpy())[rows]
        kd = dequantize(k8[b, kv].cpu().numpy(), ks[b, kv].cpu().numpy())
        vd = dequantize(v8[b, kv].cpu().numpy(), vs[b, kv].cpu().numpy(), block=s.Nk)
        ref_o, ref_l, P = attention_head(qd, kd, vd, scale, s.causal, rows=rows, nq=s.Nq, want_p=True)
        got = o[b, h, torch.from_numpy(rows).to(dev)].double().cpu().numpy()
        bound = (2.0 ** -4 * P + 2.0 ** -18 * (P > 0)) @ np.abs(vd) + 1e-5 + np.abs(got) * 2.0 ** -9
        err = np.abs(got - ref_o)
        assert np.all(err <= bound), f"{name} head {b},{h}: max excess {(err - bound).max():.3e}"
        gl = lse[b, h, torch.from_numpy(rows).to(dev)].double().cpu().numpy()
        assert np.all(np.abs(gl - ref_l) <= 1e-3)


def test_fp8_rejects_other_head_dims(cuda_device):
    dev = torch.device("cuda:0")
    x = torch.zeros((1, 1, 16, 64), dtype=torch.uint8, device=dev)
    s1 = torch.ones((1, 1, 1), device=dev)
    with pytest.raises(ab.AttnError):
        ab.attn_fwd_fp8(x, s1, x, s1, x, torch.ones((1, 1), device=dev), torch.zeros((1, 1, 16, 64), device=dev),
                        None, False, 0.1)
