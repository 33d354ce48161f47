"""GPU parity of the prefill kernels against the fp64 oracle (small sizes that still span
several tiles and a ragged tail), plus the special cases the method has."""

import math

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth
from oracle import attention, attention_rows
from parity import compare_lse, compare_o, run_prefill

pytestmark = pytest.mark.gpu


def inputs(B, Hq, Hkv, Nq, Nk, d, seed, qk_std=1.0, causal=False):
    shape = synth.PrefillShape(B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=d, causal=causal, qk_std=qk_std)
    return synth.prefill_inputs(shape, seed)


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, qk_std      (what it exercises)
    (1, 2, 2, 128, 128, 64, False, 1.0),       # the tiny d=64 workload
    (2, 8, 2, 384, 384, 128, True, 1.0),       # GQA causal, heads paired in one CTA, 3 q-tiles
    (1, 8, 2, 384, 384, 128, False, 1.0),      # GQA non-causal
    (1, 4, 4, 200, 200, 128, False, 1.0),      # MHA: consecutive q-tiles paired, ragged tail
    (1, 4, 4, 200, 200, 128, True, 1.0),
    (1, 3, 1, 333, 333, 128, True, 1.0),       # MQA with an odd group, ragged tail
    (1, 4, 2, 100, 300, 128, True, 1.0),       # Nq < Nk, mask aligned bottom-right
    (1, 4, 2, 300, 100, 128, True, 1.0),       # Nq > Nk: fully masked leading rows
    (1, 4, 2, 1, 517, 128, True, 1.0),         # one query row (decode-like prefill)
    (2, 4, 2, 257, 257, 64, True, 1.0),        # d=64 causal GQA
    (1, 2, 2, 512, 512, 256, False, 3.0),      # peaked d=256 (scores with std 9)
    (1, 2, 1, 300, 300, 256, True, 1.0),       # d=256 causal, ragged, GQA
    (1, 2, 2, 130, 70, 256, False, 1.0),       # d=256 Nk < one block
    (1, 1, 1, 128, 128, 256, False, 1.0),      # d=256 exactly one q-tile and one 128-key block
    (1, 2, 1, 1000, 1000, 256, True, 1.0),     # d=256 causal, the K/V ring wraps several times, ragged tail
    (1, 2, 2, 200, 2300, 256, False, 2.0),     # d=256 a long key row per q-tile, Nk ragged
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,qk_std", CASES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_prefill_matches_oracle(B, Hq, Hkv, Nq, Nk, d, causal, qk_std, out, cuda_device):
    q, k, v = inputs(B, Hq, Hkv, Nq, Nk, d, seed=1000 + Nq + d, qk_std=qk_std, causal=causal)
    scale = 1.0 / math.sqrt(d)
    ref_o, ref_l = attention(q, k, v, scale, causal)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    o, lse = run_prefill(q, k, v, causal, scale, out_dtype=dt)
    compare_o(o, ref_o, bf16_out=(out == "bf16"))
    compare_lse(lse, ref_l)


def test_tiny_workload_exactly(cuda_device):
    name = "tiny_mha_d64"
    s = synth.WORKLOADS[name]
    q, k, v = synth.prefill_inputs(s, synth.workload_seed(name))
    scale = synth.default_scale(s.d)
    ref_o, ref_l = attention(q, k, v, scale, s.causal)
    o, lse = run_prefill(q, k, v, s.causal, scale)
    e_max, e_mean = compare_o(o, ref_o, bf16_out=False)
    assert e_max < 2e-3
    compare_lse(lse, ref_l)


def test_lse_may_be_omitted(cuda_device):
    q, k, v = inputs(1, 2, 2, 256, 256, 128, seed=5)
    o, _ = run_prefill(q, k, v, True, 0.1, with_lse=False)
    ref_o, _ = attention(q, k, v, 0.1, True)
    compare_o(o, ref_o, bf16_out=False)


def test_no_keys_gives_zero_and_minus_inf(cuda_device):
    q, k, v = inputs(1, 2, 2, 64, 0, 128, seed=6)
    o, lse = run_prefill(q, k, v, False, 0.1)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_single_key_returns_its_value(cuda_device):
    q, k, v = inputs(1, 2, 1, 150, 1, 128, seed=7)
    o, lse = run_prefill(q, k, v, False, 0.2)
    ref = v.double().numpy()[:, [0, 0]]
    np.testing.assert_allclose(o, np.broadcast_to(ref, o.shape), atol=1e-6)
    np.testing.assert_allclose(lse, 0.2 * np.einsum("bhqd,bd->bhq", q.double().numpy(),
                                                    k.double().numpy()[:, 0, 0]), atol=1e-3)


def test_uniform_scores_give_mean_of_v(cuda_device):
    q, k, v = inputs(1, 2, 2, 256, 256, 128, seed=8)
    q.zero_()
    o, lse = run_prefill(q, k, v, True, 0.1)
    vv = v.double().numpy()
    ref = np.cumsum(vv, axis=2) / np.arange(1, 257)[None, None, :, None]
    np.testing.assert_allclose(o, ref, atol=2e-3)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, 257)), lse.shape), atol=1e-4)


def test_dominant_key_selects_its_value(cuda_device):
    q, k, v = inputs(1, 1, 1, 256, 256, 128, seed=9)
    q.zero_()
    q[..., 0] = 8.0
    k[..., 0] = 0.0
    k[0, 0, 173, 0] = 8.0          # score 64 * scale for key 173, 0 for the rest
    o, _ = run_prefill(q, k, v, False, 1.0)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v.double().numpy()[0, 0, 173], (256, 128)), atol=1e-5)


def test_gqa_equals_replicated_mha(cuda_device):
    q, k, v = inputs(1, 8, 2, 256, 256, 128, seed=10)
    o1, l1 = run_prefill(q, k, v, True, 0.09)
    o2, l2 = run_prefill(q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1), True, 0.09)
    np.testing.assert_allclose(o1, o2, atol=1e-6)
    np.testing.assert_allclose(l1, l2, atol=1e-6)


def test_key_permutation_invariance(cuda_device):
    q, k, v = inputs(1, 2, 2, 128, 384, 128, seed=11)
    perm = torch.randperm(384, generator=torch.Generator().manual_seed(0))
    o1, l1 = run_prefill(q, k, v, False, 0.09)
    o2, l2 = run_prefill(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), False, 0.09)
    np.testing.assert_allclose(o1, o2, atol=2e-3)
    np.testing.assert_allclose(l1, l2, atol=1e-4)


def test_deterministic(cuda_device):
    q, k, v = inputs(2, 8, 2, 384, 384, 128, seed=12)
    o1, l1 = run_prefill(q, k, v, True, 0.09)
    o2, l2 = run_prefill(q, k, v, True, 0.09)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_bf16_output_is_rounded_fp32_output(cuda_device):
    q, k, v = inputs(1, 4, 2, 256, 256, 128, seed=13)
    o32, _ = run_prefill(q, k, v, True, 0.09, out_dtype=torch.float32)
    o16, _ = run_prefill(q, k, v, True, 0.09, out_dtype=torch.bfloat16)
    rounded = torch.from_numpy(o32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(o16, rounded)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", [
    (1, 2, 2, 1, 77, 128, False),    # one row: a single valid row in the first warp's 32-row box
    (1, 2, 2, 33, 300, 128, True),   # the second warp of the tile holds one valid row
    (1, 3, 1, 333, 333, 128, True),  # odd group: q-tile pairs of one head, the last tile past Nq
    (2, 4, 2, 257, 257, 64, True),   # d = 64: one 64-column box per warp
    (1, 4, 4, 97, 130, 64, False),
])
def test_bf16_store_equals_rounded_fp32_output(B, Hq, Hkv, Nq, Nk, d, causal, cuda_device):
    # bf16 O leaves through staged tensor stores, fp32 O through direct stores: the same
    # accumulator and normaliser, so bf16 must be exactly the rounded fp32 output
    q, k, v = inputs(B, Hq, Hkv, Nq, Nk, d, seed=17 + Nq, causal=causal)
    scale = 1.0 / math.sqrt(d)
    o32, l32 = run_prefill(q, k, v, causal, scale, out_dtype=torch.float32)
    o16, l16 = run_prefill(q, k, v, causal, scale, out_dtype=torch.bfloat16)
    rounded = torch.from_numpy(o32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(o16, rounded)
    assert np.array_equal(l16, l32)


def test_watchdog_latches_timeout_and_device_stays_usable(cuda_device):
    assert ab.attn_get_device_status() == 0
    ab.attn_debug_watchdog(20_000_000)  # 20 ms on a barrier nothing completes
    assert ab.attn_get_device_status() == 5  # ATTN_ERR_DEVICE_TIMEOUT
    assert ab.attn_get_device_status() == 0  # cleared by the read
    q, k, v = inputs(1, 2, 2, 128, 128, 64, seed=14)
    o, lse = run_prefill(q, k, v, False, 0.125)
    ref_o, _ = attention(q, k, v, 0.125, False)
    compare_o(o, ref_o, bf16_out=False)


# ------------------------------------------------------------------ full-size workloads, sampled rows

def sampled_rows_check(name, n_rows=48, seed_rows=0):
    s = synth.WORKLOADS[name]
    q, k, v = synth.prefill_inputs(s, synth.workload_seed(name))
    scale = synth.default_scale(s.d)
    o, lse = run_prefill(q, k, v, s.causal, scale, out_dtype=torch.bfloat16)
    rng = np.random.default_rng(seed_rows)
    worst = 0.0
    for _ in range(n_rows // 8):
        b, h = int(rng.integers(s.B)), int(rng.integers(s.Hq))
        rows = np.sort(rng.choice(s.Nq, 8, replace=False))
        rows[0] = 0 if _ == 0 else rows[0]
        rows[-1] = s.Nq - 1 if _ == 1 else rows[-1]
        ro, rl = attention_rows(q, k, v, scale, s.causal, b, h, rows)
        compare_o(o[b, h, rows], ro, bf16_out=True)
        compare_lse(lse[b, h, rows], rl)
        worst = max(worst, float(np.abs(o[b, h, rows] - ro).max()))
    # properties that hold at any size: finite everywhere, LSE at least the log of the visible count's min
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    return worst


@pytest.mark.slow
@pytest.mark.parametrize("name", ["gqa_causal_2k", "gqa_causal_16k", "peaked_mha_d256"])
def test_full_size_workload_sampled(name, cuda_device):
    sampled_rows_check(name)


def test_device_is_sm100(cuda_device):
    # the library carries sm_100a code only: the device must be compute capability 10.0
    assert torch.cuda.get_device_capability(cuda_device) == (10, 0)
