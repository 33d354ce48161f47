"""GPU parity of attn_fwd_masked (sliding window, block-sparse map) against the fp64
oracle, plus the identities that tie the masked path to the unmasked one."""

import math

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth
from oracle import attention, attention_rows
from parity import compare_lse, compare_o

pytestmark = pytest.mark.gpu


def inputs(B, Hq, Hkv, Nq, Nk, d, seed):
    shape = synth.PrefillShape(B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=d, causal=True, qk_std=1.0)
    return synth.prefill_inputs(shape, seed)


def run_masked(q, k, v, causal, scale, window=0, block_mask=None, out_dtype=torch.float32):
    dev = torch.device("cuda:0")
    B, Hq, Nq, d = q.shape
    o = torch.empty((B, Hq, Nq, d), dtype=out_dtype, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    bm = None if block_mask is None else block_mask.to(dev)
    ab.attn_fwd_masked(q.to(dev), k.to(dev), v.to(dev), o, lse, causal, scale, window=window, block_mask=bm)
    status = ab.attn_get_device_status()
    assert status == 0, ab.attn_status_string(status)
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def run_plain(q, k, v, causal, scale):
    dev = torch.device("cuda:0")
    B, Hq, Nq, d = q.shape
    o = torch.empty((B, Hq, Nq, d), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    ab.attn_fwd_ex(q.to(dev), k.to(dev), v.to(dev), o, lse, causal, scale)
    return o.cpu().numpy(), lse.cpu().numpy()


WINDOW_CASES = [
    # B, Hq, Hkv, Nq, Nk, d, window
    (1, 4, 2, 384, 384, 128, 1),      # diagonal only
    (1, 4, 2, 384, 384, 128, 64),     # window inside one block
    (1, 4, 4, 333, 333, 128, 100),    # MHA q-tile pairs, ragged tail
    (2, 8, 2, 520, 520, 64, 300),     # window spanning block edges, d=64
    (1, 4, 2, 200, 600, 128, 130),    # Nq < Nk: bottom-right alignment
    (1, 2, 1, 450, 450, 256, 200),    # d=256 (64-key blocks)
    (1, 2, 2, 300, 300, 256, 1),
    (1, 4, 2, 256, 256, 128, 10000),  # window wider than the sequence = causal
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,window", WINDOW_CASES)
def test_window_matches_oracle(B, Hq, Hkv, Nq, Nk, d, window, cuda_device):
    q, k, v = inputs(B, Hq, Hkv, Nq, Nk, d, seed=3000 + Nq + window)
    scale = 1.0 / math.sqrt(d)
    ref_o, ref_l = attention(q, k, v, scale, True, window=window)
    o, lse = run_masked(q, k, v, True, scale, window=window)
    compare_o(o, ref_o, bf16_out=False)
    compare_lse(lse, ref_l)


BLOCK_CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, density
    (1, 4, 2, 512, 512, 128, False, 0.5),   # GQA: paired heads share a map row
    (1, 4, 4, 640, 640, 128, False, 0.4),   # MHA: the two tiles of a CTA use different rows
    (1, 4, 4, 640, 640, 128, True, 0.6),
    (2, 4, 2, 300, 700, 64, True, 0.5),     # ragged, Nq < Nk
    (1, 2, 2, 700, 300, 64, False, 0.3),    # Nq > Nk
    (1, 2, 1, 512, 512, 256, False, 0.5),   # d=256: bitmap of the row
    (1, 2, 2, 400, 400, 256, True, 0.7),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,density", BLOCK_CASES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_block_mask_matches_oracle(B, Hq, Hkv, Nq, Nk, d, causal, density, out, cuda_device):
    q, k, v = inputs(B, Hq, Hkv, Nq, Nk, d, seed=4000 + Nq + d)
    bm = synth.block_mask(Nq, Nk, density, seed=4100 + Nk)
    bm[0, :] = 0  # one query block sees nothing at all
    scale = 1.0 / math.sqrt(d)
    ref_o, ref_l = attention(q, k, v, scale, causal, block_mask=bm)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    o, lse = run_masked(q, k, v, causal, scale, block_mask=bm, out_dtype=dt)
    compare_o(o, ref_o, bf16_out=(out == "bf16"))
    compare_lse(lse, ref_l)
    assert np.all(o[:, :, :128] == 0) and np.all(np.isneginf(lse[:, :, :128]))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_window_and_block_mask_together(d, cuda_device):
    Nq = Nk = 777
    q, k, v = inputs(1, 4, 2, Nq, Nk, d, seed=5000 + d)
    bm = synth.block_mask(Nq, Nk, 0.6, seed=5100 + d)
    scale = 1.0 / math.sqrt(d)
    ref_o, ref_l = attention(q, k, v, scale, True, window=250, block_mask=bm)
    o, lse = run_masked(q, k, v, True, scale, window=250, block_mask=bm)
    compare_o(o, ref_o, bf16_out=False)
    compare_lse(lse, ref_l)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_map_and_wide_window_change_nothing(d, causal, cuda_device):
    # the same blocks in the same order: results identical bit for bit
    Nq, Nk = 300, 420
    q, k, v = inputs(1, 4, 2, Nq, Nk, d, seed=6000 + d)
    scale = 1.0 / math.sqrt(d)
    o0, l0 = run_plain(q, k, v, causal, scale)
    ones = torch.ones(((Nq + 127) // 128, (Nk + 127) // 128), dtype=torch.uint8)
    o1, l1 = run_masked(q, k, v, causal, scale, block_mask=ones)
    assert np.array_equal(o0, o1.astype(np.float32)) and np.array_equal(l0, l1.astype(np.float32))
    if causal:
        o2, l2 = run_masked(q, k, v, True, scale, window=Nk)  # hides nothing
        assert np.array_equal(o0, o2.astype(np.float32)) and np.array_equal(l0, l2.astype(np.float32))


@pytest.mark.parametrize("d", [128, 256])
def test_all_zero_map_gives_zero_and_minus_inf(d, cuda_device):
    q, k, v = inputs(1, 2, 2, 260, 260, d, seed=7000 + d)
    zeros = torch.zeros((3, 3), dtype=torch.uint8)
    o, lse = run_masked(q, k, v, False, 0.1, block_mask=zeros)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("Nq,Nk,d,window", [(333, 333, 128, 100), (45, 300, 64, 17)])
def test_window_bf16_store_equals_rounded_fp32_output(Nq, Nk, d, window, cuda_device):
    q, k, v = inputs(1, 4, 2, Nq, Nk, d, seed=23 + Nq)
    scale = 1.0 / math.sqrt(d)
    o32, l32 = run_masked(q, k, v, True, scale, window=window, out_dtype=torch.float32)
    o16, l16 = run_masked(q, k, v, True, scale, window=window, out_dtype=torch.bfloat16)
    rounded = torch.from_numpy(np.asarray(o32, dtype=np.float64)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(np.asarray(o16, dtype=np.float64), rounded)
    assert np.array_equal(l16, l32)


def test_bad_masked_arguments_raise(cuda_device):
    q, k, v = inputs(1, 2, 2, 128, 128, 64, seed=1)
    dev = torch.device("cuda:0")
    o = torch.empty((1, 2, 128, 64), dtype=torch.float32, device=dev)
    with pytest.raises(ab.AttnError):
        ab.attn_fwd_masked(q.to(dev), k.to(dev), v.to(dev), o, None, False, 0.1, window=16)
    with pytest.raises(ValueError):
        ab.attn_fwd_masked(q.to(dev), k.to(dev), v.to(dev), o, None, False, 0.1,
                           block_mask=torch.ones((2, 2), dtype=torch.uint8, device=dev))


@pytest.mark.slow
@pytest.mark.parametrize("d,window", [(128, 4096), (64, 1000), (256, 2048)])
def test_long_window_sampled_rows(d, window, cuda_device):
    # a long causal sequence with a window: rows sampled across the whole range
    B, Hq, Hkv, N = 1, 8, 2, 16384
    q, k, v = inputs(B, Hq, Hkv, N, N, d, seed=8000 + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_masked(q, k, v, True, scale, window=window)
    rng = np.random.default_rng(8100 + d)
    rows = np.sort(np.concatenate([[0, window - 1, window, N - 1], rng.integers(0, N, 60)]))
    for hq in (0, 5):
        ref_o, ref_l = attention_rows(q, k, v, scale, True, 0, hq, rows, window=window)
        compare_o(o[0, hq, rows], ref_o, bf16_out=False)
        compare_lse(lse[0, hq, rows], ref_l)


@pytest.mark.slow
def test_long_block_sparse_sampled_rows(cuda_device):
    B, Hq, Hkv, N, d = 1, 8, 2, 16384, 128
    q, k, v = inputs(B, Hq, Hkv, N, N, d, seed=9000)
    bm = synth.block_mask(N, N, 0.25, seed=9100)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_masked(q, k, v, True, scale, block_mask=bm)
    rng = np.random.default_rng(9200)
    rows = np.sort(rng.integers(0, N, 64))
    for hq in (1, 6):
        ref_o, ref_l = attention_rows(q, k, v, scale, True, 0, hq, rows, block_mask=bm)
        compare_o(o[0, hq, rows], ref_o, bf16_out=False)
        compare_lse(lse[0, hq, rows], ref_l)
