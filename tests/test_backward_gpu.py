"""GPU parity of the backward pass (attn_bwd) against the fp64 backward oracle.

Tolerance, derived from the arithmetic (the parity bar of the forward pass says nothing
about gradients).  The kernels compute P and dS in fp32, round both to bf16 as
tensor-core operands (relative error <= 2^-9 each) and accumulate in fp32; Delta =
rowsum(dO o O) uses the forward's bf16 O, whose own error dO_gpu - O_exact enters dS as
P (Delta_gpu - Delta).  Element by element, with eps = 2^-8 (twice the rounding unit):
    |dV err| <= eps |P|^T |dO|
    |dQ err| <= scale (eps |dS| + P |dDelta|) |K|
    |dK err| <= scale (eps |dS| + P |dDelta|)^T |Q|
plus an fp32 accumulation allowance of N 2^-22 times the same magnitudes and an absolute
floor of 1e-6 max|ref|.  dDelta is measured from the GPU's own O.
"""

import math

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth
from oracle import attention_head_backward, kv_head_of

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -8


def run_case(B, Hq, Hkv, Nq, Nk, d, causal, seed):
    shape = synth.PrefillShape(B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=d, causal=causal)
    q, k, v = synth.prefill_inputs(shape, seed)
    do = synth.upstream_grad(shape, seed)
    scale = 1.0 / math.sqrt(d)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    ab.attn_fwd(qd, kd, vd, o, lse, causal, scale)
    dq = torch.full((B, Hq, Nq, d), float("nan"), dtype=torch.float32, device=dev)
    dk = torch.full((B, Hkv, Nk, d), float("nan"), dtype=torch.float32, device=dev)
    dv = torch.full((B, Hkv, Nk, d), float("nan"), dtype=torch.float32, device=dev)
    ab.attn_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, causal, scale)
    status = ab.attn_get_device_status()
    assert status == 0, ab.attn_status_string(status)
    return (q, k, v, do, scale), o.double().cpu().numpy(), (dq.double().cpu().numpy(), dk.double().cpu().numpy(),
                                                          dv.double().cpu().numpy())


def reference_and_bounds(q, k, v, do, scale, causal, o_gpu):
    q, k, v, do = (t.double().numpy() for t in (q, k, v, do))
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    ref = [np.zeros_like(q), np.zeros((B, Hkv, Nk, d)), np.zeros((B, Hkv, Nk, d))]
    bnd = [np.zeros_like(q), np.zeros((B, Hkv, Nk, d)), np.zeros((B, Hkv, Nk, d))]
    acc = (max(Nq, Nk) + 16) * 2.0 ** -22
    for b in range(B):
        for h in range(Hq):
            kv = kv_head_of(h, Hq, Hkv)
            gq, gk, gv, P, dS, delta = attention_head_backward(q[b, h], k[b, kv], v[b, kv], do[b, h], scale, causal,
                                                               want_parts=True)
            ref[0][b, h] = gq
            ref[1][b, kv] += gk
            ref[2][b, kv] += gv
            O = P @ v[b, kv]
            d_delta = np.abs(np.sum(do[b, h] * (o_gpu[b, h] - O), axis=1))
            wq = EPS * np.abs(dS) + P * d_delta[:, None]
            bnd[0][b, h] = scale * ((wq + acc * np.abs(dS)) @ np.abs(k[b, kv]))
            bnd[1][b, kv] += scale * ((wq + acc * np.abs(dS)).T @ np.abs(q[b, h]))
            bnd[2][b, kv] += (EPS + acc) * (P.T @ np.abs(do[b, h]))
    return ref, bnd


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 2, 2, 128, 128, 64, False),
    (1, 4, 2, 256, 256, 128, True),     # GQA causal, dK/dV summed over the group
    (2, 4, 1, 200, 200, 128, False),    # MQA, ragged tail
    (1, 2, 2, 333, 333, 64, True),      # ragged, causal
    (1, 4, 2, 100, 300, 128, True),     # Nq < Nk: bottom-right alignment
    (1, 2, 1, 300, 100, 128, True),     # Nq > Nk: rows without visible keys
    (1, 2, 2, 1, 200, 64, False),       # one query row
    (1, 8, 2, 512, 512, 128, True),     # several tiles in both directions
    (1, 4, 2, 8200, 8200, 64, True),    # 65 key tiles: the grid takes them in bands of 64, a short last band
    (1, 2, 1, 8200, 8200, 128, True),   # the same at d = 128 (dQ_step shares the dP^T columns)
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", CASES)
def test_backward_matches_oracle(B, Hq, Hkv, Nq, Nk, d, causal, cuda_device):
    inputs, o_gpu, got = run_case(B, Hq, Hkv, Nq, Nk, d, causal, seed=7000 + Nq + Nk + d)
    ref, bnd = reference_and_bounds(*inputs, causal, o_gpu)
    for name, g, r, e in zip(("dq", "dk", "dv"), got, ref, bnd):
        assert np.all(np.isfinite(g)), f"{name} not finite"
        err = np.abs(g - r)
        floor = 1e-6 * max(np.abs(r).max(), 1e-30)
        bad = err > e + floor
        assert not bad.any(), (f"{name}: {bad.sum()} elements over the bound, worst excess "
                               f"{(err - e).max():.3e}, max |err| {err.max():.3e}, max |ref| {np.abs(r).max():.3e}")
        rel = err.mean() / max(np.abs(r).mean(), 1e-30)
        assert rel < EPS, f"{name}: mean relative error {rel:.3e}"


def test_backward_conservation_on_gpu(cuda_device):
    # sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i (per head, non-causal, every row sees a key)
    inputs, _, (dq, dk, dv) = run_case(1, 2, 2, 256, 256, 128, False, seed=99)
    q, k, v, do, scale = inputs
    do = do.double().numpy()
    for h in range(2):
        s = np.abs(dk[0, h]).sum(axis=0)
        assert np.all(np.abs(dk[0, h].sum(axis=0)) <= 1e-2 * s + 1e-6)
        np.testing.assert_allclose(dv[0, h].sum(axis=0), do[0, h].sum(axis=0), rtol=2e-2, atol=2e-2)


def test_no_query_or_no_key(cuda_device):
    dev = torch.device("cuda:0")
    q = torch.zeros((1, 2, 0, 64), dtype=torch.bfloat16, device=dev)
    k = torch.randn((1, 2, 130, 64), device=dev).to(torch.bfloat16)
    dk = torch.full((1, 2, 130, 64), 7.0, device=dev)
    dv = torch.full((1, 2, 130, 64), 7.0, device=dev)
    ab.attn_bwd(q, k, k, q, q, torch.zeros((1, 2, 0), device=dev), torch.zeros((1, 2, 0, 64), device=dev), dk, dv,
                False, 0.1)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0)
    q = torch.randn((1, 2, 50, 64), device=dev).to(torch.bfloat16)
    k0 = torch.zeros((1, 2, 0, 64), dtype=torch.bfloat16, device=dev)
    dq = torch.full((1, 2, 50, 64), 7.0, device=dev)
    ab.attn_bwd(q, k0, k0, q, q, torch.full((1, 2, 50), -float("inf"), device=dev), dq,
                torch.zeros((1, 2, 0, 64), device=dev), torch.zeros((1, 2, 0, 64), device=dev), False, 0.1)
    torch.cuda.synchronize()
    assert torch.all(dq == 0)


def test_backward_rejects_d256(cuda_device):
    dev = torch.device("cuda:0")
    x = torch.zeros((1, 1, 16, 256), dtype=torch.bfloat16, device=dev)
    g = torch.zeros((1, 1, 16, 256), device=dev)
    with pytest.raises(ab.AttnError):
        ab.attn_bwd(x, x, x, x, x, torch.zeros((1, 1, 16), device=dev), g, g, g, False, 0.1)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["gqa_causal_2k"])
def test_backward_full_size_one_group(name, cuda_device):
    # the whole workload on the GPU; the oracle on the query heads of one K/V head
    s = synth.WORKLOADS[name]
    seed = synth.workload_seed(name)
    q, k, v = synth.prefill_inputs(s, seed)
    do = synth.upstream_grad(s, seed)
    scale = synth.default_scale(s.d)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o = torch.empty((s.B, s.Hq, s.Nq, s.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((s.B, s.Hq, s.Nq), dtype=torch.float32, device=dev)
    ab.attn_fwd(qd, kd, vd, o, lse, s.causal, scale)
    dq = torch.empty((s.B, s.Hq, s.Nq, s.d), dtype=torch.float32, device=dev)
    dk = torch.empty((s.B, s.Hkv, s.Nk, s.d), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)
    ab.attn_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, s.causal, scale)
    assert ab.attn_get_device_status() == 0
    b, kv = s.B - 1, s.Hkv - 1
    G = s.Hq // s.Hkv
    heads = list(range(kv * G, (kv + 1) * G))
    sub = lambda t, hs: t[b:b + 1, hs]  # noqa: E731
    ref, bnd = reference_and_bounds(sub(q, heads), sub(k, [kv]), sub(v, [kv]), sub(do, heads), scale, s.causal,
                                    o[b:b + 1, heads].double().cpu().numpy())
    got = (dq[b:b + 1, heads].double().cpu().numpy(), dk[b:b + 1, [kv]].double().cpu().numpy(),
           dv[b:b + 1, [kv]].double().cpu().numpy())
    for name_, g, r, e in zip(("dq", "dk", "dv"), got, ref, bnd):
        err = np.abs(g - r)
        assert not (err > e + 1e-6 * np.abs(r).max()).any(), f"{name_}: max excess {(err - e).max():.3e}"
