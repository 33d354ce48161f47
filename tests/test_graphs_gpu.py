"""The entry points inside a CUDA graph: a prefill, its backward pass and a paged decode
step are captured once and replayed, and the replay must reproduce the eager calls bit
for bit.  The backward pass accumulates dQ by additions in L2 whose order varies from run
to run, so its dQ is compared within a few fp32 ulps of the eager call instead."""

import math

import numpy as np
import pytest
import torch

import attn_fwd_05_b200 as ab
from attn_fwd_05_b200 import synth

pytestmark = pytest.mark.gpu


def test_prefill_backward_decode_replay_matches_eager(cuda_device):
    dev = torch.device("cuda:0")
    shape = synth.PrefillShape(B=1, Hq=4, Hkv=2, Nq=300, Nk=300, d=128, causal=True)
    q, k, v = (t.to(dev) for t in synth.prefill_inputs(shape, 31))
    do = synth.upstream_grad(shape, 31).to(dev)
    scale = 1.0 / math.sqrt(shape.d)
    o = torch.empty((1, 4, 300, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 4, 300), dtype=torch.float32, device=dev)
    dq = torch.empty((1, 4, 300, 128), dtype=torch.float32, device=dev)
    dk = torch.empty((1, 2, 300, 128), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)
    bws = torch.empty(max(ab.attn_bwd_workspace_size(1, 4, 300), 16), dtype=torch.uint8, device=dev)

    dshape = synth.DecodeShape(S=4, Hq=8, Hkv=2, d=128, page_size=16, len_lo=100, len_hi=3000)
    kv = synth.decode_inputs(dshape, 32)
    dq_in, kp, vp, bt, sl = (t.to(dev) for t in (kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens))
    S, Hq, d = kv.q.shape
    do_ = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=dev)
    dlse = torch.empty((S, Hq), dtype=torch.float32, device=dev)
    dws = torch.empty(ab.attn_decode_paged_workspace_size(S, Hq, kv.k_pool.shape[1], d, kv.max_pages_per_seq,
                                                          kv.page_size), dtype=torch.uint8, device=dev)
    outs = (o, lse, dq, dk, dv, do_, dlse)

    def step():
        ab.attn_fwd(q, k, v, o, lse, True, scale)
        ab.attn_bwd(q, k, v, o, do, lse, dq, dk, dv, True, scale, bws)
        ab.attn_decode_paged(dq_in, kp, vp, bt, sl, kv.page_size, do_, dlse, 1.0 / math.sqrt(d), dws)

    # eager (also sets the kernels' shared-memory limits)
    step()
    torch.cuda.synchronize()
    assert ab.attn_get_device_status() == 0
    eager = [t.clone() for t in outs]

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in outs:
        t.fill_(float("nan"))
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert ab.attn_get_device_status() == 0
    for i, (ref, got) in enumerate(zip(eager, outs)):
        if got is dq:  # sums in L2 in an order that varies: a few fp32 roundings apart
            assert torch.isfinite(got).all()
            assert (got - ref).abs().max().item() <= 1e-5 * ref.abs().max().item()
        else:
            assert torch.equal(ref.view(torch.uint8), got.view(torch.uint8)), i
    del g
    assert np.isfinite(eager[0].float().cpu().numpy()).all()
