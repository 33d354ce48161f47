"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle on the same seeded bf16 inputs.

Tolerances (O is the attention output, compared element by element):
* fp32 O (attn_fwd_ex with an fp32 output): max |err| <= 1e-2, mean |err| <= 1e-3;
* LSE: max |err| <= 1e-3 (and -inf exactly where no key is visible);
* bf16 O: the same bounds plus the unavoidable bf16 rounding of the output itself,
  half a bf16 unit (2^-9 relative) of the exact value.
"""

from __future__ import annotations

import numpy as np
import torch

import attn_fwd_05_b200 as ab

O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def run_prefill(q, k, v, causal: bool, scale: float, out_dtype=torch.float32, with_lse=True):
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    B, Hq, Nq, d = q.shape
    o = torch.empty((B, Hq, Nq, d), dtype=out_dtype, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev) if with_lse else None
    ab.attn_fwd_ex(qd, kd, vd, o, lse, causal, scale)
    status = ab.attn_get_device_status()
    assert status == 0, ab.attn_status_string(status)
    return o.double().cpu().numpy(), (lse.double().cpu().numpy() if with_lse else None)


def compare_o(o, ref, bf16_out: bool, o_max=O_MAX, o_mean=O_MEAN):
    err = np.abs(o - ref)
    slack = np.abs(ref) * 2.0 ** -9 if bf16_out else 0.0
    excess = err - slack
    assert np.all(np.isfinite(o)), "non-finite output"
    assert excess.max() <= o_max, f"max |O err| {err.max():.3e} (excess {excess.max():.3e})"
    mean_bound = o_mean + (float(np.mean(slack)) if bf16_out else 0.0)
    assert err.mean() <= mean_bound, f"mean |O err| {err.mean():.3e} > {mean_bound:.3e}"
    return float(err.max()), float(err.mean())


def compare_lse(lse, ref, lse_max=LSE_MAX):
    inf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(lse), inf_ref), "-inf pattern of LSE differs"
    fin = ~inf_ref
    if fin.any():
        e = np.abs(lse[fin] - ref[fin]).max()
        assert e <= lse_max, f"max |LSE err| {e:.3e}"
        return float(e)
    return 0.0
