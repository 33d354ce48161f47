"""Byte-count helpers against the sizes the pages print (tests/golden/page_sizes.json),
and the FLOP counts of the five workloads against their plain definitions."""

import json
import os

import pytest

from attn_fwd_05_b200 import counts, synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_sizes.json")
CASES = json.load(open(GOLDEN))["cases"]


@pytest.mark.parametrize("case", CASES, ids=[c["helper"] + ":" + c["what"][:30] for c in CASES])
def test_page_printed_sizes(case):
    got = getattr(counts, case["helper"])(**case["args"])
    want = case["value"]
    assert abs(got - want) <= case["rel_tol"] * want + 1e-9, (got, want)


def test_workload_flops():
    s = synth.WORKLOADS["gqa_causal_2k"]
    assert counts.prefill_flops(s.B, s.Hq, s.Nq, s.Nk, s.d, s.causal) == 0.5 * 4 * 4 * 32 * 2048 * 2048 * 128
    s = synth.WORKLOADS["gqa_causal_16k"]
    assert abs(counts.prefill_flops(s.B, s.Hq, s.Nq, s.Nk, s.d, s.causal) - 4.398e12) < 1e9
    s = synth.WORKLOADS["peaked_mha_d256"]
    assert abs(counts.prefill_flops(s.B, s.Hq, s.Nq, s.Nk, s.d, s.causal) - 549.8e9) < 1e8
    s = synth.WORKLOADS["tiny_mha_d64"]
    assert counts.prefill_flops(s.B, s.Hq, s.Nq, s.Nk, s.d, s.causal) == 4 * 2 * 128 * 128 * 64


def test_decode_bytes():
    # 64 sequences of 16640 tokens, 8 KV heads, d = 128, bf16 K and V: about 4.36 GB
    assert abs(counts.decode_kv_bytes([16640] * 64, 8, 128) - 4.36e9) < 0.01e9
