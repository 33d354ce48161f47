"""The N > 1 host path of bench.py on CPU with gloo, world size 2: every rank runs its
own independent problem (no data-path collective) and timings are reduced to the
slowest rank's."""

import os
import socket
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from attn_fwd_05_b200 import synth
    d = bench.Dist()
    d.init("gloo")
    try:
        # per-rank device time: the job's time is the slowest rank's
        out[rank] = (d.max(10.0 + rank), bench.rank_seed(synth.workload_seed("gqa_causal_2k"), rank))
        d.barrier()
    finally:
        d.close()


def test_two_ranks_reduce_to_slowest_and_draw_independent_problems():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0
    assert out[0][1] != out[1][1]
    # the two seeds give different inputs of the same shape
    s = synth_shape()
    from attn_fwd_05_b200 import synth
    q0 = synth.normal_bf16((4, 8), out[0][1], 1)
    q1 = synth.normal_bf16((4, 8), out[1][1], 1)
    assert q0.shape == q1.shape and not torch.equal(q0, q1)


def synth_shape():
    from attn_fwd_05_b200 import synth
    return synth.WORKLOADS["gqa_causal_2k"]
