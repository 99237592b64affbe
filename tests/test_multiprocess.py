"""The N > 1 path on CPU: two gloo ranks over 127.0.0.1.

The hot path shards into independent (sequence, KV head) units with no
exchange step: each rank takes its own sequences, and only the timing and the
work are reduced (max of the step time, sum of the work). These tests run the
bench's reductions on gloo and check that sharding the sequences across ranks
gives the same oracle outputs as one process over all of them.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    from dynamic_block_sparse_nsa_b200 import inputs
    from tests import gpu_cases as gc
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=4, T=300, Hq=4, Hkv=1, d=32, top_n=3,
                        window=40, dtype="f32")
    inp = inputs.make_decode(w, seed=3, seq_lens=[300, 211, 64, 299])
    return w, inp, gc.oracle_params_for(dict(w, B=1))


def _oracle_decode(w, inp, op, bs):
    """Oracle decode output of sequences `bs` (one row each, at seq_len - 1)."""
    import oracle
    outs = []
    for b in bs:
        L = int(inp["seq_lens"][b])
        k = inp["k"][b:b + 1].double().numpy()
        v = inp["v"][b:b + 1].double().numpy()
        kc, vc = oracle.compress(op, k, v, inp["w_cmp"].double().numpy())
        res = oracle.nsa_rows(op, [0], [L - 1], inp["q"][b:b + 1].double().numpy(), k, v, kc, vc,
                              inp["w_gate"].double().numpy())
        outs.append(res["out"][0])
    return np.stack(outs)


def _worker(rank, port, queue):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        step_ms = [3.0, 5.0][rank]
        mx = bench.reduce_max(step_ms, WORLD)
        sm = bench.reduce_sum(100.0 * (rank + 1), WORLD)
        bench.barrier(WORLD)
        w, inp, op = _case()
        mine = list(range(rank, w["B"], WORLD))  # this rank's sequences
        out = _oracle_decode(w, inp, op, mine)
        queue.put((rank, mx, sm, mine, out))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_shard_sequences():
    port = _free_port()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, port, queue)) for r in range(WORLD)]
    for p in procs:
        p.start()
    got = [queue.get(timeout=180) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, inp, op = _case()
    full = _oracle_decode(w, inp, op, range(w["B"]))
    for rank, mx, sm, mine, out in got:
        assert mx == 5.0           # the job's step time is the slowest rank's
        assert sm == 300.0         # the job's work is every rank's work
        np.testing.assert_array_equal(out, full[mine])  # no cross-shard dependency
