"""The multi-rank path on CPU: two gloo ranks, each with its own batch; the
timing reduction (max over ranks) and the loss sum are the only exchanges."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from linear_memory_attention_b200 import dist as ldist, synth
    r, wsz, lr = ldist.env_ranks()
    assert (r, wsz, lr) == (rank, world, rank)
    assert ldist.init("gloo", timeout_s=60) == world
    w = synth.WORKLOADS["fp32-small"]
    wr = ldist.rank_workload(w, rank)
    xt, xs = synth.make_relation(wr, "Q")
    elapsed = 10.0 + rank  # the slower rank decides the job's time
    mx = ldist.max_over_ranks(elapsed)
    total = ldist.sum_over_ranks(float(rank + 1))
    rate = ldist.aggregate_rate(w.causal_logits(), 5, world, mx)
    out[rank] = (tuple(xt.shape), float(xt.double().sum()), mx, total, rate)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    a, b = out[0], out[1]
    assert a[0] == b[0], "ranks run the same shapes"
    assert a[1] != b[1], "each rank draws its own batch"
    assert a[2] == b[2] == 11.0, "time is the max over ranks"
    assert a[3] == b[3] == 3.0, "loss is summed over ranks"
    from linear_memory_attention_b200 import synth
    w = synth.WORKLOADS["fp32-small"]
    assert a[4] == pytest.approx(w.causal_logits() * 5 * world / 11e-3)


def test_single_rank_is_identity():
    from linear_memory_attention_b200 import dist as ldist
    assert ldist.max_over_ranks(3.5) == 3.5 and ldist.sum_over_ranks(2.0) == 2.0
    assert ldist.aggregate_rate(100, 2, 1, 1000.0) == 200.0
