"""The multi-rank paths on CPU (gloo ranks): weak scaling, where each rank runs
its own batch, and one job whose (relation, batch, head) units are split
across the ranks, whose only data-path exchange is the all-reduce of the
loss.  The timing reduction (max over ranks) is the other exchange."""
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


# ------------------------------------------------------------------ one job split across ranks

def test_partition_is_disjoint_complete_and_balanced():
    from linear_memory_attention_b200 import dist as ldist
    for units in ([("Q", 32), ("K", 32), ("V", 32)], [("Q", 64), ("K", 16), ("V", 16)], [("Q", 3)],
                  [("Q", 5), ("K", 1), ("V", 2)]):
        U = sum(c for _, c in units)
        for world in range(1, 12):
            seen = {}
            sizes = []
            prev_end = 0
            for rank in range(world):
                sl = ldist.partition_units(units, world, rank)
                size = 0
                for rel, lo, hi in sl:
                    assert 0 <= lo < hi <= dict(units)[rel]
                    for u in range(lo, hi):
                        assert (rel, u) not in seen, "a unit given to two ranks"
                        seen[(rel, u)] = rank
                    size += hi - lo
                # contiguous in the job's unit order, following the previous rank
                flat = [sum(c for r, c in units[:[r for r, _ in units].index(rel)]) + u
                        for rel, lo, hi in sl for u in range(lo, hi)]
                assert flat == list(range(prev_end, prev_end + size))
                prev_end += size
                sizes.append(size)
            assert len(seen) == U, "every unit is run once"
            assert max(sizes) - min(sizes) <= 1, "equal work per rank (every unit costs the same)"


def _split_worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import oracle
    from linear_memory_attention_b200 import dist as ldist, synth
    ldist.init("gloo", timeout_s=60)
    w = _split_workload()
    host = synth.make_all(w)
    loss = torch.zeros(1, dtype=torch.float64)
    mine = {}
    for rel, lo, hi in ldist.rank_slices(w, world, rank):
        xt, xs = (ldist.slice_heads(t, lo, hi).to(torch.float64).numpy() for t in host[rel])
        o = oracle.relation(xt, xt, xs, xs, w.tau, w.causal)
        loss += o["loss"]
        for k in range(hi - lo):
            mine[(rel, lo + k)] = (o["lse_s"][0, k].copy(), o["dXs"][0, k].copy())
    ldist.all_reduce_loss(loss)
    out[rank] = (float(loss.item()), mine)
    dist.barrier()
    dist.destroy_process_group()


def _split_workload():
    from linear_memory_attention_b200 import synth
    # GQA-like head counts with B = 2: 10 + 2 + 4 = 16 units, which 2 or 3 ranks cut mid-relation
    return synth.Workload("split test B2 Hq5 Hkv1/2 n37 d8 fp32", 2, {"Q": 5, "K": 1, "V": 2}, 37, 8,
                          "fp32", 1e4, 1 / 8, 7)


@pytest.mark.parametrize("world", [2, 3])
def test_job_split_across_gloo_ranks(world):
    """Each rank runs its slice of one job's units (oracle on CPU); the summed
    loss after the all-reduce equals the one-rank loss, and the per-unit
    results of the slices are the one-rank results."""
    import oracle
    from linear_memory_attention_b200 import synth
    oracle.default()  # build before the ranks start
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_split_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    w = _split_workload()
    host = synth.make_all(w)
    want = 0.0
    units = {}
    for rel in w.relations:
        xt, xs = (t.to(torch.float64).numpy() for t in host[rel])
        o = oracle.relation(xt, xt, xs, xs, w.tau, w.causal)
        want += o["loss"]
        H = w.heads[rel]
        for b in range(w.B):
            for h in range(H):
                units[(rel, b * H + h)] = (o["lse_s"][b, h], o["dXs"][b, h])
    losses = [out[r][0] for r in range(world)]
    assert all(x == losses[0] for x in losses), "every rank holds the same job loss"
    assert losses[0] == pytest.approx(want, rel=1e-12)
    got = {}
    for r in range(world):
        for key, val in out[r][1].items():
            assert key not in got
            got[key] = val
    assert set(got) == set(units)
    for key, (lse, dx) in units.items():
        assert abs(got[key][0] - lse).max() == 0.0 and abs(got[key][1] - dx).max() == 0.0
