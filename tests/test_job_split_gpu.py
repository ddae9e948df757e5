"""The data path of one job split across ranks, on one GPU: each rank's slice of
the (relation, b, h) units (dist.rank_slices) runs through the grouped C-ABI
calls as [1, h1 - h0, n, d] views of the job's tensors, one slice after the
other, as the ranks of `bench.py --scaling strong` would.  The union of the
slices' results equals the whole job's, and the slices' summed loss equals
the job's loss (what the all-reduce forms)."""
import pytest
import torch

from linear_memory_attention_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lard():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_memory_attention_b200 import lard as L
    return L


@pytest.mark.parametrize("world", [2, 3, 7])
def test_slices_reproduce_the_whole_job(lard, world):
    from linear_memory_attention_b200 import dist as ldist
    w = synth.Workload("split B2 Hq5 Hkv3/2 n700 d128 bf16", 2, {"Q": 5, "K": 3, "V": 2}, 700, 128,
                       "bf16", 1e4, 1 / 8, 11)
    host = synth.make_all(w)
    dev = {r: (xt.cuda(), xs.cuda()) for r, (xt, xs) in host.items()}
    whole, loss = lard.relations_kl([dev[r] for r in w.relations], w.tau, True, fused_self=True,
                                    grad_dtype="bf16")
    torch.cuda.synchronize()
    whole = dict(zip(w.relations, whole))
    total = 0.0
    covered = {r: torch.zeros(w.B * w.heads[r], dtype=torch.bool) for r in w.relations}
    for rank in range(world):
        sl = ldist.rank_slices(w, world, rank)
        if not sl:
            continue
        pairs = [tuple(ldist.slice_heads(t, lo, hi) for t in dev[r]) for r, lo, hi in sl]
        assert all(t.is_contiguous() and t.shape[0] == 1 for p in pairs for t in p)
        outs, part = lard.relations_kl(pairs, w.tau, True, fused_self=True, grad_dtype="bf16")
        torch.cuda.synchronize()
        lard.lard_device_status()
        total += part.item()
        for (r, lo, hi), o in zip(sl, outs):
            W = whole[r]
            for key in ("lse_t", "lse_s", "row_kl"):
                ref = ldist.slice_heads(W[key], lo, hi)
                assert torch.equal(o[key], ref), f"{r} {key} of units [{lo}, {hi})"
            assert torch.equal(o["loss_bh"], W["loss_bh"][lo:hi])
            ref = ldist.slice_heads(W["dXs"], lo, hi).double()
            bound = 2.0 ** -7 * ref.abs() + 1e-6 * ref.abs().max().item() + 1e-30
            assert bool(((o["dXs"].double() - ref).abs() <= bound).all()), f"{r} dQ of units [{lo}, {hi})"
            covered[r][lo:hi] = True
    assert all(bool(c.all()) for c in covered.values()), "every unit is run by some rank"
    assert abs(total - loss.item()) <= 1e-5 * abs(loss.item())
