"""Several layers (or relations of equal shape) in one call, as extra heads.

The method distils the relation maps of one or more layers (LinearARD notes,
实验关键数据: last layer only against all layers).  Heads are independent
units, so stacking L layers along H must give, head by head, what L separate
calls give: the same row statistics and losses bit for bit (each head's
forward is computed by the same blocks in the same order) and the same
gradients up to the order of the dX reduce-adds."""
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


@pytest.mark.parametrize("causal", [1, 0], ids=["causal", "full"])
def test_layers_as_heads(lard, causal):
    dev = torch.device("cuda:0")
    layers = []
    for seed in (31, 32, 33):
        w = synth.custom(1, 4, 777, 128, "bf16", seed=seed, causal=bool(causal))
        layers.append(synth.make_relation(w, "K"))
    tau = w.tau
    sep = [lard.relation_kl(xt.to(dev), xs.to(dev), tau, causal) for xt, xs in layers]
    Xt = torch.cat([xt for xt, _ in layers], dim=1).to(dev)
    Xs = torch.cat([xs for _, xs in layers], dim=1).to(dev)
    both = lard.relation_kl(Xt, Xs, tau, causal)
    torch.cuda.synchronize()
    lard.lard_device_status()
    for key in ("lse_t", "lse_s", "row_kl"):
        assert torch.equal(both[key], torch.cat([o[key] for o in sep], dim=1)), key
    assert torch.equal(both["loss_bh"], torch.cat([o["loss_bh"] for o in sep]))
    torch.testing.assert_close(both["loss"], sum(o["loss"] for o in sep), rtol=1e-6, atol=1e-9)
    assert torch.equal(both["dYs"], torch.cat([o["dYs"] for o in sep], dim=1))
    dx = torch.cat([o["dXs"] for o in sep], dim=1)
    torch.testing.assert_close(both["dXs"], dx, rtol=1e-5, atol=1e-6 * dx.abs().max().item())
