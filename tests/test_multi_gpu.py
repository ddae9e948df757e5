"""GPU checks of lard_kl_fwd_multi / lard_kl_bwd_multi: several relations (with
their own head counts, as Q/Q against GQA K/K and V/V) in one launch per phase
give what one call per relation gives, and match the oracle."""
import pytest
import torch

import oracle
from parity_util import TOL, assert_close_abs, assert_grad_close, assert_kl_close, f64, grad_floor
from linear_memory_attention_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lard():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_memory_attention_b200 import lard as L
    return L


def _pairs(heads, n, d, dtype, seed, causal=True):
    dev = torch.device("cuda:0")
    out = []
    for k, (rel, H) in enumerate(heads):
        w = synth.custom(2, H, n, d, dtype, seed=seed + k, causal=causal, relations=(rel,))
        Xt, Xs = synth.make_relation(w, rel)
        out.append((Xt.to(dev), Xs.to(dev)))
    return out, w.tau


@pytest.mark.parametrize("causal", [1, 0], ids=["causal", "full"])
def test_multi_equals_separate_calls(lard, causal):
    """Q with 4 heads, K and V with 1 (a GQA layout), n with a ragged tail."""
    pairs, tau = _pairs([("Q", 4), ("K", 1), ("V", 1)], 1000, 128, "bf16", 50, bool(causal))
    multi, loss = lard.relations_kl(pairs, tau, causal)
    torch.cuda.synchronize()
    lard.lard_device_status()
    total = 0.0
    for (xt, xs), m in zip(pairs, multi):
        one = lard.relation_kl(xt, xs, tau, causal)
        torch.cuda.synchronize()
        for key in ("lse_t", "lse_s", "row_kl", "loss_bh", "dYs"):
            assert torch.equal(m[key], one[key]), key
        torch.testing.assert_close(m["dXs"], one["dXs"], rtol=1e-5, atol=1e-6 * one["dXs"].abs().max().item())
        total += one["loss"].item()
    assert abs(loss.item() - total) <= 1e-5 * abs(total) + 1e-7


def test_multi_against_oracle(lard):
    pairs, tau = _pairs([("Q", 3), ("V", 2)], 333, 64, "bf16", 60)
    multi, loss = lard.relations_kl(pairs, tau, True)
    torch.cuda.synchronize()
    tol = TOL["bf16"]
    for k, ((xt, xs), m) in enumerate(zip(pairs, multi)):
        b, h = 1, xt.shape[1] - 1
        Xt, Xs = f64(xt[b, h]), f64(xs[b, h])
        o = oracle.relation(Xt, Xt, Xs, Xs, tau, True)
        what = f"multi relation {k} head ({b},{h})"
        assert_close_abs(m["lse_t"][b, h].double().cpu().numpy(), o["lse_t"], tol["lse"], what + " lse_t")
        assert_close_abs(m["lse_s"][b, h].double().cpu().numpy(), o["lse_s"], tol["lse"], what + " lse_s")
        assert_kl_close(m["row_kl"][b, h].double().cpu().numpy(), o["row_kl"], tol, what + " row_kl")
        floor = grad_floor(Xs, Xs, tau, 1.0, 333)
        assert_grad_close(m["dXs"][b, h].double().cpu().numpy(), o["dXs"], tol["grad"], what + " dXs", floor)
        assert_grad_close(m["dYs"][b, h].double().cpu().numpy(), o["dYs"], tol["grad"], what + " dYs", floor)


def test_multi_fused_self(lard):
    pairs, tau = _pairs([("Q", 2), ("K", 2), ("V", 1)], 400, 128, "bf16", 70)
    multi, _ = lard.relations_kl(pairs, tau, True, fused_self=True)
    torch.cuda.synchronize()
    lard.lard_device_status()
    for (xt, xs), m in zip(pairs, multi):
        assert "dYs" not in m
        one = lard.relation_kl(xt, xs, tau, True)
        torch.cuda.synchronize()
        want = one["dXs"] + one["dYs"]
        torch.testing.assert_close(m["dXs"], want, rtol=1e-5, atol=1e-6 * want.abs().max().item())


def test_multi_fp32(lard):
    pairs, tau = _pairs([("Q", 2), ("K", 1)], 200, 64, "fp32", 80)
    multi, loss = lard.relations_kl(pairs, tau, True)
    torch.cuda.synchronize()
    total = 0.0
    for (xt, xs), m in zip(pairs, multi):
        one = lard.relation_kl(xt, xs, tau, True)
        torch.cuda.synchronize()
        for key in ("lse_t", "lse_s", "row_kl", "loss_bh", "dXs", "dYs"):
            assert torch.equal(m[key], one[key]), key
        total += one["loss"].item()
    assert abs(loss.item() - total) <= 1e-6 * abs(total) + 1e-9
