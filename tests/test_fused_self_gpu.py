"""GPU parity of lard_kl_bwd_self: the total student gradient of a self-relation
(Y = X), dL/dX_s through both of X_s's roles, against the oracle's dXs + dYs."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import TOL, assert_grad_close, f64, grad_floor
from linear_memory_attention_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lard():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_memory_attention_b200 import lard as L
    return L


def fused(lard, Xt, Xs, tau, causal, grad_scale=1.0):
    dev = torch.device("cuda:0")
    xt, xs = Xt.to(dev), Xs.to(dev)
    out = lard.relation_kl(xt, xs, tau, causal, backward=False)
    dq = torch.empty(xs.shape, device=dev, dtype=torch.float32)
    lard.lard_kl_bwd_self(xt, xs, tau, causal, out["lse_t"], out["lse_s"], grad_scale, dq)
    torch.cuda.synchronize()
    lard.lard_device_status()
    return dq.double().cpu().numpy()


@pytest.mark.parametrize("causal", [1, 0], ids=["causal", "full"])
@pytest.mark.parametrize("shape", [(1, 2, 1, 128), (1, 2, 129, 128), (2, 1, 300, 64), (1, 3, 517, 128)],
                         ids=lambda s: "B%dH%dn%dd%d" % s)
def test_fused_self_small(lard, shape, causal):
    B, H, n, d = shape
    w = synth.custom(B, H, n, d, "bf16", seed=n + 3 * d, causal=bool(causal))
    Xt, Xs = synth.make_relation(w, "Q")
    o = oracle.relation(f64(Xt), f64(Xt), f64(Xs), f64(Xs), w.tau, causal)
    want = o["dXs"] + o["dYs"]
    got = fused(lard, Xt, Xs, w.tau, causal)
    assert_grad_close(got, want, TOL["bf16"]["grad"], f"fused dQ {shape} causal={causal}",
                      grad_floor(f64(Xs), f64(Xs), w.tau, 1.0, n))


def test_fused_self_grad_scale(lard):
    w = synth.custom(1, 2, 200, 128, "bf16", seed=21)
    Xt, Xs = synth.make_relation(w, "K")
    o = oracle.relation(f64(Xt), f64(Xt), f64(Xs), f64(Xs), w.tau, 1)
    got = fused(lard, Xt, Xs, w.tau, 1, grad_scale=-2.5)
    assert_grad_close(got, -2.5 * (o["dXs"] + o["dYs"]), TOL["bf16"]["grad"], "fused dQ grad_scale",
                      grad_floor(f64(Xs), f64(Xs), w.tau, 2.5, w.n))


def test_fused_self_workload_n4096(lard):
    """The 4K workload's Q/Q relation at full size; two whole heads against the oracle."""
    w = synth.WORKLOADS["n4096"]
    Xt, Xs = synth.make_relation(w, "Q")
    got = fused(lard, Xt, Xs, w.tau, 1)
    assert np.isfinite(got).all()
    for h in (0, 31):
        xt, xs = f64(Xt[0, h]), f64(Xs[0, h])
        o = oracle.relation(xt, xt, xs, xs, w.tau, True)
        assert_grad_close(got[0, h], o["dXs"] + o["dYs"], TOL["bf16"]["grad"], f"fused dQ n4096 head {h}",
                          grad_floor(xs, xs, w.tau, 1.0, w.n))


def test_fused_self_rejects_fp32(lard):
    dev = torch.device("cuda:0")
    x = torch.randn((1, 1, 64, 64), device=dev)
    f = torch.zeros((1, 1, 64), device=dev)
    dq = torch.empty_like(x)
    with pytest.raises(lard.LardError) as e:
        lard.lard_kl_bwd_self(x, x.clone(), 1 / math.sqrt(64), 1, f, f.clone(), 1.0, dq)
    assert e.value.status == lard.LARD_ERR_UNSUPPORTED
