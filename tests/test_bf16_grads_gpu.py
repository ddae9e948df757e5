"""GPU parity of the bf16 gradient outputs (lard_kl_bwd_multi_bf16): the
gradients, accumulated in fp32 and rounded once to bf16, against the oracle
at the bf16 gradient bar, and against the fp32 outputs of lard_kl_bwd_multi
within the bf16 rounding."""
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


def _pairs(spec, B, n, d, seed, causal):
    out = []
    for k, (rel, H) in enumerate(spec):
        w = synth.custom(B, H, n, d, "bf16", seed=seed + k, causal=causal, relations=(rel,))
        Xt, Xs = synth.make_relation(w, rel)
        out.append((Xt.cuda(), Xs.cuda()))
    return out, w.tau


def _close_to_fp32(got16, want32, what):
    """bf16 = round(fp32 accumulation): within one bf16 rounding (2^-8 relative,
    a little more for dX, whose fp32 sum is reassociated between runs)."""
    g, w = got16.double(), want32.double()
    scale = w.abs().max().item()
    err = (g - w).abs()
    bound = 2.0 ** -8 * w.abs() + 1e-6 * scale + 1e-30
    assert bool((err <= bound).all()), f"{what}: max err {err.max().item():.3e}"


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("n,d", [(1, 128), (129, 128), (300, 64), (517, 128)])
def test_bf16_outputs_match_oracle_and_fp32(lard, n, d, causal):
    pairs, tau = _pairs((("Q", 2), ("K", 1), ("V", 3)), 2, n, d, seed=n + d, causal=causal)
    o32, loss32 = lard.relations_kl(pairs, tau, causal)
    o16, loss16 = lard.relations_kl(pairs, tau, causal, grad_dtype="bf16")
    f16, _ = lard.relations_kl(pairs, tau, causal, fused_self=True, grad_dtype="bf16")
    torch.cuda.synchronize()
    lard.lard_device_status()
    assert loss16.item() == loss32.item()
    tol = TOL["bf16"]
    for k, ((xt, xs), a, b, c) in enumerate(zip(pairs, o32, o16, f16)):
        assert b["dXs"].dtype == torch.bfloat16 and c["dXs"].dtype == torch.bfloat16 and "dYs" not in c
        _close_to_fp32(b["dYs"], a["dYs"], f"relation {k} dYs")
        _close_to_fp32(b["dXs"], a["dXs"], f"relation {k} dXs")
        _close_to_fp32(c["dXs"], a["dXs"] + a["dYs"], f"relation {k} fused dQ")
        bb, hh = 1, xt.shape[1] - 1
        X_t, X_s = f64(xt[bb, hh]), f64(xs[bb, hh])
        o = oracle.relation(X_t, X_t, X_s, X_s, tau, causal)
        floor = grad_floor(X_s, X_s, tau, 1.0, n)
        what = f"bf16 outputs n={n} d={d} relation {k}"
        assert_grad_close(f64(b["dXs"][bb, hh]), o["dXs"], tol["grad"], what + " dXs", floor)
        assert_grad_close(f64(b["dYs"][bb, hh]), o["dYs"], tol["grad"], what + " dYs", floor)
        assert_grad_close(f64(c["dXs"][bb, hh]), o["dXs"] + o["dYs"], tol["grad"], what + " dQ", floor)


def test_bf16_outputs_grad_scale_and_workspace_reuse(lard):
    """grad_scale is applied before the rounding; a workspace holding another
    call's values is overwritten (it needs no clearing by the caller)."""
    pairs, tau = _pairs((("Q", 2),), 1, 700, 128, seed=5, causal=True)
    rels32, _ = lard.relations_kl(pairs, tau, True, grad_scale=-2.5)
    base, _ = lard.relations_kl(pairs, tau, True, backward=False)
    rel = [dict(Xt=pairs[0][0], Xs=pairs[0][1], lse_t=base[0]["lse_t"], lse_s=base[0]["lse_s"],
                dXs=torch.empty_like(pairs[0][0]), dYs=torch.empty_like(pairs[0][0]))]
    ws = torch.full((lard.lard_kl_bwd_bf16_workspace_bytes(rel) // 4 + 7,), 3.0e7, device="cuda")
    for _ in range(2):
        lard.lard_kl_bwd_multi_bf16(rel, tau, True, -2.5, ws)
        torch.cuda.synchronize()
        lard.lard_device_status()
        _close_to_fp32(rel[0]["dXs"], rels32[0]["dXs"], "dXs, scaled")
        _close_to_fp32(rel[0]["dYs"], rels32[0]["dYs"], "dYs, scaled")


def test_bf16_outputs_refuse_fp32_inputs(lard):
    w = synth.custom(1, 1, 64, 64, "fp32", seed=1, relations=("Q",))
    xt, xs = (t.cuda() for t in synth.make_relation(w, "Q"))
    base, _ = lard.relations_kl([(xt, xs)], w.tau, True, backward=False)
    rel = [dict(Xt=xt, Xs=xs, lse_t=base[0]["lse_t"], lse_s=base[0]["lse_s"],
                dXs=torch.empty(xt.shape, device="cuda", dtype=torch.bfloat16), dYs=None)]
    ws = torch.empty((lard.lard_kl_bwd_bf16_workspace_bytes(rel),), device="cuda", dtype=torch.uint8)
    with pytest.raises(lard.LardError) as e:
        lard.lard_kl_bwd_multi_bf16(rel, w.tau, True, 1.0, ws)
    assert e.value.status == lard.LARD_ERR_UNSUPPORTED


def test_bf16_outputs_grouped_noncausal_and_head_dim_64(lard):
    """No mask with a ragged tail (n = 2000, 16 row blocks), d = 64, three relations
    with their own head counts, fused and not, in one launch per phase: one
    whole head per relation against the oracle."""
    for causal, d in ((False, 128), (True, 64), (False, 64)):
        pairs, tau = _pairs((("Q", 3), ("K", 1), ("V", 2)), 1, 2000, d, seed=90 + d, causal=causal)
        for fused in (False, True):
            outs, _ = lard.relations_kl(pairs, tau, causal, fused_self=fused, grad_dtype="bf16")
            torch.cuda.synchronize()
            lard.lard_device_status()
            for k, ((xt, xs), g) in enumerate(zip(pairs, outs)):
                h = xt.shape[1] - 1
                X_t, X_s = f64(xt[0, h]), f64(xs[0, h])
                o = oracle.relation(X_t, X_t, X_s, X_s, tau, causal)
                floor = grad_floor(X_s, X_s, tau, 1.0, 2000)
                what = f"grouped bf16 causal={causal} d={d} fused={fused} relation {k}"
                if fused:
                    assert_grad_close(f64(g["dXs"][0, h]), o["dXs"] + o["dYs"], TOL["bf16"]["grad"], what + " dQ", floor)
                else:
                    assert_grad_close(f64(g["dXs"][0, h]), o["dXs"], TOL["bf16"]["grad"], what + " dXs", floor)
                    assert_grad_close(f64(g["dYs"][0, h]), o["dYs"], TOL["bf16"]["grad"], what + " dYs", floor)


def test_bf16_outputs_cross_relation(lard):
    """X != Y for teacher and student (a Q K^T map): bf16 dX_s and dY_s from the
    grouped call, against the oracle, with a ragged n and both masks."""
    import math
    from parity_util import random_cross
    for causal in (True, False):
        Xt, Yt, Xs, Ys = (t.cuda() for t in random_cross(1, 2, 333, 128, "bf16", seed=77, scale=1.2))
        tau = 1.0 / math.sqrt(128)
        f32 = dict(device="cuda", dtype=torch.float32)
        rel = dict(Xt=Xt, Yt=Yt, Xs=Xs, Ys=Ys, lse_t=torch.empty((1, 2, 333), **f32),
                   lse_s=torch.empty((1, 2, 333), **f32), row_kl=torch.empty((1, 2, 333), **f32))
        lard.lard_kl_fwd_multi([rel], tau, causal)
        out = dict(rel, dXs=torch.empty(Xs.shape, device="cuda", dtype=torch.bfloat16),
                   dYs=torch.empty(Xs.shape, device="cuda", dtype=torch.bfloat16))
        out.pop("row_kl")
        ws = torch.empty((lard.lard_kl_bwd_bf16_workspace_bytes([out]),), device="cuda", dtype=torch.uint8)
        lard.lard_kl_bwd_multi_bf16([out], tau, causal, 1.0, ws)
        torch.cuda.synchronize()
        lard.lard_device_status()
        for h in range(2):
            o = oracle.relation(f64(Xt[0, h]), f64(Yt[0, h]), f64(Xs[0, h]), f64(Ys[0, h]), tau, causal)
            floor = grad_floor(f64(Xs[0, h]), f64(Ys[0, h]), tau, 1.0, 333)
            what = f"cross bf16 causal={causal} head {h}"
            assert_grad_close(f64(out["dXs"][0, h]), o["dXs"], TOL["bf16"]["grad"], what + " dXs", floor)
            assert_grad_close(f64(out["dYs"][0, h]), o["dYs"], TOL["bf16"]["grad"], what + " dYs", floor)
        # a cross relation has no fused form
        bad = dict(out, dYs=None)
        with pytest.raises(lard.LardError):
            lard.lard_kl_bwd_multi_bf16([bad], tau, causal, 1.0, ws)
