"""The entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they run Phase 2 -- code inside
another framework's step whose memory pool owns the device, or a runtime
that forbids allocation once started -- so they cannot hand
lard_kl_bwd_multi_bf16 its fp32 workspace.  lard_kl_bwd_multi_bf16_noalloc
uses a fixed array inside the library instead.  These tests call it through
the C ABI and check that it gives what lard_kl_bwd_multi_bf16 gives with a
caller-allocated workspace, on two calls in a row (the array keeps the
previous call's contents, so the second call checks that it is cleared),
and that a problem larger than the array is refused.  This file is
collected last, so that a run stopping at its first failure has run every
other test first; it also passes alone in a fresh process.
"""
import ctypes

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


def _relations(lard, spec, n, d, seed, causal=True):
    rels = []
    for k, (rel, H, fused) in enumerate(spec):
        w = synth.custom(1, H, n, d, "bf16", seed=seed + k, relations=(rel,), causal=causal)
        xt, xs = (t.cuda() for t in synth.make_relation(w, rel))
        f32 = dict(device="cuda", dtype=torch.float32)
        rels.append(dict(Xt=xt, Xs=xs, lse_t=torch.empty((1, H, n), **f32), lse_s=torch.empty((1, H, n), **f32),
                         row_kl=torch.empty((1, H, n), **f32), loss_bh=torch.empty((H,), **f32), fused=fused))
    tau = w.tau
    lard.lard_kl_fwd_multi([{k: v for k, v in r.items() if k != "fused"} for r in rels], tau, causal)
    return rels, tau


def _grads(rels):
    out = []
    for r in rels:
        g = dict(r)
        g.pop("fused")
        g.pop("row_kl")
        g.pop("loss_bh")
        g["dXs"] = torch.empty(r["Xt"].shape, device="cuda", dtype=torch.bfloat16)
        g["dYs"] = None if r["fused"] else torch.empty(r["Xt"].shape, device="cuda", dtype=torch.bfloat16)
        out.append(g)
    return out


def _close(got, want, what):
    """Within one bf16 unit in the last place of each other: the fp32 sums behind
    both are the same up to the order of the dX reduce-adds, and a sum that
    lands near a rounding midpoint may round to either neighbour (one ulp is at
    most 2^-7 of the value)."""
    g, w = got.double(), want.double()
    bound = 2.0 ** -7 * w.abs() + 1e-6 * w.abs().max().item() + 1e-30
    err = (g - w).abs()
    assert bool((err <= bound).all()), f"{what}: max err {err.max().item():.3e}"


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
def test_noalloc_matches_the_workspace_entry_point(lard, causal):
    rels, tau = _relations(lard, (("Q", 3, False), ("K", 2, True)), 1000, 128, seed=31, causal=causal)
    ref = _grads(rels)
    ws = torch.empty((lard.lard_kl_bwd_bf16_workspace_bytes(ref),), device="cuda", dtype=torch.uint8)
    lard.lard_kl_bwd_multi_bf16(ref, tau, causal, 0.75, ws)
    for call in range(2):  # the second call finds the first call's sums in the array
        got = _grads(rels)
        lard.lard_kl_bwd_multi_bf16_noalloc(got, tau, causal, 0.75)
        torch.cuda.synchronize()
        lard.lard_device_status()
        for k, (a, b) in enumerate(zip(got, ref)):
            _close(a["dXs"], b["dXs"], f"call {call} relation {k} dXs")
            if b["dYs"] is not None:
                _close(a["dYs"], b["dYs"], f"call {call} relation {k} dYs")


def test_noalloc_through_the_c_abi_allocates_nothing(lard):
    """A direct C call: no device memory is taken, and the result equals the
    binding's."""
    rels, tau = _relations(lard, (("V", 2, False),), 700, 64, seed=5)
    want = _grads(rels)
    lard.lard_kl_bwd_multi_bf16_noalloc(want, tau, True, 1.0)
    torch.cuda.synchronize()
    got = _grads(rels)
    arr = (lard._Relation * 1)()
    r = got[0]
    arr[0].Xt = arr[0].Yt = r["Xt"].data_ptr()
    arr[0].Xs = arr[0].Ys = r["Xs"].data_ptr()
    arr[0].H = 2
    arr[0].lse_t, arr[0].lse_s = r["lse_t"].data_ptr(), r["lse_s"].data_ptr()
    out = (lard._Bf16Grads * 1)()
    out[0].dXs, out[0].dYs = r["dXs"].data_ptr(), r["dYs"].data_ptr()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    st = lard._lib.lard_kl_bwd_multi_bf16_noalloc(arr, out, 1, lard.LARD_DTYPE_BF16, 1, 700, 64,
                                                  ctypes.c_float(tau), 1, ctypes.c_float(1.0),
                                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == lard.LARD_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    lard.lard_device_status()
    _close(got[0]["dXs"], want[0]["dXs"], "dXs")
    _close(got[0]["dYs"], want[0]["dYs"], "dYs")


def test_noalloc_refuses_a_problem_larger_than_its_array(lard):
    # 33 heads of n = 4096, d = 128 need 66 MiB of fp32 accumulators
    rels, tau = _relations(lard, (("Q", 33, True),), 4096, 128, seed=2)
    assert lard.lard_kl_bwd_bf16_workspace_bytes(_grads(rels)) > lard.LARD_NOALLOC_WORKSPACE_BYTES
    with pytest.raises(lard.LardError) as e:
        lard.lard_kl_bwd_multi_bf16_noalloc(_grads(rels), tau, True, 1.0)
    assert e.value.status == lard.LARD_ERR_TOO_LARGE
