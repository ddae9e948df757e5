"""Out-of-bounds write check (a stand-in for a memory sanitizer): every output
of every entry point is placed inside a larger device buffer whose guard
regions before and after it hold a marker value; after the calls, the guards
must be untouched.  The ragged sizes put the last row block's TMA stores and
reduce-adds right at the end of each buffer, where an off-by-one row or box
would write past it."""
import pytest
import torch

from linear_memory_attention_b200 import synth

pytestmark = pytest.mark.gpu

CANARY = -7.25e30       # a value no output can take
GUARD = 16384           # guard elements (64 KB) on each side; keeps 16-byte alignment


@pytest.fixture(scope="module")
def lard():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_memory_attention_b200 import lard as L
    return L


class Guarded:
    """Output views carved out of guarded device buffers."""

    def __init__(self):
        self.bufs = []

    def __call__(self, *shape, dtype=torch.float32):
        numel = 1
        for s in shape:
            numel *= s
        # guards of GUARD fp32 words (64 KB) whatever the element type
        g = GUARD * 4 // torch.tensor([], dtype=dtype).element_size()
        buf = torch.full((g + numel + g,), CANARY if dtype == torch.float32 else -3.0e38,
                         device="cuda", dtype=dtype)
        self.bufs.append((buf, numel, g, buf[0].item()))
        return buf[g:g + numel].view(*shape)

    def check(self, what):
        torch.cuda.synchronize()
        for k, (buf, numel, g, mark) in enumerate(self.bufs):
            head, tail = buf[:g], buf[g + numel:]
            assert bool((head == mark).all()), f"{what}: buffer {k} written before its start"
            assert bool((tail == mark).all()), f"{what}: buffer {k} written past its end"


def _inputs(B, H, n, d, dtype, seed, rel="Q"):
    w = synth.custom(B, H, n, d, dtype, seed=seed, relations=(rel,))
    Xt, Xs = synth.make_relation(w, rel)
    return Xt.cuda(), Xs.cuda(), w.tau


CASES = [(1, 1, 1, 128), (1, 2, 127, 128), (2, 1, 129, 64), (1, 1, 8000, 128), (1, 2, 8000, 64)]


@pytest.mark.parametrize("causal", [1, 0], ids=["causal", "full"])
@pytest.mark.parametrize("shape", CASES, ids=lambda s: "B%dH%dn%dd%d" % s)
def test_single_relation_calls_stay_in_bounds(lard, shape, causal):
    B, H, n, d = shape
    xt, xs, tau = _inputs(B, H, n, d, "bf16", seed=n + d)
    G = Guarded()
    lse_t, lse_s, kl = G(B, H, n), G(B, H, n), G(B, H, n)
    loss_bh, loss = G(B * H), G(1)
    dX, dY, dQ = G(B, H, n, d), G(B, H, n, d), G(B, H, n, d)
    lard.lard_kl_fwd(xt, xt, xs, xs, tau, causal, lse_t, lse_s, kl, loss_bh, loss)
    lard.lard_kl_bwd(xt, xt, xs, xs, tau, causal, lse_t, lse_s, 1.0, dX, dY)
    lard.lard_kl_bwd_self(xt, xs, tau, causal, lse_t, lse_s, 1.0, dQ)
    lard.lard_device_status()
    G.check(f"single-relation calls {shape} causal={causal}")
    torch.testing.assert_close(dQ, dX + dY, rtol=1e-5, atol=1e-6 * (dX + dY).abs().max().item() + 1e-30)


@pytest.mark.parametrize("causal", [1, 0], ids=["causal", "full"])
@pytest.mark.parametrize("n,d", [(1, 128), (129, 128), (8000, 64), (8000, 128)])
def test_grouped_calls_stay_in_bounds(lard, n, d, causal):
    """Three relations with their own head counts, one of them fused, in one
    launch per phase."""
    G = Guarded()
    rels = []
    for k, (rel, H, fused) in enumerate((("Q", 3, False), ("K", 1, True), ("V", 2, False))):
        xt, xs, tau = _inputs(2, H, n, d, "bf16", seed=10 * k + n, rel=rel)
        r = dict(Xt=xt, Xs=xs, lse_t=G(2, H, n), lse_s=G(2, H, n), row_kl=G(2, H, n), loss_bh=G(2 * H),
                 dXs=G(2, H, n, d))
        if not fused:
            r["dYs"] = G(2, H, n, d)
        rels.append(r)
    loss = G(1)
    lard.lard_kl_fwd_multi(rels, tau, causal, loss)
    lard.lard_kl_bwd_multi(rels, tau, causal, 0.5)
    lard.lard_device_status()
    G.check(f"grouped calls n={n} d={d} causal={causal}")


@pytest.mark.parametrize("n,d", [(1, 32), (127, 64), (129, 96)])
def test_fp32_path_stays_in_bounds(lard, n, d):
    """The fp32 path parks per-row corrections in the dX rows while it builds
    dY; nothing may land outside them."""
    xt, xs, tau = _inputs(2, 2, n, d, "fp32", seed=n)
    G = Guarded()
    lse_t, lse_s, kl, loss_bh, loss = G(2, 2, n), G(2, 2, n), G(2, 2, n), G(4), G(1)
    dX, dY = G(2, 2, n, d), G(2, 2, n, d)
    lard.lard_kl_fwd(xt, xt, xs, xs, tau, True, lse_t, lse_s, kl, loss_bh, loss)
    lard.lard_kl_bwd(xt, xt, xs, xs, tau, True, lse_t, lse_s, 1.0, dX, dY)
    lard.lard_device_status()
    G.check(f"fp32 path n={n} d={d}")


@pytest.mark.parametrize("n,d", [(1, 128), (129, 64), (8000, 128)])
def test_bf16_gradient_outputs_stay_in_bounds(lard, n, d):
    """bf16 gradients and the fp32 workspace (sized exactly) inside guards."""
    G = Guarded()
    rels = []
    for k, (rel, H, fused) in enumerate((("Q", 2, False), ("V", 1, True))):
        xt, xs, tau = _inputs(1, H, n, d, "bf16", seed=7 * k + n, rel=rel)
        r = dict(Xt=xt, Xs=xs, lse_t=G(1, H, n), lse_s=G(1, H, n), row_kl=G(1, H, n), loss_bh=G(H),
                 dXs=G(1, H, n, d, dtype=torch.bfloat16))
        r["dYs"] = None if fused else G(1, H, n, d, dtype=torch.bfloat16)
        rels.append(r)
    lard.lard_kl_fwd_multi(rels, tau, True, G(1))
    need = lard.lard_kl_bwd_bf16_workspace_bytes(rels)
    ws = G(need // 4)
    lard.lard_kl_bwd_multi_bf16(rels, tau, True, 1.0, ws)
    lard.lard_device_status()
    G.check(f"bf16 outputs n={n} d={d}")
