"""The library on several streams and threads at once, and its refusal of
buffers that are not device memory (checked on the host before any launch)."""
import threading

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


def _inputs(seed, n=700, H=3):
    w = synth.custom(1, H, n, 128, "bf16", seed=seed)
    Xt, Xs = synth.make_relation(w, "Q")
    return Xt.cuda(), Xs.cuda(), w.tau


def test_two_streams_two_threads(lard):
    """Two host threads, each with its own stream, run both phases concurrently;
    each result equals the same call made alone (statistics and dY bit for bit)."""
    cases = [_inputs(91), _inputs(92)]
    alone = []
    for xt, xs, tau in cases:
        alone.append(lard.relation_kl(xt, xs, tau, True))
    torch.cuda.synchronize()
    results = [None, None]
    errors = []

    def run(k):
        try:
            s = torch.cuda.Stream()
            xt, xs, tau = cases[k]
            with torch.cuda.stream(s):
                out = None
                for _ in range(3):
                    out = lard.relation_kl(xt, xs, tau, True, stream=s)
            s.synchronize()
            results[k] = out
        except Exception as e:  # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(k,)) for k in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    lard.lard_device_status()
    for got, want in zip(results, alone):
        for key in ("lse_t", "lse_s", "row_kl", "loss_bh", "dYs"):
            assert torch.equal(got[key], want[key]), key
        torch.testing.assert_close(got["dXs"], want["dXs"], rtol=1e-5,
                                   atol=1e-6 * want["dXs"].abs().max().item())


def test_host_buffers_are_refused(lard):
    """Host memory in place of a device buffer is refused before any launch: by
    the binding's checks (ValueError), and by the C library itself when called
    directly with the raw pointers (LARD_ERR_INVALID_ARG)."""
    import ctypes
    xt, xs, tau = _inputs(93, n=256, H=1)
    f32 = dict(dtype=torch.float32)
    dev = dict(device=xt.device, **f32)
    lse_t, lse_s = torch.empty((1, 1, 256), **dev), torch.empty((1, 1, 256), **dev)
    host_kl = torch.empty((1, 1, 256), **f32).pin_memory()
    with pytest.raises(ValueError):
        lard.lard_kl_fwd(xt, xt, xs, xs, tau, True, lse_t, lse_s, host_kl)
    with pytest.raises(ValueError):
        lard.lard_kl_fwd(xt.cpu(), xt.cpu(), xs.cpu(), xs.cpu(), tau, True, lse_t, lse_s,
                         torch.empty((1, 1, 256), **dev))
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    f = ctypes.c_float(tau)
    st = lard._lib.lard_kl_fwd(p(xt), p(xt), p(xs), p(xs), 0, 1, 1, 256, 128, f, 1, p(lse_t), p(lse_s),
                               p(host_kl), None, None, s)
    assert st == lard.LARD_ERR_INVALID_ARG
    xh, sh = xt.cpu().pin_memory(), xs.cpu().pin_memory()
    kl = torch.empty((1, 1, 256), **dev)
    st = lard._lib.lard_kl_fwd(p(xh), p(xh), p(sh), p(sh), 0, 1, 1, 256, 128, f, 1, p(lse_t), p(lse_s),
                               p(kl), None, None, s)
    assert st == lard.LARD_ERR_INVALID_ARG
    lard.lard_kl_fwd(xt, xt, xs, xs, tau, True, lse_t, lse_s, kl)
    host_dx = torch.empty((1, 1, 256, 128), **f32).pin_memory()
    with pytest.raises(ValueError):
        lard.lard_kl_bwd_self(xt, xs, tau, True, lse_t, lse_s, 1.0, host_dx)
    st = lard._lib.lard_kl_bwd_self(p(xt), p(xs), 0, 1, 1, 256, 128, f, 1, p(lse_t), p(lse_s),
                                    ctypes.c_float(1.0), p(host_dx), s)
    assert st == lard.LARD_ERR_INVALID_ARG
    torch.cuda.synchronize()
    lard.lard_device_status()
