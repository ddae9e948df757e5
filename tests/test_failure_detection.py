"""Failure detection without a GPU fault: a kernel wait that runs out sets the
device fault word, the host reads LARD_ERR_TIMEOUT, and the context keeps
working.  The wait is made to run out on purpose (an mbarrier nothing arrives
at, with a 50 ms limit); no kernel traps, faults or hangs."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lard():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from linear_memory_attention_b200 import lard as L
    return L


def test_timed_out_wait_is_reported_and_context_survives(lard):
    assert lard.lard_device_status() == 0  # clean before
    lard.lard_selftest_timeout(50_000)
    with pytest.raises(lard.LardError) as ei:
        lard.lard_device_status()
    assert ei.value.status == lard.LARD_ERR_TIMEOUT
    assert ei.value.fault_bits & 0x8000       # the wait inside the loop
    assert ei.value.fault_bits & 0x100        # the block's exit wait
    assert lard.lard_device_status() == 0  # the word was cleared
    # the context still runs real work correctly
    from linear_memory_attention_b200 import synth
    w = synth.custom(1, 1, 200, 128, "bf16", seed=2)
    Xt, Xs = (t.cuda() for t in synth.make_relation(w, "Q"))
    out = lard.relation_kl(Xt, Xs, w.tau)
    torch.cuda.synchronize()
    assert torch.isfinite(out["loss"]).all() and torch.isfinite(out["dXs"]).all()
    assert lard.lard_device_status() == 0


def test_selftest_rejects_bad_limits(lard):
    for bad in (0, 10_000_000):
        with pytest.raises(lard.LardError):
            lard.lard_selftest_timeout(bad)
