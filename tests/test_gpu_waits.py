"""The bounded waits give up, report and leave the device usable.

Every wait in libq8's kernels (the shared-memory ring's mbarrier waits, the
fused layer kernel's grid barrier) is bounded: after its limit it latches a
wait-timeout flag, which q8_check reports as Q8_E_CUDA, and returns instead of
spinning.  The test hook q8_debug_wait_timeout runs one such wait that nothing
can satisfy (an mbarrier phase nothing completes; a grid barrier one arrival
short) with a limit of a few milliseconds; q8_check must then report the
timeout, q8_reset_errors must clear it, and the device must still run a
kernel correctly afterwards.  No fault, trap or endless wait is involved.
"""
import pytest
import torch

from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gemv_still_works():
    w = synth.normal((64, 128), seed=4242, std=0.02).to(DEV)
    W = q8.pack(w)
    xq, xd = q8.quantize_row(synth.normal((1, 128), seed=4243).to(DEV))
    y1 = q8.gemv(W, xq, xd)
    y2 = q8.gemv(W, xq, xd)
    q8.check(None)
    assert torch.equal(y1, y2) and not torch.isnan(y1).any()


@pytest.mark.parametrize("kind", [0, 1])
def test_wait_runs_out_reports_and_resets(kind):
    q8.reset_errors()
    q8.check(None)  # clean to start with
    bar = torch.zeros(2, dtype=torch.int32, device=DEV) if kind == 1 else None
    q8.debug_wait_timeout(kind, 5_000_000, bar)  # 5 ms
    with pytest.raises(q8.Q8Error) as e:
        q8.check(None)
    assert e.value.name == "Q8_E_CUDA" and b"gave up" in q8.load().q8_last_error()
    if kind == 1:
        assert int(bar[0]) == 2  # both CTAs arrived; the one missing arrival never came
    q8.reset_errors()
    q8.check(None)
    _gemv_still_works()

