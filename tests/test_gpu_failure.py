"""The band kernel's device-side failure path, exercised without a fault.

Every pipeline wait of the band kernel gives up after a limit, sets the
CTA's abort flag and raises bit 1 of the device status word; the kernel then
drains what it issued and ends.  A test hook shortens the limit and makes
the producers publish nothing, so the other roles wait on barriers that no
one will complete: the waits run out, lf_attn_device_status reports
LF_ERR_DEVICE_CHECK with bit 1, and the next normal call computes the right
answer (the context stays usable).  Nothing traps, faults or hangs.
"""
import pytest
import torch

from sparse_long_sequence_fwd_b200 import build, lf_attn, workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    lf_attn.load()
    yield
    lf_attn.test_hooks(0, 0)


def test_pipeline_waits_run_out_then_the_next_call_is_correct():
    w = workloads.custom("stall", "bf16", 1, 2, 700, 64, 60, dil=[1, 2], globals_per_b=[[3, 650]], seed=60)
    inp = workloads.make_inputs(w)
    lf_attn.device_status()  # clear
    lf_attn.test_hooks(1, 2_000_000)  # producers publish nothing; waits give up after 2 ms
    try:
        parity.run_gpu(w, inp)
        st, flags = lf_attn.device_status()
    finally:
        lf_attn.test_hooks(0, 0)
    assert st == 5 and flags & 2, (st, flags)
    got = parity.run_gpu(w, inp)
    parity.compare(w, got, parity.oracle_full(w, inp))
    st, flags = lf_attn.device_status()
    assert st == 0 and flags == 0, (st, flags)


def test_short_wait_limit_alone_changes_nothing():
    """A 50 ms limit is far above any wait of a healthy pipeline."""
    w = workloads.custom("short_limit", "bf16", 1, 2, 900, 64, 100, globals_per_b=[[0]], seed=61)
    inp = workloads.make_inputs(w)
    lf_attn.device_status()
    lf_attn.test_hooks(0, 50_000_000)
    try:
        got = parity.run_gpu(w, inp)
        st, flags = lf_attn.device_status()
    finally:
        lf_attn.test_hooks(0, 0)
    assert st == 0 and flags == 0
    parity.compare(w, got, parity.oracle_full(w, inp))
