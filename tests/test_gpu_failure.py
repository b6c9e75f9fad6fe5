"""Failure detection on the GPU without a GPU fault: a wait that nothing completes gives up.

Every wait inside the library's kernels (mbarriers for copies, MMAs and warp hand-offs) is bounded by
0.2 s of %globaltimer time; on timeout the kernel sets the per-device error word and returns.  The
self-test entry point launches one thread that waits on a barrier nothing will ever complete (the flag
that nothing sets); the host reads the error word, and the context must still run a correct step.
"""
import time

import pytest
import torch

from pagedattention_block_table_b200.inputs import make_batch
from tests.common import assert_close, oracle_step, to_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable(O, cuda_lib):
    B = cuda_lib
    assert B.pa_get_device_error() == B.PA_OK
    t0 = time.perf_counter()
    B.pa_selftest_bounded_wait()
    assert B.pa_get_device_error() == B.PA_EDEVICE_OOB          # the timeout was reported ...
    waited = time.perf_counter() - t0
    assert 0.15 < waited < 10.0                                   # ... after the bounded wait
    assert B.pa_get_device_error() == B.PA_OK                     # ... and cleared by reading it

    from pagedattention_block_table_b200.runner import DeviceStep
    batch = make_batch("tiny_decode")
    st = DeviceStep(batch)
    st.fill_history()
    st.step()
    torch.cuda.synchronize()
    assert B.pa_get_device_error() == B.PA_OK
    assert_close(to_f64(st.out_dec), oracle_step(batch, O)["decode"], what="decode after the timeout")
