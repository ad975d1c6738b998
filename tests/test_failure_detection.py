"""Device-side failure detection, exercised without faulting or hanging a GPU.

Every wait in the library's kernels (mbarrier phases, TMA and MMA completion)
is bounded by a wall-clock limit.  The self-test kernel waits on a barrier that
nothing completes; the wait must give up, the error flag must read
MEA_ERR_TIMEOUT, be cleared by the read, and the context must stay usable.
"""

import pytest
import torch

from synthetic_inputs import custom, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives():
    import exact_memory_efficient_b200 as m
    assert m.mea_last_device_error() == m.MEA_OK        # clean start
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.mea_selftest_bounded_wait(gave_up)
    assert m.mea_last_device_error() == m.MEA_ERR_TIMEOUT
    assert int(gave_up.item()) == 1
    assert m.mea_last_device_error() == m.MEA_OK        # the read cleared the flag
    # the context still runs the real kernels
    w = custom(1, 1, 130, 140, 64, "bf16", backward=False)
    q, k, v, _ = (x.cuda() if x is not None else None for x in make_inputs(w, 0))
    o, lse = m.attention_forward(q, k, v, w.scale)
    assert m.mea_last_device_error() == m.MEA_OK
    assert torch.isfinite(o.float()).all()
