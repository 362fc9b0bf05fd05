"""Failure reporting on the GPU without a fault: a kernel whose bounded device-side wait runs
out stops waiting, and the host reads the event from the cache's status word.

kvq_selftest_wait_timeout makes one warp wait, with the same bounded wait the pipelined
decode and prefill kernels use, on a barrier that nothing ever arrives on (no copies or
tensor memory are held); the wait gives up after the given limit. The test checks that the
status is reported once (and cleared), and that the context stays usable: a decode after it
still matches the oracle."""
import numpy as np
import pytest

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
from harness import append_both, decode_both, make_pair

pytestmark = pytest.mark.gpu


def test_timed_out_wait_is_reported_and_context_survives():
    import torch
    from quantized_mixed_precision_qx_b200 import kvq
    wl = Workload(1, 1, 2, 12, 256, 600, KVRecipe("outlier"), seed=90)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, 128)
    vmax = append_both(g, o, wl, 0, 0, 600)
    assert kvq.kvq_device_status(g.handle) == kvq.OK
    decode_both(g, o, wl, 0, 0, vmax, what="before")
    assert kvq.kvq_device_status(g.handle) == kvq.OK        # a healthy decode records nothing
    kvq.kvq_selftest_wait_timeout(g.handle, 2_000_000)      # gives up after 2 ms
    assert kvq.kvq_device_status(g.handle) == kvq.ERR_DEVICE_TIMEOUT
    assert kvq.kvq_device_status(g.handle) == kvq.OK        # reading clears it
    decode_both(g, o, wl, 0, 1, vmax, what="after")
    torch.cuda.synchronize()
    assert kvq.kvq_device_status(g.handle) == kvq.OK
