"""The error path of the tensor-core kernels' bounded waits, on the GPU: a
kernel whose wait can never be satisfied gives up after about a second, the
host reads the device error word, and the context stays usable.  Nothing here
faults or hangs the GPU."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_context_survives():
    import lut_clustered_weight_b200 as cq
    assert cq.cq_device_error() == 0
    t0 = time.perf_counter()
    cq.cq_selftest_wait_timeout()
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert 0.5 < dt < 30.0                 # the wait ran out (about 1 s), then returned
    assert cq.cq_device_error() == 1       # recorded ...
    assert cq.cq_device_error() == 0       # ... and cleared by the read
    # the context is still usable
    x = synth.activations(3, 256, seed=5, name="after_timeout", n_outliers=2)
    q, s = cq.cq_rotate_quantize(torch.from_numpy(x).cuda(), 64, 4)
    torch.cuda.synchronize()
    qr, sr = oracle.rotate_quantize(x, 64, 4)
    assert np.array_equal(oracle.unpack_codes(q.cpu().numpy(), 256, 4), qr)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32))
