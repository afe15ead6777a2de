"""Failure detection on the GPU without a fault.

Every mbarrier wait in the kernels is bounded: past its limit it records status 1 in a device
word, sets the CTA's abort flag and returns, so the kernel ends normally and the host reads the
status with sage_last_device_error().  Here a wait is made to run out (an mbarrier that nothing
arrives on), through the same wait helper the pipelines use, and the test checks the status,
that reading it clears it, and that the context still computes a correct forward pass.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_without_losing_the_context():
    import quantized_attention_02_b200 as sa

    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0  # start clean
    gave_up = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    sa.sage_debug_wait_timeout(gave_up)
    torch.cuda.synchronize()
    assert int(gave_up.item()) == 0           # the wait gave up rather than completing
    assert sa.sage_last_device_error() == 1   # kDevTimeoutBarrier, read by the host
    assert sa.sage_last_device_error() == 0   # reading clears it

    # the context is intact: the whole forward pass still matches the oracle
    w = W.Workload("after_timeout", 1, 2, 256, 128, True, True, n_out=4, out_mag=20.0)
    q, k, v = W.make_qkv(w)
    o = sa.sageattn(q.cuda(), k.cuda(), v.cuda(), w.causal, w.sm_scale, sa.SAGE_PER_BLOCK)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    ref = oracle.sage_attn(q, k, v, w.causal, w.sm_scale, per_block=True)
    og = o.float().cpu().numpy().astype(np.float64)
    assert np.abs(og - ref["o64"]).max() <= 2e-3 * float(v.abs().max())
