"""sage_attn_fwd_noalloc: the forward pass for callers that cannot allocate device memory.

Some callers cannot let a library allocate while they run: a host whose device-memory
budget is fixed at start-up, or a framework plugin whose host owns every device allocation
and does not let the library call the CUDA allocator.  sage_attn_fwd gets its workspace with a
stream-ordered allocation, so it is not usable there; sage_attn_fwd_noalloc runs the same kernels on
a fixed scratch array compiled into the library.

This file is collected last on purpose: it must pass on its own in a fresh process (where
its first call also does the per-device set-up) and after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

ATOL_FRAC = 2e-3
COS_MIN = 0.9999


def _close(a: np.ndarray, b: np.ndarray, vmax: float):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    err = float(np.abs(a - b).max())
    cos = float(np.dot(a, b) / (np.linalg.norm(a) * np.linalg.norm(b)))
    assert err <= ATOL_FRAC * vmax, err
    assert cos >= COS_MIN, cos


def test_noalloc_matches_sage_attn_fwd_on_two_calls_in_a_row():
    import quantized_attention_02_b200 as sa

    lib = sa.get_lib()
    cases = [
        W.Workload("noalloc_a", 1, 4, 1024, 128, True, True, n_out=8, out_mag=30.0),
        W.Workload("noalloc_b", 2, 3, 512, 64, False, False, n_out=4, out_mag=20.0),
        W.Workload("noalloc_c_ragged", 1, 2, 777, 128, True, False, n_out=4, out_mag=20.0),
    ]
    stream = torch.cuda.current_stream()
    for w in cases:
        gran = sa.SAGE_PER_BLOCK if w.per_block else sa.SAGE_PER_TOKEN
        assert sa.sage_noalloc_scratch_bytes(w.B, w.H, w.N, w.d, gran) <= 64 << 20
        # two calls in a row on different inputs: the second one finds the first one's
        # codes and scales in the shared scratch array and must not depend on them
        for seed in (0, 1):
            q, k, v = (t.cuda() for t in W.make_qkv(w, seed=seed))
            o_ref = torch.empty_like(q)
            sa.sage_attn_fwd(q, k, v, o_ref, w.causal, w.sm_scale, gran, stream)
            o = torch.empty_like(q)
            rc = lib.sage_attn_fwd_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                           ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                           w.B, w.H, w.N, w.d, int(w.causal), float(w.sm_scale), gran,
                                           ctypes.c_void_p(stream.cuda_stream))
            assert rc == sa.SAGE_OK, sa.sage_status_string(rc)
            torch.cuda.synchronize()
            assert sa.sage_last_device_error() == 0
            # the same kernels on the same inputs: bit-identical to sage_attn_fwd
            assert torch.equal(o, o_ref), w.name
            if w.name == "noalloc_b" and seed == 1:
                # and within the method's bar of the oracle (the second call, on a scratch
                # array that still holds the first call's codes and scales)
                import oracle
                ref = oracle.sage_attn(q.cpu(), k.cpu(), v.cpu(), w.causal, w.sm_scale, per_block=w.per_block)
                _close(o.float().cpu().numpy(), ref["o64"], float(v.abs().max()))


def test_noalloc_rejects_problems_beyond_the_scratch():
    import quantized_attention_02_b200 as sa

    lib = sa.get_lib()
    fake = ctypes.c_void_p(0x1000)  # never touched: the size check comes first
    B, H, N, d = 1, 64, 16384, 128  # 256 MiB of INT8 Q/K alone
    assert sa.sage_noalloc_scratch_bytes(B, H, N, d, sa.SAGE_PER_BLOCK) > 64 << 20
    rc = lib.sage_attn_fwd_noalloc(fake, fake, fake, fake, B, H, N, d, 0, 0.1, sa.SAGE_PER_BLOCK,
                                   ctypes.c_void_p(0))
    assert rc == sa.SAGE_ERR_TOO_LARGE
    assert "scratch" in sa.sage_status_string(rc)
