"""GPU parity of the two HBM-bound steps in front of the fused kernel, at the sizes that select
each launch shape of the K-mean kernel.

The K mean runs as one thread-block cluster of 1, 2, 4 or 8 CTAs per head (the largest power of
two <= 8 that leaves every CTA at least 2048 tokens), each CTA summing a contiguous slice of the
head's tokens; sequence lengths that are not a multiple of the cluster size leave a short last
slice.  The K mean, the INT8 codes and the scales must equal the oracle's bit for bit, for both
granularities and both head dimensions.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

# (N, CTAs per head): 1 (N < 4096), 2 (4096 <= N < 8192), 4 (8192 <= N < 16384), 8 (N >= 16384)
LENGTHS = [1000, 4095, 4096, 6001, 8192, 12289, 16384, 20000, 32768]


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    assert torch.cuda.is_available()
    return sa


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", LENGTHS)
def test_prep_bit_exact_across_cluster_sizes(sa, N, d):
    per_block = N % 2 == 0  # both granularities across the lengths
    w = W.Workload(f"prep_n{N}_d{d}", 1, 2, N, d, False, per_block, n_out=4, out_mag=20.0)
    q, k, _ = W.make_qkv(w, seed=N)
    gran = sa.SAGE_PER_BLOCK if per_block else sa.SAGE_PER_TOKEN
    qd, kd = q.cuda(), k.cuda()
    km, q8, k8, sq, sk = sa.empty_quantized(qd, gran)
    sa.sage_smooth_k(kd, km)
    sa.sage_quant_qk(qd, kd, km, q8, k8, sq, sk, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0

    gq, gk = oracle.GROUP_PER_BLOCK if per_block else oracle.GROUP_PER_TOKEN
    km_ref = oracle.smooth_k(k)
    q8_ref, sq_ref = oracle.quant(q, gq)
    k8_ref, sk_ref = oracle.quant(k, gk, km_ref)
    np.testing.assert_array_equal(km.cpu().numpy(), km_ref, err_msg="km")
    np.testing.assert_array_equal(q8.cpu().numpy(), q8_ref, err_msg="q8")
    np.testing.assert_array_equal(sq.cpu().numpy(), sq_ref, err_msg="sq")
    np.testing.assert_array_equal(k8.cpu().numpy(), k8_ref, err_msg="k8")
    np.testing.assert_array_equal(sk.cpu().numpy(), sk_ref, err_msg="sk")


def test_k_mean_of_large_values_is_exact(sa):
    """Channels near the fp16 maximum on every token: the per-thread fp32 partial sums of the
    K-mean kernel reach their largest magnitudes, and the mean must still be exact."""
    B, H, N, d = 1, 1, 16384, 128
    g = torch.Generator().manual_seed(7)
    k = (torch.rand((B, H, N, d), generator=g) * 2 - 1) * 65504.0
    k[..., :8] = 65504.0     # all tokens at the largest finite value
    k[..., 8:16] = -65504.0
    k[..., 16:24] = 2.0 ** -24  # the smallest subnormal
    k = k.to(torch.float16)
    km = torch.empty((B, H, d), dtype=torch.float32, device="cuda")
    sa.sage_smooth_k(k.cuda(), km)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    np.testing.assert_array_equal(km.cpu().numpy(), oracle.smooth_k(k))
