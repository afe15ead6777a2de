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


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 200, 1000, 4095, 6001, 12289, 16384, 20000])
@pytest.mark.parametrize("gran", [0, 1])
def test_one_launch_prep_equals_the_two_steps_and_the_oracle(sa, N, d, gran):
    """sage_prep_qk (K mean, K codes, Q codes in one launch, one cluster per head) gives the bits
    of sage_smooth_k + sage_quant_qk, and those of the oracle, at every cluster size, both
    granularities and ragged lengths (slices of whole 128-token blocks, a short last one)."""
    w = W.Workload(f"prep1_n{N}_d{d}", 1, 3, N, d, False, gran == 1, n_out=4, out_mag=20.0)
    q, k, _ = W.make_qkv(w, seed=N + 1)
    qd, kd = q.cuda(), k.cuda()
    a = sa.empty_quantized(qd, gran)
    b = sa.empty_quantized(qd, gran)
    for t in b:
        t.fill_(7)  # stale values the one-launch kernel must overwrite
    sa.sage_smooth_k(kd, a[0])
    sa.sage_quant_qk(qd, kd, a[0], *a[1:], gran)
    sa.sage_prep_qk(qd, kd, *b, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    for name, x, y in zip(("km", "q8", "k8", "sq", "sk"), a, b):
        assert torch.equal(x, y), name
    gq, gk = oracle.GROUP_PER_BLOCK if gran == 1 else oracle.GROUP_PER_TOKEN
    km_ref = oracle.smooth_k(k)
    np.testing.assert_array_equal(b[0].cpu().numpy(), km_ref)
    np.testing.assert_array_equal(b[2].cpu().numpy(), oracle.quant(k, gk, km_ref)[0])
    np.testing.assert_array_equal(b[1].cpu().numpy(), oracle.quant(q, gq)[0])
