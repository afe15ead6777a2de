"""More than 65535 heads (B*H = 70000): every kernel puts heads on grid x, so no launch
hits the 65535 limit of grid y/z.  The K mean, codes and scales stay bit-exact against the
oracle; O matches it on sampled heads; the INT32 debug product on sampled heads."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

HEADS = 70000


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    return sa


@pytest.mark.parametrize("gran", [1, 0])
def test_70000_heads_prep_and_attention(sa, gran):
    w = W.Workload("many_heads_n16_d64", 1, HEADS, 16, 64, False, gran == 1, n_out=4, out_mag=20.0)
    q, k, v = W.make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    km, q8, k8, sq, sk = sa.empty_quantized(qd, gran)
    sa.sage_smooth_k(kd, km)
    sa.sage_quant_qk(qd, kd, km, q8, k8, sq, sk, gran)
    o = torch.empty_like(qd)
    sa.sage_attn_fwd(qd, kd, vd, o, w.causal, w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    ref = oracle.sage_attn(q, k, v, w.causal, w.sm_scale, per_block=gran == 1)
    for name, got in (("km", km), ("q8", q8), ("sq", sq), ("k8", k8), ("sk", sk)):
        np.testing.assert_array_equal(got.cpu().numpy(), ref[name], err_msg=name)
    heads = [0, 1, 65534, 65535, 65536, HEADS - 1]
    og = o.view(HEADS, w.N, w.d)[heads].float().cpu().numpy()
    o64 = ref["o64"].reshape(HEADS, w.N, w.d)[heads]
    vmax = float(v.abs().max())
    assert np.abs(og - o64).max() <= 2e-3 * vmax


def test_70000_heads_int32_debug_product(sa):
    BH, N, d = HEADS, 128, 64
    g = torch.Generator().manual_seed(3)
    q8 = torch.randint(-127, 128, (1, BH, N, d), generator=g, dtype=torch.int8)
    k8 = torch.randint(-127, 128, (1, BH, N, d), generator=g, dtype=torch.int8)
    s = torch.empty((1, BH, N, N), dtype=torch.int32, device="cuda")
    sa.sage_debug_qk_int32(q8.cuda(), k8.cuda(), s)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    heads = [0, 65535, 65536, BH - 1]
    got = s[0, heads].cpu().numpy().astype(np.int64)
    want = oracle.qk_int(q8[0, heads].numpy(), k8[0, heads].numpy())
    np.testing.assert_array_equal(got, want)
