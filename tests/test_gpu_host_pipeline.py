"""sage_attn_fwd_host(_variant): host tensors in, host tensor out, copies overlapped with the
compute across chunks of heads.  Its output must equal the device entry point of the same
method or variant on the same tensors bit for bit (each head is an independent problem running
the same kernels), for any chunking, pinned or pageable host memory, ragged N and both head
dimensions."""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    assert torch.cuda.is_available()
    return sa


CASES = [
    # workload, heads_per_chunk, pinned
    (W.Workload("host_b1h5_n256_d128_blk", 1, 5, 256, 128, False, True, n_out=4, out_mag=20.0), 2, True),
    (W.Workload("host_b1h5_n256_d128_blk", 1, 5, 256, 128, False, True, n_out=4, out_mag=20.0), 0, True),
    (W.Workload("host_b2h3_n200_d64_causal_tok", 2, 3, 200, 64, True, False, n_out=4, out_mag=20.0), 1, True),
    (W.Workload("host_b2h3_n200_d64_causal_tok", 2, 3, 200, 64, True, False, n_out=4, out_mag=20.0), 64, False),
    (W.Workload("host_b1h4_n1000_d128_causal_blk", 1, 4, 1000, 128, True, True, bias_std=4.0), 3, False),
]


@pytest.mark.parametrize("w,hpc,pinned", CASES, ids=lambda x: str(x) if not hasattr(x, "name") else x.name)
def test_host_pipeline_matches_device_entry(sa, w, hpc, pinned):
    q, k, v = W.make_qkv(w)
    gran = 1 if w.per_block else 0
    ref = torch.empty_like(v.cuda())
    sa.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), ref, w.causal, w.sm_scale, gran)
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o = torch.full_like(q, float("nan"))
    if pinned:
        o = o.pin_memory()
    st = torch.cuda.current_stream()
    sa.sage_attn_fwd_host(q, k, v, o, w.causal, w.sm_scale, gran, heads_per_chunk=hpc, stream=st)
    st.synchronize()
    assert sa.sage_last_device_error(st) == 0
    np.testing.assert_array_equal(o.numpy().view(np.uint16), ref.cpu().numpy().view(np.uint16))


def test_host_pipeline_on_a_side_stream_then_reuse(sa):
    # two calls in a row on a non-default stream reuse the cached copy streams; the second
    # call's output is complete once that stream is synchronized
    w = W.Workload("host_b1h6_n384_d128_full_blk", 1, 6, 384, 128, False, True, n_out=4, out_mag=20.0)
    q, k, v = (t.pin_memory() for t in W.make_qkv(w))
    s = torch.cuda.Stream()
    o1, o2 = torch.empty_like(q).pin_memory(), torch.empty_like(q).pin_memory()
    sa.sage_attn_fwd_host(q, k, v, o1, False, w.sm_scale, 1, heads_per_chunk=2, stream=s)
    sa.sage_attn_fwd_host(q, k, v, o2, False, w.sm_scale, 1, heads_per_chunk=4, stream=s)
    s.synchronize()
    assert sa.sage_last_device_error(s) == 0
    np.testing.assert_array_equal(o1.numpy().view(np.uint16), o2.numpy().view(np.uint16))
    assert np.isfinite(o1.float().numpy()).all()


VARIANT_CASES = [
    # variant, workload, heads_per_chunk
    ("fp4", W.Workload("host_fp4_b1h5_n300_d128", 1, 5, 300, 128, False, True, n_out=4, out_mag=20.0), 2),
    ("fp4", W.Workload("host_fp4_b2h3_n200_d64_causal", 2, 3, 200, 64, True, True, bias_std=4.0), 0),
    ("fp8pv", W.Workload("host_fp8_b1h4_n384_d128_causal", 1, 4, 384, 128, True, True, n_out=4, out_mag=20.0), 3),
]


@pytest.mark.parametrize("variant,w,hpc", VARIANT_CASES, ids=lambda x: x if isinstance(x, str) else str(x))
def test_host_pipeline_variants_match_their_device_entries(sa, variant, w, hpc):
    q, k, v = W.make_qkv(w)
    ref = torch.empty_like(v.cuda())
    if variant == "fp4":
        sa.sage_attn_fwd_fp4(q.cuda(), k.cuda(), v.cuda(), ref, w.causal, w.sm_scale)
    else:
        sa.sage_attn_fwd_fp8pv(q.cuda(), k.cuda(), v.cuda(), ref, w.causal, w.sm_scale, sa.SAGE_PER_BLOCK)
    q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o = torch.full_like(q, float("nan")).pin_memory()
    st = torch.cuda.current_stream()
    sa.sage_attn_fwd_host(q, k, v, o, w.causal, w.sm_scale, sa.SAGE_PER_BLOCK, heads_per_chunk=hpc, stream=st,
                          variant=variant)
    st.synchronize()
    assert sa.sage_last_device_error(st) == 0
    np.testing.assert_array_equal(o.numpy().view(np.uint16), ref.cpu().numpy().view(np.uint16))
