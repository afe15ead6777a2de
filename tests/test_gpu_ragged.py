"""GPU parity for sequence lengths that are not a multiple of the 128-token tile.

The last query tile and the last key tile are partial: query rows past N are computed on
zeros and never stored, keys past N are masked out of the maximum and get P~ = 0, and the
per-block scale groups (128 Q / 64 K tokens) end with a partial group.  Same bar as the
whole-tile cases: quantization bit-exact, O within 2e-3 * max|V| and cosine >= 0.9999 of
the oracle, and nothing written outside [B, H, N, d].
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from test_gpu_parity import COS_EXACT_MIN, assert_o_close, gpu_prep, gran_of, groups_of, oracle_prep

pytestmark = pytest.mark.gpu

RAGGED = [
    W.Workload("ragged_n1_d64_full_tok", 1, 2, 1, 64, False, False),
    W.Workload("ragged_n37_d128_causal_blk", 1, 2, 37, 128, True, True, n_out=4, out_mag=20.0),
    W.Workload("ragged_n64_d128_full_blk", 1, 2, 64, 128, False, True, n_out=4, out_mag=20.0),
    W.Workload("ragged_n100_d64_full_blk", 2, 1, 100, 64, False, True, n_out=4, out_mag=20.0),
    W.Workload("ragged_n130_d64_causal_blk", 1, 2, 130, 64, True, True, bias_std=4.0),
    W.Workload("ragged_n200_d128_causal_tok", 1, 2, 200, 128, True, False, n_out=4, out_mag=20.0),
    W.Workload("ragged_n333_d64_causal_tok", 2, 1, 333, 64, True, False, n_out=4, out_mag=20.0),
    W.Workload("ragged_n383_d128_full_tok", 1, 3, 383, 128, False, False, n_out=4, out_mag=20.0),
    W.Workload("ragged_n1000_d128_full_blk", 1, 2, 1000, 128, False, True, q_std=1.5, n_out=2, out_mag=40.0),
    W.Workload("ragged_n1001_d128_causal_blk", 1, 1, 1001, 128, True, True, n_out=4, out_mag=20.0),
]


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    assert torch.cuda.is_available()
    return sa


@pytest.mark.parametrize("w", RAGGED, ids=lambda w: w.name)
def test_ragged_parity(sa, w):
    q, k, v = W.make_qkv(w)
    gran = gran_of(w)
    ref = oracle_prep(q, k, w.per_block)
    got = gpu_prep(sa, q, k, gran)
    for name in ("km", "q8", "sq", "k8", "sk"):
        np.testing.assert_array_equal(got[name], ref[name], err_msg=name)

    # fused kernel on the oracle's quantized tensors; O sits inside a larger buffer whose
    # guard bands must stay untouched (stores past N are clipped, not wrapped into the next head)
    o64, _ = oracle.attn(ref["q8"], ref["k8"], ref["sq"], ref["sk"], v, w.causal, w.sm_scale, groups_of(w))
    vmax = float(np.abs(v.float().numpy()).max())
    vd = v.cuda()
    guard = 4096
    sentinel = torch.full((guard * 2 + v.numel(),), 1234.0, dtype=torch.float16, device="cuda")  # exact in fp16
    o = sentinel[guard:guard + v.numel()].view(v.shape)
    sa.sage_attn_fwd_quantized(torch.from_numpy(ref["q8"]).cuda(), torch.from_numpy(ref["k8"]).cuda(),
                               torch.from_numpy(ref["sq"]).cuda(), torch.from_numpy(ref["sk"]).cuda(),
                               vd, o, w.causal, w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    band = torch.cat([sentinel[:guard], sentinel[guard + v.numel():]]).float().cpu().numpy()
    assert np.all(band == 1234.0), "a store landed outside O"
    o_q = o.float().cpu().numpy()
    assert np.isfinite(o_q).all()
    assert_o_close(o_q, o64, vmax, "fused kernel")

    # whole pipeline as a user calls it (workspace path): same kernels, identical output
    o2 = sa.sageattn(q.cuda(), k.cuda(), vd, w.causal, w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    np.testing.assert_array_equal(o2.cpu().numpy().view(np.uint16), o.cpu().numpy().view(np.uint16))

    exact = oracle.attn_fp64(q, k, v, w.causal, w.sm_scale)
    assert oracle.metrics(o_q, exact)["cos"] >= COS_EXACT_MIN


def test_ragged_tail_matches_truncated_whole_tile_problem(sa):
    # the first n tokens of a whole-tile problem, run alone, give the causal outputs of those
    # rows exactly as the whole problem does (causal rows only see earlier keys; per-token
    # scales do not depend on the other tokens; the K mean does, so smoothing is left off)
    w = W.Workload("ragged_prefix_src", 1, 2, 256, 128, True, False, n_out=4, out_mag=20.0)
    q, k, v = W.make_qkv(w)
    n = 173
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    full = torch.empty_like(vd)
    part = torch.empty_like(vd[:, :, :n]).contiguous()

    def run(qq, kk, vv, oo):
        km, q8, k8, sq, sk = sa.empty_quantized(qq, sa.SAGE_PER_TOKEN)
        sa.sage_quant_qk(qq, kk, None, q8, k8, sq, sk, sa.SAGE_PER_TOKEN)
        sa.sage_attn_fwd_quantized(q8, k8, sq, sk, vv, oo, True, w.sm_scale, sa.SAGE_PER_TOKEN)

    run(qd, kd, vd, full)
    run(qd[:, :, :n].contiguous(), kd[:, :, :n].contiguous(), vd[:, :, :n].contiguous(), part)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    # same tiles, same operations in the same order for every row < n: bit-identical
    np.testing.assert_array_equal(part.cpu().numpy().view(np.uint16),
                                  full[:, :, :n].contiguous().cpu().numpy().view(np.uint16))
