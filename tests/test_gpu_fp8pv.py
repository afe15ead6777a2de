"""GPU parity of the FP8 P.V variant (SageAttention2 abstract: (P~, V) in FP8, V smoothed,
P~V accumulated in an FP32 buffer) through the C ABI, against oracle/sage_oracle_sa2.c.

Bar:
  * V codes (E4M3), per-channel scales and channel means: bit-exact;
  * O against the oracle: cosine >= 0.9999, and element by element
        |O_gpu - O_oracle| <= 1e-3 * max|V^| + envelope,
    where envelope_c = sum over keys j whose exact weight p_j lies within a relative 2e-4 of an
    E4M3 rounding midpoint of (one E4M3 step of p_j) * |V^_jc| / l.  The kernel computes the
    weight in fp32 (a scale trimmed by up to 2^-20, exp2 approximations with relative error up
    to 7.5e-5), so a weight that close to a midpoint may round to either neighbour; both are
    correct roundings of the weight at the kernel's precision.  Every other weight rounds as the
    oracle rounds it: both use integer row offsets in log2 units, so both round on the same E4M3
    grid.  V^ = dequantized V (codes * sv).
  * against unquantized fp64 attention on the K-outlier inputs: cosine >= 0.99 (an FP8 V carries
    a relative 2^-4 rounding per element; the FP16 path's bar is 0.995).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

BASE_FRAC = 1e-3
NEAR_REL = 2e-4
COS_MIN = 0.9999
COS_EXACT_MIN = 0.99


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    return sa


def _groups(w):
    return oracle.GROUP_PER_BLOCK if w.per_block else oracle.GROUP_PER_TOKEN


def _envelope(q8h, k8h, sqh, skh, vhat, rows, N, causal, sm_scale, groups):
    """Per sampled row: sum over keys near an E4M3 midpoint of one step x |V^| / l (numpy, fp64)."""
    gq, gk = groups
    S = oracle.qk_int_rows(q8h, k8h, rows).astype(np.float64)
    sqr = np.repeat(sqh.astype(np.float64), gq)[:N][rows]
    skr = np.repeat(skh.astype(np.float64), gk)[:N]
    u = S * sqr[:, None] * skr[None, :] * sm_scale * math.log2(math.e)
    if causal:
        u = np.where(np.arange(N)[None, :] <= rows[:, None], u, -np.inf)
    M = np.ceil(u.max(axis=1, keepdims=True))
    p = np.exp2(u - M + 8)
    l = p.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(p > 0, p, 1.0)))
    step = np.where(p >= 2.0**-6, np.exp2(e - 3), 2.0**-9)
    frac = p / step - np.floor(p / step)
    near = (np.abs(frac - 0.5) * step <= NEAR_REL * p) & (p > 0)
    return (np.where(near, step, 0.0) / l) @ np.abs(vhat)


def _check_rows(o_gpu, o_ref, env, vhat_max, what):
    o_gpu = np.asarray(o_gpu, np.float64)
    err = np.abs(o_gpu - o_ref)
    bar = BASE_FRAC * vhat_max + env
    worst = np.unravel_index(np.argmax(err - bar), err.shape)
    assert np.all(err <= bar), f"{what}: err {err[worst]:.3e} > bar {bar[worst]:.3e} at {worst}"
    cos = oracle.metrics(o_gpu, o_ref)["cos"]
    assert cos >= COS_MIN, f"{what}: cosine {cos:.6f}"


def _gpu_quant_v(sa, v, smooth=True):
    vd = v.cuda()
    B, H, N, d = v.shape
    v8 = torch.empty((B, H, N, d), dtype=torch.uint8, device="cuda")
    sv = torch.empty((B, H, d), dtype=torch.float32, device="cuda")
    vm = torch.empty((B, H, d), dtype=torch.float32, device="cuda") if smooth else None
    sa.sage_quant_v_fp8(vd, v8, sv, vm)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    return v8, sv, vm


@pytest.mark.parametrize("N,d,smooth", [(128, 128, True), (1000, 128, True), (4096, 64, True), (777, 64, False),
                                        (16384, 128, True), (20000, 128, False), (1, 128, True)])
def test_quant_v_fp8_bit_exact(sa, N, d, smooth):
    w = W.Workload(f"qv_n{N}_d{d}", 1, 3, N, d, False, True, bias_std=4.0)
    _, _, v = W.make_qkv(w)
    v = (v.float() + torch.linspace(-3, 3, d)).half()  # channel offsets for the smoothing to remove
    v8, sv, vm = _gpu_quant_v(sa, v, smooth)
    r8, rsv, rvm = oracle.quant_v_fp8(v, smooth)
    np.testing.assert_array_equal(v8.cpu().numpy(), r8)
    np.testing.assert_array_equal(sv.cpu().numpy(), rsv)
    if smooth:
        np.testing.assert_array_equal(vm.cpu().numpy(), rvm)


def test_quant_v_fp8_extremes(sa):
    # fp16 extremes, a constant channel (scale 0) and a channel of one nonzero token
    v = torch.zeros((1, 1, 256, 128), dtype=torch.float16)
    v[0, 0, :, 0] = 65504.0
    v[0, 0, ::2, 1] = -65504.0
    v[0, 0, :, 2] = 0.5
    v[0, 0, 7, 3] = 2.0**-24
    v[0, 0, :, 4:] = torch.randn(256, 124).half() * 100
    for smooth in (True, False):
        v8, sv, vm = _gpu_quant_v(sa, v, smooth)
        r8, rsv, rvm = oracle.quant_v_fp8(v, smooth)
        np.testing.assert_array_equal(v8.cpu().numpy(), r8)
        np.testing.assert_array_equal(sv.cpu().numpy(), rsv)


SMALL = [
    W.Workload("fp8_tiny_tok", 1, 2, 256, 128, False, False, n_out=4, out_mag=20.0),
    W.Workload("fp8_small_causal_blk", 1, 4, 1024, 128, True, True, n_out=8, out_mag=30.0),
    W.Workload("fp8_ragged_causal_tok", 1, 2, 640, 128, True, False, q_std=1.5, n_out=2, out_mag=40.0),
    W.Workload("fp8_ragged_full_blk", 2, 1, 333, 128, False, True, bias_std=4.0),
    W.Workload("fp8_n128_causal_blk", 1, 1, 128, 128, True, True, n_out=4, out_mag=20.0),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fp8pv_small_full_parity(sa, w):
    q, k, v = W.make_qkv(w)
    gran = 1 if w.per_block else 0
    ref = oracle.sage_attn_fp8pv(q, k, v, w.causal, w.sm_scale, per_block=w.per_block)
    # the fused kernel on the oracle's own quantized tensors
    t = {n: torch.from_numpy(np.ascontiguousarray(ref[n])).cuda() for n in ("q8", "k8", "sq", "sk", "v8", "sv", "vm")}
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_fp8pv_quantized(t["q8"], t["k8"], t["sq"], t["sk"], t["v8"], t["sv"], t["vm"], o, w.causal,
                                     w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    og = o.view(w.BH, w.N, w.d).float().cpu().numpy()
    o64 = ref["o64"].reshape(w.BH, w.N, w.d)
    vhat = oracle.e4m3_decode(ref["v8"]).reshape(w.BH, w.N, w.d) * ref["sv"].reshape(w.BH, 1, w.d)
    rows = np.arange(w.N)
    for h in range(w.BH):
        env = _envelope(ref["q8"].reshape(w.BH, w.N, w.d)[h], ref["k8"].reshape(w.BH, w.N, w.d)[h],
                        ref["sq"].reshape(w.BH, -1)[h], ref["sk"].reshape(w.BH, -1)[h], vhat[h], rows, w.N, w.causal,
                        w.sm_scale, _groups(w))
        _check_rows(og[h], o64[h], env, np.abs(vhat[h]).max(), f"{w.name} head {h}")
    # the whole variant as a user calls it: same kernels on the same inputs, so identical
    o2 = torch.empty_like(o)
    sa.sage_attn_fwd_fp8pv(q.cuda(), k.cuda(), v.cuda(), o2, w.causal, w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    assert torch.equal(o2, o)
    exact = oracle.attn_fp64(q, k, v, w.causal, w.sm_scale)
    assert oracle.metrics(og.reshape(exact.shape), exact)["cos"] >= COS_EXACT_MIN


BIG = [W.HEADLINE, W.LLM, W.sweep(4096, 128, False), W.TOKEN128]


@pytest.mark.parametrize("w", BIG, ids=lambda w: w.name)
def test_fp8pv_full_size_parity(sa, w):
    q, k, v = W.make_qkv(w)
    gran = 1 if w.per_block else 0
    gq, gk = _groups(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    sa.sage_attn_fwd_fp8pv(qd, kd, vd, o, w.causal, w.sm_scale, gran)
    v8, sv, vm = _gpu_quant_v(sa, v)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    r8, rsv, rvm = oracle.quant_v_fp8(v)
    np.testing.assert_array_equal(v8.cpu().numpy(), r8)
    np.testing.assert_array_equal(sv.cpu().numpy(), rsv)
    np.testing.assert_array_equal(vm.cpu().numpy(), rvm)
    km = oracle.smooth_k(k)
    q8, sq = oracle.quant(q, gq)
    k8, sk = oracle.quant(k, gk, km)
    og = o.view(w.BH, w.N, w.d).float().cpu().numpy()
    q8, k8 = q8.reshape(w.BH, w.N, w.d), k8.reshape(w.BH, w.N, w.d)
    sq, sk = sq.reshape(w.BH, -1), sk.reshape(w.BH, -1)
    r8, rsv, rvm = r8.reshape(w.BH, w.N, w.d), rsv.reshape(w.BH, w.d), rvm.reshape(w.BH, w.d)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N // 2, w.N - 1], rng.integers(0, w.N, 30)])).astype(np.int64)
    for h in sorted({0, w.BH // 2, w.BH - 1}):
        r64 = oracle.attn_fp8pv_rows(q8[h], k8[h], sq[h], sk[h], r8[h], rsv[h], rvm[h], rows, w.causal, w.sm_scale,
                                     (gq, gk))
        vhat = oracle.e4m3_decode(r8[h]) * rsv[h][None, :]
        env = _envelope(q8[h], k8[h], sq[h], sk[h], vhat, rows, w.N, w.causal, w.sm_scale, (gq, gk))
        _check_rows(og[h, rows], r64, env, np.abs(vhat).max(), f"{w.name} head {h}")


def test_fp8pv_rejects_head_dim_64(sa):
    q = torch.zeros((1, 1, 128, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(sa.SageError) as e:
        sa.sage_attn_fwd_fp8pv(q, q, q, torch.empty_like(q), False, 0.125, 1)
    assert e.value.status == sa.SAGE_ERR_UNSUPPORTED
