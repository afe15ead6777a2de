"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bar (the tolerances the method's error analysis gives):
  * K mean, INT8 codes, scales, INT32 Q.K^T: bit-exact;
  * O: max |O_gpu - O_oracle| <= 2e-3 * max|V| and cosine >= 0.9999, element by element
    over every output the oracle computes (all of it for small cases, sampled heads and
    rows at full sizes);
  * against unquantized fp64 attention on the K-outlier workloads: cosine >= 0.995.
The oracle gets the same seeded inputs (workloads.make_qkv) and never any GPU value,
except that the fused kernel is also fed the oracle's own quantized tensors, so that its
parity is checked independently of the quantization kernels.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

ATOL_FRAC = 2e-3   # of max|V|
COS_MIN = 0.9999
COS_EXACT_MIN = 0.995


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    assert torch.cuda.is_available()
    return sa


def gran_of(w):
    return 1 if w.per_block else 0


def groups_of(w):
    return oracle.GROUP_PER_BLOCK if w.per_block else oracle.GROUP_PER_TOKEN


def gpu_prep(sa, q, k, gran, smooth=True):
    qd, kd = q.cuda(), k.cuda()
    km, q8, k8, sq, sk = sa.empty_quantized(qd, gran)
    if smooth:
        sa.sage_smooth_k(kd, km)
    sa.sage_quant_qk(qd, kd, km if smooth else None, q8, k8, sq, sk, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    return dict(km=km.cpu().numpy(), q8=q8.cpu().numpy(), k8=k8.cpu().numpy(), sq=sq.cpu().numpy(),
                sk=sk.cpu().numpy())


def oracle_prep(q, k, w_per_block, smooth=True):
    gq, gk = oracle.GROUP_PER_BLOCK if w_per_block else oracle.GROUP_PER_TOKEN
    km = oracle.smooth_k(k) if smooth else None
    q8, sq = oracle.quant(q, gq)
    k8, sk = oracle.quant(k, gk, km)
    return dict(km=km, q8=q8, sq=sq, k8=k8, sk=sk)


def assert_o_close(o_gpu, o_ref64, vmax, what=""):
    o_gpu = np.asarray(o_gpu, np.float64)
    err = np.abs(o_gpu - o_ref64).max()
    cos = oracle.metrics(o_gpu, o_ref64)["cos"]
    assert err <= ATOL_FRAC * vmax, f"{what}: max abs err {err:.3e} > {ATOL_FRAC * vmax:.3e}"
    assert cos >= COS_MIN, f"{what}: cosine {cos:.6f}"


# ------------------------------------------------------------------ small full-tensor cases
EDGE = [
    W.Workload("edge_n128_d64_causal_blk", 1, 1, 128, 64, True, True, n_out=4, out_mag=20.0),
    W.Workload("edge_n128_d128_full_tok", 1, 1, 128, 128, False, False, n_out=4, out_mag=20.0),
    W.Workload("edge_n384_d128_full_tok", 1, 3, 384, 128, False, False, n_out=4, out_mag=20.0),
    W.Workload("edge_n384_d64_causal_tok", 2, 1, 384, 64, True, False, n_out=4, out_mag=20.0),
    W.Workload("edge_n640_d128_causal_blk", 1, 2, 640, 128, True, True, q_std=1.5, n_out=2, out_mag=40.0),
    W.Workload("edge_n512_d64_full_blk", 2, 2, 512, 64, False, True, bias_std=4.0),
]
SMALL_CASES = [W.TINY, W.SMALL] + EDGE


@pytest.mark.parametrize("w", SMALL_CASES, ids=lambda w: w.name)
def test_small_full_parity(sa, w):
    q, k, v = W.make_qkv(w)
    gran = gran_of(w)
    ref = oracle_prep(q, k, w.per_block)
    got = gpu_prep(sa, q, k, gran)
    for name in ("km", "q8", "sq", "k8", "sk"):
        np.testing.assert_array_equal(got[name], ref[name], err_msg=name)

    # INT32 Q.K^T through the debug entry point, bit-exact against exact integers
    q8d, k8d = torch.from_numpy(ref["q8"]).cuda(), torch.from_numpy(ref["k8"]).cuda()
    s = torch.empty((w.B, w.H, w.N, w.N), dtype=torch.int32, device="cuda")
    sa.sage_debug_qk_int32(q8d, k8d, s)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    np.testing.assert_array_equal(s.cpu().numpy().astype(np.int64), oracle.qk_int(ref["q8"], ref["k8"]))

    # fused kernel on the oracle's quantized tensors
    o64, _ = oracle.attn(ref["q8"], ref["k8"], ref["sq"], ref["sk"], v, w.causal, w.sm_scale, groups_of(w))
    vmax = float(np.abs(v.float().numpy()).max())
    vd = v.cuda()
    o = torch.empty_like(vd)
    sa.sage_attn_fwd_quantized(q8d, k8d, torch.from_numpy(ref["sq"]).cuda(), torch.from_numpy(ref["sk"]).cuda(),
                               vd, o, w.causal, w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    o_q = o.float().cpu().numpy()
    assert_o_close(o_q, o64, vmax, "fused kernel")

    # whole pipeline as a user calls it: same kernels, so identical to the above
    o2 = sa.sageattn(q.cuda(), k.cuda(), vd, w.causal, w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    np.testing.assert_array_equal(o2.cpu().numpy().view(np.uint16), o.cpu().numpy().view(np.uint16))

    # quality against exact attention on the outlier inputs
    exact = oracle.attn_fp64(q, k, v, w.causal, w.sm_scale)
    assert oracle.metrics(o_q, exact)["cos"] >= COS_EXACT_MIN


def test_causal_first_row_equals_first_value_row(sa):
    # Row 0 sees key 0 only: O[0] = fp16(fp16(p) * V[0] / p) for the single weight p.  The
    # kernel's exponent offset may sit up to one offset quantum above the row maximum, so p
    # can be just below 1 and each fp16 rounding adds at most 2^-11 relative error.
    w = W.Workload("c0", 1, 2, 256, 128, True, True, n_out=4, out_mag=20.0)
    q, k, v = W.make_qkv(w)
    o = sa.sageattn(q.cuda(), k.cuda(), v.cuda(), True, w.sm_scale, 1).cpu()
    v0 = v[:, :, 0].double()
    assert torch.all((o[:, :, 0].double() - v0).abs() <= 2.0**-10 * v0.abs() + 1e-7)


def test_zero_queries_give_prefix_means(sa):
    w = W.Workload("zq", 1, 1, 384, 64, True, False)
    _, k, v = W.make_qkv(w)
    q = torch.zeros_like(k)
    o = sa.sageattn(q.cuda(), k.cuda(), v.cuda(), True, w.sm_scale, 0).float().cpu().numpy()[0, 0]
    vf = v.float().numpy()[0, 0].astype(np.float64)
    prefix = np.cumsum(vf, axis=0) / np.arange(1, w.N + 1)[:, None]
    assert np.abs(o - prefix).max() <= ATOL_FRAC * np.abs(vf).max()


def test_zero_key_block_gives_zero_scale(sa):
    # an all-zero K block (after smoothing a constant K) quantizes to scale 0 / codes 0
    w = W.Workload("zk", 1, 1, 256, 128, False, True)
    q, k, v = W.make_qkv(w)
    k = torch.full_like(k, 0.75)
    got = gpu_prep(sa, q, k, 1)
    ref = oracle_prep(q, k, True)
    for name in ("km", "q8", "sq", "k8", "sk"):
        np.testing.assert_array_equal(got[name], ref[name], err_msg=name)
    assert np.all(got["sk"] == 0) and np.all(got["k8"] == 0)
    o = sa.sageattn(q.cuda(), k.cuda(), v.cuda(), False, w.sm_scale, 1).float().cpu().numpy()[0, 0]
    np.testing.assert_allclose(o, np.broadcast_to(v.float().numpy()[0, 0].mean(0), o.shape),
                               atol=ATOL_FRAC * float(v.abs().max()))


def test_smoothing_off_path_matches_oracle(sa):
    q, k, v = W.make_qkv(W.TINY)
    got = gpu_prep(sa, q, k, 0, smooth=False)
    ref = oracle_prep(q, k, False, smooth=False)
    for name in ("q8", "sq", "k8", "sk"):
        np.testing.assert_array_equal(got[name], ref[name], err_msg=name)


def test_repeated_calls_are_deterministic(sa):
    w = W.SMALL
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    a = sa.sageattn(q, k, v, w.causal, w.sm_scale, 1)
    b = sa.sageattn(q, k, v, w.causal, w.sm_scale, 1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ------------------------------------------------------------------ full-size workloads
# every workload the benchmark and the measured sweep report: the LLM and video-DiT shapes, the
# per-token headline variants, and all 24 points of the N x d x causal sweep (the headline among them)
BIG = [W.LLM, W.DIT, W.TOKEN128, W.TOKEN64] + [W.sweep(n, d, c) for n in W.SWEEP_N for d in W.SWEEP_D
                                                for c in (False, True)]


def sample_rows(N, n=40, seed=0):
    r = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 255, 256, N // 2, N - 129, N - 128, N - 1]
    return np.unique(np.concatenate([fixed, r.integers(0, N, n)])).astype(np.int64)


@pytest.mark.parametrize("w", BIG, ids=lambda w: w.name)
def test_full_size_parity(sa, w):
    q, k, v = W.make_qkv(w)
    gran = gran_of(w)
    ref = oracle_prep(q, k, w.per_block)
    got = gpu_prep(sa, q, k, gran)
    for name in ("km", "q8", "sq", "k8", "sk"):
        np.testing.assert_array_equal(got[name], ref[name], err_msg=name)
    del got

    # the whole pipeline in the launch configuration the benchmark times
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    sa.sage_attn_fwd(qd, kd, vd, o, w.causal, w.sm_scale, gran)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    o = o.view(w.BH, w.N, w.d).float().cpu().numpy()
    vv = v.view(w.BH, w.N, w.d)
    q8 = ref["q8"].reshape(w.BH, w.N, w.d)
    k8 = ref["k8"].reshape(w.BH, w.N, w.d)
    sq = ref["sq"].reshape(w.BH, -1)
    sk = ref["sk"].reshape(w.BH, -1)
    heads = sorted({0, w.BH - 1, w.BH // 2})
    rows = sample_rows(w.N)
    for h in heads:
        r64, _ = oracle.attn_rows(q8[h], k8[h], sq[h], sk[h], vv[h], rows, w.causal, w.sm_scale, groups_of(w))
        vmax = float(vv[h].abs().max())
        assert_o_close(o[h, rows], r64, vmax, f"head {h}")
        exact_rows = _exact_rows(q.view(w.BH, w.N, w.d)[h], k.view(w.BH, w.N, w.d)[h], vv[h], rows, w)
        assert oracle.metrics(o[h, rows], exact_rows)["cos"] >= COS_EXACT_MIN

    # INT32 Q.K^T of one head at full N, sampled rows
    if w.N * w.N < 2**31:
        s = torch.empty((1, 1, w.N, w.N), dtype=torch.int32, device="cuda")
        q8h = torch.from_numpy(np.ascontiguousarray(q8[heads[-1]])).cuda().view(1, 1, w.N, w.d)
        k8h = torch.from_numpy(np.ascontiguousarray(k8[heads[-1]])).cuda().view(1, 1, w.N, w.d)
        sa.sage_debug_qk_int32(q8h, k8h, s)
        torch.cuda.synchronize()
        assert sa.sage_last_device_error() == 0
        srows = s[0, 0, torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.int64)
        np.testing.assert_array_equal(srows, oracle.qk_int_rows(q8[heads[-1]], k8[heads[-1]], rows))


def _exact_rows(qh, kh, vh, rows, w):
    """fp64 unquantized attention for the sampled rows of one head (numpy)."""
    qf = qh.double().numpy()[rows]
    kf = kh.double().numpy()
    vf = vh.double().numpy()
    s = (qf @ kf.T) * w.sm_scale
    if w.causal:
        s = np.where(np.arange(w.N)[None, :] <= rows[:, None], s, -np.inf)
    s -= s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ vf


@pytest.mark.parametrize("d,causal", [(128, False), (128, True), (64, True)])
def test_traced_kernel_matches_untraced_and_stamps_are_ordered(sa, d, causal):
    w = W.Workload(f"trace_b1h2_n1024_d{d}", 1, 2, 1024, d, causal, True, n_out=4, out_mag=20.0)
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    km, q8, k8, sq, sk = sa.empty_quantized(q, 1)
    sa.sage_smooth_k(k, km)
    sa.sage_quant_qk(q, k, km, q8, k8, sq, sk, 1)
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    sa.sage_attn_fwd_quantized(q8, k8, sq, sk, v, o1, w.causal, w.sm_scale, 1)
    T = w.N // 128
    ctas = 8  # every CTA of the first head: causal pairs with 8, 6, 4 and 2 key tiles
    tr = torch.zeros((ctas, 2 + 10 * T), dtype=torch.int64, device="cuda")
    sa.sage_debug_attn_trace(q8, k8, sq, sk, v, o2, w.causal, w.sm_scale, 1, tr, ctas)
    torch.cuda.synchronize()
    # 0: no wait timed out, and (2 otherwise) every CTA's final barrier held all its threads
    assert sa.sage_last_device_error() == 0
    assert torch.equal(o1, o2)
    tr = tr.cpu().numpy()
    assert np.all(tr[:, 1] > tr[:, 0])
    # the end stamp is taken after the CTA's final barrier: every event of the CTA comes before it
    assert np.all(tr[:, 2:].max(axis=1) <= tr[:, 1])
    assert np.all(tr[:, 2:][tr[:, 2:] > 0] >= np.repeat(tr[:, :1], tr.shape[1] - 2, axis=1)[tr[:, 2:] > 0])
    for t in range(2):
        s_ready = tr[:, 2 + 3 * t * T: 2 + (3 * t + 1) * T]
        p_sig = tr[:, 2 + (3 * t + 2) * T: 2 + (3 * t + 3) * T]
        done = s_ready > 0  # key tiles this query tile processed (all of them when non-causal)
        assert np.all((p_sig > s_ready)[done])
        assert np.all(p_sig[~done] == 0)
        for c in range(ctas):
            assert np.all(np.diff(s_ready[c][done[c]]) > 0)
        if not causal:
            assert done.all()


def test_mma_peak_probe_rates(sa):
    # dense per-SM rates of the three kinds; FP16 near the datasheet 4096 MAC/clk/SM, INT8 and
    # FP8 about twice that (bounds loose enough for clock and issue jitter)
    r = {k: sa.mma_peak(k, iters=2048)["macs_per_clk_per_sm"] for k in (0, 1, 2)}
    assert 2000 < r[1] < 4400, r
    assert 1.5 < r[0] / r[1] < 2.2 and 1.5 < r[2] / r[1] < 2.2, r
