"""GPU parity of the block-sparse variant (SpargeAttn abstract: a predicted attention map skips
block products, a softmax-aware filter skips more) through the C ABI, against
oracle/sage_oracle_sparse.c.

Bar:
  * stage 1: the GPU's kept key blocks equal the oracle's on every block whose decision the
    oracle does not flag as within 1e-4 of flipping (the GPU computes the block means, the
    compressed map and the similarities in fp32, the oracle in fp64);
  * the fused kernel, given the GPU's block lists: O against the oracle run on the same kept
    blocks: max |O_gpu - O_oracle| <= 2e-3 * max|V| and cosine >= 0.9999 -- the FP16 path's bar.
    Where the two sides' stage-2 decisions differ (a block maximum within rounding of the
    running maximum minus lambda), the dropped weights are all below 2^-lambda of the row's
    running maximum: at lambda = 20 a 128-key block moves O by at most 128 * 2^-20 * max|V|,
    inside the bar;
  * with every block kept and stage 2 off, the sparse kernel is bit-identical to the dense one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

ATOL_FRAC = 2e-3
COS_MIN = 0.9999
TAU, THETA, LAM = 0.99, 0.3, 20.0


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    return sa


def _groups(w):
    return oracle.GROUP_PER_BLOCK if w.per_block else oracle.GROUP_PER_TOKEN


def gpu_predict(sa, q, k, causal, sm_scale, tau=TAU, theta=THETA):
    B, H, N, d = q.shape
    nqb, nkb = sa.sparse_blocks(N)
    cnt = torch.zeros((B, H, nqb), dtype=torch.int32, device="cuda")
    idx = torch.full((B, H, nqb, nkb), -1, dtype=torch.int16, device="cuda")
    sa.sage_sparse_predict(q.cuda(), k.cuda(), causal, sm_scale, tau, theta, cnt, idx)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    return cnt, idx


def lists_to_mask(cnt, idx):
    cnt, idx = cnt.cpu().numpy(), idx.cpu().numpy().astype(np.int64)
    mask = np.zeros(idx.shape, np.uint8)
    it = np.ndindex(cnt.shape)
    for pos in it:
        c = cnt[pos]
        lst = idx[pos][:c]
        assert np.all(np.diff(lst) > 0) and (c == 0 or (lst[0] >= 0 and lst[-1] < idx.shape[-1]))
        mask[pos][lst] = 1
    return mask


def mask_to_lists(mask):
    mask = np.asarray(mask, np.uint8)
    cnt = mask.sum(axis=-1).astype(np.int32)
    idx = np.zeros(mask.shape, np.int16)
    for pos in np.ndindex(mask.shape[:-1]):
        lst = np.nonzero(mask[pos])[0]
        idx[pos][:lst.size] = lst
    return torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda()


def assert_close(o_gpu, o_ref, vmax, what):
    o_gpu = np.asarray(o_gpu, np.float64)
    err = np.abs(o_gpu - o_ref).max()
    cos = oracle.metrics(o_gpu, o_ref)["cos"]
    assert err <= ATOL_FRAC * vmax, f"{what}: max abs err {err:.3e} > {ATOL_FRAC * vmax:.3e}"
    assert cos >= COS_MIN, f"{what}: cosine {cos:.6f}"


PRED = [
    W.Workload("sp_win_n4096", 1, 4, 4096, 128, False, True, window=512, align=12.0),
    W.Workload("sp_win_causal_n3000", 1, 3, 3000, 128, True, True, window=384, align=10.0),
    W.Workload("sp_random_n2048", 2, 2, 2048, 128, False, False, n_out=4, out_mag=20.0),
]


@pytest.mark.parametrize("w", PRED, ids=lambda w: w.name)
@pytest.mark.parametrize("tau,theta", [(TAU, THETA), (0.7, 0.5), (0.5, 0.0)])
def test_predicted_blocks_match_the_oracle(sa, w, tau, theta):
    q, k, _ = W.make_qkv(w)
    cnt, idx = gpu_predict(sa, q, k, w.causal, w.sm_scale, tau, theta)
    got = lists_to_mask(cnt, idx)
    ref, unsure, _, _ = oracle.sparse_predict(q, k, w.causal, w.sm_scale, tau, theta)
    sure = unsure == 0
    mismatch = (got != ref) & sure
    assert not mismatch.any(), f"{mismatch.sum()} decided blocks differ"
    # most decisions are clear of rounding (structureless inputs give near-equal probabilities)
    assert sure.mean() > (0.5 if w.window == 0 else 0.9)


SMALL = [
    W.Workload("sp_small_win", 1, 2, 2048, 128, False, True, window=512, align=12.0),
    W.Workload("sp_small_win_causal", 1, 2, 2048, 128, True, True, window=512, align=12.0),
    W.Workload("sp_small_ragged_tok", 1, 2, 1500, 128, False, False, window=384, align=10.0),
    W.Workload("sp_small_ragged_causal_tok", 1, 2, 1100, 128, True, False, window=256, align=10.0),
    # head dimension 64 (the video-DiT kernel)
    W.Workload("sp_small_win_d64", 1, 2, 2048, 64, False, True, window=512, align=9.0, bias_std=4.0),
    W.Workload("sp_small_win_causal_d64", 1, 2, 2048, 64, True, True, window=512, align=9.0),
    W.Workload("sp_small_ragged_tok_d64", 1, 2, 1500, 64, False, False, window=384, align=8.0),
    W.Workload("sp_small_ragged_causal_tok_d64", 1, 2, 1100, 64, True, False, window=256, align=8.0),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("lam", [LAM, math.inf])
def test_sparse_fused_kernel_matches_the_oracle(sa, w, lam):
    q, k, v = W.make_qkv(w)
    gran = 1 if w.per_block else 0
    gq, gk = _groups(w)
    cnt, idx = gpu_predict(sa, q, k, w.causal, w.sm_scale)
    mask = lists_to_mask(cnt, idx)
    km = oracle.smooth_k(k)
    q8, sq = oracle.quant(q, gq)
    k8, sk = oracle.quant(k, gk, km)
    t = [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (q8, k8, sq, sk)]
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_sparse_quantized(*t, v.cuda(), o, w.causal, w.sm_scale, gran, cnt, idx, lam)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    o64, _, skipped = oracle.attn_sparse(q8, k8, sq, sk, v, mask, w.causal, w.sm_scale, lam, (gq, gk))
    vmax = float(v.abs().max())
    assert_close(o.float().cpu().numpy(), o64, vmax, w.name)
    assert mask.mean() < 0.75  # the case really is sparse
    # and the whole variant as a user calls it gives the same output
    o2 = torch.empty_like(o)
    sa.sage_attn_fwd_sparse(q.cuda(), k.cuda(), v.cuda(), o2, w.causal, w.sm_scale, gran, TAU, THETA, lam)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    assert torch.equal(o2, o)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1024, 1000])
def test_all_blocks_without_stage_two_equal_the_dense_kernel(sa, causal, N, d):
    w = W.Workload("sp_dense", 1, 3, N, d, causal, True, n_out=4, out_mag=20.0)
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    km, q8, k8, sq, sk = sa.empty_quantized(q, 1)
    sa.sage_smooth_k(k, km)
    sa.sage_quant_qk(q, k, km, q8, k8, sq, sk, 1)
    nqb, nkb = sa.sparse_blocks(N)
    full = np.ones((1, 3, nqb, nkb), np.uint8)
    if causal:  # the visible blocks of each query block
        for i in range(nqb):
            full[:, :, i, (min(N, (i + 1) * 256) - 1) // 128 + 1:] = 0
    cnt, idx = mask_to_lists(full)
    o_dense, o_sparse = torch.empty_like(q), torch.empty_like(q)
    sa.sage_attn_fwd_quantized(q8, k8, sq, sk, v, o_dense, causal, w.sm_scale, 1)
    sa.sage_attn_fwd_sparse_quantized(q8, k8, sq, sk, v, o_sparse, causal, w.sm_scale, 1, cnt, idx, math.inf)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    assert torch.equal(o_dense, o_sparse)


@pytest.mark.parametrize("d", [64, 128])
def test_random_block_lists(sa, d):
    # any ascending lists work (stage 1 bypassed), causal lists holding each query's own blocks
    N, causal = 1536, True
    w = W.Workload("sp_lists", 1, 2, N, d, causal, True, n_out=4, out_mag=20.0)
    q, k, v = W.make_qkv(w)
    nqb, nkb = sa.sparse_blocks(N)
    rng = np.random.default_rng(5)
    mask = (rng.random((1, 2, nqb, nkb)) < 0.4).astype(np.uint8)
    for i in range(nqb):
        mask[:, :, i, (min(N, (i + 1) * 256) - 1) // 128 + 1:] = 0
        mask[:, :, i, 2 * i:2 * i + 2] = 1
    cnt, idx = mask_to_lists(mask)
    km = oracle.smooth_k(k)
    q8, sq = oracle.quant(q, 128)
    k8, sk = oracle.quant(k, 64, km)
    t = [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (q8, k8, sq, sk)]
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_sparse_quantized(*t, v.cuda(), o, causal, w.sm_scale, 1, cnt, idx, 8.0)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    o64, _, _ = oracle.attn_sparse(q8, k8, sq, sk, v, mask, causal, w.sm_scale, 8.0, (128, 64))
    assert_close(o.float().cpu().numpy(), o64, float(v.abs().max()), "random lists")


BIG = [W.SPARSE, W.SPARSE_CAUSAL, W.SPARSE_DIT]


@pytest.mark.parametrize("w", BIG, ids=lambda w: w.name)
def test_sparse_full_size(sa, w):
    q, k, v = W.make_qkv(w)
    gq, gk = _groups(w)
    cnt, idx = gpu_predict(sa, q, k, w.causal, w.sm_scale)
    mask = lists_to_mask(cnt, idx)
    ref, unsure, _, _ = oracle.sparse_predict(q, k, w.causal, w.sm_scale, TAU, THETA)
    assert not ((mask != ref) & (unsure == 0)).any()
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_sparse(q.cuda(), k.cuda(), v.cuda(), o, w.causal, w.sm_scale, 1, TAU, THETA, LAM)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    og = o.view(w.BH, w.N, w.d).float().cpu().numpy()
    km = oracle.smooth_k(k)
    q8, sq = oracle.quant(q, gq)
    k8, sk = oracle.quant(k, gk, km)
    q8, k8 = q8.reshape(w.BH, w.N, w.d), k8.reshape(w.BH, w.N, w.d)
    sq, sk = sq.reshape(w.BH, -1), sk.reshape(w.BH, -1)
    vv = v.view(w.BH, w.N, w.d)
    m = mask.reshape(w.BH, *mask.shape[-2:])
    tiles = np.array([0, 1, 63, 64, 127])
    for h in (0, w.BH // 2, w.BH - 1):
        t64, _ = oracle.attn_sparse_tiles(q8[h], k8[h], sq[h], sk[h], vv[h], m[h], tiles, w.causal, w.sm_scale, LAM,
                                          (gq, gk))
        got = np.stack([og[h, 128 * t:128 * t + 128] for t in tiles])
        assert_close(got, t64, float(vv[h].abs().max()), f"{w.name} head {h}")
    # the sparse method stays close to exact attention on the windowed inputs
    rows = np.array([5, 3000, 9000, 16000])
    qf, kf, vf = (x.view(w.BH, w.N, w.d)[0].double().numpy() for x in (q, k, v))
    s = qf[rows] @ kf.T * w.sm_scale
    if w.causal:
        s = np.where(np.arange(w.N)[None, :] <= rows[:, None], s, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    exact = (e / e.sum(axis=1, keepdims=True)) @ vf
    assert oracle.metrics(og[0, rows], exact)["cos"] >= 0.99


def test_sparse_rejects_what_it_does_not_support(sa):
    # more than 512 key tiles (N > 65536): the kernels' lists hold at most 512
    q = torch.zeros((1, 1, 65536 + 256, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(sa.SageError) as e:
        sa.sage_attn_fwd_sparse(q, q, q, torch.empty_like(q), False, 0.125, 1, TAU, THETA, LAM)
    assert e.value.status == sa.SAGE_ERR_UNSUPPORTED
