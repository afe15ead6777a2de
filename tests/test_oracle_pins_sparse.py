"""Pins of the oracle's block-sparse variant (oracle/sage_oracle_sparse.c; SpargeAttn abstract:
a first stage that predicts the attention map and skips matrix products, a second softmax-aware
stage inside the online softmax that skips more) against facts that do not come from it: the
dense oracle (already pinned) when nothing is dropped, textbook attention over the kept keys,
brute-force re-derivations of the predicted map in numpy, closed forms of the self-similarity,
and hand-built cases of the second stage.  Readings: the top of sage_oracle_sparse.c.
"""
import math

import numpy as np
import pytest

import oracle
from test_oracle_pins import exact_attention, fp16

RNG = np.random.default_rng(7)
INF = float("inf")


def _rand_quant(N, d, groups=(1, 1), spread=3.0):
    gq, gk = groups
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    sq = (RNG.uniform(0.5, 1.5, (1, -(-N // gq))) * spread / 127).astype(np.float32)
    sk = (RNG.uniform(0.5, 1.5, (1, -(-N // gk))) * spread / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    return q8, k8, sq, sk, v


def _nblocks(N):
    return -(-N // 256), -(-N // 128)


# ---------------------------------------------------------------- attention over kept blocks
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("groups", [(1, 1), (128, 64)])
def test_all_kept_without_stage_two_is_the_dense_oracle(causal, groups):
    N, d = 600, 32
    q8, k8, sq, sk, v = _rand_quant(N, d, groups)
    nqb, nkb = _nblocks(N)
    mask = np.ones((1, nqb, nkb), np.uint8)
    o64, o16, skipped = oracle.attn_sparse(q8, k8, sq, sk, v, mask, causal, 0.2, INF, groups)
    d64, d16 = oracle.attn(q8, k8, sq, sk, v, causal, 0.2, groups)
    np.testing.assert_array_equal(o64, d64)
    np.testing.assert_array_equal(o16.view(np.uint16), d16.view(np.uint16))
    assert not skipped.any()


@pytest.mark.parametrize("causal", [False, True])
def test_dropped_blocks_are_textbook_attention_over_the_kept_keys(causal):
    N, d = 700, 16
    q8, k8, sq, sk, v = _rand_quant(N, d)
    nqb, nkb = _nblocks(N)
    mask = (RNG.random((1, nqb, nkb)) < 0.5).astype(np.uint8)
    for i in range(nqb):  # keep every query's own block, as stage 1 does when causal
        mask[0, i, min(nkb - 1, 2 * i):min(nkb, 2 * i + 2)] = 1
    o64, _, _ = oracle.attn_sparse(q8, k8, sq, sk, v, mask, causal, 0.3, INF)
    qf = q8[0] * sq[0][:, None].astype(np.float64)
    kf = k8[0] * sk[0][:, None].astype(np.float64)
    vf = v[0].astype(np.float64)
    s = qf @ kf.T * 0.3
    keep = mask[0][np.arange(N) // 256][:, np.arange(N) // 128].astype(bool)
    if causal:
        keep &= np.tril(np.ones((N, N), bool))
    s = np.where(keep, s, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (e / e.sum(axis=1, keepdims=True)) @ vf
    assert np.abs(o64[0] - ref).max() <= 2**-11 * np.abs(vf).max() * 1.001  # the fp16 P~ bound
    assert np.abs(o64[0] - oracle.attn(q8, k8, sq, sk, v, causal, 0.3)[0][0]).max() > 1e-3


# ---------------------------------------------------------------- stage 2
def _two_block_case(low_first: bool, gap_log2: float):
    # one query tile of 128 rows; key block 0 and 1 (256 keys).  Integer codes: every query is
    # [1, 0], block `hi` keys are [-20, 0], block `lo` keys [-70, 0]: scores differ by a fixed
    # amount per row, all keys within a block score alike, and every score is negative (so a
    # running maximum that started at 0 instead of -inf would skip a first block far below 0).
    N, d = 256, 2
    q8 = np.zeros((1, N, d), np.int8)
    q8[0, :, 0] = 1
    k8 = np.zeros((1, N, d), np.int8)
    hi, lo = (1, 0) if low_first else (0, 1)
    k8[0, hi * 128:(hi + 1) * 128, 0] = -20
    k8[0, lo * 128:(lo + 1) * 128, 0] = -20 - 50
    sq = np.ones((1, N), np.float32)
    sm = gap_log2 / 50 / math.log2(math.e)  # a 50-code gap is gap_log2 in log2 units
    sk = np.ones((1, N), np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    return q8, k8, sq, sk, v, sm, hi, lo


def test_stage_two_skips_a_block_far_below_the_running_maximum():
    q8, k8, sq, sk, v, sm, hi, lo = _two_block_case(low_first=False, gap_log2=30.0)
    mask = np.ones((1, 1, 2), np.uint8)
    o64, _, skipped = oracle.attn_sparse(q8, k8, sq, sk, v, mask, False, sm, 20.0)
    assert skipped[0, :, lo].all() and not skipped[0, :, hi].any()
    only_hi = mask.copy()
    only_hi[0, 0, lo] = 0
    ref, _, _ = oracle.attn_sparse(q8, k8, sq, sk, v, only_hi, False, sm, INF)
    np.testing.assert_array_equal(o64, ref)
    # a gap below lambda is not skipped
    _, _, skipped2 = oracle.attn_sparse(q8, k8, sq, sk, v, mask, False, sm, 40.0)
    assert not skipped2.any()


def test_stage_two_never_skips_the_first_block_and_uses_the_running_maximum():
    # the low block comes first: at that point the running maximum is its own, so it is kept;
    # the result is the full (dense) attention
    q8, k8, sq, sk, v, sm, hi, lo = _two_block_case(low_first=True, gap_log2=30.0)
    mask = np.ones((1, 1, 2), np.uint8)
    o64, _, skipped = oracle.attn_sparse(q8, k8, sq, sk, v, mask, False, sm, 20.0)
    assert not skipped.any()
    dense, _ = oracle.attn(q8, k8, sq, sk, v, False, sm)
    np.testing.assert_array_equal(o64, dense)


def test_stage_two_needs_every_row_of_the_tile():
    # one row of the tile scores the low block high: the tile keeps the block for all rows
    q8, k8, sq, sk, v, sm, hi, lo = _two_block_case(low_first=False, gap_log2=30.0)
    q8[0, 77, 0] = -1  # row 77 prefers the low block
    mask = np.ones((1, 1, 2), np.uint8)
    _, _, skipped = oracle.attn_sparse(q8, k8, sq, sk, v, mask, False, sm, 20.0)
    assert not skipped[0, 0].any()
    # rows of the second query tile decide for themselves (they are all [1, 0])
    assert skipped[0, 1, lo]


# ---------------------------------------------------------------- stage 1
def _numpy_predict(q, k, causal, sm_scale, tau, theta):
    """Re-derivation of the stage-1 reading in numpy for one head [N, d]."""
    N, d = q.shape
    qf, kf = q.astype(np.float64), k.astype(np.float64)
    nqb, nkb = _nblocks(N)

    def stats(x, b, size):
        blk = x[b * size:min(N, (b + 1) * size)]
        nrm = np.linalg.norm(blk, axis=1, keepdims=True)
        unit = np.divide(blk, nrm, out=np.zeros_like(blk), where=nrm > 0)
        return blk.mean(axis=0), float(np.sum(unit.sum(axis=0) ** 2) / blk.shape[0] ** 2)

    qs = [stats(qf, i, 256) for i in range(nqb)]
    ks = [stats(kf, j, 128) for j in range(nkb)]
    mask = np.zeros((nqb, nkb), np.uint8)
    for i in range(nqb):
        last_q = min(N, (i + 1) * 256) - 1
        nvis = last_q // 128 + 1 if causal else nkb
        s = np.array([qs[i][0] @ ks[j][0] * sm_scale for j in range(nvis)])
        p = np.exp(s - s.max())
        p /= p.sum()
        order = sorted(range(nvis), key=lambda j: (-p[j], j))
        cum = 0.0
        for j in order:
            if cum >= tau:
                break
            mask[i, j] = 1
            cum += p[j]
        for j in range(nvis):
            if qs[i][1] < theta or ks[j][1] < theta:
                mask[i, j] = 1
            if causal and (j + 1) * 128 > i * 256:
                mask[i, j] = 1
    return mask, np.array([x[1] for x in qs]), np.array([x[1] for x in ks])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau,theta", [(0.5, 0.0), (0.9, 0.02), (0.99, 0.5)])
def test_predicted_map_matches_a_numpy_rederivation(causal, tau, theta):
    N, d = 1500, 32
    # structured inputs: windows of 384 tokens share a direction, so the map is far from uniform
    base = RNG.standard_normal((4, d))
    win = np.arange(N) // 384
    q = fp16(RNG.standard_normal((1, N, d)) * 0.7 + 2 * base[win])
    k = fp16(RNG.standard_normal((1, N, d)) * 0.7 + 2 * base[win])
    mask, unsure, qsim, ksim = oracle.sparse_predict(q, k, causal, 1 / math.sqrt(d), tau, theta)
    ref, rq, rk = _numpy_predict(q[0], k[0], causal, 1 / math.sqrt(d), tau, theta)
    np.testing.assert_allclose(qsim[0], rq, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ksim[0], rk, rtol=1e-12, atol=1e-12)
    sure = unsure[0] == 0
    np.testing.assert_array_equal(mask[0][sure], ref[sure])
    assert 0 < mask.mean() < 1 or theta >= 0.5  # the case is neither empty nor trivially dense


def test_self_similarity_closed_forms():
    d = 8
    one = np.zeros((1, 256, d))
    one[0, :, 0] = 3.0                              # identical tokens: 1
    opp = np.zeros((1, 256, d))
    opp[0, ::2, 1], opp[0, 1::2, 1] = 1.0, -1.0    # opposite pairs: 0
    orth = np.zeros((1, 256, d))
    for t in range(256):
        orth[0, t, t % d] = 2.0                     # d orthogonal directions, 32 tokens each: 1/d
    zero = np.zeros((1, 256, d))                    # zero tokens count as cosine 0: 0
    for x, expect in ((one, 1.0), (opp, 0.0), (orth, 1.0 / d), (zero, 0.0)):
        _, _, qsim, ksim = oracle.sparse_predict(fp16(x), fp16(x), False, 0.3, 0.9, 0.0)
        assert abs(qsim[0, 0] - expect) < 1e-12 and abs(ksim[0, 0] - expect) < 1e-12


def test_predicted_map_limits():
    N, d = 1024, 16
    q = fp16(RNG.standard_normal((1, N, d)) + 3 * RNG.standard_normal((1, 1, d)))
    k = fp16(RNG.standard_normal((1, N, d)) + 3 * RNG.standard_normal((1, 1, d)))
    nqb, nkb = _nblocks(N)
    # theta above every similarity: every visible block is kept
    m, _, _, _ = oracle.sparse_predict(q, k, False, 0.25, 0.1, 1.5)
    assert m.all()
    m, _, _, _ = oracle.sparse_predict(q, k, True, 0.25, 0.1, 1.5)
    vis = np.array([[(j * 128 <= min(N, (i + 1) * 256) - 1) for j in range(nkb)] for i in range(nqb)])
    np.testing.assert_array_equal(m[0].astype(bool), vis)
    # theta 0 and a tiny tau: exactly the most probable block (non-causal)
    m, _, _, _ = oracle.sparse_predict(q, k, False, 0.25, 1e-9, 0.0)
    assert np.all(m.sum(axis=-1) == 1)
    # causal: never a block beyond the last query, always the diagonal ones
    m, _, _, _ = oracle.sparse_predict(q, k, True, 0.25, 1e-9, 0.0)
    assert not (m[0] & ~vis).any()
    for i in range(nqb):
        assert m[0, i, 2 * i] and (2 * i + 1 >= nkb or m[0, i, 2 * i + 1])


def test_sparse_method_on_a_windowed_workload_is_close_to_exact_attention():
    # with tau = 0.95 the kept blocks carry the attention of the windowed inputs
    from workloads import Workload, make_qkv
    w = Workload("sparse_pin", 1, 1, 2048, 64, False, True, window=512, align=10.0)
    q, k, v = make_qkv(w)
    mask, _, _, _ = oracle.sparse_predict(q, k, w.causal, w.sm_scale, 0.95, 0.3)
    assert mask.mean() < 0.5
    km = oracle.smooth_k(k)
    q8, sq = oracle.quant(q, 128)
    k8, sk = oracle.quant(k, 64, km)
    o64, _, _ = oracle.attn_sparse(q8, k8, sq, sk, v, mask, w.causal, w.sm_scale, 20.0, (128, 64))
    exact = oracle.attn_fp64(q, k, v, w.causal, w.sm_scale)
    assert oracle.metrics(o64, exact)["cos"] >= 0.99


def test_tiles_match_the_whole_head():
    N, d = 500, 16
    q8, k8, sq, sk, v = _rand_quant(N, d, (128, 64))
    nqb, nkb = _nblocks(N)
    mask = (RNG.random((1, nqb, nkb)) < 0.6).astype(np.uint8)
    mask[0, :, 0] = 1
    for causal in (False, True):
        if causal:
            for i in range(nqb):
                mask[0, i, min(nkb - 1, 2 * i):min(nkb, 2 * i + 2)] = 1
        o64, _, skipped = oracle.attn_sparse(q8, k8, sq, sk, v, mask, causal, 0.3, 6.0, (128, 64))
        tiles = np.array([3, 0, 2])
        t64, tsk = oracle.attn_sparse_tiles(q8[0], k8[0], sq[0], sk[0], v[0], mask[0], tiles, causal, 0.3, 6.0,
                                            (128, 64))
        for r, t in enumerate(tiles):
            n = min(128, N - 128 * t)
            np.testing.assert_array_equal(t64[r, :n], o64[0, 128 * t:128 * t + n])
            assert np.isnan(t64[r, n:]).all()
            np.testing.assert_array_equal(tsk[r], skipped[0, t])
