"""Pins of the oracle's microscaling FP4 variant (oracle/sage_oracle_sa3.c) against facts that
do not come from the oracle: the independent E2M1 type of ml_dtypes and E4M3 type of PyTorch,
brute-force nearest-value search, the format's extremes, hand-derived rows
(tests/golden/fp4_online_frames.json) and an error bound against textbook attention on the
dequantized inputs.

The variant follows the SageAttention3 entry (microscaling FP4 attention on FP4 tensor cores); its
open points are the readings written at the top of sage_oracle_sa3.c.
tests/test_oracle_mutations.py plants slips in that file and checks that this file fails on
each of them.
"""
import json
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import fp16

RNG = np.random.default_rng(4242)
E2M1 = ml_dtypes.float4_e2m1fn
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp4_online_frames.json")


def e4m3_torch(x) -> np.ndarray:
    """Round to E4M3 with PyTorch's float8_e4m3fn (round to nearest even), as values."""
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).double().numpy()


# ---------------------------------------------------------------- the E2M1 format
def test_decode_matches_ml_dtypes_e2m1():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(E2M1).astype(np.float64)
    np.testing.assert_array_equal(oracle.e2m1_decode(codes), ref)
    assert oracle.e2m1_decode(np.array([7, 1, 15], np.uint8)).tolist() == [6.0, 0.5, -6.0]


def test_encode_matches_ml_dtypes_e2m1():
    # ties (the seven midpoints), saturation, signed zeros and random values
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    x = np.concatenate([mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 10), [6.0, 6.5, 100.0, -7.0, 0.0, -0.0,
                                                                                     -0.1, 1e-30],
                        RNG.standard_normal(20000) * 3, RNG.uniform(-7, 7, 20000)]).astype(np.float32)
    ref = x.astype(E2M1).view(np.uint8)
    got = oracle.e2m1_encode(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_encode_is_the_nearest_value_ties_to_even():
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    x = np.concatenate([RNG.uniform(0, 6, 5000), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]])
    for xi, ci in zip(x.tolist(), oracle.e2m1_encode(x).tolist()):
        err = np.abs(grid - xi)
        cand = np.nonzero(err == err.min())[0]
        if cand.size > 1:
            cand = cand[cand % 2 == 0]
        assert ci == cand[0], (xi, ci)


# ---------------------------------------------------------------- one microscaled group
def test_microscale_worked_examples():
    # max 6.5: 6.5 / 6 = 1.0833 rounds to the E4M3 value 1.125 (code 0x39); 1 / 1.125 = 0.8889:
    # 0.889 -> 1 (code 2), 1.778 -> 2 (code 4), 2.667 -> 3 (code 5), -5.778 -> -6 (code 15)
    s8, c = oracle.fp4_microscale([1.0, 2.0, 3.0, -6.5])
    assert s8 == 0x39 and c.tolist() == [2, 4, 5, 15]
    # saturation: 6.9 / 6 = 1.15 rounds down to 1.125, and 6.9 / 1.125 = 6.13 saturates at 6;
    # 0.2 / 1.125 = 0.178 rounds to 0
    s8, c = oracle.fp4_microscale([6.9, 0.2])
    assert s8 == 0x39 and c.tolist() == [7, 0]
    # an all-zero group: scale 0, zero codes
    s8, c = oracle.fp4_microscale(np.zeros(16))
    assert s8 == 0 and not c.any()


def test_microscale_rule_and_error_bound():
    for _ in range(300):
        n = int(RNG.integers(1, 17))
        z = (RNG.standard_normal(n) * 10.0 ** RNG.uniform(-4, 3)).astype(np.float32)
        s8, c = oracle.fp4_microscale(z)
        gm = np.float32(np.abs(z).max())
        s = oracle.e4m3_decode(np.array([s8], np.uint8))[0]
        assert s == e4m3_torch(gm / np.float32(6.0))  # the scale is the E4M3 rounding of max/6
        zq = oracle.e2m1_decode(c) * s
        # every element within one scale unit (half the widest E2M1 step, 4 -> 6) of its value,
        # plus what a scale rounded below max/6 (by at most max/96 when normal, 2^-10 when
        # subnormal or zero) loses to saturation at 6
        bound = s + max(gm / 16.0, 6 * 2.0**-10)
        assert np.all(np.abs(zq - z.astype(np.float64)) <= bound + 1e-12), (z, zq, s)


# ---------------------------------------------------------------- Q and K
def _qk_input(N=300, d=64, outliers=True):
    x = RNG.standard_normal((1, 2, N, d)) * 2.0
    if outliers:
        x[..., 5] += 40.0
    return torch.from_numpy(x).half()


def test_quant_fp4_tile_scale_extremes_and_bound():
    x = _qk_input()
    codes, s8, g = oracle.quant_fp4(x)
    xb = x.double().numpy()
    B, H, N, d = xb.shape
    nt = -(-N // 128)
    assert g.shape == (B, H, nt) and s8.shape == (B, H, N, d // 16)
    for h in range(H):
        for t in range(nt):
            blk = xb[0, h, 128 * t:128 * t + 128]
            a = np.float32(np.abs(blk).max())
            assert g[0, h, t] == np.float32(a / np.float32(2688.0))  # fl32(a / 2688)
            # the tile's largest element: z = 2688 exactly or within an ulp, scale 448, code +-6
            i, c = np.unravel_index(np.abs(blk).argmax(), blk.shape)
            assert s8[0, h, 128 * t + i, c // 16] == 0x7E
            assert codes[0, h, 128 * t + i, c] & 7 == 7
    # dequantized values: within one group scale unit times the tile scale of the input
    sc = np.repeat(oracle.e4m3_decode(s8), 16, axis=-1)
    gt = np.repeat(g.astype(np.float64), 128, axis=-1)[..., :N, None]
    xq = oracle.e2m1_decode(codes) * sc * gt
    assert np.all(np.abs(xq - xb) <= sc * gt * 1.0 + 1e-9)
    assert np.abs(xq - xb).max() <= 0.2 * np.abs(xb).max()


def test_quant_fp4_smooths_k_by_its_mean():
    k = _qk_input(N=200, d=32)
    km = oracle.smooth_k(k)
    codes, s8, g = oracle.quant_fp4(k, km)
    sc = np.repeat(oracle.e4m3_decode(s8), 16, axis=-1)
    gt = np.repeat(g.astype(np.float64), 128, axis=-1)[..., :200, None]
    kq = oracle.e2m1_decode(codes) * sc * gt + km[..., None, :]
    kb = k.double().numpy()
    assert np.all(np.abs(kq - kb) <= sc * gt + 1e-6)
    # the outlier channel is gone after smoothing: the tile scale follows the spread, not the bias
    _, _, g_raw = oracle.quant_fp4(k)
    assert g.max() < 0.5 * g_raw.max()


# ---------------------------------------------------------------- V
def test_quant_v_fp4_channel_scale_groups_and_mean():
    v = _qk_input(N=150, d=32)
    codes, s8, gv, vm = oracle.quant_v_fp4(v, smooth=True)
    assert s8.shape == (1, 2, 10, 32) and gv.shape == (1, 2, 32)
    # the channel means are those of the FP8 variant's V smoothing (the same exact mean)
    _, _, vm8 = oracle.quant_v_fp8(v, smooth=True)
    np.testing.assert_array_equal(vm, vm8)
    vb = v.double().numpy()
    x = (v.float().numpy() - vm[..., None, :]).astype(np.float32)
    a = np.abs(x).max(axis=-2)
    np.testing.assert_array_equal(gv, (a / np.float32(2688.0)).astype(np.float32))
    for h in range(2):
        for c in range(32):
            t = int(np.abs(x[0, h, :, c]).argmax())
            assert s8[0, h, t // 16, c] == 0x7E and codes[0, h, t, c] & 7 == 7
    sc = np.repeat(oracle.e4m3_decode(s8), 16, axis=-2)[..., :150, :]
    vq = oracle.e2m1_decode(codes) * sc * gv[..., None, :] + vm[..., None, :]
    assert np.all(np.abs(vq - vb) <= sc * gv[..., None, :] + 1e-6)
    # without smoothing no mean is subtracted
    codes0, _, gv0, vm0 = oracle.quant_v_fp4(v, smooth=False)
    assert vm0 is None
    a0 = np.abs(v.float().numpy()).max(axis=-2)
    np.testing.assert_array_equal(gv0, (a0 / np.float32(2688.0)).astype(np.float32))


# ---------------------------------------------------------------- attention
def _golden_inputs(case):
    d = 16
    if case == "near_far":
        N = 17
        q4 = np.zeros((1, N, d), np.uint8); q4[0, 0, 0] = 2
        k4 = np.zeros((1, N, d), np.uint8); k4[0, 1:16, 0] = 15; k4[0, 16, 0] = 13  # -6, -3
        ks = np.full((1, N, 1), 0x38, np.uint8); ks[0, 1:16, 0] = 0x7E; ks[0, 16, 0] = 0x49  # 448, 4.5
        v4 = np.zeros((1, N, d), np.uint8); v4[0, 0, 0] = 2; v4[0, 16, 0] = 7
        vs = np.full((1, 2, d), 0x38, np.uint8); vs[0, 1, 0] = 0x7E
        gv = np.ones((1, d), np.float32); gv[0, 0] = 0.5
        vm = np.zeros((1, d), np.float32); vm[0, 0] = 0.25
    else:
        N = 144
        q4 = np.zeros((1, N, d), np.uint8); q4[0, 0, 0:2] = 2
        k4 = np.zeros((1, N, d), np.uint8); k4[0, 0, 0] = 15; k4[0, 0, 1] = 9  # -6, -0.5
        k4[0, 1:128, 0] = 15; k4[0, 129:, 0] = 15
        ks = np.full((1, N, 1), 0x7E, np.uint8); ks[0, 0, 0] = 0x45; ks[0, 128, 0] = 0x38  # 3.25
        v4 = np.zeros((1, N, d), np.uint8); v4[0, 0, 0] = 7; v4[0, 128, 0] = 2
        vs = np.full((1, 9, d), 0x38, np.uint8); vs[0, 0, 0] = 0x7E
        gv = np.ones((1, d), np.float32)
        vm = np.zeros((1, d), np.float32)
    qs = np.full((1, N, 1), 0x38, np.uint8)
    nt = -(-N // 128)
    gq = np.ones((1, nt), np.float32)
    gk = np.ones((1, nt), np.float32)
    return q4, qs, gq, k4, ks, gk, v4, vs, gv, vm


@pytest.mark.parametrize("case", ["near_far", "two_frames"])
def test_attention_hand_derived_rows(case):
    gold = {c["name"]: c for c in json.load(open(GOLDEN))["cases"]}[case]
    args = _golden_inputs(case)
    o64, o16, env, unsure = oracle.attn_fp4(*args, causal=False, sm_scale=math.log(2.0))
    assert abs(o64[0, 0, 0] - gold["o_row0_ch0"]) <= 1e-12 * max(1.0, abs(gold["o_row0_ch0"]))
    assert np.all(o64[0, 0, 1:] == 0.0)
    assert unsure[0, 0] == gold["unsure_row0"]
    assert env[0, 0, 0] == 0.0  # no decision of this row lies near a rounding midpoint
    # the rows function agrees
    r64, renv, run = oracle.attn_fp4_rows(*args, bh=0, rows=[0], causal=False, sm_scale=math.log(2.0))
    np.testing.assert_array_equal(r64[0], o64[0, 0])


def test_attention_within_the_fp4_bound_of_textbook_attention():
    """O against softmax attention on the dequantized Q^, K^, V^ (numpy, fp64): each P~ lies
    within s + max(gm/16, 6 * 2^-10) of p (test_microscale_rule_and_error_bound), and the
    scale s within (17/16) gm/6 + 2^-10, so |O - O_exact| <= sum_j (0.2396 gm_j + 7 * 2^-10)
    |v^_j| gv / l in the frame of the row's largest score (earlier frames only shrink the
    absolute terms)."""
    for causal in (False, True):
        N, d = 260, 32
        q = torch.from_numpy(RNG.standard_normal((1, 1, N, d)) * 1.5).half()
        k = torch.from_numpy(RNG.standard_normal((1, 1, N, d))).half()
        v = torch.from_numpy(RNG.standard_normal((1, 1, N, d))).half()
        sm = d ** -0.5
        r = oracle.sage_attn_fp4(q, k, v, causal, sm)
        qs = np.repeat(oracle.e4m3_decode(r["qs"]), 16, axis=-1)
        ks = np.repeat(oracle.e4m3_decode(r["ks"]), 16, axis=-1)
        gqt = np.repeat(r["gq"].astype(np.float64), 128, axis=-1)[..., :N, None]
        gkt = np.repeat(r["gk"].astype(np.float64), 128, axis=-1)[..., :N, None]
        qh = (oracle.e2m1_decode(r["q4"]) * qs * gqt)[0, 0]
        kh = (oracle.e2m1_decode(r["k4"]) * ks * gkt)[0, 0]
        vs = np.repeat(oracle.e4m3_decode(r["vs"]), 16, axis=-2)[..., :N, :]
        vh = (oracle.e2m1_decode(r["v4"]) * vs)[0, 0]  # without gv
        gv = r["gv"][0, 0].astype(np.float64)
        u = qh @ kh.T * sm / math.log(2.0)
        if causal:
            u = np.where(np.arange(N)[None, :] <= np.arange(N)[:, None], u, -np.inf)
        M = np.ceil(u.max(axis=1, keepdims=True))
        p = np.exp2(u - M + 10.0)
        l = p.sum(axis=1, keepdims=True)
        exact = (p @ vh) / l * gv + r["vm"][0, 0]
        ng = -(-N // 16)
        pg = np.zeros((N, ng * 16))
        pg[:, :N] = p
        gm = pg.reshape(N, ng, 16).max(axis=2)
        per_key = np.repeat(gm * (17.0 / 96.0 + 1.0 / 16.0) + 7 * 2.0**-10, 16, axis=1)[:, :N]
        if causal:
            per_key = np.where(np.arange(N)[None, :] <= np.arange(N)[:, None], per_key, 0.0)
        bound = per_key @ np.abs(vh) / l * gv
        err = np.abs(r["o64"][0, 0] - exact)
        assert np.all(err <= bound + 1e-12), float((err - bound).max())
        assert oracle.metrics(r["o64"][0, 0], exact)["cos"] > 0.98
        assert np.array_equal(r["o16"][0, 0], fp16(r["o64"][0, 0]))


def test_envelope_counts_keys_near_a_midpoint():
    """Key 0 scores -0.375 (codes -0.5 at scale 0.75): m = 0, p0 = 2^9.625 = 789.7, whose
    max/6 = 131.6 rounds to the E4M3 value 128.  Key 1 scores -5 (code -4 at scale 1.25):
    p1 = 2^5 = 32 and 32/128 = 0.25, exactly the midpoint between the E2M1 values 0 and 0.5
    (ties to even: 0).  Its envelope is one E2M1 step (at most 2) times the scale:
    2 * 128 * |v^1| / l.  At score -4 (code -4 at scale 1.0) p1 = 64, 64/128 = 0.5 is a code
    and the envelope is 0."""
    d, N = 16, 2

    def run(k1_code, k1_scale):
        q4 = np.zeros((1, N, d), np.uint8); q4[0, :, 0] = 2
        k4 = np.zeros((1, N, d), np.uint8); k4[0, 0, 0] = 9; k4[0, 1, 0] = k1_code
        ks = np.full((1, N, 1), 0x34, np.uint8); ks[0, 1, 0] = k1_scale  # 0.75
        v4 = np.zeros((1, N, d), np.uint8); v4[0, :, 0] = 2
        vs = np.full((1, 1, d), 0x38, np.uint8)
        ones = np.ones((1, 1), np.float32)
        return oracle.attn_fp4(q4, np.full((1, N, 1), 0x38, np.uint8), ones, k4, ks, ones, v4, vs,
                               np.ones((1, d), np.float32), None, False, math.log(2.0))
    p0 = 2.0 ** 9.625
    o64, _, env, unsure = run(14, 0x3A)  # -4 * 1.25 = -5
    l = p0 + 32.0
    assert abs(env[0, 0, 0] - 2 * 128 / l) <= 1e-12
    assert abs(o64[0, 0, 0] - 768.0 / l) <= 1e-12  # P~0 = e2m1(789.7/128 = 6.17 -> 6) * 128, P~1 = 0
    assert unsure[0, 0] == 0
    o64, _, env, _ = run(14, 0x38)  # -4 * 1.0 = -4
    assert env[0, 0, 0] == 0.0
    assert abs(o64[0, 0, 0] - (768.0 + 64.0) / (p0 + 64.0)) <= 1e-12
