"""Pins of the oracle's FP8 P.V variant (oracle/sage_oracle_sa2.c) against facts that do not
come from the oracle: PyTorch's independent E4M3 type, brute-force nearest-value search,
exact rational arithmetic, hand-derived two-key cases (tests/golden/fp8_pv_two_keys.json),
an error bound against textbook attention, and the V-shift invariance of smoothing.

The variant follows the SageAttention2 abstract ((P~, V) quantized to FP8, V smoothed, P~V
accumulated in an FP32 buffer); its open points are the readings written at the top of
sage_oracle_sa2.c.  tests/test_oracle_mutations.py plants slips in that file and checks that
this file fails on each of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import exact_attention, fp16, round_to_f32_exact

RNG = np.random.default_rng(99)
ALL_CODES = np.arange(256, dtype=np.uint8)


def torch_e4m3_values() -> np.ndarray:
    """Value of every E4M3 code according to PyTorch's float8_e4m3fn type."""
    return torch.from_numpy(ALL_CODES.copy()).view(torch.float8_e4m3fn).double().numpy()


# ---------------------------------------------------------------- the E4M3 format
def test_decode_matches_torch_float8_e4m3fn():
    mine = oracle.e4m3_decode(ALL_CODES)
    ref = torch_e4m3_values()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2  # 0x7F and 0xFF
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0**-9


def test_encode_is_nearest_with_ties_to_even_and_saturates():
    vals = torch_e4m3_values()
    finite = ~np.isnan(vals)
    codes, grid = ALL_CODES[finite], vals[finite]
    x = np.concatenate([RNG.standard_normal(20000) * 30, RNG.standard_normal(5000) * 0.01,
                        (RNG.integers(-900, 900, 4000) + 0.5) / 2.0 ** RNG.integers(-3, 9, 4000),
                        np.array([447.9, 448.0, 463.9, 464.0, 465.0, 1e6, -1e6, 2.0**-10, 3 * 2.0**-11,
                                  -(2.0**-10), 0.0])])
    got = oracle.e4m3_encode(x)
    for xi, ci in zip(x.tolist(), got.tolist()):
        if abs(xi) >= 448.0:  # saturation
            assert oracle.e4m3_decode(np.array([ci], np.uint8))[0] == math.copysign(448.0, xi)
            continue
        err = np.abs(grid - xi)
        best = err.min()
        cand = codes[err == best]
        if cand.size > 1:  # a tie between two grid values: the even mantissa wins
            cand = cand[(cand & 1) == 0]
            cand = cand[(cand & 0x80) == (0x80 if math.copysign(1.0, xi) < 0 else 0)] if cand.size > 1 else cand
        assert ci in cand.tolist(), (xi, ci, cand)
    inr = np.abs(x) < 448
    t = torch.from_numpy(x[inr]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    nz = x[inr] != 0  # torch keeps -0.0 as 0x80 too; compare the nonzero values bit for bit
    np.testing.assert_array_equal(got[inr][nz], t[nz])


# ---------------------------------------------------------------- V to FP8
def test_quant_v_fp8_mean_scales_and_codes():
    BH, N, d = 2, 256, 16
    v = fp16(RNG.standard_normal((BH, N, d)) * np.exp(RNG.standard_normal((1, 1, d))) + RNG.standard_normal((BH, 1, d)) * 5)
    v8, sv, vm = oracle.quant_v_fp8(v)
    vf = v.astype(np.float64)
    for h in range(BH):
        for c in range(d):
            exact = sum(Fraction(x) for x in vf[h, :, c].tolist()) / N  # N a power of two
            assert vm[h, c] == round_to_f32_exact(exact)
            x = v[h, :, c].astype(np.float32) - vm[h, c]  # fl32(V - vm)
            a = np.abs(x).max()
            assert sv[h, c] == round_to_f32_exact(Fraction(float(a)) / 448)
            inv = round_to_f32_exact(Fraction(448) / Fraction(float(a)))
            y = (x * inv).astype(np.float64)  # fl32(x * inv)
            np.testing.assert_array_equal(v8[h, :, c], oracle.e4m3_encode(y))
            dec = oracle.e4m3_decode(v8[h, :, c])
            assert np.abs(dec).max() == 448.0  # the channel's absmax maps to +-448
            # round trip: within half an E4M3 step (relative 2^-4) or 2^-10 of a unit in the subnormals
            err = np.abs(dec * float(sv[h, c]) - x.astype(np.float64))
            assert np.all(err <= (2.0**-4 * np.abs(x) + 2.0**-10 * float(sv[h, c])) * (1 + 2.0**-20))


def test_quant_v_fp8_without_smoothing_and_zero_channel():
    v = fp16(RNG.standard_normal((1, 64, 8)))
    v[0, :, 3] = 0
    v8, sv, vm = oracle.quant_v_fp8(v, smooth=False)
    assert vm is None and sv[0, 3] == 0 and np.all(v8[0, :, 3] == 0)
    a = np.abs(v[0].astype(np.float32)).max(axis=0)
    for c in (0, 1, 7):
        assert sv[0, c] == round_to_f32_exact(Fraction(float(a[c])) / 448)


def test_v_shift_moves_the_output_by_the_shift():
    # With V smoothed, adding a per-channel constant to V (exact in fp16) leaves the codes and
    # scales unchanged and moves O by exactly that constant (the mean is added back).
    BH, N, d = 1, 128, 16
    q8 = RNG.integers(-127, 128, (BH, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (BH, N, d), dtype=np.int8)
    s = (RNG.uniform(0.5, 1.5, (BH, N)) / 127).astype(np.float32)
    v = fp16(np.round(RNG.standard_normal((BH, N, d)) * 64) / 64)
    shift = np.round(RNG.standard_normal((BH, 1, d)) * 8)
    v2 = fp16(v.astype(np.float64) + shift)
    assert np.array_equal(v2.astype(np.float64), v.astype(np.float64) + shift)
    a8, asv, avm = oracle.quant_v_fp8(v)
    b8, bsv, bvm = oracle.quant_v_fp8(v2)
    np.testing.assert_array_equal(a8, b8)
    np.testing.assert_array_equal(asv, bsv)
    np.testing.assert_array_equal(bvm.astype(np.float64), avm.astype(np.float64) + shift[:, 0])
    for causal in (False, True):
        oa, _ = oracle.attn_fp8pv(q8, k8, s, s, a8, asv, avm, causal, 0.3)
        ob, _ = oracle.attn_fp8pv(q8, k8, s, s, b8, bsv, bvm, causal, 0.3)
        np.testing.assert_allclose(ob, oa + shift, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- attention with FP8 P~ and V
def test_fp8_two_keys_hand_derived():
    path = os.path.join(os.path.dirname(__file__), "golden", "fp8_pv_two_keys.json")
    with open(path) as f:
        cases = json.load(f)["cases"]
    q8 = np.ones((1, 2, 1), np.int8)
    k8 = np.ones((1, 2, 1), np.int8)
    sq = np.ones((1, 2), np.float32)
    v = fp16(np.array([[[0.0], [1.0]]]))
    v8, sv, _ = oracle.quant_v_fp8(v, smooth=False)
    assert v8.ravel().tolist() == [0, 0x7E] and sv[0, 0] == np.float32(1) / np.float32(448)
    for c in cases:
        sk = np.array([[float.fromhex(h) for h in c["sk_hex"]]], np.float32)
        u = [float(x) * math.log2(math.e) for x in sk[0]]
        M = math.ceil(max(u))
        p = [2.0 ** (x - M + 8) for x in u]
        pt0, pt1 = c["p_tilde_hand"]
        expect = pt1 * 448 * float(sv[0, 0]) / (p[0] + p[1])  # P~_0 multiplies V_0 = 0
        o64, _ = oracle.attn_fp8pv(q8, k8, sq, sk, v8, sv, None, False, 1.0)
        for i in range(2):
            assert abs(o64[0, i, 0] - expect) <= 1e-15, (c["name"], o64[0, i, 0], expect)
        # the hand-rounded weights are E4M3 values of the unrounded ones
        assert oracle.e4m3_decode(oracle.e4m3_encode(np.array(p))).tolist() == [pt0, pt1]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("groups", [(1, 1), (128, 64)])
def test_fp8_attention_within_the_p_rounding_bound(causal, groups):
    # Against textbook attention of the dequantized operands (q8 sq, k8 sk, dec(v8) sv + vm),
    # only the E4M3 rounding of P~ differs: each weight moves by at most 2^-4 of itself (normal
    # range) or 2^-10 (subnormal range, with the row's largest weight above 2^7).
    N, d = 300, 32
    gq, gk = groups
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    sq = (RNG.uniform(0.5, 1.5, (1, -(-N // gq))) * 3 / 127).astype(np.float32)
    sk = (RNG.uniform(0.5, 1.5, (1, -(-N // gk))) * 3 / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)) + 2)
    v8, sv, vm = oracle.quant_v_fp8(v)
    sm = 1 / math.sqrt(d)
    o64, o16 = oracle.attn_fp8pv(q8, k8, sq, sk, v8, sv, vm, causal, sm, groups)
    qf = q8[0] * np.repeat(sq[0].astype(np.float64), gq)[:N, None]
    kf = k8[0] * np.repeat(sk[0].astype(np.float64), gk)[:N, None]
    vc = oracle.e4m3_decode(v8[0]) * sv[0].astype(np.float64)  # dequantized V - vm
    ref = exact_attention(qf, kf, vc, causal, sm) + vm[0].astype(np.float64)
    bound = (2.0**-4 + N * 2.0**-10 / 2.0**7) * np.abs(vc).max(axis=0)
    assert np.all(np.abs(o64[0] - ref) <= bound * 1.001)
    assert np.array_equal(o16.view(np.uint16), fp16(o64).view(np.uint16))
    # and the rounding is really there (a bound that unrounded weights would also meet)
    assert np.abs(o64[0] - ref).max() > 1e-6 * np.abs(vc).max()


def test_fp8_causal_first_row():
    # Row 0 sees key 0 only: its weight is 2^(u0 - ceil(u0) + 8), rounded to E4M3, over itself.
    N, d = 64, 16
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    s = (RNG.uniform(0.5, 1.5, (1, N)) / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    v8, sv, vm = oracle.quant_v_fp8(v)
    o64, _ = oracle.attn_fp8pv(q8, k8, s, s, v8, sv, vm, True, 0.125)
    u0 = float(np.dot(q8[0, 0].astype(np.int64), k8[0, 0].astype(np.int64))) * float(s[0, 0]) * float(s[0, 0]) \
        * 0.125 * math.log2(math.e)
    p0 = 2.0 ** (u0 - math.ceil(u0) + 8)
    pt0 = oracle.e4m3_decode(oracle.e4m3_encode(np.array([p0])))[0]
    expect = pt0 / p0 * oracle.e4m3_decode(v8[0, 0]) * sv[0].astype(np.float64) + vm[0].astype(np.float64)
    np.testing.assert_allclose(o64[0, 0], expect, rtol=1e-13, atol=1e-13)


def test_fp8_rows_match_full_attention():
    N, d = 200, 16
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    sq = (RNG.uniform(0.5, 1.5, (1, 2)) / 127).astype(np.float32)
    sk = (RNG.uniform(0.5, 1.5, (1, 4)) / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    v8, sv, vm = oracle.quant_v_fp8(v)
    o64, _ = oracle.attn_fp8pv(q8, k8, sq, sk, v8, sv, vm, True, 0.2, (128, 64))
    rows = np.array([0, 5, 127, 128, 199])
    r64 = oracle.attn_fp8pv_rows(q8[0], k8[0], sq[0], sk[0], v8[0], sv[0], vm[0], rows, True, 0.2, (128, 64))
    np.testing.assert_array_equal(r64, o64[0, rows])


def test_fp8_method_quality_on_the_outlier_workload():
    # the FP8 variant stays close to exact attention on the tiny K-outlier workload
    from workloads import TINY, make_qkv
    q, k, v = make_qkv(TINY)
    exact = oracle.attn_fp64(q, k, v, TINY.causal, TINY.sm_scale)
    r = oracle.sage_attn_fp8pv(q, k, v, TINY.causal, TINY.sm_scale, per_block=False)
    assert oracle.metrics(r["o64"], exact)["cos"] >= 0.99
