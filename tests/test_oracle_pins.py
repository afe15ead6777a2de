"""Pins of the CPU oracle against facts that do not come from the oracle itself.

The page ("SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
Acceleration", research.elamur.ai summary) prints no worked example, so every
pin here is a closed form, an invariant the page states (idea I1: removing a
component shared by all tokens of K leaves the softmax unchanged), a special
case that reduces to textbook attention / exact integer arithmetic, an error
bound, or brute force on tiny inputs.  Each is chosen so that a plausible slip
in the oracle (dropped term, wrong sign, swapped index, transposed operand,
wrong group boundary, wrong rounding) fails at least one test;
tests/test_oracle_mutations.py plants such slips in copies of the oracle and
checks that this file fails on every one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from workloads import TINY, make_qkv

RNG = np.random.default_rng(1234)


def exact_attention(qf, kf, vf, causal, sm_scale):
    """Textbook softmax(q k^T * scale) v in fp64 for one head (numpy)."""
    s = (qf @ kf.T) * sm_scale
    if causal:
        n = s.shape[0]
        s = np.where(np.tril(np.ones((n, n), bool)), s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ vf


def fp16(x):
    return np.asarray(x, np.float64).astype(np.float16)


def round_to_f32_exact(fr: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 of an exact rational,
    found by comparing neighbouring fp32 candidates exactly."""
    c = np.float32(float(fr))
    best = None
    for cand in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        err = abs(Fraction(float(cand)) - fr)
        key = (err, int(np.frombuffer(np.float32(cand).tobytes(), np.uint32)[0]) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return np.float32(best[1])


# ---------------------------------------------------------------- fp16 rounding
def test_round_fp16_matches_numpy_direct_conversion():
    x = np.concatenate([
        RNG.standard_normal(20000) * 10,
        RNG.standard_normal(2000) * 1e-6,  # subnormal range of fp16
        np.array([1 + 2**-11, 1 + 3 * 2**-11, 2**-24 * 0.5, 65504.0, 65519.99, -0.0, 1e-30]),
    ])
    got = oracle.round_fp16(x)
    ref = x.astype(np.float16)  # numpy rounds fp64 -> fp16 directly
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


# ---------------------------------------------------------------- K smoothing
def test_smooth_k_power_of_two_n_is_correctly_rounded_mean():
    BH, N, d = 3, 256, 16
    k = fp16(RNG.standard_normal((BH, N, d)) * 3 + RNG.standard_normal((BH, 1, d)) * 20)
    km = oracle.smooth_k(k)
    for h in range(BH):
        for c in range(d):
            exact = sum(Fraction(float(x)) for x in k[h, :, c].astype(np.float64)) / N
            assert km[h, c] == round_to_f32_exact(exact), (h, c)


def test_smooth_k_general_n_within_two_ulps_of_exact_mean():
    BH, N, d = 2, 1000, 8
    k = fp16(RNG.standard_normal((BH, N, d)) + 5)
    km = oracle.smooth_k(k)
    exact = k.astype(np.float64).mean(axis=1)
    ulp = np.spacing(np.abs(km).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(km - exact) <= 2 * ulp)


def test_smooth_k_shift_by_token_constant_gives_same_codes():
    # K on a coarse grid and an integer per-channel shift keep every value exact
    # in fp16, so the smoothed K -- and its INT8 codes -- must not change.
    BH, N, d = 2, 128, 32
    k = fp16(np.round(RNG.standard_normal((BH, N, d)) * 8) / 8)
    shift = np.round(RNG.standard_normal((BH, 1, d)) * 10)
    k2 = fp16(k.astype(np.float64) + shift)
    assert np.array_equal(k2.astype(np.float64), k.astype(np.float64) + shift)
    km, km2 = oracle.smooth_k(k), oracle.smooth_k(k2)
    np.testing.assert_array_equal(km2.astype(np.float64), km.astype(np.float64) + shift[:, 0, :])
    for g in (1, 64):
        q1, s1 = oracle.quant(k, g, km)
        q2, s2 = oracle.quant(k2, g, km2)
        np.testing.assert_array_equal(q1, q2)
        np.testing.assert_array_equal(s1, s2)


def test_smoothed_k_has_zero_channel_mean():
    BH, N, d = 2, 512, 16
    k = fp16(RNG.standard_normal((BH, N, d)) + RNG.standard_normal((BH, 1, d)) * 30)
    km = oracle.smooth_k(k)
    centred = k.astype(np.float64) - km[:, None, :].astype(np.float64)
    assert np.abs(centred.mean(axis=1)).max() < 1e-5


# ---------------------------------------------------------------- quantization
@pytest.mark.parametrize("g", [1, 64, 128, 100])
def test_quant_group_properties(g):
    BH, N, d = 2, 300, 24  # ragged last group for g = 64, 128, 100
    x = fp16(RNG.standard_normal((BH, N, d)) * np.exp(RNG.standard_normal((BH, N, 1))))
    q, s = oracle.quant(x, g)
    assert s.shape == (BH, -(-N // g))
    xf = x.astype(np.float64)
    for h in range(BH):
        for gi in range(s.shape[1]):
            blk = slice(gi * g, min(N, (gi + 1) * g))
            a = np.abs(xf[h, blk]).max()
            qs = q[h, blk].astype(np.int64)
            # the group's absmax maps to +-127 and nothing exceeds it
            assert np.abs(qs).max() == 127
            # the scale is absmax / 127 to fp32 accuracy
            assert abs(float(s[h, gi]) - a / 127) <= 2**-23 * a / 127
            # round trip: every value is within half a step of its code, plus the
            # fp32 rounding of x * (127 / a) (three roundings of 2^-24 on codes
            # of magnitude <= 127, i.e. below 2^-15 of a step)
            err = np.abs(xf[h, blk] - qs * float(s[h, gi]))
            assert err.max() <= float(s[h, gi]) * (0.5 + 2**-15)


def test_quant_scale_and_inverse_are_single_fp32_roundings():
    # The reading of "quantized to INT8" (Summary bullet 1): s = fl32(a / 127) and
    # inv = fl32(127 / a), each ONE correctly rounded fp32 division.  Checked against exact
    # rational arithmetic over every positive finite fp16 absmax (Q groups) and a spread of
    # fp32 absmax values (smoothed K groups); the set includes values where the tempting
    # shortcuts a * fl32(1/127) and 1 / fl32(a / 127) round differently, so they would fail.
    a16 = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    a32 = (np.exp(RNG.uniform(-20, 12, 3000)) * RNG.uniform(1, 2, 3000)).astype(np.float32)
    a = np.concatenate([a16, a32, np.array([0.0], np.float32)])
    s, inv = oracle.quant_scale(a)
    assert s[-1] == 0 and inv[-1] == 0
    a, s, inv = a[:-1], s[:-1], inv[:-1]
    with np.errstate(over="ignore"):
        shortcut_s = a * np.float32(1 / 127)
        shortcut_inv = np.float32(1) / (a / np.float32(127))
    assert np.count_nonzero(shortcut_s != s) > 100 and np.count_nonzero(shortcut_inv != inv) > 100
    for ai, si, ii in zip(a.tolist(), s.tolist(), inv.tolist()):
        fa = Fraction(ai)
        assert np.float32(si) == round_to_f32_exact(fa / 127), ai
        assert np.float32(ii) == round_to_f32_exact(Fraction(127) / fa), ai


@pytest.mark.parametrize("g", [1, 64])
def test_quant_codes_are_rounded_products_with_the_inverse(g):
    # code = round_half_even(fl32(x * inv)) with inv the group's fl32(127 / a)
    BH, N, d = 2, 192, 16
    x = fp16(RNG.standard_normal((BH, N, d)) * 3)
    q, s = oracle.quant(x, g)
    xf = x.astype(np.float32)
    for h in range(BH):
        for gi in range(s.shape[1]):
            blk = slice(gi * g, min(N, (gi + 1) * g))
            a = np.abs(xf[h, blk]).max()
            s_ref, inv = oracle.quant_scale(np.array([a], np.float32))
            assert s[h, gi] == s_ref[0]
            y = xf[h, blk] * inv[0]  # fp32 product, rounded once
            np.testing.assert_array_equal(q[h, blk], np.rint(y).astype(np.int8))


def test_quant_integer_grid_is_identity_and_rounds_half_to_even():
    # A group whose absmax is exactly 127 has scale 1, so integer values map to
    # themselves and halves round to the even neighbour.
    vals = np.array([127.0, -127.0, 0.0, 3.0, -5.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, 126.5])
    x = np.zeros((1, 1, vals.size))
    x[0, 0] = vals
    q, s = oracle.quant(fp16(x), 1)
    assert s[0, 0] == 1.0
    assert q[0, 0].tolist() == [127, -127, 0, 3, -5, 2, 4, -2, -4, 0, 2, 126]


def test_quant_zero_group_has_zero_scale_and_codes():
    x = np.zeros((1, 128, 8))
    x[0, 64:] = 1.0
    q, s = oracle.quant(fp16(x), 64)
    assert s[0, 0] == 0.0 and not np.isnan(s).any()
    assert np.all(q[0, :64] == 0) and np.all(q[0, 64:] == 127)


def test_quant_subtracts_channel_mean_not_token_mean():
    # Channel c holds the constant c + noise on every token; after subtracting
    # the channel means only the noise is left, so codes match quantizing the
    # noise alone (noise and offsets chosen exact in fp16 and fp32).
    BH, N, d = 1, 64, 8
    noise = np.round(RNG.standard_normal((BH, N, d)) * 4) / 4
    noise -= noise.mean(axis=1, keepdims=True)
    noise = np.round(noise * 64) / 64
    off = np.arange(d, dtype=np.float64)[None, None, :] * 3
    mu = (off[:, 0, :] + noise.mean(axis=1)).astype(np.float32)
    x = fp16(noise + off)
    q1, s1 = oracle.quant(x, 64, mu)
    resid = x.astype(np.float32) - mu[:, None, :]
    q2, s2 = oracle.quant(fp16(resid), 64)
    assert np.array_equal(fp16(resid).astype(np.float32), resid)
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(s1, s2)


# ---------------------------------------------------------------- integer QK^T
def test_qk_int_matches_brute_force_and_int64_matmul():
    BH, N, d = 2, 12, 8
    q8 = RNG.integers(-127, 128, (BH, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (BH, N, d), dtype=np.int8)
    S = oracle.qk_int(q8, k8)
    for h in range(BH):
        for i in range(N):
            for j in range(N):
                assert S[h, i, j] == sum(int(q8[h, i, c]) * int(k8[h, j, c]) for c in range(d))
    q8b = RNG.integers(-127, 128, (1, 96, 128), dtype=np.int8)
    k8b = RNG.integers(-127, 128, (1, 96, 128), dtype=np.int8)
    ref = q8b[0].astype(np.int64) @ k8b[0].astype(np.int64).T
    np.testing.assert_array_equal(oracle.qk_int(q8b, k8b)[0], ref)


def test_qk_int_rows_matches_full_product():
    q8 = RNG.integers(-127, 128, (1, 40, 16), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, 40, 16), dtype=np.int8)
    rows = np.array([0, 7, 39])
    np.testing.assert_array_equal(oracle.qk_int_rows(q8[0], k8[0], rows), oracle.qk_int(q8, k8)[0, rows])


def test_qk_int_extreme_values_fit():
    q8 = np.full((1, 4, 128), 127, np.int8)
    k8 = np.full((1, 4, 128), -127, np.int8)
    assert np.all(oracle.qk_int(q8, k8) == -127 * 127 * 128)


# ---------------------------------------------------------------- attention
def _dequant_attention_bound_check(N, d, causal, groups, scale_spread):
    gq, gk = groups
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    sq = (RNG.uniform(0.5, 1.5, (1, -(-N // gq))) * scale_spread / 127).astype(np.float32)
    sk = (RNG.uniform(0.5, 1.5, (1, -(-N // gk))) * scale_spread / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    sm_scale = 1 / math.sqrt(d)
    o64, o16 = oracle.attn(q8, k8, sq, sk, v, causal, sm_scale, groups)
    qf = q8[0].astype(np.float64) * np.repeat(sq[0].astype(np.float64), gq)[:N, None]
    kf = k8[0].astype(np.float64) * np.repeat(sk[0].astype(np.float64), gk)[:N, None]
    ref = exact_attention(qf, kf, v[0].astype(np.float64), causal, sm_scale)
    vmax = np.abs(v.astype(np.float64)).max()
    # only P~ is rounded (relative 2^-11 per weight): |O - exact| <= 2^-11 max|V|
    assert np.abs(o64[0] - ref).max() <= 2**-11 * vmax * 1.001
    # fp16 output is the fp16 rounding of the fp64 output
    assert np.array_equal(o16.view(np.uint16), fp16(o64).view(np.uint16))
    return o64


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("groups", [(1, 1), (128, 64), (16, 8)])
def test_attn_is_dequantized_attention_within_fp16_p_bound(causal, groups):
    _dequant_attention_bound_check(200, 32, causal, groups, scale_spread=3.0)


def test_attn_large_scores_still_within_bound():
    _dequant_attention_bound_check(96, 64, False, (1, 1), scale_spread=40.0)


def test_attn_zero_queries_give_prefix_means():
    # all scores 0 -> every weight 1 (exact in fp16): O_i is the mean of V over
    # the visible keys -- all keys, or keys 0..i when causal.
    N, d = 50, 8
    q8 = np.zeros((1, N, d), np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    s = np.ones((1, N), np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    vf = v[0].astype(np.float64)
    o64, _ = oracle.attn(q8, k8, s, s, v, False, 0.3)
    np.testing.assert_allclose(o64[0], np.broadcast_to(vf.mean(axis=0), (N, d)), rtol=0, atol=1e-14)
    o64c, _ = oracle.attn(q8, k8, s, s, v, True, 0.3)
    prefix = np.cumsum(vf, axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(o64c[0], prefix, rtol=0, atol=1e-14)


def test_attn_causal_first_row_is_first_value_row():
    N, d = 64, 16
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    s = (RNG.uniform(0.5, 1.5, (1, N)) / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    _, o16 = oracle.attn(q8, k8, s, s, v, True, 0.125)
    assert np.array_equal(o16[0, 0].view(np.uint16), v[0, 0].view(np.uint16))


def test_attn_causal_rows_ignore_later_keys():
    N, d = 40, 8
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    s = (RNG.uniform(0.5, 1.5, (1, N)) / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    o_a, _ = oracle.attn(q8, k8, s, s, v, True, 0.2)
    k8b, vb = k8.copy(), v.copy()
    k8b[0, 25:] = RNG.integers(-127, 128, (N - 25, d), dtype=np.int8)
    vb[0, 25:] = fp16(RNG.standard_normal((N - 25, d)))
    o_b, _ = oracle.attn(q8, k8b, s, s, vb, True, 0.2)
    np.testing.assert_array_equal(o_a[0, :25], o_b[0, :25])
    assert np.abs(o_a[0, 25:] - o_b[0, 25:]).max() > 1e-3


@pytest.mark.parametrize("causal", [False, True])
def test_attn_probability_rows_sum_to_one(causal):
    N, d = 70, 16
    q8 = RNG.integers(-127, 128, (N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (N, d), dtype=np.int8)
    s = (RNG.uniform(0.5, 1.5, (N,)) * 4 / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((N, d)))
    P = oracle.attn_probs(q8, k8, s, s, v, causal, 0.25)
    assert np.abs(P.sum(axis=1) - 1).max() <= 1e-12
    assert np.all(P >= 0)
    if causal:
        assert np.all(P[np.triu_indices(N, 1)] == 0)


def test_attn_rows_matches_full_attention():
    N, d = 300, 32
    q8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    k8 = RNG.integers(-127, 128, (1, N, d), dtype=np.int8)
    sq = (RNG.uniform(0.5, 1.5, (1, 3)) / 127).astype(np.float32)
    sk = (RNG.uniform(0.5, 1.5, (1, 5)) / 127).astype(np.float32)
    v = fp16(RNG.standard_normal((1, N, d)))
    o64, o16 = oracle.attn(q8, k8, sq, sk, v, True, 0.2, (128, 64))
    rows = np.array([0, 1, 127, 128, 299])
    r64, r16 = oracle.attn_rows(q8[0], k8[0], sq[0], sk[0], v[0], rows, True, 0.2, (128, 64))
    np.testing.assert_array_equal(r64, o64[0, rows])
    np.testing.assert_array_equal(r16.view(np.uint16), o16[0, rows].view(np.uint16))


# ---------------------------------------------------------------- fp64 attention
def test_attn_fp64_matches_textbook_and_is_shift_invariant():
    # idea I1: adding one vector to every key leaves each softmax row unchanged
    BH, N, d = 2, 48, 16
    q = fp16(RNG.standard_normal((BH, N, d)))
    k = fp16(np.round(RNG.standard_normal((BH, N, d)) * 16) / 16)
    v = fp16(RNG.standard_normal((BH, N, d)))
    shift = np.round(RNG.standard_normal((BH, 1, d)) * 8)
    k2 = fp16(k.astype(np.float64) + shift)
    for causal in (False, True):
        o = oracle.attn_fp64(q, k, v, causal, 0.25)
        o2 = oracle.attn_fp64(q, k2, v, causal, 0.25)
        assert np.abs(o - o2).max() < 1e-10
        for h in range(BH):
            ref = exact_attention(q[h].astype(np.float64), k[h].astype(np.float64),
                                  v[h].astype(np.float64), causal, 0.25)
            assert np.abs(o[h] - ref).max() < 1e-12


def test_p_tilde_is_rounded_once_to_fp16():
    # Summary bullet 2: P.V runs on 16-bit floating-point operands, so the unnormalized
    # probabilities are rounded to fp16 -- once, from the exact value (no detour via fp32), and
    # the row sum uses the unrounded weights.  Two keys with scores 0 and -sm_scale: the case
    # file derives O = (fp16(e) * 1) / (1 + e) by hand, with fp16(e) given as a multiple of
    # 2^-12; 'tie_plus' sits 2^-40 above an fp16 midpoint, so an unrounded weight or a rounding
    # via fp32 lands on a different value.
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "p_rounding_two_keys.json")
    with open(path) as f:
        cases = json.load(f)["cases"]
    q8 = np.array([[[1], [1]]], np.int8)
    k8 = np.array([[[0], [-1]]], np.int8)
    ones = np.ones((1, 2), np.float32)
    v = fp16(np.array([[[0.0], [1.0]]]))
    for c in cases:
        e_target = c["e_target"][0] / c["e_target"][1]  # exact rational, to the nearest fp64
        sm_scale = -math.log(e_target)
        e = math.exp(-sm_scale)  # the weight the oracle computes, exp(s1 - m) with m = s0 = 0
        expect = (c["fp16_e_times_4096"] / 4096) / (1 + e)
        o64, o16 = oracle.attn(q8, k8, ones, ones, v, False, sm_scale)
        for i in range(2):
            assert abs(o64[0, i, 0] - expect) <= 1e-16, (c["name"], o64[0, i, 0], expect)
        if c["fp32_detour_times_4096"] != c["fp16_e_times_4096"]:
            detour = (c["fp32_detour_times_4096"] / 4096) / (1 + e)
            assert abs(expect - detour) > 1e-5 and abs(expect - e / (1 + e)) > 1e-5


def test_closed_form_two_keys():
    # N = 2, d = 1, non-causal: O_i = v0 + (v1 - v0) * sigmoid(q_i (k1 - k0) s).
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "closed_form_two_keys.json")
    with open(path) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = fp16(np.array(c["q"], np.float64).reshape(1, 2, 1))
        k = fp16(np.array(c["k"], np.float64).reshape(1, 2, 1))
        v = fp16(np.array(c["v"], np.float64).reshape(1, 2, 1))
        o = oracle.attn_fp64(q, k, v, False, c["sm_scale"])
        for i in range(2):
            z = c["q"][i] * (c["k"][1] - c["k"][0]) * c["sm_scale"]
            expect = c["v"][0] + (c["v"][1] - c["v"][0]) / (1 + math.exp(-z))
            assert abs(o[0, i, 0] - expect) < 1e-14
            assert abs(o[0, i, 0] - c["expected"][i]) < 1e-12


# ---------------------------------------------------------------- method level
def test_method_quality_and_smoothing_direction_on_tiny_workload():
    # Key points ("Effect of smoothing K"): with per-token INT8, smoothing K
    # lifts attention cosine from poor to near 1.  On the synthetic K-outlier
    # inputs the same direction must show, and with smoothing the cosine
    # against exact attention must be at least 0.995.
    q, k, v = make_qkv(TINY)
    exact = oracle.attn_fp64(q, k, v, TINY.causal, TINY.sm_scale)
    on = oracle.sage_attn(q, k, v, TINY.causal, TINY.sm_scale, per_block=False, smooth=True)
    off = oracle.sage_attn(q, k, v, TINY.causal, TINY.sm_scale, per_block=False, smooth=False)
    m_on = oracle.metrics(on["o64"], exact)
    m_off = oracle.metrics(off["o64"], exact)
    assert m_on["cos"] >= 0.995
    assert m_on["rel_l1"] < m_off["rel_l1"]
    assert m_on["cos"] > m_off["cos"]


def test_metrics_definitions():
    a = np.array([1.0, 2.0, 3.0])
    b = np.array([1.0, 2.0, 4.0])
    m = oracle.metrics(a, b)
    assert abs(m["cos"] - 17 / math.sqrt(14 * 21)) < 1e-15
    assert abs(m["rel_l1"] - 1 / 7) < 1e-15
    assert abs(m["rmse"] - math.sqrt(1 / 3)) < 1e-15
