"""GPU parity of the microscaling FP4 variant (SageAttention3 entry: both products of the
attention on FP4 tensor cores with microscaling) through the C ABI, against
oracle/sage_oracle_sa3.c.

Bar:
  * E2M1 codes, UE4M3 scales (read back out of the tensor cores' scale atoms), fp32 tile and
    channel scales and the channel means of Q, K and V: bit-exact;
  * O against the oracle run on the same codes, on every row whose offset decisions are clear
    of an integer (the oracle's "unsure" flag):
        |O_gpu - O_oracle| <= 1e-3 * max|V^| + envelope,
    the envelope being the oracle's per-element sum, over keys whose P~ code or group scale lies
    within a relative 1e-4 of a rounding midpoint, of the change the other rounding makes
    (times |v^| / l): the kernel computes p in fp32 (fp32 scores, exp2 approximations), so such
    a decision may go either way; the base term covers fp32 accumulation and the fp16 output.
    Unsure rows (an offset one integer apart changes which P~ groups have subnormal scales):
    cosine >= 0.99 each; all rows together: cosine >= 0.9999;
  * against textbook attention (fp64, unquantized inputs): the kernel's cosine within 1e-3 of the
    oracle's, and the oracle's >= 0.95 on structured inputs (FP4 codes carry up to ~17 %
    rounding per element; measured 0.969 here).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

BASE_FRAC = 1e-3


@pytest.fixture(scope="module")
def sa():
    import quantized_attention_02_b200 as sa
    return sa


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[..., n/2] bytes -> [..., n] E2M1 codes (the even element in the low nibble)."""
    lo, hi = packed & 15, packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))


def atoms_to_scales(atoms: np.ndarray) -> np.ndarray:
    """[..., tiles, A, 512] scale atoms -> [..., tiles * 128, 4A] scales per (row, group of 16)."""
    lead = atoms.shape[:-3]
    t, a = atoms.shape[-3], atoms.shape[-2]
    r = np.arange(128)
    out = np.empty(lead + (t, 128, 4 * a), np.uint8)
    for g in range(4 * a):
        out[..., g] = atoms[..., g // 4, :][..., (r % 32) * 16 + (r // 32) * 4 + g % 4]
    return out.reshape(lead + (t * 128, 4 * a))


def atoms64_to_scales(atoms: np.ndarray) -> np.ndarray:
    """[..., halves, A, 512] scale atoms with 64 rows each (K's tokens, or V's channels at d = 64)
    -> [..., halves * 64, 4A]; also checks that the atoms' other rows are zero."""
    lead = atoms.shape[:-3]
    t, a = atoms.shape[-3], atoms.shape[-2]
    r = np.arange(64)
    out = np.empty(lead + (t, 64, 4 * a), np.uint8)
    for g in range(4 * a):
        out[..., g] = atoms[..., g // 4, :][..., (r % 32) * 16 + (r // 32) * 4 + g % 4]
    lines = atoms.reshape(lead + (t, a, 32, 16))
    assert not lines[..., 8:].any(), "rows 64..127 of 64-row scale atoms must be zero"
    return out.reshape(lead + (t * 64, 4 * a))


def gpu_quant(sa, q, k, v, smooth_v=True):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    b = sa.empty_fp4(qd, smooth_v)
    sa.sage_smooth_k(kd, b["km"])
    sa.sage_quant_qk_fp4(qd, kd, b["km"], b["q4"], b["sfq"], b["gq"], b["k4"], b["sfk"], b["gk"])
    sa.sage_quant_v_fp4(vd, b["v4t"], b["sfv"], b["gv"], b["vm"])
    torch.cuda.synchronize()
    return b


def check_codes(b, ref, N):
    cpu = {k: (v.cpu().numpy() if v is not None else None) for k, v in b.items()}
    for name, gname, sname in (("q4", "gq", "sfq"), ("k4", "gk", "sfk")):
        codes = unpack_codes(cpu[name])
        want = ref[name]
        diff = codes != want
        assert not diff.any(), f"{name}: {diff.sum()} codes differ (first at {np.argwhere(diff)[0]})"
        np.testing.assert_array_equal(cpu[gname], ref[gname], err_msg=gname)
        sc = atoms_to_scales(cpu[sname]) if name == "q4" else atoms64_to_scales(cpu[sname])
        np.testing.assert_array_equal(sc[..., :N, :], ref["qs" if name == "q4" else "ks"], err_msg=sname)
        assert not sc[..., N:, :].any(), f"{sname}: rows past N must carry zero scales"
    np.testing.assert_array_equal(cpu["gv"], ref["gv"], err_msg="gv")
    if ref["vm"] is not None:
        np.testing.assert_array_equal(cpu["vm"], ref["vm"], err_msg="vm")
    vt = unpack_codes(cpu["v4t"])                   # [B,H,d,tiles*128]
    vcodes = np.swapaxes(vt, -1, -2)[..., :N, :]   # token-major
    diff = vcodes != ref["v4"]
    assert not diff.any(), f"v4: {diff.sum()} codes differ (first at {np.argwhere(diff)[0]})"
    assert not vt[..., N:].any(), "V codes past N must be zero"
    d = vt.shape[-2]
    # [B,H,tiles*d (channels per tile), 8]
    vs = atoms_to_scales(cpu["sfv"]) if d == 128 else atoms64_to_scales(cpu["sfv"])
    B, H = vs.shape[:2]
    t = cpu["sfv"].shape[2]
    vs = vs.reshape(B, H, t, d, 8).transpose(0, 1, 2, 4, 3).reshape(B, H, t * 8, d)
    ng = -(-N // 16)
    np.testing.assert_array_equal(vs[..., :ng, :], ref["vs"], err_msg="sfv")


def vhat_max(ref):
    vs = np.repeat(oracle.e4m3_decode(ref["vs"]), 16, axis=-2)[..., :ref["v4"].shape[-2], :]
    return float(np.abs(oracle.e2m1_decode(ref["v4"]) * vs * ref["gv"][..., None, :]).max())


def check_o(o_gpu, o_ref, env, unsure, vmax, what):
    o_gpu = np.asarray(o_gpu, np.float64)
    sure = unsure == 0
    assert sure.mean() > 0.9, f"{what}: too many unsure rows ({(~sure).sum()})"
    err = np.abs(o_gpu - o_ref)
    bar = BASE_FRAC * vmax + env
    bad = (err > bar) & sure[..., None]
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: err {err[i]:.3e} > bar {bar[i]:.3e} at {i} ({bad.sum()} elements)")
    for idx in zip(*np.nonzero(~sure)):
        c = oracle.metrics(o_gpu[idx], o_ref[idx])["cos"]
        assert c >= 0.99, f"{what}: unsure row {idx} cosine {c:.5f}"
    c = oracle.metrics(o_gpu, o_ref)["cos"]
    assert c >= 0.9999, f"{what}: cosine {c:.6f}"


SMALL = [
    W.Workload("fp4_n256", 1, 2, 256, 128, False, True, n_out=4, out_mag=20.0),
    W.Workload("fp4_n384_causal", 1, 2, 384, 128, True, True, n_out=4, out_mag=20.0),
    W.Workload("fp4_ragged_n1000", 2, 1, 1000, 128, False, True, q_std=1.5),
    W.Workload("fp4_ragged_causal_n700", 1, 2, 700, 128, True, True, bias_std=4.0),
    W.Workload("fp4_win_n2048", 1, 2, 2048, 128, False, True, window=256, align=10.0),
    W.Workload("fp4_d64_n256", 1, 2, 256, 64, False, True, n_out=4, out_mag=20.0),
    W.Workload("fp4_d64_ragged_causal_n700", 1, 2, 700, 64, True, True, bias_std=4.0),
    W.Workload("fp4_d64_win_n2048", 2, 1, 2048, 64, False, True, window=256, align=12.0, bias_std=4.0),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fp4_codes_and_output_match_the_oracle(sa, w):
    q, k, v = W.make_qkv(w)
    b = gpu_quant(sa, q, k, v)
    ref = oracle.sage_attn_fp4(q, k, v, w.causal, w.sm_scale)
    check_codes(b, ref, w.N)
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_fp4_quantized(b["q4"], b["sfq"], b["gq"], b["k4"], b["sfk"], b["gk"], b["v4t"], b["sfv"],
                                   b["gv"], b["vm"], o, w.causal, w.sm_scale)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    check_o(o.float().cpu().numpy(), ref["o64"], ref["env"], ref["unsure"], vhat_max(ref), w.name)
    # the whole variant as a user calls it gives the same output
    o2 = torch.empty_like(o)
    sa.sage_attn_fwd_fp4(q.cuda(), k.cuda(), v.cuda(), o2, w.causal, w.sm_scale)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    assert torch.equal(o2, o)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 129, 200])
def test_fp4_edge_sizes(sa, N, causal, d):
    # a single token, partial 64-key tiles, a partial 128-token scale tile, one key tile plus one key
    w = W.Workload(f"fp4_edge_{N}", 1, 2, N, d, causal, True, n_out=2, out_mag=10.0)
    q, k, v = W.make_qkv(w)
    b = gpu_quant(sa, q, k, v)
    ref = oracle.sage_attn_fp4(q, k, v, causal, w.sm_scale)
    check_codes(b, ref, N)
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_fp4_quantized(b["q4"], b["sfq"], b["gq"], b["k4"], b["sfk"], b["gk"], b["v4t"], b["sfv"],
                                   b["gv"], b["vm"], o, causal, w.sm_scale)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    o_gpu = o.float().cpu().numpy().astype(np.float64)
    err = np.abs(o_gpu - ref["o64"])
    bar = BASE_FRAC * vhat_max(ref) + ref["env"]
    sure = ref["unsure"] == 0
    assert np.all((err <= bar) | ~sure[..., None]), f"N={N}: max excess {(err - bar).max():.3e}"
    if causal:  # row 0 sees only key 0: O[0] = v^0 (one P~ code times its own scale, over p itself)
        assert np.isfinite(o_gpu).all()


def test_fp4_without_v_smoothing(sa):
    w = W.Workload("fp4_nosmooth", 1, 2, 512, 128, False, True, n_out=2, out_mag=10.0)
    q, k, v = W.make_qkv(w)
    v = v + 3.0  # a channel offset that smoothing would remove
    b = gpu_quant(sa, q, k, v, smooth_v=False)
    km = oracle.smooth_k(k)
    q4, qs, gq = oracle.quant_fp4(q)
    k4, ks, gk = oracle.quant_fp4(k, km)
    v4, vs, gv, vm = oracle.quant_v_fp4(v, smooth=False)
    ref = dict(q4=q4, qs=qs, gq=gq, k4=k4, ks=ks, gk=gk, v4=v4, vs=vs, gv=gv, vm=None)
    check_codes(b, ref, w.N)
    o64, _, env, unsure = oracle.attn_fp4(q4, qs, gq, k4, ks, gk, v4, vs, gv, None, False, w.sm_scale)
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_fp4_quantized(b["q4"], b["sfq"], b["gq"], b["k4"], b["sfk"], b["gk"], b["v4t"], b["sfv"],
                                   b["gv"], None, o, False, w.sm_scale)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    ref["v4"], ref["vs"], ref["gv"] = v4, vs, gv
    check_o(o.float().cpu().numpy(), o64, env, unsure, vhat_max(ref), "no V smoothing")


@pytest.mark.parametrize("w", [W.HEADLINE, W.SPARSE, W.SPARSE_DIT, W.LLM, W.DIT, W.SPARSE_CAUSAL],
                         ids=lambda w: w.name)
def test_fp4_full_size_sampled_rows(sa, w):
    q, k, v = W.make_qkv(w)
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_fp4(q.cuda(), k.cuda(), v.cuda(), o, w.causal, w.sm_scale)
    torch.cuda.synchronize()
    assert sa.sage_last_device_error() == 0
    og = o.view(w.BH, w.N, w.d).float().cpu().numpy()
    # first rows, tile edges, the causal diagonal's 64-key halves, a middle row and the last one
    rows = np.unique(np.clip(np.array([0, 1, 63, 64, 127, 128, 2047, 4095, 5000, 8191, 12345, w.N - 1]), 0, w.N - 1))
    for h in (0, w.BH // 2, w.BH - 1):
        qh, kh, vh = (x.view(w.BH, w.N, w.d)[h:h + 1] for x in (q, k, v))
        km = oracle.smooth_k(kh)
        q4, qs, gq = oracle.quant_fp4(qh)
        k4, ks, gk = oracle.quant_fp4(kh, km)
        v4, vs, gv, vm = oracle.quant_v_fp4(vh)
        o64, env, unsure = oracle.attn_fp4_rows(q4, qs, gq, k4, ks, gk, v4, vs, gv, vm, 0, rows, w.causal, w.sm_scale)
        vsd = np.repeat(oracle.e4m3_decode(vs), 16, axis=-2)[..., :w.N, :]
        vmax = float(np.abs(oracle.e2m1_decode(v4) * vsd * gv[..., None, :]).max())
        got = og[h, rows]
        err = np.abs(got - o64)
        bar = BASE_FRAC * vmax + env
        sure = unsure == 0
        assert np.all((err <= bar) | ~sure[:, None]), f"{w.name} head {h}: max excess {(err - bar).max():.3e}"
        assert oracle.metrics(got, o64)["cos"] >= 0.9999


def test_fp4_close_to_exact_attention(sa):
    # FP4 is lossy by design: the kernel must be as close to textbook attention as the method
    # itself (the oracle), and the method close enough to be useful
    w = W.Workload("fp4_exact", 1, 2, 1024, 128, False, True, window=256, align=10.0)
    q, k, v = W.make_qkv(w)
    o = torch.empty_like(q, device="cuda")
    sa.sage_attn_fwd_fp4(q.cuda(), k.cuda(), v.cuda(), o, w.causal, w.sm_scale)
    torch.cuda.synchronize()
    exact = oracle.attn_fp64(q, k, v, w.causal, w.sm_scale)
    c_gpu = oracle.metrics(o.float().cpu().numpy(), exact)["cos"]
    c_ref = oracle.metrics(oracle.sage_attn_fp4(q, k, v, w.causal, w.sm_scale)["o64"], exact)["cos"]
    assert abs(c_gpu - c_ref) <= 1e-3, (c_gpu, c_ref)
    assert c_ref >= 0.95, f"the method's cosine to exact attention {c_ref:.4f}"


def test_fp4_rejects_other_head_dimensions(sa):
    q = torch.zeros((1, 1, 256, 96), dtype=torch.float16, device="cuda")
    with pytest.raises(sa.SageError) as e:
        sa.sage_attn_fwd_fp4(q, q, q, torch.empty_like(q), False, 0.125)
    assert e.value.status == sa.SAGE_ERR_UNSUPPORTED


@pytest.mark.parametrize("d", [64, 128])
def test_sageattn_variants_match_their_entry_points(sa, d):
    w = W.Workload(f"variants_d{d}", 1, 2, 320, d, True, True, n_out=2, out_mag=10.0)
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    calls = [("fp16pv", lambda o: sa.sage_attn_fwd(q, k, v, o, True, w.sm_scale, sa.SAGE_PER_BLOCK)),
             ("fp4", lambda o: sa.sage_attn_fwd_fp4(q, k, v, o, True, w.sm_scale))]
    calls.append(("sparse", lambda o: sa.sage_attn_fwd_sparse(q, k, v, o, True, w.sm_scale, sa.SAGE_PER_BLOCK,
                                                              0.99, 0.3, 20.0)))
    if d == 128:
        calls.append(("fp8pv", lambda o: sa.sage_attn_fwd_fp8pv(q, k, v, o, True, w.sm_scale, sa.SAGE_PER_BLOCK)))
    for variant, direct in calls:
        want = torch.empty_like(q)
        direct(want)
        got = sa.sageattn(q, k, v, causal=True, sm_scale=w.sm_scale, variant=variant)
        torch.cuda.synchronize()
        assert torch.equal(got, want), variant
