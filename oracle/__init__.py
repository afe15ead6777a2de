"""CPU oracle for the SageAttention-style 8-bit attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import this package.  The
product library never loads it, and this package never imports the product.

The arithmetic lives in ``sage_oracle.c`` (plain C, fp64 / exact integers,
``-ffp-contract=off``); this module only marshals numpy arrays through ctypes.
Every function cites the passage it follows on the page "SageAttention:
Accurate 8-Bit Attention for Plug-and-play Inference Acceleration"
(research.elamur.ai summary), sections Summary, Key points and Interesting
ideas.

Parity status (which functions are pinned by checks other than themselves):
  smooth_k ........ pinned (exact fp64 mean for power-of-two N; shift of K by a
                    constant; numpy mean within 1 ulp)
  quant ........... pinned (scale fl32(a/127) and inverse fl32(127/a) against exact
                    rationals over every positive fp16 absmax; codes = rne(fl32(x*inv));
                    integer grid identity, round-trip bound, +-127 at the absmax,
                    all-zero group)
  qk_int .......... pinned (brute-force Python loops; int64 numpy matmul)
  attn ............ pinned (P~ rounded once fp64 -> fp16: hand-derived two-key
                    case next to an fp16 midpoint in tests/golden; identity-quantizer
                    special case vs exact fp64 attention within the fp16 error bound;
                    causal row 0 equals V[0]; causal rows ignore later keys; rows of P
                    sum to 1)
  e4m3_encode/decode, quant_v_fp8, attn_fp8pv (FP8 P.V variant, SageAttention2 abstract;
                    sage_oracle_sa2.c) ... pinned (PyTorch's float8_e4m3fn values and
                    brute-force nearest search; exact rational scales and mean; hand-
                    derived two-key cases in tests/golden; the P~-rounding bound against
                    textbook attention; V-shift invariance; causal row 0)
  sparse_predict, attn_sparse, attn_sparse_tiles (block-sparse variant, SpargeAttn
                    abstract; sage_oracle_sparse.c) ... pinned (the dense oracle when every
                    block is kept; textbook attention over the kept keys; a numpy re-
                    derivation of the predicted map; closed forms of the self-similarity;
                    hand-built second-stage cases; limits of tau and theta)
  e2m1_encode/decode, fp4_microscale, quant_fp4, quant_v_fp4, attn_fp4 (microscaling FP4
                    variant, SageAttention3 abstract; sage_oracle_sa3.c) ... pinned (the
                    E2M1 type of ml_dtypes and PyTorch's E4M3; brute-force nearest search;
                    worked groups; the tile and channel scales' extremes; hand-derived rows
                    in tests/golden (the online frames, a subnormal group scale); the FP4
                    error bound against textbook attention on dequantized inputs; the
                    envelope of a key on an E2M1 midpoint)
Every pin is itself checked by tests/test_oracle_mutations.py: planted slips
(dropped or re-routed roundings, signs, indices, group sizes, operands), each of which
makes the pins fail.
  attn_fp64 ....... pinned (softmax shift invariance; hand-derived closed forms
                    in tests/golden)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, f) for f in ("sage_oracle.c", "sage_oracle_sa2.c", "sage_oracle_sparse.c",
                                           "sage_oracle_sa3.c")]
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libsage_oracle.so")
_lock = threading.Lock()
_lib = None

GROUP_PER_TOKEN = (1, 1)
GROUP_PER_BLOCK = (128, 64)  # (Q tokens, K tokens) per quantization group


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no FMA contraction, OpenMP)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(s) for s in _SRCS):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, *_SRCS, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # SAGE_ORACLE_LIB: a deliberately broken build of this file, loaded by the
            # mutation tests (tests/test_oracle_mutations.py) to show that the pins fail on it
            lib = ctypes.CDLL(os.environ.get("SAGE_ORACLE_LIB") or build())
            i64, i32, f64, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
            lib.oracle_smooth_k.argtypes = [vp, i64, i64, i64, vp]
            lib.oracle_quant.argtypes = [vp, vp, i64, i64, i64, i64, vp, vp]
            lib.oracle_qk_int.argtypes = [vp, vp, i64, i64, i64, vp]
            lib.oracle_qk_int_rows.argtypes = [vp, vp, i64, i64, vp, i64, vp]
            lib.oracle_attn.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, f64, i64, i64, vp, vp]
            lib.oracle_attn_rows.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, f64, i64, i64, vp,
                                             i64, vp, vp]
            lib.oracle_attn_probs.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, f64, i64, i64, vp]
            lib.oracle_attn_fp64.argtypes = [vp, vp, vp, i64, i64, i64, i32, f64, vp]
            lib.oracle_round_fp16.argtypes = [vp, i64, vp]
            lib.oracle_round_fp16.restype = None
            lib.oracle_quant_scale.argtypes = [vp, i64, vp, vp]
            lib.oracle_quant_scale.restype = None
            lib.oracle_e4m3_encode_n.argtypes = [vp, i64, vp]
            lib.oracle_e4m3_encode_n.restype = None
            lib.oracle_e4m3_decode_n.argtypes = [vp, i64, vp]
            lib.oracle_e4m3_decode_n.restype = None
            lib.oracle_quant_v_fp8.argtypes = [vp, i64, i64, i64, vp, vp, vp]
            lib.oracle_attn_fp8pv.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, f64, i64, i64, vp, vp]
            lib.oracle_attn_fp8pv_rows.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i32, f64, i64, i64, vp,
                                                   i64, vp]
            for name in ("oracle_quant_v_fp8", "oracle_attn_fp8pv", "oracle_attn_fp8pv_rows"):
                getattr(lib, name).restype = i32
            lib.oracle_sparse_predict.argtypes = [vp, vp, i64, i64, i64, i32, f64, f64, f64, f64, vp, vp, vp, vp]
            lib.oracle_sparse_predict.restype = i32
            lib.oracle_attn_sparse.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, f64, i64, i64, vp, f64, vp,
                                               vp, vp]
            lib.oracle_attn_sparse.restype = i32
            lib.oracle_attn_sparse_tiles.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, f64, i64, i64, vp, f64, vp,
                                                     i64, vp, vp]
            lib.oracle_attn_sparse_tiles.restype = i32
            lib.oracle_e2m1_encode_n.argtypes = [vp, i64, vp]
            lib.oracle_e2m1_encode_n.restype = None
            lib.oracle_e2m1_decode_n.argtypes = [vp, i64, vp]
            lib.oracle_e2m1_decode_n.restype = None
            lib.oracle_fp4_microscale.argtypes = [vp, i32, vp]
            lib.oracle_fp4_microscale.restype = ctypes.c_uint8
            lib.oracle_quant_fp4.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp]
            lib.oracle_quant_v_fp4.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp, vp]
            lib.oracle_attn_fp4.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, f64, vp, vp,
                                            vp, vp]
            lib.oracle_attn_fp4_rows.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, f64,
                                                 vp, i64, vp, vp, vp]
            for name in ("oracle_quant_fp4", "oracle_quant_v_fp4", "oracle_attn_fp4", "oracle_attn_fp4_rows"):
                getattr(lib, name).restype = i32
            for name in ("oracle_smooth_k", "oracle_quant", "oracle_qk_int", "oracle_qk_int_rows", "oracle_attn",
                         "oracle_attn_rows", "oracle_attn_probs", "oracle_attn_fp64"):
                getattr(lib, name).restype = i32
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_fp16_bits(x) -> np.ndarray:
    """Accept a numpy float16 array or a torch fp16 tensor; return uint16 bits."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().contiguous().numpy()
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16)
    if x.dtype == np.uint16:
        return x
    raise TypeError(f"expected fp16 data, got {x.dtype}")


def _check(rc: int, name: str) -> None:
    if rc != 0:
        raise RuntimeError(f"{name} failed with status {rc}")


def _bhnd(x: np.ndarray):
    if x.ndim == 4:
        B, H, N, d = x.shape
        return B * H, N, d
    if x.ndim == 3:
        return x.shape
    raise ValueError("expected [B,H,N,d] or [BH,N,d]")


def smooth_k(k) -> np.ndarray:
    """Per-(b,h) channel mean of K over tokens (Summary bullet 1; idea I1).

    Returns fp32 [*lead, d] where lead = k.shape[:-2]."""
    kb = _as_fp16_bits(k)
    BH, N, d = _bhnd(kb)
    km = np.empty(kb.shape[:-2] + (d,), np.float32)
    _check(_load().oracle_smooth_k(_ptr(kb), BH, N, d, _ptr(km)), "oracle_smooth_k")
    return km


def scale_count(N: int, g: int) -> int:
    return (N + g - 1) // g


def quant_scale(a) -> tuple[np.ndarray, np.ndarray]:
    """(scale, inverse) = (fl32(a/127), fl32(127/a)) for group absmax values a (fp32);
    both 0 where a = 0.  The two roundings the INT8 reading fixes (Summary bullet 1)."""
    a = np.ascontiguousarray(a, np.float32)
    s = np.empty_like(a)
    inv = np.empty_like(a)
    _load().oracle_quant_scale(_ptr(a), a.size, _ptr(s), _ptr(inv))
    return s, inv


def quant(x, g: int, mu=None):
    """Symmetric absmax INT8 quantization over groups of g tokens (Summary
    bullet 1; Key points on per-token granularity).  mu: optional fp32 channel
    mean subtracted first (K smoothing).  Returns (int8 codes, fp32 scales)."""
    xb = _as_fp16_bits(x)
    BH, N, d = _bhnd(xb)
    q = np.empty(xb.shape, np.int8)
    s = np.empty(xb.shape[:-2] + (scale_count(N, g),), np.float32)
    mu_arr = None
    if mu is not None:
        mu_arr = np.ascontiguousarray(mu, dtype=np.float32)
        if mu_arr.size != BH * d:
            raise ValueError("mu must hold one value per (head, channel)")
    _check(_load().oracle_quant(_ptr(xb), _ptr(mu_arr) if mu_arr is not None else None, BH, N, d, g,
                                _ptr(q), _ptr(s)), "oracle_quant")
    return q, s


def qk_int(q8: np.ndarray, k8: np.ndarray) -> np.ndarray:
    """Exact integer q8 . k8^T per head (int64 [*lead, N, N])."""
    q8 = np.ascontiguousarray(q8, np.int8)
    k8 = np.ascontiguousarray(k8, np.int8)
    BH, N, d = _bhnd(q8)
    S = np.empty(q8.shape[:-1] + (N,), np.int64)
    _check(_load().oracle_qk_int(_ptr(q8), _ptr(k8), BH, N, d, _ptr(S)), "oracle_qk_int")
    return S


def qk_int_rows(q8h: np.ndarray, k8h: np.ndarray, rows) -> np.ndarray:
    """Exact integer products of the listed query rows of one head [N,d] with
    all N keys (int64 [len(rows), N])."""
    q8h = np.ascontiguousarray(q8h, np.int8)
    k8h = np.ascontiguousarray(k8h, np.int8)
    N, d = q8h.shape
    rows = np.ascontiguousarray(rows, np.int64)
    S = np.empty((rows.size, N), np.int64)
    _check(_load().oracle_qk_int_rows(_ptr(q8h), _ptr(k8h), N, d, _ptr(rows), rows.size, _ptr(S)),
           "oracle_qk_int_rows")
    return S


def attn(q8, k8, sq, sk, v, causal: bool, sm_scale: float, groups=GROUP_PER_TOKEN):
    """Quantized attention: dequantized scores, fp64 softmax, P rounded to fp16,
    fp64 P.V (Summary bullets 1-2).  Returns (O fp64, O fp16)."""
    q8 = np.ascontiguousarray(q8, np.int8)
    k8 = np.ascontiguousarray(k8, np.int8)
    sq = np.ascontiguousarray(sq, np.float32)
    sk = np.ascontiguousarray(sk, np.float32)
    vb = _as_fp16_bits(v)
    BH, N, d = _bhnd(vb)
    o64 = np.empty(vb.shape, np.float64)
    o16 = np.empty(vb.shape, np.uint16)
    gq, gk = groups
    _check(_load().oracle_attn(_ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), _ptr(vb), BH, N, d,
                               int(bool(causal)), float(sm_scale), gq, gk, _ptr(o64), _ptr(o16)),
           "oracle_attn")
    return o64, o16.view(np.float16)


def attn_rows(q8h, k8h, sqh, skh, vh, rows, causal: bool, sm_scale: float, groups=GROUP_PER_TOKEN):
    """Like attn() for one head [N,d] but only for the listed query rows."""
    q8h = np.ascontiguousarray(q8h, np.int8)
    k8h = np.ascontiguousarray(k8h, np.int8)
    sqh = np.ascontiguousarray(sqh, np.float32)
    skh = np.ascontiguousarray(skh, np.float32)
    vb = _as_fp16_bits(vh)
    N, d = vb.shape
    rows = np.ascontiguousarray(rows, np.int64)
    o64 = np.empty((rows.size, d), np.float64)
    o16 = np.empty((rows.size, d), np.uint16)
    gq, gk = groups
    _check(_load().oracle_attn_rows(_ptr(q8h), _ptr(k8h), _ptr(sqh), _ptr(skh), _ptr(vb), N, d,
                                    int(bool(causal)), float(sm_scale), gq, gk, _ptr(rows),
                                    rows.size, _ptr(o64), _ptr(o16)), "oracle_attn_rows")
    return o64, o16.view(np.float16)


def attn_probs(q8h, k8h, sqh, skh, vh, causal: bool, sm_scale: float, groups=GROUP_PER_TOKEN):
    """Normalized softmax probabilities of one head (N x N fp64)."""
    q8h = np.ascontiguousarray(q8h, np.int8)
    k8h = np.ascontiguousarray(k8h, np.int8)
    sqh = np.ascontiguousarray(sqh, np.float32)
    skh = np.ascontiguousarray(skh, np.float32)
    vb = _as_fp16_bits(vh)
    N, d = vb.shape
    P = np.empty((N, N), np.float64)
    gq, gk = groups
    _check(_load().oracle_attn_probs(_ptr(q8h), _ptr(k8h), _ptr(sqh), _ptr(skh), _ptr(vb), N, d,
                                     int(bool(causal)), float(sm_scale), gq, gk, _ptr(P)),
           "oracle_attn_probs")
    return P


def attn_fp64(q, k, v, causal: bool, sm_scale: float) -> np.ndarray:
    """Exact (unquantized) attention in fp64 (idea I5's tensor-level reference)."""
    qb, kb, vb = _as_fp16_bits(q), _as_fp16_bits(k), _as_fp16_bits(v)
    BH, N, d = _bhnd(qb)
    o = np.empty(qb.shape, np.float64)
    _check(_load().oracle_attn_fp64(_ptr(qb), _ptr(kb), _ptr(vb), BH, N, d, int(bool(causal)),
                                    float(sm_scale), _ptr(o)), "oracle_attn_fp64")
    return o


def round_fp16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_round_fp16(_ptr(x), x.size, _ptr(out))
    return out.view(np.float16)


def sage_attn(q, k, v, causal: bool, sm_scale: float, per_block: bool, smooth: bool = True):
    """The whole method in the page's order: smooth K, quantize Q and K, then
    attention (Summary bullets 1-2).  Returns a dict with every intermediate."""
    gq, gk = GROUP_PER_BLOCK if per_block else GROUP_PER_TOKEN
    km = smooth_k(k) if smooth else None
    q8, sq = quant(q, gq)
    k8, sk = quant(k, gk, km)
    o64, o16 = attn(q8, k8, sq, sk, v, causal, sm_scale, (gq, gk))
    return dict(km=km, q8=q8, sq=sq, k8=k8, sk=sk, o64=o64, o16=o16)


# ------------------------------------------------------------------ FP8 P.V variant
# (SageAttention2 abstract: (P~, V) quantized to FP8, V smoothed, P~V in an FP32 buffer;
# readings in sage_oracle_sa2.c)
def e4m3_encode(x) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even, saturating at +-448): uint8 codes."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e4m3_encode_n(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(b) -> np.ndarray:
    """Value of E4M3 codes (fp64)."""
    b = np.ascontiguousarray(b, np.uint8)
    out = np.empty(b.shape, np.float64)
    _load().oracle_e4m3_decode_n(_ptr(b), b.size, _ptr(out))
    return out


def quant_v_fp8(v, smooth: bool = True):
    """V to E4M3 with one fp32 scale per (head, channel), after subtracting the channel mean
    when smooth.  Returns (v8 uint8 codes, sv fp32 [*lead, d], vm fp32 [*lead, d] or None)."""
    vb = _as_fp16_bits(v)
    BH, N, d = _bhnd(vb)
    v8 = np.empty(vb.shape, np.uint8)
    sv = np.empty(vb.shape[:-2] + (d,), np.float32)
    vm = np.empty(vb.shape[:-2] + (d,), np.float32) if smooth else None
    _check(_load().oracle_quant_v_fp8(_ptr(vb), BH, N, d, _ptr(vm) if smooth else None, _ptr(sv), _ptr(v8)),
           "oracle_quant_v_fp8")
    return v8, sv, vm


def attn_fp8pv(q8, k8, sq, sk, v8, sv, vm, causal: bool, sm_scale: float, groups=GROUP_PER_TOKEN):
    """INT8 Q.K^T attention with P~ and V in E4M3 (readings in sage_oracle_sa2.c).
    Returns (O fp64, O fp16)."""
    q8 = np.ascontiguousarray(q8, np.int8)
    k8 = np.ascontiguousarray(k8, np.int8)
    sq = np.ascontiguousarray(sq, np.float32)
    sk = np.ascontiguousarray(sk, np.float32)
    v8 = np.ascontiguousarray(v8, np.uint8)
    sv = np.ascontiguousarray(sv, np.float32)
    vm_arr = None if vm is None else np.ascontiguousarray(vm, np.float32)
    BH, N, d = _bhnd(v8)
    o64 = np.empty(v8.shape, np.float64)
    o16 = np.empty(v8.shape, np.uint16)
    gq, gk = groups
    _check(_load().oracle_attn_fp8pv(_ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), _ptr(v8), _ptr(sv),
                                     _ptr(vm_arr) if vm_arr is not None else None, BH, N, d, int(bool(causal)),
                                     float(sm_scale), gq, gk, _ptr(o64), _ptr(o16)), "oracle_attn_fp8pv")
    return o64, o16.view(np.float16)


def attn_fp8pv_rows(q8h, k8h, sqh, skh, v8h, svh, vmh, rows, causal: bool, sm_scale: float,
                    groups=GROUP_PER_TOKEN) -> np.ndarray:
    """Like attn_fp8pv() for one head [N,d], only the listed query rows (fp64)."""
    q8h = np.ascontiguousarray(q8h, np.int8)
    k8h = np.ascontiguousarray(k8h, np.int8)
    sqh = np.ascontiguousarray(sqh, np.float32)
    skh = np.ascontiguousarray(skh, np.float32)
    v8h = np.ascontiguousarray(v8h, np.uint8)
    svh = np.ascontiguousarray(svh, np.float32)
    vmh = None if vmh is None else np.ascontiguousarray(vmh, np.float32)
    N, d = v8h.shape
    rows = np.ascontiguousarray(rows, np.int64)
    o64 = np.empty((rows.size, d), np.float64)
    gq, gk = groups
    _check(_load().oracle_attn_fp8pv_rows(_ptr(q8h), _ptr(k8h), _ptr(sqh), _ptr(skh), _ptr(v8h), _ptr(svh),
                                          _ptr(vmh) if vmh is not None else None, N, d, int(bool(causal)),
                                          float(sm_scale), gq, gk, _ptr(rows), rows.size, _ptr(o64)),
           "oracle_attn_fp8pv_rows")
    return o64


def sage_attn_fp8pv(q, k, v, causal: bool, sm_scale: float, per_block: bool, smooth_v: bool = True):
    """The FP8 P.V variant in order: smooth K, quantize Q and K to INT8, quantize V to E4M3
    (smoothed), attention with P~ in E4M3.  Returns every intermediate."""
    gq, gk = GROUP_PER_BLOCK if per_block else GROUP_PER_TOKEN
    km = smooth_k(k)
    q8, sq = quant(q, gq)
    k8, sk = quant(k, gk, km)
    v8, sv, vm = quant_v_fp8(v, smooth_v)
    o64, o16 = attn_fp8pv(q8, k8, sq, sk, v8, sv, vm, causal, sm_scale, (gq, gk))
    return dict(km=km, q8=q8, sq=sq, k8=k8, sk=sk, v8=v8, sv=sv, vm=vm, o64=o64, o16=o16)


# ------------------------------------------------------------------ microscaling FP4 variant
# (SageAttention3 entry: microscaling FP4 attention on FP4 tensor cores; readings in
# sage_oracle_sa3.c)
FP4_TILE, FP4_GROUP = 128, 16


def e2m1_encode(x) -> np.ndarray:
    """Round to the nearest E2M1 value (ties to the even mantissa bit, saturating at +-6):
    4-bit codes, one per uint8 (bit 3 the sign)."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e2m1_encode_n(_ptr(x), x.size, _ptr(out))
    return out


def e2m1_decode(c) -> np.ndarray:
    """Value of E2M1 codes (fp64)."""
    c = np.ascontiguousarray(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().oracle_e2m1_decode_n(_ptr(c), c.size, _ptr(out))
    return out


def fp4_microscale(z):
    """One group of at most 16 fp32 values: (UE4M3 scale byte, E2M1 codes)."""
    z = np.ascontiguousarray(z, np.float32)
    if z.ndim != 1 or z.size > FP4_GROUP:
        raise ValueError("a group holds at most 16 values")
    codes = np.zeros(z.size, np.uint8)
    s8 = _load().oracle_fp4_microscale(_ptr(z), z.size, _ptr(codes))
    return int(s8), codes


def quant_fp4(x, km=None):
    """Q (km None) or smoothed K to FP4: (codes uint8 [*lead, N, d] one per byte, UE4M3 scales
    uint8 [*lead, N, d/16], fp32 tile scales [*lead, ceil(N/128)])."""
    xb = _as_fp16_bits(x)
    BH, N, d = _bhnd(xb)
    codes = np.empty(xb.shape, np.uint8)
    s8 = np.empty(xb.shape[:-1] + (d // FP4_GROUP,), np.uint8)
    g = np.empty(xb.shape[:-2] + (-(-N // FP4_TILE),), np.float32)
    kmv = None if km is None else np.ascontiguousarray(km, np.float32)
    _check(_load().oracle_quant_fp4(_ptr(xb), _ptr(kmv) if kmv is not None else None, BH, N, d, _ptr(codes),
                                    _ptr(s8), _ptr(g)), "oracle_quant_fp4")
    return codes, s8, g


def quant_v_fp4(v, smooth: bool = True):
    """V to FP4 along the tokens: (codes uint8 [*lead, N, d], UE4M3 scales uint8
    [*lead, ceil(N/16), d], channel scales gv fp32 [*lead, d], channel means vm or None)."""
    vb = _as_fp16_bits(v)
    BH, N, d = _bhnd(vb)
    codes = np.empty(vb.shape, np.uint8)
    s8 = np.empty(vb.shape[:-2] + (-(-N // FP4_GROUP), d), np.uint8)
    gv = np.empty(vb.shape[:-2] + (d,), np.float32)
    vm = np.empty(vb.shape[:-2] + (d,), np.float32) if smooth else None
    _check(_load().oracle_quant_v_fp4(_ptr(vb), BH, N, d, int(bool(smooth)), _ptr(vm) if smooth else None,
                                      _ptr(gv), _ptr(codes), _ptr(s8)), "oracle_quant_v_fp4")
    return codes, s8, gv, vm


def _fp4_args(q4, qs, gq, k4, ks, gk, v4, vs, gv, vm):
    u8 = lambda a: np.ascontiguousarray(a, np.uint8)  # noqa: E731
    f32 = lambda a: np.ascontiguousarray(a, np.float32)  # noqa: E731
    return (u8(q4), u8(qs), f32(gq), u8(k4), u8(ks), f32(gk), u8(v4), u8(vs), f32(gv),
            None if vm is None else f32(vm))


def attn_fp4(q4, qs, gq, k4, ks, gk, v4, vs, gv, vm, causal: bool, sm_scale: float):
    """Microscaling FP4 attention (readings in sage_oracle_sa3.c).  Returns (O fp64, O fp16,
    envelope fp64 [*lead, N, d], unsure uint8 [*lead, N])."""
    a = _fp4_args(q4, qs, gq, k4, ks, gk, v4, vs, gv, vm)
    BH, N, d = _bhnd(a[6])
    o64 = np.empty(a[6].shape, np.float64)
    o16 = np.empty(a[6].shape, np.uint16)
    env = np.empty(a[6].shape, np.float64)
    unsure = np.empty(a[6].shape[:-1], np.uint8)
    ptrs = [_ptr(x) if x is not None else None for x in a]
    _check(_load().oracle_attn_fp4(*ptrs, BH, N, d, int(bool(causal)), float(sm_scale), _ptr(o64), _ptr(o16),
                                   _ptr(env), _ptr(unsure)), "oracle_attn_fp4")
    return o64, o16.view(np.float16), env, unsure


def attn_fp4_rows(q4, qs, gq, k4, ks, gk, v4, vs, gv, vm, bh: int, rows, causal: bool, sm_scale: float):
    """attn_fp4() for the listed query rows of head bh only (arrays flattened to [BH, ...]).
    Returns (O fp64 [rows, d], envelope [rows, d], unsure [rows])."""
    a = _fp4_args(q4, qs, gq, k4, ks, gk, v4, vs, gv, vm)
    BH, N, d = _bhnd(a[6])
    if not 0 <= bh < BH:
        raise ValueError("head index out of range")
    rows = np.ascontiguousarray(rows, np.int64)
    o64 = np.empty((rows.size, d), np.float64)
    env = np.empty((rows.size, d), np.float64)
    unsure = np.empty(rows.size, np.uint8)
    ptrs = [_ptr(x) if x is not None else None for x in a]
    _check(_load().oracle_attn_fp4_rows(*ptrs, bh, N, d, int(bool(causal)), float(sm_scale), _ptr(rows),
                                        rows.size, _ptr(o64), _ptr(env), _ptr(unsure)), "oracle_attn_fp4_rows")
    return o64, env, unsure


def sage_attn_fp4(q, k, v, causal: bool, sm_scale: float, smooth_v: bool = True):
    """The FP4 variant in order: smooth K, Q and K to FP4, V to FP4 (smoothed), attention with
    microscaled FP4 P~.  Returns every intermediate."""
    km = smooth_k(k)
    q4, qs, gq = quant_fp4(q)
    k4, ks, gk = quant_fp4(k, km)
    v4, vs, gv, vm = quant_v_fp4(v, smooth_v)
    o64, o16, env, unsure = attn_fp4(q4, qs, gq, k4, ks, gk, v4, vs, gv, vm, causal, sm_scale)
    return dict(km=km, q4=q4, qs=qs, gq=gq, k4=k4, ks=ks, gk=gk, v4=v4, vs=vs, gv=gv, vm=vm, o64=o64, o16=o16,
                env=env, unsure=unsure)


# ------------------------------------------------------------------ block-sparse variant
# (SpargeAttn abstract: a first stage that predicts the attention map and skips matrix
# products, a second softmax-aware stage that skips more; readings in sage_oracle_sparse.c)
SPARSE_BQ, SPARSE_BK = 256, 128


def sparse_predict(q, k, causal: bool, sm_scale: float, tau: float, theta: float, eps: float = 1e-4):
    """Stage 1: the kept (query block of 256, key block of 128) pairs.  Returns (mask uint8
    [*lead, NQB, NKB], unsure uint8 (decisions within eps of flipping), qsim [*lead, NQB],
    ksim [*lead, NKB])."""
    qb, kb = _as_fp16_bits(q), _as_fp16_bits(k)
    BH, N, d = _bhnd(qb)
    nqb, nkb = -(-N // SPARSE_BQ), -(-N // SPARSE_BK)
    lead = qb.shape[:-2]
    mask = np.empty(lead + (nqb, nkb), np.uint8)
    unsure = np.empty(lead + (nqb, nkb), np.uint8)
    qsim = np.empty(lead + (nqb,), np.float64)
    ksim = np.empty(lead + (nkb,), np.float64)
    _check(_load().oracle_sparse_predict(_ptr(qb), _ptr(kb), BH, N, d, int(bool(causal)), float(sm_scale),
                                         float(tau), float(theta), float(eps), _ptr(mask), _ptr(unsure), _ptr(qsim),
                                         _ptr(ksim)), "oracle_sparse_predict")
    return mask, unsure, qsim, ksim


def attn_sparse(q8, k8, sq, sk, v, mask, causal: bool, sm_scale: float, lam: float, groups=GROUP_PER_TOKEN):
    """Block-sparse quantized attention over the kept blocks of `mask`, with the stage-2 filter
    lam (log2 units; inf = none).  Returns (O fp64, O fp16, skipped uint8 [*lead, NQT, NKB])."""
    q8 = np.ascontiguousarray(q8, np.int8)
    k8 = np.ascontiguousarray(k8, np.int8)
    sq = np.ascontiguousarray(sq, np.float32)
    sk = np.ascontiguousarray(sk, np.float32)
    vb = _as_fp16_bits(v)
    BH, N, d = _bhnd(vb)
    mask = np.ascontiguousarray(mask, np.uint8)
    if mask.size != BH * (-(-N // SPARSE_BQ)) * (-(-N // SPARSE_BK)):
        raise ValueError("mask must be [BH, ceil(N/256), ceil(N/128)]")
    nqt = -(-N // 128)
    o64 = np.empty(vb.shape, np.float64)
    o16 = np.empty(vb.shape, np.uint16)
    skipped = np.empty(vb.shape[:-2] + (nqt, -(-N // SPARSE_BK)), np.uint8)
    gq, gk = groups
    _check(_load().oracle_attn_sparse(_ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), _ptr(vb), BH, N, d, int(bool(causal)),
                                      float(sm_scale), gq, gk, _ptr(mask), float(lam), _ptr(o64), _ptr(o16),
                                      _ptr(skipped)), "oracle_attn_sparse")
    return o64, o16.view(np.float16), skipped


def attn_sparse_tiles(q8h, k8h, sqh, skh, vh, maskh, tiles, causal: bool, sm_scale: float, lam: float,
                      groups=GROUP_PER_TOKEN):
    """attn_sparse() for the listed 128-row query tiles of one head [N, d] only.  Returns
    (O fp64 [len(tiles), 128, d] -- rows past N are NaN --, skipped uint8 [len(tiles), NKB])."""
    q8h = np.ascontiguousarray(q8h, np.int8)
    k8h = np.ascontiguousarray(k8h, np.int8)
    sqh = np.ascontiguousarray(sqh, np.float32)
    skh = np.ascontiguousarray(skh, np.float32)
    vb = _as_fp16_bits(vh)
    N, d = vb.shape
    maskh = np.ascontiguousarray(maskh, np.uint8)
    tiles = np.ascontiguousarray(tiles, np.int64)
    o64 = np.full((tiles.size, 128, d), np.nan, np.float64)
    skipped = np.empty((tiles.size, -(-N // SPARSE_BK)), np.uint8)
    gq, gk = groups
    _check(_load().oracle_attn_sparse_tiles(_ptr(q8h), _ptr(k8h), _ptr(sqh), _ptr(skh), _ptr(vb), N, d,
                                            int(bool(causal)), float(sm_scale), gq, gk, _ptr(maskh), float(lam),
                                            _ptr(tiles), tiles.size, _ptr(o64), _ptr(skipped)),
           "oracle_attn_sparse_tiles")
    return o64, skipped


def metrics(a: np.ndarray, b: np.ndarray) -> dict:
    """Tensor-level accuracy metrics named by idea I5: cosine similarity,
    relative L1 (sum|a-b| / sum|b|) and RMSE, with b the reference."""
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    cos = float(np.dot(a, b) / (np.linalg.norm(a) * np.linalg.norm(b)))
    rel_l1 = float(np.abs(a - b).sum() / np.abs(b).sum())
    rmse = float(np.sqrt(np.mean((a - b) ** 2)))
    return dict(cos=cos, rel_l1=rel_l1, rmse=rmse)
