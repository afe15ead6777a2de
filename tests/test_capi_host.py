"""Host-side checks of the C-ABI library that need no GPU: it loads, exports every
function include/sage_attn.h declares, and rejects invalid calls before launching
anything (argument validation happens ahead of any CUDA call)."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sa():
    from quantized_attention_02_b200 import build
    build.build()
    import quantized_attention_02_b200 as sa
    return sa


def test_library_exports_every_header_function(sa):
    names = sa.header_functions()
    assert set(names) >= {"sage_smooth_k", "sage_quant_qk", "sage_attn_fwd", "sage_attn_fwd_quantized",
                          "sage_debug_qk_int32", "sage_status_string", "sage_scale_count",
                          "sage_last_device_error"}
    lib = ctypes.CDLL(sa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_library_has_no_driver_link_dependency(sa):
    # the driver is reached through the runtime's entry-point query only
    import subprocess
    out = subprocess.run(["ldd", sa.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_status_strings_and_scale_counts(sa):
    for s in (0, -1, -2, -3, -4, -5, 42):
        assert isinstance(sa.sage_status_string(s), str) and sa.sage_status_string(s)
    assert sa.sage_scale_count(1024, sa.SAGE_PER_TOKEN, True) == 1024
    assert sa.sage_scale_count(1024, sa.SAGE_PER_BLOCK, True) == 8
    assert sa.sage_scale_count(1024, sa.SAGE_PER_BLOCK, False) == 16
    assert sa.sage_scale_count(300, sa.SAGE_PER_BLOCK, False) == 5
    assert sa.sage_scale_count(0, sa.SAGE_PER_BLOCK, False) == 0
    assert sa.sage_scale_count(128, 7, False) == 0


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("args,expect", [
    # (B, H, N, d)
    ((1, 1, 128, 96), -2),   # d not 64/128
    ((0, 1, 128, 64), -1),   # empty batch
    ((1, 1, 0, 64), -1),     # empty sequence
    ((1, -1, 128, 64), -1),
    ((4096, 4096, 1024, 128), -2),  # too many elements for 32-bit indexing
])
def test_shape_validation(sa, args, expect):
    B, H, N, d = args
    L = sa.get_lib()
    s = ctypes.c_void_p(0)
    assert L.sage_smooth_k(FAKE, FAKE, B, H, N, d, s) == expect
    assert L.sage_quant_qk(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, B, H, N, d, 1, s) == expect
    assert L.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, B, H, N, d, 0, 0.1, 1, s) == expect
    assert L.sage_attn_fwd_quantized(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, H, N, d, 0, 0.1, 1, s) == expect
    assert L.sage_debug_qk_int32(FAKE, FAKE, FAKE, B, H, N, d, s) == expect


def test_ragged_n_rejected_only_by_the_int32_debug_entry(sa):
    # any N >= 1 is supported by the method's entry points (exercised on the GPU); the INT32
    # debug entry needs whole 128 x 128 tiles and refuses before touching its pointers
    L = sa.get_lib()
    s = ctypes.c_void_p(0)
    for n in (1, 100, 200, 1000):
        assert L.sage_debug_qk_int32(FAKE, FAKE, FAKE, 1, 1, n, 64, s) == -2


def test_null_pointers_and_bad_scalars(sa):
    L = sa.get_lib()
    s = ctypes.c_void_p(0)
    assert L.sage_smooth_k(None, FAKE, 1, 1, 128, 64, s) == -1
    assert L.sage_quant_qk(FAKE, FAKE, None, FAKE, None, FAKE, FAKE, 1, 1, 128, 64, 1, s) == -1
    assert L.sage_attn_fwd(FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 0, 0.1, 1, s) == -1
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert L.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, bad, 1, s) == -1
        assert L.sage_attn_fwd_quantized(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, bad, 1, s) == -1
    for g in (-1, 2, 17):
        assert L.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, 0.1, g, s) == -1
        assert L.sage_quant_qk(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, g, s) == -1
    misaligned = ctypes.c_void_p(0x1008)
    assert L.sage_smooth_k(misaligned, FAKE, 1, 1, 128, 64, s) == -1
    assert L.sage_debug_qk_int32(FAKE, FAKE, None, 1, 1, 128, 64, s) == -1
    assert L.sage_debug_wait_timeout(None, s) == -1


def test_variant_entries_validate_before_any_cuda_call(sa):
    # FP8 P.V, block-sparse and FP4 entry points: null pointers, unsupported head dimensions and
    # sizes, bad scalars and misaligned buffers are rejected before anything is enqueued
    L = sa.get_lib()
    s = ctypes.c_void_p(0)
    mis = ctypes.c_void_p(0x1008)
    inv, uns = sa.SAGE_ERR_INVALID, sa.SAGE_ERR_UNSUPPORTED
    # microscaling FP4: head dimension 64 or 128
    assert L.sage_attn_fwd_fp4(FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 96, 0, 0.1, s) == uns
    assert L.sage_attn_fwd_fp4_quantized(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                         1, 1, 256, 32, 0, 0.1, s) == uns
    assert L.sage_attn_fwd_fp4(FAKE, FAKE, FAKE, None, 1, 1, 256, 128, 0, 0.1, s) == inv
    assert L.sage_attn_fwd_fp4(mis, FAKE, FAKE, FAKE, 1, 1, 256, 128, 0, 0.1, s) == inv
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert L.sage_attn_fwd_fp4(FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 128, 0, bad, s) == inv
        assert L.sage_attn_fwd_fp4_quantized(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                             1, 1, 256, 128, 0, bad, s) == inv
    assert L.sage_quant_qk_fp4(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 256, 128, s) == inv
    assert L.sage_quant_qk_fp4(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 256, s) == uns
    assert L.sage_quant_qk_fp4(FAKE, FAKE, None, mis, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 128, s) == inv
    assert L.sage_quant_v_fp4(FAKE, None, FAKE, FAKE, None, 1, 1, 256, 128, s) == inv
    assert L.sage_quant_v_fp4(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 256, 96, s) == uns
    assert L.sage_attn_fwd_fp4_quantized(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, mis, FAKE, None, FAKE,
                                         1, 1, 256, 128, 0, 0.1, s) == inv
    # FP8 P.V: head dimension 128 only
    assert L.sage_attn_fwd_fp8pv(FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 64, 0, 0.1, 1, s) == uns
    # block-sparse: at most 512 key blocks; tau in (0, 1]; lambda > 0
    assert L.sage_attn_fwd_sparse(FAKE, FAKE, FAKE, FAKE, 1, 1, 65536 + 256, 64, 0, 0.1, 1, 0.9, 0.3, 20.0, s) == uns
    for tau in (0.0, -0.5, 1.5, float("nan")):
        assert L.sage_attn_fwd_sparse(FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 64, 0, 0.1, 1, tau, 0.3, 20.0, s) == inv
    for lam in (0.0, -1.0, float("nan")):
        assert L.sage_attn_fwd_sparse(FAKE, FAKE, FAKE, FAKE, 1, 1, 256, 128, 0, 0.1, 1, 0.9, 0.3, lam, s) == inv


def test_host_pipeline_validation(sa):
    # every failure below is found before any CUDA call (no GPU is needed)
    L = sa.get_lib()
    s = ctypes.c_void_p(0)
    ok_args = (1, 2, 256, 64, 0, 0.1, 1)
    assert L.sage_attn_fwd_host(None, FAKE, FAKE, FAKE, *ok_args, 0, s) == -1
    assert L.sage_attn_fwd_host(FAKE, FAKE, FAKE, None, *ok_args, 0, s) == -1
    assert L.sage_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, *ok_args, -1, s) == -1       # heads_per_chunk < 0
    assert L.sage_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 96, 0, 0.1, 1, 0, s) == -2  # d
    assert L.sage_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, 1, 2, 0, 64, 0, 0.1, 1, 0, s) == -1    # N
    assert L.sage_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 64, 0, float("nan"), 1, 0, s) == -1
    assert L.sage_attn_fwd_host(FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 64, 0, 0.1, 5, 0, s) == -1  # granularity
    V = L.sage_attn_fwd_host_variant
    assert V(FAKE, FAKE, FAKE, FAKE, *ok_args, 0, 3, s) == -1                            # unknown variant
    assert V(FAKE, FAKE, FAKE, FAKE, *ok_args, 0, -1, s) == -1
    assert V(FAKE, FAKE, FAKE, FAKE, *ok_args, 0, sa.SAGE_VARIANT_FP8PV, s) == -2       # FP8 P.V: d = 128 only
    assert V(FAKE, FAKE, FAKE, FAKE, 1, 2, 256, 96, 0, 0.1, 1, 0, sa.SAGE_VARIANT_FP4, s) == -2
    assert V(FAKE, FAKE, FAKE, None, *ok_args, 0, sa.SAGE_VARIANT_FP4, s) == -1


def test_binding_rejects_cpu_tensors(sa):
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        sa.sageattn(q, q, q)


def _declared_arity():
    """Parameter count of every function declared in include/sage_attn.h (comments stripped)."""
    import re
    from pathlib import Path
    root = Path(__file__).resolve().parents[1]
    text = (root / "include" / "sage_attn.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    out = {}
    for m in re.finditer(r"\b(sage_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_header(sa):
    """Every function the binding declares ctypes argument types for takes exactly as many
    arguments as its declaration in the header."""
    arity = _declared_arity()
    lib = sa.get_lib()
    checked = 0
    for name, n in arity.items():
        argtypes = getattr(lib, name).argtypes
        if argtypes is not None:
            assert len(argtypes) == n, (name, len(argtypes), n)
            checked += 1
    assert checked >= 12


def test_noalloc_validates_like_sage_attn_fwd(sa):
    # the allocation-free entry point returns the status sage_attn_fwd returns for the same
    # invalid arguments (both decide before any CUDA call)
    L = sa.get_lib()
    s = ctypes.c_void_p(0)
    mis = ctypes.c_void_p(0x1008)
    cases = [
        ((None, FAKE, FAKE, FAKE), (1, 1, 128, 64, 0, 0.1, 1)),
        ((FAKE,) * 4, (0, 1, 128, 64, 0, 0.1, 1)),
        ((FAKE,) * 4, (1, 1, 128, 96, 0, 0.1, 1)),
        ((FAKE,) * 4, (1, 1, 128, 96, 0, 0.1, 7)),          # bad d and granularity: d decides
        ((FAKE,) * 4, (4096, 4096, 1024, 128, 0, 0.1, 1)),
        ((FAKE,) * 4, (1, 1, 128, 64, 0, float("inf"), 1)),
        ((FAKE,) * 4, (1, 1, 128, 64, 0, float("nan"), 1)),
        ((FAKE,) * 4, (1, 1, 128, 64, 0, -0.5, 1)),
        ((FAKE,) * 4, (1, 1, 128, 64, 0, 0.0, 1)),
        ((FAKE,) * 4, (1, 1, 128, 64, 0, 0.1, 3)),
        ((FAKE, FAKE, mis, FAKE), (1, 1, 128, 64, 0, 0.1, 1)),
    ]
    for ptrs, args in cases:
        a = L.sage_attn_fwd(*ptrs, *args, s)
        b = L.sage_attn_fwd_noalloc(*ptrs, *args, s)
        assert a == b and a < 0, (args, a, b)
