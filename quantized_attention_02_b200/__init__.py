"""Python binding of the B200 SageAttention-style 8-bit attention library.

Argument marshalling only: every step of the method runs in the CUDA kernels of
``libsage_attn.so`` (built in-tree by ``python -m quantized_attention_02_b200.build``).
The functions mirror the C ABI of ``include/sage_attn.h`` one to one and take
torch CUDA tensors, passing their device pointers and the current CUDA stream.
There is no CPU fallback: a missing library raises at import time, and a call
on tensors that are not on a CUDA device raises before anything is launched.

The method follows "SageAttention: Accurate 8-Bit Attention for Plug-and-play
Inference Acceleration" (research.elamur.ai summary page, Summary and idea I1).
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage_attn.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "sage_attn.h")

SAGE_OK = 0
SAGE_ERR_INVALID = -1
SAGE_ERR_UNSUPPORTED = -2
SAGE_ERR_CUDA = -3
SAGE_ERR_TIMEOUT = -4
SAGE_ERR_NOMEM = -5
SAGE_ERR_TOO_LARGE = -6
SAGE_PER_TOKEN = 0
SAGE_PER_BLOCK = 1

_lib = None


def get_lib() -> ctypes.CDLL:
    """The loaded libsage_attn.so (loaded on first use; raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m quantized_attention_02_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        _i, _f, _p, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
        lib.sage_status_string.argtypes = [_i]
        lib.sage_status_string.restype = ctypes.c_char_p
        lib.sage_scale_count.argtypes = [_i, _i, _i]
        lib.sage_scale_count.restype = _sz
        lib.sage_smooth_k.argtypes = [_p, _p, _i, _i, _i, _i, _p]
        lib.sage_quant_qk.argtypes = [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
        lib.sage_attn_fwd.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _p]
        lib.sage_attn_fwd_quantized.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _p]
        lib.sage_debug_qk_int32.argtypes = [_p, _p, _p, _i, _i, _i, _i, _p]
        lib.sage_quant_v_fp8.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _p]
        lib.sage_prep_qk.argtypes = [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p]
        lib.sage_attn_fwd_fp8pv_quantized.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _p]
        lib.sage_attn_fwd_fp8pv.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _p]
        lib.sage_quant_qk_fp4.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _p]
        lib.sage_quant_v_fp4.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _p]
        lib.sage_attn_fwd_fp4_quantized.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i,
                                                    _f, _p]
        lib.sage_attn_fwd_fp4.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _p]
        lib.sage_sparse_predict.argtypes = [_p, _p, _i, _i, _i, _i, _i, _f, _f, _f, _p, _p, _p]
        lib.sage_attn_fwd_sparse_quantized.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _p, _p, _f,
                                                       _p]
        lib.sage_attn_fwd_sparse.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _f, _f, _f, _p]
        lib.sage_last_device_error.argtypes = [_p]
        lib.sage_attn_fwd_noalloc.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _p]
        lib.sage_noalloc_scratch_bytes.argtypes = [_i, _i, _i, _i, _i]
        lib.sage_noalloc_scratch_bytes.restype = _sz
        lib.sage_debug_attn_trace.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _p, _i, _p]
        lib.sage_debug_mma_peak.argtypes = [_i, _i, _i, _p, _p, _p]
        lib.sage_debug_wait_timeout.argtypes = [_p, _p]
        lib.sage_attn_fwd_host.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _i, _p]
        lib.sage_attn_fwd_host_variant.argtypes = [_p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _i, _i, _i, _p]
        for n in ("sage_smooth_k", "sage_quant_qk", "sage_attn_fwd", "sage_attn_fwd_quantized",
                  "sage_debug_qk_int32", "sage_last_device_error", "sage_attn_fwd_noalloc",
                  "sage_debug_attn_trace", "sage_debug_mma_peak", "sage_attn_fwd_host",
                  "sage_debug_wait_timeout", "sage_quant_v_fp8", "sage_attn_fwd_fp8pv_quantized", "sage_prep_qk",
                  "sage_attn_fwd_fp8pv", "sage_sparse_predict", "sage_attn_fwd_sparse_quantized",
                  "sage_attn_fwd_sparse", "sage_attn_fwd_host_variant", "sage_quant_qk_fp4", "sage_quant_v_fp4",
                  "sage_attn_fwd_fp4_quantized", "sage_attn_fwd_fp4"):
            getattr(lib, n).restype = _i
        _lib = lib
    return _lib


class SageError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {sage_status_string(status)} ({status})")
        self.status = status


def header_functions() -> list[str]:
    """Names of the functions declared in include/sage_attn.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))


def sage_status_string(status: int) -> str:
    return get_lib().sage_status_string(int(status)).decode()


def sage_scale_count(N: int, granularity: int, is_q: bool) -> int:
    return int(get_lib().sage_scale_count(int(N), int(granularity), int(bool(is_q))))


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _shape(x: torch.Tensor):
    if x.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    return tuple(int(s) for s in x.shape)


def _check(rc: int, where: str) -> None:
    if rc != SAGE_OK:
        raise SageError(rc, where)


def sage_smooth_k(k: torch.Tensor, km: torch.Tensor, stream=None) -> None:
    B, H, N, d = _shape(k)
    _check(get_lib().sage_smooth_k(_ptr(k), _ptr(km), B, H, N, d, _stream(stream)), "sage_smooth_k")


def sage_quant_qk(q, k, km, q8, k8, sq, sk, granularity: int, stream=None) -> None:
    B, H, N, d = _shape(q)
    _check(get_lib().sage_quant_qk(_ptr(q), _ptr(k), _ptr(km), _ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk),
                             B, H, N, d, int(granularity), _stream(stream)), "sage_quant_qk")


def sage_prep_qk(q, k, km, q8, k8, sq, sk, granularity: int, stream=None) -> None:
    """K mean, K and Q codes and scales in one launch (the results of sage_smooth_k then sage_quant_qk)."""
    B, H, N, d = _shape(q)
    _check(get_lib().sage_prep_qk(_ptr(q), _ptr(k), _ptr(km), _ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), B, H, N, d,
                                  int(granularity), _stream(stream)), "sage_prep_qk")


def sage_attn_fwd(q, k, v, o, causal: bool, sm_scale: float, granularity: int, stream=None) -> None:
    B, H, N, d = _shape(q)
    _check(get_lib().sage_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, int(bool(causal)),
                             float(sm_scale), int(granularity), _stream(stream)), "sage_attn_fwd")


def sage_attn_fwd_quantized(q8, k8, sq, sk, v, o, causal: bool, sm_scale: float, granularity: int,
                            stream=None) -> None:
    B, H, N, d = _shape(v)
    _check(get_lib().sage_attn_fwd_quantized(_ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), _ptr(v), _ptr(o), B, H, N,
                                       d, int(bool(causal)), float(sm_scale), int(granularity),
                                       _stream(stream)), "sage_attn_fwd_quantized")


def sage_quant_v_fp8(v, v8, sv, vm=None, stream=None) -> None:
    """V to E4M3 codes (uint8 tensor) with per-(head, channel) scales sv; channel means into vm
    (V smoothed) unless vm is None (FP8 P.V variant, SageAttention2 abstract)."""
    B, H, N, d = _shape(v)
    _check(get_lib().sage_quant_v_fp8(_ptr(v), _ptr(v8), _ptr(sv), _ptr(vm), B, H, N, d, _stream(stream)),
           "sage_quant_v_fp8")


def sage_attn_fwd_fp8pv_quantized(q8, k8, sq, sk, v8, sv, vm, o, causal: bool, sm_scale: float, granularity: int,
                                  stream=None) -> None:
    B, H, N, d = _shape(o)
    _check(get_lib().sage_attn_fwd_fp8pv_quantized(_ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), _ptr(v8), _ptr(sv),
                                                   _ptr(vm), _ptr(o), B, H, N, d, int(bool(causal)), float(sm_scale),
                                                   int(granularity), _stream(stream)),
           "sage_attn_fwd_fp8pv_quantized")


def sage_attn_fwd_fp8pv(q, k, v, o, causal: bool, sm_scale: float, granularity: int, stream=None) -> None:
    B, H, N, d = _shape(q)
    _check(get_lib().sage_attn_fwd_fp8pv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, int(bool(causal)),
                                         float(sm_scale), int(granularity), _stream(stream)), "sage_attn_fwd_fp8pv")


def fp4_tiles(N: int) -> int:
    """Tiles of 128 tokens of the microscaling FP4 variant: ceil(N/128)."""
    return (N + 127) // 128


def empty_fp4(q, smooth_v: bool = True) -> dict:
    """Device buffers of the FP4 variant's quantized operands for q-shaped [B,H,N,d] inputs
    (d = 64 or 128, A = d/64 scale atoms per row group): q4/k4 uint8 [B,H,N,d/2], sfq uint8
    [B,H,tiles,A,512], sfk uint8 [B,H,ceil(N/64),A,512], sfv uint8 [B,H,tiles,2,512], gq/gk fp32
    [B,H,tiles], v4t uint8 [B,H,d,tiles*64], gv/vm fp32 [B,H,d] (vm None when not smoothed), km
    fp32 [B,H,d]."""
    B, H, N, d = _shape(q)
    t = fp4_tiles(N)
    a = d // 64
    u8 = dict(dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    return dict(q4=torch.empty((B, H, N, d // 2), **u8), k4=torch.empty((B, H, N, d // 2), **u8),
                sfq=torch.empty((B, H, t, a, 512), **u8), sfk=torch.empty((B, H, (N + 63) // 64, a, 512), **u8),
                sfv=torch.empty((B, H, t, 2, 512), **u8), gq=torch.empty((B, H, t), **f32),
                gk=torch.empty((B, H, t), **f32), v4t=torch.empty((B, H, d, t * 64), **u8),
                gv=torch.empty((B, H, d), **f32), vm=torch.empty((B, H, d), **f32) if smooth_v else None,
                km=torch.empty((B, H, d), **f32))


def sage_quant_qk_fp4(q, k, km, q4, sfq, gq, k4, sfk, gk, stream=None) -> None:
    """Q and K (minus km unless None) to E2M1 codes with UE4M3 scale atoms and fp32 tile scales
    (microscaling FP4 variant, SageAttention3 entry: title and abstract)."""
    B, H, N, d = _shape(q)
    _check(get_lib().sage_quant_qk_fp4(_ptr(q), _ptr(k), _ptr(km), _ptr(q4), _ptr(sfq), _ptr(gq), _ptr(k4), _ptr(sfk),
                                       _ptr(gk), B, H, N, d, _stream(stream)), "sage_quant_qk_fp4")


def sage_quant_v_fp4(v, v4t, sfv, gv, vm=None, stream=None) -> None:
    """V to E2M1 codes along the tokens (transposed), UE4M3 scale atoms, fp32 channel scales;
    channel means into vm (V smoothed) unless vm is None."""
    B, H, N, d = _shape(v)
    _check(get_lib().sage_quant_v_fp4(_ptr(v), _ptr(v4t), _ptr(sfv), _ptr(gv), _ptr(vm), B, H, N, d, _stream(stream)),
           "sage_quant_v_fp4")


def sage_attn_fwd_fp4_quantized(q4, sfq, gq, k4, sfk, gk, v4t, sfv, gv, vm, o, causal: bool, sm_scale: float,
                                stream=None) -> None:
    B, H, N, d = _shape(o)
    _check(get_lib().sage_attn_fwd_fp4_quantized(_ptr(q4), _ptr(sfq), _ptr(gq), _ptr(k4), _ptr(sfk), _ptr(gk),
                                                 _ptr(v4t), _ptr(sfv), _ptr(gv), _ptr(vm), _ptr(o), B, H, N, d,
                                                 int(bool(causal)), float(sm_scale), _stream(stream)),
           "sage_attn_fwd_fp4_quantized")


def sage_attn_fwd_fp4(q, k, v, o, causal: bool, sm_scale: float, stream=None) -> None:
    """The whole microscaling FP4 variant (smooth K, FP4 Q, K and V, the fused FP4 kernel)."""
    B, H, N, d = _shape(q)
    _check(get_lib().sage_attn_fwd_fp4(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, int(bool(causal)),
                                       float(sm_scale), _stream(stream)), "sage_attn_fwd_fp4")


def sparse_blocks(N: int) -> tuple[int, int]:
    """(query blocks, key blocks) of the block-sparse variant: ceil(N/256), ceil(N/128)."""
    return (N + 255) // 256, (N + 127) // 128


def sage_sparse_predict(q, k, causal: bool, sm_scale: float, tau: float, theta: float, kv_count, kv_index,
                        stream=None) -> None:
    """Stage 1 of the block-sparse variant (SpargeAttn abstract): kv_count int32 [B,H,QB] and
    kv_index int16 [B,H,QB,KB] receive each query block's kept key blocks."""
    B, H, N, d = _shape(q)
    _check(get_lib().sage_sparse_predict(_ptr(q), _ptr(k), B, H, N, d, int(bool(causal)), float(sm_scale), float(tau),
                                         float(theta), _ptr(kv_count), _ptr(kv_index), _stream(stream)),
           "sage_sparse_predict")


def sage_attn_fwd_sparse_quantized(q8, k8, sq, sk, v, o, causal: bool, sm_scale: float, granularity: int, kv_count,
                                   kv_index, skip_lambda: float, stream=None) -> None:
    B, H, N, d = _shape(v)
    _check(get_lib().sage_attn_fwd_sparse_quantized(_ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), _ptr(v), _ptr(o), B, H, N,
                                                    d, int(bool(causal)), float(sm_scale), int(granularity),
                                                    _ptr(kv_count), _ptr(kv_index), float(skip_lambda),
                                                    _stream(stream)), "sage_attn_fwd_sparse_quantized")


def sage_attn_fwd_sparse(q, k, v, o, causal: bool, sm_scale: float, granularity: int, tau: float, theta: float,
                         skip_lambda: float, stream=None) -> None:
    B, H, N, d = _shape(q)
    _check(get_lib().sage_attn_fwd_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, int(bool(causal)),
                                          float(sm_scale), int(granularity), float(tau), float(theta),
                                          float(skip_lambda), _stream(stream)), "sage_attn_fwd_sparse")


def sage_debug_qk_int32(q8, k8, s, stream=None) -> None:
    B, H, N, d = _shape(q8)
    _check(get_lib().sage_debug_qk_int32(_ptr(q8), _ptr(k8), _ptr(s), B, H, N, d, _stream(stream)),
           "sage_debug_qk_int32")


def sage_debug_attn_trace(q8, k8, sq, sk, v, o, causal: bool, sm_scale: float, granularity: int, trace,
                          trace_ctas: int, stream=None) -> None:
    """sage_attn_fwd_quantized with pipeline clock stamps (see include/sage_attn.h)."""
    B, H, N, d = _shape(v)
    _check(get_lib().sage_debug_attn_trace(_ptr(q8), _ptr(k8), _ptr(sq), _ptr(sk), _ptr(v), _ptr(o), B, H, N, d,
                                           int(bool(causal)), float(sm_scale), int(granularity), _ptr(trace),
                                           int(trace_ctas), _stream(stream)), "sage_debug_attn_trace")


MMA_PEAK_KINDS = {0: ("kind::i8", 32), 1: ("kind::f16", 16), 2: ("kind::f8f6f4 e4m3", 32)}


def mma_peak(kind: int, iters: int = 4096) -> dict:
    """Dense tensor-core rate of this GPU for one MMA kind (0 = INT8, 1 = FP16, 2 = FP8 E4M3):
    one CTA per SM, two warps issuing M=128 N=256 MMAs back to back.  Returns multiply-
    accumulates per SM clock and the whole-GPU rate in TOPS (2 ops per multiply-accumulate,
    CUDA events on the current stream, at whatever clock the GPU runs)."""
    dev = torch.cuda.current_device()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    name, K = MMA_PEAK_KINDS[kind]
    st = torch.cuda.current_stream()
    lib = get_lib()
    _check(lib.sage_debug_mma_peak(kind, 64, sms, _ptr(cycles), _ptr(status), _stream(st)), "mma_peak")  # warm-up
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    _check(lib.sage_debug_mma_peak(kind, iters, sms, _ptr(cycles), _ptr(status), _stream(st)), "mma_peak")
    e1.record(st)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError("mma_peak wait gave up")
    macs = 2 * iters * 128 * 256 * K  # per CTA: two warps
    cyc = float(cycles.double().median())
    return {"kind": name, "shape": [128, 256, K], "macs_per_clk_per_sm": macs / cyc,
            "tops": 2.0 * macs * sms / (e0.elapsed_time(e1) * 1e-3) / 1e12}


def sage_attn_fwd_noalloc(q, k, v, o, causal: bool, sm_scale: float, granularity: int, stream=None) -> None:
    """sage_attn_fwd for callers that cannot allocate device memory during the call: the
    workspace is the library's fixed scratch array (SAGE_NOALLOC_SCRATCH_BYTES per GPU).
    Calls that overlap on the GPU race on that array."""
    B, H, N, d = _shape(q)
    _check(get_lib().sage_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, int(bool(causal)),
                                     float(sm_scale), int(granularity), _stream(stream)),
           "sage_attn_fwd_noalloc")


def _host_ptr(t):
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if t.is_cuda:
        raise ValueError("sage_attn_fwd_host takes host tensors (pinned memory lets the copies overlap)")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if t.dtype != torch.float16:
        raise ValueError("expected float16")
    return ctypes.c_void_p(t.data_ptr())


SAGE_VARIANT_FP16PV, SAGE_VARIANT_FP8PV, SAGE_VARIANT_FP4 = 0, 1, 2
_VARIANT_CODES = {"fp16pv": SAGE_VARIANT_FP16PV, "fp8pv": SAGE_VARIANT_FP8PV, "fp4": SAGE_VARIANT_FP4}


def sage_attn_fwd_host(q, k, v, o, causal: bool, sm_scale: float, granularity: int, heads_per_chunk: int = 0,
                       stream=None, variant: str = "fp16pv") -> None:
    """Whole forward pass on HOST tensors [B, H, N, d] (fp16): copies in, compute and copies
    out overlap across chunks of heads.  variant: "fp16pv" (the method), "fp8pv" or "fp4".
    Asynchronous on `stream` (the current CUDA stream by default): synchronize it before reading
    o or changing q, k, v."""
    if variant not in _VARIANT_CODES:
        raise ValueError(f"variant must be one of {tuple(_VARIANT_CODES)}, not {variant!r}")
    B, H, N, d = _shape(q)
    for t in (k, v, o):
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError("q, k, v, o must have the same shape")
    _check(get_lib().sage_attn_fwd_host_variant(_host_ptr(q), _host_ptr(k), _host_ptr(v), _host_ptr(o), B, H, N, d,
                                                int(bool(causal)), float(sm_scale), int(granularity),
                                                int(heads_per_chunk), _VARIANT_CODES[variant], _stream(stream)),
           "sage_attn_fwd_host_variant")


def sage_noalloc_scratch_bytes(B: int, H: int, N: int, d: int, granularity: int) -> int:
    return int(get_lib().sage_noalloc_scratch_bytes(B, H, N, d, granularity))


def sage_last_device_error(stream=None) -> int:
    return int(get_lib().sage_last_device_error(_stream(stream)))


def sage_debug_wait_timeout(gave_up: torch.Tensor, stream=None) -> None:
    """One warp waits, with the pipelines' bounded wait, on an mbarrier that nothing arrives on;
    gave_up (int32 [1], CUDA) receives 0 when the wait gave up."""
    _check(get_lib().sage_debug_wait_timeout(_ptr(gave_up), _stream(stream)), "sage_debug_wait_timeout")


# ------------------------------------------------------------------ conveniences
def empty_quantized(q: torch.Tensor, granularity: int):
    """Allocate (km, q8, k8, sq, sk) for inputs shaped like q."""
    B, H, N, d = _shape(q)
    dev = q.device
    km = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    q8 = torch.empty((B, H, N, d), dtype=torch.int8, device=dev)
    k8 = torch.empty((B, H, N, d), dtype=torch.int8, device=dev)
    sq = torch.empty((B, H, sage_scale_count(N, granularity, True)), dtype=torch.float32, device=dev)
    sk = torch.empty((B, H, sage_scale_count(N, granularity, False)), dtype=torch.float32, device=dev)
    return km, q8, k8, sq, sk


VARIANTS = ("fp16pv", "fp8pv", "fp4", "sparse")


def sageattn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
             sm_scale: float | None = None, granularity: int = SAGE_PER_BLOCK, variant: str = "fp16pv",
             stream=None, tau: float = 0.99, theta: float = 0.3, skip_lambda: float = 20.0) -> torch.Tensor:
    """O = softmax(Q K^T sm_scale) V on fp16 [B, H, N, d] CUDA tensors; sm_scale defaults to d^-1/2.
    variant: "fp16pv" the method (smoothed K, INT8 Q K^T with per-token or per-block scales, FP16 P V);
    "fp8pv" its FP8 P~ V variant (E4M3 P~ and smoothed V; d = 128); "fp4" the microscaling FP4 variant
    (E2M1 Q, K, P~, V with UE4M3 scales per 16 elements; granularity does not apply); "sparse" the
    block-sparse variant (stage 1 keeps the key blocks reaching cumulative probability tau, theta the
    self-similarity below which a block is always kept; stage 2 drops a block whose scores all lie
    skip_lambda log2 units below the running row maximum; N <= 65536)."""
    if variant not in VARIANTS:
        raise ValueError(f"variant must be one of {VARIANTS}, not {variant!r}")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(q.shape[-1])
    o = torch.empty_like(q)
    if variant == "fp4":
        sage_attn_fwd_fp4(q, k, v, o, causal, sm_scale, stream)
    elif variant == "sparse":
        sage_attn_fwd_sparse(q, k, v, o, causal, sm_scale, granularity, tau, theta, skip_lambda, stream)
    elif variant == "fp8pv":
        sage_attn_fwd_fp8pv(q, k, v, o, causal, sm_scale, granularity, stream)
    else:
        sage_attn_fwd(q, k, v, o, causal, sm_scale, granularity, stream)
    return o
