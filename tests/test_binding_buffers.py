"""Host-side checks of the Python binding's buffer helpers and the high-level entry point (no GPU):
the shapes empty_fp4 / empty_quantized allocate are the layouts include/sage_attn.h documents, for
both head dimensions, and sageattn rejects an unknown variant before any CUDA call."""
import pytest
import torch

import quantized_attention_02_b200 as sa


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 64, 65, 200, 256])
def test_empty_fp4_shapes_follow_the_header(N, d):
    B, H = 2, 3
    q = torch.zeros((B, H, N, d), dtype=torch.float16)
    b = sa.empty_fp4(q)
    t, a = (N + 127) // 128, d // 64
    want = {
        "q4": (B, H, N, d // 2), "k4": (B, H, N, d // 2),
        "sfq": (B, H, t, a, 512), "sfk": (B, H, (N + 63) // 64, a, 512), "sfv": (B, H, t, 2, 512),
        "gq": (B, H, t), "gk": (B, H, t), "v4t": (B, H, d, t * 64),
        "gv": (B, H, d), "vm": (B, H, d), "km": (B, H, d),
    }
    assert set(b) == set(want)
    for name, shape in want.items():
        assert tuple(b[name].shape) == shape, name
    assert b["q4"].dtype == torch.uint8 and b["sfk"].dtype == torch.uint8 and b["gq"].dtype == torch.float32
    assert sa.empty_fp4(q, smooth_v=False)["vm"] is None


@pytest.mark.parametrize("gran", [sa.SAGE_PER_TOKEN, sa.SAGE_PER_BLOCK])
def test_empty_quantized_shapes(gran):
    q = torch.zeros((1, 2, 300, 64), dtype=torch.float16)
    km, q8, k8, sq, sk = sa.empty_quantized(q, gran)
    assert km.shape == (1, 2, 64) and q8.shape == k8.shape == (1, 2, 300, 64) and q8.dtype == torch.int8
    if gran == sa.SAGE_PER_TOKEN:
        assert sq.shape == sk.shape == (1, 2, 300)
    else:  # one scale per 128 Q tokens / 64 K tokens
        assert sq.shape == (1, 2, 3) and sk.shape == (1, 2, 5)


def test_sageattn_rejects_an_unknown_variant():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.float16)
    with pytest.raises(ValueError):
        sa.sageattn(q, q, q, variant="int4")


def test_binding_constants_match_the_header():
    import re
    text = open(sa.HEADER_PATH).read()
    consts = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(SAGE_[A-Z0-9_]+)\s*=\s*(-?\d+)", text)}
    for name in ("SAGE_PER_TOKEN", "SAGE_PER_BLOCK", "SAGE_VARIANT_FP16PV", "SAGE_VARIANT_FP8PV", "SAGE_VARIANT_FP4",
                 "SAGE_OK", "SAGE_ERR_INVALID", "SAGE_ERR_UNSUPPORTED"):
        assert getattr(sa, name) == consts[name], name
