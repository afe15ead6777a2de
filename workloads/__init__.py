"""Seeded synthetic Q/K/V workloads shared by the tests, the oracle checks and
the benchmark.

This module holds no step of the attention method: it only draws random
tensors.  The shapes and value distributions stand in for the LLM and
video-DiT attention inputs the SageAttention page evaluates on (Summary; Key
points: "RTX3090 speedups" lists LLMs, CogvideoX video generation and TIMM);
no dataset or trained weights are used.  K carries a per-channel bias that is
constant over tokens -- the channel-wise outliers the page's Summary names as
the reason plain INT8 attention fails -- so that K smoothing has work to do.

Recipe (every config, one CPU torch.Generator seeded with ``seed``; draws in
this order, all in fp32, then rounded to fp16):
  1. Q      ~ N(0, q_std^2)                      shape [B,H,N,d]
  2. noise  ~ N(0, 1)                            shape [B,H,N,d]
  3. bias   ~ N(0, bias_std^2)                   shape [B,H,1,d]
  4. outlier channels: first n_out columns of a random permutation per (b,h)
  5. outlier signs: +-1 uniformly per (b,h, outlier)
  6. V      ~ N(0, 1)                            shape [B,H,N,d]
  K = noise + bias, where the outlier channels' bias is replaced by sign * mag.
Windowed (block-sparse) workloads, window > 0, draw one more tensor after V:
  7. u      ~ N(0, 1), each row scaled to unit length, shape [B,H,ceil(N/window),d]
  and add align * u[t // window] to both Q and K: tokens of one window share a direction, so the
  attention concentrates inside windows -- the locality of the video-DiT inputs the sparse
  attention pages evaluate on (SpargeAttn abstract: attention maps are often sparse).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    per_block: bool
    q_std: float = 1.0
    bias_std: float = 1.0
    n_out: int = 0
    out_mag: float = 0.0
    window: int = 0        # > 0: tokens in windows of this many share a direction of length align
    align: float = 0.0

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def ops(self) -> float:
        """Attention work 4 N^2 d B H, halved when causal."""
        w = 4.0 * self.N * self.N * self.d * self.B * self.H
        return w / 2 if self.causal else w

    def describe(self) -> str:
        g = "per-block 128Q/64K" if self.per_block else "per-token"
        return (f"B={self.B},H={self.H},N={self.N},d={self.d} {'causal' if self.causal else 'non-causal'}, "
                f"{g}, Q~N(0,{self.q_std}^2), K~N(0,1)+bias(N(0,{self.bias_std}^2)"
                + (f", {self.n_out} ch +-{self.out_mag:g}" if self.n_out else "") + "), V~N(0,1)"
                + (f", Q and K + {self.align:g} x a unit direction shared by each window of {self.window} tokens"
                   if self.window else ""))


# The five workload families: a tiny per-token case, a small causal per-block
# case, an LLM-shaped case, a video-DiT-shaped case and the N/d sweep.
TINY = Workload("tiny_d64_n256", 1, 2, 256, 64, False, False, n_out=4, out_mag=20.0)
SMALL = Workload("small_d128_n1024_causal", 1, 8, 1024, 128, True, True, n_out=8, out_mag=30.0)
LLM = Workload("llm_b4h32_n4096_d128_causal", 4, 32, 4096, 128, True, True, q_std=1.5,
               n_out=2, out_mag=40.0)
DIT = Workload("dit_b2h48_n16384_d64", 2, 48, 16384, 64, False, True, bias_std=4.0)


def sweep(N: int, d: int, causal: bool) -> Workload:
    """Sweep point: B=1, H = 2^20 / N (B*H*N = 2^20 tokens), 4 channels +-20."""
    H = (1 << 20) // N
    return Workload(f"sweep_n{N}_d{d}_{'causal' if causal else 'full'}", 1, H, N, d, causal, True,
                    n_out=4, out_mag=20.0)


SWEEP_N = (1024, 2048, 4096, 8192, 16384, 32768)
SWEEP_D = (64, 128)
HEADLINE = sweep(16384, 128, False)
# a quarter of the headline problem (inputs still larger than L2) for profiler captures
PROFILE = Workload("profile_b1h16_n16384_d128", 1, 16, 16384, 128, False, True, n_out=4, out_mag=20.0)
# the video-DiT shape with a sixth of its heads: small enough for a full profiler capture
PROFILE64 = Workload("profile_b1h16_n16384_d64", 1, 16, 16384, 64, False, True, bias_std=4.0)

# the headline sweep point with per-token scales (one per query / key token) instead of per-block
TOKEN128 = Workload("token_n16384_d128_full", 1, 64, 16384, 128, False, False, n_out=4, out_mag=20.0)
TOKEN64 = Workload("token_n16384_d64_full", 1, 64, 16384, 64, False, False, n_out=4, out_mag=20.0)

# block-sparse stand-in for the video-DiT attention maps (SpargeAttn abstract): the headline
# shape with windows of 2048 tokens (16 key tiles) whose Q and K share a direction of length 14
# (in-window scores about 17 above the rest, natural log units, at d^-1/2 = 0.088)
SPARSE = Workload("sparse_n16384_d128_win2048", 1, 64, 16384, 128, False, True, window=2048, align=14.0)
SPARSE_CAUSAL = Workload("sparse_n16384_d128_win2048_causal", 1, 64, 16384, 128, True, True, window=2048, align=14.0)

# the video-DiT shape (d = 64) with the same window structure: direction length 12 gives
# in-window scores about 18 above the rest at d^-1/2 = 0.125
SPARSE_DIT = Workload("sparse_dit_b2h48_n16384_d64_win2048", 2, 48, 16384, 64, False, True, bias_std=4.0,
                      window=2048, align=12.0)

# a quarter of the block-sparse workload's heads, for profiler captures
SPARSE_PROFILE = Workload("sparse_profile_b1h16_n16384_d128_win2048", 1, 16, 16384, 128, False, True, window=2048,
                          align=14.0)

ALL = {w.name: w for w in (TINY, SMALL, LLM, DIT, PROFILE, PROFILE64, TOKEN128, TOKEN64, SPARSE, SPARSE_CAUSAL,
                           SPARSE_DIT, SPARSE_PROFILE)}
for _n in SWEEP_N:
    for _d in SWEEP_D:
        for _c in (False, True):
            _w = sweep(_n, _d, _c)
            ALL[_w.name] = _w


def make_qkv(w: Workload, seed: int = 0):
    """Return (q, k, v) as contiguous CPU fp16 tensors of shape [B,H,N,d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (w.B, w.H, w.N, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32) * w.q_std
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    bias = torch.randn((w.B, w.H, 1, w.d), generator=g, dtype=torch.float32) * w.bias_std
    if w.n_out:
        perm = torch.argsort(torch.rand((w.B, w.H, w.d), generator=g), dim=-1)[..., : w.n_out]
        signs = torch.randint(0, 2, (w.B, w.H, w.n_out), generator=g).to(torch.float32) * 2 - 1
        bias.view(w.B, w.H, w.d).scatter_(-1, perm, signs * w.out_mag)
    k += bias
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.window:
        n_win = -(-w.N // w.window)
        u = torch.randn((w.B, w.H, n_win, w.d), generator=g, dtype=torch.float32)
        u = u / u.norm(dim=-1, keepdim=True)
        shared = u[:, :, torch.arange(w.N) // w.window] * w.align
        q += shared
        k += shared
    return q.half().contiguous(), k.half().contiguous(), v.half().contiguous()


def head_slice(x: torch.Tensor, heads) -> torch.Tensor:
    """Select flat (b*H + h) head indices from a [B,H,N,d] tensor -> [len, N, d]."""
    B, H, N, d = x.shape
    return x.reshape(B * H, N, d)[list(heads)].contiguous()
