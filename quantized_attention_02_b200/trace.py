"""Pipeline trace of the fused attention kernel.

    python -m quantized_attention_02_b200.trace [--workload NAME] [--ctas C]

Runs ``sage_debug_attn_trace`` (the fused kernel built with SM clock stamps) on a
synthetic workload and summarises, over the traced CTAs and the steady-state key tiles,
where a softmax warpgroup spends its cycles:

  softmax   S ready -> P~ signalled           (TMEM loads, max, exp2, P~ store)
  head      S ready -> max / offset done      (part of softmax)
  mma_wait  P~ signalled -> next S ready      (P.V + next Q.K^T on the tensor core, plus
                                               the signalling latency both ways)
  period    S ready -> next S ready           (one key tile for one query tile)
  prologue  CTA start -> first S ready       (set-up, first loads, first Q.K^T)
  epilogue  last event -> CTA end            (last P.V, normalisation and store, final barrier)

and the kernel-wide rate: cycles per (query tile x key tile) per SM.
"""
from __future__ import annotations

import argparse
import json
import sys

import numpy as np
import torch


def run(workload, ctas: int = 8):
    import workloads as W

    import quantized_attention_02_b200 as sa

    w = workload
    gran = sa.SAGE_PER_BLOCK
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    km, q8, k8, sq, sk = sa.empty_quantized(q, gran)
    sa.sage_smooth_k(k, km)
    sa.sage_quant_qk(q, k, km, q8, k8, sq, sk, gran)
    o = torch.empty_like(q)
    T = w.N // 128
    tr = torch.zeros((ctas, 2 + 10 * T), dtype=torch.int64, device="cuda")
    for _ in range(2):  # warm-up, then the traced run
        tr.zero_()
        sa.sage_debug_attn_trace(q8, k8, sq, sk, v, o, w.causal, w.sm_scale, gran, tr, ctas)
    torch.cuda.synchronize()
    if sa.sage_last_device_error() != 0:
        raise RuntimeError("kernel wait timed out")
    return summarize(tr.cpu().numpy(), T, w.causal)


def summarize(tr: np.ndarray, T: int, causal: bool) -> dict:
    def ev(t, e):
        return tr[:, 2 + (3 * t + e) * T: 2 + (3 * t + e + 1) * T]

    def mma(t, e):
        return tr[:, 2 + (6 + 2 * t + e) * T: 2 + (6 + 2 * t + e + 1) * T]

    out = {}
    for t in range(2):
        s_ready, max_done, p_sig = ev(t, 0), ev(t, 1), ev(t, 2)
        pv_iss, qk_iss = mma(t, 0), mma(t, 1)
        valid = (s_ready[:, 1:] > 0) & (p_sig[:, :-1] > 0)
        sm = (p_sig - s_ready)[s_ready > 0]
        hd = (max_done - s_ready)[s_ready > 0]
        wait = (s_ready[:, 1:] - p_sig[:, :-1])[valid]
        per = (s_ready[:, 1:] - s_ready[:, :-1])[valid]
        react = (pv_iss - p_sig)[(pv_iss > 0) & (p_sig > 0)]
        tens = (s_ready[:, 1:] - qk_iss[:, :-1])[valid & (qk_iss[:, :-1] > 0)]
        out[f"tile{t}"] = {"softmax": float(np.median(sm)), "head": float(np.median(hd)),
                           "mma_wait": float(np.median(wait)), "period": float(np.median(per)),
                           "mma_react": float(np.median(react)) if react.size else None,
                           "qk_issue_to_s_ready": float(np.median(tens)) if tens.size else None}
    # phase of the two groups: P~ of tile 1 relative to P~ of tile 0 for the same key tile
    p0, p1 = ev(0, 2), ev(1, 2)
    both = (p0 > 0) & (p1 > 0)
    out["p1_minus_p0"] = float(np.median((p1 - p0)[both])) if both.any() else None
    dur = tr[:, 1] - tr[:, 0]
    n_tiles = 2 * (T if not causal else (T + 1) // 2)
    # per CTA: start -> first S ready (set-up, first loads, first Q.K^T) and last recorded event
    # -> end (last P.V, epilogue, final barrier); the end stamp is taken after the CTA barrier
    big = np.iinfo(np.int64).max
    s0, s1 = ev(0, 0)[:, 0], ev(1, 0)[:, 0]
    first_s = np.minimum(np.where(s0 > 0, s0, big), np.where(s1 > 0, s1, big))
    last = np.where(tr[:, 2:] > 0, tr[:, 2:], 0).max(axis=1)
    out["prologue"] = float(np.median(first_s - tr[:, 0]))
    out["epilogue"] = float(np.median(tr[:, 1] - last))
    out["cta_cycles"] = float(np.median(dur))
    out["cycles_per_tile_pair"] = float(np.median(dur)) / max(1, (T if not causal else T // 2))
    out["note"] = "cycles are SM clocks; 'cycles_per_tile_pair' = CTA cycles / key tiles (2 query tiles each)"
    out["tiles_per_cta"] = n_tiles
    return out


def main(argv=None) -> int:
    import workloads as W

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default=W.PROFILE.name, choices=sorted(W.ALL))
    ap.add_argument("--ctas", type=int, default=8)
    a = ap.parse_args(argv)
    print(json.dumps(run(W.ALL[a.workload], a.ctas), indent=1))
    return 0


if __name__ == "__main__":
    sys.exit(main())
