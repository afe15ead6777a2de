"""The trace summary (quantized_attention_02_b200/trace.py) on a synthetic stamp array, on CPU.

Layout per CTA row: [0] start, [1] end, then for key tile j: softmax group t event e at
2 + (3t+e)*T + j (e: 0 S ready, 1 maximum done, 2 P~ signalled) and MMA event e of tile t at
2 + (6+2t+e)*T + j (e: 0 P.V issued, 1 next Q.K^T issued).
"""
import numpy as np

from quantized_attention_02_b200.trace import summarize


def _row(T, start, end, s, m, p, pv, qk):
    r = np.zeros(2 + 10 * T, dtype=np.int64)
    r[0], r[1] = start, end
    for t in range(2):
        for e, arr in enumerate((s, m, p)):
            r[2 + (3 * t + e) * T: 2 + (3 * t + e + 1) * T] = np.asarray(arr[t])
        for e, arr in enumerate((pv, qk)):
            r[2 + (6 + 2 * t + e) * T: 2 + (6 + 2 * t + e + 1) * T] = np.asarray(arr[t])
    return r


def test_summary_of_a_two_tile_trace():
    T = 2
    row = _row(T, 1000, 20000,
               s=[[1500, 5000], [1600, 5100]], m=[[2000, 5600], [2100, 5700]], p=[[4000, 8000], [4100, 8100]],
               pv=[[4500, 8500], [4600, 8400]], qk=[[4300, 0], [4400, 0]])
    out = summarize(np.stack([row, row]), T, causal=False)
    assert out["tile0"]["softmax"] == 2750.0      # median of 4000-1500 and 8000-5000
    assert out["tile0"]["head"] == 550.0          # median of 500 and 600
    assert out["tile0"]["period"] == 3500.0
    assert out["tile0"]["mma_wait"] == 1000.0     # 5000 - 4000
    assert out["prologue"] == 500.0               # start -> first S ready
    assert out["epilogue"] == 11500.0             # last event (P.V issued at 8500) -> end
    assert out["cta_cycles"] == 19000.0
    assert out["p1_minus_p0"] == 100.0
