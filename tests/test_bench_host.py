"""Host logic of bench.py's accuracy report, on CPU.

bench.py compares, outside its timed region, the library's output on the cpu_baseline sample's
head with the oracle rows that leg computes anyway.  Here a stand-in for the binding returns the
oracle's own fp16 output, so the report must show agreement; a stand-in that fails must give an
error entry instead of an exception (the bench line is never lost to the report).
"""
import types

import numpy as np
import torch

import oracle
import workloads as W


def _fake_binding(fail: bool = False):
    def sageattn(q, k, v, causal, sm_scale, gran):
        if fail:
            raise RuntimeError("no device")
        ref = oracle.sage_attn(q, k, v, causal, sm_scale, per_block=(gran == 1))
        return torch.from_numpy(ref["o16"].view(np.float16))
    return types.SimpleNamespace(SAGE_PER_TOKEN=0, SAGE_PER_BLOCK=1, sageattn=sageattn)


def test_accuracy_report_agrees_with_the_oracle_it_samples():
    import bench
    w = W.Workload("bench_acc_n256", 1, 2, 256, 64, True, True, n_out=4, out_mag=20.0)
    tops, cores, desc, sample = bench.oracle_sample(w, budget_s=0.5, keep=True)
    assert tops > 0 and cores >= 1 and "query rows" in desc
    acc = bench.sample_accuracy(_fake_binding(), w, sample, torch.device("cpu"))
    assert "error" not in acc, acc
    assert acc["rows"] == sample[3].size
    assert acc["max_abs_err_over_max_v"] <= 2e-3 and acc["cos_vs_oracle"] >= 0.9999
    assert acc["cos_vs_fp64_exact"] >= 0.995


def test_accuracy_report_never_raises():
    import bench
    w = W.Workload("bench_acc_fail", 1, 1, 128, 64, False, False)
    sample = bench.oracle_sample(w, budget_s=0.2, keep=True)[3]
    acc = bench.sample_accuracy(_fake_binding(fail=True), w, sample, torch.device("cpu"))
    assert set(acc) == {"error"} and "no device" in acc["error"]
