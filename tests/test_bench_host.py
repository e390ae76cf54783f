"""Host-side accounting of bench.py, on the CPU.

The CPU baseline converts the oracle's time on a sample of query rows into
pairs per second with bench.allowed_keys (keys a row may attend to under a
workload's mask).  Summed over every row of a head it must equal the pair
count of the oracle's brute-force mask enumeration, for every mask kind the
workloads use.  The exponential-unit ceiling and the sustained figures are
plain arithmetic on the measured peaks, checked here as well."""
import dataclasses

import numpy as np
import pytest

import bench
from io_aware_exact_34_b200 import synth


@pytest.mark.parametrize("Lq,Lk,causal,wl,wr", [
    (300, 300, False, -1, -1), (300, 300, True, -1, -1), (257, 257, False, 40, 40),
    (400, 400, True, 100, 0), (129, 300, True, -1, -1), (300, 129, True, -1, -1),
    (200, 200, False, 0, 0), (333, 333, False, 17, 5), (64, 64, True, 1000, 0)])
def test_allowed_keys_sum_to_pair_count(oracle, Lq, Lk, causal, wl, wr):
    w = synth.Workload("adhoc", "prefill", 1, 1, Lq, Lk, 64, "bf16", causal=causal, window_left=wl,
                       window_right=wr)
    per_row = bench.allowed_keys(w, np.arange(Lq))
    assert per_row.min() >= 0
    assert int(per_row.sum()) == oracle.count_blocks(Lq, Lk, causal, wl, wr, 128, 128)["pairs"]


def test_allowed_keys_on_the_workloads(oracle):
    # the long workloads at a reduced length (same masks), and the headline as it is
    for name, L in [("window_bidir_32k", 8192), ("window_causal_32k", 8192), ("causal_64k_qscale", 4096),
                    ("causal_4k", 4096)]:
        w = dataclasses.replace(synth.WORKLOADS[name], Lq=L, Lk=L)
        total = int(bench.allowed_keys(w, np.arange(L)).sum())
        assert total == oracle.count_blocks(L, L, w.causal, w.window_left, w.window_right, 128, 128)["pairs"]


PEAKS = {"hbm_gbs": 6543.4, "bf16_tflops": 1683.0, "bf16_tflops_sustained": 1390.2}


def test_exp_ceiling_is_d_over_128_of_the_tensor_peak():
    # 16 exp2 per clock per SM against 8192 bf16 FLOPs, 4 d FLOPs per pair
    for d in (64, 128):
        r = bench.exp_roofline(500.0, PEAKS, "measured", d)
        assert r["bound"] == "alu"
        assert r["peak"] == pytest.approx(PEAKS["bf16_tflops"] * 16 * 4 * d / 8192)
        assert r["frac"] == pytest.approx(500.0 / r["peak"])


def test_sustained_entry_against_the_sustained_peak():
    flops = 2.749e11
    e = bench.sustained_entry(2, 0.25, flops, PEAKS)
    per_gpu = flops / 0.25e-3 / 1e12
    assert e["value"] == pytest.approx(2 * per_gpu)           # whole job over the ranks
    assert e["frac"] == pytest.approx(per_gpu / PEAKS["bf16_tflops_sustained"])
    e8 = bench.sustained_entry(1, 0.25, flops, PEAKS, 2.0)
    assert e8["peak"] == pytest.approx(2 * PEAKS["bf16_tflops_sustained"])
    assert bench.sustained_entry(1, None, flops, PEAKS) is None


def test_no_sustained_switch_skips_the_soak(monkeypatch):
    calls = []
    monkeypatch.setattr(bench, "SUSTAINED", False)
    assert bench.timed_sustained(1, lambda: calls.append(1), 5) is None
    assert calls == []
