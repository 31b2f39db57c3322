"""Host-side pieces of bench.py on CPU: the CPU-oracle baseline records (core counts, the
measured or extrapolated full-problem time) and the choice of roofline peak per kernel."""
import dataclasses
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)


@pytest.mark.parametrize("name", ["oracle_1280", "train_480p_fwd_bwd", "q8_720p", "wan1.3b_480p_cfg"])
def test_cpu_baseline_record(name):
    import bench
    import synth
    w = dataclasses.replace(synth.WORKLOADS[name], S=200, H=2, name=f"{name}@small")
    r = bench.cpu_baseline(w, 8)
    assert r["kind"] == "oracle" and r["unit"] == "TFLOP/s" and r["value"] > 0
    assert r["cores"] >= 1 and r["nproc"] >= 1 and 1 <= r["cpus_allowed"] <= r["nproc"]
    full = w.fwd_flop * (3.5 if w.backward else 1.0)
    assert r["full_problem_s_extrapolated"] == pytest.approx(full / (r["_flop"] / r["sample_s"]))
    everything = bench.cpu_baseline(w, 200)           # every row of a forward is the full problem
    if not w.backward:
        assert "full_problem_s" in everything and "full_problem_s_extrapolated" not in everything


def test_roofline_peak_per_kernel():
    import bench
    peaks = {"bf16": 1700.0, "bf16_sustained": 1400.0, "source": "measured"}
    bf16 = object.__new__(bench.Path)
    bf16.peak_key = "bf16"
    assert bench.peak_for(bf16, peaks, {})[0] == 1700.0
    q8 = object.__new__(bench.Path)
    q8.peak_key = "fp8"
    assert bench.peak_for(q8, peaks, {})[0] == 3400.0                   # nominal 2 x bf16 fallback
    got = bench.peak_for(q8, peaks, {"fp8_e4m3_tflops": 3000.0, "int8_tops": 2000.0})[0]
    assert got == pytest.approx(2400.0)                                  # half the work at each rate
    gemm = object.__new__(bench.GemmPath)
    gemm.peak_key = "fp8"
    assert bench.peak_for(gemm, peaks, {"fp8_e4m3_tflops": 3000.0, "int8_tops": 2000.0})[0] == 3000.0


def test_union_fraction_of_the_block_sparse_tiles():
    import numpy as np
    import bench
    m = np.zeros((1, 1, 3, 4), dtype=np.uint8)
    m[0, 0, 0, [0, 2]] = 1            # tile 0: query blocks 0 and 1 -> union {0, 2, 3}
    m[0, 0, 1, [2, 3]] = 1
    m[0, 0, 2, [1]] = 1               # tile 1: query block 2 alone -> {1}
    assert bench.union_fraction(m) == pytest.approx((3 + 1) / (2 * 4))
    rng = np.random.default_rng(0)    # independent rows at density d: 1 - (1 - d)^2
    r = (rng.random((1, 8, 64, 4096)) < 0.125).astype(np.uint8)
    assert bench.union_fraction(r) == pytest.approx(1 - 0.875 ** 2, abs=3e-3)
