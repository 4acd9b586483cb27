"""The tensor-core rate probe behind the benchmark's MMA peaks (GPU).

bench.py calls the same probe in every run and reports the GEMM and the whole
layer against these rates; here the rates are checked for plausibility
against the part's nominal dense peaks (2.25 PF bf16, 4.5 PF FP8/INT8,
9 PF FP4): a probe that measured nothing, or twice the hardware, fails.
"""
import pytest

import rank_gemm_svdq_b200 as sv

pytestmark = pytest.mark.gpu


def test_tensor_peak_probe_rates_are_plausible(gpu):
    import torch
    import bench
    peaks = bench.probe_tensor_peaks(sv, torch)
    print(peaks)
    nominal = {"mxf4nvf4_pair": 9000.0, "mxf4nvf4": 9000.0, "bf16": 2250.0, "e4m3": 4500.0, "s8": 4500.0}
    for name, nom in nominal.items():
        assert 0.3 * nom < peaks[name] < 1.2 * nom, (name, peaks[name])
    assert peaks["mxf4nvf4_pair"] >= peaks["mxf4nvf4"] * 0.95


def test_probe_rejects_bad_arguments(gpu):
    import torch
    cycles = torch.zeros(8, dtype=torch.int64, device="cuda")
    for op, iters, ctas in ((5, 10, 1), (-1, 10, 1), (0, 0, 1), (0, 10, 0)):
        with pytest.raises(sv.SVDQError):
            sv.probe_tc(op, iters, ctas, cycles)
