"""The benchmark's host-side logic on the CPU: roofline selection, peaks,
config naming, the layer-level fractions (no GPU)."""
import bench
import synth

PEAKS = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}
PROBED = {"mxf4nvf4_pair": 8000.0, "e4m3": 3800.0}


def test_headline_layer_is_tensor_bound_against_fp4():
    wl = synth.make_workload("flux_ffn_up_nvfp4", with_x=False, with_w=False)
    r = bench.gemm_roofline(wl, 0.1, 0.03, 0.12, PEAKS, PROBED)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["kernel"] == "gemm_nvfp4_pair_kernel"
    assert r["peak"] == 1600.0 * 4
    f = bench.flops(4608, 3072, 12288, 32)
    assert abs(r["achieved"] - f / 1e-4 / 1e12) < 1e-6
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    assert abs(r["frac_of_nominal"] - r["achieved"] / 9000.0) < 1e-12
    assert abs(r["frac_of_probed_mma"] - r["achieved"] / 8000.0) < 1e-12
    # the whole step (both kernels) against the same three peaks
    lay = r["layer"]
    assert abs(lay["achieved_tflops"] - f / 1.2e-4 / 1e12) < 1e-6
    assert abs(lay["frac_of_measured"] - lay["achieved_tflops"] / 6400.0) < 1e-12
    assert abs(lay["frac_of_nominal"] - lay["achieved_tflops"] / 9000.0) < 1e-12
    assert abs(lay["frac_of_probed_mma"] - lay["achieved_tflops"] / 8000.0) < 1e-12
    assert lay["frac_of_measured"] < r["frac"]


def test_int4_layer_uses_the_fp8_ratio():
    wl = synth.make_workload("flux_qkv_int4", with_x=False, with_w=False)
    r = bench.gemm_roofline(wl, 0.36, 0.03, 0.39, PEAKS, PROBED)
    assert r["bound"] == "tensor" and r["kernel"] == "gemm_int4_kernel" and r["peak"] == 1600.0 * 2
    assert r["traffic"] is None and r["probed_mma_tflops"] == 3800.0
    assert abs(r["frac_of_nominal"] - r["achieved"] / 4500.0) < 1e-12


def test_few_tokens_are_hbm_bound():
    wl = synth.make_workload("var_up_nvfp4", with_x=False, with_w=False)
    wl.M = 1
    r = bench.gemm_roofline(wl, 0.02, 0.01, 0.025, PEAKS, PROBED)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6500.0
    assert abs(r["achieved"] - bench.gemm_alg_bytes(1, 4096, 16384, 32, "nvfp4") / 2e-5 / 1e9) < 1e-6
    lb = bench.layer_alg_bytes(1, 4096, 16384, 32, "nvfp4")
    assert abs(r["layer"]["achieved_gbs"] - lb / 2.5e-5 / 1e9) < 1e-6
    r2 = bench.gemm_roofline(wl, 0.02, 0.01, 0.025, None, None)
    assert r2["peak"] == 6650.0 and r2["peak_source"].startswith("of fallback")


def test_layer_bytes_count_x_and_y_once():
    M, K, N, r = 4608, 3072, 12288, 32
    b = bench.layer_alg_bytes(M, K, N, r, "nvfp4")
    assert b == M * K * 2 + M * N * 2 + N * K // 2 + N * K // 16 + K * r * 2 + r * N * 2 + N * 4 + K * 4


def test_config_names():
    wl = synth.make_workload("flux_ffn_up_nvfp4", with_x=False, with_w=False)
    d = bench.config_dict(wl, 1, small=False)
    assert d["workload"].startswith("flux_ffn_up_nvfp4: FLUX.1-like FFN up projection")
    assert d["l2"].startswith("flushed")
    wl = synth.make_workload("tiny_int4", with_x=False, with_w=False)
    d = bench.config_dict(wl, 2, small=True)
    assert d["workload"].startswith("tiny_int4: M=256 K=512 N=512") and d["format"] == "int4"
    assert d["act_dtype"] == "fp16" and d["parallelism"].startswith("replicas x2")
    assert "graph" in d["l2"]
