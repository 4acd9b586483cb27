"""The benchmark's host-side logic on the CPU: roofline selection, peaks,
config naming (no GPU)."""
import bench
import synth

PEAKS = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}


def test_headline_layer_is_tensor_bound_against_fp4():
    wl = synth.make_workload("flux_ffn_up_nvfp4")
    r = bench.gemm_roofline(wl, 0.1, 0.03, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["kernel"] == "gemm_nvfp4_pair_kernel"
    assert r["peak"] == 1600.0 * 4
    assert abs(r["achieved"] - bench.flops(4608, 3072, 12288, 32) / 1e-4 / 1e12) < 1e-6
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    assert "frac_of_nominal_fp4" in r


def test_int4_layer_uses_the_fp8_ratio():
    wl = synth.make_workload("flux_qkv_int4")
    r = bench.gemm_roofline(wl, 0.36, 0.03, PEAKS)
    assert r["bound"] == "tensor" and r["kernel"] == "gemm_int4_kernel" and r["peak"] == 1600.0 * 2
    assert r["traffic"] is None and "frac_of_nominal_fp4" not in r


def test_few_tokens_are_hbm_bound():
    wl = synth.make_workload("var_up_nvfp4")
    wl.M = 1
    r = bench.gemm_roofline(wl, 0.02, 0.01, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6500.0
    assert abs(r["achieved"] - bench.gemm_alg_bytes(1, 4096, 16384, 32, "nvfp4") / 2e-5 / 1e9) < 1e-6
    r2 = bench.gemm_roofline(wl, 0.02, 0.01, None)
    assert r2["peak"] == 6650.0 and r2["peak_source"].startswith("of fallback")


def test_config_names():
    wl = synth.make_workload("flux_ffn_up_nvfp4")
    assert bench.config_dict(wl)["workload"].startswith("flux_ffn_up_nvfp4: FLUX.1-like FFN up projection")
    wl = synth.make_workload("tiny_int4")
    d = bench.config_dict(wl, {"parallelism": "x"})
    assert d["workload"].startswith("tiny_int4: M=256 K=512 N=512") and d["format"] == "int4"
    assert d["act_dtype"] == "fp16" and d["parallelism"] == "x"
