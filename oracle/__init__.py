"""CPU oracle for the SVDQuant W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct.  Only the test-suite, the smoke check and the
benchmark's CPU-baseline leg may import this package; the product path
(`rank_gemm_svdq_b200`) never does, and this package imports nothing from it.

What it follows (pages, by title and section):
  * "SVDQuant是什么？…" (zhuoshang.net), 技术原理: smoothing migrates activation
    outliers into the weight, the weight is split by SVD into a 16-bit low-rank
    branch and a 4-bit residual; Eckart-Young-Mirsky bounds the residual.
  * "AI图像生成4-bit量化技术解析与应用", section 2.2 (the three SVD steps:
    W = U S V^T, keep the top k, quantise R = W - W_k to 4 bits) and 3.1/3.2
    (INT4 group quantisation with dynamic activation ranges; NVFP4).
  * "W4A8量化技术在边缘计算中的实践与优化", 3.1 (symmetric absmax quantiser
    scale = max|w| / (2^(b-1)-1), q = clamp(round(w/scale), -2^(b-1), 2^(b-1)-1)).
  * "DeepCompressor…", SVDQuant section: the low-rank branch and the 4-bit
    branch are summed in one layer output.

Modules:
  formats    E2M1 / E4M3 codes, round-to-nearest-even to fp16 / bf16
  quant      INT4 group-64 and NVFP4 quantisers (fp32 arithmetic)
  svd        one-sided Jacobi SVD in float64 (plain C helper, _jacobi.c)
  svdquant   smoothing, truncated factors, residual, Y
  kvcache    asymmetric per-channel INT8 KV-cache codec ("VAR-Compressor…",
             INT8 KV缓存量化)

Pins: tests/test_oracle_*.py check every function against what the pages and
the mathematics fix (closed forms, invariants, brute force, format tables);
tests/test_kv.py (a hand-worked fixture and the codec's invariants),
tests/test_lora.py (the appended layer against plain X A B products) and
tests/test_shard.py (a shard against the full layer's columns) pin the
next-row functions, and tests/test_oracle_mutations*.py plant mistakes that
the pins must catch.
Functions whose result is not pinned say "parity unpinned" in their docstring;
there are none at present.
"""
