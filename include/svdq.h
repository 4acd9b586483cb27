/*
 * svdq.h -- C ABI of the SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (SVDQuant; "SVDQuant是什么？" 技术原理, "AI图像生成4-bit量化技术解析与应用"
 * 2.2/3.1/3.2, "DeepCompressor…" SVDQuant section):
 *
 *     X^ = X diag(lambda)^-1,  W^ = diag(lambda) W         smoothing
 *     W^ ~ L1 L2  (rank r, truncated SVD, 16-bit)          low-rank branch
 *     R  = W^ - L1 L2                                       4-bit residual
 *     Y  = Q(X^) Q(R) + (X^ L1) L2 + b
 *
 * Q is INT4 with symmetric per-group-of-64 fp32 scales, or NVFP4 (E2M1 values,
 * one E4M3 scale per 16 values, one fp32 tensor scale).
 *
 * Two halves:
 *   svdq_prepare  host, offline: smoothing factors, truncated SVD, residual,
 *                 weight quantisation, packing into one self-describing blob.
 *   svdq_linear   device, per call: activation quantisation + down projection
 *                 (one kernel), then the 4-bit GEMM whose epilogue adds the
 *                 low-rank up projection and the bias (one kernel).
 *
 * Layout conventions (all row-major, C order):
 *   Wt    N x K  fp32, nn.Linear layout (W = Wt^T is K x N); host memory.
 *   X     M x K  fp16 or bf16 (params.act_dtype); device memory.
 *   Y     M x N  bf16; device memory.
 *   bias  N fp32 or NULL (zero bias); host memory.
 *
 * Ownership: the caller allocates and owns every buffer (host and device).
 * The library allocates no device memory and keeps no per-call state; one
 * device-global status word per GPU records device-side failures.
 *
 * Errors: every function returns an svdq_status and never aborts.  Device
 * work is launched asynchronously; failures inside a kernel (a bounded wait
 * that gave up) are recorded in the status word and read by svdq_get_status.
 *
 * Constraints: K % 256 == 0 (both formats), N % 256 == 0,
 * 0 <= rank <= 128, rank % 16 == 0,
 * M >= 0 (M = 0 is a no-op), device pointers 16-byte aligned, inputs finite.
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,    /* null pointer, bad size or unsupported shape   */
  SVDQ_ERR_UNSUPPORTED = 2,    /* no sm_100 device or unsupported format         */
  SVDQ_ERR_ALIGNMENT = 3,      /* a device pointer is not 16-byte aligned        */
  SVDQ_ERR_WORKSPACE = 4,      /* workspace smaller than svdq_workspace_bytes    */
  SVDQ_ERR_BLOB = 5,           /* blob header, size or checksum mismatch         */
  SVDQ_ERR_NO_CONVERGENCE = 6, /* truncated SVD did not converge                 */
  SVDQ_ERR_CUDA = 7,           /* a CUDA runtime call or launch failed           */
  SVDQ_ERR_TIMEOUT = 8         /* a device-side bounded wait gave up             */
} svdq_status;

typedef enum { SVDQ_INT4_G64 = 1, SVDQ_NVFP4 = 2 } svdq_format;
typedef enum { SVDQ_F16 = 1, SVDQ_BF16 = 2 } svdq_dtype;

typedef struct svdq_params {
  int32_t K;          /* input features                                   */
  int32_t N;          /* output features                                  */
  int32_t rank;       /* r, rank of the 16-bit branch (0 disables it)     */
  int32_t fmt;        /* svdq_format                                      */
  int32_t act_dtype;  /* svdq_dtype of X (and of the stored L1, L2)       */
  int32_t smooth;     /* 1: smoothing on; 0: lambda = 1                   */
  float alpha;        /* smoothing migration strength, in [0, 1]          */
  int32_t reserved;   /* must be 0                                        */
} svdq_params;

/* An opaque CUDA stream handle (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st* svdq_stream;

/* ---------------------------------------------------------------- host side */

/* Bytes of the blob svdq_prepare writes for these parameters (0 if invalid). */
size_t svdq_blob_bytes(const svdq_params* p);

/*
 * Offline preparation ("SVDQuant是什么？" 技术原理; 4-bit page 2.2).
 *   lambda_j = a_j^alpha / w_j^(1-alpha), a_j = max_m |X_cal[m,j]|,
 *   w_j = max_n |W[j,n]| (1 where either is 0 or smoothing is off);
 *   W^ = diag(lambda) W; (L1, L2) = top-r singular triplets of W^ as
 *   L1 = U_r S_r, L2 = V_r^T rounded to act_dtype; R = W^ - L1 L2 (float64,
 *   then fp32); R quantised per output channel along K; NVFP4 also stores the
 *   static activation tensor scale amax(X_cal diag(lambda)^-1) / 2688.
 * Wt: N x K fp32 host.  bias: N fp32 host or NULL.  X_cal: M_cal x K host,
 * act_dtype bits (calibration activations; may be the layer's own input).
 * blob: host buffer of blob_bytes >= svdq_blob_bytes(p); copy it to device
 * memory (16-byte aligned) before svdq_linear.  sigma_out: NULL or rank+1
 * doubles, the leading singular values of W^ (estimates).
 * Uses the host's cores (OpenMP).  Deterministic for a given input.
 */
svdq_status svdq_prepare(const svdq_params* p, const float* Wt, const float* bias,
                         const void* X_cal, int64_t M_cal, void* blob, size_t blob_bytes,
                         double* sigma_out);

/* Validate a host blob against p: magic, version, parameters, size, checksum. */
svdq_status svdq_blob_check(const svdq_params* p, const void* blob, size_t blob_bytes);

/*
 * Copy a host blob's contents out in a canonical, layout-independent form
 * (for tests and inspection).  Any output pointer may be NULL.
 *   inv_lambda  K fp32
 *   L1          K x r  act_dtype bits (uint16)
 *   L2          r x N  act_dtype bits (uint16)
 *   wcodes      N x K  one code per byte: INT4 as int8 in [-8, 7];
 *               NVFP4 as the E2M1 code in the low nibble
 *   wscales     INT4: N x K/64 fp32;  NVFP4: N x K/16 E4M3 codes (uint8)
 *   tscales     2 fp32: [s_gX, s_gW] (NVFP4 tensor scales; 1 for INT4)
 *   bias        N fp32
 */
svdq_status svdq_blob_export(const svdq_params* p, const void* blob, float* inv_lambda,
                             uint16_t* L1, uint16_t* L2, uint8_t* wcodes, void* wscales,
                             float* tscales, float* bias);

/*
 * Add a LoRA branch to a prepared layer without re-quantising it
 * ("SVDQuant是什么？" 概述简介 and 功能特色, LoRA集成: off-the-shelf low-rank
 * adapters plug into the quantised model with no new quantisation).  The
 * layer then computes Y' = Y + X A B.  Since X = X^ diag(lambda), the
 * adapter joins the 16-bit low-rank branch:
 *   L1' = [L1 | act_dtype(lambda_eff (.) A)]   K x (r + r_lora),
 *   L2' = [L2 ; act_dtype(B)]                  (r + r_lora) x N,
 * with lambda_eff_j = 1 / inv_lambda_j as stored; the 4-bit residual, its
 * scales, lambda, the tensor scales and the bias are copied unchanged.
 * A: K x r_lora fp32 host (row-major); B: r_lora x N fp32 host (any LoRA
 * scaling already folded in).  r_lora > 0, r_lora % 16 == 0 and
 * p->rank + r_lora <= 128, else SVDQ_ERR_INVALID_ARG.  blob_in (blob_in_bytes,
 * checked as by svdq_blob_check) is read only; blob_out is a host buffer of
 * blob_out_bytes >= svdq_blob_bytes(p_out), written in full; *p_out receives
 * p with rank = p->rank + r_lora.  Adapters stack by calling it again.
 */
svdq_status svdq_append_lora(const svdq_params* p, const void* blob_in, size_t blob_in_bytes, const float* A,
                             const float* B, int32_t r_lora, svdq_params* p_out, void* blob_out,
                             size_t blob_out_bytes);

/*
 * Column shard of a prepared layer, for column-parallel use on several GPUs
 * (one shard per GPU, each writing its own slice of Y): output features
 * [n0, n1) of the layer, with n0 and n1 multiples of 256, 0 <= n0 < n1 <= N.
 * The shard keeps lambda, L1 and the tensor scales of the whole layer and
 * takes the features' rows of L2, of the 4-bit residual and its scales, and
 * of the bias, so svdq_linear on the shard gives columns [n0, n1) of the full
 * layer's output (bit for bit when both run the same GEMM schedule, i.e.
 * outside the few-token K split).  blob_in (blob_in_bytes, checked as by
 * svdq_blob_check) is read only; blob_out is a host buffer of blob_out_bytes
 * >= svdq_blob_bytes(p_out); *p_out receives p with N = n1 - n0.  Errors:
 * SVDQ_ERR_INVALID_ARG (range, sizes), SVDQ_ERR_BLOB (blob_in).
 */
svdq_status svdq_shard_columns(const svdq_params* p, const void* blob_in, size_t blob_in_bytes, int32_t n0,
                               int32_t n1, svdq_params* p_out, void* blob_out, size_t blob_out_bytes);

/* ------------------------------------------------- INT8 KV-cache codec
 * Asymmetric per-channel INT8 for a block of cached keys or values
 * ("VAR-Compressor：在边缘GPU上实现80亿参数视觉自回归模型的高效量化部署",
 * INT8 KV缓存量化 and KV缓存特性研究: the cache's variance is driven by channels
 * and its distribution is skewed, so each channel gets its own scale and a
 * non-centred zero point).  For a block X of T tokens x C channels
 * (row-major, act dtype), per channel c, in fp32 with round to nearest even:
 *   lo = min(0, min_t X[t,c]), hi = max(0, max_t X[t,c]),
 *   scale = (hi - lo) / 255 (1 when hi == lo), zero = clamp(rint(-lo/scale), 0, 255),
 *   code  = clamp(rint(X/scale) + zero, 0, 255)        (uint8)
 * and decoding gives (code - zero) * scale rounded to the dtype.  A zero
 * entry decodes to exactly 0.
 */

/* Device workspace bytes of svdq_kv_encode for a T x C block (0 if invalid). */
size_t svdq_kv_workspace_bytes(int64_t T, int32_t C);

/*
 * Encode a device block.  X: T x C, dtype an svdq_dtype value (SVDQ_BF16 /
 * SVDQ_F16).  codes: T x C uint8; scale: C fp32; zero: C uint8; workspace:
 * ws_bytes >= svdq_kv_workspace_bytes(T, C).  All device pointers, 16-byte
 * aligned, owned by the caller.  T >= 1, C % 256 == 0.  Asynchronous on
 * `stream` (two kernels).  Errors: SVDQ_ERR_INVALID_ARG, SVDQ_ERR_WORKSPACE,
 * SVDQ_ERR_ALIGNMENT, SVDQ_ERR_UNSUPPORTED (no sm_100 device), SVDQ_ERR_CUDA.
 */
svdq_status svdq_kv_encode(const void* X, int64_t T, int32_t C, int32_t dtype, uint8_t* codes, float* scale,
                           uint8_t* zero, void* workspace, size_t ws_bytes, svdq_stream stream);

/*
 * Decode a device block back to dtype: Y[t,c] = dtype((codes[t,c] - zero[c]) * scale[c]).
 * T >= 1, C % 8 == 0; device pointers 16-byte aligned; asynchronous.
 */
svdq_status svdq_kv_decode(const uint8_t* codes, const float* scale, const uint8_t* zero, int64_t T, int32_t C,
                           int32_t dtype, void* Y, svdq_stream stream);

/*
 * Attention reads over INT8 caches (the read side of the codec above): scaled
 * dot-product attention of Mq query rows against T cached keys and values
 * held as codes, per head, without materialising the decoded cache:
 *   for head h (channels [h d, (h + 1) d), d = C / heads),
 *   S[i,t] = sum_c Q[i,c] K^[t,c] / sqrt(d),  P = softmax over t,
 *   out[i,c] = sum_t P[i,t] V^[t,c],   K^ = (kcodes - kzero) kscale, V^ likewise
 * (the decoded values in fp32).  Q: Mq x C, dtype (SVDQ_BF16 / SVDQ_F16);
 * kcodes, vcodes: T x C uint8; kscale, vscale: C fp32; kzero, vzero: C uint8
 * (as svdq_kv_encode writes them); out: Mq x C fp32.  All device pointers,
 * 16-byte aligned, owned by the caller; workspace >= the bytes below.
 * 1 <= Mq <= 16, T >= 1, d = 64 or 128 (else SVDQ_ERR_UNSUPPORTED).
 * Asynchronous on `stream` (two kernels: 256-token chunks, then a combine in
 * chunk order, so results are reproducible bit for bit).  Errors:
 * SVDQ_ERR_INVALID_ARG, SVDQ_ERR_WORKSPACE, SVDQ_ERR_ALIGNMENT,
 * SVDQ_ERR_UNSUPPORTED, SVDQ_ERR_CUDA.
 */
size_t svdq_kv_attention_workspace_bytes(int64_t T, int32_t C, int32_t heads, int32_t Mq);
svdq_status svdq_kv_attention(const void* Q, int32_t Mq, const uint8_t* kcodes, const float* kscale,
                              const uint8_t* kzero, const uint8_t* vcodes, const float* vscale, const uint8_t* vzero,
                              int64_t T, int32_t C, int32_t heads, int32_t dtype, float* out, void* workspace,
                              size_t ws_bytes, svdq_stream stream);

/* Device workspace bytes svdq_linear needs for M tokens. */
size_t svdq_workspace_bytes(const svdq_params* p, int64_t M);

/* ---------------------------------------------------------------- device side */

/*
 * Y = Q(X^) Q(R) + (X^ L1) L2 + b for M tokens ("DeepCompressor…" SVDQuant
 * section: the low-rank branch is fused into the low-bit kernel).
 *   Kernel 1 reads X once: X^ = fp32(X) * inv_lambda, per-token dynamic
 *   quantisation (INT4 groups of 64 / NVFP4 blocks of 16 with the static
 *   tensor scale) and u = X^16 L1 (X^ rounded to act_dtype, fp32 accumulate).
 *   Kernel 2: TMA-fed tcgen05 GEMM with TMEM accumulators; the epilogue adds
 *   u L2 (as extra tensor-core K-steps into the same accumulator) and b, and
 *   writes bf16 Y.
 * blob_dev: device copy of the svdq_prepare blob for the same p.
 * X: M x K act_dtype, device.  Y: M x N bf16, device.
 * workspace: device, >= svdq_workspace_bytes(p, M); holds the quantised
 * activations between the kernels (read back by svdq_export_act).
 * Asynchronous on `stream`; returns SVDQ_ERR_CUDA if a launch fails.
 */
svdq_status svdq_linear(const svdq_params* p, const void* blob_dev, const void* X, int64_t M,
                        void* Y, void* workspace, size_t ws_bytes, svdq_stream stream);

/*
 * The two halves of svdq_linear as separate launches (same arguments and
 * rules).  svdq_quantize_act runs kernel 1 (X -> workspace); svdq_gemm runs
 * kernel 2 (workspace -> Y) and must follow a svdq_quantize_act for the same
 * M and workspace in stream order.  svdq_linear == quantize_act + gemm.
 */
svdq_status svdq_quantize_act(const svdq_params* p, const void* blob_dev, const void* X, int64_t M,
                              void* workspace, size_t ws_bytes, svdq_stream stream);
svdq_status svdq_gemm(const svdq_params* p, const void* blob_dev, int64_t M, void* Y, void* workspace,
                      size_t ws_bytes, svdq_stream stream);

/*
 * Chained layers: this layer's GEMM emits the NEXT layer's quantised input,
 * so this layer's output never makes a bf16 round trip through HBM (the
 * fusion argument of the "DeepCompressor…" SVDQuant section, where the
 * low-rank branch rides in the low-bit kernel to save activation traffic,
 * carried to the boundary between two layers).  The next layer's input is
 * this layer's bf16 output y; its quantised form is what the next layer's
 * activation kernel would make of y: x^' = fp32(y) * inv_lambda', NVFP4
 * codes and E4M3 block scales under the next layer's static tensor scale,
 * and u' = X^'16 L1' with X^'16 = bf16(x^').
 * Call it where svdq_gemm would be called: `workspace` holds this layer's
 * quantised input (from svdq_quantize_act, or from a previous chained call
 * as its ws_next).  On return (stream order) ws_next holds the next layer's
 * quantised input exactly as svdq_quantize_act(p_next, blob_next, y, M,
 * ws_next) leaves it, codes and scales bit for bit; u' equal up to fp32
 * summation order (per output tile, then across tiles in order).  Finish
 * with svdq_gemm(p_next, blob_next, M, Y', ws_next) or chain again.
 *   Both layers NVFP4; p_next->K == p->N; p_next->act_dtype == SVDQ_BF16;
 *   p_next->rank 0, 16 or 32 (else SVDQ_ERR_UNSUPPORTED / INVALID_ARG).
 *   workspace >= svdq_chain_workspace_bytes(p, p_next, M) (this layer's
 *   workspace plus the next layer's partial down projections, one per
 *   256-column output tile, fp32); ws_next >= svdq_workspace_bytes(p_next, M).
 *   Above 128 tokens this is one GEMM launch whose epilogue quantises and
 *   runs the partial down projection on the tensor cores, plus a small
 *   kernel that adds the partials; up to 128 tokens (this layer's output at
 *   most 128 rows) the GEMM writes y into the workspace and the next
 *   layer's activation kernel reads it.
 * All pointers device, 16-byte aligned, owned by the caller.  Asynchronous on
 * `stream`; errors as svdq_gemm.
 */
size_t svdq_chain_workspace_bytes(const svdq_params* p, const svdq_params* p_next, int64_t M);
svdq_status svdq_gemm_chain(const svdq_params* p, const void* blob_dev, int64_t M, const svdq_params* p_next,
                            const void* blob_next_dev, void* workspace, size_t ws_bytes, void* ws_next,
                            size_t ws_next_bytes, svdq_stream stream);

/*
 * After svdq_linear: copy the quantised activations out of the workspace in
 * canonical form (synchronises `stream`).  Any output pointer may be NULL.
 *   codes   M x K host, one code per byte (INT4 int8 / NVFP4 E2M1 low nibble)
 *   scales  INT4: M x K/64 fp32;  NVFP4: M x K/16 E4M3 codes (uint8)
 *   u       M x r host fp32: the down projection X^16 L1 as used by kernel 2
 *           (hi + lo parts summed, before the tensor-scale division)
 */
svdq_status svdq_export_act(const svdq_params* p, const void* workspace, int64_t M,
                            uint8_t* codes, void* scales, float* u, svdq_stream stream);

/* Synchronise `stream`, read and clear this device's status word. */
svdq_status svdq_get_status(svdq_stream stream);

const char* svdq_status_string(svdq_status s);

/* The CUDA error behind the most recent SVDQ_ERR_CUDA returned on this host
 * thread ("" if none): the failing step and cudaGetErrorString's text. */
const char* svdq_last_error_string(void);

/*
 * Test hook: the GPU's own fp32 -> E2M1 and fp32 -> E4M3 conversions
 * (cvt.rn.satfinite), used to pin the host encoders.  in: n fp32 device;
 * e2m1, e4m3: n bytes device (one code per byte).  Asynchronous.
 */
svdq_status svdq_probe_cvt(const float* in, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                           svdq_stream stream);

/*
 * Test hook: the quotient v[i] / d[i] as the activation kernel computes it
 * (one round-to-nearest reciprocal per block, then an FMA-corrected product)
 * into q, and the IEEE round-to-nearest division into q_ieee, so that tests
 * can check the two agree bit for bit.  All pointers: n fp32, device.
 */
svdq_status svdq_probe_div(const float* v, const float* d, int64_t n, float* q, float* q_ieee,
                           svdq_stream stream);

/*
 * Test hook for the device-side failure path: one thread waits, with the
 * kernels' bounded mbarrier wait, on a barrier that nothing arrives on.  After
 * limit_ns (1 .. 2e9) it gives up and records SVDQ_ERR_TIMEOUT in the device
 * status word, which the next svdq_get_status returns (and clears).  Nothing
 * hangs and the context stays usable.  Asynchronous on `stream`.
 */
svdq_status svdq_probe_timeout(int64_t limit_ns, svdq_stream stream);

/*
 * Measurement hook: tensor-core MMA rate, the denominators of the GEMM
 * rooflines.  Launches `ctas` CTAs (rounded up to whole CTA pairs for op 1);
 * in each, one thread issues `iters` (1 .. 2^24) back-to-back tcgen05 MMAs of
 * kind `op` on zeroed shared memory and writes the clock64 cycles it took
 * (issue to completion) to cycles[cta] (device, one entry per launched CTA).
 *   0 mxf4nvf4 128x256x64   1 mxf4nvf4 256x256x64 (CTA pair)
 *   2 bf16 128x256x16       3 E4M3 128x256x32      4 s8 128x256x32
 * Time the launch with events on `stream` for the chip-wide rate
 * (2 M N K flops per MMA).  Asynchronous; SVDQ_ERR_INVALID_ARG outside these ranges.
 */
svdq_status svdq_probe_tc(int op, int iters, int ctas, unsigned long long* cycles, svdq_stream stream);

/*
 * svdq_linear without a caller-supplied workspace: the quantised activations
 * and the down projection go to a scratch buffer that the library holds in
 * static device memory (SVDQ_NOALLOC_SCRATCH_BYTES per device, 256-byte
 * aligned, part of the library's device image).  Nothing is allocated by this
 * call: no cudaMalloc, no cudaFree, no allocating library routine.  The
 * SVDQuant pages have no counterpart; this entry point exists for callers that
 * must not allocate device memory at the point of the call (for example a
 * host framework whose allocator is not reachable from where the layer runs,
 * or code running while allocation is forbidden).
 *
 *   p, blob_dev, X, M, Y, stream   as for svdq_linear.
 *
 * Limit: the workspace that svdq_workspace_bytes(p, M) reports must fit in
 * SVDQ_NOALLOC_SCRATCH_BYTES, otherwise the call returns SVDQ_ERR_WORKSPACE
 * and svdq_last_error_string names both sizes; nothing is launched.  16 MiB
 * covers, e.g., K = 3072 layers at 4608 tokens in both formats.
 * Nothing in the scratch has to start at zero: the first kernel writes every
 * byte that the second reads.
 * The first call on each device performs one-time set-up with that device
 * current (device query, kernel attributes, and the lookup of the scratch
 * buffer's device address); make that first call before any stream capture.
 * That set-up is kept for the life of the process: after cudaDeviceReset on a
 * device the kept address and attributes are stale, so do not call the
 * library on that device again in the same process.
 * There is ONE scratch buffer per device: calls that may overlap on the GPU
 * (different streams, or different host threads, without ordering between
 * them) race on it and corrupt each other's results.  Order such calls.
 */
#define SVDQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
svdq_status svdq_linear_noalloc(const svdq_params* p, const void* blob_dev, const void* X, int64_t M,
                                void* Y, svdq_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
