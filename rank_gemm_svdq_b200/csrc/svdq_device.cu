// Device half of libsvdq: the kernels of svdq_linear and their launchers.
//
//   kernel 1 reads X once: X^ = fp32(X) * inv_lambda, per-token dynamic 4-bit
//       quantisation (NVFP4 blocks of 16 / INT4 groups of 64) and the low-rank
//       down projection u = X^16 L1 on the tensor cores
//       ("AI图像生成4-bit量化技术解析与应用" 3.1: dynamic activation ranges;
//       "SVDQuant是什么？" 技术原理: 16-bit low-rank branch):
//     act_nvfp4_kernel  NVFP4 above 256 tokens: 128-token tiles, tcgen05;
//     act_quant_kernel  INT4, and NVFP4 up to 256 tokens: 32-token groups,
//                       mma.sync, K split over clusters (and the workspace).
//   kernel 2, the 4-bit GEMM Q(X^) Q(R) on tcgen05 with TMEM accumulators;
//       the low-rank up projection u L2 runs as extra bf16 K-steps into the
//       same accumulator and the epilogue adds the bias and writes bf16 Y
//       ("DeepCompressor…" SVDQuant section: the low-rank branch fused into
//       the low-bit kernel so it costs no extra activation traffic):
//     gemm_nvfp4_pair_kernel<false>  NVFP4 above 128 tokens, CTA pairs;
//     gemm_nvfp4_small_kernel<TOK>   NVFP4 up to 128 tokens, weight tile as A;
//     gemm_int4_kernel               INT4 (E4M3-coded), group scales folded.
//   chained layers: gemm_nvfp4_pair_kernel<true> writes the next layer's
//       quantised input instead of Y, chain_u_kernel adds its per-tile
//       partial down projections.
//
// Every wait on an mbarrier is bounded (about 1 s); a wait that gives up
// records SVDQ_ERR_TIMEOUT in a device status word and the CTA winds down.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <mutex>
#include <vector>

#include "layout.h"
#include "ptx.cuh"

namespace svdq {
namespace dev {

// ------------------------------------------------------------ conversions
// fp32 pair -> two E4M3 codes (hi -> upper byte), RNE, saturating to 448.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// fp32 pair -> two E2M1 codes (hi -> upper nibble), RNE, saturating to 6.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// E4M3 code -> fp32 value (exact).
__device__ __forceinline__ float e4m3_val(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  const float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
  return (b & 0x80u) ? -v : v;
}

template <int DT>
__device__ __forceinline__ float half_to_f32(uint16_t h) {
  if constexpr (DT == SVDQ_BF16) return __uint_as_float((uint32_t)h << 16);
  else return __half2float(__ushort_as_half(h));
}

template <int DT>
__device__ __forceinline__ uint16_t f32_to_half_rn(float f) {
  if constexpr (DT == SVDQ_BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(f));
  else return __half_as_ushort(__float2half_rn(f));
}

__device__ __forceinline__ uint16_t bf16_rn(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }

// ------------------------------------------------------------ kernel 1
struct ActArgs {
  const uint16_t* X;
  int64_t M, Mp;
  int K, r, lrw, nseg;
  const float* inv_lambda;
  const uint16_t* l1t;
  const BlobHeader* hdr;
  uint8_t* xq;
  uint8_t* xs;
  uint16_t* ux;
  int ks;   // K split: ks CTAs share one group of 32 tokens
  int* gemm_cnt;   // GEMM K-split arrival counters to clear (or null)
  int n_cnt;
  // workspace split (the GS kernels, ks > 8): clusters of 8 add their partial
  // down projections through distributed shared memory, and the ks / 8
  // cluster sums of a group meet in the workspace, where the last to arrive
  // adds them (see act_small_ks)
  unsigned long long epoch;   // nonzero, distinct per call
  float* upart;               // [groups][ks / 8][32 r] fp32, in mma fragment order
  unsigned long long* ucnt;   // one arrival word per group
};

constexpr int kActRows = 32;     // tokens per CTA
constexpr int kActThreads = 512;
constexpr int kActSmemMax = 232448 - 4096;   // dynamic; the kernel also has 2 KB of static tables
constexpr int kActChunk = 256;   // K elements per step
constexpr int kActStride = kActChunk + 8;  // padded smem row (bf16/fp16 elements)

// Correctly rounded fp32 quotient v / d given r = RN(1 / d): q = RN(v r) is
// within one ulp, the remainder e = v - q d is exact with one FMA, and
// RN(q + e r) is the correctly rounded quotient (Markstein's theorem; see
// Muller et al., Handbook of Floating-Point Arithmetic, the FMA-based division
// section).  Valid while the remainder is representable and nothing
// overflows: the callers use it only for 2^-100 <= d <= 2^125 (recip_ok), and
// for quotients below 2^-2 (where the exact remainder may underflow) every
// 4-bit code is zero either way, with the sign preserved.
__device__ __forceinline__ bool recip_ok(float d) { return d >= 0x1p-100f && d <= 0x1p+125f; }

__device__ __forceinline__ float div_by_recip(float v, float d, float r) {
  const float q = __fmul_rn(v, r);
  const float e = __fmaf_rn(-q, d, v);
  return __fmaf_rn(e, r, q);
}

// Two fp32 lanes per instruction (mul / fma .rn.f32x2): each lane is rounded
// exactly as the scalar operation would be.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// div_by_recip on two lanes: v2 / d, given nd2 = (-d, -d) and r2 = (r, r).
__device__ __forceinline__ uint64_t div2_by_recip(uint64_t v2, uint64_t nd2, uint64_t r2) {
  const uint64_t q = f2_mul(v2, r2);
  const uint64_t e = f2_fma(q, nd2, v2);
  return f2_fma(e, r2, q);
}

__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Number of L1^T chunk buffers the activation kernel keeps in shared memory
// (3 lets the copies run two chunks ahead; rank 128 only fits 2).
SVDQ_HD inline int act_l1_bufs(int r) {
  return (2 * kActRows + 3 * r) * kActStride * 2 <= kActSmemMax ? 3 : 2;
}
SVDQ_HD inline int act_ring_bytes(int r) { return (2 * kActRows + act_l1_bufs(r) * r) * kActStride * 2; }
// The CTA's slice of inv_lambda (k_range floats) also sits in shared memory when it fits.
SVDQ_HD inline bool act_il_in_smem(int r, int k_range) { return act_ring_bytes(r) + k_range * 4 <= kActSmemMax; }
SVDQ_HD inline int act_smem_bytes(int r, int k_range) {
  return act_ring_bytes(r) + (act_il_in_smem(r, k_range) ? k_range * 4 : 0);
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& a0, uint32_t& a1, uint32_t& a2,
                                            uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& b0, uint32_t& b1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(addr));
}

template <int DT>
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  if constexpr (DT == SVDQ_BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

template <int DT>
__device__ __forceinline__ uint32_t pack_half2_rn(float lo, float hi) {
  if constexpr (DT == SVDQ_BF16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

// Quantise 16 consecutive smoothed activations of one token (one NVFP4
// block, or a quarter of an INT4 group of 64 spread over 4 lanes) and store
// codes / scales.
// Destinations (per thread and chunk, precomputed by the caller):
//   NVFP4: tile = this token's activation tile of the chunk's slab (null for
//          rows past Mp), code_off / sf_off = the lane's codes and scale byte in it;
//   INT4:  codes = the lane's 16 code bytes (null past M), sx = its group scale
//          (null unless the lane leads its group of 4 and the row is below Mp).
struct QuantDst {
  uint8_t* tile;
  uint32_t code_off, sf_off;
  uint8_t* codes;
  float* sx;
};
// The steps of quantize16's NVFP4 branch as separate helpers, for the chained
// GEMM epilogue (the activation kernel keeps its own inline copy).
// max |x| over 16 values (exact: no rounding in a max).
__device__ __forceinline__ float absmax16(const float (&xh)[16]) {
  float m8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m8[i] = fmaxf(fabsf(xh[i]), fabsf(xh[i + 8]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m8[i] = fmaxf(m8[i], m8[i + 4]);
  return fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3]));
}

// NVFP4 block scale code: E4M3_RNE_satfinite(amax / (6 s_gX)), the quotient
// correctly rounded (r6 = the reciprocal of six_sg when the FMA-corrected
// route is exact for it, else 0 and an IEEE division).
__device__ __forceinline__ uint32_t nvfp4_scale_code(float amax, float six_sg, float r6) {
  const float ratio = r6 != 0.0f ? div_by_recip(amax, six_sg, r6) : __fdiv_rn(amax, six_sg);
  return cvt_e4m3x2(0.0f, ratio) & 0xFFu;
}

// The 16 E2M1 codes E2M1_RNE_satfinite(x / d) of one block, packed two per
// byte (even element in the low nibble): p0 elements 0-7, p1 elements 8-15.
// d = E4M3(e) s_gX; rd = its round-to-nearest reciprocal when the
// FMA-corrected quotient is exact, else 0 (IEEE division).  d == 0: all zero.
__device__ __forceinline__ void nvfp4_codes16(const float (&xh)[16], float d, float rd, uint32_t& p0,
                                              uint32_t& p1) {
  p0 = 0; p1 = 0;
  if (d == 0.0f) return;
  if (rd != 0.0f) {
    const uint64_t nd2 = f2_pack(-d, -d), r2 = f2_pack(rd, rd);
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float q0, q1;
      f2_unpack(div2_by_recip(f2_pack(xh[2 * i], xh[2 * i + 1]), nd2, r2), q0, q1);
      b[i] = cvt_e2m1x2(q1, q0);
    }
    p0 = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    p1 = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      p0 |= cvt_e2m1x2(__fdiv_rn(xh[2 * i + 1], d), __fdiv_rn(xh[2 * i], d)) << (8 * i);
      p1 |= cvt_e2m1x2(__fdiv_rn(xh[2 * i + 9], d), __fdiv_rn(xh[2 * i + 8], d)) << (8 * i);
    }
  }
}

template <int FMT>
// dq: NVFP4 per-code tables in shared memory, dq[e] = E4M3(e) * s_gX and
// dq[256 + e] = its round-to-nearest reciprocal (0 where the FMA-corrected
// division is not valid); unused for INT4.
__device__ __forceinline__ void quantize16(const float (&xh)[16], const QuantDst& dst, float six_sg, float r6,
                                           const float* dq) {
  float m8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m8[i] = fmaxf(fabsf(xh[i]), fabsf(xh[i + 8]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m8[i] = fmaxf(m8[i], m8[i + 4]);
  float amax = fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3]));
  if constexpr (FMT == SVDQ_NVFP4) {
    const float ratio = r6 != 0.0f ? div_by_recip(amax, six_sg, r6) : __fdiv_rn(amax, six_sg);
    const uint32_t e = cvt_e4m3x2(0.0f, ratio) & 0xFFu;
    const float d = dq[e];
    const float rd = dq[256 + e];
    uint32_t p0 = 0, p1 = 0;
    if (d != 0.0f) {
      if (rd != 0.0f) {
        const uint64_t nd2 = f2_pack(-d, -d), r2 = f2_pack(rd, rd);
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float q0, q1;
          f2_unpack(div2_by_recip(f2_pack(xh[2 * i], xh[2 * i + 1]), nd2, r2), q0, q1);
          b[i] = cvt_e2m1x2(q1, q0);
        }
        p0 = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
        p1 = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          p0 |= cvt_e2m1x2(__fdiv_rn(xh[2 * i + 1], d), __fdiv_rn(xh[2 * i], d)) << (8 * i);
          p1 |= cvt_e2m1x2(__fdiv_rn(xh[2 * i + 9], d), __fdiv_rn(xh[2 * i + 8], d)) << (8 * i);
        }
      }
    }
    // activation tile (m / 128, slab): swizzled codes, then the slab's scale atoms
    if (dst.tile) {
      *reinterpret_cast<uint2*>(dst.tile + dst.code_off) = make_uint2(p0, p1);
      dst.tile[dst.sf_off] = (uint8_t)e;
    }
  } else {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));   // group of 64 = 4 lanes
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float s = __fdiv_rn(amax, 7.0f);
    uint32_t w[8];
    if (amax == 0.0f) {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = 0;
    } else {
      const bool fast = recip_ok(s);
      const float rs = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float t0 = fast ? div_by_recip(xh[2 * i], s, rs) : __fdiv_rn(xh[2 * i], s);
        const float t1 = fast ? div_by_recip(xh[2 * i + 1], s, rs) : __fdiv_rn(xh[2 * i + 1], s);
        const int q0 = min(7, max(-8, __float2int_rn(t0)));
        const int q1 = min(7, max(-8, __float2int_rn(t1)));
        w[i] = cvt_e4m3x2((float)q1, (float)q0);
      }
    }
    if (dst.codes)
      *reinterpret_cast<uint4*>(dst.codes) =
          make_uint4(w[0] | (w[1] << 16), w[2] | (w[3] << 16), w[4] | (w[5] << 16), w[6] | (w[7] << 16));
    if (dst.sx) *dst.sx = s;
  }
}

// One CTA = 32 tokens x K / ks, 16 warps (with ks > 1 the ks CTAs of a
// cluster split K and CTA 0 adds their partial down projections in rank
// order through distributed shared memory, so u is deterministic).  Per 256-wide chunk, warp w owns
// tokens 2w (lanes 0-15) and 2w+1 (lanes 16-31); lane l owns elements
// 16(l%16) .. 16(l%16)+15 (two 16-byte loads).  X loads run two chunks ahead
// in registers; the L1^T chunks arrive by cp.async into a ring of 3 (2 at
// rank 128) shared buffers, issued two (one) chunks ahead; the X^16 tile is
// double-buffered, so a chunk costs one __syncthreads.  The down projection
// u = X^16 L1 runs on mma.sync (m16n8k16, fp32 accumulate): 2 x r/8 tiles of
// 16 tokens x 8 ranks, tile t on warp t % 16.
template <int FMT, int DT, bool GS>
__global__ void __launch_bounds__(kActThreads, 1) act_quant_kernel(const ActArgs a) {
  extern __shared__ __align__(16) uint16_t act_smem[];
  const int K = a.K, r = a.r;
  const int nbuf = act_l1_bufs(r), lead = nbuf - 1;
  uint16_t* const xs16_base = act_smem;
  uint16_t* const l1s_base = act_smem + 2 * kActRows * kActStride;
  auto xs16 = [&](int b) { return xs16_base + b * kActRows * kActStride; };
  auto l1sb = [&](int b) { return l1s_base + b * r * kActStride; };

  griddep_launch();   // the GEMM may start its prologue on idle SMs
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (blockIdx.x == 0 && a.gemm_cnt)
    for (int i = tid; i < a.n_cnt; i += kActThreads) a.gemm_cnt[i] = 0;
  const int KS = a.ks;
  // K part of this CTA; with the workspace split the ks parts run as ks / 8
  // clusters of 8 (cluster rank = kidx % 8)
  const int kidx = GS ? (int)(blockIdx.x % KS) : (KS > 1 ? (int)cluster_ctarank() : 0);
  const int64_t m0 = (int64_t)(blockIdx.x / KS) * kActRows;
  const float s_gx = a.hdr->s_gx;
  const float six_sg = __fmul_rn(6.0f, s_gx);
  const float r6 = recip_ok(six_sg) ? __frcp_rn(six_sg) : 0.0f;
  const float inv_alpha = FMT == SVDQ_NVFP4 ? 1.0f / (a.hdr->s_gx * a.hdr->s_gw) : 1.0f;
  const int n_mma = 2 * (r / 8);   // (16-token, 8-rank) tiles of u

  float acc[2][4], acc2[2][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = acc2[t][i] = 0.0f;

  const int rw = warp * 2 + (lane >> 4);     // token row inside the CTA
  const int64_t m = m0 + rw;
  const int col = (lane & 15) * 16;          // element offset inside the chunk
  const bool live = m < a.M;
  const uint16_t* xrow = a.X + (live ? m : 0) * K + col;
  const int cpk = K / kActChunk / KS;      // chunks of this CTA: [c0, c0 + cpk)
  const int c0 = kidx * cpk;
  // per-thread output locations (see QuantDst): only the chunk's offset varies
  uint8_t* const row_tiles =
      (FMT == SVDQ_NVFP4 && m < a.Mp) ? a.xq + (size_t)(m >> 7) * (size_t)(K / 256) * kATile : nullptr;
  const uint32_t code_off = sw128((uint32_t)(m & 127), (uint32_t)col >> 1);
  const uint32_t sf_off = kTileCodes + tile_sf((uint32_t)(m & 127), (uint32_t)col >> 4);
  uint8_t* const row_codes = (FMT != SVDQ_NVFP4 && live) ? a.xq + (size_t)m * K + col : nullptr;
  const bool sx_lead = FMT != SVDQ_NVFP4 && (lane & 3) == 0 && m < a.Mp;
  const size_t sx_base = (size_t)(m / 128) * 256 + (size_t)(m % 128);   // int4_sx_index without the group part
  const size_t sx_pitch = (size_t)(a.Mp / 128) * 256;
  auto load_x = [&](int c, uint4 (&x)[2]) {
    if (live && c < cpk) {
      c += c0;
      x[0] = __ldg(reinterpret_cast<const uint4*>(xrow + c * kActChunk));
      x[1] = __ldg(reinterpret_cast<const uint4*>(xrow + c * kActChunk + 8));
    } else {
      x[0] = make_uint4(0, 0, 0, 0);
      x[1] = make_uint4(0, 0, 0, 0);
    }
  };
  uint4 xc[2], xn[2], xnn[2];
  load_x(0, xc);
  load_x(1, xn);

  // one cp.async group per chunk (empty past the end, so the counts stay uniform)
  auto stage_l1 = [&](int chunk) {
    if (chunk < cpk) {
      uint16_t* dst = l1sb(chunk % nbuf);
      for (int idx = tid; idx < r * (kActChunk / 8); idx += kActThreads) {
        const int i = idx / (kActChunk / 8), c8 = idx % (kActChunk / 8);
        cp_async_16(dst + i * kActStride + c8 * 8, a.l1t + (size_t)i * K + (c0 + chunk) * kActChunk + c8 * 8);
      }
    }
    cp_async_commit();
  };
  for (int c = 0; c < lead; ++c) stage_l1(c);

  // inv_lambda of this CTA's K range, read by every token.  In shared memory
  // (when it fits) each 256-wide chunk is stored as [q][l][4] -- element
  // 16 l + 4 q + j at (16 q + l) * 4 + j -- so that lane l's four float4
  // reads of its 16 elements hit distinct banks.
  const int k_range = cpk * kActChunk;
  const bool il_smem = act_il_in_smem(r, k_range);
  // NVFP4 per-code block-scale tables (see quantize16): same values as
  // computing them per block, looked up instead
  __shared__ float dq_tab[512];
  if (FMT == SVDQ_NVFP4 && tid < 256) {
    const float d = __fmul_rn(e4m3_val((uint32_t)tid), s_gx);
    dq_tab[tid] = d;
    dq_tab[256 + tid] = (d != 0.0f && recip_ok(d)) ? __frcp_rn(d) : 0.0f;
  }
  const float* il_s = reinterpret_cast<const float*>(act_smem + act_ring_bytes(r) / 2);
  if (il_smem) {
    float* dst = reinterpret_cast<float*>(act_smem + act_ring_bytes(r) / 2);
    const float4* src = reinterpret_cast<const float4*>(a.inv_lambda + (size_t)c0 * kActChunk);
    for (int i = tid; i < k_range / 4; i += kActThreads) {
      const int ch = i / 64, w = i % 64, l = w >> 2, q = w & 3;   // float4 w of chunk ch = lane l, quarter q
      reinterpret_cast<float4*>(dst + ch * kActChunk)[q * 16 + l] = __ldg(src + i);
    }
  }
  __syncthreads();

  for (int c = 0; c < cpk; ++c) {
    const int k0 = (c0 + c) * kActChunk;
    const int buf = c & 1;
    load_x(c + 2, xnn);
    const int kk = k0 + col;
    float il[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = il_smem ? reinterpret_cast<const float4*>(il_s + c * kActChunk)[i * 16 + (lane & 15)]
                               : __ldg(reinterpret_cast<const float4*>(a.inv_lambda + kk + 4 * i));
      il[4 * i] = f.x; il[4 * i + 1] = f.y; il[4 * i + 2] = f.z; il[4 * i + 3] = f.w;
    }
    const uint16_t* x16 = reinterpret_cast<const uint16_t*>(xc);
    float xh[16];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      f2_unpack(f2_mul(f2_pack(half_to_f32<DT>(x16[2 * i]), half_to_f32<DT>(x16[2 * i + 1])),
                       f2_pack(il[2 * i], il[2 * i + 1])),
                xh[2 * i], xh[2 * i + 1]);
    QuantDst qd;
    if (FMT == SVDQ_NVFP4) {
      qd.tile = row_tiles ? row_tiles + (size_t)(c0 + c) * kATile : nullptr;
      qd.code_off = code_off;
      qd.sf_off = sf_off;
      qd.codes = nullptr;
      qd.sx = nullptr;
    } else {
      qd.tile = nullptr;
      qd.code_off = qd.sf_off = 0;
      qd.codes = row_codes ? row_codes + (size_t)k0 : nullptr;
      const int grp = (c0 + c) * 4 + (col >> 6);   // this lane's group of 64 (int4_sx_index)
      qd.sx = sx_lead ? reinterpret_cast<float*>(a.xs) + (size_t)(grp >> 1) * sx_pitch + sx_base + (size_t)(grp & 1) * 128
                      : nullptr;
    }
    quantize16<FMT>(xh, qd, six_sg, r6, dq_tab);
    uint4 o0, o1;
    o0.x = pack_half2_rn<DT>(xh[0], xh[1]);   o0.y = pack_half2_rn<DT>(xh[2], xh[3]);
    o0.z = pack_half2_rn<DT>(xh[4], xh[5]);   o0.w = pack_half2_rn<DT>(xh[6], xh[7]);
    o1.x = pack_half2_rn<DT>(xh[8], xh[9]);   o1.y = pack_half2_rn<DT>(xh[10], xh[11]);
    o1.z = pack_half2_rn<DT>(xh[12], xh[13]); o1.w = pack_half2_rn<DT>(xh[14], xh[15]);
    uint4* dst = reinterpret_cast<uint4*>(xs16(buf) + rw * kActStride + col);
    dst[0] = o0;
    dst[1] = o1;
    // this chunk's L1^T group is complete once at most lead-1 newer ones remain
    if (lead == 2) cp_async_wait_1(); else cp_async_wait_all();
    __syncthreads();
    // the buffer refilled here was last read by the previous chunk's MMAs
    stage_l1(c + lead);
    const uint16_t* l1c = l1sb(c % nbuf);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int tt = warp + 16 * t;
      if (tt < n_mma) {
        const int mt = tt & 1, nt = tt >> 1;
        const uint32_t a_base = smem_u32(xs16(buf) + (mt * 16 + (lane & 15)) * kActStride + (lane >> 4) * 8);
        const uint32_t b_base = smem_u32(l1c + (nt * 8 + (lane & 7)) * kActStride + ((lane >> 3) & 1) * 8);
        // two accumulators (even / odd k-steps) halve the dependent MMA chain
#pragma unroll 4
        for (int ks = 0; ks < kActChunk / 16; ks += 2) {
          uint32_t a0, a1, a2, a3, b0, b1;
          ldmatrix_x4(a_base + ks * 32, a0, a1, a2, a3);
          ldmatrix_x2(b_base + ks * 32, b0, b1);
          mma_16816<DT>(acc[t], a0, a1, a2, a3, b0, b1);
          ldmatrix_x4(a_base + ks * 32 + 32, a0, a1, a2, a3);
          ldmatrix_x2(b_base + ks * 32 + 32, b0, b1);
          mma_16816<DT>(acc2[t], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    xc[0] = xn[0]; xc[1] = xn[1];
    xn[0] = xnn[0]; xn[1] = xnn[1];
  }
  cp_async_wait_all();
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] += acc2[t][i];
  if (KS > 1) {
    // 1. a cluster's partials -> its CTA 0 through distributed shared memory, in rank order
    const int CL = GS ? kActClusterKs : KS;   // CTAs per cluster
    const int crank = kidx % CL;
    float* red = reinterpret_cast<float*>(act_smem);
    __syncthreads();   // the last chunk's MMAs have read their operands
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int tt = warp + 16 * t;
      if (tt < n_mma)
        *reinterpret_cast<float4*>(red + (tt * 32 + lane) * 4) = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
    }
    cluster_sync();
    if (crank == 0) {
      for (int src = 1; src < CL; ++src) {
        const uint32_t base = mapa_shared(smem_u32(red), (uint32_t)src);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int tt = warp + 16 * t;
          if (tt < n_mma) {
            const float4 v = ld_cluster_f32x4(base + (uint32_t)((tt * 32 + lane) * 16));
            acc[t][0] += v.x; acc[t][1] += v.y; acc[t][2] += v.z; acc[t][3] += v.w;
          }
        }
      }
    }
    cluster_sync();   // every partial stays in place until CTA 0 has read it
    if (crank != 0) return;
    if constexpr (GS) {
      // 2. the ks / 8 cluster sums meet in the workspace: each counts in on the
      //    group's arrival word; the last one adds them in K order
      const int g = (int)(blockIdx.x / KS);
      const int nc = KS / CL, kc = kidx / CL;
      float* mine = a.upart + ((size_t)g * nc + kc) * (size_t)(32 * r);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int tt = warp + 16 * t;
        if (tt < n_mma)
          __stcg(reinterpret_cast<float4*>(mine + (tt * 32 + lane) * 4), make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]));
      }
      __threadfence();
      __syncthreads();
      __shared__ int last_sh;
      if (tid == 0) {
        unsigned long long* w = a.ucnt + g;
        unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(w), seen;
        int last = 0;
        for (;;) {
          const bool same = (old >> 8) == a.epoch;
          const unsigned long long cnt = same ? (old & 0xFF) : 0ull;
          const unsigned long long next = (cnt + 1 == (unsigned long long)nc) ? 0ull : ((a.epoch << 8) | (cnt + 1));
          seen = atomicCAS(w, old, next);
          if (seen == old) { last = cnt + 1 == (unsigned long long)nc; break; }
          old = seen;
        }
        last_sh = last;
      }
      __syncthreads();
      if (!last_sh) return;
      __threadfence();
      const float* base = a.upart + (size_t)g * nc * (size_t)(32 * r);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int tt = warp + 16 * t;
        if (tt < n_mma) {
          const float4* src = reinterpret_cast<const float4*>(base) + tt * 32 + lane;
          const size_t step = (size_t)(32 * r) / 4;   // float4s per partial
          float4 w[kActGMaxKs / kActClusterKs];
#pragma unroll
          for (int i = 0; i < kActGMaxKs / kActClusterKs; ++i)
            w[i] = i < nc ? __ldcg(src + (size_t)i * step) : make_float4(0.f, 0.f, 0.f, 0.f);
          float4 s4 = w[0];
#pragma unroll
          for (int i = 1; i < kActGMaxKs / kActClusterKs; ++i)
            if (i < nc) { s4.x += w[i].x; s4.y += w[i].y; s4.z += w[i].z; s4.w += w[i].w; }
          acc[t][0] = s4.x; acc[t][1] = s4.y; acc[t][2] = s4.z; acc[t][3] = s4.w;
        }
      }
    }
  }
  // u' = u * inv_alpha, split into bf16 hi + lo: [hi | lo (| hi) | 0 pad];
  // NVFP4 keeps it as swizzled low-rank tiles over the padded rows
  const int64_t u_rows = FMT == SVDQ_NVFP4 ? a.Mp : a.M;
  auto ux_at = [&](int64_t mm, int e) -> uint32_t* {
    if constexpr (FMT == SVDQ_NVFP4) {
      uint8_t* tile = reinterpret_cast<uint8_t*>(a.ux) + ((size_t)(mm >> 7) * (a.lrw / 64) + e / 64) * kLRTile;
      return reinterpret_cast<uint32_t*>(tile + sw128((uint32_t)(mm & 127), (uint32_t)(e & 63) * 2));
    } else {
      return reinterpret_cast<uint32_t*>(a.ux + (size_t)mm * a.lrw + e);
    }
  };
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int tt = warp + 16 * t;
    if (tt < n_mma) {
      const int mt = tt & 1, nt = tt >> 1;
      const int ucol = nt * 8 + 2 * (lane & 3);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int64_t mu = m0 + mt * 16 + (lane >> 2) + half * 8;
        if (mu < u_rows) {
          uint16_t hi[2], lo[2];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const float v = acc[t][half * 2 + cc] * inv_alpha;
            hi[cc] = bf16_rn(v);
            lo[cc] = bf16_rn(v - __uint_as_float((uint32_t)hi[cc] << 16));
          }
          *ux_at(mu, ucol) = hi[0] | ((uint32_t)hi[1] << 16);
          *ux_at(mu, r + ucol) = lo[0] | ((uint32_t)lo[1] << 16);
          if (a.nseg == 3) *ux_at(mu, 2 * r + ucol) = hi[0] | ((uint32_t)hi[1] << 16);
        }
      }
    }
  }
  const int used = a.nseg * r;
  const int pad = a.lrw - used;
  if (pad > 0) {
    for (int idx = tid; idx < kActRows * (pad / 2); idx += kActThreads) {
      const int64_t mu = m0 + idx / (pad / 2);
      if (mu < u_rows) *ux_at(mu, used + 2 * (idx % (pad / 2))) = 0;
    }
  }
}

// ------------------------------------------------------------ kernel 2 (shared parts)
constexpr int kBM = 128;          // tokens per tile (TMEM lanes)
constexpr int kABytes = kBM * 128;   // one 128-byte-wide K slab of A

struct GemmArgs {
  int64_t M;
  int N, K;
  int lr_iters;       // low-rank K-steps of 64 bf16
  int k_iters;        // 4-bit K slabs of 128 bytes
  const uint8_t* sfa; // activation scales (workspace)
  const uint8_t* sfb; // weight scales (blob)
  const float* bias;
  const BlobHeader* hdr;
  uint16_t* Y;
  int64_t Mp;
};

// Bounded wait that ignores the abort flag (used to drain copies in flight).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      record_status(kStatusTimeout);
      return;
    }
  }
}

// ------------------------------------------------------------ kernel 1, NVFP4 form
// NVFP4 activations on 128-token tiles (one TMEM lane per token), with the K
// range of a tile split over ks CTAs (act_nv_ks) so that the grid fills the
// SMs.  Per 128-wide half of a 256-wide K slab (one ring stage):
//   producer   TMA-loads the X half slab (128 tokens x 128: two 128-byte-
//              swizzled atoms), the matching L1^T columns and inv_lambda;
//   quantiser  16 warps; warp w owns 16-element block w % 8 of the half for
//              tokens 64 (w / 8) + lane + {0, 32}: X^ = fp32(x) * inv_lambda,
//              block amax -> E4M3 scale -> E2M1 codes, written straight into
//              the GEMM's activation tile in shared memory; X^ rounded to the
//              16-bit dtype overwrites x in place, which makes the stage the A
//              operand of the down projection;
//   MMA thread issues u += X^16 L1 on tcgen05 (M = 128 tokens, N = r, fp32 in
//              TMEM), frees the stage, and once both halves of a slab are
//              quantised writes the 18 KB activation tile out with one bulk copy.
// After the last slab four warps read the partial u from TMEM.  With ks = 1
// they write u' = u / (s_gX s_gW) as bf16 hi + lo into the low-rank input
// tile.  With ks > 1 every CTA writes its partial to the workspace and
// counts in on its tile's arrival word (tagged with this call's epoch, so no
// initial value is needed); the last CTA to arrive adds the ks partials in K
// order (deterministic), writes u' and clears the word.  Tokens past M stay
// zero (TMA fills them, and zeros quantise to zero codes and scale 0).
struct ActNvArgs {
  int64_t M, Mp;
  int K, r, lrw, nseg;
  int slabs;          // 256-wide K slabs per CTA
  int ks;             // CTAs per 128-token tile (K split)
  int stages;         // ring depth
  unsigned long long epoch;   // nonzero, distinct per call (K split arrivals)
  const float* inv_lambda;
  const BlobHeader* hdr;
  uint8_t* xq;        // activation tiles [Mp/128][K/256]
  uint8_t* ux;        // low-rank input tiles [Mp/128][lrw/64]
  float* upart;       // ks > 1: partial u [Mp/128][ks][128][r]
  unsigned long long* ucnt;   // ks > 1: arrival word per 128-token tile
  int* gemm_cnt;      // GEMM K-split arrival counters to clear (or null)
  int n_cnt;
};

constexpr int kAN_Quant = 16;
constexpr int kAN_Threads = (2 + kAN_Quant) * 32;
constexpr int kAN_XBytes = 128 * 128 * 2;        // X half slab: two 16 KB atoms
constexpr int kAN_IlBytes = 128 * 4;             // inv_lambda of the half slab
constexpr int kAN_Budget = 232448 - 4096;        // dynamic shared memory budget (static tables aside)
constexpr int kAN_MaxStages = 6;

// stage: [X atoms | L1^T atoms (2 x r rows x 128 bytes) | inv_lambda], 1024-aligned
SVDQ_HD inline int an_stage_bytes(int r) { return (kAN_XBytes + 2 * r * 128 + kAN_IlBytes + 1023) / 1024 * 1024; }
SVDQ_HD inline int an_stages(int r) {
  const int s = (kAN_Budget - 1024 - 2 * kATile) / an_stage_bytes(r);
  return s > kAN_MaxStages ? kAN_MaxStages : s;
}
SVDQ_HD inline int an_smem_bytes(int r) { return 1024 + an_stages(r) * an_stage_bytes(r) + 2 * kATile; }

// One NVFP4 block of 16 smoothed activations -> 8 code bytes (p0, p1) and
// the E4M3 scale code (same arithmetic as quantize16).
__device__ __forceinline__ void nv_block(const float (&xh)[16], float six_sg, float r6, const float* dq,
                                         uint32_t& p0, uint32_t& p1, uint32_t& e) {
  float m8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m8[i] = fmaxf(fabsf(xh[i]), fabsf(xh[i + 8]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m8[i] = fmaxf(m8[i], m8[i + 4]);
  const float amax = fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3]));
  const float ratio = r6 != 0.0f ? div_by_recip(amax, six_sg, r6) : __fdiv_rn(amax, six_sg);
  e = cvt_e4m3x2(0.0f, ratio) & 0xFFu;
  const float d = dq[e];
  const float rd = dq[256 + e];
  p0 = 0; p1 = 0;
  if (d != 0.0f) {
    if (rd != 0.0f) {
      const uint64_t nd2 = f2_pack(-d, -d), r2 = f2_pack(rd, rd);
      uint32_t b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float q0, q1;
        f2_unpack(div2_by_recip(f2_pack(xh[2 * i], xh[2 * i + 1]), nd2, r2), q0, q1);
        b[i] = cvt_e2m1x2(q1, q0);
      }
      p0 = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
      p1 = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        p0 |= cvt_e2m1x2(__fdiv_rn(xh[2 * i + 1], d), __fdiv_rn(xh[2 * i], d)) << (8 * i);
        p1 |= cvt_e2m1x2(__fdiv_rn(xh[2 * i + 9], d), __fdiv_rn(xh[2 * i + 8], d)) << (8 * i);
      }
    }
  }
}

template <int DT>
__device__ __forceinline__ void unpack8(const uint4 v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (DT == SVDQ_BF16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(kAN_Threads, 1)
    act_nvfp4_kernel(const ActNvArgs a, const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_l1) {
  extern __shared__ __align__(1024) uint8_t an_raw[];
  __shared__ uint64_t full_bar[kAN_MaxStages], empty_bar[kAN_MaxStages], qdone_bar[kAN_MaxStages];
  __shared__ uint64_t tfree_bar[2], accf_bar;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh, last_sh;
  __shared__ float dq_tab[512];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(an_raw) + 1023) & ~uintptr_t(1023));
  const int S = a.stages, r = a.r;
  const int sbytes = an_stage_bytes(r);
  const int off_il = kAN_XBytes + 2 * r * 128;
  const uint32_t stage_tx = (uint32_t)(kAN_XBytes + 2 * r * 128 + kAN_IlBytes);
  uint8_t* ctile = smem + S * sbytes;            // two activation tiles being assembled
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = a.ks;
  const int kq = blockIdx.x % KS;                // K part of the tile
  const int mtile = blockIdx.x / KS;             // 128-token tile
  const int64_t m0 = (int64_t)mtile * 128;
  const int slab0 = kq * a.slabs;
  const int nhalf = 2 * a.slabs;
  const int ksl = a.K / 256;
  const uint32_t tcols = r <= 32 ? 32u : (r <= 64 ? 64u : 128u);
  // a tile wholly past the last token (M rounded up to the GEMM's 256 rows)
  // loads nothing: its activation tiles and low-rank rows are written as zeros
  const bool live_tile = m0 < a.M;
  const int rows_live = live_tile ? (int)(a.M - m0 < 128 ? a.M - m0 : 128) : 0;
  volatile int* abort_flag = &abort_sh;

  griddep_launch();   // the GEMM may start its prologue on idle SMs
  // ring stage c: X half slab, L1^T columns and inv_lambda at K offset (2 slab0 + c) * 128
  auto issue_half = [&](int c) {
    const int s = c % S;
    uint8_t* st = smem + s * sbytes;
    const int k0 = slab0 * 256 + c * 128;
    mbar_arrive_expect_tx(&full_bar[s], stage_tx);
    tma_load_2d(st, &tm_x, &full_bar[s], k0, (int)m0);
    tma_load_2d(st + 16384, &tm_x, &full_bar[s], k0 + 64, (int)m0);
    if (r > 0) {
      tma_load_2d(st + kAN_XBytes, &tm_l1, &full_bar[s], k0, 0);
      tma_load_2d(st + kAN_XBytes + r * 128, &tm_l1, &full_bar[s], k0 + 64, 0);
    }
    bulk_load(st + off_il, a.inv_lambda + k0, kAN_IlBytes, &full_bar[s]);
  };
  const int first = nhalf < S ? nhalf : S;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); mbar_init(&qdone_bar[s], kAN_Quant);
    }
    mbar_init(&tfree_bar[0], 1); mbar_init(&tfree_bar[1], 1);
    mbar_init(&accf_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    if (live_tile)   // the first stages load while the rest of the CTA sets up
      for (int c = 0; c < first; ++c) issue_half(c);
  }
  const float s_gx = a.hdr->s_gx;
  if (threadIdx.x < 256) {
    const float d = __fmul_rn(e4m3_val((uint32_t)threadIdx.x), s_gx);
    dq_tab[threadIdx.x] = d;
    dq_tab[256 + threadIdx.x] = (d != 0.0f && recip_ok(d)) ? __frcp_rn(d) : 0.0f;
  }
  if (rows_live < 128)   // rows past M keep zero codes and scales (never written below)
    for (int i = threadIdx.x; i < 2 * kATile / 16; i += kAN_Threads)
      reinterpret_cast<uint4*>(ctile)[i] = make_uint4(0, 0, 0, 0);
  if (blockIdx.x == 0 && a.gemm_cnt)
    for (int i = threadIdx.x; i < a.n_cnt; i += kAN_Threads) a.gemm_cnt[i] = 0;
  if (warp == 1) { tmem_alloc(&tmem_sh, tcols); tmem_relinquish(); }
  fence_proxy_async_smem();   // zeroed tiles are read by bulk copies
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_sh;
  uint8_t* const xq_tile = a.xq + (size_t)mtile * ksl * kATile;   // + slab * kATile

  if (!live_tile) {
    if (warp == 1 && lane == 0) {
      for (int t = 0; t < a.slabs; ++t) bulk_store(xq_tile + (size_t)(slab0 + t) * kATile, ctile, kATile);
      bulk_commit();
      bulk_wait_all();
    }
  } else if (warp == 0) {
    if (lane == 0) {
      int issued = first;
      for (int c = first; c < nhalf; ++c) {
        const int s = c % S;
        if (!mbar_wait(&empty_bar[s], ((c / S) & 1) ^ 1, abort_flag)) break;
        issue_half(c);
        issued = c + 1;
      }
      if (*abort_flag)
        for (int i = issued - 1; i >= 0 && i >= issued - S; --i) mbar_drain(&full_bar[i % S], (i / S) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = DT == SVDQ_BF16 ? idesc_f16_bf16(128, r) : idesc_f16_f16(128, r);
      bool dead = false;
      for (int c = 0; c < nhalf; ++c) {
        const int s = c % S;
        if (!mbar_wait(&qdone_bar[s], (c / S) & 1, abort_flag)) { dead = true; break; }
        tc_fence_after();
        if (r > 0) {
          const uint32_t a_addr = smem_u32(smem + s * sbytes);
          const uint32_t b_addr = a_addr + kAN_XBytes;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mma_f16(tbase, desc_k_sw128(a_addr + h * 16384 + 32 * q), desc_k_sw128(b_addr + h * r * 128 + 32 * q),
                      idesc, (c | h | q) != 0);
        }
        mma_commit(&empty_bar[s]);
        if (c & 1) {
          // both halves of slab t are in the tile buffer: one bulk copy out
          const int t = c >> 1;
          bulk_store(xq_tile + (size_t)(slab0 + t) * kATile, ctile + (t & 1) * kATile, kATile);
          bulk_commit();
          bulk_wait_read<0>();
          mbar_arrive(&tfree_bar[t & 1]);
        }
      }
      mma_commit(&accf_bar);
      if (dead) mbar_drain(&accf_bar, 0);
      bulk_wait_all();
    }
  } else {
    // quantiser warps
    const int qw = warp - 2;
    const int jb = qw & 7;                         // 16-element block inside the half slab
    const int row0 = (qw >> 3) * 64 + lane;        // tokens row0 and row0 + 32 of the tile
    const int cc = (jb & 3) * 2;                   // its first 16-byte chunk in a 128-byte atom row
    const float six_sg = __fmul_rn(6.0f, s_gx);
    const float r6 = recip_ok(six_sg) ? __frcp_rn(six_sg) : 0.0f;
    // rows of this warp past the last token are zero and stay unquantised
    const int nrow = (qw >> 3) * 64 < rows_live ? ((qw >> 3) * 64 + 32 < rows_live ? 2 : 1) : 0;
    for (int c = 0; c < nhalf; ++c) {
      const int s = c % S, t = c >> 1, h = c & 1;
      if (h == 0 && t >= 2)
        if (!mbar_wait(&tfree_bar[t & 1], ((t >> 1) - 1) & 1, abort_flag)) break;
      if (!mbar_wait(&full_bar[s], (c / S) & 1, abort_flag)) break;
      uint8_t* st = smem + s * sbytes;
      float il[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = reinterpret_cast<const float4*>(st + off_il)[4 * jb + i];
        il[4 * i] = f.x; il[4 * i + 1] = f.y; il[4 * i + 2] = f.z; il[4 * i + 3] = f.w;
      }
      uint8_t* xatom = st + (jb >> 2) * 16384;
      uint8_t* tileb = ctile + (t & 1) * kATile;
      const int j16 = 8 * h + jb;                  // block inside the 256-wide slab
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (i >= nrow) break;
        const int row = row0 + 32 * i;
        uint8_t* rowp = xatom + row * 128;
        uint4* c0p = reinterpret_cast<uint4*>(rowp + ((cc ^ (row & 7)) << 4));
        uint4* c1p = reinterpret_cast<uint4*>(rowp + (((cc + 1) ^ (row & 7)) << 4));
        float xf[16];
        unpack8<DT>(*c0p, xf);
        unpack8<DT>(*c1p, xf + 8);
        float xh[16];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          f2_unpack(f2_mul(f2_pack(xf[2 * k], xf[2 * k + 1]), f2_pack(il[2 * k], il[2 * k + 1])), xh[2 * k],
                    xh[2 * k + 1]);
        uint32_t p0, p1, e;
        nv_block(xh, six_sg, r6, dq_tab, p0, p1, e);
        *reinterpret_cast<uint2*>(tileb + sw128((uint32_t)row, 8u * (uint32_t)j16)) = make_uint2(p0, p1);
        tileb[kTileCodes + tile_sf((uint32_t)row, (uint32_t)j16)] = (uint8_t)e;
        uint4 o0, o1;
        o0.x = pack_half2_rn<DT>(xh[0], xh[1]);   o0.y = pack_half2_rn<DT>(xh[2], xh[3]);
        o0.z = pack_half2_rn<DT>(xh[4], xh[5]);   o0.w = pack_half2_rn<DT>(xh[6], xh[7]);
        o1.x = pack_half2_rn<DT>(xh[8], xh[9]);   o1.y = pack_half2_rn<DT>(xh[10], xh[11]);
        o1.z = pack_half2_rn<DT>(xh[12], xh[13]); o1.w = pack_half2_rn<DT>(xh[14], xh[15]);
        *c0p = o0;
        *c1p = o1;
      }
      fence_proxy_async_smem();   // X^16 and the tile are read by the tensor core and a bulk copy
      __syncwarp();
      if (lane == 0) mbar_arrive(&qdone_bar[s]);
    }
  }

  // ---- partial u: TMEM -> the workspace (ks > 1) or shared memory (ks = 1),
  // live rows only (warps 2..5, one TMEM lane quarter each)
  const bool epi = warp >= 2 && warp < 6;
  const int rs = r + 4;                            // row stride of the shared-memory copy
  if (epi && r > 0 && live_tile && __all_sync(0xffffffffu, mbar_wait(&accf_bar, 0, abort_flag))) {
    tc_fence_after();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    float* part = a.upart + (((size_t)mtile * KS + kq) * 128 + row) * r;
    for (int c0 = 0; c0 < r; c0 += 16) {
      uint32_t v[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
          "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
            "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
          : "r"(tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)c0));
      tmem_ld_wait();
      if (row < rows_live) {
        float4* dst = KS > 1 ? reinterpret_cast<float4*>(part + c0)
                             : reinterpret_cast<float4*>(reinterpret_cast<float*>(smem) + row * rs + c0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 f = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                       __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
          if (KS > 1) __stcg(dst + k, f); else dst[k] = f;
        }
      }
    }
    if (KS > 1) __threadfence();   // the partial is visible before this CTA counts in
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, tcols);
  }
  // ---- K split: count in; the last CTA of the tile adds the partials
  bool finisher = true;
  if (KS > 1 && r > 0 && live_tile) {
    if (threadIdx.x == 64) {
      __threadfence();
      unsigned long long* w = a.ucnt + mtile;
      unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(w), seen;
      int last = 0;
      for (;;) {
        const bool same = (old >> 8) == a.epoch;
        const unsigned long long cnt = same ? (old & 0xFF) : 0ull;
        const unsigned long long next = (cnt + 1 == (unsigned long long)KS) ? 0ull : ((a.epoch << 8) | (cnt + 1));
        seen = atomicCAS(w, old, next);
        if (seen == old) { last = cnt + 1 == (unsigned long long)KS; break; }
        old = seen;
      }
      last_sh = last;
    }
    __syncthreads();
    finisher = last_sh != 0;
    if (finisher) __threadfence();
  }
  if (!finisher || a.lrw == 0) return;
  // ---- u' = u / (s_gX s_gW) as bf16 hi + lo into the low-rank input tile.
  // Work items are (live row, 4 columns); a group of `lpi` lanes shares an
  // item, lane i of the group adding partials i, i + lpi, ... in K order, and
  // the group combines its lanes with a fixed shuffle tree (the same order on
  // every call for a given shape).
  const float inv_alpha = 1.0f / (a.hdr->s_gx * a.hdr->s_gw);
  uint8_t* utiles = a.ux + (size_t)mtile * (a.lrw / 64) * kLRTile;
  auto store4 = [&](int row, int col, uint32_t w0, uint32_t w1) {   // 4 bf16 at columns col..col+3
    uint8_t* tile = utiles + (size_t)(col / 64) * kLRTile;
    *reinterpret_cast<uint2*>(tile + sw128((uint32_t)row, (uint32_t)(col % 64) * 2)) = make_uint2(w0, w1);
  };
  const int c4 = r / 4;
  const int items = rows_live * c4;
  int lpi = 1;
  if (KS > 1)
    while (lpi < 32 && lpi < KS && items * lpi * 2 <= kAN_Threads) lpi *= 2;
  const int groups = kAN_Threads / lpi;
  const int gid = (int)threadIdx.x / lpi, gl = (int)threadIdx.x % lpi;
  for (int it0 = 0; it0 < items; it0 += groups) {   // uniform trip count: the shuffles need every lane
    const int it = it0 + gid;
    const bool act = it < items;
    const int row = act ? it / c4 : 0, col = act ? (it % c4) * 4 : 0;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (act) {
      if (KS > 1) {
        // this lane's partials (at most kActMaxKs / lpi), all loads in flight before the K-ordered sum
        const float* base = a.upart + ((size_t)mtile * KS * 128 + row) * r + col;
        const int nsrc = (KS - gl + lpi - 1) / lpi;
        for (int b0 = 0; b0 < nsrc; b0 += 4) {
          float4 w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (b0 + i < nsrc) w[i] = __ldcg(reinterpret_cast<const float4*>(base + (size_t)(gl + (b0 + i) * lpi) * 128 * r));
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (b0 + i < nsrc) { u.x += w[i].x; u.y += w[i].y; u.z += w[i].z; u.w += w[i].w; }
        }
      } else {
        u = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(smem) + row * rs + col);
      }
    }
    for (int off = 1; off < lpi; off <<= 1) {
      u.x += __shfl_xor_sync(0xffffffffu, u.x, off);
      u.y += __shfl_xor_sync(0xffffffffu, u.y, off);
      u.z += __shfl_xor_sync(0xffffffffu, u.z, off);
      u.w += __shfl_xor_sync(0xffffffffu, u.w, off);
    }
    if (act && gl == 0) {
      const float v[4] = {u.x * inv_alpha, u.y * inv_alpha, u.z * inv_alpha, u.w * inv_alpha};
      uint32_t hi[2], lo[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t h0 = bf16_rn(v[2 * k]), h1 = bf16_rn(v[2 * k + 1]);
        const uint32_t l0 = bf16_rn(v[2 * k] - __uint_as_float(h0 << 16));
        const uint32_t l1 = bf16_rn(v[2 * k + 1] - __uint_as_float(h1 << 16));
        hi[k] = h0 | (h1 << 16);
        lo[k] = l0 | (l1 << 16);
      }
      store4(row, col, hi[0], hi[1]);
      store4(row, r + col, lo[0], lo[1]);
      if (a.nseg == 3) store4(row, 2 * r + col, hi[0], hi[1]);
    }
  }
  // zero padding columns of the live rows and every column of the rows past M
  const int pad0 = a.nseg * r;
  const int npad = (a.lrw - pad0) / 4;
  const int zitems = rows_live * npad + (128 - rows_live) * (a.lrw / 4);
  for (int it = threadIdx.x; it < zitems; it += kAN_Threads) {
    int row, col;
    if (it < rows_live * npad) { row = it / npad; col = pad0 + (it % npad) * 4; }
    else { const int j = it - rows_live * npad; row = rows_live + j / (a.lrw / 4); col = (j % (a.lrw / 4)) * 4; }
    store4(row, col, 0u, 0u);
  }
}

// Epilogue store: 32 consecutive fp32 accumulator columns of one row -> bf16.
__device__ __forceinline__ void store_row32(uint16_t* dst, const float* v, const float* bias, float alpha) {
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float y0 = fmaf(alpha, v[2 * j], bias[2 * j]);
    const float y1 = fmaf(alpha, v[2 * j + 1], bias[2 * j + 1]);
    w[j] = (uint32_t)bf16_rn(y0) | ((uint32_t)bf16_rn(y1) << 16);
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

// ------------------------------------------------------------ kernel 2, NVFP4 (CTA pairs)
// Persistent, clusters of 2 CTAs; each pair walks 256 x 256 output tiles
// (pair p: tile p, p + pairs, ..., n fastest).  In a pair, CTA r holds A rows
// [128r, 128r + 128) of the tile and B rows (output features) [128r, 128r+128)
// in its shared memory; the leader (rank 0) issues cta_group::2 MMAs
// (M = 256, N = 256) that read both CTAs' operands and accumulate each CTA's
// 128 rows in its own TMEM, so every B byte is fetched once per pair.
//
// Data path: the operands are stored as ready-made tiles (swizzled codes
// followed by their scale atoms), so a K slab of one CTA is two bulk copies
// (activation tile 18 KB, weight tile 20 KB) into a 5-deep stage ring.  Each
// CTA's copies signal its own `landed` barrier.
// Scale factors: four scale warps per CTA (one per TMEM lane quarter) wait
// for their stage to land, copy its scale atoms to that stage's TMEM slot
// with tcgen05.st, and arrive on the leader's `ready` barrier; the MMA
// issuer waits only for `ready` (all eight scale warps of both CTAs), which
// implies both CTAs' bytes landed.  The leader's tcgen05.commit (CTA mask
// 0b11) frees the stage in both CTAs.  A stage refills only after its MMAs
// completed, so the TMEM scale slot needs no separate release.
//
// Warps (four warpgroups, register budgets set with setmaxnreg so that the
// sum fits the 64K-register file): 0 producer, 1 TMEM owner + MMA issuer
// (leader), 2-3 idle [56 regs]; 4-7 scale warps [80]; 8-15 epilogue, lane
// quarter warp % 4, column half (warp - 8) / 4 [184].  The
// epilogue copies its 128 accumulator columns to registers with four
// back-to-back tcgen05.ld, releases TMEM, then adds alpha / bias and stores
// bf16 rows while the next tile runs.
// TMEM: [0,256) accumulator; stage s scale slot at 256 + 48 s (SFA 16, SFB 32 columns).
constexpr int kS_SFA = kTileCodes;                 // stage: [A codes | SFA | B codes | SFB]
constexpr int kS_B = kATile;
constexpr int kS_SFB = kATile + kTileCodes;
constexpr int kS_Size = kATile + kWTile;           // 38912
constexpr int kP_Stages = 5;
constexpr int kEpiWarps = 8;
constexpr int kP_Threads = 16 * 32;
constexpr int kEpiChunk = 32 * 128;               // 32 rows x 64 bf16 columns, 128-byte swizzled
constexpr int kP_Smem = kP_Stages * kS_Size + kEpiWarps * kEpiChunk + 1024;
// Chained form (the epilogue emits the next layer's quantised input): a
// 4-deep ring; the tile's X^16 (128 rows x 256 columns bf16, four 64-column
// swizzled tiles) and this CTA's half of the next layer's L1^T rows for the
// tile's 256 columns replace the output chunks; the partial down projection
// (next rank <= 32 columns) sits in TMEM after the scale slots.
constexpr int kC_Stages = 4;
constexpr int kC_MaxR = 32;
constexpr int kC_XHat = 4 * kLRTile;                      // 65536
constexpr int kC_L1 = 4 * (kC_MaxR / 2) * 128;            // 8192
constexpr int kC_Smem = kC_Stages * kS_Size + kC_XHat + kC_L1 + 1024;
constexpr uint32_t kC_UCol = 256 + 48 * kC_Stages;        // 448
static_assert(kC_UCol + kC_MaxR <= 512, "TMEM columns");
static_assert((kC_Stages * kS_Size) % 1024 == 0, "X^16 tiles must start on a 1024-byte boundary");

struct PairArgs {
  int64_t M, Mp;
  int N, K;
  int lr_iters;            // low-rank K steps (64 bf16 each)
  int k_iters;             // 4-bit K slabs (256 elements each)
  const uint8_t* atiles;   // activation tiles [Mp/128][K/256]
  const uint8_t* wtiles;   // weight tiles [N/128][K/256]
  const uint8_t* utiles;   // low-rank input tiles [Mp/128][lr_iters]
  const uint8_t* l2tiles;  // low-rank weight tiles [N/128][lr_iters]
  const float* bias;
  const BlobHeader* hdr;
  uint16_t* Y;
  int ks;                  // K split (few output tiles): items = tiles x ks
  float* part;             // ks > 1: fp32 partial sums [ks][M][N]
  int* cnt;                // ks > 1: arrival counters [tiles][16] (zero between calls)
  // chained form only: the next layer's input instead of Y
  const float* nx_inv_lambda;   // next layer's 1/lambda (N values)
  const BlobHeader* nx_hdr;     // next layer's header (activation tensor scale)
  uint8_t* nx_atiles;           // next layer's activation tiles [Mp/128][N/256]
  float* nx_upart;              // partial down projections [N/256][Mp][nx_r]
  int nx_r;                     // next layer's rank: 0, 16 or 32
};

template <bool CHAIN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kP_Threads, 1)
    gemm_nvfp4_pair_kernel(const PairArgs g, const __grid_constant__ CUtensorMap tm_y,
                           const __grid_constant__ CUtensorMap tm_l1n) {
  constexpr int kStages = CHAIN ? kC_Stages : kP_Stages;
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  __shared__ uint64_t landed_bar[kStages], empty_bar[kStages], ready_bar[kStages], accf_bar, acce_bar;
  __shared__ uint64_t xready_bar, ufull_bar, l1_bar;   // chained form
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ychunks = smem + kStages * kS_Size;   // one 4 KB output chunk per epilogue warp
  uint8_t* xhat = smem + kStages * kS_Size;      // chained form: X^16 tiles, then the L1^T half
  uint8_t* l1buf = xhat + kC_XHat;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
  const int n_tiles = g.N / 256;
  const int num_tiles = n_tiles * (int)(g.Mp / 256);
  const int ksl = g.K / 256;
  // Work items: output tile x K range.  With g.ks > 1 item (t, kq) covers
  // slabs [kq cpk, (kq + 1) cpk); only kq = 0 adds the low-rank steps.
  const int num_items = num_tiles * g.ks;
  const int cpk = g.k_iters / g.ks;
  auto item_lr = [&](int item) { return (item % g.ks) == 0 ? g.lr_iters : 0; };
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&landed_bar[s], 1); mbar_init(&empty_bar[s], 1); mbar_init(&ready_bar[s], 2 * 4);
    }
    mbar_init(&accf_bar, 1);
    mbar_init(&acce_bar, 2 * kEpiWarps);
    mbar_init(&xready_bar, 2 * kEpiWarps);
    mbar_init(&ufull_bar, 1);
    mbar_init(&l1_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc_pair(&tmem_base_sh, 512); tmem_relinquish_pair(); }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tbase = tmem_base_sh;
  const uint32_t peer_abort = mapa_shared(smem_u32(&abort_sh), rank ^ 1u);
  auto give_up_both = [&]() { st_cluster_u32(peer_abort, 1u); };

  if (warp == 0) {
    regs_dec<56>();
    if (lane == 0) {
      // The weights do not depend on the activation kernel: when every pair
      // has a single tile (few tokens), pull this CTA's weight tiles into L2
      // while that kernel runs; then wait for it before touching the workspace.
      if (num_items <= pairs && pair < num_items) {   // one item per pair: weight streaming dominates
        const int t0 = pair / g.ks, kq0 = pair % g.ks;
        const size_t nb0 = (size_t)(2 * (t0 % n_tiles) + (int)rank);
        for (int kt = kq0 * cpk; kt < (kq0 + 1) * cpk; ++kt)
          bulk_prefetch_l2(g.wtiles + (nb0 * ksl + kt) * kWTile, kWTile);
      }
      griddep_wait();
      int it = 0, issued = 0;
      bool dead = false;
      for (int item = pair; item < num_items && !dead; item += pairs) {
        const int tile = item / g.ks, kq = item % g.ks, lr = item_lr(item);
        const int mt = tile / n_tiles, nt = tile % n_tiles;
        const size_t mb = (size_t)(2 * mt + (int)rank), nb = (size_t)(2 * nt + (int)rank);
        for (int j = 0; j < lr + cpk; ++j, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&empty_bar[s], ((it / kStages) & 1) ^ 1, abort_flag)) { give_up_both(); dead = true; break; }
          uint8_t* st = smem + s * kS_Size;
          if (j < lr) {
            mbar_arrive_expect_tx(&landed_bar[s], 2 * kLRTile);
            bulk_load(st, g.utiles + (mb * g.lr_iters + j) * kLRTile, kLRTile, &landed_bar[s]);
            bulk_load(st + kS_B, g.l2tiles + (nb * g.lr_iters + j) * kLRTile, kLRTile, &landed_bar[s]);
          } else {
            const int kt = kq * cpk + (j - lr);
            mbar_arrive_expect_tx(&landed_bar[s], kS_Size);
            bulk_load(st, g.atiles + (mb * ksl + kt) * kATile, kATile, &landed_bar[s]);
            bulk_load(st + kS_B, g.wtiles + (nb * ksl + kt) * kWTile, kWTile, &landed_bar[s]);
          }
          issued = it + 1;
        }
      }
      if (*abort_flag) {
        for (int i = issued - 1; i >= 0 && i >= issued - kStages; --i)
          mbar_drain(&landed_bar[i % kStages], (i / kStages) & 1);
      }
    }
  } else if (warp < 4) {
    regs_dec<56>();
    if (warp == 1 && leader && lane == 0) {
      const uint32_t id_lr = idesc_f16_bf16(256, 256);
      const uint32_t id_f4 = idesc_nvf4(256, 256);
      int it = 0, tcount = 0;
      bool dead = false;
      // chained form: tile t's partial down projection X^16 L1 (M = 256, N =
      // next rank, K = the tile's 256 columns) once its epilogue has staged
      // X^16 and the L1^T halves in both CTAs: between the stages of the next
      // tile's main loop as soon as the hand-off has landed (polled, never
      // waited on there), else at that loop's end
      const bool down = CHAIN && g.nx_r > 0;
      int pend = -1;   // the tile whose down projection is still to be issued
      auto issue_down = [&](int t) {
        tc_fence_after();
        const uint32_t id_u = idesc_f16_bf16(256, g.nx_r);
        const uint32_t xa = smem_u32(xhat), la = smem_u32(l1buf);
        const uint32_t lc = (uint32_t)(g.nx_r / 2) * 128u;   // bytes of one 64-column L1^T chunk
#pragma unroll 1
        for (int cq = 0; cq < 16; ++cq) {   // 64-column chunk cq / 4, K step cq % 4 (a loop: this warp has 56 registers)
          const int c = cq >> 2, q = cq & 3;
          mma_f16_pair(tbase + kC_UCol, desc_k_sw128(xa + c * kLRTile + 32 * q), desc_k_sw128(la + c * lc + 32 * q),
                       id_u, cq != 0);
        }
        mma_commit_pair(&ufull_bar, 0x3);
        pend = -1;
      };
      // blocking form (end of a main loop, or after the last tile)
      auto down_proj = [&](int t) -> bool {
        if (!mbar_wait_cluster(&xready_bar, (uint32_t)t & 1u, abort_flag)) { give_up_both(); return false; }
        issue_down(t);
        return true;
      };
      for (int item = pair; item < num_items && !dead; item += pairs, ++tcount) {
        const int lr = item_lr(item);
        if (!mbar_wait(&acce_bar, (tcount & 1) ^ 1, abort_flag)) { give_up_both(); break; }
        tc_fence_after();
        if (down && tcount > 0) pend = tcount - 1;
        for (int j = 0; j < lr + cpk; ++j, ++it) {
          const int s = it % kStages;
          // the previous tile's down projection as soon as its epilogue has staged X^16
          if (pend >= 0 && mbar_try_wait_cluster(&xready_bar, (uint32_t)pend & 1u)) issue_down(pend);
          if (!mbar_wait(&ready_bar[s], (it / kStages) & 1, abort_flag)) { give_up_both(); dead = true; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * kS_Size);
          const uint32_t b_addr = a_addr + kS_B;
          if (j < lr) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mma_f16_pair(tbase, desc_k_sw128(a_addr + 32 * q), desc_k_sw128(b_addr + 32 * q), id_lr,
                           (j | q) != 0);
          } else {
            const uint32_t sfa_t = tbase + 256 + 48 * s;
            const uint32_t sfb_t = sfa_t + 16;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mma_nvf4_pair(tbase, desc_k_sw128(a_addr + 32 * q), desc_k_sw128(b_addr + 32 * q), id_f4,
                            sfa_t + 4 * q, sfb_t + 8 * q, (j | q) != 0);
          }
          mma_commit_pair(&empty_bar[s], 0x3);
        }
        if (!dead && pend >= 0 && !down_proj(pend)) dead = true;
        if (!dead) mma_commit_pair(&accf_bar, 0x3);
      }
      if (down && !dead && tcount > 0) down_proj(tcount - 1);
      if (*abort_flag) {
        mma_commit_pair(&accf_bar, 0x3);
        mbar_drain(&accf_bar, tcount & 1);
      }
    }
  } else if (warp < 8) {
    regs_dec<80>();
    // scale warps: landed stage -> this CTA's TMEM lane quarter of the stage's scale slot
    const int q = warp & 3;
    const uint32_t lane_base = tbase + ((uint32_t)(q * 32) << 16);
    int it = 0;
    bool dead = false;
    for (int item = pair; item < num_items && !dead; item += pairs) {
      const int lr = item_lr(item);
      for (int j = 0; j < lr + cpk; ++j, ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&landed_bar[s], (it / kStages) & 1, abort_flag)) { give_up_both(); dead = true; break; }
        if (j >= lr) {
          const uint8_t* st = smem + s * kS_Size;
          uint32_t wa[16], wb[32];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 x = *reinterpret_cast<const uint4*>(st + kS_SFA + 512 * k + lane * 16);
            wa[4 * k] = x.x; wa[4 * k + 1] = x.y; wa[4 * k + 2] = x.z; wa[4 * k + 3] = x.w;
            const uint4 y0 = *reinterpret_cast<const uint4*>(st + kS_SFB + 512 * k + lane * 16);
            const uint4 y1 = *reinterpret_cast<const uint4*>(st + kS_SFB + 2048 + 512 * k + lane * 16);
            wb[8 * k] = y0.x; wb[8 * k + 1] = y0.y; wb[8 * k + 2] = y0.z; wb[8 * k + 3] = y0.w;
            wb[8 * k + 4] = y1.x; wb[8 * k + 5] = y1.y; wb[8 * k + 6] = y1.z; wb[8 * k + 7] = y1.w;
          }
          tc_fence_after();
          tmem_st_16cols(lane_base + 256 + 48 * s, wa);
          tmem_st_32cols(lane_base + 256 + 48 * s + 16, wb);
          tmem_st_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&ready_bar[s]), 0));
      }
    }
  } else {
    regs_inc<184>();
    // epilogue warps 8..15 (both CTAs): TMEM -> registers, release TMEM,
    // then y = alpha * acc + bias -> bf16, written through a swizzled 4 KB
    // shared-memory chunk (32 rows x 64 columns) by TMA stores, so that
    // global writes are whole 128-byte row segments.
    const int q = warp & 3;
    const int h = (warp - 8) >> 2;
    const uint32_t taddr = tbase + ((uint32_t)(q * 32) << 16) + h * 128;
    const uint32_t acce_leader = mapa_shared(smem_u32(&acce_bar), 0);
    const float alpha = g.hdr->s_gx * g.hdr->s_gw;
    uint8_t* ybuf = ychunks + (warp - 8) * kEpiChunk;
    int tcount = 0;
    for (int item = pair; item < num_items; item += pairs, ++tcount) {
      const int tile = item / g.ks, kq = item % g.ks;
      const int mt = tile / n_tiles, nt = tile % n_tiles;
      const int col0 = nt * 256 + h * 128;
      float bl[4];   // bias of columns col0 + 32 j + lane
#pragma unroll
      for (int j = 0; j < 4; ++j) bl[j] = __ldg(g.bias + col0 + 32 * j + lane);
      if (CHAIN && g.nx_r > 0 && warp == 8 && lane == 0) {
        // this CTA's half of the next layer's L1^T rows, the tile's 256
        // columns (the buffer is free: the previous tile's down projection
        // completed before this warp read its result)
        const int rh = g.nx_r / 2;
        mbar_arrive_expect_tx(&l1_bar, (uint32_t)(256 * g.nx_r));
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tma_load_2d(l1buf + c * rh * 128, &tm_l1n, &l1_bar, nt * 256 + 64 * c, (int)rank * rh);
      }
      if (!mbar_wait(&accf_bar, tcount & 1, abort_flag)) { give_up_both(); break; }
      tc_fence_after();
      uint32_t v[128];
      tmem_ld_32cols(taddr + 0, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
      tmem_ld_32cols(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_ld_32cols(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
      tmem_ld_32cols(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_leader);
      const int64_t row0 = (int64_t)mt * 256 + 128 * rank + q * 32;
      if constexpr (CHAIN) {
        // The next layer's input, as its activation kernel would make it from
        // this layer's bf16 output y: x^ = fp32(y) * inv_lambda', one NVFP4
        // block per 16 columns (codes and E4M3 scale into the next layer's
        // activation tile (row tile, K slab nt)), and X^16 = bf16(x^) staged
        // for the partial down projection.  Rows past M quantise zeros.
        const int rl = q * 32 + lane;                     // row inside this CTA's 128
        const bool live = row0 + lane < g.M;
        const float s_gx = g.nx_hdr->s_gx;
        const float six_sg = __fmul_rn(6.0f, s_gx);
        const float r6 = recip_ok(six_sg) ? __frcp_rn(six_sg) : 0.0f;
        uint8_t* ntile = g.nx_atiles + ((size_t)(2 * mt + (int)rank) * (size_t)n_tiles + (size_t)nt) * kATile;
        const float4* il4 = reinterpret_cast<const float4*>(g.nx_inv_lambda + col0);
        uint32_t sc = 0, cw[4];
#pragma unroll
        for (int b = 0; b < 8; ++b) {                     // block b: columns 16 b .. 16 b + 15 of this half
          float xh[16];
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 il = __ldg(il4 + 4 * b + j4);
            const float ilv[4] = {il.x, il.y, il.z, il.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = 16 * b + 4 * j4 + j;
              const float bb = __shfl_sync(0xffffffffu, bl[e >> 5], e & 31);
              const float yv = __uint_as_float((uint32_t)bf16_rn(fmaf(alpha, __uint_as_float(v[e]), bb)) << 16);
              xh[4 * j4 + j] = live ? __fmul_rn(yv, ilv[j]) : 0.0f;
            }
          }
          const uint32_t e8 = nvfp4_scale_code(absmax16(xh), six_sg, r6);
          const float d = __fmul_rn(e4m3_val(e8), s_gx);
          const float rd = (d != 0.0f && recip_ok(d)) ? __frcp_rn(d) : 0.0f;
          nvfp4_codes16(xh, d, rd, cw[2 * (b & 1)], cw[2 * (b & 1) + 1]);
          sc |= e8 << (8 * (b & 3));
          if (b & 1)   // two blocks = one 16-byte chunk of the row's codes
            *reinterpret_cast<uint4*>(ntile + sw128((uint32_t)rl, (uint32_t)(16 * (4 * h + (b >> 1))))) =
                make_uint4(cw[0], cw[1], cw[2], cw[3]);
          if ((b & 3) == 3) {   // four scale bytes of one atom
            *reinterpret_cast<uint32_t*>(ntile + kTileCodes + (2 * h + (b >> 2)) * 512 + (rl & 31) * 16 +
                                         (rl >> 5) * 4) = sc;
            sc = 0;
          }
          if (g.nx_r > 0) {   // X^16 of the block: two 16-byte pieces of its 64-column tile
            uint32_t x16[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              x16[i] = (uint32_t)bf16_rn(xh[2 * i]) | ((uint32_t)bf16_rn(xh[2 * i + 1]) << 16);
            uint8_t* xt = xhat + (2 * h + (b >> 2)) * kLRTile + rl * 128;
            const int p0 = 2 * (b & 3);
            *reinterpret_cast<uint4*>(xt + ((p0 ^ (rl & 7)) << 4)) = make_uint4(x16[0], x16[1], x16[2], x16[3]);
            *reinterpret_cast<uint4*>(xt + (((p0 + 1) ^ (rl & 7)) << 4)) = make_uint4(x16[4], x16[5], x16[6], x16[7]);
          }
        }
        if (g.nx_r > 0) {
          // hand X^16 (and, from warp 8, the landed L1^T half) to the MMA
          // thread, then take this tile's partial down projection: lane
          // quarter q, columns [h r/2, (h + 1) r/2) of the next rank
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (warp == 8 && !mbar_wait(&l1_bar, tcount & 1, abort_flag)) give_up_both();
            mbar_arrive_cluster_release(mapa_shared(smem_u32(&xready_bar), 0));
          }
          __syncwarp();
          if (!mbar_wait(&ufull_bar, tcount & 1, abort_flag)) { give_up_both(); break; }
          tc_fence_after();
          const int rh = g.nx_r / 2;
          const uint32_t ua = tbase + ((uint32_t)(q * 32) << 16) + kC_UCol + (uint32_t)(h * rh);
          float* dst = g.nx_upart + ((size_t)nt * (size_t)g.Mp + (size_t)(row0 + lane)) * g.nx_r + h * rh;
          if (rh == 16) {
            uint32_t uv[16];
            tmem_ld_16cols(ua, uv);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c)
              reinterpret_cast<float4*>(dst)[c] =
                  make_float4(__uint_as_float(uv[4 * c]), __uint_as_float(uv[4 * c + 1]),
                              __uint_as_float(uv[4 * c + 2]), __uint_as_float(uv[4 * c + 3]));
          } else {
            uint32_t uv[8];
            tmem_ld_8cols(ua, uv);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 2; ++c)
              reinterpret_cast<float4*>(dst)[c] =
                  make_float4(__uint_as_float(uv[4 * c]), __uint_as_float(uv[4 * c + 1]),
                              __uint_as_float(uv[4 * c + 2]), __uint_as_float(uv[4 * c + 3]));
          }
          tc_fence_before();
        }
        continue;
      }
      if (g.ks > 1) {
        // K split: this item's raw sums -> part[kq]; the warp that completes a
        // region adds the ks partials in K order (deterministic), then applies
        // alpha and the bias.
        const int64_t m = row0 + lane;
        if (m < g.M) {
          float4* dst = reinterpret_cast<float4*>(g.part + ((size_t)kq * g.M + m) * g.N + col0);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            dst[c] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                                 __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
        }
        __threadfence();
        __syncwarp();
        int* cnt = g.cnt + (size_t)tile * 16 + rank * 8 + (warp - 8);
        int old = 0;
        if (lane == 0) old = atomicAdd(cnt, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == g.ks - 1) {
          __threadfence();
          // lane l reduces columns col0 + 4 l .. + 3 of every live row of the
          // region, four rows at a time so that their loads overlap
          const int64_t left = g.M - row0;
          const int live = left <= 0 ? 0 : (left >= 32 ? 32 : (int)left);
          const float4 b4 = __ldg(reinterpret_cast<const float4*>(g.bias + col0) + lane);
          for (int r0 = 0; r0 < live; r0 += 4) {
            float4 t[4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              t[rr] = make_float4(0.f, 0.f, 0.f, 0.f);
              if (r0 + rr < live)
                t[rr] = __ldcg(reinterpret_cast<const float4*>(g.part + (size_t)(row0 + r0 + rr) * g.N + col0) + lane);
            }
            for (int k = 1; k < g.ks; ++k) {
#pragma unroll
              for (int rr = 0; rr < 4; ++rr) {
                if (r0 + rr < live) {
                  const float4 w = __ldcg(reinterpret_cast<const float4*>(
                                              g.part + ((size_t)k * g.M + row0 + r0 + rr) * g.N + col0) + lane);
                  t[rr].x += w.x; t[rr].y += w.y; t[rr].z += w.z; t[rr].w += w.w;
                }
              }
            }
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              if (r0 + rr < live) {
                const uint32_t w0 = (uint32_t)bf16_rn(fmaf(alpha, t[rr].x, b4.x)) |
                                    ((uint32_t)bf16_rn(fmaf(alpha, t[rr].y, b4.y)) << 16);
                const uint32_t w1 = (uint32_t)bf16_rn(fmaf(alpha, t[rr].z, b4.z)) |
                                    ((uint32_t)bf16_rn(fmaf(alpha, t[rr].w, b4.w)) << 16);
                *reinterpret_cast<uint2*>(g.Y + (size_t)(row0 + r0 + rr) * g.N + col0 + 4 * lane) = make_uint2(w0, w1);
              }
            }
          }
          if (lane == 0) *cnt = 0;   // ready for the next call
        }
        continue;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint4 pk[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int e = 64 * k + 8 * c + 2 * j;
            const float b0 = __shfl_sync(0xffffffffu, bl[e >> 5], e & 31);
            const float b1 = __shfl_sync(0xffffffffu, bl[(e + 1) >> 5], (e + 1) & 31);
            const float y0 = fmaf(alpha, __uint_as_float(v[e]), b0);
            const float y1 = fmaf(alpha, __uint_as_float(v[e + 1]), b1);
            w[j] = (uint32_t)bf16_rn(y0) | ((uint32_t)bf16_rn(y1) << 16);
          }
          pk[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // the chunk buffer is free once the previous TMA store has read it
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(ybuf + lane * 128 + ((c ^ (lane & 7)) << 4)) = pk[c];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < g.M) {
          tma_store_2d(&tm_y, ybuf, col0 + 64 * k, (int)row0);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

// ------------------------------------------------------------ chained form: next low-rank input
// u'[m, i] = (sum over the output tile columns t, in order, of the chained
// GEMM's partial X^16 L1 [t][m][i]) / (s_gX s_gW) of the next layer, written
// as bf16 hi + lo into the next layer's low-rank input tiles in the format
// its activation kernel writes ([u'_hi | u'_lo | 0 pad], 128 x 64 swizzled
// tiles).  One thread per (token, 4 columns of the low-rank row).
constexpr int kCU_Threads = 256;
__global__ void __launch_bounds__(kCU_Threads) chain_u_kernel(const float* upart, int tiles, int64_t Mp, int r,
                                                              int lrw, const BlobHeader* nx_hdr, uint8_t* ux) {
  griddep_wait();   // the partials come from the chained GEMM
  const int per_row = lrw / 4;
  const int64_t idx = (int64_t)blockIdx.x * kCU_Threads + threadIdx.x;
  if (idx >= Mp * per_row) return;
  const int64_t m = idx / per_row;
  const int j = (int)(idx % per_row);
  const int c4 = r / 4;
  if (j >= c4 && j < 2 * c4) return;   // the lo half is written with its hi half
  uint8_t* const utile = ux + (size_t)(m / 128) * (size_t)(lrw / 64) * kLRTile;
  auto store4 = [&](int col, uint32_t w0, uint32_t w1) {   // 4 bf16 at columns col .. col + 3
    uint8_t* tile = utile + (size_t)(col / 64) * kLRTile;
    *reinterpret_cast<uint2*>(tile + sw128((uint32_t)(m % 128), (uint32_t)(col % 64) * 2)) = make_uint2(w0, w1);
  };
  if (j >= 2 * c4) {
    store4(4 * j, 0u, 0u);
    return;
  }
  const float4* src = reinterpret_cast<const float4*>(upart + (size_t)m * r) + j;
  const size_t tstride = (size_t)Mp * (size_t)r / 4;   // float4s per tile column
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  int t = 0;
  for (; t + 8 <= tiles; t += 8) {   // eight loads in flight, added in order
    float4 w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = __ldcg(src + (size_t)(t + i) * tstride);
#pragma unroll
    for (int i = 0; i < 8; ++i) { acc.x += w[i].x; acc.y += w[i].y; acc.z += w[i].z; acc.w += w[i].w; }
  }
  for (; t < tiles; ++t) {
    const float4 w = __ldcg(src + (size_t)t * tstride);
    acc.x += w.x; acc.y += w.y; acc.z += w.z; acc.w += w.w;
  }
  const float inv_alpha = 1.0f / (nx_hdr->s_gx * nx_hdr->s_gw);
  const float v[4] = {acc.x * inv_alpha, acc.y * inv_alpha, acc.z * inv_alpha, acc.w * inv_alpha};
  uint32_t hi[2], lo[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint32_t h0 = bf16_rn(v[2 * k]), h1 = bf16_rn(v[2 * k + 1]);
    const uint32_t l0 = bf16_rn(v[2 * k] - __uint_as_float(h0 << 16));
    const uint32_t l1 = bf16_rn(v[2 * k + 1] - __uint_as_float(h1 << 16));
    hi[k] = h0 | (h1 << 16);
    lo[k] = l0 | (l1 << 16);
  }
  store4(4 * j, hi[0], hi[1]);
  store4(r + 4 * j, lo[0], lo[1]);
}

// ------------------------------------------------------------ kernel 2, NVFP4, few tokens
// Up to 128 tokens: the layer streams its weights, so the weight tile is the
// 128-row A operand of a 1-CTA kind::mxf4nvf4 MMA and the tokens are a
// TOK-column B operand (M = 128 output features, N = TOK = 16, 64 or 128
// tokens, K = 64): D[feature, token] accumulates in TOK TMEM columns.  One CTA per (128-feature
// tile, K part); with ks > 1 K parts add through fp32 partials (the last CTA
// of a tile adds them in K order, as in the pair kernel).
// Per 256-wide K slab a ring stage holds the tile's codes (16 KB) and its
// 128 rows of scale atoms (2 KB), and the first TOK rows of the activation
// tile's codes (TOK x 128 bytes) and its scale atoms (2 KB): four bulk copies.  The
// weight halves of the first stages are issued before the wait for the
// activation kernel.  Four scale warps (one per TMEM lane quarter) move a
// landed stage's eight scale atoms to its TMEM slot with tcgen05.st and
// release it to the MMA thread, which then only issues the stage's four MMAs
// (with the scale copies on the MMA thread, the measured issue cost was
// ~0.5 us per stage, slower than the weight stream).  The low-rank up
// projection u' L2 runs last as kind::f16 K-steps (A = the L2 tile of the 128
// features, B = the first TOK rows of the low-rank input tile) into the same
// accumulator.
// Warps: 0 producer, 1 TMEM owner + MMA issuer, 2-5 scale warps, then the
// epilogue (lane quarters).
constexpr int kSM_MaxTokens = (int)kFewTokens;
constexpr int kSM_Threads = 6 * 32;
// stage: [W codes | W scales | X codes (TOK rows) | X scales]
SVDQ_HD constexpr int sm_stage(int tok) { return kTileCodes + 2048 + tok * 128 + 2048; }
SVDQ_HD constexpr int sm_stages(int tok) { return (232448 - 4096 - 1024) / sm_stage(tok) > 9 ? 9 : (232448 - 4096 - 1024) / sm_stage(tok); }
SVDQ_HD constexpr int sm_smem(int tok) { return sm_stages(tok) * sm_stage(tok) + 1024; }
constexpr int kSM_MaxStages = 9;

template <int TOK>
__global__ void __launch_bounds__(kSM_Threads, 1)
    gemm_nvfp4_small_kernel(const PairArgs g) {
  constexpr int kSM_Tokens = TOK;
  constexpr int kSM_Stage = sm_stage(TOK);
  constexpr int kSM_Stages = sm_stages(TOK);
  constexpr int kSM_WS = kTileCodes, kSM_X = kTileCodes + 2048, kSM_XS = kSM_X + TOK * 128;
  constexpr uint32_t kSF0 = TOK < 32 ? 32u : (uint32_t)TOK;   // scale slots after the accumulator's columns
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  __shared__ uint64_t full_bar[kSM_MaxStages], empty_bar[kSM_MaxStages], ready_bar[kSM_MaxStages], accf_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ks = g.ks;
  const int nt = blockIdx.x / ks, kq = blockIdx.x % ks;
  const int ksl = g.K / 256;
  const int cpk = g.k_iters / ks;                 // slabs of this CTA: [kq cpk, (kq + 1) cpk)
  const int lr = kq == 0 ? g.lr_iters : 0;        // the low-rank steps ride with K part 0
  const int steps = cpk + lr;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSM_Stages; ++s) {
      mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); mbar_init(&ready_bar[s], 4);
    }
    mbar_init(&accf_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base_sh, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      // step j < cpk: slab kq cpk + j; step j >= cpk: low-rank K step j - cpk
      auto weight_part = [&](int j, uint8_t* st) {
        if (j < cpk) {
          const uint8_t* wt = g.wtiles + ((size_t)nt * ksl + (size_t)(kq * cpk + j)) * kWTile;
          bulk_load(st, wt, kTileCodes, &full_bar[j % kSM_Stages]);
          bulk_load(st + kSM_WS, wt + kTileCodes + 2048 * (nt & 1), 2048, &full_bar[j % kSM_Stages]);
        } else {
          bulk_load(st, g.l2tiles + ((size_t)nt * g.lr_iters + (j - cpk)) * kLRTile, kLRTile,
                    &full_bar[j % kSM_Stages]);
        }
      };
      auto act_part = [&](int j, uint8_t* st) {
        if (j < cpk) {
          const uint8_t* at = g.atiles + (size_t)(kq * cpk + j) * kATile;   // tokens 0..127, slab
          bulk_load(st + kSM_X, at, kSM_Tokens * 128, &full_bar[j % kSM_Stages]);
          bulk_load(st + kSM_XS, at + kTileCodes, 2048, &full_bar[j % kSM_Stages]);
        } else {
          bulk_load(st + kSM_X, g.utiles + (size_t)(j - cpk) * kLRTile, kSM_Tokens * 128, &full_bar[j % kSM_Stages]);
        }
      };
      auto stage_bytes = [&](int j) -> uint32_t {
        return j < cpk ? (uint32_t)(kTileCodes + 2048 + kSM_Tokens * 128 + 2048) : (uint32_t)(kLRTile + kSM_Tokens * 128);
      };
      // the weights do not depend on the activation kernel: start them now,
      // the first stages into shared memory and the rest of this CTA's slabs
      // into L2
      const int first = steps < kSM_Stages ? steps : kSM_Stages;
      for (int j = 0; j < first; ++j) {
        mbar_arrive_expect_tx(&full_bar[j], stage_bytes(j));
        weight_part(j, smem + j * kSM_Stage);
      }
      for (int j = first; j < cpk; ++j)
        bulk_prefetch_l2(g.wtiles + ((size_t)nt * ksl + (size_t)(kq * cpk + j)) * kWTile, kWTile);
      griddep_wait();   // activation tiles and low-rank rows come from the activation kernel
      for (int j = 0; j < first; ++j) act_part(j, smem + j * kSM_Stage);
      int issued = first;
      for (int j = first; j < steps; ++j) {
        const int s = j % kSM_Stages;
        if (!mbar_wait(&empty_bar[s], ((j / kSM_Stages) & 1) ^ 1, abort_flag)) break;
        uint8_t* st = smem + s * kSM_Stage;
        mbar_arrive_expect_tx(&full_bar[s], stage_bytes(j));
        weight_part(j, st);
        act_part(j, st);
        issued = j + 1;
      }
      if (*abort_flag)
        for (int i = issued - 1; i >= 0 && i >= issued - kSM_Stages; --i)
          mbar_drain(&full_bar[i % kSM_Stages], (i / kSM_Stages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_f4 = idesc_nvf4(128, kSM_Tokens);
      const uint32_t id_lr = idesc_f16_bf16(128, kSM_Tokens);
      bool dead = false;
      for (int j = 0; j < steps; ++j) {
        const int s = j % kSM_Stages;
        // ready: the scale warps saw the stage land and wrote its scale slot
        if (!mbar_wait(&ready_bar[s], (j / kSM_Stages) & 1, abort_flag)) { dead = true; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * kSM_Stage);
        const uint32_t b_addr = a_addr + kSM_X;
        if (j < cpk) {
          const uint32_t sfa_t = tbase + kSF0 + 32 * s, sfb_t = sfa_t + 16;   // the stage's scale slot
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mma_nvf4(tbase, desc_k_sw128(a_addr + 32 * q), desc_k_sw128(b_addr + 32 * q), id_f4, sfa_t + 4 * q,
                     sfb_t + 4 * q, (j | q) != 0);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mma_f16(tbase, desc_k_sw128(a_addr + 32 * q), desc_k_sw128(b_addr + 32 * q), id_lr, (j | q) != 0);
        }
        mma_commit(&empty_bar[s]);
      }
      mma_commit(&accf_bar);
      if (dead) mbar_drain(&accf_bar, 0);
    }
  } else {
    const int q = warp & 3;
    // scale warps: a landed stage's scale atoms -> this lane quarter of its TMEM slot
    {
      const uint32_t lane_base = tbase + ((uint32_t)(q * 32) << 16);
      for (int j = 0; j < steps; ++j) {
        const int s = j % kSM_Stages;
        if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[s], (j / kSM_Stages) & 1, abort_flag))) break;
        if (j < cpk) {
          const uint8_t* st = smem + s * kSM_Stage;
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 a4 = *reinterpret_cast<const uint4*>(st + kSM_WS + 512 * k + lane * 16);
            w[4 * k] = a4.x; w[4 * k + 1] = a4.y; w[4 * k + 2] = a4.z; w[4 * k + 3] = a4.w;
          }
          tc_fence_after();
          tmem_st_16cols(lane_base + kSF0 + 32 * s, w);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 b4 = *reinterpret_cast<const uint4*>(st + kSM_XS + 512 * k + lane * 16);
            w[4 * k] = b4.x; w[4 * k + 1] = b4.y; w[4 * k + 2] = b4.z; w[4 * k + 3] = b4.w;
          }
          tmem_st_16cols(lane_base + kSF0 + 32 * s + 16, w);
          tmem_st_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ready_bar[s]);
      }
    }
    // epilogue: lane quarter q holds features 32 q + lane of the tile
    const int n = nt * 128 + q * 32 + lane;
    const float alpha = g.hdr->s_gx * g.hdr->s_gw;
    const float b = __ldg(g.bias + n);
    if (__all_sync(0xffffffffu, mbar_wait(&accf_bar, 0, abort_flag))) {
      tc_fence_after();
      const int M = (int)g.M;
      int* cnt = g.cnt + (size_t)nt * 4 + q;
      for (int m0 = 0; m0 < TOK && m0 < M; m0 += 16) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)m0));
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + j;
          if (m < M) {
            if (ks == 1) g.Y[(size_t)m * g.N + n] = bf16_rn(fmaf(alpha, __uint_as_float(v[j]), b));
            else __stcg(g.part + ((size_t)kq * g.M + m) * g.N + n, __uint_as_float(v[j]));
          }
        }
      }
      if (ks > 1) {
        // the warp completing its 32 features adds the K parts in order
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(cnt, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == ks - 1) {
          __threadfence();
          // eight tokens' ks loads in flight at once, each token's added in K order
#pragma unroll 8
          for (int m = 0; m < M; ++m) {
            float pk[kMaxKSplit];
#pragma unroll
            for (int k = 0; k < kMaxKSplit; ++k)
              pk[k] = k < ks ? __ldcg(g.part + ((size_t)k * g.M + m) * g.N + n) : 0.0f;
            float t = 0.0f;
#pragma unroll
            for (int k = 0; k < kMaxKSplit; ++k)
              if (k < ks) t += pk[k];
            g.Y[(size_t)m * g.N + n] = bf16_rn(fmaf(alpha, t, b));
          }
          if (lane == 0) *cnt = 0;   // ready for the next call
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------ kernel 2, INT4
// INT4 codes live as E4M3 bytes (exact for -8..7), so each group of 64 is two
// kind::f8f6f4 MMAs whose fp32 partial sum is an exact integer.  The per-group
// scales sx[m,g] sw[n,g] cannot enter the MMA, so every group's partial is
// drained from TMEM and folded on the CUDA cores, two columns per instruction
// (f32x2):  acc += (P_g * sw) * sx.
// Persistent, one CTA per SM over 128 x 128 output tiles (n fastest).
// TMEM: four 128-column partial buffers in a ring that runs across tile
// boundaries; the MMA issuer fills one while the fold warps drain the others.
// The hand-off (commit -> fold warps load -> release -> next MMA) has a round
// trip of about a microsecond whatever the work, so the time it bounds is
// (partial columns per SM / 512) x that round trip.  128-column partials keep
// that product while letting each fold warp hold a whole share (32 rows x 64
// columns) of a partial in registers after one load, so the buffer is
// released before any folding arithmetic.  The low-rank product u L2 is each
// tile's first partial (scale 1).
// The fold reads TMEM in the 16x256b shape: a thread holds 4 rows x 16
// columns instead of 1 row x 64, so it needs 16 column scales sw (not 64)
// from shared memory per partial.  Broadcasting sw to every lane was the
// kernel's bottleneck (shared-memory load wavefronts ~70 % busy) with the
// row-per-lane shape.
// Shared memory: a 6-deep ring of K slabs (128 bytes = two groups: A 16 KB,
// B 16 KB, by 2D TMA), a ring of the slabs' group scales (two 1 KB bulk
// copies from the blocked scale arrays), and one 2 KB output chunk per fold
// warp (32 rows x 32 bf16 columns, 64-byte swizzle) for TMA stores.
// Warps: 0 producer, 1 TMEM owner + MMA issuer, 2-3 idle [72 regs];
// 4-11 fold / epilogue, lane quarter warp % 4, column half (warp - 4) / 4 [216]
// (4 x 32 x 72 + 8 x 32 x 216 = the 384 x 168 registers of the launch).
constexpr int kI4BN = 128;                         // output features per tile
constexpr int kI4BBytes = kI4BN * 128;             // one 128-byte-wide K slab of B
constexpr int kI4Stages = 6;
constexpr int kI4Bufs = 4;                         // TMEM partial buffers of kI4BN columns
constexpr int kI4StageBytes = kABytes + kI4BBytes; // A/B ring: 2 groups per stage
constexpr int kI4ScaleSlot = 2 * kBM * 4 + 2 * kI4BN * 4;  // sx[2][128] + sw[2][128] fp32 = 2048
constexpr int kI4Epi = 8;
constexpr int kI4Threads = (4 + kI4Epi) * 32;
constexpr int kI4Chunk = 32 * 64;                  // 32 rows x 32 bf16 columns
constexpr int kI4Smem = kI4Stages * (kI4StageBytes + kI4ScaleSlot) + kI4Epi * kI4Chunk + 1024;
static_assert(kI4Bufs * kI4BN == 512, "the partial buffers fill TMEM");

__global__ void __launch_bounds__(kI4Threads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_ua, const __grid_constant__ CUtensorMap tm_ub,
                     const __grid_constant__ CUtensorMap tm_y, const GemmArgs g) {
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  __shared__ uint64_t full_bar[kI4Stages], empty_bar[kI4Stages], sfull_bar[kI4Stages], sempty_bar[kI4Stages];
  __shared__ uint64_t pfull_bar[kI4Bufs], pempty_bar[kI4Bufs], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sring = smem + kI4Stages * kI4StageBytes;   // scale slots
  uint8_t* ychunks = sring + kI4Stages * kI4ScaleSlot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = g.N / kI4BN;
  const int num_tiles = n_tiles * (int)(g.Mp / kBM);
  const int total = g.lr_iters + g.k_iters;   // ring steps per tile
  const int has_lr = g.lr_iters > 0;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kI4Stages; ++s) {
      mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1);
      mbar_init(&sfull_bar[s], 1); mbar_init(&sempty_bar[s], kI4Epi);
    }
    for (int b = 0; b < kI4Bufs; ++b) { mbar_init(&pfull_bar[b], 1); mbar_init(&pempty_bar[b], kI4Epi); }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a); prefetch_tmap(&tm_b); prefetch_tmap(&tm_y);
    if (has_lr) { prefetch_tmap(&tm_ua); prefetch_tmap(&tm_ub); }
  }
  if (warp == 1) { tmem_alloc(&tmem_base_sh, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_sh;

  if (warp < 4) {
    regs_dec<72>();
    if (warp == 0 && lane == 0) {
      griddep_wait();   // the workspace comes from the activation kernel
      int it = 0, issued = 0, sk = 0, sissued = 0;
      bool dead = false;
      for (int tile = blockIdx.x; tile < num_tiles && !dead; tile += gridDim.x) {
        const int mt = tile / n_tiles, nt = tile % n_tiles;
        const int n0 = nt * kI4BN;
        const int64_t m0 = (int64_t)mt * kBM;
        for (int j = 0; j < total; ++j, ++it) {
          const int s = it % kI4Stages;
          if (!mbar_wait(&empty_bar[s], ((it / kI4Stages) & 1) ^ 1, abort_flag)) { dead = true; break; }
          uint8_t* st = smem + s * kI4StageBytes;
          mbar_arrive_expect_tx(&full_bar[s], kABytes + kI4BBytes);
          if (j < g.lr_iters) {
            tma_load_2d(st, &tm_ua, &full_bar[s], j * 64, (int)m0);
            tma_load_2d(st + kABytes, &tm_ub, &full_bar[s], j * 64, n0);
          } else {
            const int kt = j - g.lr_iters;
            tma_load_2d(st, &tm_a, &full_bar[s], kt * 128, (int)m0);
            tma_load_2d(st + kABytes, &tm_b, &full_bar[s], kt * 128, n0);
            // the slab's two groups of scales (blocked layouts: one copy each)
            const int ss = sk % kI4Stages;
            if (!mbar_wait(&sempty_bar[ss], ((sk / kI4Stages) & 1) ^ 1, abort_flag)) { issued = it + 1; dead = true; break; }
            uint8_t* slot = sring + ss * kI4ScaleSlot;
            const float* sx = reinterpret_cast<const float*>(g.sfa) + ((size_t)kt * (size_t)(g.Mp / kBM) + mt) * 256;
            const float* sw = reinterpret_cast<const float*>(g.sfb) + ((size_t)kt * n_tiles + nt) * (2 * kI4BN);
            mbar_arrive_expect_tx(&sfull_bar[ss], kI4ScaleSlot);
            bulk_load(slot, sx, 2 * kBM * 4, &sfull_bar[ss]);
            bulk_load(slot + 2 * kBM * 4, sw, 2 * kI4BN * 4, &sfull_bar[ss]);
            ++sk;
            sissued = sk;
          }
          issued = it + 1;
        }
      }
      if (*abort_flag) {
        for (int i = issued - 1; i >= 0 && i >= issued - kI4Stages; --i)
          mbar_drain(&full_bar[i % kI4Stages], (i / kI4Stages) & 1);
        for (int i = sissued - 1; i >= 0 && i >= sissued - kI4Stages; --i)
          mbar_drain(&sfull_bar[i % kI4Stages], (i / kI4Stages) & 1);
      }
    } else if (warp == 1 && lane == 0) {
      const uint32_t id_lr = idesc_f16_bf16(kBM, kI4BN);
      const uint32_t id_f8 = idesc_f8_e4m3(kBM, kI4BN);
      int it = 0, seq = 0;   // seq: partial-buffer sequence over all tiles
      bool dead = false;
      for (int tile = blockIdx.x; tile < num_tiles && !dead; tile += gridDim.x) {
        for (int j = 0; j < total && !dead; ++j, ++it) {
          const int s = it % kI4Stages;
          if (!mbar_wait(&full_bar[s], (it / kI4Stages) & 1, abort_flag)) { dead = true; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * kI4StageBytes);
          const uint32_t b_addr = a_addr + kABytes;
          if (j < g.lr_iters) {
            const int buf = seq % kI4Bufs;
            if (j == 0) {
              if (!mbar_wait(&pempty_bar[buf], ((seq / kI4Bufs) & 1) ^ 1, abort_flag)) { dead = true; break; }
              tc_fence_after();
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mma_f16(tbase + kI4BN * buf, desc_k_sw128(a_addr + 32 * q), desc_k_sw128(b_addr + 32 * q), id_lr,
                      (j | q) != 0);
            if (j == g.lr_iters - 1) { mma_commit(&pfull_bar[buf]); ++seq; }
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int buf = seq % kI4Bufs;
              if (!mbar_wait(&pempty_bar[buf], ((seq / kI4Bufs) & 1) ^ 1, abort_flag)) { dead = true; break; }
              tc_fence_after();
              const uint32_t d = tbase + kI4BN * buf;
#pragma unroll
              for (int q = 0; q < 2; ++q)
                mma_f8(d, desc_k_sw128(a_addr + 64 * h + 32 * q), desc_k_sw128(b_addr + 64 * h + 32 * q), id_f8,
                       q != 0);
              mma_commit(&pfull_bar[buf]);
              ++seq;
            }
          }
          mma_commit(&empty_bar[s]);
        }
      }
      if (*abort_flag) {
        // wait for this thread's MMAs before TMEM is released
        mma_commit(&drain_bar);
        mbar_drain(&drain_bar, 0);
      }
    }
  } else {
    regs_inc<216>();
    // fold / epilogue warps 4..11
    const int e = warp - 4;
    const int q = warp & 3;                 // TMEM lane quarter
    const int ch = e >> 2;                  // column half of the tile
    const int t4 = lane >> 2;               // row within an 8-row group
    const int c2 = 2 * (lane & 3);          // column pair within an 8-column block
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    uint8_t* ybuf = ychunks + e * kI4Chunk;
    int seq = 0, sk = 0;
    bool ok = true;
    // acc[8 * s + k]: rows 32q + 8s + t4 (s = 0..3), columns 64ch + 8k + c2 + {0, 1}
    uint64_t acc[32];
    // drain partial buffer `buf` into acc: acc += (P * sw) * sx; the buffer is
    // released as soon as this warp's 32 x 64 share is in registers
    auto fold = [&](int buf, const float* swp, const float* sxp, bool plain) {
      uint32_t v[64];   // v[32 h + 4k + 2i + j]: row 16h + 8i + t4, column 8k + c2 + j
      tmem_ld_16x256b_x8(tbase + lane_addr + kI4BN * buf + ch * 64, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld_16x256b_x8(tbase + lane_addr + (16u << 16) + kI4BN * buf + ch * 64,
                         *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pempty_bar[buf]);
      if (plain) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int i = 0; i < 2; ++i)
              acc[8 * (2 * h + i) + k] =
                  f2_pack(__uint_as_float(v[32 * h + 4 * k + 2 * i]), __uint_as_float(v[32 * h + 4 * k + 2 * i + 1]));
      } else {
        uint64_t sx2[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float x = sxp[8 * r + t4];
          sx2[r] = f2_pack(x, x);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 w = *reinterpret_cast<const float2*>(swp + 8 * k + c2);
          const uint64_t w2 = f2_pack(w.x, w.y);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int rs = 2 * h + i;
              const uint64_t pp = f2_mul(
                  f2_pack(__uint_as_float(v[32 * h + 4 * k + 2 * i]), __uint_as_float(v[32 * h + 4 * k + 2 * i + 1])),
                  w2);
              acc[8 * rs + k] = f2_fma(pp, sx2[rs], acc[8 * rs + k]);
            }
        }
      }
    };
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int mt = tile / n_tiles, nt = tile % n_tiles;
      const int col0 = nt * kI4BN + ch * 64;
      const int64_t m0 = (int64_t)mt * kBM;
      if (has_lr) {
        const int buf = seq % kI4Bufs;
        if (!mbar_wait(&pfull_bar[buf], (seq / kI4Bufs) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        fold(buf, nullptr, nullptr, true);
        ++seq;
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0ull;
      }
      for (int kt = 0; kt < g.k_iters && ok; ++kt, ++sk) {
        const int ss = sk % kI4Stages;
        if (!mbar_wait(&sfull_bar[ss], (sk / kI4Stages) & 1, abort_flag)) { ok = false; break; }
        const float* slot = reinterpret_cast<const float*>(sring + ss * kI4ScaleSlot);
        for (int h = 0; h < 2; ++h) {
          const int buf = seq % kI4Bufs;
          if (!mbar_wait(&pfull_bar[buf], (seq / kI4Bufs) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          fold(buf, slot + 2 * kBM + h * kI4BN + ch * 64, slot + h * kBM + q * 32, false);
          ++seq;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty_bar[ss]);
      }
      if (!ok) break;
      // epilogue: y = acc + bias -> bf16, two 32-column chunks through shared
      // memory (64-byte rows, 16-byte unit u of row r stored at u ^ ((r >> 1) & 3))
      const int64_t row0 = m0 + q * 32;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float2 bl[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) bl[kk] = __ldg(reinterpret_cast<const float2*>(g.bias + col0 + 32 * c + 8 * kk + c2));
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int rs = 0; rs < 4; ++rs) {
          const int r = 8 * rs + t4;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            float y0, y1;
            f2_unpack(acc[8 * rs + 4 * c + kk], y0, y1);
            const uint32_t w = (uint32_t)bf16_rn(y0 + bl[kk].x) | ((uint32_t)bf16_rn(y1 + bl[kk].y) << 16);
            *reinterpret_cast<uint32_t*>(ybuf + r * 64 + ((kk ^ ((r >> 1) & 3)) << 4) + 2 * c2) = w;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < g.M) {
          tma_store_2d(&tm_y, ybuf, col0 + 32 * c, (int)row0);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA of this CTA has been consumed by the fold warps (or the CTA
    // gave up and drained); release TMEM
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------ probe (test hook)
__global__ void probe_cvt_kernel(const float* in, int64_t n, uint8_t* e2m1, uint8_t* e4m3) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float x = in[i];
    e2m1[i] = (uint8_t)(cvt_e2m1x2(0.0f, x) & 0xF);
    e4m3[i] = (uint8_t)(cvt_e4m3x2(0.0f, x) & 0xFF);
  }
}


// ------------------------------------------------------------ tensor-core rate probe
// Measures the issue-limited throughput of tcgen05 MMAs on this GPU: one
// thread per CTA issues `iters` MMAs back to back on zeroed shared memory,
// then waits (bounded) for their completion.  These are the tensor peaks the
// kernels are held against (dense FP4 / FP8 / INT8 / BF16 as this part runs
// them):
//   op 0  kind::mxf4nvf4 block16, M=128 N=256 K=64        (1 CTA)
//   op 1  kind::mxf4nvf4 block16, M=256 N=256 K=64        (CTA pair)
//   op 2  kind::f16 (bf16),      M=128 N=256 K=16
//   op 3  kind::f8f6f4 (E4M3),   M=128 N=256 K=32
//   op 4  kind::i8 (s8),         M=128 N=256 K=32
constexpr int kProbeSmem = 16384 + 32768 + 16384 + 1024;

template <bool kPair>
__device__ __forceinline__ void probe_body(int op, int iters, unsigned long long* cycles) {
  // every tcgen05 instruction of a kernel uses the same cta_group, so the
  // pair kernel only runs op 1 and the single-CTA kernel ops 0 and 2-4
  extern __shared__ __align__(1024) uint8_t psm_raw[];
  __shared__ uint64_t done_bar;
  __shared__ uint32_t tbase_sh;
  __shared__ int abort_sh;
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(psm_raw) + 1023) & ~uintptr_t(1023));
  for (int i = threadIdx.x; i < (kProbeSmem - 1024) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) { mbar_init(&done_bar, 1); abort_sh = 0; fence_mbar_init(); }
  if (warp == 0) {
    if constexpr (kPair) { tmem_alloc_pair(&tbase_sh, 512); tmem_relinquish_pair(); }
    else { tmem_alloc(&tbase_sh, 512); tmem_relinquish(); }
  }
  tc_fence_before();
  if constexpr (kPair) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t t = tbase_sh;
  bool issuer = threadIdx.x == 0;
  if constexpr (kPair) issuer = issuer && cluster_ctarank() == 0;
  if (issuer) {
    const uint32_t a = smem_u32(sm), b = a + 16384, sf = b + 32768;
    // zero the scale-factor columns [256, 352) from zeroed shared memory
    for (int q = 0; q < 24; ++q) {
      if constexpr (kPair) tmem_cp_32x128b_x4_pair(t + 256 + 4 * q, desc_sf_32x16(sf + 512 * (q & 15)));
      else tmem_cp_32x128b_x4(t + 256 + 4 * q, desc_sf_32x16(sf + 512 * (q & 15)));
    }
    const unsigned long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
      const uint32_t acc = i > 0;
      if constexpr (kPair) {
        mma_nvf4_pair(t, desc_k_sw128(a), desc_k_sw128(b), idesc_nvf4(256, 256), t + 256 + 4 * (i & 3),
                      t + 288 + 8 * (i & 3), acc);
      } else {
        switch (op) {
          case 0: mma_nvf4(t, desc_k_sw128(a), desc_k_sw128(b), idesc_nvf4(128, 256), t + 256, t + 288, acc); break;
          case 2: mma_f16(t, desc_k_sw128(a), desc_k_sw128(b), idesc_f16_bf16(128, 256), acc); break;
          case 3: mma_f8(t, desc_k_sw128(a), desc_k_sw128(b), idesc_f8_e4m3(128, 256), acc); break;
          case 4: mma_i8(t, desc_k_sw128(a), desc_k_sw128(b), idesc_i8(128, 256), acc); break;
          default: break;
        }
      }
    }
    if constexpr (kPair) mma_commit_pair(&done_bar, 0x3); else mma_commit(&done_bar);
    mbar_wait(&done_bar, 0, &abort_sh);
    cycles[blockIdx.x] = clock64() - t0;
  }
  if constexpr (kPair) {
    if (!issuer && threadIdx.x == 0) mbar_wait(&done_bar, 0, &abort_sh);
  }
  tc_fence_before();
  if constexpr (kPair) cluster_sync(); else __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(t, 512); else tmem_dealloc(t, 512);
  }
}

__global__ void __launch_bounds__(128, 1) tc_probe_kernel(int op, int iters, unsigned long long* cycles) {
  probe_body<false>(op, iters, cycles);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
    tc_probe_pair_kernel(int op, int iters, unsigned long long* cycles) {
  probe_body<true>(op, iters, cycles);
}

// Test hook: one thread waits, through the same bounded wait as the kernels,
// on an mbarrier that nothing arrives on; after limit_ns it gives up and
// records a timeout in the status word instead of hanging.
__global__ void probe_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_sh = 0;
    fence_mbar_init();
    (void)mbar_wait(&bar, 0, &abort_sh, limit_ns);
  }
}

// Test hook: the activation kernel's quotient (reciprocal + FMA correction)
// next to the IEEE division, on the same inputs.
__global__ void probe_div_kernel(const float* v, const float* d, int64_t n, float* q, float* q_ieee) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float dv = d[i];
    q[i] = recip_ok(dv) ? div_by_recip(v[i], dv, __frcp_rn(dv)) : __fdiv_rn(v[i], dv);
    q_ieee[i] = __fdiv_rn(v[i], dv);
  }
}

}  // namespace dev
}  // namespace svdq

// ======================================================================= host launchers
using namespace svdq;

extern "C" svdq_status svdq_decode_act_host(const svdq_params* p, const uint8_t* ws, int64_t M,
                                            uint8_t* codes, void* scales, float* u);

namespace {

thread_local char g_last_error[256] = "";

// Record a failed CUDA call for svdq_last_error_string and return SVDQ_ERR_CUDA.
svdq_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
  return SVDQ_ERR_CUDA;
}

svdq_status launch_status(const char* where) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SVDQ_OK : cuda_fail(e, where);
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device capability check and one-time kernel attributes.
struct DevState {
  bool checked = false, ok = false;
  int sms = 0;
};
std::mutex g_dev_mu;
DevState g_dev[64];

svdq_status device_ready() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SVDQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevState& d = g_dev[dev];
  if (!d.checked) {
    d.checked = true;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SVDQ_ERR_CUDA;
    d.ok = prop.major == 10 && prop.minor == 0;
    d.sms = prop.multiProcessorCount;
    if (d.ok) {
      const int i4_smem = dev::kI4Smem;
      d.ok = cudaFuncSetAttribute(dev::gemm_nvfp4_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dev::kP_Smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::gemm_nvfp4_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dev::kC_Smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::gemm_nvfp4_small_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dev::sm_smem(16)) == cudaSuccess &&
             cudaFuncSetAttribute(dev::gemm_nvfp4_small_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dev::sm_smem(64)) == cudaSuccess &&
             cudaFuncSetAttribute(dev::gemm_nvfp4_small_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dev::sm_smem(128)) == cudaSuccess &&
             cudaFuncSetAttribute(dev::gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  i4_smem) == cudaSuccess;
      const int act_smem = dev::kActSmemMax;
      d.ok = d.ok &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_NVFP4, SVDQ_BF16, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_NVFP4, SVDQ_F16, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_NVFP4, SVDQ_BF16, true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_NVFP4, SVDQ_F16, true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_INT4_G64, SVDQ_BF16, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_INT4_G64, SVDQ_F16, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_nvfp4_kernel<SVDQ_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dev::kAN_Budget) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_nvfp4_kernel<SVDQ_F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dev::kAN_Budget) == cudaSuccess;
      d.ok = d.ok && encoder();
    }
  }
  return d.ok ? SVDQ_OK : SVDQ_ERR_UNSUPPORTED;
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < 64 && g_dev[dev].sms > 0) ? g_dev[dev].sms : 148;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svdq_status check_params_dev(const svdq_params* p) {
  // same rules as the host half; the shape limits follow from the tile sizes
  if (!p) return SVDQ_ERR_INVALID_ARG;
  if (svdq_blob_bytes(p) == 0) {
    if (p->fmt != SVDQ_INT4_G64 && p->fmt != SVDQ_NVFP4) return SVDQ_ERR_UNSUPPORTED;
    if (p->act_dtype != SVDQ_F16 && p->act_dtype != SVDQ_BF16) return SVDQ_ERR_UNSUPPORTED;
    return SVDQ_ERR_INVALID_ARG;
  }
  return SVDQ_OK;
}

// K split of the activation kernel: with few 32-token groups, clusters of
// ks CTAs share a group's K range so that more SMs work (ks | K / 256, ks <= 8).
int act_k_split(int64_t Mp, int K) {
  const int64_t groups = Mp / dev::kActRows;
  const int chunks = K / dev::kActChunk;
  int ks = 1;
  while (ks < 8 && groups * ks * 2 <= num_sms() && chunks % (ks * 2) == 0) ks *= 2;
  return ks;
}

// Per-call tag of the activation kernel's K-split arrivals (56 bits, never 0),
// started from the clock so that another process's leftovers never match.
std::atomic<unsigned long long> g_act_epoch{
    ((unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull) >> 8};

template <int FMT>
cudaError_t launch_act(const svdq_params* p, dev::ActArgs a, int64_t Mp, cudaStream_t stream) {
  a.ks = act_k_split(Mp, p->K);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(dev::kActThreads);
  cfg.stream = stream;
  if constexpr (FMT == SVDQ_NVFP4) if (a.upart != nullptr) {
    // few live 32-token groups: only they run (rows past them are never read
    // for live tokens), ks > 8 CTAs each as clusters of 8; the clusters'
    // partials meet in the workspace
    a.ks = act_small_ks(a.M, p->K);
    a.epoch = g_act_epoch.fetch_add(1) & 0x00FFFFFFFFFFFFFFull;
    if (a.epoch == 0) a.epoch = g_act_epoch.fetch_add(1) & 0x00FFFFFFFFFFFFFFull;
    cfg.gridDim = dim3((unsigned)((a.M + dev::kActRows - 1) / dev::kActRows * a.ks));
    cfg.dynamicSmemBytes = (size_t)dev::act_smem_bytes(p->rank, p->K / a.ks);
    cudaLaunchAttribute cat[1];
    cat[0].id = cudaLaunchAttributeClusterDimension;
    cat[0].val.clusterDim.x = (unsigned)kActClusterKs;
    cat[0].val.clusterDim.y = 1;
    cat[0].val.clusterDim.z = 1;
    cfg.attrs = cat;
    cfg.numAttrs = 1;
    if (p->act_dtype == SVDQ_BF16) return cudaLaunchKernelEx(&cfg, dev::act_quant_kernel<FMT, SVDQ_BF16, true>, a);
    return cudaLaunchKernelEx(&cfg, dev::act_quant_kernel<FMT, SVDQ_F16, true>, a);
  }
  cfg.gridDim = dim3((unsigned)(Mp / dev::kActRows * a.ks));
  cfg.dynamicSmemBytes = (size_t)dev::act_smem_bytes(p->rank, p->K / a.ks);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)a.ks;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (p->act_dtype == SVDQ_BF16) return cudaLaunchKernelEx(&cfg, dev::act_quant_kernel<FMT, SVDQ_BF16, false>, a);
  return cudaLaunchKernelEx(&cfg, dev::act_quant_kernel<FMT, SVDQ_F16, false>, a);
}

}  // namespace

namespace {

svdq_status common_checks(const svdq_params* p, const void* blob_dev, int64_t M, const void* workspace,
                          size_t ws_bytes) {
  svdq_status st = check_params_dev(p);
  if (st != SVDQ_OK) return st;
  if (M < 0 || M > ((int64_t)1 << 30)) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!blob_dev || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(blob_dev) || !aligned16(workspace)) return SVDQ_ERR_ALIGNMENT;
  if (ws_bytes < ws_layout(*p, M).total) return SVDQ_ERR_WORKSPACE;
  return device_ready();
}

svdq_status launch_quantize(const svdq_params* p, const void* blob_dev, const void* X, int64_t M,
                            void* workspace, cudaStream_t stream) {
  const WsLayout W = ws_layout(*p, M);
  const BlobLayout B = blob_layout(*p);
  const uint8_t* blob = static_cast<const uint8_t*>(blob_dev);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  dev::ActArgs a;
  a.X = static_cast<const uint16_t*>(X);
  a.M = M; a.Mp = W.Mp; a.K = p->K; a.r = p->rank; a.lrw = lr_width(*p); a.nseg = nseg_of(*p);
  a.inv_lambda = reinterpret_cast<const float*>(blob + B.off_inv_lambda);
  a.l1t = reinterpret_cast<const uint16_t*>(blob + B.off_l1t);
  a.hdr = reinterpret_cast<const BlobHeader*>(blob);
  a.xq = ws + W.off_xq; a.xs = ws + W.off_xs;
  a.ux = reinterpret_cast<uint16_t*>(ws + W.off_ux);
  a.gemm_cnt = W.off_cnt > W.off_part ? reinterpret_cast<int*>(ws + W.off_cnt) : nullptr;
  a.n_cnt = (p->N / 256) * (int)(W.Mp / 256) * 16;
  // the 32-token kernel's workspace K split (NVFP4, few tokens; see ws_layout)
  const bool gsplit = p->fmt == SVDQ_NVFP4 && M <= 256 && W.off_ucnt > W.off_upart;
  a.upart = gsplit ? reinterpret_cast<float*>(ws + W.off_upart) : nullptr;
  a.ucnt = gsplit ? reinterpret_cast<unsigned long long*>(ws + W.off_ucnt) : nullptr;
  a.epoch = 0;
  // NVFP4 above 256 tokens: the 128-token-tile kernel (tcgen05 down projection).
  // Up to 256 tokens the 32-token kernel wins: its latency chain per call is
  // shorter (measured 12-22 us against 20-25 us at one token on the VAR shapes).
  if (p->fmt == SVDQ_NVFP4 && M > 256) {
    dev::ActNvArgs n;
    n.M = M; n.Mp = W.Mp; n.K = p->K; n.r = p->rank; n.lrw = lr_width(*p); n.nseg = nseg_of(*p);
    n.ks = act_nv_ks(W.Mp, p->K);
    n.slabs = p->K / 256 / n.ks;
    n.stages = dev::an_stages(p->rank);
    n.epoch = g_act_epoch.fetch_add(1) & 0x00FFFFFFFFFFFFFFull;
    if (n.epoch == 0) n.epoch = g_act_epoch.fetch_add(1) & 0x00FFFFFFFFFFFFFFull;
    n.inv_lambda = a.inv_lambda;
    n.hdr = a.hdr;
    n.xq = a.xq;
    n.ux = reinterpret_cast<uint8_t*>(a.ux);
    n.upart = reinterpret_cast<float*>(ws + W.off_upart);
    n.ucnt = reinterpret_cast<unsigned long long*>(ws + W.off_ucnt);
    n.gemm_cnt = a.gemm_cnt;
    n.n_cnt = a.n_cnt;
    const CUtensorMapDataType dt =
        p->act_dtype == SVDQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tm_x, tm_l1;
    bool ok = make_map(&tm_x, dt, X, (uint64_t)p->K, (uint64_t)M, (uint64_t)p->K * 2, 64, 128);
    if (p->rank > 0)
      ok = ok && make_map(&tm_l1, dt, a.l1t, (uint64_t)p->K, (uint64_t)p->rank, (uint64_t)p->K * 2, 64,
                          (uint32_t)p->rank);
    else
      tm_l1 = tm_x;   // not read at rank 0
    if (!ok) return cuda_fail(cudaErrorInvalidValue, "tensor map encode (activation kernel)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(W.Mp / 128 * n.ks));
    cfg.blockDim = dim3(dev::kAN_Threads);
    cfg.dynamicSmemBytes = (size_t)dev::an_smem_bytes(p->rank);
    cfg.stream = stream;
    const cudaError_t e = p->act_dtype == SVDQ_BF16
                              ? cudaLaunchKernelEx(&cfg, dev::act_nvfp4_kernel<SVDQ_BF16>, n, tm_x, tm_l1)
                              : cudaLaunchKernelEx(&cfg, dev::act_nvfp4_kernel<SVDQ_F16>, n, tm_x, tm_l1);
    if (e != cudaSuccess) return cuda_fail(e, "act_nvfp4_kernel launch");
    return launch_status("act_nvfp4_kernel launch");
  }
  const cudaError_t e = p->fmt == SVDQ_NVFP4 ? launch_act<SVDQ_NVFP4>(p, a, W.Mp, stream)
                                             : launch_act<SVDQ_INT4_G64>(p, a, W.Mp, stream);
  if (e != cudaSuccess) return cuda_fail(e, "act_quant_kernel launch");
  return launch_status("act_quant_kernel launch");
}

svdq_status launch_gemm(const svdq_params* p, const void* blob_dev, int64_t M, void* Y, void* workspace,
                        cudaStream_t stream) {
  const WsLayout W = ws_layout(*p, M);
  const BlobLayout B = blob_layout(*p);
  const uint8_t* blob = static_cast<const uint8_t*>(blob_dev);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int K = p->K, N = p->N, r = p->rank, lrw = lr_width(*p);
  const bool fp4 = p->fmt == SVDQ_NVFP4;
  if (fp4) {
    dev::PairArgs g{};
    g.M = M; g.Mp = W.Mp; g.N = N; g.K = K;
    g.lr_iters = r > 0 ? lrw / 64 : 0;
    g.k_iters = K / 256;
    g.atiles = ws + W.off_xq;
    g.wtiles = blob + B.off_wq;
    g.utiles = ws + W.off_ux;
    g.l2tiles = blob + B.off_l2x;
    g.bias = reinterpret_cast<const float*>(blob + B.off_bias);
    g.hdr = reinterpret_cast<const BlobHeader*>(blob);
    g.Y = static_cast<uint16_t*>(Y);
    CUtensorMap tm_y;
    if (!make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, (uint64_t)N, (uint64_t)M, (uint64_t)N * 2, 64, 32))
      return cuda_fail(cudaErrorInvalidValue, "tensor map encode (Y)");
    g.part = reinterpret_cast<float*>(ws + W.off_part);
    g.cnt = reinterpret_cast<int*>(ws + W.off_cnt);
    if (M <= dev::kSM_MaxTokens) {
      // up to 128 tokens: the weight tile as the A operand of a 1-CTA MMA, K
      // split over idle SMs when the workspace holds the partials
      const int n_tiles = N / 128;
      g.ks = 1;
      if (W.off_cnt > W.off_part)
        while (g.ks < kMaxKSplit && n_tiles * g.ks * 2 <= num_sms() && g.k_iters % (g.ks * 2) == 0 &&
               g.k_iters / (g.ks * 2) >= 2)
          g.ks *= 2;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(n_tiles * g.ks));
      cfg.blockDim = dim3(dev::kSM_Threads);
      cfg.stream = stream;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      at[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      cudaError_t e;
      if (M <= 16) {
        cfg.dynamicSmemBytes = dev::sm_smem(16);
        e = cudaLaunchKernelEx(&cfg, dev::gemm_nvfp4_small_kernel<16>, g);
      } else if (M <= 64) {
        cfg.dynamicSmemBytes = dev::sm_smem(64);
        e = cudaLaunchKernelEx(&cfg, dev::gemm_nvfp4_small_kernel<64>, g);
      } else {
        cfg.dynamicSmemBytes = dev::sm_smem(128);
        e = cudaLaunchKernelEx(&cfg, dev::gemm_nvfp4_small_kernel<128>, g);
      }
      if (e != cudaSuccess) return cuda_fail(e, "gemm_nvfp4_small_kernel launch");
      return launch_status("gemm_nvfp4_small_kernel launch");
    }
    const int tiles = (N / 256) * (int)(W.Mp / 256);
    g.ks = 1;
    if (W.off_cnt > W.off_part) {   // few tokens and tiles: split K over the idle pairs
      while (g.ks < kMaxKSplit && tiles * g.ks * 2 <= num_sms() / 2 && g.k_iters % (g.ks * 2) == 0 &&
             g.k_iters / (g.ks * 2) >= 2)
        g.ks *= 2;
    }
    const int pairs = std::max(1, std::min(tiles * g.ks, num_sms() / 2));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(dev::kP_Threads);
    cfg.dynamicSmemBytes = dev::kP_Smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, dev::gemm_nvfp4_pair_kernel<false>, g, tm_y, tm_y);
    if (e != cudaSuccess) return cuda_fail(e, "gemm_nvfp4_pair_kernel launch");
    return launch_status("gemm_nvfp4_pair_kernel launch");
  }
  CUtensorMap tm_a, tm_b, tm_ua, tm_ub, tm_y;
  const uint64_t krow = (uint64_t)K;
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + W.off_xq, krow, (uint64_t)M, krow, 128, dev::kBM) &&
            make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, blob + B.off_wq, krow, (uint64_t)N, krow, 128, dev::kI4BN) &&
            make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, (uint64_t)N, (uint64_t)M, (uint64_t)N * 2, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B);
  if (r > 0) {
    ok = ok && make_map(&tm_ua, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws + W.off_ux, (uint64_t)lrw, (uint64_t)M,
                        (uint64_t)lrw * 2, 64, dev::kBM) &&
         make_map(&tm_ub, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, blob + B.off_l2x, (uint64_t)lrw, (uint64_t)N,
                  (uint64_t)lrw * 2, 64, dev::kI4BN);
  } else {
    tm_ua = tm_a; tm_ub = tm_b;   // not read when rank is 0
  }
  if (!ok) return cuda_fail(cudaErrorInvalidValue, "tensor map encode");
  dev::GemmArgs g;
  g.M = M; g.N = N; g.K = K;
  g.lr_iters = r > 0 ? lrw / 64 : 0;
  g.k_iters = K / 128;
  g.sfa = ws + W.off_xs;
  g.sfb = blob + B.off_ws;
  g.bias = reinterpret_cast<const float*>(blob + B.off_bias);
  g.hdr = reinterpret_cast<const BlobHeader*>(blob);
  g.Y = static_cast<uint16_t*>(Y);
  g.Mp = W.Mp;
  const int tiles = (N / dev::kI4BN) * (int)(W.Mp / dev::kBM);
  const int grid = std::max(1, std::min(tiles, num_sms()));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(dev::kI4Threads);
  cfg.dynamicSmemBytes = dev::kI4Smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, dev::gemm_int4_kernel, tm_a, tm_b, tm_ua, tm_ub, tm_y, g);
  if (e != cudaSuccess) return cuda_fail(e, "gemm_int4_kernel launch");
  return launch_status("gemm kernel launch");
}

// This layer's GEMM writing the next layer's quantised input into ws_next
// (its activation tiles and low-rank input tiles) instead of Y.
svdq_status launch_gemm_chain(const svdq_params* p, const void* blob_dev, int64_t M, const svdq_params* pn,
                              const void* blob_next, void* workspace, void* ws_next, cudaStream_t stream) {
  const ChainLayout C = chain_layout(*p, *pn, M);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (M <= kFewTokens) {
    // a few tokens: Y is at most 128 rows, so it goes through the workspace
    // to the next layer's activation kernel
    void* y = ws + C.off_extra;
    const svdq_status st = launch_gemm(p, blob_dev, M, y, workspace, stream);
    if (st != SVDQ_OK) return st;
    return launch_quantize(pn, blob_next, y, M, ws_next, stream);
  }
  const WsLayout W = ws_layout(*p, M);
  const WsLayout Wn = ws_layout(*pn, M);
  const BlobLayout B = blob_layout(*p);
  const BlobLayout Bn = blob_layout(*pn);
  const uint8_t* blob = static_cast<const uint8_t*>(blob_dev);
  const uint8_t* nblob = static_cast<const uint8_t*>(blob_next);
  uint8_t* wsn = static_cast<uint8_t*>(ws_next);
  const int K = p->K, N = p->N, r = p->rank, lrw = lr_width(*p), rn = pn->rank;
  dev::PairArgs g{};
  g.M = M; g.Mp = W.Mp; g.N = N; g.K = K;
  g.lr_iters = r > 0 ? lrw / 64 : 0;
  g.k_iters = K / 256;
  g.atiles = ws + W.off_xq;
  g.wtiles = blob + B.off_wq;
  g.utiles = ws + W.off_ux;
  g.l2tiles = blob + B.off_l2x;
  g.bias = reinterpret_cast<const float*>(blob + B.off_bias);
  g.hdr = reinterpret_cast<const BlobHeader*>(blob);
  g.ks = 1;
  g.nx_inv_lambda = reinterpret_cast<const float*>(nblob + Bn.off_inv_lambda);
  g.nx_hdr = reinterpret_cast<const BlobHeader*>(nblob);
  g.nx_atiles = wsn + Wn.off_xq;
  g.nx_upart = reinterpret_cast<float*>(ws + C.off_extra);
  g.nx_r = rn;
  CUtensorMap tm_l1n{};
  if (rn > 0 && !make_map(&tm_l1n, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, nblob + Bn.off_l1t, (uint64_t)N, (uint64_t)rn,
                          (uint64_t)N * 2, 64, (uint32_t)(rn / 2)))
    return cuda_fail(cudaErrorInvalidValue, "tensor map encode (next layer L1)");
  const int tiles = (N / 256) * (int)(W.Mp / 256);
  const int pairs = std::max(1, std::min(tiles, num_sms() / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(dev::kP_Threads);
  cfg.dynamicSmemBytes = dev::kC_Smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, dev::gemm_nvfp4_pair_kernel<true>, g, tm_l1n, tm_l1n);
  if (e != cudaSuccess) return cuda_fail(e, "gemm_nvfp4_pair_kernel (chained) launch");
  if (rn > 0) {
    const int lrw_n = lr_width(*pn);
    const int64_t items = Wn.Mp * (lrw_n / 4);
    cfg.gridDim = dim3((unsigned)((items + dev::kCU_Threads - 1) / dev::kCU_Threads));
    cfg.blockDim = dim3(dev::kCU_Threads);
    cfg.dynamicSmemBytes = 0;
    e = cudaLaunchKernelEx(&cfg, dev::chain_u_kernel, (const float*)g.nx_upart, N / 256, (int64_t)Wn.Mp, rn, lrw_n,
                           g.nx_hdr, wsn + Wn.off_ux);
    if (e != cudaSuccess) return cuda_fail(e, "chain_u_kernel launch");
  }
  return launch_status("chained gemm launch");
}

}  // namespace

extern "C" {

svdq_status svdq_quantize_act(const svdq_params* p, const void* blob_dev, const void* X, int64_t M,
                              void* workspace, size_t ws_bytes, svdq_stream stream) {
  svdq_status st = common_checks(p, blob_dev, M, workspace, ws_bytes);
  if (st != SVDQ_OK || M == 0) return st;
  if (!X) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X)) return SVDQ_ERR_ALIGNMENT;
  return launch_quantize(p, blob_dev, X, M, workspace, reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_gemm(const svdq_params* p, const void* blob_dev, int64_t M, void* Y, void* workspace,
                      size_t ws_bytes, svdq_stream stream) {
  svdq_status st = common_checks(p, blob_dev, M, workspace, ws_bytes);
  if (st != SVDQ_OK || M == 0) return st;
  if (!Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(Y)) return SVDQ_ERR_ALIGNMENT;
  return launch_gemm(p, blob_dev, M, Y, workspace, reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_gemm_chain(const svdq_params* p, const void* blob_dev, int64_t M, const svdq_params* p_next,
                            const void* blob_next_dev, void* workspace, size_t ws_bytes, void* ws_next,
                            size_t ws_next_bytes, svdq_stream stream) {
  svdq_status st = check_params_dev(p_next);
  if (st != SVDQ_OK) return st;
  if ((st = chain_supported(*p, *p_next)) != SVDQ_OK) return st;
  st = common_checks(p, blob_dev, M, workspace, ws_bytes);
  if (st != SVDQ_OK || M == 0) return st;
  if (ws_bytes < chain_layout(*p, *p_next, M).total) return SVDQ_ERR_WORKSPACE;
  if (!blob_next_dev || !ws_next) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(blob_next_dev) || !aligned16(ws_next)) return SVDQ_ERR_ALIGNMENT;
  if (ws_next_bytes < ws_layout(*p_next, M).total) return SVDQ_ERR_WORKSPACE;
  return launch_gemm_chain(p, blob_dev, M, p_next, blob_next_dev, workspace, ws_next,
                           reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_linear(const svdq_params* p, const void* blob_dev, const void* X, int64_t M, void* Y,
                        void* workspace, size_t ws_bytes, svdq_stream stream_) {
  svdq_status st = common_checks(p, blob_dev, M, workspace, ws_bytes);
  if (st != SVDQ_OK || M == 0) return st;
  if (!X || !Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y)) return SVDQ_ERR_ALIGNMENT;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  st = launch_quantize(p, blob_dev, X, M, workspace, stream);
  if (st != SVDQ_OK) return st;
  return launch_gemm(p, blob_dev, M, Y, workspace, stream);
}

svdq_status svdq_export_act(const svdq_params* p, const void* workspace, int64_t M, uint8_t* codes,
                            void* scales, float* u, svdq_stream stream) {
  svdq_status st = check_params_dev(p);
  if (st != SVDQ_OK) return st;
  if (!workspace || M < 0) return SVDQ_ERR_INVALID_ARG;
  const WsLayout W = ws_layout(*p, M);
  std::vector<uint8_t> host(W.total);
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "svdq_export_act sync");
  e = cudaMemcpy(host.data(), workspace, W.total, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "svdq_export_act copy");
  return svdq_decode_act_host(p, host.data(), M, codes, scales, u);
}

svdq_status svdq_get_status(svdq_stream stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "svdq_get_status sync");
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, dev::g_status, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "svdq_get_status read");
  if (v != 0) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(dev::g_status, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_fail(e, "svdq_get_status clear");
    return (svdq_status)v;
  }
  return SVDQ_OK;
}

const char* svdq_last_error_string(void) { return g_last_error; }

svdq_status svdq_probe_cvt(const float* in, int64_t n, uint8_t* e2m1, uint8_t* e4m3, svdq_stream stream) {
  if (n < 0 || (n > 0 && (!in || !e2m1 || !e4m3))) return SVDQ_ERR_INVALID_ARG;
  if (n == 0) return SVDQ_OK;
  svdq_status st = device_ready();
  if (st != SVDQ_OK) return st;
  const int64_t blocks = (n + 255) / 256;
  dev::probe_cvt_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(in, n, e2m1, e4m3);
  return launch_status("probe_cvt launch");
}

svdq_status svdq_probe_tc(int op, int iters, int ctas, unsigned long long* cycles, svdq_stream stream) {
  if (op < 0 || op > 4 || iters <= 0 || iters > (1 << 24) || ctas <= 0 || ctas > 4096 || !cycles)
    return SVDQ_ERR_INVALID_ARG;
  svdq_status st = device_ready();
  if (st != SVDQ_OK) return st;
  cudaError_t e = cudaFuncSetAttribute(dev::tc_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev::kProbeSmem);
  if (e != cudaSuccess) return cuda_fail(e, "tc_probe_kernel attribute");
  e = cudaFuncSetAttribute(dev::tc_probe_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dev::kProbeSmem);
  if (e != cudaSuccess) return cuda_fail(e, "tc_probe_pair_kernel attribute");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (op == 1) dev::tc_probe_pair_kernel<<<(ctas + 1) / 2 * 2, 128, dev::kProbeSmem, s>>>(op, iters, cycles);
  else dev::tc_probe_kernel<<<ctas, 128, dev::kProbeSmem, s>>>(op, iters, cycles);
  return launch_status("tc_probe launch");
}

svdq_status svdq_probe_timeout(int64_t limit_ns, svdq_stream stream) {
  if (limit_ns <= 0 || limit_ns > 2000000000ll) return SVDQ_ERR_INVALID_ARG;
  svdq_status st = device_ready();
  if (st != SVDQ_OK) return st;
  dev::probe_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)limit_ns);
  return launch_status("probe_timeout launch");
}

svdq_status svdq_probe_div(const float* v, const float* d, int64_t n, float* q, float* q_ieee,
                           svdq_stream stream) {
  if (n < 0 || (n > 0 && (!v || !d || !q || !q_ieee))) return SVDQ_ERR_INVALID_ARG;
  if (n == 0) return SVDQ_OK;
  svdq_status st = device_ready();
  if (st != SVDQ_OK) return st;
  const int64_t blocks = (n + 255) / 256;
  dev::probe_div_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(v, d, n, q, q_ieee);
  return launch_status("probe_div launch");
}

}  // extern "C"

// ======================================================================= allocation-free entry point
// Some callers cannot allocate device memory where the layer runs (their
// allocator is out of reach there, or allocation is forbidden at that point),
// so this entry point takes its workspace from a buffer in the library's own
// static device memory instead of from the caller.  One buffer per device;
// overlapping calls on one device share it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SVDQ_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

// Device address of the static scratch on the current device, looked up once
// per device (with that device current) and cached.
svdq_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "svdq_linear_noalloc cudaGetDevice");
  if (dev < 0 || dev >= 64) {
    snprintf(g_last_error, sizeof(g_last_error), "svdq_linear_noalloc: device index %d outside 0..63", dev);
    return SVDQ_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* a = nullptr;
    e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "svdq_linear_noalloc cudaGetSymbolAddress");
    g_scratch_addr[dev] = a;
  }
  *out = g_scratch_addr[dev];
  return SVDQ_OK;
}

}  // namespace

extern "C" svdq_status svdq_linear_noalloc(const svdq_params* p, const void* blob_dev, const void* X, int64_t M,
                                           void* Y, svdq_stream stream) {
  svdq_status st = check_params_dev(p);
  if (st != SVDQ_OK) return st;
  if (M < 0 || M > ((int64_t)1 << 30)) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  const size_t need = ws_layout(*p, M).total;
  if (need > SVDQ_NOALLOC_SCRATCH_BYTES) {
    snprintf(g_last_error, sizeof(g_last_error),
             "svdq_linear_noalloc: workspace of %zu bytes exceeds the static scratch of %zu bytes", need,
             (size_t)SVDQ_NOALLOC_SCRATCH_BYTES);
    return SVDQ_ERR_WORKSPACE;
  }
  st = device_ready();
  if (st != SVDQ_OK) return st;
  void* ws = nullptr;
  st = noalloc_scratch(&ws);
  if (st != SVDQ_OK) return st;
  return svdq_linear(p, blob_dev, X, M, Y, ws, SVDQ_NOALLOC_SCRATCH_BYTES, stream);
}
