// Device half of libsvdq: the two kernels of svdq_linear and their launchers.
//
//   act_quant_kernel  (kernel 1)  reads X once: X^ = fp32(X) * inv_lambda,
//       per-token dynamic 4-bit quantisation (NVFP4 blocks of 16 / INT4 groups
//       of 64) and the low-rank down projection u = X^16 L1 on the tensor cores
//       ("AI图像生成4-bit量化技术解析与应用" 3.1: dynamic activation ranges;
//       "SVDQuant是什么？" 技术原理: 16-bit low-rank branch).
//   gemm_nvfp4_kernel / gemm_int4_kernel  (kernel 2)  the 4-bit GEMM
//       Q(X^) Q(R) on tcgen05 with TMEM accumulators, fed by TMA; the low-rank
//       up projection u L2 runs as extra bf16 K-steps into the same
//       accumulator and the epilogue adds the bias and writes bf16 Y
//       ("DeepCompressor…" SVDQuant section: the low-rank branch fused into
//       the low-bit kernel so it costs no extra activation traffic).
//
// Every wait on an mbarrier is bounded (about 1 s); a wait that gives up
// records SVDQ_ERR_TIMEOUT in a device status word and the CTA winds down.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <string.h>

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
};

constexpr int kActRows = 32;     // tokens per CTA
constexpr int kActChunk = 256;   // K elements per step
constexpr int kActStride = kActChunk + 8;  // padded smem row (bf16/fp16 elements)

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

// One CTA = 32 tokens x all of K, 8 warps.  Warp w owns tokens 4w..4w+3; lane
// l owns elements 8l..8l+7 of each 256-wide chunk (one 16-byte load per row).
template <int FMT, int DT>
__global__ void __launch_bounds__(256) act_quant_kernel(const ActArgs a) {
  extern __shared__ __align__(16) uint16_t act_smem[];
  uint16_t* xs16 = act_smem;                          // [32][kActStride]
  uint16_t* l1s = act_smem + kActRows * kActStride;   // [r][kActStride]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kActRows;
  const int K = a.K, r = a.r;
  const float s_gx = a.hdr->s_gx;
  const float six_sg = __fmul_rn(6.0f, s_gx);
  const float inv_alpha = FMT == SVDQ_NVFP4 ? 1.0f / (a.hdr->s_gx * a.hdr->s_gw) : 1.0f;

  // u tiles: (32/16) x (r/8) tiles of m16n8, spread over the 8 warps
  const int n_tiles = 2 * (r / 8);
  float acc[4][4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;

  for (int k0 = 0; k0 < K; k0 += kActChunk) {
    // stage this chunk of L1^T (r rows x 256) in shared memory
    for (int idx = tid; idx < r * (kActChunk / 8); idx += 256) {
      const int i = idx / (kActChunk / 8), c8 = idx % (kActChunk / 8);
      *reinterpret_cast<uint4*>(l1s + i * kActStride + c8 * 8) =
          __ldg(reinterpret_cast<const uint4*>(a.l1t + (size_t)i * K + k0 + c8 * 8));
    }
    const int kk = k0 + lane * 8;
    const float4 il0 = __ldg(reinterpret_cast<const float4*>(a.inv_lambda + kk));
    const float4 il1 = __ldg(reinterpret_cast<const float4*>(a.inv_lambda + kk + 4));
    const float il[8] = {il0.x, il0.y, il0.z, il0.w, il1.x, il1.y, il1.z, il1.w};

    uint4 xin[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t m = m0 + warp * 4 + j;
      xin[j] = m < a.M ? __ldg(reinterpret_cast<const uint4*>(a.X + m * K + kk)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int rw = warp * 4 + j;
      const int64_t m = m0 + rw;
      const uint16_t* xh16 = reinterpret_cast<const uint16_t*>(&xin[j]);
      float xh[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) xh[i] = __fmul_rn(half_to_f32<DT>(xh16[i]), il[i]);

      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(xh[i]));

      if constexpr (FMT == SVDQ_NVFP4) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));       // block of 16 = 2 lanes
        const float ratio = __fdiv_rn(amax, six_sg);
        const uint32_t e = cvt_e4m3x2(0.0f, ratio) & 0xFFu;
        const float d = __fmul_rn(e4m3_val(e), s_gx);
        uint32_t packed = 0;
        if (d != 0.0f) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            packed |= cvt_e2m1x2(__fdiv_rn(xh[2 * i + 1], d), __fdiv_rn(xh[2 * i], d)) << (8 * i);
        }
        if (m < a.M) *reinterpret_cast<uint32_t*>(a.xq + (size_t)m * (K / 2) + kk / 2) = packed;
        if ((lane & 1) == 0 && m < a.Mp) a.xs[sf_offset(m, kk / 16, K / 16)] = (uint8_t)e;
      } else {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));       // group of 64 = 8 lanes
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        const float s = __fdiv_rn(amax, 7.0f);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          int q0 = 0, q1 = 0;
          if (amax != 0.0f) {
            q0 = min(7, max(-8, __float2int_rn(__fdiv_rn(xh[2 * i], s))));
            q1 = min(7, max(-8, __float2int_rn(__fdiv_rn(xh[2 * i + 1], s))));
          }
          w[i] = cvt_e4m3x2((float)q1, (float)q0);
        }
        if (m < a.M)
          *reinterpret_cast<uint2*>(a.xq + (size_t)m * K + kk) =
              make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
        if ((lane & 7) == 0 && m < a.Mp)
          reinterpret_cast<float*>(a.xs)[(size_t)(kk / 64) * a.Mp + m] = s;
      }
      // X^ rounded to the 16-bit dtype: the low-rank branch's input
      uint4 o;
      uint16_t* o16 = reinterpret_cast<uint16_t*>(&o);
#pragma unroll
      for (int i = 0; i < 8; ++i) o16[i] = f32_to_half_rn<DT>(xh[i]);
      *reinterpret_cast<uint4*>(xs16 + rw * kActStride + lane * 8) = o;
    }
    __syncthreads();

    // u += X^16[32 x 256] * L1[256 x r]   (mma.sync m16n8k16, fp32 accumulate)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int tile = warp + 8 * t;
      if (tile < n_tiles) {
        const int mt = tile & 1, nt = tile >> 1;
        const uint32_t a_base =
            smem_u32(xs16 + (mt * 16 + (lane & 15)) * kActStride + (lane >> 4) * 8);
        const uint32_t b_base = smem_u32(l1s + (nt * 8 + (lane & 7)) * kActStride + ((lane >> 3) & 1) * 8);
#pragma unroll 4
        for (int ks = 0; ks < kActChunk / 16; ++ks) {
          uint32_t a0, a1, a2, a3, b0, b1;
          ldmatrix_x4(a_base + ks * 32, a0, a1, a2, a3);
          ldmatrix_x2(b_base + ks * 32, b0, b1);
          mma_16816<DT>(acc[t], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    __syncthreads();
  }

  // u' = u * inv_alpha, split into bf16 hi + lo: [hi | lo (| hi) | 0 pad]
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int tile = warp + 8 * t;
    if (tile < n_tiles) {
      const int mt = tile & 1, nt = tile >> 1;
      const int col = nt * 8 + 2 * (lane & 3);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int64_t m = m0 + mt * 16 + (lane >> 2) + half * 8;
        if (m < a.M) {
          uint16_t hi[2], lo[2];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const float v = acc[t][half * 2 + c] * inv_alpha;
            hi[c] = bf16_rn(v);
            lo[c] = bf16_rn(v - __uint_as_float((uint32_t)hi[c] << 16));
          }
          uint16_t* row = a.ux + (size_t)m * a.lrw;
          *reinterpret_cast<uint32_t*>(row + col) = hi[0] | ((uint32_t)hi[1] << 16);
          *reinterpret_cast<uint32_t*>(row + r + col) = lo[0] | ((uint32_t)lo[1] << 16);
          if (a.nseg == 3) *reinterpret_cast<uint32_t*>(row + 2 * r + col) = hi[0] | ((uint32_t)hi[1] << 16);
        }
      }
    }
  }
  const int used = a.nseg * r;
  const int pad = a.lrw - used;
  if (pad > 0) {
    for (int idx = tid; idx < kActRows * pad; idx += 256) {
      const int64_t m = m0 + idx / pad;
      if (m < a.M) a.ux[(size_t)m * a.lrw + used + idx % pad] = 0;
    }
  }
}

// ------------------------------------------------------------ kernel 2 (shared parts)
constexpr int kBM = 128;          // tokens per tile (TMEM lanes)
constexpr int kBN = 256;          // output features per tile (TMEM columns)
constexpr int kABytes = kBM * 128;   // one 128-byte-wide K slab of A
constexpr int kBBytes = kBN * 128;   // ... of B
constexpr int kStages = 4;

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

// ------------------------------------------------------------ kernel 2, NVFP4
// One CTA per 128 x 256 output tile.  Warp 0: TMA producer.  Warp 1: TMEM
// owner and MMA issuer.  Warps 2-5: epilogue (TMEM lane quarter = warp % 4).
// TMEM: columns [0,256) accumulator; [256,288) and [288,352) two buffers of
// activation / weight scale factors.
constexpr int kSfaBytes = 4 * 512;                 // 128 rows x 16 scale blocks
constexpr int kSfbBytes = 2 * 4 * 512;             // 256 rows x 16 scale blocks
constexpr int kFp4StageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;   // 55296

__global__ void __launch_bounds__(192, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_ua, const __grid_constant__ CUtensorMap tm_ub,
                      const GemmArgs g) {
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], accum_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = blockIdx.x, mt = blockIdx.y;
  const int n0 = nt * kBN;
  const int64_t m0 = (int64_t)mt * kBM;
  const int total = g.lr_iters + g.k_iters;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    mbar_init(&accum_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a); prefetch_tmap(&tm_b);
    if (g.lr_iters) { prefetch_tmap(&tm_ua); prefetch_tmap(&tm_ub); }
  }
  if (warp == 1) { tmem_alloc(&tmem_base_sh, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1, abort_flag)) break;
        uint8_t* st = smem + s * kFp4StageBytes;
        if (it < g.lr_iters) {
          mbar_arrive_expect_tx(&full_bar[s], kABytes + kBBytes);
          tma_load_2d(st, &tm_ua, &full_bar[s], it * 64, (int)m0);
          tma_load_2d(st + kABytes, &tm_ub, &full_bar[s], it * 64, n0);
        } else {
          const int kt = it - g.lr_iters;
          const int katoms = g.K / 64;
          mbar_arrive_expect_tx(&full_bar[s], kFp4StageBytes);
          tma_load_2d(st, &tm_a, &full_bar[s], kt * 128, (int)m0);
          tma_load_2d(st + kABytes, &tm_b, &full_bar[s], kt * 128, n0);
          uint8_t* sf = st + kABytes + kBBytes;
          bulk_load(sf, g.sfa + ((size_t)mt * katoms + kt * 4) * 512, kSfaBytes, &full_bar[s]);
          bulk_load(sf + kSfaBytes, g.sfb + ((size_t)(2 * nt) * katoms + kt * 4) * 512, 2048, &full_bar[s]);
          bulk_load(sf + kSfaBytes + 2048, g.sfb + ((size_t)(2 * nt + 1) * katoms + kt * 4) * 512, 2048,
                    &full_bar[s]);
        }
        issued = it + 1;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        for (int it = issued - 1; it >= 0 && it >= issued - kStages; --it)
          mbar_drain(&full_bar[it % kStages], (it / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_lr = idesc_f16_bf16(kBM, kBN);
      const uint32_t id_f4 = idesc_nvf4(kBM, kBN);
      for (int it = 0; it < total; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&full_bar[s], ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * kFp4StageBytes);
        const uint32_t b_addr = a_addr + kABytes;
        if (it < g.lr_iters) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_f16(tbase, desc_k_sw128(a_addr + 32 * j), desc_k_sw128(b_addr + 32 * j), id_lr,
                    (it | j) != 0);
        } else {
          const int kt = it - g.lr_iters;
          const uint32_t sfa_t = tbase + 256 + 16 * (kt & 1);
          const uint32_t sfb_t = tbase + 288 + 32 * (kt & 1);
          const uint32_t sf_addr = b_addr + kBBytes;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_cp_32x128b_x4(sfa_t + 4 * j, desc_sf_32x16(sf_addr + 512 * j));
            tmem_cp_32x128b_x4(sfb_t + 8 * j, desc_sf_32x16(sf_addr + kSfaBytes + 512 * j));
            tmem_cp_32x128b_x4(sfb_t + 8 * j + 4, desc_sf_32x16(sf_addr + kSfaBytes + 2048 + 512 * j));
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvf4(tbase, desc_k_sw128(a_addr + 32 * j), desc_k_sw128(b_addr + 32 * j), id_f4,
                     sfa_t + 4 * j, sfb_t + 8 * j, (it | j) != 0);
        }
        mma_commit(&empty_bar[s]);
      }
      mma_commit(&accum_bar);
      if (*abort_flag) mbar_drain(&accum_bar, 0);
    }
  } else {
    // epilogue: warps 2..5
    const int q = warp & 3;
    const bool ok = mbar_wait(&accum_bar, 0, abort_flag);
    tc_fence_after();
    if (ok) {
      const float alpha = g.hdr->s_gx * g.hdr->s_gw;
      const int64_t m = m0 + q * 32 + lane;
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32cols(tbase + ((uint32_t)(q * 32) << 16) + c * 32, v);
        tmem_ld_wait();
        if (m < g.M) {
          float bias[32], f[32];
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(g.bias + n0 + c * 32 + j));
            bias[j] = b4.x; bias[j + 1] = b4.y; bias[j + 2] = b4.z; bias[j + 3] = b4.w;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
          store_row32(g.Y + (size_t)m * g.N + n0 + c * 32, f, bias, alpha);
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
// drained from TMEM and folded on the CUDA cores:  acc += P_g * sx * sw.
// TMEM: two 256-column partial buffers (MMA writes one while the epilogue
// folds the other).  The low-rank product u L2 is sequence step 0 (scale 1).
// Warps: 0 TMA producer, 1 MMA issuer, 2-9 fold/epilogue (lane quarter
// warp % 4, column half (warp - 2) / 4).
constexpr int kI4StageBytes = kABytes + kBBytes;   // A/B ring: 2 groups per stage
constexpr int kI4ScaleSlot = 2 * kBM * 4 + 2 * kBN * 4;  // sx[2][128] + sw[2][256] fp32 = 3072
constexpr int kI4Epi = 8;

__global__ void __launch_bounds__(320, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_ua, const __grid_constant__ CUtensorMap tm_ub,
                     const GemmArgs g) {
  extern __shared__ __align__(1024) uint8_t gsmem_raw[];
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], sfull_bar[kStages], sempty_bar[kStages];
  __shared__ uint64_t pfull_bar[2], pempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sring = smem + kStages * kI4StageBytes;   // scale slots
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = blockIdx.x, mt = blockIdx.y;
  const int n0 = nt * kBN;
  const int64_t m0 = (int64_t)mt * kBM;
  const int total = g.lr_iters + g.k_iters;
  const int has_lr = g.lr_iters > 0;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1);
      mbar_init(&sfull_bar[s], 1); mbar_init(&sempty_bar[s], kI4Epi);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&pfull_bar[b], 1); mbar_init(&pempty_bar[b], kI4Epi); }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a); prefetch_tmap(&tm_b);
    if (has_lr) { prefetch_tmap(&tm_ua); prefetch_tmap(&tm_ub); }
  }
  if (warp == 1) { tmem_alloc(&tmem_base_sh, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0, sissued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1, abort_flag)) break;
        uint8_t* st = smem + s * kI4StageBytes;
        if (it < g.lr_iters) {
          mbar_arrive_expect_tx(&full_bar[s], kABytes + kBBytes);
          tma_load_2d(st, &tm_ua, &full_bar[s], it * 64, (int)m0);
          tma_load_2d(st + kABytes, &tm_ub, &full_bar[s], it * 64, n0);
        } else {
          const int kt = it - g.lr_iters;
          mbar_arrive_expect_tx(&full_bar[s], kABytes + kBBytes);
          tma_load_2d(st, &tm_a, &full_bar[s], kt * 128, (int)m0);
          tma_load_2d(st + kABytes, &tm_b, &full_bar[s], kt * 128, n0);
          // group scales of this slab go to the scale ring (read by the fold warps)
          const int ss = kt % kStages;
          if (!mbar_wait(&sempty_bar[ss], ((kt / kStages) & 1) ^ 1, abort_flag)) { issued = it + 1; break; }
          uint8_t* slot = sring + ss * kI4ScaleSlot;
          const float* sx = reinterpret_cast<const float*>(g.sfa);
          const float* sw = reinterpret_cast<const float*>(g.sfb);
          mbar_arrive_expect_tx(&sfull_bar[ss], kI4ScaleSlot);
          for (int h = 0; h < 2; ++h) {
            const int grp = 2 * kt + h;
            bulk_load(slot + h * kBM * 4, sx + (size_t)grp * g.Mp + m0, kBM * 4, &sfull_bar[ss]);
            bulk_load(slot + 2 * kBM * 4 + h * kBN * 4, sw + (size_t)grp * g.N + n0, kBN * 4, &sfull_bar[ss]);
          }
          sissued = kt + 1;
        }
        issued = it + 1;
      }
      if (*abort_flag) {
        for (int it = issued - 1; it >= 0 && it >= issued - kStages; --it)
          mbar_drain(&full_bar[it % kStages], (it / kStages) & 1);
        for (int kt = sissued - 1; kt >= 0 && kt >= sissued - kStages; --kt)
          mbar_drain(&sfull_bar[kt % kStages], (kt / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_lr = idesc_f16_bf16(kBM, kBN);
      const uint32_t id_f8 = idesc_f8_e4m3(kBM, kBN);
      int seq = 0;     // partial-buffer sequence: LR product (if any), then groups
      bool dead = false;
      for (int it = 0; it < total && !dead; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&full_bar[s], ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * kI4StageBytes);
        const uint32_t b_addr = a_addr + kABytes;
        if (it < g.lr_iters) {
          if (it == 0) {
            if (!mbar_wait(&pempty_bar[0], 1, abort_flag)) break;
            tc_fence_after();
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_f16(tbase, desc_k_sw128(a_addr + 32 * j), desc_k_sw128(b_addr + 32 * j), id_lr,
                    (it | j) != 0);
          if (it == g.lr_iters - 1) { mma_commit(&pfull_bar[0]); seq = 1; }
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int buf = seq & 1;
            if (!mbar_wait(&pempty_bar[buf], ((seq >> 1) & 1) ^ 1, abort_flag)) { dead = true; break; }
            tc_fence_after();
            const uint32_t d = tbase + 256 * buf;
#pragma unroll
            for (int j = 0; j < 2; ++j)
              mma_f8(d, desc_k_sw128(a_addr + 64 * h + 32 * j), desc_k_sw128(b_addr + 64 * h + 32 * j), id_f8,
                     j != 0);
            mma_commit(&pfull_bar[buf]);
            ++seq;
          }
        }
        mma_commit(&empty_bar[s]);
      }
      if (*abort_flag) {
        // wait for this thread's MMAs before TMEM is released
        mma_commit(&drain_bar);
        mbar_drain(&drain_bar, 0);
      }
    }
  } else {
    // fold / epilogue warps 2..9
    const int e = warp - 2;
    const int q = warp & 3;                 // TMEM lane quarter
    const int ch = e >> 2;                  // column half
    const int64_t m = m0 + q * 32 + lane;
    const int row_in_tile = q * 32 + lane;
    float acc[128];
#pragma unroll
    for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
    int seq = 0;
    bool ok = true;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    if (has_lr) {
      ok = mbar_wait(&pfull_bar[0], 0, abort_flag);
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld_32cols(tbase + lane_addr + ch * 128 + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[c * 32 + j] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pempty_bar[0]);
      seq = 1;
    }
    for (int kt = 0; kt < g.k_iters && ok; ++kt) {
      const int ss = kt % kStages;
      if (!mbar_wait(&sfull_bar[ss], (kt / kStages) & 1, abort_flag)) { ok = false; break; }
      const float* slot = reinterpret_cast<const float*>(sring + ss * kI4ScaleSlot);
      for (int h = 0; h < 2; ++h) {
        const int buf = seq & 1;
        if (!mbar_wait(&pfull_bar[buf], (seq >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const float sxm = slot[h * kBM + row_in_tile];
        const float* swp = slot + 2 * kBM + h * kBN + ch * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld_32cols(tbase + lane_addr + 256 * buf + ch * 128 + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            acc[c * 32 + j] = fmaf(__uint_as_float(v[j]), sxm * swp[c * 32 + j], acc[c * 32 + j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty_bar[buf]);
        ++seq;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty_bar[ss]);
    }
    if (ok && m < g.M) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float bias[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 b4 = __ldg(reinterpret_cast<const float4*>(g.bias + n0 + ch * 128 + c * 32 + j));
          bias[j] = b4.x; bias[j + 1] = b4.y; bias[j + 2] = b4.z; bias[j + 3] = b4.w;
        }
        store_row32(g.Y + (size_t)m * g.N + n0 + ch * 128 + c * 32, acc + c * 32, bias, 1.0f);
      }
    }
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

}  // namespace dev
}  // namespace svdq

// ======================================================================= host launchers
using namespace svdq;

extern "C" svdq_status svdq_decode_act_host(const svdq_params* p, const uint8_t* ws, int64_t M,
                                            uint8_t* codes, void* scales, float* u);

namespace {

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
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device capability check and one-time kernel attributes.
struct DevState {
  bool checked = false, ok = false;
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
    if (d.ok) {
      const int fp4_smem = dev::kStages * dev::kFp4StageBytes + 1024;
      const int i4_smem = dev::kStages * (dev::kI4StageBytes + dev::kI4ScaleSlot) + 1024;
      d.ok = cudaFuncSetAttribute(dev::gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  fp4_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  i4_smem) == cudaSuccess;
      const int act_smem = (dev::kActRows + 128) * dev::kActStride * 2;
      d.ok = d.ok &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_NVFP4, SVDQ_BF16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_NVFP4, SVDQ_F16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_INT4_G64, SVDQ_BF16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess &&
             cudaFuncSetAttribute(dev::act_quant_kernel<SVDQ_INT4_G64, SVDQ_F16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, act_smem) == cudaSuccess;
      d.ok = d.ok && encoder();
    }
  }
  return d.ok ? SVDQ_OK : SVDQ_ERR_UNSUPPORTED;
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

template <int FMT>
void launch_act(const svdq_params* p, const dev::ActArgs& a, int64_t Mp, cudaStream_t stream) {
  const dim3 grid((unsigned)(Mp / dev::kActRows));
  const size_t smem = (size_t)(dev::kActRows + p->rank) * dev::kActStride * 2;
  if (p->act_dtype == SVDQ_BF16) dev::act_quant_kernel<FMT, SVDQ_BF16><<<grid, 256, smem, stream>>>(a);
  else dev::act_quant_kernel<FMT, SVDQ_F16><<<grid, 256, smem, stream>>>(a);
}

}  // namespace

extern "C" {

svdq_status svdq_linear(const svdq_params* p, const void* blob_dev, const void* X, int64_t M, void* Y,
                        void* workspace, size_t ws_bytes, svdq_stream stream_) {
  svdq_status st = check_params_dev(p);
  if (st != SVDQ_OK) return st;
  if (M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!blob_dev || !X || !Y || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(blob_dev) || !aligned16(X) || !aligned16(Y) || !aligned16(workspace)) return SVDQ_ERR_ALIGNMENT;
  if (M > (int64_t)1 << 30) return SVDQ_ERR_INVALID_ARG;
  const WsLayout W = ws_layout(*p, M);
  if (ws_bytes < W.total) return SVDQ_ERR_WORKSPACE;
  st = device_ready();
  if (st != SVDQ_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

  const BlobLayout B = blob_layout(*p);
  const uint8_t* blob = static_cast<const uint8_t*>(blob_dev);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int K = p->K, N = p->N, r = p->rank, lrw = lr_width(*p);

  dev::ActArgs a;
  a.X = static_cast<const uint16_t*>(X);
  a.M = M; a.Mp = W.Mp; a.K = K; a.r = r; a.lrw = lrw; a.nseg = nseg_of(*p);
  a.inv_lambda = reinterpret_cast<const float*>(blob + B.off_inv_lambda);
  a.l1t = reinterpret_cast<const uint16_t*>(blob + B.off_l1t);
  a.hdr = reinterpret_cast<const BlobHeader*>(blob);
  a.xq = ws + W.off_xq; a.xs = ws + W.off_xs;
  a.ux = reinterpret_cast<uint16_t*>(ws + W.off_ux);
  if (p->fmt == SVDQ_NVFP4) launch_act<SVDQ_NVFP4>(p, a, W.Mp, stream);
  else launch_act<SVDQ_INT4_G64>(p, a, W.Mp, stream);
  if (cudaGetLastError() != cudaSuccess) return SVDQ_ERR_CUDA;

  CUtensorMap tm_a, tm_b, tm_ua, tm_ub;
  const bool fp4 = p->fmt == SVDQ_NVFP4;
  const uint64_t krow = fp4 ? (uint64_t)K / 2 : (uint64_t)K;
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, ws + W.off_xq, krow, (uint64_t)M, krow, 128, dev::kBM) &&
            make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, blob + B.off_wq, krow, (uint64_t)N, krow, 128, dev::kBN);
  if (r > 0) {
    ok = ok && make_map(&tm_ua, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws + W.off_ux, (uint64_t)lrw, (uint64_t)M,
                        (uint64_t)lrw * 2, 64, dev::kBM) &&
         make_map(&tm_ub, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, blob + B.off_l2x, (uint64_t)lrw, (uint64_t)N,
                  (uint64_t)lrw * 2, 64, dev::kBN);
  } else {
    tm_ua = tm_a; tm_ub = tm_b;   // unused
  }
  if (!ok) return SVDQ_ERR_CUDA;

  dev::GemmArgs g;
  g.M = M; g.N = N; g.K = K;
  g.lr_iters = r > 0 ? lrw / 64 : 0;
  g.k_iters = fp4 ? K / 256 : K / 128;
  g.sfa = ws + W.off_xs;
  g.sfb = blob + B.off_ws;
  g.bias = reinterpret_cast<const float*>(blob + B.off_bias);
  g.hdr = reinterpret_cast<const BlobHeader*>(blob);
  g.Y = static_cast<uint16_t*>(Y);
  g.Mp = W.Mp;
  const dim3 grid((unsigned)(N / dev::kBN), (unsigned)(W.Mp / dev::kBM));
  if (fp4) {
    dev::gemm_nvfp4_kernel<<<grid, 192, dev::kStages * dev::kFp4StageBytes + 1024, stream>>>(tm_a, tm_b, tm_ua,
                                                                                        tm_ub, g);
  } else {
    dev::gemm_int4_kernel<<<grid, 320, dev::kStages * (dev::kI4StageBytes + dev::kI4ScaleSlot) + 1024, stream>>>(
        tm_a, tm_b, tm_ua, tm_ub, g);
  }
  if (cudaGetLastError() != cudaSuccess) return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

svdq_status svdq_export_act(const svdq_params* p, const void* workspace, int64_t M, uint8_t* codes,
                            void* scales, float* u, svdq_stream stream) {
  svdq_status st = check_params_dev(p);
  if (st != SVDQ_OK) return st;
  if (!workspace || M < 0) return SVDQ_ERR_INVALID_ARG;
  const WsLayout W = ws_layout(*p, M);
  std::vector<uint8_t> host(W.total);
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (cudaMemcpy(host.data(), workspace, W.total, cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  return svdq_decode_act_host(p, host.data(), M, codes, scales, u);
}

svdq_status svdq_get_status(svdq_stream stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, dev::g_status, sizeof(v)) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (v != 0) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(dev::g_status, &z, sizeof(z)) != cudaSuccess) return SVDQ_ERR_CUDA;
    return (svdq_status)v;
  }
  return SVDQ_OK;
}

svdq_status svdq_probe_cvt(const float* in, int64_t n, uint8_t* e2m1, uint8_t* e4m3, svdq_stream stream) {
  if (n < 0 || (n > 0 && (!in || !e2m1 || !e4m3))) return SVDQ_ERR_INVALID_ARG;
  if (n == 0) return SVDQ_OK;
  svdq_status st = device_ready();
  if (st != SVDQ_OK) return st;
  const int64_t blocks = (n + 255) / 256;
  dev::probe_cvt_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(in, n, e2m1, e4m3);
  return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

}  // extern "C"
