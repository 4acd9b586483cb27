// Asymmetric per-channel INT8 KV-cache codec ("VAR-Compressor：在边缘GPU上实现
// 80亿参数视觉自回归模型的高效量化部署", INT8 KV缓存量化 and KV缓存特性研究: the
// cache's variance is driven by channels and its distribution is skewed, so it
// is stored as INT8 per channel with a non-centred zero point).
//
// A block of T cached tokens x C channels (row-major fp16 / bf16) gets one
// (scale, zero point) per channel from the channel's range over the block,
// widened to contain 0; all arithmetic in fp32, round to nearest even:
//   lo = min(0, min_t x), hi = max(0, max_t x), s = (hi - lo) / 255 (1 if 0),
//   z = clamp(rint(-lo / s), 0, 255), q = clamp(rint(x / s) + z, 0, 255),
//   decode: (q - z) * s rounded to the cache dtype.
//
// Encode is two HBM-bound kernels over 256-channel x 256-token tiles: the
// first writes each tile's per-channel min / max to the workspace, the second
// combines a channel's tile ranges (every tile of a column does the same
// arithmetic, so all agree), derives s and z, and writes the tile's codes.
// A lane owns 8 adjacent channels (16-byte loads, 8-byte code stores: 512 /
// 256 contiguous bytes per warp and token); the 8 warps of a CTA take every
// 8th token of the tile, 8 loads in flight each.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/svdq.h"

namespace svdq {
namespace kv {

constexpr int kTileC = 256;   // channels per CTA (32 lanes x 8)
constexpr int kTileT = 256;   // tokens per CTA
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

template <int DT>
__device__ __forceinline__ float to_f32(uint32_t h) {
  if constexpr (DT == SVDQ_BF16) return __uint_as_float(h << 16);
  else return __half2float(__ushort_as_half((unsigned short)h));
}

template <int DT>
__device__ __forceinline__ uint16_t from_f32(float f) {
  if constexpr (DT == SVDQ_BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(f));
  else return __half_as_ushort(__float2half_rn(f));
}

template <int DT>
__device__ __forceinline__ void unpack8(const uint4& w, float (&v)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = to_f32<DT>(u[i] & 0xFFFFu);
    v[2 * i + 1] = to_f32<DT>(u[i] >> 16);
  }
}

// part: [2][n_tiles_t][C] fp32, minima then maxima of each token tile
template <int DT>
__global__ void __launch_bounds__(kThreads) kv_range_kernel(const uint16_t* __restrict__ X, int64_t T, int C,
                                                            float* __restrict__ part) {
  __shared__ float red[2][kWarps][kTileC];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * kTileC + 8 * lane;
  const int64_t t0 = (int64_t)blockIdx.y * kTileT;
  const int64_t t1 = t0 + kTileT < T ? t0 + kTileT : T;
  float lo[8], hi[8];   // ranges widened to contain 0
#pragma unroll
  for (int i = 0; i < 8; ++i) lo[i] = hi[i] = 0.0f;
#pragma unroll 8
  for (int64_t t = t0 + warp; t < t1; t += kWarps) {
    float v[8];
    unpack8<DT>(__ldg(reinterpret_cast<const uint4*>(X + t * C + c)), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) { lo[i] = fminf(lo[i], v[i]); hi[i] = fmaxf(hi[i], v[i]); }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) { red[0][warp][8 * lane + i] = lo[i]; red[1][warp][8 * lane + i] = hi[i]; }
  __syncthreads();
  const int cc = threadIdx.x;   // one channel of the tile per thread
  float l = 0.0f, h = 0.0f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) { l = fminf(l, red[0][w][cc]); h = fmaxf(h, red[1][w][cc]); }
  const size_t nt = gridDim.y;
  part[(size_t)blockIdx.y * C + blockIdx.x * kTileC + cc] = l;
  part[(nt + blockIdx.y) * (size_t)C + blockIdx.x * kTileC + cc] = h;
}

__device__ __forceinline__ void channel_params(float lo, float hi, float& s, int& z) {
  s = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
  if (s == 0.0f) s = 1.0f;
  const float zf = rintf(__fdiv_rn(-lo, s));
  z = (int)fminf(fmaxf(zf, 0.0f), 255.0f);
}

// x / s rounded to nearest as IEEE division gives it, from rs = RN(1 / s):
// q = RN(x rs) is within an ulp, e = x - q s is exact (one FMA) and RN(q + e rs)
// is the correctly rounded quotient (Markstein; Muller et al., Handbook of
// Floating-Point Arithmetic, FMA-based division), valid while nothing over- or
// underflows: rs is 0 (use the division) outside 2^-100 <= s <= 2^125.  Codes
// of tiny quotients are 0 or z either way.
__device__ __forceinline__ float quot(float x, float s, float rs) {
  if (rs == 0.0f) return __fdiv_rn(x, s);
  const float q = __fmul_rn(x, rs);
  const float e = __fmaf_rn(-q, s, x);
  return __fmaf_rn(e, rs, q);
}

__device__ __forceinline__ uint32_t code(float x, float s, float rs, int z) {
  const int q = __float2int_rn(quot(x, s, rs)) + z;
  return (uint32_t)(q < 0 ? 0 : (q > 255 ? 255 : q));
}

template <int DT>
__global__ void __launch_bounds__(kThreads) kv_quant_kernel(const uint16_t* __restrict__ X, int64_t T, int C,
                                                            const float* __restrict__ part, uint8_t* __restrict__ q,
                                                            float* __restrict__ scale, uint8_t* __restrict__ zero) {
  __shared__ float s_sc[kTileC];
  __shared__ int s_z[kTileC];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    // one channel per thread: combine the tile ranges of its column
    const int cc = blockIdx.x * kTileC + threadIdx.x;
    const size_t nt = gridDim.y;
    float l = 0.0f, h = 0.0f;
    for (size_t i = 0; i < nt; ++i) {
      l = fminf(l, __ldcg(part + i * C + cc));
      h = fmaxf(h, __ldcg(part + (nt + i) * C + cc));
    }
    float sc;
    int z;
    channel_params(l, h, sc, z);
    s_sc[threadIdx.x] = sc;
    s_z[threadIdx.x] = z;
    if (blockIdx.y == 0) {
      scale[cc] = sc;
      zero[cc] = (uint8_t)z;
    }
  }
  __syncthreads();
  float sc[8], rs[8];
  int z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sc[i] = s_sc[8 * lane + i];
    z[i] = s_z[8 * lane + i];
    rs[i] = (sc[i] >= 0x1p-100f && sc[i] <= 0x1p+125f) ? __frcp_rn(sc[i]) : 0.0f;
  }
  const int c = blockIdx.x * kTileC + 8 * lane;
  const int64_t t0 = (int64_t)blockIdx.y * kTileT;
  const int64_t t1 = t0 + kTileT < T ? t0 + kTileT : T;
#pragma unroll 8
  for (int64_t t = t0 + warp; t < t1; t += kWarps) {
    float v[8];
    unpack8<DT>(__ldg(reinterpret_cast<const uint4*>(X + t * C + c)), v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i >> 2] |= code(v[i], sc[i], rs[i], z[i]) << (8 * (i & 3));
    *reinterpret_cast<uint2*>(q + t * C + c) = make_uint2(w[0], w[1]);
  }
}

// Each thread decodes 8 consecutive channels of one token (8-byte code load,
// 16-byte store).
template <int DT>
__global__ void __launch_bounds__(256) kv_decode_kernel(const uint8_t* __restrict__ q, const float* __restrict__ scale,
                                                        const uint8_t* __restrict__ zero, int64_t T, int C,
                                                        uint16_t* __restrict__ Y) {
  const int64_t n8 = T * (int64_t)(C / 8);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / (C / 8);
    const int c = (int)(i % (C / 8)) * 8;
    const uint2 qq = __ldg(reinterpret_cast<const uint2*>(q + t * C + c));
    const uint2 zz = __ldg(reinterpret_cast<const uint2*>(zero + c));
    const float4 sa = __ldg(reinterpret_cast<const float4*>(scale + c));
    const float4 sb = __ldg(reinterpret_cast<const float4*>(scale + c + 4));
    const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const uint32_t qw = j < 4 ? qq.x : qq.y, zw = j < 4 ? zz.x : zz.y;
      const int sh = 8 * (j & 3);
      const int d0 = (int)((qw >> sh) & 0xFFu) - (int)((zw >> sh) & 0xFFu);
      const int d1 = (int)((qw >> (sh + 8)) & 0xFFu) - (int)((zw >> (sh + 8)) & 0xFFu);
      out[j / 2] = (uint32_t)from_f32<DT>(__fmul_rn((float)d0, sv[j])) |
                   ((uint32_t)from_f32<DT>(__fmul_rn((float)d1, sv[j + 1])) << 16);
    }
    *reinterpret_cast<uint4*>(Y + t * C + c) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}


// ------------------------------------------------------------ attention reads
// Scaled dot-product attention of a few query rows against an INT8 cache,
// read straight from the codes (split over 256-token chunks, then combined):
//   S[i,t] = sum_c Q[i,c] K^[t,c] / sqrt(d),  K^[t,c] = (kq[t,c] - kz[c]) ks[c]
//          = (sum_c (Q[i,c] ks[c]) kq[t,c] - sum_c Q[i,c] ks[c] kz[c]) / sqrt(d),
//   O[i,c] = sum_t P[i,t] V^[t,c] = vs[c] (sum_t P[i,t] vq[t,c] - vz[c] sum_t P[i,t]).
// kv_attn_partial: one CTA per (head, chunk); the chunk's key and value rows
// of the head are staged in shared memory once; each thread scores one token
// for every query; per query the chunk's max m, sum l of exp(S - m) and the
// unnormalised o[c] = sum_t exp(S - m) vq[t,c] go to the workspace.
// kv_attn_combine: per (head, query), the chunks in order: M = max m_k,
// L = sum exp(m_k - M) l_k, O = sum exp(m_k - M) o_k, out = vs (O / L - vz).
constexpr int kAttnChunk = 256;
constexpr int kAttnMaxQ = 16;
constexpr int attn_smem_bytes(int D, int QB) {
  return kAttnChunk * (D + 16) + kAttnChunk * D + QB * D * 4 + QB * kAttnChunk * 4 + QB * 8 * 4 + QB * 4;
}

__device__ __forceinline__ void codes16(const uint4 w, float (&f)[16]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int b = 0; b < 4; ++b) f[4 * i + b] = (float)((u[i] >> (8 * b)) & 0xFFu);
}

// QB: query bucket (1, 4 or 16) >= Mq; loops over queries run QB times
template <int DT, int D, int QB>
__global__ void __launch_bounds__(256) kv_attn_partial(const uint16_t* __restrict__ Q, int Mq,
                                                       const uint8_t* __restrict__ kq, const float* __restrict__ ks,
                                                       const uint8_t* __restrict__ kz, const uint8_t* __restrict__ vq,
                                                       int64_t T, int C, float* __restrict__ part) {
  constexpr int KS = D + 16;                      // padded key row (bank-conflict free 16-byte reads)
  extern __shared__ __align__(16) uint8_t attn_smem[];
  uint8_t* kc = attn_smem;                                                      // [chunk][KS]
  uint8_t* vc = kc + kAttnChunk * KS;                                           // [chunk][D]
  float (*qp)[D] = reinterpret_cast<float (*)[D]>(vc + kAttnChunk * D);        // [MaxQ][D]
  float (*pr)[kAttnChunk] = reinterpret_cast<float (*)[kAttnChunk]>(&qp[QB][0]);
  float (*red)[8] = reinterpret_cast<float (*)[8]>(&pr[QB][0]);
  float* bk = &red[QB][0];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid: heads fastest, so that the CTAs running together read whole cache rows
  const int h = blockIdx.x;
  const int64_t t0 = (int64_t)blockIdx.y * kAttnChunk;
  const int nt = (int)(T - t0 < kAttnChunk ? T - t0 : kAttnChunk);
  const int c0 = h * D;
  // stage the chunk's rows of this head (rows past T as zero codes): every
  // load of the thread in flight before the first store
  constexpr int kPer = kAttnChunk * (D / 16) / 256;   // 16-byte pieces per thread and operand
  uint4 ka[kPer], va[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int e = tid + 256 * r, t = e / (D / 16), j = e % (D / 16);
    ka[r] = va[r] = make_uint4(0, 0, 0, 0);
    if (t < nt) {
      ka[r] = __ldg(reinterpret_cast<const uint4*>(kq + (t0 + t) * C + c0) + j);
      va[r] = __ldg(reinterpret_cast<const uint4*>(vq + (t0 + t) * C + c0) + j);
    }
  }
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int e = tid + 256 * r, t = e / (D / 16), j = e % (D / 16);
    *reinterpret_cast<uint4*>(kc + t * KS + 16 * j) = ka[r];
    *reinterpret_cast<uint4*>(vc + t * D + 16 * j) = va[r];
  }
  // queries times the key scales, and their dot with the key zero points
  for (int e = tid; e < Mq * D; e += 256) {
    const int i = e / D, c = e % D;
    const uint32_t hq = Q[(size_t)i * C + c0 + c];
    const float q = DT == SVDQ_BF16 ? __uint_as_float(hq << 16) : __half2float(__ushort_as_half((unsigned short)hq));
    qp[i][c] = __fmul_rn(q, __ldg(ks + c0 + c));
  }
  __syncthreads();
  for (int i = warp; i < Mq; i += 8) {
    float acc = 0.0f;
    for (int c = lane; c < D; c += 32) acc = fmaf(qp[i][c], (float)kz[c0 + c], acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) bk[i] = acc;
  }
  __syncthreads();
  // scores: thread = token of the chunk, all queries
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  float sc[QB];
#pragma unroll
  for (int i = 0; i < QB; ++i) sc[i] = 0.0f;
  for (int j = 0; j < D / 16; ++j) {
    float f[16];
    codes16(*reinterpret_cast<const uint4*>(kc + tid * KS + 16 * j), f);
#pragma unroll
    for (int i = 0; i < QB; ++i) {
      if (i < Mq) {
        const float4* qv = reinterpret_cast<const float4*>(&qp[i][16 * j]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 w = qv[k];
          sc[i] = fmaf(w.x, f[4 * k], sc[i]);
          sc[i] = fmaf(w.y, f[4 * k + 1], sc[i]);
          sc[i] = fmaf(w.z, f[4 * k + 2], sc[i]);
          sc[i] = fmaf(w.w, f[4 * k + 3], sc[i]);
        }
      }
    }
  }
  const bool live = tid < nt;
  // per query: chunk max, exp, chunk sum (warp shuffle trees, then the 8 warps in order)
  // (every loop over the queries is unrolled to QB with a guard, so
  // that the per-query values stay in registers)
#pragma unroll
  for (int i = 0; i < QB; ++i) {
    if (i < Mq) {
      const float s = live ? (sc[i] - bk[i]) * inv_sqrt_d : -INFINITY;
      float m = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (lane == 0) red[i][warp] = m;
      sc[i] = s;
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < QB; ++i) {
    if (i < Mq) {
      float m = red[i][0];
#pragma unroll
      for (int w = 1; w < 8; ++w) m = fmaxf(m, red[i][w]);
      sc[i] = live ? expf(sc[i] - m) : 0.0f;
      if (tid == 0) bk[i] = m;   // the chunk max, kept for the partial record
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < QB; ++i) {
    if (i < Mq) {
      const float e = sc[i];
      pr[i][tid] = e;
      float l = e;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      if (lane == 0) red[i][warp] = l;
    }
  }
  __syncthreads();
  // o[i][c] = sum_t pr[i][t] vq[t][c]: warp w takes tokens 32 w .. 32 w + 31,
  // lane l channels l, l + 32, ... (D / 32 of them); then the 8 warps' sums
  // are added in warp order through shared memory (over the staged keys,
  // which are no longer read)
  constexpr int CPL = D / 32;                      // channels per lane
  float acc[QB][CPL];
#pragma unroll
  for (int i = 0; i < QB; ++i)
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[i][k] = 0.0f;
  const int tw = warp * 32;
  const int tn = nt - tw < 32 ? (nt - tw > 0 ? nt - tw : 0) : 32;
  for (int u = 0; u < tn; ++u) {
    const int t = tw + u;
    float v[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) v[k] = (float)vc[t * D + lane + 32 * k];
#pragma unroll
    for (int i = 0; i < QB; ++i)
      if (i < Mq) {
        const float pt = pr[i][t];
#pragma unroll
        for (int k = 0; k < CPL; ++k) acc[i][k] = fmaf(pt, v[k], acc[i][k]);
      }
  }
  float* wsum = reinterpret_cast<float*>(kc);        // [8 warps][Mq][D] over the staged keys and values
  __syncthreads();                                   // every warp is done reading the staged values
#pragma unroll
  for (int i = 0; i < QB; ++i)
    if (i < Mq)
#pragma unroll
      for (int k = 0; k < CPL; ++k) wsum[(warp * Mq + i) * D + lane + 32 * k] = acc[i][k];
  __syncthreads();
  float* out = part + ((size_t)h * gridDim.y + blockIdx.y) * (size_t)Mq * (D + 2);
  for (int e = tid; e < Mq * D; e += 256) {
    const int i = e / D, c = e % D;
    float o = wsum[i * D + c];
#pragma unroll
    for (int w = 1; w < 8; ++w) o += wsum[(w * Mq + i) * D + c];
    out[(size_t)i * (D + 2) + 2 + c] = o;
    if (c == 0) {
      float l = red[i][0];
#pragma unroll
      for (int w = 1; w < 8; ++w) l += red[i][w];
      out[(size_t)i * (D + 2)] = bk[i];
      out[(size_t)i * (D + 2) + 1] = l;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) kv_attn_combine(const float* __restrict__ part, int n_chunks, int Mq, int C,
                                                     const float* __restrict__ vs, const uint8_t* __restrict__ vz,
                                                     float* __restrict__ O) {
  const int h = blockIdx.x, i = blockIdx.y, c = threadIdx.x;
  const float* p = part + ((size_t)h * n_chunks * Mq + i) * (D + 2);
  const size_t stride = (size_t)Mq * (D + 2);
  // the chunks in order, eight records in flight at a time
  float M = -INFINITY;
  for (int k0 = 0; k0 < n_chunks; k0 += 8) {
    float m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = k0 + j < n_chunks ? __ldcg(p + (k0 + j) * stride) : -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) M = fmaxf(M, m[j]);
  }
  float L = 0.0f, o = 0.0f;
  for (int k0 = 0; k0 < n_chunks; k0 += 8) {
    float m[8], l[8], x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = k0 + j < n_chunks;
      m[j] = in ? __ldcg(p + (k0 + j) * stride) : -INFINITY;
      l[j] = in ? __ldcg(p + (k0 + j) * stride + 1) : 0.0f;
      x[j] = in ? __ldcg(p + (k0 + j) * stride + 2 + c) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (k0 + j < n_chunks) {
        const float w = expf(m[j] - M);
        L = fmaf(w, l[j], L);
        o = fmaf(w, x[j], o);
      }
    }
  }
  const int cc = h * D + c;
  O[(size_t)i * C + cc] = __fmul_rn(__ldg(vs + cc), __fsub_rn(__fdiv_rn(o, L), (float)vz[cc]));
}

// sm_100 check, cached per device (cudaGetDeviceProperties costs milliseconds)
bool device_ok() {
  static std::atomic<int> state[64];   // 0 unknown, 1 ok, 2 not ok (zero-initialised)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  if (dev < 64) {
    const int known = state[dev].load(std::memory_order_relaxed);
    if (known) return known == 1;
  }
  int major = 0, minor = 0;
  const bool ok = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
                  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
                  major == 10 && minor == 0;
  if (dev < 64) state[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
  return ok;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

svdq_status launched() { return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA; }

}  // namespace kv
}  // namespace svdq

using namespace svdq::kv;

extern "C" {

size_t svdq_kv_workspace_bytes(int64_t T, int32_t C) {
  if (T < 1 || C < 1) return 0;
  return 2 * (size_t)((T + kTileT - 1) / kTileT) * (size_t)C * sizeof(float);
}

svdq_status svdq_kv_encode(const void* X, int64_t T, int32_t C, int32_t dtype, uint8_t* codes, float* scale,
                           uint8_t* zero, void* workspace, size_t ws_bytes, svdq_stream stream) {
  if (T < 1 || C < kTileC || C % kTileC != 0 || (dtype != SVDQ_BF16 && dtype != SVDQ_F16) || !X || !codes ||
      !scale || !zero || !workspace)
    return SVDQ_ERR_INVALID_ARG;
  if (ws_bytes < svdq_kv_workspace_bytes(T, C)) return SVDQ_ERR_WORKSPACE;
  if (!aligned(X, 16) || !aligned(codes, 16) || !aligned(scale, 16) || !aligned(zero, 16) || !aligned(workspace, 16))
    return SVDQ_ERR_ALIGNMENT;
  if (!device_ok()) return SVDQ_ERR_UNSUPPORTED;
  const dim3 grid(C / kTileC, (unsigned)((T + kTileT - 1) / kTileT));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t* x = static_cast<const uint16_t*>(X);
  float* part = static_cast<float*>(workspace);
  if (dtype == SVDQ_BF16) {
    kv_range_kernel<SVDQ_BF16><<<grid, kThreads, 0, s>>>(x, T, C, part);
    kv_quant_kernel<SVDQ_BF16><<<grid, kThreads, 0, s>>>(x, T, C, part, codes, scale, zero);
  } else {
    kv_range_kernel<SVDQ_F16><<<grid, kThreads, 0, s>>>(x, T, C, part);
    kv_quant_kernel<SVDQ_F16><<<grid, kThreads, 0, s>>>(x, T, C, part, codes, scale, zero);
  }
  return launched();
}

svdq_status svdq_kv_decode(const uint8_t* codes, const float* scale, const uint8_t* zero, int64_t T, int32_t C,
                           int32_t dtype, void* Y, svdq_stream stream) {
  if (T < 1 || C < 8 || C % 8 != 0 || (dtype != SVDQ_BF16 && dtype != SVDQ_F16) || !codes || !scale || !zero || !Y)
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scale, 16) || !aligned(zero, 16) || !aligned(Y, 16))
    return SVDQ_ERR_ALIGNMENT;
  if (!device_ok()) return SVDQ_ERR_UNSUPPORTED;
  const int64_t n8 = T * (int64_t)(C / 8);
  const int64_t blocks64 = (n8 + 255) / 256;
  const unsigned blocks = (unsigned)(blocks64 < 148 * 16 ? blocks64 : 148 * 16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SVDQ_BF16)
    kv_decode_kernel<SVDQ_BF16><<<blocks, 256, 0, s>>>(codes, scale, zero, T, C, static_cast<uint16_t*>(Y));
  else
    kv_decode_kernel<SVDQ_F16><<<blocks, 256, 0, s>>>(codes, scale, zero, T, C, static_cast<uint16_t*>(Y));
  return launched();
}

size_t svdq_kv_attention_workspace_bytes(int64_t T, int32_t C, int32_t heads, int32_t Mq) {
  if (T < 1 || C < 1 || heads < 1 || C % heads != 0 || Mq < 1) return 0;
  const int64_t d = C / heads, chunks = (T + kAttnChunk - 1) / kAttnChunk;
  return (size_t)heads * (size_t)chunks * (size_t)Mq * (size_t)(d + 2) * sizeof(float);
}

svdq_status svdq_kv_attention(const void* Q, int32_t Mq, const uint8_t* kcodes, const float* kscale,
                              const uint8_t* kzero, const uint8_t* vcodes, const float* vscale, const uint8_t* vzero,
                              int64_t T, int32_t C, int32_t heads, int32_t dtype, float* out, void* workspace,
                              size_t ws_bytes, svdq_stream stream) {
  if (Mq < 1 || Mq > kAttnMaxQ || T < 1 || heads < 1 || C < 1 || C % heads != 0 ||
      (dtype != SVDQ_BF16 && dtype != SVDQ_F16) || !Q || !kcodes || !kscale || !kzero || !vcodes || !vscale ||
      !vzero || !out || !workspace)
    return SVDQ_ERR_INVALID_ARG;
  const int d = C / heads;
  if (d != 64 && d != 128) return SVDQ_ERR_UNSUPPORTED;
  if (ws_bytes < svdq_kv_attention_workspace_bytes(T, C, heads, Mq)) return SVDQ_ERR_WORKSPACE;
  if (!aligned(Q, 16) || !aligned(kcodes, 16) || !aligned(vcodes, 16) || !aligned(kscale, 16) ||
      !aligned(vscale, 16) || !aligned(out, 16) || !aligned(workspace, 16))
    return SVDQ_ERR_ALIGNMENT;
  if (!device_ok()) return SVDQ_ERR_UNSUPPORTED;
  static std::atomic<int> attr_done[64];   // per device: the kernels' shared-memory attributes are set
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev < 0 || dev >= 64) return SVDQ_ERR_UNSUPPORTED;
#define SVDQ_ATTN_ATTR(DT_, D_, QB_)                                                                    \
  cudaFuncSetAttribute(kv_attn_partial<DT_, D_, QB_>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                       attn_smem_bytes(D_, QB_)) == cudaSuccess
  if (!attr_done[dev].load()) {
    const bool ok = SVDQ_ATTN_ATTR(SVDQ_BF16, 64, 1) && SVDQ_ATTN_ATTR(SVDQ_BF16, 64, 4) &&
                    SVDQ_ATTN_ATTR(SVDQ_BF16, 64, 16) && SVDQ_ATTN_ATTR(SVDQ_F16, 64, 1) &&
                    SVDQ_ATTN_ATTR(SVDQ_F16, 64, 4) && SVDQ_ATTN_ATTR(SVDQ_F16, 64, 16) &&
                    SVDQ_ATTN_ATTR(SVDQ_BF16, 128, 1) && SVDQ_ATTN_ATTR(SVDQ_BF16, 128, 4) &&
                    SVDQ_ATTN_ATTR(SVDQ_BF16, 128, 16) && SVDQ_ATTN_ATTR(SVDQ_F16, 128, 1) &&
                    SVDQ_ATTN_ATTR(SVDQ_F16, 128, 4) && SVDQ_ATTN_ATTR(SVDQ_F16, 128, 16);
    if (!ok) return SVDQ_ERR_CUDA;
    attr_done[dev].store(1);
  }
#undef SVDQ_ATTN_ATTR
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int chunks = (int)((T + kAttnChunk - 1) / kAttnChunk);
  const dim3 grid(heads, chunks);
  const uint16_t* q = static_cast<const uint16_t*>(Q);
  float* part = static_cast<float*>(workspace);
  const int qb = Mq <= 1 ? 1 : (Mq <= 4 ? 4 : 16);
#define SVDQ_ATTN_LAUNCH(DT_, D_, QB_)                                                                           \
  kv_attn_partial<DT_, D_, QB_><<<grid, 256, attn_smem_bytes(D_, QB_), s>>>(q, Mq, kcodes, kscale, kzero, vcodes, T, \
                                                                           C, part)
#define SVDQ_ATTN_QB(DT_, D_)                           \
  do {                                                  \
    if (qb == 1) SVDQ_ATTN_LAUNCH(DT_, D_, 1);          \
    else if (qb == 4) SVDQ_ATTN_LAUNCH(DT_, D_, 4);     \
    else SVDQ_ATTN_LAUNCH(DT_, D_, 16);                 \
  } while (0)
  if (d == 64) {
    if (dtype == SVDQ_BF16) SVDQ_ATTN_QB(SVDQ_BF16, 64); else SVDQ_ATTN_QB(SVDQ_F16, 64);
    kv_attn_combine<64><<<dim3(heads, Mq), 64, 0, s>>>(part, chunks, Mq, C, vscale, vzero, out);
  } else {
    if (dtype == SVDQ_BF16) SVDQ_ATTN_QB(SVDQ_BF16, 128); else SVDQ_ATTN_QB(SVDQ_F16, 128);
    kv_attn_combine<128><<<dim3(heads, Mq), 128, 0, s>>>(part, chunks, Mq, C, vscale, vzero, out);
  }
#undef SVDQ_ATTN_QB
#undef SVDQ_ATTN_LAUNCH
  return launched();
}

}  // extern "C"
