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

__device__ __forceinline__ uint32_t code(float x, float s, int z) {
  const int q = __float2int_rn(__fdiv_rn(x, s)) + z;
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
  float sc[8];
  int z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { sc[i] = s_sc[8 * lane + i]; z[i] = s_z[8 * lane + i]; }
  const int c = blockIdx.x * kTileC + 8 * lane;
  const int64_t t0 = (int64_t)blockIdx.y * kTileT;
  const int64_t t1 = t0 + kTileT < T ? t0 + kTileT : T;
#pragma unroll 8
  for (int64_t t = t0 + warp; t < t1; t += kWarps) {
    float v[8];
    unpack8<DT>(__ldg(reinterpret_cast<const uint4*>(X + t * C + c)), v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i >> 2] |= code(v[i], sc[i], z[i]) << (8 * (i & 3));
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

}  // extern "C"
