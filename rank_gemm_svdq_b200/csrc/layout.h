// Internal layouts of the blob (prepared weights) and of the per-call workspace.
//
// Blob (one contiguous buffer, every section 1024-byte aligned):
//   header      BlobHeader
//   inv_lambda  K fp32                                  smoothing, device multiplies X by it
//   l1t         r x K act_dtype (L1 transposed)          B operand of the down projection
//   l2x         N x lrw bf16, K-major                    B operand of the up projection
//               (NVFP4: as low-rank tiles, below; INT4: row-major)
//               (lrw = nseg*r rounded up to 64, zero padded):
//               bf16 X: [L2 ; L2]             (pairs with [u_hi | u_lo])
//               fp16 X: [L2h ; L2h ; L2l]     (pairs with [u_hi | u_lo | u_hi]; L2 = L2h + L2l exactly)
//   wq          NVFP4: weight tiles (below), [N/128][K/256] x 20480 bytes
//               INT4:  N x K bytes, the code as an E4M3 byte (exact for -8..7)
//   ws          NVFP4: empty (the scales live in the weight tiles)
//               INT4:  fp32 group scales, blocked [K/128][N/128][2][128]
//               (one 128-wide K slab of a 256-column tile is one contiguous 2 KB)
//   bias        N fp32
//
// Workspace for M tokens:
//   xq   NVFP4: activation tiles (below), [Mp/128][K/256] x 18432 bytes
//        INT4:  M x K bytes (code as E4M3 byte)
//   xs   NVFP4: empty;  INT4: fp32 group scales, blocked [K/128][Mp/128][2][128],
//        Mp = ceil(M/128)*128 (one K slab of a 128-token tile is one contiguous 1 KB)
//   ux   M x lrw bf16: [u'_hi | u'_lo (| u'_hi) | 0 pad], u' = u / (s_gX s_gW) (NVFP4) or u (INT4)
//        (NVFP4: as low-rank tiles over Mp rows; INT4: row-major)
//   part, cnt   NVFP4 K-split scratch when nvfp4_split_k_eligible (below), else empty
//   upart, ucnt NVFP4 activation kernel K split (act_nv_ks > 1): fp32 partial down
//               projections [Mp/128][ks][128][r] and one 64-bit arrival word per
//               128-token tile (need no initial value: each call tags its
//               arrivals with a fresh epoch)
//
// NVFP4 operand tiles (what one bulk copy brings into shared memory, ready
// for the tensor core): 128 rows x one K slab of 256 elements.  The E2M1
// codes (two per byte, even element in the low nibble) sit as 128 rows of
// 128 bytes with the 128-byte swizzle -- 16-byte chunk c of row r stored at
// chunk c ^ (r % 8) -- followed by the slab's E4M3 scale atoms:
//   activation tile: 16384 bytes of codes + 2048 bytes of scales (its 128 rows)
//   weight tile:     16384 bytes of codes + 4096 bytes of scales of the 256 rows
//                    (two row blocks 2p, 2p+1) that one CTA pair multiplies
// Low-rank tiles: 128 rows x 64 bf16 (128 bytes), same swizzle, 16384 bytes.
//
// Scale-factor atom layout (the operand format of tcgen05 block-scaled MMA
// scale factors once copied to tensor memory by tcgen05.cp 32x128b.warpx4):
// rows are grouped by 128, scale blocks along K by 4 (64 elements); each group
// is a 512-byte atom, atoms ordered [row_group][k_group]; inside an atom the
// scale of row r (0..127) and block j (0..3) sits at byte (r%32)*16 + (r/32)*4 + j.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/svdq.h"

namespace svdq {

constexpr uint32_t kMagic0 = 0x51445653u;  // "SVDQ"
constexpr uint32_t kMagic1 = 0x30303242u;  // "B200"
constexpr uint32_t kVersion = 1;
constexpr size_t kAlign = 1024;
constexpr int kGroupInt4 = 64;
constexpr int kBlockFp4 = 16;
constexpr int kTileCodes = 16384;   // 128 rows x 128 bytes
constexpr int kATile = 18432;       // activation tile: codes + 128 rows of scales
constexpr int kWTile = 20480;       // weight tile: codes + 256 rows of scales
constexpr int kLRTile = 16384;      // low-rank tile: 128 rows x 64 bf16

struct BlobHeader {
  uint32_t magic0, magic1, version, header_bytes;
  svdq_params params;
  uint64_t total_bytes;
  uint64_t off_inv_lambda, off_l1t, off_l2x, off_wq, off_ws, off_bias;
  float s_gx, s_gw;
  int32_t nseg, pad0;
  uint64_t checksum;  // FNV-1a 64 over bytes [header_bytes, total_bytes)
};
static_assert(sizeof(BlobHeader) <= kAlign, "header too large");

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

#ifdef __CUDACC__
#define SVDQ_HD __host__ __device__
#else
#define SVDQ_HD
#endif

inline int nseg_of(const svdq_params& p) { return p.act_dtype == SVDQ_F16 ? 3 : 2; }
// Width (bf16 elements) of one row of the low-rank operands.
inline int lr_width(const svdq_params& p) { return (nseg_of(p) * p.rank + 63) / 64 * 64; }

struct BlobLayout {
  size_t off_inv_lambda, off_l1t, off_l2x, off_wq, off_ws, off_bias, total;
  int nseg;
};

inline BlobLayout blob_layout(const svdq_params& p) {
  BlobLayout L{};
  const size_t K = (size_t)p.K, N = (size_t)p.N, r = (size_t)p.rank;
  L.nseg = nseg_of(p);
  size_t off = kAlign;
  L.off_inv_lambda = off; off = align_up(off + K * 4);
  L.off_l1t = off;        off = align_up(off + r * K * 2);
  L.off_l2x = off;        off = align_up(off + N * (size_t)lr_width(p) * 2);
  L.off_wq = off;
  off = align_up(off + (p.fmt == SVDQ_NVFP4 ? (N / 128) * (K / 256) * (size_t)kWTile : N * K));
  L.off_ws = off;
  off = align_up(off + (p.fmt == SVDQ_NVFP4 ? 0 : (K / kGroupInt4) * N * 4));
  L.off_bias = off;       off = align_up(off + N * 4);
  L.total = off;
  return L;
}

struct WsLayout {
  size_t off_xq, off_xs, off_ux, off_part, off_cnt, off_upart, off_ucnt, total;
  int64_t Mp;  // M rounded up to the GEMM's row tile (256 NVFP4, 128 INT4)
};

// NVFP4 with few tokens and few output tiles: the GEMM may split K over up to
// kMaxKSplit CTA pairs per tile; the workspace then also holds the fp32
// partial sums [ks][M][N] and one arrival counter per tile region [tiles][16]
// (zeroed by the activation kernel of the same call).
constexpr int kMaxKSplit = 8;
inline bool nvfp4_split_k_eligible(const svdq_params& p, int64_t M) {
  return p.fmt == SVDQ_NVFP4 && M >= 1 && M <= 64 && p.N / 256 <= 37;
}

// K split of the NVFP4 activation kernel: ks CTAs (a power of two dividing
// K / 256, at most 16, which bounds the contention on a tile's arrival word)
// share each 128-token tile so that the grid fills about the 148 SMs of a
// B200.  A fixed function of the shape, so that the host sizes the workspace
// the same way the launcher splits.
constexpr int kActSizingSMs = 148;
constexpr int kActMaxKs = 16;
SVDQ_HD inline int act_nv_ks(int64_t Mp, int K) {
  const int64_t tiles = Mp / 128;
  const int slabs = K / 256;
  int ks = 1;
  while (ks < kActMaxKs && tiles * ks * 2 <= kActSizingSMs && slabs % (ks * 2) == 0) ks *= 2;
  return ks;
}

// NVFP4 up to 256 tokens (the 32-token activation kernel): with few live
// 32-token groups and K >= 8192, ks CTAs split a group's K range (a power of
// two dividing K / 256, at most kActGMaxKs).  Clusters of up to 8 add their partial down
// projections through distributed shared memory; above 8 the ks / 8 cluster
// sums meet in the workspace ([groups][ks / 8][32][r] fp32 plus one 64-bit
// arrival word per group, tagged per call like the 128-token kernel's).
constexpr int kActGMaxKs = 32;
constexpr int kActClusterKs = 8;
SVDQ_HD inline int act_small_ks(int64_t M, int K) {
  const int64_t groups = (M + 31) / 32;
  const int chunks = K / 256;
  if (chunks < 4 * kActClusterKs) return 1;   // a cluster of 8 leaves <= 3 slabs per CTA: no workspace split
  int ks = 1;
  while (ks < kActGMaxKs && groups * ks * 2 <= kActSizingSMs && chunks % (ks * 2) == 0) ks *= 2;
  return ks;
}

inline WsLayout ws_layout(const svdq_params& p, int64_t M) {
  WsLayout L{};
  const size_t K = (size_t)p.K;
  // NVFP4 pads tokens to whole 256-row tiles (one CTA pair), INT4 to 128
  const int64_t pad = p.fmt == SVDQ_NVFP4 ? 256 : 128;
  L.Mp = (M + pad - 1) / pad * pad;
  const size_t Mp = (size_t)L.Mp;
  size_t off = 0;
  L.off_xq = off;
  off = align_up(off + (p.fmt == SVDQ_NVFP4 ? (Mp / 128) * (K / 256) * (size_t)kATile : (size_t)M * K));
  L.off_xs = off;
  off = align_up(off + (p.fmt == SVDQ_NVFP4 ? 0 : (K / kGroupInt4) * Mp * 4));
  L.off_ux = off;
  off = align_up(off + (p.fmt == SVDQ_NVFP4 ? Mp : (size_t)M) * (size_t)lr_width(p) * 2);
  L.off_part = L.off_cnt = off;
  if (nvfp4_split_k_eligible(p, M)) {
    off = align_up(off + (size_t)kMaxKSplit * (size_t)M * (size_t)p.N * 4);
    L.off_cnt = off;
    off = align_up(off + (size_t)(p.N / 256) * (Mp / 256) * 16 * 4);
  }
  L.off_upart = L.off_ucnt = off;
  if (p.fmt == SVDQ_NVFP4 && M > 256) {   // the 128-token-tile activation kernel (see the launcher)
    const int ks = act_nv_ks(L.Mp, p.K);
    if (ks > 1 && p.rank > 0) {
      off = align_up(off + (Mp / 128) * (size_t)ks * 128 * (size_t)p.rank * 4);
      L.off_ucnt = off;
      off = align_up(off + (Mp / 128) * 8);
    }
  } else if (p.fmt == SVDQ_NVFP4 && M >= 1) {   // the 32-token kernel with its K split in the workspace
    const int ks = act_small_ks(M, p.K);
    if (ks > kActClusterKs && p.rank > 0) {
      const size_t groups = (size_t)((M + 31) / 32);
      off = align_up(off + groups * (size_t)(ks / kActClusterKs) * 32 * (size_t)p.rank * 4);
      L.off_ucnt = off;
      off = align_up(off + groups * 8);
    }
  }
  L.total = off > 0 ? off : kAlign;
  return L;
}

// NVFP4 up to this many tokens: the GEMM streams each weight tile as the A
// operand of a 1-CTA MMA with the tokens as a narrow B operand.
constexpr int64_t kFewTokens = 128;

// Chained layers (svdq_gemm_chain): this layer's GEMM emits the next layer's
// quantised input.  Both NVFP4, the next layer's input bf16 (this layer's
// output type) and its rank 0, 16 or 32.
inline svdq_status chain_supported(const svdq_params& p, const svdq_params& pn) {
  if (p.fmt != SVDQ_NVFP4 || pn.fmt != SVDQ_NVFP4 || pn.act_dtype != SVDQ_BF16) return SVDQ_ERR_UNSUPPORTED;
  if (pn.K != p.N) return SVDQ_ERR_INVALID_ARG;
  if (pn.rank != 0 && pn.rank != 16 && pn.rank != 32) return SVDQ_ERR_UNSUPPORTED;
  return SVDQ_OK;
}

// Workspace of a chained call: this layer's workspace, then above kFewTokens
// the partial down projections of the next layer, [N/256][Mp][r'] fp32 (one
// per output tile column), or up to kFewTokens an M x N bf16 buffer for this
// layer's output (there the call runs the GEMM and the next layer's
// activation kernel one after the other).
struct ChainLayout {
  size_t off_extra, total;
};
inline ChainLayout chain_layout(const svdq_params& p, const svdq_params& pn, int64_t M) {
  ChainLayout L{};
  const WsLayout W = ws_layout(p, M);
  L.off_extra = align_up(W.total);
  const size_t extra = M <= kFewTokens ? (size_t)M * (size_t)p.N * 2
                                       : (size_t)(p.N / 256) * (size_t)W.Mp * (size_t)pn.rank * 4;
  L.total = L.off_extra + align_up(extra);
  return L;
}

// Byte offset of scale (row, block) inside a scale-factor atom array whose
// rows span `kblocks` blocks of 16 along K (kblocks % 4 == 0).
SVDQ_HD inline size_t sf_offset(int64_t row, int64_t blk, int64_t kblocks) {
  const int64_t atom = (row / 128) * (kblocks / 4) + blk / 4;
  const int64_t r = row % 128;
  return (size_t)(atom * 512 + (r % 32) * 16 + (r / 32) * 4 + (blk % 4));
}

// Index (in floats) of INT4 group scale g of token m / output feature n in the
// blocked scale arrays described above.
SVDQ_HD inline size_t int4_sx_index(int64_t g, int64_t m, int64_t Mp) {
  return ((size_t)(g >> 1) * (size_t)(Mp / 128) + (size_t)(m / 128)) * 256 + (size_t)(g & 1) * 128 + (size_t)(m % 128);
}
SVDQ_HD inline size_t int4_sw_index(int64_t g, int64_t n, int64_t N) {
  return ((size_t)(g >> 1) * (size_t)(N / 128) + (size_t)(n / 128)) * 256 + (size_t)(g & 1) * 128 + (size_t)(n % 128);
}

// Byte offset of (row r, byte c) inside a 128 x 128-byte tile with the 128-byte swizzle.
SVDQ_HD inline uint32_t sw128(uint32_t r, uint32_t c) {
  return r * 128u + ((((c >> 4) ^ (r & 7u)) & 7u) << 4) + (c & 15u);
}

// Byte offset of the scale of tile row rr (0..127) and scale block j (0..15
// inside the slab) within a tile's scale atoms.
SVDQ_HD inline uint32_t tile_sf(uint32_t rr, uint32_t j) {
  return (j >> 2) * 512u + (rr & 31u) * 16u + (rr >> 5) * 4u + (j & 3u);
}

}  // namespace svdq
