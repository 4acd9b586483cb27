// Host half of libsvdq: parameter checks, offline preparation (smoothing,
// truncated SVD, residual quantisation, packing) and blob export.
//
// The method: "SVDQuant是什么？" 技术原理 (smoothing moves activation outliers
// into the weight; SVD splits the weight into a 16-bit low-rank branch and a
// residual quantised to 4 bits; Eckart-Young-Mirsky); "AI图像生成4-bit量化技术
// 解析与应用" 2.2 (W = U S V^T, keep the top k, quantise R = W - W_k) and 3.1/3.2
// (INT4 groups, NVFP4); W4A8 page 3.1 (symmetric absmax quantiser).
//
// Compiled with -ffp-contract=off: the residual and the quantisers are fixed
// sequences of IEEE operations, so their results are reproducible bit for bit.
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "layout.h"

using namespace svdq;

namespace {

// ------------------------------------------------------------ parameters
svdq_status check_params(const svdq_params* p) {
  if (!p) return SVDQ_ERR_INVALID_ARG;
  // the activation kernel and the NVFP4 GEMM work in whole 256-wide K slabs
  if (p->K <= 0 || p->N <= 0 || p->K % 256 != 0 || p->N % 256 != 0) return SVDQ_ERR_INVALID_ARG;
  if (p->rank < 0 || p->rank > 128 || p->rank % 16 != 0 || p->rank > std::min(p->K, p->N))
    return SVDQ_ERR_INVALID_ARG;
  if (p->fmt != SVDQ_INT4_G64 && p->fmt != SVDQ_NVFP4) return SVDQ_ERR_UNSUPPORTED;
  if (p->act_dtype != SVDQ_F16 && p->act_dtype != SVDQ_BF16) return SVDQ_ERR_UNSUPPORTED;
  if (!(p->alpha >= 0.0f && p->alpha <= 1.0f)) return SVDQ_ERR_INVALID_ARG;
  if (p->smooth != 0 && p->smooth != 1) return SVDQ_ERR_INVALID_ARG;
  if (p->reserved != 0) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

// ------------------------------------------------------------ 16-bit floats
// Round a double to `sig` significant bits with minimum normal exponent emin
// (subnormal grid below), ties to even, in one step (no double rounding).
double round_sig(double x, int sig, int emin) {
  if (x == 0.0) return x;
  int e;
  frexp(x, &e);                 // |x| = m 2^e, m in [0.5, 1)
  int lead = std::max(e - 1, emin);
  double quantum = ldexp(1.0, lead - (sig - 1));
  return nearbyint(x / quantum) * quantum;   // default rounding mode: to nearest even
}

double bf16_round(double x) { return round_sig(x, 8, -126); }
double fp16_round(double x) { return round_sig(x, 11, -14); }

uint16_t bf16_bits_exact(double v) {          // v already a bf16 value
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

uint16_t fp16_bits_exact(double v) {          // v already an fp16 value, |v| <= 65504
  uint16_t s = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (a == 0.0) return s;
  if (a < ldexp(1.0, -14)) return s | (uint16_t)llround(a / ldexp(1.0, -24));
  int e;
  frexp(a, &e);
  int ex = e - 1;                                              // a in [2^ex, 2^(ex+1))
  uint16_t mant = (uint16_t)llround((a / ldexp(1.0, ex) - 1.0) * 1024.0);
  return s | (uint16_t)((ex + 15) << 10) | mant;
}

double fp16_value(uint16_t b) {
  int s = b >> 15, e = (b >> 10) & 31, m = b & 1023;
  double v = e == 0 ? ldexp((double)m, -24) : ldexp(1.0 + m / 1024.0, e - 15);
  return s ? -v : v;
}

double dtype_round(double x, int dt) { return dt == SVDQ_F16 ? fp16_round(x) : bf16_round(x); }
uint16_t dtype_bits(double v, int dt) { return dt == SVDQ_F16 ? fp16_bits_exact(v) : bf16_bits_exact(v); }
double dtype_value(uint16_t b, int dt) { return dt == SVDQ_F16 ? fp16_value(b) : bf16_value(b); }

// ------------------------------------------------------------ 4/8-bit floats
// fp32 -> E4M3 (OCP E4M3FN) code, round to nearest even, saturating to 448.
uint8_t e4m3_encode(float x) {
  uint8_t s = signbit(x) ? 0x80 : 0;
  double a = fabs((double)x);
  if (a >= 448.0) return s | 0x7E;
  if (a < ldexp(1.0, -6)) {                       // subnormal grid 2^-9 (code 8 = 2^-6)
    return s | (uint8_t)nearbyint(a * 512.0);
  }
  int e;
  frexp(a, &e);
  int ex = e - 1;                                 // a in [2^ex, 2^(ex+1)), ex in [-6, 8]
  double q = nearbyint((a / ldexp(1.0, ex) - 1.0) * 8.0);
  if (q == 8.0) { q = 0.0; ++ex; }
  int code = ((ex + 7) << 3) | (int)q;
  return s | (uint8_t)std::min(code, 0x7E);
}

double e4m3_value(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

// fp32 -> E2M1 code (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), ties to even, saturating.
uint8_t e2m1_encode(float x) {
  uint8_t s = signbit(x) ? 0x8 : 0;
  double a = fabs((double)x);
  uint8_t c;
  if (a >= 6.0) c = 7;
  else if (a < 2.0) c = (uint8_t)nearbyint(a * 2.0);            // 0 .. 4 on a 0.5 grid
  else if (a < 4.0) c = (uint8_t)(2 + (int)nearbyint(a));       // 2,3,4 -> codes 4,5,6
  else c = (uint8_t)(4 + (int)nearbyint(a * 0.5));              // 4,6 -> codes 6,7
  return s | c;
}

double e2m1_value(uint8_t c) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  return (c & 8) ? -mag[c & 7] : mag[c & 7];
}

// ------------------------------------------------------------ quantisers
// INT4 symmetric group quantiser: s = m / 7, q = clamp(rint(v / s), -8, 7).
void int4_quant_row(const float* v, int K, int8_t* q, float* s_out /* K/64 */) {
  for (int g = 0; g < K / kGroupInt4; ++g) {
    const float* vg = v + g * kGroupInt4;
    float m = 0.0f;
    for (int j = 0; j < kGroupInt4; ++j) m = std::max(m, fabsf(vg[j]));
    float s = m / 7.0f;
    s_out[g] = s;
    for (int j = 0; j < kGroupInt4; ++j) {
      int qi = 0;
      if (m != 0.0f) {
        float t = vg[j] / s;
        qi = (int)nearbyintf(t);
        qi = std::min(7, std::max(-8, qi));
      }
      q[g * kGroupInt4 + j] = (int8_t)qi;
    }
  }
}

// NVFP4 row quantiser with fp32 tensor scale s_g.
void nvfp4_quant_row(const float* v, int K, float s_g, uint8_t* codes, uint8_t* scales) {
  const float six_sg = 6.0f * s_g;
  for (int b = 0; b < K / kBlockFp4; ++b) {
    const float* vb = v + b * kBlockFp4;
    float m = 0.0f;
    for (int j = 0; j < kBlockFp4; ++j) m = std::max(m, fabsf(vb[j]));
    float ratio = m / six_sg;
    uint8_t e = e4m3_encode(ratio);
    scales[b] = e;
    float d = (float)e4m3_value(e) * s_g;
    for (int j = 0; j < kBlockFp4; ++j)
      codes[b * kBlockFp4 + j] = d == 0.0f ? 0 : e2m1_encode(vb[j] / d);
  }
}

float nvfp4_tensor_scale(float amax) {
  float s = amax / 2688.0f;
  return s == 0.0f ? 1.0f : s;
}

// ------------------------------------------------------------ dense helpers
// C (rows x l) = A (rows x cols, row-major) * B (cols x l, row-major)
void matmul_rows(const double* A, int64_t rows, int64_t cols, const double* B, int l, double* C) {
  const int RB = 16;
#pragma omp parallel for schedule(static)
  for (int64_t r0 = 0; r0 < rows; r0 += RB) {
    const int nr = (int)std::min<int64_t>(RB, rows - r0);
    std::vector<double> acc((size_t)RB * l, 0.0);
    for (int64_t c = 0; c < cols; ++c) {
      const double* b = B + c * l;
      for (int i = 0; i < nr; ++i) {
        const double a = A[(r0 + i) * cols + c];
        double* o = acc.data() + (size_t)i * l;
        for (int j = 0; j < l; ++j) o[j] += a * b[j];
      }
    }
    memcpy(C + r0 * l, acc.data(), sizeof(double) * (size_t)nr * l);
  }
}

// C (cols x l) = A^T * B, A rows x cols row-major, B rows x l row-major
void matmul_tn(const double* A, int64_t rows, int64_t cols, const double* B, int l, double* C) {
  const int CB = 32;
#pragma omp parallel for schedule(static)
  for (int64_t c0 = 0; c0 < cols; c0 += CB) {
    const int nc = (int)std::min<int64_t>(CB, cols - c0);
    std::vector<double> acc((size_t)CB * l, 0.0);
    for (int64_t r = 0; r < rows; ++r) {
      const double* b = B + r * l;
      const double* a = A + r * cols + c0;
      for (int i = 0; i < nc; ++i) {
        const double av = a[i];
        double* o = acc.data() + (size_t)i * l;
        for (int j = 0; j < l; ++j) o[j] += av * b[j];
      }
    }
    memcpy(C + c0 * l, acc.data(), sizeof(double) * (size_t)nc * l);
  }
}

// Orthonormalise the l columns of Y (n x l, row-major) in place by
// Gram-Schmidt applied twice; columns that vanish are set to zero.
void orthonormalise(double* Y, int64_t n, int l) {
  std::vector<double> col((size_t)n);
  for (int j = 0; j < l; ++j) {
    double norm0 = 0.0;
    for (int64_t i = 0; i < n; ++i) norm0 += Y[i * l + j] * Y[i * l + j];
    norm0 = sqrt(norm0);
    for (int pass = 0; pass < 2; ++pass) {
      for (int k = 0; k < j; ++k) {
        double d = 0.0;
        for (int64_t i = 0; i < n; ++i) d += Y[i * l + k] * Y[i * l + j];
        for (int64_t i = 0; i < n; ++i) Y[i * l + j] -= d * Y[i * l + k];
      }
    }
    double nrm = 0.0;
    for (int64_t i = 0; i < n; ++i) nrm += Y[i * l + j] * Y[i * l + j];
    nrm = sqrt(nrm);
    const bool keep = nrm > 1e-13 * norm0 && nrm > 0.0;
    for (int64_t i = 0; i < n; ++i) Y[i * l + j] = keep ? Y[i * l + j] / nrm : 0.0;
  }
}

// Symmetric eigen-decomposition by cyclic two-sided Jacobi rotations:
// G (l x l) = E diag(w) E^T.  Returns false if it does not converge.
bool sym_eig_jacobi(std::vector<double>& G, int l, std::vector<double>& w, std::vector<double>& E) {
  E.assign((size_t)l * l, 0.0);
  for (int i = 0; i < l; ++i) E[(size_t)i * l + i] = 1.0;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < l; ++i)
      for (int j = 0; j < l; ++j) (i == j ? diag : off) += G[(size_t)i * l + j] * G[(size_t)i * l + j];
    if (off <= 1e-30 * diag || off == 0.0) {
      w.resize(l);
      for (int i = 0; i < l; ++i) w[i] = G[(size_t)i * l + i];
      return true;
    }
    for (int p = 0; p < l - 1; ++p)
      for (int q = p + 1; q < l; ++q) {
        const double gpq = G[(size_t)p * l + q];
        if (gpq == 0.0) continue;
        const double gpp = G[(size_t)p * l + p], gqq = G[(size_t)q * l + q];
        const double theta = (gqq - gpp) / (2.0 * gpq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
        const double c = 1.0 / sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < l; ++k) {                  // G <- G J (columns p, q)
          const double a = G[(size_t)k * l + p], b = G[(size_t)k * l + q];
          G[(size_t)k * l + p] = c * a - s * b;
          G[(size_t)k * l + q] = s * a + c * b;
        }
        for (int k = 0; k < l; ++k) {                  // G <- J^T G (rows p, q)
          const double a = G[(size_t)p * l + k], b = G[(size_t)q * l + k];
          G[(size_t)p * l + k] = c * a - s * b;
          G[(size_t)q * l + k] = s * a + c * b;
        }
        for (int k = 0; k < l; ++k) {                  // E <- E J
          const double a = E[(size_t)k * l + p], b = E[(size_t)k * l + q];
          E[(size_t)k * l + p] = c * a - s * b;
          E[(size_t)k * l + q] = s * a + c * b;
        }
      }
  }
  return false;
}

// Standard normals from a SplitMix64 counter stream (Box-Muller), seeded.
void gaussian_fill(double* x, size_t n, uint64_t seed) {
  auto mix = [](uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  };
  for (size_t i = 0; i < n; i += 2) {
    const double u1 = ((mix(seed + (2 * i + 1) * 0x9E3779B97F4A7C15ull) >> 11) + 0.5) * 0x1p-53;
    const double u2 = ((mix(seed + (2 * i + 2) * 0x9E3779B97F4A7C15ull) >> 11) + 0.5) * 0x1p-53;
    const double r = sqrt(-2.0 * log(u1));
    x[i] = r * cos(6.283185307179586 * u2);
    if (i + 1 < n) x[i + 1] = r * sin(6.283185307179586 * u2);
  }
}

// Top-`rank` singular triplets of A (n x k, row-major) by randomized subspace
// iteration: block size l = rank + 32, `iters` power iterations with
// re-orthonormalisation, then the exact SVD of the l x k projected matrix
// through the eigen-decomposition of its Gram matrix.
// Output: P (n x rank, orthonormal columns), sigma (rank + 1 estimates).
svdq_status truncated_svd(const double* A, int64_t n, int64_t k, int rank, int iters,
                          std::vector<double>& P, std::vector<double>& sigma) {
  const int l = (int)std::min<int64_t>(rank + 32, std::min(n, k));
  std::vector<double> Om((size_t)k * l), Y((size_t)n * l), Z((size_t)k * l);
  gaussian_fill(Om.data(), Om.size(), 0x5344564451ull);
  matmul_rows(A, n, k, Om.data(), l, Y.data());          // Y = A Om
  orthonormalise(Y.data(), n, l);
  for (int it = 0; it < iters; ++it) {
    matmul_tn(A, n, k, Y.data(), l, Z.data());           // Z = A^T Y
    orthonormalise(Z.data(), k, l);
    matmul_rows(A, n, k, Z.data(), l, Y.data());         // Y = A Z
    orthonormalise(Y.data(), n, l);
  }
  // B^T = A^T Y (k x l); G = B B^T = Y^T A A^T Y (l x l)
  matmul_tn(A, n, k, Y.data(), l, Z.data());
  std::vector<double> G((size_t)l * l, 0.0);
  for (int i = 0; i < l; ++i)
    for (int j = 0; j < l; ++j) {
      double s = 0.0;
      for (int64_t r = 0; r < k; ++r) s += Z[(size_t)r * l + i] * Z[(size_t)r * l + j];
      G[(size_t)i * l + j] = s;
    }
  std::vector<double> w, E;
  if (!sym_eig_jacobi(G, l, w, E)) return SVDQ_ERR_NO_CONVERGENCE;
  std::vector<int> order(l);
  for (int i = 0; i < l; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return w[a] > w[b]; });
  sigma.assign(rank + 1, 0.0);
  for (int i = 0; i <= rank && i < l; ++i) sigma[i] = sqrt(std::max(0.0, w[order[i]]));
  // left singular vectors of A: P = Y E (columns in descending order)
  P.assign((size_t)n * rank, 0.0);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n; ++r)
    for (int c = 0; c < rank; ++c) {
      double s = 0.0;
      for (int j = 0; j < l; ++j) s += Y[(size_t)r * l + j] * E[(size_t)j * l + order[c]];
      P[(size_t)r * rank + c] = sigma[c] > 0.0 ? s : 0.0;
    }
  return SVDQ_OK;
}

uint64_t fnv1a(const uint8_t* p, size_t n) {
  uint64_t h = 0xcbf29ce484222325ull;
  for (size_t i = 0; i < n; ++i) { h ^= p[i]; h *= 0x100000001b3ull; }
  return h;
}

// Write the low-rank factors (act_dtype values, as doubles) in their device
// layouts: l1t = L1^T (r x K), and l2x, the N x lrw B operand of the up
// projection, [L2 ; L2] for bf16 X or [L2h ; L2h ; L2l] for fp16 X (L2 =
// L2h + L2l exactly), row-major (INT4) or as swizzled low-rank tiles (NVFP4).
void write_factors(const svdq_params* p, const BlobLayout& L, uint8_t* base, const double* L1, const double* L2) {
  const int K = p->K, N = p->N, r = p->rank, dt = p->act_dtype;
  uint16_t* l1t = (uint16_t*)(base + L.off_l1t);
  for (int i = 0; i < r; ++i)
    for (int j = 0; j < K; ++j) l1t[(size_t)i * K + j] = dtype_bits(L1[(size_t)j * r + i], dt);
  uint16_t* l2x = (uint16_t*)(base + L.off_l2x);
  const int w2 = lr_width(*p);
  auto l2x_at = [&](int n, int e) -> uint16_t& {
    if (p->fmt != SVDQ_NVFP4) return l2x[(size_t)n * w2 + e];
    uint8_t* tile = base + L.off_l2x + ((size_t)(n / 128) * (w2 / 64) + e / 64) * kLRTile;
    return *reinterpret_cast<uint16_t*>(tile + sw128(n % 128, (e % 64) * 2));
  };
  for (int n = 0; n < N; ++n)
    for (int i = 0; i < r; ++i) {
      const double v = L2[(size_t)i * N + n];
      const double hi = bf16_round(v), lo = v - hi;                  // lo exact in bf16
      l2x_at(n, i) = bf16_bits_exact(hi);
      l2x_at(n, r + i) = bf16_bits_exact(hi);
      if (L.nseg == 3) l2x_at(n, 2 * r + i) = bf16_bits_exact(lo);
    }
}

// Read the low-rank factors back as act_dtype values (the inverse of write_factors).
void read_factors(const svdq_params* p, const BlobLayout& L, const uint8_t* base, double* L1, double* L2) {
  const int K = p->K, N = p->N, r = p->rank, dt = p->act_dtype;
  const uint16_t* l1t = (const uint16_t*)(base + L.off_l1t);
  for (int j = 0; j < K; ++j)
    for (int i = 0; i < r; ++i) L1[(size_t)j * r + i] = dtype_value(l1t[(size_t)i * K + j], dt);
  const uint16_t* l2x = (const uint16_t*)(base + L.off_l2x);
  const int w2 = lr_width(*p);
  auto at = [&](int n, int e) -> uint16_t {
    if (p->fmt != SVDQ_NVFP4) return l2x[(size_t)n * w2 + e];
    const uint8_t* tile = base + L.off_l2x + ((size_t)(n / 128) * (w2 / 64) + e / 64) * kLRTile;
    return *reinterpret_cast<const uint16_t*>(tile + sw128(n % 128, (e % 64) * 2));
  };
  for (int i = 0; i < r; ++i)
    for (int n = 0; n < N; ++n) {
      double v = bf16_value(at(n, i));
      if (L.nseg == 3) v += bf16_value(at(n, 2 * r + i));
      L2[(size_t)i * N + n] = v;
    }
}

void finish_header(const svdq_params* p, const BlobLayout& L, uint8_t* base) {
  BlobHeader* h = (BlobHeader*)base;
  h->magic0 = kMagic0; h->magic1 = kMagic1; h->version = kVersion; h->header_bytes = (uint32_t)kAlign;
  h->params = *p;
  h->total_bytes = L.total;
  h->off_inv_lambda = L.off_inv_lambda; h->off_l1t = L.off_l1t; h->off_l2x = L.off_l2x;
  h->off_wq = L.off_wq; h->off_ws = L.off_ws; h->off_bias = L.off_bias;
  h->nseg = L.nseg;
  h->checksum = fnv1a(base + kAlign, L.total - kAlign);
}

}  // namespace

// ======================================================================= C ABI
extern "C" {

size_t svdq_blob_bytes(const svdq_params* p) {
  if (check_params(p) != SVDQ_OK) return 0;
  return blob_layout(*p).total;
}

size_t svdq_workspace_bytes(const svdq_params* p, int64_t M) {
  if (check_params(p) != SVDQ_OK || M < 0) return 0;
  return ws_layout(*p, M).total;
}

size_t svdq_chain_workspace_bytes(const svdq_params* p, const svdq_params* p_next, int64_t M) {
  if (check_params(p) != SVDQ_OK || check_params(p_next) != SVDQ_OK || M < 0) return 0;
  if (chain_supported(*p, *p_next) != SVDQ_OK) return 0;
  return chain_layout(*p, *p_next, M).total;
}

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED: return "unsupported";
    case SVDQ_ERR_ALIGNMENT: return "misaligned device pointer";
    case SVDQ_ERR_WORKSPACE: return "workspace too small";
    case SVDQ_ERR_BLOB: return "blob mismatch";
    case SVDQ_ERR_NO_CONVERGENCE: return "SVD did not converge";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

svdq_status svdq_prepare(const svdq_params* p, const float* Wt, const float* bias,
                         const void* X_cal, int64_t M_cal, void* blob, size_t blob_bytes,
                         double* sigma_out) {
  svdq_status st = check_params(p);
  if (st != SVDQ_OK) return st;
  if (!Wt || !blob || M_cal < 0 || (M_cal > 0 && !X_cal)) return SVDQ_ERR_INVALID_ARG;
  const BlobLayout L = blob_layout(*p);
  if (blob_bytes < L.total) return SVDQ_ERR_INVALID_ARG;
  const int K = p->K, N = p->N, r = p->rank, dt = p->act_dtype;
  uint8_t* base = (uint8_t*)blob;
  memset(base, 0, L.total);

  // --- 1. smoothing factors: lambda_j = a_j^alpha / w_j^(1-alpha)
  std::vector<double> a(K, 0.0), w(K, 0.0);
  const uint16_t* xc = (const uint16_t*)X_cal;
  for (int64_t m = 0; m < M_cal; ++m)
    for (int j = 0; j < K; ++j) a[j] = std::max(a[j], fabs(dtype_value(xc[m * K + j], dt)));
  for (int n = 0; n < N; ++n)
    for (int j = 0; j < K; ++j) w[j] = std::max(w[j], fabs((double)Wt[(size_t)n * K + j]));
  float* inv_lambda = (float*)(base + L.off_inv_lambda);
  std::vector<double> lam_eff(K);
  for (int j = 0; j < K; ++j) {
    double lam = 1.0;
    if (p->smooth && a[j] > 0.0 && w[j] > 0.0)
      lam = pow(a[j], (double)p->alpha) / pow(w[j], 1.0 - (double)p->alpha);
    inv_lambda[j] = (float)(1.0 / lam);
    lam_eff[j] = 1.0 / (double)inv_lambda[j];
  }

  // --- 2. smoothed weight, stored transposed: At[n][k] = W^[k][n] = Wt[n][k] * lambda_k
  std::vector<double> At((size_t)N * K);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    for (int j = 0; j < K; ++j) At[(size_t)n * K + j] = (double)Wt[(size_t)n * K + j] * lam_eff[j];

  // --- 3. truncated SVD: At = P S Q^T  =>  W^ = Q S P^T, L1 = Q S (= W^ P), L2 = P^T
  std::vector<double> L1((size_t)K * r, 0.0), L2((size_t)r * N, 0.0);  // dtype values
  if (r > 0) {
    std::vector<double> P, sigma;
    st = truncated_svd(At.data(), N, K, r, 6, P, sigma);
    if (st != SVDQ_OK) return st;
    if (sigma_out) for (int i = 0; i <= r; ++i) sigma_out[i] = sigma[i];
    std::vector<double> L1f((size_t)K * r);
    matmul_tn(At.data(), N, K, P.data(), r, L1f.data());      // L1 = At^T P  (K x r)
    for (size_t i = 0; i < L1f.size(); ++i) L1[i] = dtype_round(L1f[i], dt);
    for (int i = 0; i < r; ++i)
      for (int n = 0; n < N; ++n) L2[(size_t)i * N + n] = dtype_round(P[(size_t)n * r + i], dt);
  } else if (sigma_out) {
    sigma_out[0] = 0.0;
  }

  // --- 4. residual R = W^ - L1 L2 (float64, rank-1 terms in ascending order,
  //        each product rounded then added), rounded to fp32; quantised per
  //        output channel n along K.
  uint8_t* wq = base + L.off_wq;
  uint8_t* wsb = base + L.off_ws;
  (void)wsb;
  std::vector<float> R((size_t)N * K);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    for (int j = 0; j < K; ++j) {
      double s = 0.0;
      for (int i = 0; i < r; ++i) s = s + L1[(size_t)j * r + i] * L2[(size_t)i * N + n];
      R[(size_t)n * K + j] = (float)(At[(size_t)n * K + j] - s);
    }
  At.clear(); At.shrink_to_fit();

  BlobHeader* h = (BlobHeader*)base;
  h->s_gw = 1.0f;
  if (p->fmt == SVDQ_INT4_G64) {
    float* sw = (float*)wsb;                                   // blocked, int4_sw_index
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
      std::vector<int8_t> q(K);
      std::vector<float> s(K / kGroupInt4);
      int4_quant_row(&R[(size_t)n * K], K, q.data(), s.data());
      for (int j = 0; j < K; ++j) wq[(size_t)n * K + j] = e4m3_encode((float)q[j]);
      for (int g = 0; g < K / kGroupInt4; ++g) sw[int4_sw_index(g, n, N)] = s[g];
    }
  } else {
    float amax = 0.0f;
    for (size_t i = 0; i < R.size(); ++i) amax = std::max(amax, fabsf(R[i]));
    const float s_g = nvfp4_tensor_scale(amax);
    h->s_gw = s_g;
    // weight tiles [n/128][slab]: swizzled codes + the scales of the tile's 256-row pair
    const int kb = K / kBlockFp4, ksl = K / 256;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
      std::vector<uint8_t> c(K), e(kb);
      nvfp4_quant_row(&R[(size_t)n * K], K, s_g, c.data(), e.data());
      const int nb = n / 128, rr = n % 128, half = nb & 1, pb = nb & ~1;
      for (int t = 0; t < ksl; ++t) {
        uint8_t* tile = wq + ((size_t)nb * ksl + t) * kWTile;
        for (int cb = 0; cb < 128; ++cb) {
          const int j = t * 256 + 2 * cb;
          tile[sw128(rr, cb)] = (uint8_t)(c[j] | (c[j + 1] << 4));
        }
        for (int b = 0; b < 16; ++b) {
          const uint8_t sc = e[t * 16 + b];
          // both tiles of the pair carry the pair's scales
          for (int q = 0; q < 2; ++q)
            wq[((size_t)(pb + q) * ksl + t) * kWTile + kTileCodes + half * 2048 + tile_sf(rr, b)] = sc;
        }
      }
    }
  }

  // --- 5. static activation tensor scale (NVFP4): amax(fp32(X_cal) * inv_lambda) / 2688
  h->s_gx = 1.0f;
  if (p->fmt == SVDQ_NVFP4) {
    float amax = 0.0f;
    for (int64_t m = 0; m < M_cal; ++m)
      for (int j = 0; j < K; ++j)
        amax = std::max(amax, fabsf((float)dtype_value(xc[m * K + j], dt) * inv_lambda[j]));
    h->s_gx = nvfp4_tensor_scale(amax);
  }

  // --- 6. factors in device layouts
  write_factors(p, L, base, L1.data(), L2.data());
  float* bb = (float*)(base + L.off_bias);
  for (int n = 0; n < N; ++n) bb[n] = bias ? bias[n] : 0.0f;

  // --- 7. header
  finish_header(p, L, base);
  return SVDQ_OK;
}

svdq_status svdq_blob_check(const svdq_params* p, const void* blob, size_t blob_bytes) {
  svdq_status st = check_params(p);
  if (st != SVDQ_OK) return st;
  if (!blob || blob_bytes < sizeof(BlobHeader)) return SVDQ_ERR_BLOB;
  const BlobHeader* h = (const BlobHeader*)blob;
  const BlobLayout L = blob_layout(*p);
  if (h->magic0 != kMagic0 || h->magic1 != kMagic1 || h->version != kVersion) return SVDQ_ERR_BLOB;
  if (memcmp(&h->params, p, sizeof(svdq_params)) != 0) return SVDQ_ERR_BLOB;
  if (h->total_bytes != L.total || blob_bytes < L.total) return SVDQ_ERR_BLOB;
  if (h->off_wq != L.off_wq || h->off_ws != L.off_ws || h->off_bias != L.off_bias) return SVDQ_ERR_BLOB;
  if (fnv1a((const uint8_t*)blob + kAlign, L.total - kAlign) != h->checksum) return SVDQ_ERR_BLOB;
  return SVDQ_OK;
}

svdq_status svdq_blob_export(const svdq_params* p, const void* blob, float* inv_lambda,
                             uint16_t* L1, uint16_t* L2, uint8_t* wcodes, void* wscales,
                             float* tscales, float* bias) {
  svdq_status st = check_params(p);
  if (st != SVDQ_OK) return st;
  if (!blob) return SVDQ_ERR_INVALID_ARG;
  const BlobLayout L = blob_layout(*p);
  const BlobHeader* h = (const BlobHeader*)blob;
  if (h->magic0 != kMagic0 || h->magic1 != kMagic1 || memcmp(&h->params, p, sizeof(svdq_params)))
    return SVDQ_ERR_BLOB;
  const uint8_t* base = (const uint8_t*)blob;
  const int K = p->K, N = p->N, r = p->rank, dt = p->act_dtype;
  if (inv_lambda) memcpy(inv_lambda, base + L.off_inv_lambda, (size_t)K * 4);
  if (L1) {
    const uint16_t* l1t = (const uint16_t*)(base + L.off_l1t);
    for (int j = 0; j < K; ++j)
      for (int i = 0; i < r; ++i) L1[(size_t)j * r + i] = l1t[(size_t)i * K + j];
  }
  if (L2) {
    const uint16_t* l2x = (const uint16_t*)(base + L.off_l2x);
    const int w2 = lr_width(*p);
    auto at = [&](int n, int e) -> uint16_t {
      if (p->fmt != SVDQ_NVFP4) return l2x[(size_t)n * w2 + e];
      const uint8_t* tile = base + L.off_l2x + ((size_t)(n / 128) * (w2 / 64) + e / 64) * kLRTile;
      return *reinterpret_cast<const uint16_t*>(tile + sw128(n % 128, (e % 64) * 2));
    };
    for (int i = 0; i < r; ++i)
      for (int n = 0; n < N; ++n) {
        double v = bf16_value(at(n, i));
        if (L.nseg == 3) v += bf16_value(at(n, 2 * r + i));
        L2[(size_t)i * N + n] = dtype_bits(v, dt);
      }
  }
  const uint8_t* wq = base + L.off_wq;
  const uint8_t* wsb = base + L.off_ws;
  if (wcodes) {
    for (int n = 0; n < N; ++n)
      for (int j = 0; j < K; ++j) {
        if (p->fmt == SVDQ_NVFP4) {
          const uint8_t* tile = wq + ((size_t)(n / 128) * (K / 256) + j / 256) * kWTile;
          const uint8_t byte = tile[sw128(n % 128, (j % 256) / 2)];
          wcodes[(size_t)n * K + j] = (j & 1) ? (byte >> 4) : (byte & 15);
        } else {
          wcodes[(size_t)n * K + j] = (uint8_t)(int8_t)llround(e4m3_value(wq[(size_t)n * K + j]));
        }
      }
  }
  if (wscales) {
    if (p->fmt == SVDQ_NVFP4) {
      uint8_t* o = (uint8_t*)wscales;
      const int kb = K / kBlockFp4;
      for (int n = 0; n < N; ++n)
        for (int b = 0; b < kb; ++b) {
          // read from the tile of the row's own block (its pair partner holds the same bytes)
          const uint8_t* tile = wq + ((size_t)(n / 128) * (K / 256) + b / 16) * kWTile;
          o[(size_t)n * kb + b] = tile[kTileCodes + ((n / 128) & 1) * 2048 + tile_sf(n % 128, b % 16)];
        }
    } else {
      float* o = (float*)wscales;
      const float* sw = (const float*)wsb;
      const int G = K / kGroupInt4;
      for (int n = 0; n < N; ++n)
        for (int g = 0; g < G; ++g) o[(size_t)n * G + g] = sw[int4_sw_index(g, n, N)];
    }
  }
  if (tscales) { tscales[0] = h->s_gx; tscales[1] = h->s_gw; }
  if (bias) memcpy(bias, base + L.off_bias, (size_t)N * 4);
  return SVDQ_OK;
}

svdq_status svdq_shard_columns(const svdq_params* p, const void* blob_in, size_t blob_in_bytes, int32_t n0,
                               int32_t n1, svdq_params* p_out, void* blob_out, size_t blob_out_bytes) {
  svdq_status st = svdq_blob_check(p, blob_in, blob_in_bytes);
  if (st != SVDQ_OK) return st;
  if (!p_out || !blob_out || n0 < 0 || n1 > p->N || n0 >= n1 || n0 % 256 != 0 || n1 % 256 != 0)
    return SVDQ_ERR_INVALID_ARG;
  svdq_params q = *p;
  q.N = n1 - n0;
  const BlobLayout Li = blob_layout(*p), Lo = blob_layout(q);
  if (blob_out_bytes < Lo.total) return SVDQ_ERR_INVALID_ARG;
  const int K = p->K, N = p->N, Ns = q.N;
  const uint8_t* in = (const uint8_t*)blob_in;
  uint8_t* out = (uint8_t*)blob_out;
  memset(out, 0, Lo.total);
  memcpy(out, in, sizeof(BlobHeader));   // tensor scales s_gX, s_gW stay those of the whole layer
  memcpy(out + Lo.off_inv_lambda, in + Li.off_inv_lambda, (size_t)K * 4);
  memcpy(out + Lo.off_l1t, in + Li.off_l1t, (size_t)p->rank * K * 2);
  // every per-column array is ordered by output feature first, so a column
  // range [n0, n1) (whole 256-column tiles) is one contiguous run of each
  const size_t w2 = (size_t)lr_width(*p);
  memcpy(out + Lo.off_l2x, in + Li.off_l2x + (size_t)n0 * w2 * 2, (size_t)Ns * w2 * 2);
  if (p->fmt == SVDQ_NVFP4) {
    const size_t tile_row = (size_t)(K / 256) * kWTile;   // one 128-row block over all K slabs
    memcpy(out + Lo.off_wq, in + Li.off_wq + (size_t)(n0 / 128) * tile_row, (size_t)(Ns / 128) * tile_row);
  } else {
    memcpy(out + Lo.off_wq, in + Li.off_wq + (size_t)n0 * K, (size_t)Ns * K);
    // blocked scales [K/128][N/128][2][128]: one run per 128-wide K slab
    for (int kt = 0; kt < K / 128; ++kt)
      memcpy(out + Lo.off_ws + (size_t)kt * (Ns / 128) * 1024,
             in + Li.off_ws + ((size_t)kt * (N / 128) + n0 / 128) * 1024, (size_t)(Ns / 128) * 1024);
  }
  memcpy(out + Lo.off_bias, in + Li.off_bias + (size_t)n0 * 4, (size_t)Ns * 4);
  finish_header(&q, Lo, out);
  *p_out = q;
  return SVDQ_OK;
}

svdq_status svdq_append_lora(const svdq_params* p, const void* blob_in, size_t blob_in_bytes, const float* A,
                             const float* B, int32_t r_lora, svdq_params* p_out, void* blob_out,
                             size_t blob_out_bytes) {
  svdq_status st = svdq_blob_check(p, blob_in, blob_in_bytes);
  if (st != SVDQ_OK) return st;
  if (!A || !B || !p_out || !blob_out || r_lora <= 0 || r_lora % 16 != 0 || p->rank + r_lora > 128)
    return SVDQ_ERR_INVALID_ARG;
  svdq_params q = *p;
  q.rank = p->rank + r_lora;
  if ((st = check_params(&q)) != SVDQ_OK) return st;
  const BlobLayout Li = blob_layout(*p), Lo = blob_layout(q);
  if (blob_out_bytes < Lo.total) return SVDQ_ERR_INVALID_ARG;
  const int K = p->K, N = p->N, r = p->rank, r2 = q.rank, dt = p->act_dtype;
  const uint8_t* in = (const uint8_t*)blob_in;
  uint8_t* out = (uint8_t*)blob_out;

  // L1' = [L1 | dtype(lambda_eff (.) A)], L2' = [L2 ; dtype(B)], since X A B = X^ (diag(lambda) A) B
  std::vector<double> L1((size_t)K * r), L2((size_t)r * N);
  read_factors(p, Li, in, L1.data(), L2.data());
  const float* inv_lambda = (const float*)(in + Li.off_inv_lambda);
  std::vector<double> L1o((size_t)K * r2), L2o((size_t)r2 * N);
  for (int j = 0; j < K; ++j) {
    const double lam = 1.0 / (double)inv_lambda[j];
    for (int i = 0; i < r; ++i) L1o[(size_t)j * r2 + i] = L1[(size_t)j * r + i];
    for (int i = 0; i < r_lora; ++i)
      L1o[(size_t)j * r2 + r + i] = dtype_round(lam * (double)A[(size_t)j * r_lora + i], dt);
  }
  for (int i = 0; i < r; ++i)
    for (int n = 0; n < N; ++n) L2o[(size_t)i * N + n] = L2[(size_t)i * N + n];
  for (int i = 0; i < r_lora; ++i)
    for (int n = 0; n < N; ++n) L2o[(size_t)(r + i) * N + n] = dtype_round((double)B[(size_t)i * N + n], dt);

  // everything else is carried over unchanged: the residual is not re-quantised
  memset(out, 0, Lo.total);
  memcpy(out, in, sizeof(BlobHeader));
  memcpy(out + Lo.off_inv_lambda, in + Li.off_inv_lambda, (size_t)K * 4);
  memcpy(out + Lo.off_wq, in + Li.off_wq, Li.off_ws - Li.off_wq);
  memcpy(out + Lo.off_ws, in + Li.off_ws, Li.off_bias - Li.off_ws);
  memcpy(out + Lo.off_bias, in + Li.off_bias, (size_t)N * 4);
  write_factors(&q, Lo, out, L1o.data(), L2o.data());
  finish_header(&q, Lo, out);
  *p_out = q;
  return SVDQ_OK;
}

// Host-side decoding of the activation workspace (device copy done by the caller).
svdq_status svdq_decode_act_host(const svdq_params* p, const uint8_t* ws, int64_t M,
                                 uint8_t* codes, void* scales, float* u) {
  svdq_status st = check_params(p);
  if (st != SVDQ_OK) return st;
  const WsLayout W = ws_layout(*p, M);
  const int K = p->K, r = p->rank, w2 = lr_width(*p);
  if (codes) {
    for (int64_t m = 0; m < M; ++m)
      for (int j = 0; j < K; ++j) {
        if (p->fmt == SVDQ_NVFP4) {
          const uint8_t* tile = ws + W.off_xq + ((size_t)(m / 128) * (K / 256) + j / 256) * kATile;
          const uint8_t byte = tile[sw128((uint32_t)(m % 128), (j % 256) / 2)];
          codes[(size_t)m * K + j] = (j & 1) ? (byte >> 4) : (byte & 15);
        } else {
          codes[(size_t)m * K + j] = (uint8_t)(int8_t)llround(e4m3_value(ws[W.off_xq + (size_t)m * K + j]));
        }
      }
  }
  if (scales) {
    if (p->fmt == SVDQ_NVFP4) {
      uint8_t* o = (uint8_t*)scales;
      const int kb = K / kBlockFp4;
      for (int64_t m = 0; m < M; ++m)
        for (int b = 0; b < kb; ++b) {
          const uint8_t* tile = ws + W.off_xq + ((size_t)(m / 128) * (K / 256) + b / 16) * kATile;
          o[(size_t)m * kb + b] = tile[kTileCodes + tile_sf((uint32_t)(m % 128), b % 16)];
        }
    } else {
      float* o = (float*)scales;
      const float* sx = (const float*)(ws + W.off_xs);
      const int G = K / kGroupInt4;
      for (int64_t m = 0; m < M; ++m)
        for (int g = 0; g < G; ++g) o[(size_t)m * G + g] = sx[int4_sx_index(g, m, W.Mp)];
    }
  }
  if (u) {
    const uint16_t* ux = (const uint16_t*)(ws + W.off_ux);
    auto at = [&](int64_t m, int e) -> uint16_t {
      if (p->fmt != SVDQ_NVFP4) return ux[(size_t)m * w2 + e];
      const uint8_t* tile = ws + W.off_ux + ((size_t)(m / 128) * (w2 / 64) + e / 64) * kLRTile;
      return *reinterpret_cast<const uint16_t*>(tile + sw128((uint32_t)(m % 128), (e % 64) * 2));
    };
    for (int64_t m = 0; m < M; ++m)
      for (int i = 0; i < r; ++i)
        u[(size_t)m * r + i] = (float)(bf16_value(at(m, i)) + bf16_value(at(m, r + i)));
  }
  return SVDQ_OK;
}

}  // extern "C"
