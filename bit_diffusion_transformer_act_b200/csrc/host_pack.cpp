// Host side of libsvdq: status strings, sizes, the weight packer and the
// scale-layout helpers.  No CUDA here.
//
// The packer quantizes the residual R to NVFP4 ("Nunchaku Lite", section
// "Supported quantization types": svdq_w4a4 / nvfp4 / group 16):
//   g_w = smallest power of two with g_w * 6 * 448 >= amax(R)  (1 if R == 0)
//   S   = RNE onto E4M3 of amax_block / (6 g_w), saturating at 448
//   c   = RNE onto E2M1 of clamp(x / (S g_w), -6, 6), sign kept; 0 if S == 0
// All quotients are taken in double precision.  Their inputs have at most 24
// significant bits and S g_w at most 4, so a quotient that is not exactly on a
// rounding midpoint is at least 2^-24 (relative) away from it, while double
// rounding errs by 2^-53: the decisions equal those of exact arithmetic.

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "../../include/svdq.h"
#include "layout.h"

namespace {

// E4M3 (FN) code of a non-negative finite double, round to nearest even,
// saturating at 448 (0x7E).
uint8_t e4m3_code_rne(double v) {
  if (!(v > 0.0)) return 0;
  if (v >= 448.0) return 0x7E;
  if (v < std::ldexp(1.0, -6)) {                  // subnormal range: units of 2^-9
    const double q = std::nearbyint(std::ldexp(v, 9));   // FE_TONEAREST: ties to even
    return static_cast<uint8_t>(q);               // q == 8 is the smallest normal, code 0x08
  }
  int e2;
  (void)std::frexp(v, &e2);                       // v = f 2^e2, f in [0.5, 1)
  int E = e2 - 1;                                 // v in [2^E, 2^(E+1))
  double q = std::nearbyint(std::ldexp(v, 3 - E));  // in [8, 16]
  if (q == 16.0) { q = 8.0; ++E; }
  const int field = E + 7;
  if (field > 15 || (field == 15 && q - 8.0 >= 7.0)) return 0x7E;
  return static_cast<uint8_t>((field << 3) | static_cast<int>(q - 8.0));
}

double e4m3_value(uint8_t code) {
  const int e = (code >> 3) & 0xF, m = code & 7;
  if (e == 0) return std::ldexp(static_cast<double>(m), -9);
  return std::ldexp(1.0 + m / 8.0, e - 7);
}

// E2M1 magnitude code of |v| clamped to 6, ties to the even code, by
// comparison with the midpoints of the grid {0, .5, 1, 1.5, 2, 3, 4, 6}.
uint8_t e2m1_code_rne(double v) {
  const double a = std::fmin(std::fabs(v), 6.0);
  uint8_t c;
  if (a <= 0.25) c = 0;          // tie 0.25 -> code 0
  else if (a < 0.75) c = 1;      // tie 0.75 -> code 2
  else if (a <= 1.25) c = 2;     // tie 1.25 -> code 2
  else if (a < 1.75) c = 3;      // tie 1.75 -> code 4
  else if (a <= 2.5) c = 4;      // tie 2.5  -> code 4
  else if (a < 3.5) c = 5;       // tie 3.5  -> code 6
  else if (a <= 5.0) c = 6;      // tie 5    -> code 6
  else c = 7;
  return static_cast<uint8_t>(c | (std::signbit(v) ? 8 : 0));
}

double pow2_global_scale(double amax) {
  if (amax == 0.0) return 1.0;
  const double limit = 6.0 * 448.0;
  int e;
  (void)std::frexp(amax / limit, &e);
  double g = std::ldexp(1.0, e);
  while (g * limit < amax) g *= 2.0;
  while ((g * 0.5) * limit >= amax) g *= 0.5;
  return g;
}

// bf16 nearest (ties to even) to a double, rounded once (8 significant bits, bf16 subnormal
// steps of 2^-133); finite inputs.
uint16_t double_to_bf16_rne(double v) {
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  const double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e;
  (void)std::frexp(a, &e);
  const int step = std::max(e - 8, -133);
  const double r = std::ldexp(std::nearbyint(std::ldexp(a, -step)), step);
  const float f = static_cast<float>(r);            // exact (or infinity)
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(sign | (u >> 16));
}

float bf16_to_float(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t float_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);   // finite inputs only
  return static_cast<uint16_t>(u >> 16);
}

}  // namespace

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SVDQ_ERR_ARCH: return "device is not sm_100 (B200)";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "kernel wait timed out";
    case SVDQ_ERR_SCALE_RANGE: return "device-side scale product out of range (clamped)";
    default: return "unknown status";
  }
}

int svdq_abi_version(void) { return svdq::kAbiVersion; }

size_t svdq_packed_weight_bytes(int N, int K, int rank) {
  if (N <= 0 || K <= 0 || N % 64 != 0 || K % 64 != 0 || rank != svdq::kRank) return 0;
  return svdq::blob_layout(N, K, rank).total;
}

size_t svdq_act_scale_bytes(int M, int K) {
  if (M < 0 || K <= 0 || K % 64 != 0) return 0;
  return svdq::swizzled_scale_bytes(static_cast<size_t>(M), static_cast<size_t>(K));
}

int svdq_pack_weights(const float* R, const uint16_t* L1, const uint16_t* L2,
                      const uint16_t* bias, const uint16_t* smooth_inv, int N, int K, int rank,
                      void* out, size_t out_bytes, float* w_global_scale) {
  if (!R || !L1 || !L2 || !smooth_inv || !out || !w_global_scale) return SVDQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || N % 64 != 0 || K % 64 != 0 || rank != svdq::kRank)
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  const svdq::BlobLayout L = svdq::blob_layout(N, K, rank);
  if (out_bytes < L.total) return SVDQ_ERR_INVALID_ARG;

  const size_t n = static_cast<size_t>(N), k = static_cast<size_t>(K);
  double amax = 0.0;
  for (size_t i = 0; i < n * k; ++i) {
    const double a = std::fabs(static_cast<double>(R[i]));
    if (!std::isfinite(a)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    if (a > amax) amax = a;
  }
  const double g = pow2_global_scale(amax);

  uint8_t* blob = static_cast<uint8_t*>(out);
  std::memset(blob, 0, L.total);

  uint8_t* codes = blob + L.codes;
  uint8_t* scales = blob + L.scales;
  const size_t groups = k / 16;
  for (size_t row = 0; row < n; ++row) {
    const float* x = R + row * k;
    for (size_t gi = 0; gi < groups; ++gi) {
      double bmax = 0.0;
      for (int t = 0; t < 16; ++t) bmax = std::fmax(bmax, std::fabs(static_cast<double>(x[gi * 16 + t])));
      const uint8_t s = e4m3_code_rne(bmax / (6.0 * g));
      scales[svdq::swizzled_scale_offset(row, gi, k)] = s;
      const double Sg = e4m3_value(s) * g;
      for (int t = 0; t < 16; t += 2) {
        uint8_t c0 = 0, c1 = 0;
        if (s != 0) {
          c0 = e2m1_code_rne(static_cast<double>(x[gi * 16 + t]) / Sg);
          c1 = e2m1_code_rne(static_cast<double>(x[gi * 16 + t + 1]) / Sg);
        }
        codes[row * (k / 2) + (gi * 16 + t) / 2] = static_cast<uint8_t>(c0 | (c1 << 4));
      }
    }
  }

  // smooth_inv[k] * L1[k][j] is a product of two bf16 values (at most 16 significant
  // bits, exact in float); it splits exactly into hi = RN_bf16(p) and lo = p - hi.
  uint16_t* l1s_hi = reinterpret_cast<uint16_t*>(blob + L.l1s);
  uint16_t* l1s_lo = l1s_hi + static_cast<size_t>(rank) * k;
  for (size_t j = 0; j < static_cast<size_t>(rank); ++j)
    for (size_t kk = 0; kk < k; ++kk) {
      const float prod = bf16_to_float(smooth_inv[kk]) * bf16_to_float(L1[kk * rank + j]);
      const uint16_t hi = float_to_bf16_rne(prod);
      l1s_hi[j * k + kk] = hi;
      l1s_lo[j * k + kk] = float_to_bf16_rne(prod - bf16_to_float(hi));
    }
  // L2 / g_w: g_w is a power of two, so the division only moves the exponent.
  uint16_t* l2t = reinterpret_cast<uint16_t*>(blob + L.l2t);
  for (size_t row = 0; row < n; ++row)
    for (size_t j = 0; j < static_cast<size_t>(rank); ++j)
      l2t[row * rank + j] = float_to_bf16_rne(static_cast<float>(bf16_to_float(L2[j * n + row]) / g));
  if (bias) std::memcpy(blob + L.bias, bias, n * 2);

  svdq::BlobHeader h;
  std::memset(&h, 0, sizeof(h));
  std::memcpy(h.magic, "SVDQNVF4", 8);
  h.abi_version = svdq::kAbiVersion;
  h.N = N; h.K = K; h.rank = rank;
  h.w_global_scale = static_cast<float>(g);
  std::memcpy(blob, &h, sizeof(h));
  *w_global_scale = static_cast<float>(g);
  return SVDQ_OK;
}

size_t svdq_int4_packed_weight_bytes(int N, int K, int rank) {
  if (N <= 0 || K <= 0 || N % 128 != 0 || K % 64 != 0 || rank != svdq::kRank) return 0;
  return svdq::blob_layout_int4(N, K, rank).total;
}

int svdq_int4_pack_weights(const float* R, const uint16_t* L1, const uint16_t* L2, const uint16_t* bias,
                           const uint16_t* smooth_inv, int N, int K, int rank, void* out, size_t out_bytes) {
  if (!R || !L1 || !L2 || !smooth_inv || !out) return SVDQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || N % 128 != 0 || K % 64 != 0 || rank != svdq::kRank) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  const svdq::BlobLayout L = svdq::blob_layout_int4(N, K, rank);
  if (out_bytes < L.total) return SVDQ_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(N), k = static_cast<size_t>(K);
  for (size_t i = 0; i < n * k; ++i)
    if (!std::isfinite(R[i])) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  uint8_t* blob = static_cast<uint8_t*>(out);
  std::memset(blob, 0, L.total);
  uint8_t* codes = blob + L.codes;
  float* scales = reinterpret_cast<float*>(blob + L.scales);       // [K/64][N]
  // per (row, 64-group): s = RNE_bf16(amax / 7) rounded once from the double quotient (amax has
  // at most 24 significant bits, 7 three: a quotient on a bf16 midpoint is exact in double, one
  // off it is far more than double's error away); c = clamp(RNE(x / s), -8, 7), by the same
  // argument decided exactly; c stored as its E4M3 byte
  for (size_t row = 0; row < n; ++row) {
    const float* x = R + row * k;
    for (size_t gi = 0; gi < k / 64; ++gi) {
      double amax = 0.0;
      for (int t = 0; t < 64; ++t) amax = std::fmax(amax, std::fabs(static_cast<double>(x[gi * 64 + t])));
      const uint16_t sb = double_to_bf16_rne(amax / 7.0);
      scales[gi * n + row] = bf16_to_float(sb);
      const double s = bf16_to_float(sb);
      for (int t = 0; t < 64; ++t) {
        double c = 0.0;
        if (s != 0.0) c = std::fmin(7.0, std::fmax(-8.0, std::nearbyint(static_cast<double>(x[gi * 64 + t]) / s)));
        const uint8_t mag = e4m3_code_rne(std::fabs(c));      // integers up to 8 are exact in E4M3
        codes[row * k + gi * 64 + t] = static_cast<uint8_t>(mag | (c < 0.0 ? 0x80 : 0));
      }
    }
  }
  uint16_t* l1s_hi = reinterpret_cast<uint16_t*>(blob + L.l1s);
  uint16_t* l1s_lo = l1s_hi + static_cast<size_t>(rank) * k;
  for (size_t j = 0; j < static_cast<size_t>(rank); ++j)
    for (size_t kk = 0; kk < k; ++kk) {
      const float prod = bf16_to_float(smooth_inv[kk]) * bf16_to_float(L1[kk * rank + j]);
      const uint16_t hi = float_to_bf16_rne(prod);
      l1s_hi[j * k + kk] = hi;
      l1s_lo[j * k + kk] = float_to_bf16_rne(prod - bf16_to_float(hi));
    }
  uint16_t* l2t = reinterpret_cast<uint16_t*>(blob + L.l2t);
  for (size_t row = 0; row < n; ++row)
    for (size_t j = 0; j < static_cast<size_t>(rank); ++j) l2t[row * rank + j] = L2[j * n + row];
  if (bias) std::memcpy(blob + L.bias, bias, n * 2);
  svdq::BlobHeader h;
  std::memset(&h, 0, sizeof(h));
  std::memcpy(h.magic, "SVDQINT4", 8);
  h.abi_version = svdq::kAbiVersion;
  h.N = N; h.K = K; h.rank = rank;
  h.w_global_scale = 1.0f;
  std::memcpy(blob, &h, sizeof(h));
  return SVDQ_OK;
}

int svdq_unswizzle_scales(const void* swizzled, int rows, int K, uint8_t* out) {
  if (!swizzled || !out || rows < 0 || K <= 0 || K % 64 != 0) return SVDQ_ERR_INVALID_ARG;
  const uint8_t* s = static_cast<const uint8_t*>(swizzled);
  const size_t groups = static_cast<size_t>(K) / 16;
  for (size_t r = 0; r < static_cast<size_t>(rows); ++r)
    for (size_t gi = 0; gi < groups; ++gi)
      out[r * groups + gi] = s[svdq::swizzled_scale_offset(r, gi, K)];
  return SVDQ_OK;
}

int svdq_swizzle_scales(const uint8_t* plain, int rows, int K, void* swizzled) {
  if (!plain || !swizzled || rows < 0 || K <= 0 || K % 64 != 0) return SVDQ_ERR_INVALID_ARG;
  uint8_t* s = static_cast<uint8_t*>(swizzled);
  std::memset(s, 0, svdq::swizzled_scale_bytes(rows, K));
  const size_t groups = static_cast<size_t>(K) / 16;
  for (size_t r = 0; r < static_cast<size_t>(rows); ++r)
    for (size_t gi = 0; gi < groups; ++gi)
      s[svdq::swizzled_scale_offset(r, gi, K)] = plain[r * groups + gi];
  return SVDQ_OK;
}

}  // extern "C"
