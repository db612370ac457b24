// Fixed-table 4-bit formats through the any4 kernels.
//
// The any4 explainer's comparison table (10100.com, article 149119421,
// section 1) sets any4 against int4 (uniform scaling with the integer map
// -8..7), NF4 (a fixed table of 16 Gaussian-fitted values) and FP4. Each is a
// 16-entry table shared by every row, so a weight in one of these formats is
// an any4 weight whose per-row tables are all the same: it is packed with the
// format's table and runs through the same dequant and linear kernels.
//
// The tables are built here on the host from their definitions:
//  * int4: -8, -7, ..., 7;
//  * NF4: the normal-quantile construction of the 4-bit NormalFloat type
//    (8 positive and 7 negative quantiles of the standard normal at evenly
//    spaced probabilities up to 1 - delta, delta = (1/32 + 1/30) / 2, plus an
//    exact 0, divided by the largest magnitude), quantiles found by bisection
//    on the normal CDF 0.5 * erfc(-x / sqrt 2);
//  * FP4: the E2M1 element type (sign bit, 2 exponent bits with bias 1, 1
//    mantissa bit; exponent 0 is subnormal), code 8 being -0.
// Every value is rounded once from double to bf16, nearest-even.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/any4.h"
#include "kernels.cuh"

namespace {

uint16_t double_to_bf16(double v) {
  uint64_t u;
  std::memcpy(&u, &v, sizeof u);
  const uint16_t sign = (uint16_t)((u >> 63) << 15);
  const int exp = (int)((u >> 52) & 0x7FF);
  if (exp == 0) return sign;   // zero (the tables hold no subnormal doubles)
  const uint64_t mant = u & ((1ull << 52) - 1);
  // bf16 keeps the top 7 mantissa bits; round the other 45 to nearest-even
  uint64_t keep = mant >> 45;
  const uint64_t rest = mant & ((1ull << 45) - 1);
  const uint64_t half = 1ull << 44;
  int e = exp - 1023 + 127;
  if (rest > half || (rest == half && (keep & 1))) {
    if (++keep == 128) {
      keep = 0;
      ++e;
    }
  }
  return (uint16_t)(sign | (uint16_t)(e << 7) | (uint16_t)keep);
}

double normal_quantile(double p) {
  double lo = -12.0, hi = 12.0;
  for (int i = 0; i < 200 && hi - lo > 0.0; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p) lo = mid;
    else hi = mid;
  }
  return 0.5 * (lo + hi);
}

void nf4_levels(double (&v)[16]) {
  const double delta = 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
  const double top = 1.0 - delta;
  int n = 0;
  for (int j = 7; j >= 1; --j) v[n++] = -normal_quantile(0.5 + j * (top - 0.5) / 7.0);
  v[n++] = 0.0;
  for (int i = 1; i <= 8; ++i) v[n++] = normal_quantile(0.5 + i * (top - 0.5) / 8.0);
  const double m = v[15] > -v[0] ? v[15] : -v[0];
  for (double& x : v) x /= m;
}

}  // namespace

namespace any4 {

bool format_table(int format, uint16_t (&lut)[16]) {
  double v[16];
  switch (format) {
    case ANY4_FORMAT_INT4:
      for (int q = 0; q < 16; ++q) v[q] = q - 8;
      break;
    case ANY4_FORMAT_NF4:
      nf4_levels(v);
      break;
    case ANY4_FORMAT_FP4:
      for (int q = 0; q < 16; ++q) {
        const int e = (q >> 1) & 3, m = q & 1;
        const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
        v[q] = (q & 8) ? -mag : mag;
      }
      v[8] = -0.0;
      break;
    default:
      return false;
  }
  for (int q = 0; q < 16; ++q) lut[q] = double_to_bf16(v[q]);
  return true;
}

}  // namespace any4

namespace {
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
}  // namespace

extern "C" {

ANY4_API int any4_format_lut(int format, uint16_t* lut) {
  if (!lut) return ANY4_EINVAL;
  uint16_t t[16];
  if (!any4::format_table(format, t)) return ANY4_EINVAL;
  for (int q = 0; q < 16; ++q) lut[q] = t[q];
  return ANY4_OK;
}

ANY4_API int any4_pack_format(int format, const uint8_t* idx_nib, const uint16_t* alpha,
                              const uint16_t* beta, int n, int k, int group, void* packed,
                              size_t packed_bytes, any4_stream_t stream) {
  if (!idx_nib || !alpha || !beta || !packed) return ANY4_EINVAL;
  uint16_t t[16];
  if (!any4::format_table(format, t)) return ANY4_EINVAL;
  if (!any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  if (!aligned16(packed)) return ANY4_EALIGN;
  const any4::Layout L = any4::make_layout(n, k, group);
  if (packed_bytes < L.total) return ANY4_EWORKSPACE;
  const cudaError_t e = any4::launch_pack_fixed(idx_nib, t, alpha, beta, L,
                                                static_cast<uint8_t*>(packed),
                                                (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : any4::record_cuda_error(e);
}

}  // extern "C"
