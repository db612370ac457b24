// any4_quantize: the any4 quantizer (group scaling + per-row weighted
// k-means) on the GPU, one warp per row.
//
// Method (any4 explainer, 10100.com article 149119421):
//  * section 2.1, group scaling: each row is cut into contiguous groups of G
//    columns; per group alpha and beta map the weights into the quantizable
//    range. Read as asymmetric min-max onto the signed b-bit map
//    [-2^(b-1), 2^(b-1)-1]: alpha = (max - min) / (2^b - 1), beta = min +
//    2^(b-1) * alpha, both rounded to bf16 and used rounded; w_s = (w - beta)
//    / alpha (0 for a constant group).
//  * section 2.1, calibration: E|x| per input channel (an input here).
//  * section 2.2, weighted k-means per row: E-step = nearest table value
//    (lowest index on ties); M-step LUT_q = sum(c * w_s) / sum(c) over the
//    weights assigned to q with c = alpha * E|x|, evaluated as LUT_q +
//    sum(c * (w_s - LUT_q)) / sum(c); an empty cluster keeps its value.
//    Start: the row's sorted distinct w_s values when there are at most 2^b
//    of them (the last repeated), else the integer map. After the rounds the
//    table is rounded to bf16 and a last E-step runs against it.
// Every double operation is written with an explicit round-to-nearest
// intrinsic in a fixed order (no contraction into fused multiply-adds), and
// each cluster sum runs over the row's columns in increasing order (one lane
// per cluster folds the staged terms), so the result is a deterministic
// function of the inputs, the same as a sequential evaluation.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/any4.h"
#include "kernels.cuh"

namespace any4 {

namespace {

constexpr int kQuantWarps = 8;     // rows per block, one warp each
constexpr int kQuantChunk = 256;   // columns whose M-step terms are staged per fold

// double -> bf16 bits, round to nearest even (normal, subnormal, zero; the
// values here are finite)
__device__ uint16_t d2bf16(double v) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  const uint16_t sign = (uint16_t)((u >> 63) << 15);
  const int exp = (int)((u >> 52) & 0x7FF);
  unsigned long long mant = u & ((1ull << 52) - 1);
  if (exp == 0) return sign;   // zero or a double subnormal (far below bf16 range)
  int e = exp - 1023 + 127;    // bf16 biased exponent
  mant |= 1ull << 52;          // explicit leading one
  int shift = 45;              // keep 8 significant bits (1 + 7)
  if (e <= 0) {                // bf16 subnormal: fewer bits survive
    shift += 1 - e;
    e = 0;
    if (shift > 60) return sign;
  }
  unsigned long long keep = mant >> shift;
  const unsigned long long rest = mant & ((1ull << shift) - 1);
  const unsigned long long half = 1ull << (shift - 1);
  if (rest > half || (rest == half && (keep & 1))) ++keep;
  // keep holds the significand with its leading one at bit 7 (normal) or
  // below (subnormal); a carry into bit 8 bumps the exponent
  uint32_t bits;
  if (e == 0) {
    bits = (uint32_t)keep;                       // subnormal (or rounded up to the smallest normal)
  } else {
    if (keep >> 8) {
      keep >>= 1;
      ++e;
    }
    bits = ((uint32_t)e << 7) | (uint32_t)(keep & 0x7F);
  }
  return (uint16_t)(sign | bits);
}

__device__ __forceinline__ double bf2d(uint16_t b) {
  return (double)__uint_as_float((uint32_t)b << 16);
}

// One warp per row. Everything per column (scaling, the E-step, the M-step
// terms) runs on the warp's lanes in parallel; the cluster sums, whose
// floating-point result depends on their order, are folded in increasing
// column order by one lane per cluster from a shared-memory stage of the
// terms, so the result equals the sequential definition bit for bit.
template <int BITS>
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_kernel(const uint16_t* __restrict__ w, const double* __restrict__ ex, int n, int k,
                    int g, int iters, uint8_t* __restrict__ idx_nib, uint16_t* __restrict__ lut_out,
                    uint16_t* __restrict__ alpha, uint16_t* __restrict__ beta) {
  constexpr int size = 1 << BITS;
  __shared__ double s_term[kQuantWarps][kQuantChunk];
  __shared__ double s_c[kQuantWarps][kQuantChunk];
  __shared__ uint8_t s_q[kQuantWarps][kQuantChunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kQuantWarps + warp;
  if (r >= n) return;   // the whole warp
  const int groups = k / g;
  const double levels = (double)(size - 1), half = (double)(size / 2);
  const uint16_t* wr = w + (size_t)r * k;
  uint16_t* ar = alpha + (size_t)r * groups;
  uint16_t* br = beta + (size_t)r * groups;

  // ---- group scaling: one lane per group, its columns in order
  for (int gi = lane; gi < groups; gi += 32) {
    double lo = bf2d(wr[gi * g]), hi = lo;
    for (int j = 1; j < g; ++j) {
      const double v = bf2d(wr[gi * g + j]);
      lo = v < lo ? v : lo;
      hi = v > hi ? v : hi;
    }
    const uint16_t a = d2bf16(__ddiv_rn(__dsub_rn(hi, lo), levels));
    const uint16_t b = d2bf16(__dadd_rn(lo, __dmul_rn(half, bf2d(a))));
    ar[gi] = a;
    br[gi] = b;
  }
  __syncwarp();
  auto scaled = [&](int col, double& a_out) {
    const int gi = col / g;
    const double a = bf2d(ar[gi]);
    a_out = a;
    if (a == 0.0) return 0.0;
    return __ddiv_rn(__dsub_rn(bf2d(wr[col]), bf2d(br[gi])), a);
  };

  // ---- starting table (lane 0): the distinct scaled values if few enough,
  // else the grid
  double lut[size];
  {
    double mine[size];
    if (lane == 0) {
      double uniq[size + 1];
      int nu = 0;
      bool many = false;
      for (int col = 0; col < k && !many; ++col) {
        double a;
        const double v = scaled(col, a);
        int pos = 0;
        while (pos < nu && uniq[pos] < v) ++pos;
        if (pos < nu && uniq[pos] == v) continue;
        if (nu == size) {
          many = true;
          break;
        }
        for (int i = nu; i > pos; --i) uniq[i] = uniq[i - 1];
        uniq[pos] = v;
        ++nu;
      }
#pragma unroll
      for (int q = 0; q < size; ++q) mine[q] = many ? (double)(q - size / 2) : uniq[q < nu ? q : nu - 1];
    }
#pragma unroll
    for (int q = 0; q < size; ++q) lut[q] = __shfl_sync(0xffffffffu, mine[q], 0);
  }

  auto nearest = [&](double v) {
    int best = 0;
    double bd = fabs(__dsub_rn(v, lut[0]));
#pragma unroll
    for (int q = 1; q < size; ++q) {
      const double d = fabs(__dsub_rn(v, lut[q]));
      if (d < bd) {
        bd = d;
        best = q;
      }
    }
    return best;
  };

  // ---- weighted k-means rounds
  for (int it = 0; it < iters; ++it) {
    double num = 0.0, den = 0.0;   // lane q < size: cluster q
    for (int c0 = 0; c0 < k; c0 += kQuantChunk) {
      const int len = min(kQuantChunk, k - c0);
      for (int j = lane; j < len; j += 32) {
        double a;
        const double v = scaled(c0 + j, a);
        const double c = __dmul_rn(a, ex[c0 + j]);
        const int q = nearest(v);
        double lq = lut[0];
#pragma unroll
        for (int i = 1; i < size; ++i) lq = q == i ? lut[i] : lq;
        s_term[warp][j] = __dmul_rn(c, __dsub_rn(v, lq));
        s_c[warp][j] = c;
        s_q[warp][j] = (uint8_t)q;
      }
      __syncwarp();
      if (lane < size) {
        for (int j = 0; j < len; ++j) {
          if (s_q[warp][j] == lane) {
            num = __dadd_rn(num, s_term[warp][j]);
            den = __dadd_rn(den, s_c[warp][j]);
          }
        }
      }
      __syncwarp();
    }
    double cur = lut[0];
#pragma unroll
    for (int i = 1; i < size; ++i) cur = lane == i ? lut[i] : cur;
    const double upd = (lane < size && den > 0.0) ? __dadd_rn(cur, __ddiv_rn(num, den)) : cur;
#pragma unroll
    for (int q = 0; q < size; ++q) lut[q] = __shfl_sync(0xffffffffu, upd, q);
  }

  // ---- store the bf16 table (padded to 16) and assign against it
  uint16_t lb[size];
#pragma unroll
  for (int q = 0; q < size; ++q) {
    lb[q] = d2bf16(lut[q]);
    lut[q] = bf2d(lb[q]);
  }
  if (lane < 16) {
    uint16_t v = lb[size - 1];
#pragma unroll
    for (int q = 0; q < size; ++q) v = lane == q ? lb[q] : v;
    lut_out[(size_t)r * 16 + lane] = v;
  }
  uint8_t* ir = idx_nib + (size_t)r * (k / 2);
  for (int col = 2 * lane; col < k; col += 64) {
    double a;
    const int q0 = nearest(scaled(col, a));
    const int q1 = nearest(scaled(col + 1, a));
    ir[col / 2] = (uint8_t)(q0 | (q1 << 4));
  }
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* w, const double* ex, int n, int k, int g, int bits,
                            int iters, uint8_t* idx_nib, uint16_t* lut, uint16_t* alpha,
                            uint16_t* beta, cudaStream_t stream) {
  const int blocks = (n + kQuantWarps - 1) / kQuantWarps;
  if (bits == 4)
    quantize_kernel<4><<<blocks, kQuantWarps * 32, 0, stream>>>(w, ex, n, k, g, iters, idx_nib, lut, alpha, beta);
  else if (bits == 3)
    quantize_kernel<3><<<blocks, kQuantWarps * 32, 0, stream>>>(w, ex, n, k, g, iters, idx_nib, lut, alpha, beta);
  else
    quantize_kernel<2><<<blocks, kQuantWarps * 32, 0, stream>>>(w, ex, n, k, g, iters, idx_nib, lut, alpha, beta);
  return cudaGetLastError();
}

}  // namespace any4

extern "C" {

ANY4_API int any4_quantize(const uint16_t* w, const double* ex, int n, int k, int group, int bits,
                           int iters, uint8_t* idx_nib, uint16_t* lut, uint16_t* alpha,
                           uint16_t* beta, any4_stream_t stream) {
  if (!w || !ex || !idx_nib || !lut || !alpha || !beta) return ANY4_EINVAL;
  if (bits < 2 || bits > 4 || iters < 0 || iters > 1000) return ANY4_EINVAL;
  if (!any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  const cudaError_t e = any4::launch_quantize(w, ex, n, k, group, bits, iters, idx_nib, lut, alpha,
                                              beta, (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : any4::record_cuda_error(e);
}

}  // extern "C"
