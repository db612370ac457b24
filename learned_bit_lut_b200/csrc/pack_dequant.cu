// any4_pack and any4_dequant kernels.
//
// Pack reorders the canonical tensors (per-row 4-bit indices, per-row 16-entry
// bf16 table, per-group bf16 scale and offset; any4 explainer, 10100.com
// article 149119421, sections 2 and 2.1) into the device layout of layout.cuh
// (the "weights pre-arranged in the compute format" of section 3). Rows past N
// (padding up to a multiple of 128) are written as zeros.
// Dequant reads that layout back and evaluates w_hat = fma(alpha, LUT[idx],
// beta) in fp32, rounded to bf16: the bit-exact debug view of the weights.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace any4 {

// One thread per 16 output bytes: 32 indices of one row.
__global__ void pack_weights_kernel(const uint8_t* __restrict__ idx_nib, Layout L,
                                    uint4* __restrict__ out) {
  const size_t total = (size_t)L.n_pad * L.k / 32;
  const size_t row_bytes = (size_t)L.k / 2;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int lane = (int)(e & 31);
    const int half = (int)((e >> 5) & 1);
    const int quarter = (int)((e >> 6) & 3);
    const size_t unit = e >> 8;
    const size_t tile = unit / L.chunks;
    const int chunk = (int)(unit - tile * L.chunks);
    const size_t row = tile * kTileRows + quarter * 32 + lane;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (row < (size_t)L.n) {
      const uint8_t* src = idx_nib + row * row_bytes + (size_t)chunk * (kChunkK / 2) + half * 16;
#pragma unroll
      for (int b = 0; b < 16; ++b) w[b >> 2] |= (uint32_t)src[b] << (8 * (b & 3));
    }
    out[e] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__global__ void pack_lut_kernel(const uint16_t* __restrict__ lut, Layout L,
                                uint16_t* __restrict__ out) {
  const size_t total = (size_t)L.n_pad * 16;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x)
    out[e] = e < (size_t)L.n * 16 ? lut[e] : (uint16_t)0;
}

__global__ void pack_scales_kernel(const uint16_t* __restrict__ alpha,
                                   const uint16_t* __restrict__ beta, Layout L,
                                   uint32_t* __restrict__ out) {
  const size_t total = (size_t)L.n_pad * L.groups;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(e % kTileRows);
    const size_t tg = e / kTileRows;
    const int grp = (int)(tg % L.groups);
    const size_t tile = tg / L.groups;
    const size_t row = tile * kTileRows + r;
    out[e] = row < (size_t)L.n ? ((uint32_t)alpha[row * L.groups + grp] |
                                  ((uint32_t)beta[row * L.groups + grp] << 16))
                               : 0u;
  }
}

// One thread per packed 32-bit word: 8 consecutive columns of one row.
__global__ void dequant_kernel(const uint8_t* __restrict__ packed, Layout L,
                               uint16_t* __restrict__ w) {
  const uint32_t* words = reinterpret_cast<const uint32_t*>(packed + L.w_off);
  const uint16_t* lutsec = reinterpret_cast<const uint16_t*>(packed + L.lut_off);
  const uint32_t* ab = reinterpret_cast<const uint32_t*>(packed + L.ab_off);
  const size_t total = (size_t)L.n * L.k / 8;
  const int words_per_row = L.k / 8;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t row = e / words_per_row;
    const int wi = (int)(e - row * words_per_row);      // word within the row
    const int col0 = wi * 8;
    const size_t tile = row / kTileRows;
    const int r = (int)(row - tile * kTileRows);
    const int chunk = col0 / kChunkK;
    const int in_chunk = col0 - chunk * kChunkK;         // 0, 8, ..., 56
    const int half = in_chunk / 32;
    const int word_in_16 = (in_chunk % 32) / 8;
    const size_t off = (tile * L.chunks + chunk) * (size_t)kUnitBytes + (r / 32) * 1024 +
                       half * 512 + (r % 32) * 16 + word_in_16 * 4;
    const uint32_t word = words[off / 4];
    const uint32_t s = ab[(tile * L.groups + col0 / L.g) * kTileRows + r];
    const float a = bf16_bits_to_float(s & 0xFFFF);
    const float b = bf16_bits_to_float(s >> 16);
    for (int i = 0; i < 8; ++i) {
      const uint32_t q = (word >> (4 * i)) & 0xF;
      const float l = bf16_bits_to_float(lutsec[row * 16 + q]);
      const float v = fmaf(a, l, b);                        // one fp32 rounding
      const __nv_bfloat16 h = __float2bfloat16_rn(v);       // then bf16, nearest-even
      w[row * L.k + col0 + i] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

static int grid_for(size_t work, int threads) {
  size_t b = (work + threads - 1) / threads;
  if (b > 65535u * 8u) b = 65535u * 8u;
  return (int)(b ? b : 1);
}

cudaError_t launch_pack(const uint8_t* idx_nib, const uint16_t* lut, const uint16_t* alpha,
                        const uint16_t* beta, const Layout& L, uint8_t* packed,
                        cudaStream_t stream) {
  const int th = 256;
  pack_weights_kernel<<<grid_for((size_t)L.n_pad * L.k / 32, th), th, 0, stream>>>(
      idx_nib, L, reinterpret_cast<uint4*>(packed + L.w_off));
  pack_lut_kernel<<<grid_for((size_t)L.n_pad * 16, th), th, 0, stream>>>(
      lut, L, reinterpret_cast<uint16_t*>(packed + L.lut_off));
  pack_scales_kernel<<<grid_for((size_t)L.n_pad * L.groups, th), th, 0, stream>>>(
      alpha, beta, L, reinterpret_cast<uint32_t*>(packed + L.ab_off));
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* packed, const Layout& L, uint16_t* w,
                           cudaStream_t stream) {
  const int th = 256;
  dequant_kernel<<<grid_for((size_t)L.n * L.k / 8, th), th, 0, stream>>>(packed, L, w);
  return cudaGetLastError();
}

}  // namespace any4
