// any4_pack and any4_dequant kernels.
//
// Pack reorders the canonical tensors (per-row 4-bit indices, per-row 16-entry
// bf16 table, per-group bf16 scale and offset; any4 explainer, 10100.com
// article 149119421, sections 2 and 2.1) into the device layout of layout.cuh
// (the "weights pre-arranged in the compute format" of section 3). Rows past N
// (padding up to a multiple of 32) are written as zeros.
// Dequant reads that layout back and evaluates w_hat = fma(alpha, LUT[idx],
// beta) in fp32, rounded to bf16: the bit-exact debug view of the weights.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace any4 {

// One thread per packed 32-bit word.
__global__ void pack_weights_kernel(const uint8_t* __restrict__ idx_nib, Layout L,
                                    uint32_t* __restrict__ out) {
  const size_t total = (size_t)L.n_pad * L.k / 8;
  const size_t row_bytes = (size_t)L.k / 2;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int step = (int)(e & 3);
    const int lane = (int)((e >> 2) & 31);
    const size_t tile_atom = e >> 7;
    const int atom = (int)(tile_atom % L.katoms);
    const size_t tile = tile_atom / L.katoms;
    const int g = lane >> 2, t = lane & 3;
    const size_t row0 = tile * kTileRows + g, row1 = row0 + 8;
    const size_t j0 = (size_t)atom * (kAtomK / 2) + t * 8 + step * 2;   // column 64a+16t+4s
    const size_t j1 = j0 + 1;                                            // column +2
    uint32_t v = 0;
    if (row0 < (size_t)L.n)
      v |= (uint32_t)idx_nib[row0 * row_bytes + j0] | ((uint32_t)idx_nib[row0 * row_bytes + j1] << 8);
    if (row1 < (size_t)L.n)
      v |= ((uint32_t)idx_nib[row1 * row_bytes + j0] << 16) |
           ((uint32_t)idx_nib[row1 * row_bytes + j1] << 24);
    out[e] = v;
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
    const int r16 = (int)(e % kTileRows);
    const size_t tg = e / kTileRows;
    const int grp = (int)(tg % L.groups);
    const size_t tile = tg / L.groups;
    const size_t row = tile * kTileRows + r16;
    out[e] = row < (size_t)L.n ? ((uint32_t)alpha[row * L.groups + grp] |
                                  ((uint32_t)beta[row * L.groups + grp] << 16))
                               : 0u;
  }
}

// One thread per packed 32-bit word: 8 weights (4 in row g, 4 in row g+8).
__global__ void dequant_kernel(const uint8_t* __restrict__ packed, Layout L,
                               uint16_t* __restrict__ w) {
  const uint32_t* words = reinterpret_cast<const uint32_t*>(packed + L.w_off);
  const uint16_t* lutsec = reinterpret_cast<const uint16_t*>(packed + L.lut_off);
  const uint32_t* ab = reinterpret_cast<const uint32_t*>(packed + L.ab_off);
  const size_t total = (size_t)L.n_pad * L.k / 8;
  const int col_off[4] = {0, 1, 2, 3};
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int step = (int)(e & 3);
    const int lane = (int)((e >> 2) & 31);
    const size_t tile_atom = e >> 7;
    const int atom = (int)(tile_atom % L.katoms);
    const size_t tile = tile_atom / L.katoms;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t word = words[e];
    const int c = atom * kAtomK + t * 16 + step * 4;
    for (int half = 0; half < 2; ++half) {
      const int r16 = g + 8 * half;
      const size_t row = tile * kTileRows + r16;
      if (row >= (size_t)L.n) continue;
      for (int i = 0; i < 4; ++i) {
        const int col = c + col_off[i];
        const uint32_t q = (word >> (16 * half + 4 * i)) & 0xF;
        const uint32_t s = ab[(tile * L.groups + col / L.g) * kTileRows + r16];
        const float a = bf16_bits_to_float(s & 0xFFFF);
        const float b = bf16_bits_to_float(s >> 16);
        const float v = fmaf(a, bf16_bits_to_float(lutsec[row * 16 + q]), b);   // one fp32 rounding
        const __nv_bfloat16 h = __float2bfloat16_rn(v);                          // then bf16
        w[row * L.k + col] = *reinterpret_cast<const uint16_t*>(&h);
      }
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
  pack_weights_kernel<<<grid_for((size_t)L.n_pad * L.k / 8, th), th, 0, stream>>>(
      idx_nib, L, reinterpret_cast<uint32_t*>(packed + L.w_off));
  pack_lut_kernel<<<grid_for((size_t)L.n_pad * 16, th), th, 0, stream>>>(
      lut, L, reinterpret_cast<uint16_t*>(packed + L.lut_off));
  pack_scales_kernel<<<grid_for((size_t)L.n_pad * L.groups, th), th, 0, stream>>>(
      alpha, beta, L, reinterpret_cast<uint32_t*>(packed + L.ab_off));
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* packed, const Layout& L, uint16_t* w,
                           cudaStream_t stream) {
  const int th = 256;
  dequant_kernel<<<grid_for((size_t)L.n_pad * L.k / 8, th), th, 0, stream>>>(packed, L, w);
  return cudaGetLastError();
}

}  // namespace any4
