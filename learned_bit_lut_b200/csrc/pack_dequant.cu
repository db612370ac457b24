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

// Word e of the weight section: e = ((panel*kchunks + chunk)*2 + h)*128 + lane*4 + i,
// step s = 4*h + i of the chunk, lane = 4*g + t, columns c0 = 64*chunk + 16t + 2s
// and c0 + 1.
struct WordPos {
  size_t panel;
  int g, t, c0;
};

__device__ __forceinline__ WordPos word_pos(size_t e, int kchunks) {
  WordPos q;
  const int i = (int)(e & 3);
  const int lane = (int)((e >> 2) & 31);
  const int h = (int)((e >> 7) & 1);
  const size_t pc = e >> 8;
  const int chunk = (int)(pc % kchunks);
  q.panel = pc / kchunks;
  q.g = lane >> 2;
  q.t = lane & 3;
  q.c0 = chunk * kChunkCols + 16 * q.t + 2 * (4 * h + i);
  return q;
}

// Byte b of a word: rows (r, r+16) with r = g + 8*(b & 1), column c0 + (b >> 1).
__device__ __forceinline__ int byte_row(int g, int b) { return g + 8 * (b & 1); }

// One thread per packed 32-bit word.
__global__ void pack_weights_kernel(const uint8_t* __restrict__ idx_nib, Layout L,
                                    uint32_t* __restrict__ out) {
  const size_t total = (size_t)L.n_pad * L.k / 8;
  const size_t row_bytes = (size_t)L.k / 2;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const WordPos q = word_pos(e, L.kchunks);
    uint32_t v = 0;
    for (int b = 0; b < 4; ++b) {
      const int col = q.c0 + (b >> 1);
      for (int u = 0; u < 2; ++u) {
        const size_t row = q.panel * kPanelRows + byte_row(q.g, b) + 16 * u;
        if (row >= (size_t)L.n) continue;
        const uint32_t nib = (idx_nib[row * row_bytes + col / 2] >> (4 * (col & 1))) & 0xFu;
        v |= nib << (8 * b + 4 * u);
      }
    }
    out[e] = v;
  }
}

// b-bit weights (b = 2, 3; layout.cuh): one thread per (panel, chunk, lane)
// builds the lane's 32 row-pair codes and writes its 2b packed words.
template <int B>
__global__ void pack_weights_bits_kernel(const uint8_t* __restrict__ idx_nib, Layout L,
                                         uint32_t* __restrict__ out) {
  constexpr int W = 2 * B;
  constexpr uint32_t mask = (1u << B) - 1u;
  const size_t total = (size_t)L.panels * L.kchunks * 32;
  const size_t row_bytes = (size_t)L.k / 2;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int lane = (int)(e & 31);
    const size_t pc = e >> 5;
    const int chunk = (int)(pc % L.kchunks);
    const size_t panel = pc / L.kchunks;
    const int g = lane >> 2, t = lane & 3;
    uint32_t wd[W];
    for (int j = 0; j < W; ++j) wd[j] = 0u;
    for (int f = 0; f < 32; ++f) {
      const int st = f >> 2, q = f & 3;
      const int col = chunk * kChunkCols + 16 * t + 2 * st + (q >> 1);
      uint32_t code = 0;
      for (int u = 0; u < 2; ++u) {
        const size_t row = panel * kPanelRows + g + 8 * (q & 1) + 16 * u;
        if (row >= (size_t)L.n) continue;
        const uint32_t nib = (idx_nib[row * row_bytes + col / 2] >> (4 * (col & 1))) & mask;
        code |= nib << (B * u);
      }
      const int bit = 2 * B * f, word = bit >> 5, off = bit & 31;
      wd[word] |= code << off;
      if (off + 2 * B > 32) wd[word + 1] |= code >> (32 - off);
    }
    const size_t base = (panel * L.kchunks + chunk) * (size_t)L.chunk_bytes / 4;
    for (int j = 0; j < W; ++j) {
      const size_t at = j < 4 ? base + (size_t)lane * 4 + j : base + 128 + (size_t)lane * (W - 4) + (j - 4);
      out[at] = wd[j];
    }
  }
}

__global__ void pack_lut_kernel(const uint16_t* __restrict__ lut, Layout L,
                                uint16_t* __restrict__ out) {
  const size_t total = (size_t)L.n_pad * 16;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x)
    out[e] = e < (size_t)L.n * 16 ? lut[e] : (uint16_t)0;
}

// The same 16-entry table in every row (fixed-table formats).
struct Table16 {
  uint16_t v[16];
};

__global__ void pack_lut_fixed_kernel(Table16 t, Layout L, uint16_t* __restrict__ out) {
  const size_t total = (size_t)L.n_pad * 16;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x)
    out[e] = e < (size_t)L.n * 16 ? t.v[e & 15] : (uint16_t)0;
}

// One thread per scale word: [panel][group][g][j], j = 2*half + (beta ? 1 : 0),
// value = v(r) | v(r+16) << 16 with r = 32*panel + g + 8*half.
__global__ void pack_scales_kernel(const uint16_t* __restrict__ alpha,
                                   const uint16_t* __restrict__ beta, Layout L,
                                   uint32_t* __restrict__ out) {
  const size_t total = (size_t)L.panels * L.groups * 32;
  const size_t padded = (L.total - L.ab_off) / 4;   // the section's tail padding is written as 0
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < padded;
       e += (size_t)gridDim.x * blockDim.x) {
    if (e >= total) {
      out[e] = 0u;
      continue;
    }
    const int j = (int)(e & 3);
    const int g = (int)((e >> 2) & 7);
    const size_t pg = e >> 5;
    const int grp = (int)(pg % L.groups);
    const size_t panel = pg / L.groups;
    const uint16_t* src = (j & 1) ? beta : alpha;
    const size_t r0 = panel * kPanelRows + g + 8 * (j >> 1), r1 = r0 + 16;
    uint32_t v = 0;
    if (r0 < (size_t)L.n) v |= src[r0 * L.groups + grp];
    if (r1 < (size_t)L.n) v |= (uint32_t)src[r1 * L.groups + grp] << 16;
    out[e] = v;
  }
}

// One thread per packed 32-bit word: 8 weights (two columns of four rows).
__global__ void dequant_kernel(const uint8_t* __restrict__ packed, Layout L,
                               uint16_t* __restrict__ w) {
  const uint32_t* words = reinterpret_cast<const uint32_t*>(packed + L.w_off);
  const uint16_t* lutsec = reinterpret_cast<const uint16_t*>(packed + L.lut_off);
  const uint32_t* ab = reinterpret_cast<const uint32_t*>(packed + L.ab_off);
  const size_t total = (size_t)L.n_pad * L.k / 8;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const WordPos q = word_pos(e, L.kchunks);
    const uint32_t word = words[e];
    for (int b = 0; b < 4; ++b) {
      const int col = q.c0 + (b >> 1);
      const int half = b & 1;
      const uint32_t* s = ab + ((q.panel * L.groups + col / L.g) * 8 + q.g) * 4 + 2 * half;
      for (int u = 0; u < 2; ++u) {
        const size_t row = q.panel * kPanelRows + byte_row(q.g, b) + 16 * u;
        if (row >= (size_t)L.n) continue;
        const uint32_t idx = (word >> (8 * b + 4 * u)) & 0xFu;
        const float a = bf16_bits_to_float((s[0] >> (16 * u)) & 0xFFFFu);
        const float c = bf16_bits_to_float((s[1] >> (16 * u)) & 0xFFFFu);
        const float v = fmaf(a, bf16_bits_to_float(lutsec[row * 16 + idx]), c);   // one fp32 rounding
        const __nv_bfloat16 h = __float2bfloat16_rn(v);                            // then bf16
        w[row * L.k + col] = *reinterpret_cast<const uint16_t*>(&h);
      }
    }
  }
}

// b-bit dequant (b = 2, 3): one thread per (panel, chunk, lane); same
// arithmetic as dequant_kernel.
template <int B>
__global__ void dequant_bits_kernel(const uint8_t* __restrict__ packed, Layout L, uint16_t* __restrict__ w) {
  constexpr int W = 2 * B;
  constexpr uint32_t mask = (1u << B) - 1u;
  const uint32_t* words = reinterpret_cast<const uint32_t*>(packed + L.w_off);
  const uint16_t* lutsec = reinterpret_cast<const uint16_t*>(packed + L.lut_off);
  const uint32_t* ab = reinterpret_cast<const uint32_t*>(packed + L.ab_off);
  const size_t total = (size_t)L.panels * L.kchunks * 32;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int lane = (int)(e & 31);
    const size_t pc = e >> 5;
    const int chunk = (int)(pc % L.kchunks);
    const size_t panel = pc / L.kchunks;
    const int g = lane >> 2, t = lane & 3;
    const size_t base = (panel * L.kchunks + chunk) * (size_t)L.chunk_bytes / 4;
    uint32_t wd[W + 1];
    for (int j = 0; j < W; ++j)
      wd[j] = words[j < 4 ? base + (size_t)lane * 4 + j : base + 128 + (size_t)lane * (W - 4) + (j - 4)];
    wd[W] = 0u;
    for (int f = 0; f < 32; ++f) {
      const int st = f >> 2, q = f & 3;
      const int col = chunk * kChunkCols + 16 * t + 2 * st + (q >> 1);
      const int bit = 2 * B * f, word = bit >> 5, off = bit & 31;
      const uint32_t code = (uint32_t)((((uint64_t)wd[word + 1] << 32) | wd[word]) >> off);
      const uint32_t* sc = ab + ((panel * L.groups + col / L.g) * 8 + g) * 4 + 2 * (q & 1);
      for (int u = 0; u < 2; ++u) {
        const size_t row = panel * kPanelRows + g + 8 * (q & 1) + 16 * u;
        if (row >= (size_t)L.n) continue;
        const uint32_t idx = (code >> (B * u)) & mask;
        const float a = bf16_bits_to_float((sc[0] >> (16 * u)) & 0xFFFFu);
        const float c = bf16_bits_to_float((sc[1] >> (16 * u)) & 0xFFFFu);
        const float v = fmaf(a, bf16_bits_to_float(lutsec[row * 16 + idx]), c);
        const __nv_bfloat16 hv = __float2bfloat16_rn(v);
        w[row * L.k + col] = *reinterpret_cast<const uint16_t*>(&hv);
      }
    }
  }
}

// Tiled dequant: one thread block per (panel, 8 chunks = 512 columns). The
// block decodes its words into a shared [32 rows][512 columns] bf16 tile
// (same fp32 fma + round-to-nearest-even as dequant_kernel) and writes each
// row segment with 16-byte stores, so the N x K output is written coalesced.
constexpr int kDqChunks = 8;
constexpr int kDqRow = kDqChunks * kChunkCols + 8;   // bf16 per tile row (16-byte pad)

__global__ void __launch_bounds__(256) dequant_tile_kernel(const uint8_t* __restrict__ packed, Layout L,
                                                           uint16_t* __restrict__ w) {
  __shared__ __align__(16) uint16_t tile[kPanelRows * kDqRow];
  __shared__ float lut[kPanelRows * 16];
  const uint32_t* words = reinterpret_cast<const uint32_t*>(packed + L.w_off);
  const uint16_t* lutsec = reinterpret_cast<const uint16_t*>(packed + L.lut_off);
  const uint32_t* ab = reinterpret_cast<const uint32_t*>(packed + L.ab_off);
  const int P = blockIdx.y;
  const int c_begin = blockIdx.x * kDqChunks;
  const int nch = min(kDqChunks, L.kchunks - c_begin);
  // word j of this thread: e = threadIdx.x + 256 j (chunk j of the strip, word
  // threadIdx.x of the chunk); its weights and scales are loaded before the
  // table barrier so the loads overlap
  const int wi = threadIdx.x;
  const int i = wi & 3, ln = (wi >> 2) & 31, h = wi >> 7;
  const int g = ln >> 2, t = ln & 3;
  const int c0 = 16 * t + 2 * (4 * h + i);   // column within a chunk
  const int gshift = __ffs(L.g) - 1;         // G is a power of two
  const uint32_t* wsrc = words + ((size_t)P * L.kchunks + c_begin) * 256 + wi;
  const uint4* ssrc = reinterpret_cast<const uint4*>(ab) + (size_t)P * L.groups * 8 + g;
  uint32_t word[kDqChunks];
  uint4 sc[kDqChunks];
#pragma unroll
  for (int j = 0; j < kDqChunks; ++j) {
    if (j < nch) {
      const int col0 = (c_begin + j) * kChunkCols + c0;
      word[j] = __ldg(wsrc + j * 256);
      sc[j] = __ldg(ssrc + (size_t)(col0 >> gshift) * 8);
    }
  }
  for (int e = threadIdx.x; e < kPanelRows * 16; e += blockDim.x)
    lut[e] = bf16_bits_to_float(lutsec[(size_t)P * kPanelRows * 16 + e]);
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kDqChunks; ++j) {
    if (j < nch) {
      const uint32_t sw[4] = {sc[j].x, sc[j].y, sc[j].z, sc[j].w};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int r = g + 8 * half + 16 * u;
          const float a = bf16_bits_to_float((sw[2 * half] >> (16 * u)) & 0xFFFFu);
          const float c = bf16_bits_to_float((sw[2 * half + 1] >> (16 * u)) & 0xFFFFu);
          const uint32_t i0 = (word[j] >> (8 * half + 4 * u)) & 0xFu;         // column c0
          const uint32_t i1 = (word[j] >> (8 * (half + 2) + 4 * u)) & 0xFu;   // column c0 + 1
          // one fp32 rounding each, then bf16 nearest-even
          const __nv_bfloat162 v = __floats2bfloat162_rn(fmaf(a, lut[r * 16 + i0], c), fmaf(a, lut[r * 16 + i1], c));
          *reinterpret_cast<__nv_bfloat162*>(&tile[r * kDqRow + j * kChunkCols + c0]) = v;
        }
      }
    }
  }
  __syncthreads();
  uint16_t* wp = w + (size_t)P * kPanelRows * L.k + (size_t)c_begin * kChunkCols;
  const int rows = min(kPanelRows, L.n - P * kPanelRows);
  if (nch == kDqChunks) {   // full strip: 64 16-byte units per row, 4 rows per pass
    const int u = threadIdx.x & 63;
#pragma unroll
    for (int r = threadIdx.x >> 6; r < kPanelRows; r += 4)
      if (r < rows)
        *reinterpret_cast<uint4*>(wp + (size_t)r * L.k + u * 8) =
            *reinterpret_cast<const uint4*>(&tile[r * kDqRow + u * 8]);
  } else {
    const int units = nch * kChunkCols / 8;   // 16-byte units per row
    for (int e = threadIdx.x; e < kPanelRows * units; e += blockDim.x) {
      const int r = e / units, u = e % units;
      if (r < rows)
        *reinterpret_cast<uint4*>(wp + (size_t)r * L.k + u * 8) =
            *reinterpret_cast<const uint4*>(&tile[r * kDqRow + u * 8]);
    }
  }
}

static int grid_for(size_t work, int threads) {
  size_t b = (work + threads - 1) / threads;
  if (b > 65535u * 8u) b = 65535u * 8u;
  return (int)(b ? b : 1);
}

static void launch_pack_weights(const uint8_t* idx_nib, const Layout& L, uint8_t* packed, cudaStream_t stream) {
  const int th = 256;
  uint32_t* out = reinterpret_cast<uint32_t*>(packed + L.w_off);
  const size_t lanes = (size_t)L.panels * L.kchunks * 32;
  if (L.bits == 3)
    pack_weights_bits_kernel<3><<<grid_for(lanes, th), th, 0, stream>>>(idx_nib, L, out);
  else if (L.bits == 2)
    pack_weights_bits_kernel<2><<<grid_for(lanes, th), th, 0, stream>>>(idx_nib, L, out);
  else
    pack_weights_kernel<<<grid_for((size_t)L.n_pad * L.k / 8, th), th, 0, stream>>>(idx_nib, L, out);
}

cudaError_t launch_pack(const uint8_t* idx_nib, const uint16_t* lut, const uint16_t* alpha,
                        const uint16_t* beta, const Layout& L, uint8_t* packed,
                        cudaStream_t stream) {
  const int th = 256;
  launch_pack_weights(idx_nib, L, packed, stream);
  pack_lut_kernel<<<grid_for((size_t)L.n_pad * 16, th), th, 0, stream>>>(
      lut, L, reinterpret_cast<uint16_t*>(packed + L.lut_off));
  pack_scales_kernel<<<grid_for((L.total - L.ab_off) / 4, th), th, 0, stream>>>(
      alpha, beta, L, reinterpret_cast<uint32_t*>(packed + L.ab_off));
  return cudaGetLastError();
}

cudaError_t launch_pack_fixed(const uint8_t* idx_nib, const uint16_t (&lut)[16],
                              const uint16_t* alpha, const uint16_t* beta, const Layout& L,
                              uint8_t* packed, cudaStream_t stream) {
  const int th = 256;
  Table16 t;
  for (int q = 0; q < 16; ++q) t.v[q] = lut[q];
  launch_pack_weights(idx_nib, L, packed, stream);
  pack_lut_fixed_kernel<<<grid_for((size_t)L.n_pad * 16, th), th, 0, stream>>>(
      t, L, reinterpret_cast<uint16_t*>(packed + L.lut_off));
  pack_scales_kernel<<<grid_for((L.total - L.ab_off) / 4, th), th, 0, stream>>>(
      alpha, beta, L, reinterpret_cast<uint32_t*>(packed + L.ab_off));
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* packed, const Layout& L, uint16_t* w,
                           cudaStream_t stream) {
  const int th = 256;
  const size_t lanes = (size_t)L.panels * L.kchunks * 32;
  if (L.bits == 3) {
    dequant_bits_kernel<3><<<grid_for(lanes, th), th, 0, stream>>>(packed, L, w);
  } else if (L.bits == 2) {
    dequant_bits_kernel<2><<<grid_for(lanes, th), th, 0, stream>>>(packed, L, w);
  } else if ((reinterpret_cast<uintptr_t>(w) & 15) == 0) {   // 16-byte stores need a 16-byte aligned w
    const dim3 grid((L.kchunks + kDqChunks - 1) / kDqChunks, L.panels);
    dequant_tile_kernel<<<grid, th, 0, stream>>>(packed, L, w);
  } else {
    dequant_kernel<<<grid_for((size_t)L.n_pad * L.k / 8, th), th, 0, stream>>>(packed, L, w);
  }
  return cudaGetLastError();
}

}  // namespace any4
