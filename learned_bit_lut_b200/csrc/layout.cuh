// Device layout of a packed any4 weight (written by any4_pack).
//
// The explainer's tinygemm notes (10100.com, article 149119421, section 3) keep
// the table next to the arithmetic and pre-arrange the weights in the compute
// format. This layout is built for the way the linear kernel of this library
// decodes and contracts the weights:
//
//  * rows are grouped in 32-row panels (N is padded with zero rows up to a
//    multiple of 32); inside a panel, rows r and r+16 form a "row pair";
//  * one index byte holds the 4-bit indices of BOTH rows of a pair at the same
//    column (row r in the low nibble, row r+16 in the high nibble), so a byte
//    selects one entry of a 256-entry row-pair table (LUT_r[lo], LUT_r+16[hi]);
//  * K is cut into chunks of 64 columns, a chunk into 8 steps. In step s of a
//    chunk, lane (g = lane/4, t = lane%4) of a warp owns one 32-bit word
//    covering the chunk's columns c0 = 16t+2s and c1 = c0+1 (a permutation of
//    K inside the chunk that gives every lane 16 contiguous activation
//    columns over the chunk, i.e. two 128-bit loads):
//        byte 0  rows (g,   g+16) at c0      byte 2  rows (g,   g+16) at c1
//        byte 1  rows (g+8, g+24) at c0      byte 3  rows (g+8, g+24) at c1
//    so the four bf16 pairs the bytes select are, in order, the four operand
//    registers of one m16n8k16 tensor-core tile whose 16 "rows" are the 16
//    row pairs (see linear.cu);
//  * a chunk is 1 KB: [half h][lane][4 words], word i of half h being step
//    4h+i. Chunks of a panel follow each other, then the next panel, so any
//    range of chunks of a panel is one byte range.
//
// Sections (each starts on a 256-byte boundary), Np = N rounded up to 32:
//   weights  [Np/32 panels][K/64 chunks][2][32 lanes][4 x u32]   Np*K/2 bytes
//   lut      [Np rows][16 x bf16]  (canonical order)               32*Np bytes
//   scales   [Np/32 panels][K/G groups][8 g][4 x u32]             4*Np*K/G bytes
//            word 0: alpha(g)   | alpha(g+16) << 16   (row pair g)
//            word 1: beta(g)    | beta(g+16)  << 16
//            word 2: alpha(g+8) | alpha(g+24) << 16   (row pair g+8)
//            word 3: beta(g+8)  | beta(g+24)  << 16
//
// any3 / any2 (b = 3, 2 bits per index; the variants named in the abstract
// of the "any4: Learned 4-bit Numeric Representation for LLMs" summary
// page): the same panels, chunks, lanes and steps, but a lane's 32
// row-pair codes of a chunk (code f = 4s + q of step s; q = 0: pair g at c0,
// 1: pair g+8 at c0, 2: pair g at c1, 3: pair g+8 at c1; a code is
// idx(r) | idx(r+16) << b) are packed densely, code f at bit 2b*f of the
// lane's 64b-bit string: b = 2 -> 4 words per lane, chunk [lane][4 words]
// (512 B); b = 3 -> 6 words per lane, chunk [lane][words 0-3] then
// [lane][words 4-5] (768 B). Weights take Np*K*b/8 bytes.
#pragma once

#include <cstddef>
#include <cstdint>

namespace any4 {

constexpr int kPanelRows = 32;
constexpr int kTileRows = 16;
constexpr int kChunkCols = 64;
constexpr int kChunkBytes = 1024;
constexpr int kGroupScaleBytes = 128;   // one panel, one group
constexpr int kAlign = 256;
constexpr int kMaxRows = 1 << 20;
constexpr int kMaxTokens = 1 << 20;     // M of any4_linear (M > 16 takes the prefill GEMM)

struct Layout {
  int n, k, g;
  int bits;         // bits per index: 4 (any4), 3 (any3), 2 (any2)
  int chunk_bytes;  // 1024, 768, 512
  int n_pad;        // n rounded up to a multiple of 32
  int tiles;        // n_pad / 16
  int panels;       // n_pad / 32
  int kchunks;      // k / 64
  int groups;       // k / g
  size_t w_off, lut_off, ab_off, total;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool shape_ok(int n, int k, int g) {
  if (n <= 0 || k <= 0 || n > kMaxRows) return false;
  if (n % 16 || k % kChunkCols) return false;
  if (!(g == 64 || g == 128 || g == 256 || g == 512 || g == 1024)) return false;
  return k % g == 0;
}

inline bool bits_ok(int bits) { return bits == 2 || bits == 3 || bits == 4; }

inline Layout make_layout(int n, int k, int g, int bits = 4) {
  Layout L{};
  L.n = n; L.k = k; L.g = g;
  L.bits = bits;
  L.chunk_bytes = kChunkBytes * bits / 4;
  L.n_pad = (int)align_up((size_t)n, kPanelRows);
  L.tiles = L.n_pad / kTileRows;
  L.panels = L.n_pad / kPanelRows;
  L.kchunks = k / kChunkCols;
  L.groups = k / g;
  L.w_off = 0;
  L.lut_off = align_up((size_t)L.panels * L.kchunks * L.chunk_bytes, kAlign);
  L.ab_off = L.lut_off + align_up((size_t)L.n_pad * 32, kAlign);
  L.total = L.ab_off + align_up((size_t)L.panels * L.groups * kGroupScaleBytes, kAlign);
  return L;
}

}  // namespace any4
