// Device layout of a packed any4 weight (written by any4_pack).
//
// The explainer's tinygemm notes (10100.com, article 149119421, section 3) keep
// the table next to the arithmetic and pre-arrange the weights in the compute
// format. This layout is built for the operand layout of the m16n8k16 bf16
// tensor-core tile used by the linear kernel of this library:
//
//  * rows are grouped in 16-row tiles (N is padded with zero rows up to a
//    multiple of 32, so tiles pair up into 32-row blocks);
//  * K is cut into 64-column "atoms"; an atom of a tile is 512 contiguous
//    bytes, 16 per lane of a warp, so a warp streams it with one 128-bit load
//    per lane; atoms of a tile follow each other, then the next tile;
//  * inside an atom, lane (g = lane/4, t = lane%4) owns, for each of the four
//    tensor-core steps s, one 32-bit word (c = 64*atom + 16*t + 4*s):
//        bits  0..7   idx[row g  ][c], idx[row g  ][c+1]      (low nibble = c)
//        bits  8..15  idx[row g  ][c+2], idx[row g  ][c+3]
//        bits 16..23  idx[row g+8][c], idx[row g+8][c+1]
//        bits 24..31  idx[row g+8][c+2], idx[row g+8][c+3]
//    Every byte is one (even, odd) column pair of the canonical nibble layout.
//    The m16n8k16 tile's columns 2t, 2t+1 | 2t+8, 2t+9 of step s are mapped
//    to weight columns c, c+1 | c+2, c+3: a permutation of K inside the atom,
//    applied identically to the activations, chosen so that the 16
//    activation columns a lane needs over the four steps, 64*atom+16*t ..
//    +15, are contiguous (two 128-bit loads).
//
// Sections (each starts on a 256-byte boundary), Np = N rounded up to 32:
//   weights  [Np/16 tiles][K/64 atoms][32 lanes][4 x u32]      Np*K/2 bytes
//   lut      [Np rows][16 x bf16]  (canonical order)             32*Np bytes
//   scales   [Np/16 tiles][K/G groups][16 rows] u32 = alpha | beta << 16
#pragma once

#include <cstddef>
#include <cstdint>

namespace any4 {

constexpr int kTileRows = 16;
constexpr int kBlockRows = 32;     // two tiles share one activation fragment
constexpr int kAtomK = 64;
constexpr int kAtomBytes = 512;
constexpr int kAlign = 256;
constexpr int kMaxRows = 1 << 20;

struct Layout {
  int n, k, g;
  int n_pad;        // n rounded up to a multiple of 32
  int tiles;        // n_pad / 16
  int katoms;       // k / 64
  int groups;       // k / g
  size_t w_off, lut_off, ab_off, total;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool shape_ok(int n, int k, int g) {
  if (n <= 0 || k <= 0 || n > kMaxRows) return false;
  if (n % 16 || k % kAtomK) return false;
  if (!(g == 64 || g == 128 || g == 256 || g == 512 || g == 1024)) return false;
  return k % g == 0;
}

inline Layout make_layout(int n, int k, int g) {
  Layout L{};
  L.n = n; L.k = k; L.g = g;
  L.n_pad = (int)align_up((size_t)n, kBlockRows);
  L.tiles = L.n_pad / kTileRows;
  L.katoms = k / kAtomK;
  L.groups = k / g;
  L.w_off = 0;
  L.lut_off = align_up((size_t)L.n_pad * k / 2, kAlign);
  L.ab_off = L.lut_off + align_up((size_t)L.n_pad * 32, kAlign);
  L.total = L.ab_off + align_up((size_t)L.n_pad * L.groups * 4, kAlign);
  return L;
}

}  // namespace any4
