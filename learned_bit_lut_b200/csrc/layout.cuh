// Device layout of a packed any4 weight (written by any4_pack).
//
// The explainer's tinygemm notes (10100.com, article 149119421, section 3) keep
// the table in registers and pre-arrange the weights in the compute format.
// This layout is built for the B200 decode path of this library: every 16-row
// tile of W is cut along K into 64-column "atoms"; one atom is 512 contiguous
// bytes, 16 per lane of a warp, so a warp streams it with one 128-bit load per
// lane. Inside an atom, lane (g = lane/4, t = lane%4) owns, for each of the four
// 16-column steps s, one 32-bit word:
//
//   bits  0..7   idx[row g  ][c], idx[row g  ][c+1]      (low nibble = c)
//   bits  8..15  idx[row g  ][c+8], idx[row g  ][c+9]
//   bits 16..23  idx[row g+8][c], idx[row g+8][c+1]
//   bits 24..31  idx[row g+8][c+8], idx[row g+8][c+9]
//
// with c = 64*atom + 16*s + 2*t. These are exactly the operand positions of
// the m16n8k16 tensor-core tile (rows g and g+8, columns 2t, 2t+1, 2t+8, 2t+9),
// and every byte is one (even, odd) column pair of the canonical nibble layout.
//
// Sections (each starts on a 256-byte boundary):
//   weights  [N/16 tiles][K/64 atoms][32 lanes][4 x u32]      N*K/2 bytes
//   lut      [N rows][16 low bytes | 16 high bytes]            32*N bytes
//            (byte q of each half = low / high byte of LUT entry q)
//   scales   [N/16 tiles][K/G groups][16 rows] u32 = alpha | beta << 16
#pragma once

#include <cstddef>
#include <cstdint>

namespace any4 {

constexpr int kTileRows = 16;
constexpr int kAtomK = 64;
constexpr int kAtomBytes = 512;
constexpr int kAlign = 256;

struct Layout {
  int n, k, g;
  int tiles;        // n / 16
  int katoms;       // k / 64
  int groups;       // k / g
  size_t w_off, lut_off, ab_off, total;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool shape_ok(int n, int k, int g) {
  if (n <= 0 || k <= 0) return false;
  if (n > 16 * 65536) return false;   // the linear's counter header covers 65536 tiles
  if (n % kTileRows || k % kAtomK) return false;
  if (!(g == 64 || g == 128 || g == 256 || g == 512 || g == 1024)) return false;
  return k % g == 0;
}

inline Layout make_layout(int n, int k, int g) {
  Layout L{};
  L.n = n; L.k = k; L.g = g;
  L.tiles = n / kTileRows;
  L.katoms = k / kAtomK;
  L.groups = k / g;
  L.w_off = 0;
  L.lut_off = align_up((size_t)n * k / 2, kAlign);
  L.ab_off = L.lut_off + align_up((size_t)n * 32, kAlign);
  L.total = L.ab_off + align_up((size_t)n * L.groups * 4, kAlign);
  return L;
}

}  // namespace any4
