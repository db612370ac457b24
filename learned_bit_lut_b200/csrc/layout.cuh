// Device layout of a packed any4 weight (written by any4_pack).
//
// The explainer's tinygemm notes (10100.com, article 149119421, section 3) keep
// the table close to the arithmetic and pre-arrange the weights in the compute
// format. This layout is built for the B200 linear kernel of this library, in
// which each decoder thread owns one weight row (one Tensor Memory lane):
//
//  * rows are grouped in tiles of 128 (N is padded up with zero rows);
//  * K is cut into chunks of 64 columns; one (tile, chunk) "unit" is 4096
//    contiguous bytes, and units are stored tile by tile, chunk by chunk, so
//    any run of consecutive units is one contiguous byte range;
//  * inside a unit, warp quarter q (rows 32q..32q+31) owns 1024 bytes: first
//    the 16 bytes of columns 0..31 of each of its 32 rows, then the 16 bytes of
//    columns 32..63. A row's 16 bytes are its canonical index bytes (byte j
//    holds columns 2j and 2j+1, low nibble first), so a warp reads 512
//    contiguous bytes per 128-bit load.
//
// Sections (each starts on a 256-byte boundary):
//   weights  [tiles][chunks][4 quarters][2 halves][32 rows][16 B]   Np*K/2 bytes
//   lut      [Np rows][16 x bf16]  (canonical order)               32*Np bytes
//   scales   [tiles][K/G groups][128 rows] u32 = alpha | beta << 16 4*Np*K/G bytes
// with Np = N rounded up to a multiple of 128.
#pragma once

#include <cstddef>
#include <cstdint>

namespace any4 {

constexpr int kTileRows = 128;
constexpr int kChunkK = 64;
constexpr int kUnitBytes = kTileRows * kChunkK / 2;   // 4096
constexpr int kAlign = 256;
constexpr int kMaxRows = 1 << 20;

struct Layout {
  int n, k, g;
  int n_pad;        // n rounded up to a multiple of 128
  int tiles;        // n_pad / 128
  int chunks;       // k / 64
  int groups;       // k / g
  size_t w_off, lut_off, ab_off, total;
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool shape_ok(int n, int k, int g) {
  if (n <= 0 || k <= 0 || n > kMaxRows) return false;
  if (n % 16 || k % kChunkK) return false;
  if (!(g == 64 || g == 128 || g == 256 || g == 512 || g == 1024)) return false;
  return k % g == 0;
}

inline Layout make_layout(int n, int k, int g) {
  Layout L{};
  L.n = n; L.k = k; L.g = g;
  L.n_pad = (int)align_up((size_t)n, kTileRows);
  L.tiles = L.n_pad / kTileRows;
  L.chunks = k / kChunkK;
  L.groups = k / g;
  L.w_off = 0;
  L.lut_off = align_up((size_t)L.n_pad * k / 2, kAlign);
  L.ab_off = L.lut_off + align_up((size_t)L.n_pad * 32, kAlign);
  L.total = L.ab_off + align_up((size_t)L.n_pad * L.groups * 4, kAlign);
  return L;
}

}  // namespace any4
