// any4 decode with the row tables held in registers (byte permutes).
//
// The explainer (10100.com, article 149119421, section 3) keeps each row's
// 16-entry table in registers and decodes with native instructions. Here a
// lane holds the table of each of its rows as byte planes: the low and the
// high bytes of entries 0-7 and of entries 15-8 (reversed), 8 registers per
// row. A 16-bit selector of four 4-bit indices picks 4 bytes from entries
// 0-7 with one prmt (an index >= 8 has bit 3 set, which makes prmt replicate
// a sign bit instead: a don't-care), the complemented selector picks 4 bytes
// from entries 15-8 (it maps index 8+m to byte 7-m and sets bit 3 of the
// indices < 8), one prmt per plane takes each byte from the right half (bit 3
// of the index moved to bit 2 of the selector) and two prmt interleave the
// planes into bf16 pairs: 8 byte permutes per 4 weights of a row.
//
// On B200 prmt issues at half rate (64 lanes per clock per SM), so this
// decode is bound by the integer pipe: it suits the tensor-core GEMM of
// prefill, where each decoded weight feeds 64 or more tokens, not the
// memory-bound decode of 1-16 tokens (linear.cu).
#pragma once

#include <cstdint>

#include "device_ops.cuh"

namespace any4 {

// A row's table as byte planes: low / high bytes of entries 0-3, 4-7 and of
// entries 15-12, 11-8.
struct Planes {
  uint32_t l0, l1, lq0, lq1, h0, h1, hq0, hq1;
};

// a = entries 0..7 of a row, b = entries 8..15 (as loaded: word i holds
// entries 2i (low half) and 2i+1).
__device__ __forceinline__ Planes to_planes(const uint4& a, const uint4& b) {
  Planes P;
  P.l0 = prmt(a.x, a.y, 0x6420u);   // lo(0), lo(1), lo(2), lo(3)
  P.h0 = prmt(a.x, a.y, 0x7531u);
  P.l1 = prmt(a.z, a.w, 0x6420u);   // entries 4..7
  P.h1 = prmt(a.z, a.w, 0x7531u);
  P.lq0 = prmt(b.w, b.z, 0x4602u);  // lo(15), lo(14), lo(13), lo(12)
  P.hq0 = prmt(b.w, b.z, 0x5713u);
  P.lq1 = prmt(b.y, b.x, 0x4602u);  // entries 11..8
  P.hq1 = prmt(b.y, b.x, 0x5713u);
  return P;
}

// Four weights of one row: s holds four 4-bit indices (low 16 bits used), ns
// its complement, s2 the half selector; o0 = (w0, w1), o1 = (w2, w3) as bf16.
__device__ __forceinline__ void decode4(const Planes& P, uint32_t s, uint32_t ns, uint32_t s2, uint32_t& o0,
                                        uint32_t& o1) {
  const uint32_t aL = prmt(P.l0, P.l1, s), bL = prmt(P.lq0, P.lq1, ns);
  const uint32_t aH = prmt(P.h0, P.h1, s), bH = prmt(P.hq0, P.hq1, ns);
  const uint32_t rL = prmt(aL, bL, s2), rH = prmt(aH, bH, s2);
  o0 = prmt(rL, rH, 0x5140u);
  o1 = prmt(rL, rH, 0x7362u);
}

// Eight weights: word w holds row A's selector (low half) and row B's (high
// half); a = {A(w0,w1), B(w0,w1), A(w2,w3), B(w2,w3)}.
__device__ __forceinline__ void decode8(const Planes& A, const Planes& B, uint32_t w, uint32_t (&a)[4]) {
  uint32_t nw, s2;
  asm("sub.u32 %0, -1, %1;" : "=r"(nw) : "r"(w));   // ~w on the integer-add path
  asm("lop3.b32 %0, %1, 0x44444444, 0x32103210, 0xEA;" : "=r"(s2) : "r"(w >> 1));
  decode4(A, w, nw, s2, a[0], a[2]);
  decode4(B, w >> 16, nw >> 16, s2 >> 16, a[1], a[3]);
}

// Row-pair words (layout.cuh: byte b of step s holds pair g (b even) or
// g+8 (b odd) at column c0 + b/2, row r in the low nibble and r+16 in the
// high nibble) of steps 2j (w0, columns c0, c0+1) and 2j+1 (w1, c0+2, c0+3)
// -> per-row selectors of the four columns: t0 = rows g | g+8 << 16,
// t1 = rows g+16 | g+24 << 16.
__device__ __forceinline__ void rowpair_to_selectors(uint32_t w0, uint32_t w1, uint32_t& t0, uint32_t& t1) {
  const uint32_t e0 = w0 & 0x0F0F0F0Fu, e1 = w1 & 0x0F0F0F0Fu;                 // rows g, g+8
  const uint32_t o0 = (w0 >> 4) & 0x0F0F0F0Fu, o1 = (w1 >> 4) & 0x0F0F0F0Fu;   // rows g+16, g+24
  // bytes [c0, c2, c0', c2'] and [c1, c3, c1', c3'] of the two rows
  t0 = prmt(e0, e1, 0x5140u) | (prmt(e0, e1, 0x7362u) << 4);
  t1 = prmt(o0, o1, 0x5140u) | (prmt(o0, o1, 0x7362u) << 4);
}

// Scale record (layout.cuh) of one panel and group for lane g: alpha/beta of
// rows g, g+16 (words 0, 1) and g+8, g+24 (words 2, 3) -> (value, value)
// bf16 pairs for rows g, g+8, g+16, g+24 (index 0..3).
__device__ __forceinline__ void scale_pairs(const uint4& rec, uint32_t (&al)[4], uint32_t (&be)[4]) {
  al[0] = prmt(rec.x, 0u, 0x1010u);
  be[0] = prmt(rec.y, 0u, 0x1010u);
  al[1] = prmt(rec.z, 0u, 0x1010u);
  be[1] = prmt(rec.w, 0u, 0x1010u);
  al[2] = prmt(rec.x, 0u, 0x3232u);
  be[2] = prmt(rec.y, 0u, 0x3232u);
  al[3] = prmt(rec.z, 0u, 0x3232u);
  be[3] = prmt(rec.w, 0u, 0x3232u);
}

}  // namespace any4
