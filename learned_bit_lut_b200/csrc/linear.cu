// any4_linear on B200 (sm_100a): y = x . W_hat^T with W stored as any4.
//
// Method (any4 explainer, 10100.com article 149119421): every row of W has its
// own table (LUT) of 16 bf16 values and every weight is a 4-bit index into it
// (section 2); each contiguous group of G columns has a scale alpha and an
// offset beta (section 2.1); w_hat = fma(alpha, LUT[idx], beta). tinygemm
// (section 3) keeps the table next to the arithmetic and runs batch 1-16 on
// the tensor cores. This kernel is designed from B200 measurements:
//
//  * Contraction: mma.sync m16n8k16 (bf16 in, fp32 accumulate), weights as
//    the 16-row operand, tokens as the 8-wide one (two of them for M > 8).
//    For this skinny shape it consumes ~128 weights per clock per SM, where a
//    tcgen05.mma of 128 x 16 x 16 costs ~198 cycles whatever N is (~10
//    weights per clock per SM), so the narrow-N path is the faster one here.
//  * Decode, split across two pipes. In the m16n8k16 operand a lane holds 4
//    weights of row g and 4 of row g+8 of a 16-row tile:
//      - row g: byte permutes from the row's table held in registers as a
//        low-byte and a high-byte plane (two 8-entry halves per plane, one
//        select on index bit 3, one interleave): integer pipe only;
//      - row g+8: each index byte (two adjacent columns) picks a bf16 pair
//        from a 256-entry pair table (LUT[lo nibble], LUT[hi nibble]) in
//        shared memory with one load; the byte permute that forms the address
//        is the only integer op. Four bank copies per row make every warp-wide
//        lookup conflict free.
//    alpha/beta are applied with one bf16x2 fma per pair (w_hat rounded once
//    to bf16), then the tile goes to the tensor core.
//  * A thread block works on 32-row blocks (two 16-row tiles, so every
//    activation fragment serves two MMAs); its 8 warps split the block's K
//    range and share the pair tables; the fp32 tiles are summed across warps
//    in shared memory in a fixed order.
//  * Stream-K: the (block, 64-column atom) sequence is cut into equal
//    contiguous shares, one per thread block (two blocks per SM). A block
//    split between thread blocks is finished by the last one to arrive: each
//    publishes an fp32 partial and bumps the block's counter; the last sums
//    all partials in thread-block order (deterministic) and writes y. Nothing
//    waits on another thread block.
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.cuh"

namespace any4 {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kCtasPerSm = 2;
constexpr int kMinAtomsPerCta = 16;
constexpr uint32_t kTableBytes = 256 * 256;   // 256 entries x 64 words (2 tiles x 8 rows x 4 copies)

struct Params {
  const uint16_t* x;
  const uint8_t* packed;
  uint16_t* y;
  float* partials;
  unsigned* counters;
  int m, n, k;
  int katoms, groups, apg_shift;           // atoms per group = 1 << apg_shift
  int ctas;
  long long atoms;                          // blocks * katoms
  size_t w_off, lut_off, ab_off;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Thread block that owns atom a under the split a_begin(c) = floor(c * A / C).
__device__ __forceinline__ int cta_of_atom(long long a, long long A, int C) {
  return (int)(((a + 1) * (long long)C - 1) / A);
}

// Decode one packed word into the four bf16x2 operand registers of the
// m16n8k16 tile (before alpha/beta). Row g (bits 0..15) from the register
// planes, row g+8 (bytes 2 and 3) from the shared pair table.
__device__ __forceinline__ void decode_word(uint32_t w, const uint32_t (&lo)[4],
                                            const uint32_t (&hi)[4], uint32_t tab, uint32_t off,
                                            uint32_t (&a)[4]) {
  const uint32_t w7 = w & 0x7777u;                          // entry within a half table
  const uint32_t sel = ((w >> 1) & 0x4444u) | 0x3210u;      // half 0 (byte j) or 1 (byte j+4)
  const uint32_t pa = prmt(lo[0], lo[1], w7), pb = prmt(lo[2], lo[3], w7);
  const uint32_t qa = prmt(hi[0], hi[1], w7), qb = prmt(hi[2], hi[3], w7);
  const uint32_t l = prmt(pa, pb, sel), h = prmt(qa, qb, sel);
  a[0] = prmt(l, h, 0x5140u);                               // tile columns 2t, 2t+1
  a[2] = prmt(l, h, 0x7362u);                               // tile columns 2t+8, 2t+9
  a[1] = lds32(tab + prmt(w, off, 0x5524u));                // entry = byte 2, times 256, + off
  a[3] = lds32(tab + prmt(w, off, 0x5534u));                // entry = byte 3
}

template <int NT>
__device__ __forceinline__ void store_y(const Params& p, int tile0, int lane,
                                        const float (&v)[2][NT][4]) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int tau = 0; tau < 2; ++tau)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 8 * j + 2 * t + (i & 1);
        const int n = (tile0 + tau) * kTileRows + g + 8 * (i >> 1);
        if (m < p.m && n < p.n) {
          const __nv_bfloat16 h = __float2bfloat16_rn(v[tau][j][i]);
          p.y[(size_t)m * p.n + n] = *reinterpret_cast<const uint16_t*>(&h);
        }
      }
}

// cp.async of 16 bytes global -> shared (no registers involved)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// The 32 rows x 16 LUT entries of one 32-row block (1 KB) into a shared slot.
__device__ __forceinline__ void stage_lut(const Params& p, int block, uint32_t slot) {
  if (threadIdx.x < 64)
    cp_async16(slot + 16u * threadIdx.x,
               p.packed + p.lut_off + (size_t)block * kBlockRows * 32 + 16u * threadIdx.x);
  cp_async_commit();
}

template <int NT, int PF>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) linear_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t tab = smem_u32(smem);
  // warp partial tiles for the cross-warp sum; they reuse the table space,
  // which is dead between the end of a block's streaming and the next build
  float* red = reinterpret_cast<float*>(smem);
  constexpr int kF = 2 * NT * 4;
  const uint32_t lut_slot0 = tab + kTableBytes;   // 2 x 1 KB
  const uint8_t* lut_smem = smem + kTableBytes;
  // per-warp ring of PF atoms x 2 tiles x 512 bytes, filled by cp.async; each
  // lane copies and later reads only its own 16 bytes per tile and atom
  const uint32_t ring = lut_slot0 + 2048u + (uint32_t)(threadIdx.x >> 5) * (PF * 1024u) + 16u * (threadIdx.x & 31);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int KA = p.katoms, K = p.k;
  const int apg = 1 << p.apg_shift;
  const long long A = p.atoms;
  const long long a_lo = (long long)blockIdx.x * A / p.ctas;
  const long long a_hi = (long long)(blockIdx.x + 1) * A / p.ctas;
  const int b_first = (int)(a_lo / KA);

  // activation rows of this lane's B fragments: token 8j+g, columns
  // 64*atom + 16*t .. +15 for the four steps of an atom. Tokens >= M repeat
  // token M-1; their outputs are never stored.
  const uint8_t* xrow[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j)
    xrow[j] = reinterpret_cast<const uint8_t*>(p.x + (size_t)min(8 * j + g, p.m - 1) * K) + 32 * t;

  // pair-table slice this thread builds: entry quarter, tile, row, bank copy
  const int bq = threadIdx.x >> 6, btau = (threadIdx.x >> 5) & 1;
  const int brow = (threadIdx.x >> 2) & 7, bcopy = threadIdx.x & 3;
  const uint32_t build_addr = tab + (uint32_t)bq * 64u * 256u + 128u * btau + 16u * brow + 4u * bcopy;
  // byte offset of this lane's bank copy inside an entry row, per tile
  const uint32_t off[2] = {16u * g + 4u * t, 16u * g + 4u * t + 128u};

  // ---- per-warp streaming state, primed one segment ahead
  uint32_t xf[2][NT][4][2];
  uint32_t sraw[4], snext[4];
  auto seg_bounds = [&](long long sa, int& b, long long& se, int& wa0, int& wa1) {
    b = (int)(sa / KA);
    const long long bstart = (long long)b * KA;
    se = min(a_hi, bstart + KA);
    const int ka0 = (int)(sa - bstart), n_at = (int)(se - sa);
    wa0 = ka0 + (int)((long long)warp * n_at / kWarps);
    wa1 = ka0 + (int)((long long)(warp + 1) * n_at / kWarps);
  };
  auto wptr = [&](int b) {
    return p.packed + p.w_off + (size_t)(2 * b) * KA * kAtomBytes + (size_t)lane * 16;
  };
  auto abptr = [&](int b) {
    return reinterpret_cast<const uint32_t*>(p.packed + p.ab_off) +
           (size_t)(2 * b) * p.groups * kTileRows + g;
  };
  auto load_x = [&](int atom, uint32_t (&dst)[NT][4][2]) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const uint8_t* src = xrow[j] + (size_t)atom * (kAtomK * 2);
      const uint4 u0 = ld_nc_v4(src), u1 = ld_nc_v4(src + 16);
      dst[j][0][0] = u0.x; dst[j][0][1] = u0.y; dst[j][1][0] = u0.z; dst[j][1][1] = u0.w;
      dst[j][2][0] = u1.x; dst[j][2][1] = u1.y; dst[j][3][0] = u1.z; dst[j][3][1] = u1.w;
    }
  };
  auto load_s = [&](const uint32_t* ab0, int atom, uint32_t (&dst)[4]) {
    const uint32_t* ab1 = ab0 + (size_t)p.groups * kTileRows;
    const size_t o = (size_t)(atom >> p.apg_shift) * kTileRows;
    dst[0] = ld_nc_u32(ab0 + o); dst[1] = ld_nc_u32(ab0 + o + 8);
    dst[2] = ld_nc_u32(ab1 + o); dst[3] = ld_nc_u32(ab1 + o + 8);
  };
  // weights of atom `atom` of block b into ring slot `slot` (one commit group,
  // possibly empty, per call so that group counting stays uniform)
  auto fetch = [&](int b, int atom, bool valid, int slot) {
    if (valid) {
      const uint8_t* w0 = wptr(b) + (size_t)atom * kAtomBytes;
      cp_async16(ring + (uint32_t)slot * 1024u, w0);
      cp_async16(ring + (uint32_t)slot * 1024u + 512u, w0 + (size_t)KA * kAtomBytes);
    }
    cp_async_commit();
  };
  // first loads of a warp's range: weights of the first PF atoms, activations
  // and scales of the first atom
  auto prime = [&](int b, int wa0, int wa1, bool with_x) {
#pragma unroll
    for (int j = 0; j < PF; ++j) fetch(b, wa0 + j, wa0 + j < wa1, j);
    if (wa0 >= wa1) return;
    if (with_x) load_x(wa0, xf[0]);
    load_s(abptr(b), wa0, sraw);
  };

  long long sa = a_lo;
  int b, wa0, wa1;
  long long se;
  seg_bounds(sa, b, se, wa0, wa1);
  // Only the packed weight (immutable) is read before the grid dependency
  // resolves, so with programmatic dependent launch this prologue overlaps the
  // previous kernel on the stream; activations, y and the workspace are
  // touched only after griddepcontrol.wait.
  prime(b, wa0, wa1, false);
  uint32_t lut_cur = lut_slot0;
  stage_lut(p, b, lut_cur);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cp_async_wait_all();
  __syncthreads();
  bool first_seg = true;
  int split0 = -1, split1 = -1;   // split blocks whose partials await the final count

  while (true) {
    const int tile0 = 2 * b;
    const uint8_t* lut_here = lut_smem + (lut_cur - lut_slot0);
    {
      // pair tables of rows 8..15 of both tiles: entry e = (LUT[e & 15], LUT[e >> 4])
      const uint4* src = reinterpret_cast<const uint4*>(lut_here + (16 * btau + 8 + brow) * 32);
      const uint4 u0 = src[0], u1 = src[1];
      const uint32_t L[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      // high nibbles of this quarter are 4*bq .. 4*bq+3, i.e. pairs L[2bq], L[2bq+1]
      const uint32_t h0 = bq == 0 ? u0.x : bq == 1 ? u0.z : bq == 2 ? u1.x : u1.z;
      const uint32_t h1 = bq == 0 ? u0.y : bq == 1 ? u0.w : bq == 2 ? u1.y : u1.w;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const uint32_t sel = ((j & 1) ? 0x32u : 0x10u) | ((((j >> 4) & 1) ? 0x76u : 0x54u) << 8);
        sts32(build_addr + (uint32_t)j * 256u, prmt(L[(j & 15) >> 1], (j >> 5) ? h1 : h0, sel));
      }
    }
    // this lane's row-g tables of both tiles as low-byte / high-byte planes
    uint32_t lo[2][4], hi[2][4];
#pragma unroll
    for (int tau = 0; tau < 2; ++tau) {
      const uint4* src = reinterpret_cast<const uint4*>(lut_here + (16 * tau + g) * 32);
      const uint4 u0 = src[0], u1 = src[1];
      const uint32_t L[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        lo[tau][i] = prmt(L[2 * i], L[2 * i + 1], 0x6420u);
        hi[tau][i] = prmt(L[2 * i], L[2 * i + 1], 0x7531u);
      }
    }
    // next segment (if any): its LUT rows start moving now
    const bool has_next = se < a_hi;
    int nb = 0, nwa0 = 0, nwa1 = 0;
    long long nse = 0;
    if (has_next) {
      seg_bounds(se, nb, nse, nwa0, nwa1);
      lut_cur = lut_slot0 + (lut_cur == lut_slot0 ? 1024u : 0u);
      stage_lut(p, nb, lut_cur);
    }
    __syncthreads();   // tables ready
    if (first_seg) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      if (wa0 < wa1) load_x(wa0, xf[0]);
      first_seg = false;
    }

    float acc[2][NT][4];
#pragma unroll
    for (int tau = 0; tau < 2; ++tau)
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[tau][j][i] = 0.0f;

    if (wa0 < wa1) {
      const uint32_t* ab0 = abptr(b);
      uint32_t al[4], be[4];   // (alpha, alpha), (beta, beta): rows g, g+8 of both tiles
#pragma unroll
      for (int i = 0; i < 4; ++i) { al[i] = prmt(sraw[i], sraw[i], 0x1010u); be[i] = prmt(sraw[i], sraw[i], 0x3232u); }
      if (wa0 + 1 < wa1 && ((wa0 + 1) & (apg - 1)) == 0) load_s(ab0, wa0 + 1, snext);

      for (int a0 = wa0; a0 < wa1; a0 += PF) {
#pragma unroll
        for (int jj = 0; jj < PF; ++jj) {
          const int a = a0 + jj;
          if (a >= wa1) break;
          cp_async_wait<PF - 1>();                      // this atom's weights have landed
          const uint4 v0 = lds128(ring + (uint32_t)jj * 1024u);
          const uint4 v1 = lds128(ring + (uint32_t)jj * 1024u + 512u);
          fetch(b, a + PF, a + PF < wa1, jj);
          uint32_t (&xc)[NT][4][2] = xf[jj & 1];
          if (a + 1 < wa1) load_x(a + 1, xf[(jj + 1) & 1]);
          if (a != wa0 && (a & (apg - 1)) == 0) {          // first atom of a new group
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              al[i] = prmt(snext[i], snext[i], 0x1010u);
              be[i] = prmt(snext[i], snext[i], 0x3232u);
            }
          }
          if (a + 1 < wa1 && ((a + 1) & (apg - 1)) == 0) load_s(ab0, a + 1, snext);
          const uint32_t words[2][4] = {{v0.x, v0.y, v0.z, v0.w}, {v1.x, v1.y, v1.z, v1.w}};
#pragma unroll
          for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int tau = 0; tau < 2; ++tau) {
              uint32_t af[4];
              decode_word(words[tau][s], lo[tau], hi[tau], tab, off[tau], af);
              af[0] = fma_bf16x2(af[0], al[2 * tau], be[2 * tau]);
              af[2] = fma_bf16x2(af[2], al[2 * tau], be[2 * tau]);
              af[1] = fma_bf16x2(af[1], al[2 * tau + 1], be[2 * tau + 1]);
              af[3] = fma_bf16x2(af[3], al[2 * tau + 1], be[2 * tau + 1]);
#pragma unroll
              for (int j = 0; j < NT; ++j) mma_m16n8k16(acc[tau][j], af, xc[j][s][0], xc[j][s][1]);
            }
        }
      }
    }
    // the next segment's first loads leave before this one's reduction
    if (has_next) prime(nb, nwa0, nwa1, true);

    // ---- sum the warps' tiles in warp order (the table space is free once
    // every warp is past its lookups)
    __syncthreads();
    {
      float4* dst = reinterpret_cast<float4*>(red + ((size_t)warp * 32 + lane) * kF);
#pragma unroll
      for (int tau = 0; tau < 2; ++tau)
#pragma unroll
        for (int j = 0; j < NT; ++j)
          dst[tau * NT + j] = make_float4(acc[tau][j][0], acc[tau][j][1], acc[tau][j][2], acc[tau][j][3]);
    }
    __syncthreads();
    if (warp == 0) {
      const long long bstart = (long long)b * KA;
      float v[2][NT][4];
#pragma unroll
      for (int tau = 0; tau < 2; ++tau)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) v[tau][j][i] = 0.0f;
      for (int w = 0; w < kWarps; ++w) {
        const float4* src = reinterpret_cast<const float4*>(red + ((size_t)w * 32 + lane) * kF);
#pragma unroll
        for (int tau = 0; tau < 2; ++tau)
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const float4 f = src[tau * NT + j];
            v[tau][j][0] += f.x; v[tau][j][1] += f.y; v[tau][j][2] += f.z; v[tau][j][3] += f.w;
          }
      }
      if (sa == bstart && se == bstart + KA) {
        store_y<NT>(p, tile0, lane, v);                       // the whole block is ours
      } else {
        // split block: store the fp32 partial now; the arrival count (and the
        // sum, if this thread block turns out to be the last) waits for the end
        // of the thread block, off the streaming path
        const int my_slot = 2 * blockIdx.x + (b == b_first ? 0 : 1);
        float4* dst = reinterpret_cast<float4*>(p.partials + ((size_t)my_slot * 32 + lane) * kF);
#pragma unroll
        for (int tau = 0; tau < 2; ++tau)
#pragma unroll
          for (int j = 0; j < NT; ++j)
            __stcg(dst + tau * NT + j, make_float4(v[tau][j][0], v[tau][j][1], v[tau][j][2], v[tau][j][3]));
        if (b == b_first) split0 = b; else split1 = b;
      }
    }
    if (!has_next) break;
    cp_async_wait<PF>();   // the LUT rows (older than the PF weight groups of prime)
    __syncthreads();       // reduction reads done, next LUT rows visible
    sa = se;
    b = nb; se = nse; wa0 = nwa0; wa1 = nwa1;
  }

  // ---- arrival counts of the split blocks; the last thread block of a block
  // sums all partials in thread-block order and writes y
  if (warp == 0 && (split0 >= 0 || split1 >= 0)) {
    __threadfence();   // this warp's partial stores before the counts
    __syncwarp();
    for (int q = 0; q < 2; ++q) {
      const int sb = q == 0 ? split0 : split1;
      if (sb < 0) continue;
      unsigned prev = 0;
      if (lane == 0) prev = atomicAdd(p.counters + sb, 1u);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      const long long bstart = (long long)sb * KA;
      const int c_first = cta_of_atom(bstart, A, p.ctas);
      const int c_last = cta_of_atom(bstart + KA - 1, A, p.ctas);
      if (prev != (unsigned)(c_last - c_first)) continue;
      __threadfence();
      float sum[2][NT][4];
#pragma unroll
      for (int tau = 0; tau < 2; ++tau)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) sum[tau][j][i] = 0.0f;
      constexpr int kBatch = 4;
      for (int c0 = c_first; c0 <= c_last; c0 += kBatch) {
        float4 f[kBatch][2 * NT];
#pragma unroll
        for (int qq = 0; qq < kBatch; ++qq) {
          const int c = c0 + qq;
          if (c <= c_last) {
            const long long cb = (long long)c * A / p.ctas;
            const int slot = 2 * c + ((long long)sb == cb / KA ? 0 : 1);
            const float4* src = reinterpret_cast<const float4*>(p.partials + ((size_t)slot * 32 + lane) * kF);
#pragma unroll
            for (int u = 0; u < 2 * NT; ++u) f[qq][u] = __ldcg(src + u);
          } else {
#pragma unroll
            for (int u = 0; u < 2 * NT; ++u) f[qq][u] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int qq = 0; qq < kBatch; ++qq)
#pragma unroll
          for (int tau = 0; tau < 2; ++tau)
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              const float4 u = f[qq][tau * NT + j];
              sum[tau][j][0] += u.x; sum[tau][j][1] += u.y; sum[tau][j][2] += u.z; sum[tau][j][3] += u.w;
            }
      }
      store_y<NT>(p, 2 * sb, lane, sum);
      if (lane == 0) p.counters[sb] = 0u;   // ready for the next call
    }
  }
}

constexpr int kRing = 4;   // atoms in flight per warp through the shared-memory ring

size_t smem_bytes(int nt) {
  (void)nt;   // the cross-warp sum reuses the table space
  return kTableBytes + 2 * 1024 + (size_t)kWarps * kRing * 1024;
}

cudaError_t allow_large_smem() {
  static std::atomic<unsigned long long> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(linear_kernel<1, kRing>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(1));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(linear_kernel<2, kRing>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(2));
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

}  // namespace

LinearPlan plan_linear(int m, const Layout& L, int num_sms) {
  LinearPlan pl{};
  pl.nt = m > 8 ? 2 : 1;
  pl.atoms = (long long)(L.tiles / 2) * L.katoms;
  long long c = pl.atoms / kMinAtomsPerCta;
  const long long cap = (long long)num_sms * kCtasPerSm;
  if (c > cap) c = cap;
  if (c < 1) c = 1;
  pl.ctas = (int)c;
  pl.partials_bytes = (size_t)2 * pl.ctas * 32 * (2 * pl.nt * 4) * sizeof(float);
  pl.workspace_bytes = kHeaderBytes + pl.partials_bytes;
  return pl;
}

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream) {
  cudaError_t e = allow_large_smem();
  if (e != cudaSuccess) return e;
  Params p{};
  p.x = x;
  p.packed = packed;
  p.y = y;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  p.counters = reinterpret_cast<unsigned*>(ws);
  p.partials = reinterpret_cast<float*>(ws + kHeaderBytes);
  p.m = m; p.n = L.n; p.k = L.k;
  p.katoms = L.katoms; p.groups = L.groups;
  p.apg_shift = 0;
  while ((kAtomK << p.apg_shift) < L.g) ++p.apg_shift;
  p.ctas = plan.ctas;
  p.atoms = plan.atoms;
  p.w_off = L.w_off; p.lut_off = L.lut_off; p.ab_off = L.ab_off;
  // programmatic dependent launch: this kernel's weight prologue may overlap the
  // tail of the previous kernel on the stream (see griddepcontrol in the kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes(plan.nt);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (plan.nt == 1) return cudaLaunchKernelEx(&cfg, linear_kernel<1, kRing>, p);
  return cudaLaunchKernelEx(&cfg, linear_kernel<2, kRing>, p);
}

}  // namespace any4
