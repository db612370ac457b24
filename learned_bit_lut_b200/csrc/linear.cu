// any4_linear: y = x . W_hat^T with W stored as any4 (per-row 16-entry bf16
// table, 4-bit indices, per-group bf16 scale/offset).
//
// Method: any4 explainer (10100.com, article 149119421) section 2 (per-row LUT,
// index lookup at inference), section 2.1 (per-group alpha/beta), section 3
// (table kept in registers, pre-arranged weights, batch 1-16 on tensor cores).
//
// Kernel structure (B200):
//  * Work is the flat sequence of 512-byte atoms (16 rows x 64 columns) of the
//    packed weight; atoms of consecutive tiles are contiguous, so a warp's share
//    is one contiguous byte range that it streams with 128-bit loads, several
//    atoms in flight.
//  * Every warp gets an equal share (stream-K over atoms), so all SMs finish
//    together whatever N and K are.
//  * Decode: each lane keeps the low and high bytes of its two rows' tables in
//    registers (16 registers) and looks up 4 indices at a time with byte
//    permutes (2 lookups per byte plane + 1 select on index bit 3, then the
//    bytes are interleaved into bf16 pairs). The group scale and offset are
//    applied with one bf16x2 fma per pair, giving the operand of an m16n8k16
//    bf16 tensor-core tile (weights as the 16-row side, tokens as the 8-wide
//    side, fp32 accumulation).
//  * A tile whose atoms are split between warps is finished by the last warp
//    to arrive: each contributor stores its fp32 partial tile and bumps the
//    tile's counter; the one that completes the count sums all partials in
//    warp order (deterministic) and writes y. Nobody waits on anybody.
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.cuh"

namespace any4 {

namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kCtasPerSm = 2;
constexpr int kMinAtomsPerWarp = 4;
constexpr int kPrefetch = 4;
constexpr size_t kMaxSmemPerCta = 100 * 1024;   // keeps two CTAs per SM

struct LinearArgs {
  const uint16_t* x;
  const uint8_t* packed;
  uint16_t* y;
  float* partials;
  unsigned* counters;
  Layout L;
  int m;
  int warps;
  long long atoms;
};

// Warp that owns atom a under the split a_begin(w) = floor(w * A / W).
__device__ __forceinline__ int warp_of_atom(long long a, long long A, int W) {
  return (int)(((a + 1) * (long long)W - 1) / A);
}

// Decode one packed word (8 indices: 4 of row g in bits 0..15, 4 of row g+8 in
// bits 16..31) into the four bf16x2 A-operand registers of the m16n8k16 tile.
__device__ __forceinline__ void decode_word(uint32_t w, const uint32_t (&lo0)[4],
                                            const uint32_t (&hi0)[4], const uint32_t (&lo1)[4],
                                            const uint32_t (&hi1)[4], uint32_t (&a)[4]) {
  const uint32_t w7 = w & 0x77777777u;                          // entry within a half table
  const uint32_t sel = ((w >> 1) & 0x44444444u) | 0x32103210u;  // byte j of half (bit 3)
  const uint32_t w7h = w7 >> 16, selh = sel >> 16;
  {
    const uint32_t pa = prmt(lo0[0], lo0[1], w7), pb = prmt(lo0[2], lo0[3], w7);
    const uint32_t qa = prmt(hi0[0], hi0[1], w7), qb = prmt(hi0[2], hi0[3], w7);
    const uint32_t lo = prmt(pa, pb, sel), hi = prmt(qa, qb, sel);
    a[0] = prmt(lo, hi, 0x5140u);   // columns 2t, 2t+1
    a[2] = prmt(lo, hi, 0x7362u);   // columns 2t+8, 2t+9
  }
  {
    const uint32_t pa = prmt(lo1[0], lo1[1], w7h), pb = prmt(lo1[2], lo1[3], w7h);
    const uint32_t qa = prmt(hi1[0], hi1[1], w7h), qb = prmt(hi1[2], hi1[3], w7h);
    const uint32_t lo = prmt(pa, pb, selh), hi = prmt(qa, qb, selh);
    a[1] = prmt(lo, hi, 0x5140u);
    a[3] = prmt(lo, hi, 0x7362u);
  }
}

template <int NT>
__device__ __forceinline__ void store_tile(const LinearArgs& p, int tile, int lane,
                                           const float (&acc)[NT][4]) {
  const int g = lane >> 2, t = lane & 3;
  const int n0 = tile * kTileRows + g;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = 8 * j + 2 * t + (i & 1);
      const int n = n0 + 8 * (i >> 1);
      if (m < p.m) {
        const __nv_bfloat16 h = __float2bfloat16_rn(acc[j][i]);
        p.y[(size_t)m * p.L.n + n] = *reinterpret_cast<const uint16_t*>(&h);
      }
    }
  }
}

// End of a warp's run over tile `tile` covering atoms [sb, se). Rarely taken
// (at most once per tile a warp touches), so it is kept out of line to leave
// the registers of the streaming loop alone.
template <int NT>
__device__ __noinline__ void finish_segment(const LinearArgs& p, int wid, int lane, int tile,
                                               long long sb, long long se, long long a_begin,
                                               const float (&acc)[NT][4]) {
  const int KA = p.L.katoms;
  const long long t0 = (long long)tile * KA, t1 = t0 + KA;
  if (sb == t0 && se == t1) {          // the whole tile: no one else contributes
    store_tile<NT>(p, tile, lane, acc);
    return;
  }
  constexpr int kSlot = 32 * 4 * NT;   // floats per partial tile
  const int slot = 2 * wid + ((long long)tile == a_begin / KA ? 0 : 1);
  float* dst = p.partials + (size_t)slot * kSlot + lane * 4 * NT;
#pragma unroll
  for (int j = 0; j < NT; ++j)
    __stcg(reinterpret_cast<float4*>(dst) + j, make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]));
  __threadfence();
  __syncwarp();
  const int w_first = warp_of_atom(t0, p.atoms, p.warps);
  const int w_last = warp_of_atom(t1 - 1, p.atoms, p.warps);
  unsigned prev = 0;
  if (lane == 0) prev = atomicAdd(p.counters + tile, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev != (unsigned)(w_last - w_first)) return;   // not the last contributor
  __threadfence();
  float sum[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) sum[j][i] = 0.0f;
  // contributors in warp order, loads of a batch issued before they are summed
  constexpr int kBatch = 4;
  for (int w0 = w_first; w0 <= w_last; w0 += kBatch) {
    float part[kBatch][NT][4];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int w = w0 + b;
      if (w <= w_last) {
        const long long wb = (long long)w * p.atoms / p.warps;
        const int s = 2 * w + ((long long)tile == wb / KA ? 0 : 1);
        const float4* src = reinterpret_cast<const float4*>(p.partials + (size_t)s * kSlot + lane * 4 * NT);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const float4 v = __ldcg(src + j);
          part[b][j][0] = v.x; part[b][j][1] = v.y; part[b][j][2] = v.z; part[b][j][3] = v.w;
        }
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (w0 + b <= w_last)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) sum[j][i] += part[b][j][i];
  }
  store_tile<NT>(p, tile, lane, sum);
  if (lane == 0) p.counters[tile] = 0u;   // ready for the next call
}

template <int NT>
__global__ void __launch_bounds__(kWarpsPerCta * 32, kCtasPerSm) linear_kernel(const LinearArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const long long A = p.atoms;
  const int KA = p.L.katoms, K = p.L.k, G = p.L.g, NG = p.L.groups;
  const int atoms_per_group = G / kAtomK;

  // ---- this CTA's atom range, and the tables / scales it covers
  const int w_lo = blockIdx.x * kWarpsPerCta;
  const int w_hi = min(w_lo + kWarpsPerCta, p.warps) - 1;
  const long long cta_a0 = (long long)w_lo * A / p.warps;
  const long long cta_a1 = (long long)(w_hi + 1) * A / p.warps;
  const int t_lo = (int)(cta_a0 / KA);
  const int t_hi = (int)((cta_a1 - 1) / KA);
  const long long rec_lo = (long long)t_lo * NG + (int)(cta_a0 - (long long)t_lo * KA) / atoms_per_group;
  const long long rec_hi = (long long)t_hi * NG + (int)(cta_a1 - 1 - (long long)t_hi * KA) / atoms_per_group;
  const int lut_bytes = (t_hi - t_lo + 1) * kTileRows * 32;
  uint8_t* s_lut = smem;
  uint32_t* s_ab = reinterpret_cast<uint32_t*>(smem + lut_bytes);

  const bool active = wid < p.warps;
  const long long a_begin = active ? (long long)wid * A / p.warps : 0;
  const long long a_end = active ? (long long)(wid + 1) * A / p.warps : 0;
  const uint8_t* wsec = p.packed + p.L.w_off + (size_t)lane * 16;

  // weights first: the first atoms are in flight while the tables are staged
  uint4 buf[kPrefetch];
#pragma unroll
  for (int j = 0; j < kPrefetch; ++j)
    if (a_begin + j < a_end) buf[j] = ld_stream_v4(wsec + (size_t)(a_begin + j) * kAtomBytes);

  {
    const uint4* src = reinterpret_cast<const uint4*>(p.packed + p.L.lut_off + (size_t)t_lo * kTileRows * 32);
    uint4* dst = reinterpret_cast<uint4*>(s_lut);
    for (int i = threadIdx.x; i < lut_bytes / 16; i += blockDim.x) dst[i] = __ldg(src + i);
    const uint4* asrc = reinterpret_cast<const uint4*>(p.packed + p.L.ab_off) + rec_lo * 4;
    uint4* adst = reinterpret_cast<uint4*>(s_ab);
    const int nrec4 = (int)(rec_hi - rec_lo + 1) * 4;   // 16 rows x u32 = 4 x uint4 per record
    for (int i = threadIdx.x; i < nrec4; i += blockDim.x) adst[i] = __ldg(asrc + i);
  }
  __syncthreads();
  if (!active) return;

  const int g = lane >> 2, t = lane & 3;
  // x rows feeding this lane's B fragments (token 8j+g). Columns of tokens
  // >= M repeat token M-1; their outputs are never stored.
  const uint32_t* xrow[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int m = min(8 * j + g, p.m - 1);
    xrow[j] = reinterpret_cast<const uint32_t*>(p.x + (size_t)m * K) + t;
  }
  // B fragments of one atom: [j][step][b0, b1]; c = first column / 2 of the atom
  uint32_t xf[2][NT][4][2];
  auto load_x = [&](int c, uint32_t (&dst)[NT][4][2]) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        dst[j][s][0] = __ldg(xrow[j] + c + 8 * s);
        dst[j][s][1] = __ldg(xrow[j] + c + 8 * s + 4);
      }
  };

  // Position of the current atom, advanced incrementally (no divisions in the loop).
  int tile = (int)(a_begin / KA);
  int ka = (int)(a_begin - (long long)tile * KA);   // atom within the tile
  int grp = ka / atoms_per_group;
  int kg = ka - grp * atoms_per_group;               // atom within the group
  load_x(ka * (kAtomK / 2), xf[0]);

  float acc[NT][4];
  uint32_t lo0[4], hi0[4], lo1[4], hi1[4];
  uint32_t al0 = 0, be0 = 0, al1 = 0, be1 = 0;
  int cur_tile = -1;
  long long seg_begin = a_begin;

  for (long long a0 = a_begin; a0 < a_end; a0 += kPrefetch) {
#pragma unroll
    for (int jj = 0; jj < kPrefetch; ++jj) {
      const long long a = a0 + jj;
      if (a >= a_end) break;
      const uint4 wv = buf[jj];
      if (a + kPrefetch < a_end) buf[jj] = ld_stream_v4(wsec + (size_t)(a + kPrefetch) * kAtomBytes);
      // kPrefetch is even, so jj's parity is the atom's parity within the run
      uint32_t (&xc)[NT][4][2] = xf[jj & 1];
      const int ka_next = ka + 1 == KA ? 0 : ka + 1;
      if (a + 1 < a_end) load_x(ka_next * (kAtomK / 2), xf[(jj + 1) & 1]);

      if (tile != cur_tile) {
        if (cur_tile >= 0) finish_segment<NT>(p, wid, lane, cur_tile, seg_begin, a, a_begin, acc);
        const uint4* r0 = reinterpret_cast<const uint4*>(s_lut + ((tile - t_lo) * kTileRows + g) * 32);
        const uint4* r1 = r0 + 16;   // row g+8 is 8 rows * 32 bytes further
        const uint4 l0 = r0[0], h0 = r0[1], l1 = r1[0], h1 = r1[1];
        lo0[0] = l0.x; lo0[1] = l0.y; lo0[2] = l0.z; lo0[3] = l0.w;
        hi0[0] = h0.x; hi0[1] = h0.y; hi0[2] = h0.z; hi0[3] = h0.w;
        lo1[0] = l1.x; lo1[1] = l1.y; lo1[2] = l1.z; lo1[3] = l1.w;
        hi1[0] = h1.x; hi1[1] = h1.y; hi1[2] = h1.z; hi1[3] = h1.w;
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[j][i] = 0.0f;
        cur_tile = tile;
        seg_begin = a;
      }
      if (kg == 0 || a == a_begin) {
        const uint32_t* sr = s_ab + ((long long)tile * NG + grp - rec_lo) * kTileRows + g;
        const uint32_t s0 = sr[0], s1 = sr[8];
        al0 = prmt(s0, s0, 0x1010u); be0 = prmt(s0, s0, 0x3232u);   // (alpha, alpha), (beta, beta)
        al1 = prmt(s1, s1, 0x1010u); be1 = prmt(s1, s1, 0x3232u);
      }
      const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t af[4];
        decode_word(words[s], lo0, hi0, lo1, hi1, af);
        af[0] = fma_bf16x2(af[0], al0, be0);
        af[2] = fma_bf16x2(af[2], al0, be0);
        af[1] = fma_bf16x2(af[1], al1, be1);
        af[3] = fma_bf16x2(af[3], al1, be1);
#pragma unroll
        for (int j = 0; j < NT; ++j) mma_m16n8k16(acc[j], af, xc[j][s][0], xc[j][s][1]);
      }
      // advance to the next atom
      if (++kg == atoms_per_group) { kg = 0; ++grp; }
      ka = ka_next;
      if (ka == 0) { ++tile; grp = 0; kg = 0; }
    }
  }
  if (cur_tile >= 0) finish_segment<NT>(p, wid, lane, cur_tile, seg_begin, a_end, a_begin, acc);
}

// Dynamic shared memory of one CTA: the LUTs of the tiles and the scale
// records of the groups its atom range touches (bounded by the widest CTA).
size_t linear_smem_bytes(const Layout& L, long long atoms, int warps) {
  const long long per_warp = (atoms + warps - 1) / warps;
  const long long per_cta = per_warp * kWarpsPerCta + 1;
  const long long tiles = per_cta / L.katoms + 2;
  const long long recs = per_cta * kAtomK / L.g + 2;
  return (size_t)(tiles * kTileRows * 32 + recs * kTileRows * 4);
}

// Opt the kernels in to more than 48 KB of dynamic shared memory (once per
// device; the attribute is per function and device).
cudaError_t allow_large_smem() {
  static std::atomic<unsigned long long> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(linear_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kMaxSmemPerCta);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(linear_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kMaxSmemPerCta);
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

}  // namespace

LinearPlan plan_linear(int m, const Layout& L, int num_sms) {
  LinearPlan pl{};
  pl.nt = m > 8 ? 2 : 1;
  pl.atoms = (long long)L.tiles * L.katoms;
  long long w = pl.atoms / kMinAtomsPerWarp;
  const long long cap = (long long)num_sms * kCtasPerSm * kWarpsPerCta;
  if (w > cap) w = cap;
  if (w < 1) w = 1;
  pl.warps = (int)w;
  pl.ctas = (pl.warps + kWarpsPerCta - 1) / kWarpsPerCta;
  pl.counters_bytes = (size_t)kMaxTiles * sizeof(unsigned);   // same for every shape
  pl.partials_bytes = align_up((size_t)2 * pl.warps * 32 * 4 * pl.nt * sizeof(float), kAlign);
  pl.workspace_bytes = pl.counters_bytes + pl.partials_bytes;
  pl.smem_bytes = linear_smem_bytes(L, pl.atoms, pl.warps);
  return pl;
}

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream) {
  LinearArgs p{};
  p.x = x;
  p.packed = packed;
  p.y = y;
  p.counters = reinterpret_cast<unsigned*>(workspace);
  p.partials = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + plan.counters_bytes);
  p.L = L;
  p.m = m;
  p.warps = plan.warps;
  p.atoms = plan.atoms;
  const dim3 block(kWarpsPerCta * 32);
  const size_t smem = linear_smem_bytes(L, plan.atoms, plan.warps);
  if (smem > kMaxSmemPerCta) return cudaErrorInvalidValue;
  cudaError_t e = smem > 48 * 1024 ? allow_large_smem() : cudaSuccess;
  if (e != cudaSuccess) return e;
  if (plan.nt == 1)
    linear_kernel<1><<<plan.ctas, block, smem, stream>>>(p);
  else
    linear_kernel<2><<<plan.ctas, block, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace any4
