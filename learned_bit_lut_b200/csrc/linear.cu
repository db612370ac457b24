// any4_linear on B200 (sm_100a): y = x . W_hat^T with W stored as any4.
//
// Method (any4 explainer, 10100.com article 149119421): every row of W has its
// own table (LUT) of 16 bf16 values and every weight is a 4-bit index into it
// (section 2); each contiguous group of G columns has a scale alpha and an
// offset beta (section 2.1); w_hat = fma(alpha, LUT[idx], beta). tinygemm
// (section 3) keeps the table next to the arithmetic and runs batch 1-16 on
// the tensor cores; this kernel is a fresh design for Blackwell.
//
// One persistent CTA per SM, 14 warps with fixed roles:
//  * warps 0-7, two decoder warpgroups. Thread r of a warpgroup owns weight
//    row r of the current 128-row tile, which is also Tensor Memory lane r.
//    For every (tile, 64-column chunk) "unit" the warpgroup's threads read
//    their row's 32 index bytes (one 512-byte coalesced load per warp and
//    half), turn each byte -- the indices of two adjacent columns -- into a
//    bf16 pair with ONE shared-memory load from a per-row pair table
//    (256 entries: (LUT[lo nibble], LUT[hi nibble])), apply alpha/beta with
//    one bf16x2 fma, and store the 64 weights of the row into a Tensor Memory
//    operand buffer (tcgen05.st). The two warpgroups take alternate units.
//  * warp 13 loads the matching 16 x 64 activation chunk with TMA (128-byte
//    swizzle; rows past M are zero-filled by TMA).
//  * warp 12 issues tcgen05.mma (M=128, N=16, K=16; A from Tensor Memory, B =
//    activations from shared memory) accumulating fp32 in Tensor Memory.
//  * warps 8-11 read the accumulator back at the end of each tile segment and
//    write y (bf16) or, for a tile split between CTAs, an fp32 partial; the
//    last CTA to finish a split tile sums the partials in CTA order (fixed,
//    deterministic) and writes y. Nobody waits for another CTA.
//  Stages hand over through mbarriers; every wait has a time limit after which
//  the CTA records an error bit in the workspace, skips the remaining work and
//  still releases its Tensor Memory.
//
// Work split: the units of all tiles form one sequence; CTA c gets an equal
// contiguous share (stream-K), so every SM streams the same number of bytes.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.cuh"

namespace any4 {

namespace {

constexpr int kDecoderThreads = 256;       // warps 0-7
constexpr int kEpilogueWarp0 = 8;          // warps 8-11
constexpr int kMmaWarp = 12;
constexpr int kThreads = 14 * 32;          // + warp 13: TMA
constexpr int kAStages = 4;                // Tensor Memory operand buffers per warpgroup
constexpr int kPrefetch = 4;               // units in flight per decoder thread (== kAStages)
constexpr int kXStages = 8;                // activation chunks in shared memory
constexpr int kTokens = 16;                // MMA N
constexpr int kXStageBytes = kTokens * kChunkK * 2;   // 2048
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDCol0 = 0;             // two 16-column fp32 accumulators
constexpr uint32_t kACol0 = 32;            // 8 operand buffers of 32 columns
constexpr uint32_t kACols = kChunkK / 2;
constexpr uint32_t kTableAddr = 65536;     // shared-window address of the pair tables
constexpr uint32_t kTableBlock = 65536;    // 256 entries x 64 rows x 4 bytes
constexpr int kSmemBytes = 232448;         // 227 KB: the per-block maximum
constexpr long long kWaitCycles = 4000000000ll;   // about 2 s, then give up

static_assert(kPrefetch == kAStages, "decoder ring slot doubles as operand slot");

// tcgen05 instruction descriptor (kind::f16): D fp32, A and B bf16, both
// K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            ((uint32_t)(kTokens >> 3) << 17) | ((uint32_t)(kTileRows >> 4) << 24);

enum : unsigned {
  kErrAEmpty = 1u, kErrAFull = 2u, kErrXEmpty = 4u, kErrXFull = 8u, kErrDEmpty = 16u,
  kErrDFull = 32u, kErrSmem = 64u, kErrDrain = 128u
};

struct Params {
  const uint8_t* packed;
  uint16_t* y;
  float* partials;
  unsigned* counters;
  unsigned* error;
  int m, n, k, g;
  int chunks, groups, gshift;
  int ctas;
  long long units;
  size_t w_off, lut_off, ab_off;
};

struct SmemCtl {
  uint64_t a_full[2][kAStages];
  uint64_t a_empty[2][kAStages];
  uint64_t x_full[kXStages];
  uint64_t x_empty[kXStages];
  uint64_t d_full[2];
  uint64_t d_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  unsigned ticket;
};

// ------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
      : "memory");
}

__device__ __forceinline__ void tc_st_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tc_ld_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor of one 16-token x 16-column activation slice:
// K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t x_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Bounded wait on an mbarrier phase. Gives up (returns false) when the CTA is
// already aborting, or after kWaitCycles, in which case it starts the abort.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned* err, unsigned code) {
  if (*abort_flag) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      atomicOr(err, code);
      return false;
    }
  }
}

// CTA that owns unit u under the split U0(c) = floor(c * U / C).
__device__ __forceinline__ int cta_of_unit(long long u, long long units, int ctas) {
  return (int)(((u + 1) * (long long)ctas - 1) / units);
}

// ----------------------------------------------------------- pair tables

// Build this warpgroup's half (entries 128*wg .. 128*wg+127) of the pair table
// of row r: entry e = (LUT[e & 15], LUT[e >> 4]) as a bf16 pair, so the index
// byte of two adjacent columns looks up both weights at once. `lut` holds the
// row's 16 bf16 values as 8 pairs. Framed by decoder barriers so no thread
// still reads the previous table and none reads this one half-built.
__device__ __noinline__ void build_table(uint32_t row_base, const uint32_t* lut, int wg) {
  named_bar_sync(1, kDecoderThreads);
  uint32_t lo[8], hi[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) lo[i] = lut[i];
#pragma unroll
  for (int h = 0; h < 4; ++h) hi[h] = wg ? lo[4 + h] : lo[h];
  const uint32_t addr0 = row_base + (uint32_t)wg * 128u * 256u;
#pragma unroll
  for (int i = 0; i < 128; ++i) {
    const int lo_idx = i & 15, hi_idx = i >> 4;     // high nibble = 8 * wg + hi_idx
    const uint32_t sel = ((lo_idx & 1) ? 0x32u : 0x10u) | (((hi_idx & 1) ? 0x76u : 0x54u) << 8);
    sts32(addr0 + (uint32_t)i * 256u, prmt(lo[lo_idx >> 1], hi[hi_idx >> 1], sel));
  }
  named_bar_sync(1, kDecoderThreads);
}

__device__ __forceinline__ void load_lut(const Params& p, int tile, int r, uint32_t (&lut)[8]) {
  const uint4* src = reinterpret_cast<const uint4*>(p.packed + p.lut_off +
                                                    ((size_t)tile * kTileRows + r) * 32);
  const uint4 a = ld_nc_v4(src), b = ld_nc_v4(src + 1);
  lut[0] = a.x; lut[1] = a.y; lut[2] = a.z; lut[3] = a.w;
  lut[4] = b.x; lut[5] = b.y; lut[6] = b.z; lut[7] = b.w;
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kThreads, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmap, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(base + kXStages * kXStageBytes);
  const uint32_t x_addr0 = base_addr;

  // The pair tables sit at a fixed shared address so one byte permute forms a
  // lookup address; the ring and control block must fit below it.
  if (smem_u32(ctl + 1) > kTableAddr || kTableAddr + 2 * kTableBlock > raw_addr + kSmemBytes) {
    if (threadIdx.x == 0) atomicOr(p.error, kErrSmem);
    return;
  }

  const long long U = p.units;
  const long long U0 = (long long)blockIdx.x * U / p.ctas;
  const long long U1 = (long long)(blockIdx.x + 1) * U / p.ctas;
  const long long nunits = U1 - U0;
  const int C = p.chunks;
  const int t_first = (int)(U0 / C);
  const int t_last = (int)((U1 - 1) / C);

  volatile int* abort_flag = &ctl->abort_flag;
  if (threadIdx.x == 0) {
    for (int w = 0; w < 2; ++w)
      for (int s = 0; s < kAStages; ++s) {
        mbar_init(smem_u32(&ctl->a_full[w][s]), 4);    // one arrival per decoder warp
        mbar_init(smem_u32(&ctl->a_empty[w][s]), 1);   // tcgen05.commit
      }
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(smem_u32(&ctl->x_full[s]), 1);         // expect_tx arrival + bytes
      mbar_init(smem_u32(&ctl->x_empty[s]), 1);        // tcgen05.commit
    }
    for (int d = 0; d < 2; ++d) {
      mbar_init(smem_u32(&ctl->d_full[d]), 1);         // tcgen05.commit
      mbar_init(smem_u32(&ctl->d_empty[d]), 4);        // one arrival per epilogue warp
    }
    mbar_init(smem_u32(&ctl->mma_done), 1);
    ctl->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ctl->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < 8) {
    // ------------------------------------------------------------ decoders
    const int wg = warp >> 2, q = warp & 3, r = q * 32 + lane;
    const uint32_t row_base = kTableAddr + (uint32_t)(r >> 6) * kTableBlock + 4u * (r & 63);
    const uint32_t addr_bytes = (4u * (r & 63)) | ((1u + (uint32_t)(r >> 6)) << 16);
    const uint32_t lane_tmem = tmem + ((uint32_t)(q * 32) << 16);
    const uint8_t* wsrc = p.packed + p.w_off + (size_t)q * 1024 + (size_t)lane * 16;
    const uint32_t* absrc = reinterpret_cast<const uint32_t*>(p.packed + p.ab_off) + r;

    // the prefetch head walks this warpgroup's units (every second one)
    long long up = U0 + wg;
    int tile_p = (int)(up / C), chunk_p = (int)(up - (long long)tile_p * C);
    uint4 v0[kPrefetch], v1[kPrefetch];
    uint32_t ab[kPrefetch];
    auto issue = [&](int s) {
      const uint8_t* src = wsrc + (size_t)up * kUnitBytes;
      v0[s] = ld_stream_v4(src);
      v1[s] = ld_stream_v4(src + 512);
      ab[s] = ld_nc_u32(absrc + ((size_t)tile_p * p.groups + (chunk_p >> p.gshift)) * kTileRows);
      up += 2;
      chunk_p += 2;
      while (chunk_p >= C) { chunk_p -= C; ++tile_p; }
    };
#pragma unroll
    for (int s = 0; s < kPrefetch; ++s)
      if (up < U1) issue(s);

    long long uc = U0 + wg;                        // unit being decoded
    int tile_c = (int)(uc / C), chunk_c = (int)(uc - (long long)tile_c * C);
    int built = t_first - 1;                       // last tile whose table is built
    uint32_t lut_next[8];
    load_lut(p, t_first, r, lut_next);

    for (int n0 = 0;; n0 += kPrefetch) {
      bool done = false;
#pragma unroll
      for (int s = 0; s < kPrefetch; ++s) {
        if (uc >= U1) { done = true; break; }
        while (built < tile_c) {
          build_table(row_base, lut_next, wg);
          ++built;
          if (built < t_last) load_lut(p, built + 1, r, lut_next);
        }
        const uint4 a = v0[s], b = v1[s];
        const uint32_t sab = ab[s];
        if (up < U1) issue(s);
        const uint32_t use = (uint32_t)(n0 / kPrefetch);
        if (wait_bar(smem_u32(&ctl->a_empty[wg][s]), (use & 1u) ^ 1u, abort_flag, p.error,
                     kErrAEmpty)) {
          const uint32_t al = prmt(sab, sab, 0x1010u), be = prmt(sab, sab, 0x3232u);
          const uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          uint32_t out[32];
#pragma unroll
          for (int wi = 0; wi < 8; ++wi)
#pragma unroll
            for (int bi = 0; bi < 4; ++bi) {
              const uint32_t addr = prmt(words[wi], addr_bytes, 0x7604u | ((uint32_t)bi << 4));
              out[wi * 4 + bi] = fma_bf16x2(lds32(addr), al, be);
            }
          tc_st_x32(lane_tmem + kACol0 + (uint32_t)(wg * kAStages + s) * kACols, out);
          tc_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->a_full[wg][s]));
        uc += 2;
        chunk_c += 2;
        while (chunk_c >= C) { chunk_c -= C; ++tile_c; }
      }
      if (done) break;
    }
    // both warpgroups build every tile's table, so their barriers pair up
    while (built < t_last) {
      build_table(row_base, lut_next, wg);
      ++built;
      if (built < t_last) load_lut(p, built + 1, r, lut_next);
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_tmem = tmem + ((uint32_t)(q * 32) << 16);
    for (int t = t_first; t <= t_last; ++t) {
      const int s = t - t_first, d = s & 1;
      const long long sb = max(U0, (long long)t * C), se = min(U1, (long long)(t + 1) * C);
      uint32_t raw[16];
      const bool ok = wait_bar(smem_u32(&ctl->d_full[d]), (uint32_t)(s >> 1) & 1u, abort_flag,
                               p.error, kErrDFull);
      if (ok) {
        tc_fence_after();
        tc_ld_x16(lane_tmem + kDCol0 + 16u * d, raw);
        tc_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->d_empty[d]));
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = ok ? __uint_as_float(raw[i]) : 0.0f;
      const int n_row = t * kTileRows + r;
      const bool full = sb == (long long)t * C && se == (long long)(t + 1) * C;
      if (full) {
        if (ok && n_row < p.n)
          for (int m = 0; m < p.m; ++m) {
            const __nv_bfloat16 h = __float2bfloat16_rn(v[m]);
            p.y[(size_t)m * p.n + n_row] = *reinterpret_cast<const uint16_t*>(&h);
          }
        continue;
      }
      // split tile: publish this CTA's fp32 partial (the token columns that
      // exist); the last CTA to arrive sums them
      const int nq = (p.m + 3) >> 2;
      const int my_slot = 2 * blockIdx.x + (t == t_first ? 0 : 1);
      float4* dst = reinterpret_cast<float4*>(p.partials + ((size_t)my_slot * kTileRows + r) * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i < nq) __stcg(dst + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
      __threadfence();
      named_bar_sync(2, 128);
      if (warp == kEpilogueWarp0 && lane == 0) ctl->ticket = atomicAdd(p.counters + t, 1u);
      named_bar_sync(2, 128);
      const int c_first = cta_of_unit((long long)t * C, U, p.ctas);
      const int c_last = cta_of_unit((long long)(t + 1) * C - 1, U, p.ctas);
      if (ctl->ticket != (unsigned)(c_last - c_first)) continue;
      __threadfence();
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
      // contributors in CTA order; a batch's loads are all issued before it is summed
      constexpr int kBatch = 8;
      for (int i = 0; i < nq; ++i)
        for (int c0 = c_first; c0 <= c_last; c0 += kBatch) {
          float4 f[kBatch];
#pragma unroll
          for (int b = 0; b < kBatch; ++b) {
            const int c = c0 + b;
            f[b] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c <= c_last) {
              const long long cu0 = (long long)c * U / p.ctas;
              const int slot = 2 * c + ((long long)t == cu0 / C ? 0 : 1);
              f[b] = __ldcg(reinterpret_cast<const float4*>(
                                p.partials + ((size_t)slot * kTileRows + r) * 16) + i);
            }
          }
#pragma unroll
          for (int b = 0; b < kBatch; ++b) {
            acc[4 * i] += f[b].x; acc[4 * i + 1] += f[b].y;
            acc[4 * i + 2] += f[b].z; acc[4 * i + 3] += f[b].w;
          }
        }
      if (n_row < p.n && !*abort_flag)
        for (int m = 0; m < p.m; ++m) {
          const __nv_bfloat16 h = __float2bfloat16_rn(acc[m]);
          p.y[(size_t)m * p.n + n_row] = *reinterpret_cast<const uint16_t*>(&h);
        }
      if (warp == kEpilogueWarp0 && lane == 0) p.counters[t] = 0u;   // ready for the next call
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      long long j = 0;
      for (int t = t_first; t <= t_last; ++t) {
        const int s = t - t_first, d = s & 1;
        const long long se = min(U1, (long long)(t + 1) * C);
        wait_bar(smem_u32(&ctl->d_empty[d]), ((uint32_t)(s >> 1) & 1u) ^ 1u, abort_flag, p.error,
                 kErrDEmpty);
        tc_fence_after();
        bool first = true;
        for (; U0 + j < se; ++j) {
          const int wg = (int)(j & 1), slot = (int)((j >> 1) & (kAStages - 1));
          const uint32_t use = (uint32_t)(j >> 3);
          const int xs = (int)(j & (kXStages - 1));
          const bool ok =
              wait_bar(smem_u32(&ctl->a_full[wg][slot]), use & 1u, abort_flag, p.error, kErrAFull) &&
              wait_bar(smem_u32(&ctl->x_full[xs]), (uint32_t)(j >> 3) & 1u, abort_flag, p.error,
                       kErrXFull);
          if (ok) {
            tc_fence_after();
            const uint32_t a_col = tmem + kACol0 + (uint32_t)(wg * kAStages + slot) * kACols;
            const uint64_t desc = x_desc(x_addr0 + (uint32_t)xs * kXStageBytes);
#pragma unroll
            for (int i = 0; i < kChunkK / 16; ++i)
              tc_mma(tmem + kDCol0 + 16u * d, a_col + 8u * i, desc + 2u * i,
                     (first && i == 0) ? 0u : 1u);
            first = false;
          }
          tc_commit(smem_u32(&ctl->a_empty[wg][slot]));
          tc_commit(smem_u32(&ctl->x_empty[xs]));
        }
        tc_commit(smem_u32(&ctl->d_full[d]));
      }
      // every MMA has completed before Tensor Memory is released
      tc_commit(smem_u32(&ctl->mma_done));
      const long long t0 = clock64();
      while (!mbar_try_wait(smem_u32(&ctl->mma_done), 0)) {
        if (clock64() - t0 > kWaitCycles) { atomicOr(p.error, kErrDrain); break; }
      }
    }
  } else {
    // ----------------------------------------------------------------- TMA
    if (lane == 0) {
      int chunk = (int)(U0 - (long long)t_first * C);
      int last_use[kXStages];
#pragma unroll
      for (int s = 0; s < kXStages; ++s) last_use[s] = -1;
      for (long long j = 0; j < nunits; ++j) {
        const int xs = (int)(j & (kXStages - 1));
        const uint32_t use = (uint32_t)(j >> 3);
        if (wait_bar(smem_u32(&ctl->x_empty[xs]), (use & 1u) ^ 1u, abort_flag, p.error, kErrXEmpty)) {
          mbar_arrive_expect_tx(smem_u32(&ctl->x_full[xs]), kXStageBytes);
          tma_load_2d(x_addr0 + (uint32_t)xs * kXStageBytes, &tmap, chunk * kChunkK, 0,
                      smem_u32(&ctl->x_full[xs]));
          last_use[xs] = (int)use;
        }
        if (++chunk == C) chunk = 0;
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int s = 0; s < kXStages; ++s) {
        if (last_use[s] < 0) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(smem_u32(&ctl->x_full[s]), (uint32_t)last_use[s] & 1u)) {
          if (clock64() - t0 > kWaitCycles) { atomicOr(p.error, kErrDrain); break; }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<void*> fn{nullptr};
  void* f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn.store(f, std::memory_order_release);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

cudaError_t allow_large_smem() {
  static std::atomic<unsigned long long> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

}  // namespace

LinearPlan plan_linear(int m, const Layout& L, int num_sms) {
  (void)m;
  LinearPlan pl{};
  pl.units = (long long)L.tiles * L.chunks;
  long long c = pl.units / 2;                  // at least two units per CTA
  if (c > num_sms) c = num_sms;
  if (c < 1) c = 1;
  pl.ctas = (int)c;
  pl.partials_bytes = (size_t)2 * pl.ctas * kTileRows * 16 * sizeof(float);
  pl.workspace_bytes = kHeaderBytes + pl.partials_bytes;
  return pl;
}

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  cudaError_t e = allow_large_smem();
  if (e != cudaSuccess) return e;

  // activations: K x M bf16 (inner dimension first), 64 x 16 boxes, 128-byte
  // swizzle; rows past M read as zero.
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)L.k, (cuuint64_t)m};
  const cuuint64_t strides[1] = {(cuuint64_t)L.k * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kChunkK, (cuuint32_t)kTokens};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  Params p{};
  p.packed = packed;
  p.y = y;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  p.counters = reinterpret_cast<unsigned*>(ws);
  p.error = reinterpret_cast<unsigned*>(ws + kCountersBytes);
  p.partials = reinterpret_cast<float*>(ws + kHeaderBytes);
  p.m = m; p.n = L.n; p.k = L.k; p.g = L.g;
  p.chunks = L.chunks; p.groups = L.groups;
  p.gshift = 0;
  while ((kChunkK << p.gshift) < L.g) ++p.gshift;
  p.ctas = plan.ctas;
  p.units = plan.units;
  p.w_off = L.w_off; p.lut_off = L.lut_off; p.ab_off = L.ab_off;
  linear_tc_kernel<<<plan.ctas, kThreads, kSmemBytes, stream>>>(tmap, p);
  return cudaGetLastError();
}

}  // namespace any4
