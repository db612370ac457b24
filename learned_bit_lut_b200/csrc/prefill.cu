// any4_linear for M > 16 (prefill): y = x . W_hat^T as a tensor-core GEMM.
//
// Beyond the explainer's batch 1-16 regime (10100.com article 149119421,
// section 3: tinygemm runs small batches on the tensor cores) the product is
// compute bound. Both paths run tcgen05 MMAs (M = 128 weight rows, N = the
// token tile, K = 16 per instruction) from 128-byte-swizzled K-major tiles
// in shared memory into fp32 accumulators in tensor memory, with 4 pipeline
// stages and two accumulators so the epilogue of one tile overlaps the main
// loop of the next; when there are fewer output tiles than SMs, up to 4
// blocks share a tile's K range (split-K) and the last one to arrive adds
// the fp32 partials in split order (deterministic).
//
//  * any4, M <= 512 (prefill_fused_kernel): decoder warps expand the packed
//    weight tile straight into the A stages, with every row's table held in
//    registers (regdecode.cuh) and w_hat = fma(alpha, LUT[idx], beta)
//    (sections 2-2.1) rounded once to bf16; TMA brings the activation tile.
//    Each packed weight byte crosses HBM once and no bf16 copy of W exists.
//    On B200 a tcgen05.mma costs ~143 cycles whatever N is (measured for
//    N = 16..256), so at small M the MMA count, not the FLOPs, bounds the
//    tensor side, and the byte-permute decode (integer pipe) bounds the rest.
//  * any4 M > 512, any3 / any2: dequantize W into a bf16 N x K scratch in the
//    caller's workspace (dequant_tile_kernel in pack_dequant.cu, bit-exact
//    like any4_dequant), then prefill_gemm_kernel brings both operands in by
//    TMA (tiles of 128 rows x 256 tokens). The decode then runs once per
//    call instead of once per 256-token tile.
//
// Warps of prefill_gemm_kernel: 0 = TMA producer, 1 = MMA issuer (and
// tensor-memory owner), 2-5 = epilogue (warp w reads tensor-memory lanes
// 32*(w%4) .. +31). Every mbarrier wait is bounded (~2 s); a timeout sets the
// workspace status word and the block winds down.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.cuh"
#include "regdecode.cuh"

namespace any4 {

namespace {

constexpr int kBM = 128;                       // weight rows per tile (MMA M)
constexpr int kBN = 256;                       // tokens per tile (MMA N)
constexpr int kBK = 64;                        // K per stage: one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kAStageBytes = kBM * kBK * 2;    // 16 KB
constexpr int kBStageBytes = kBN * kBK * 2;    // 32 KB
constexpr int kStageBytes = kAStageBytes + kBStageBytes;
constexpr int kGemmThreads = 192;
constexpr uint32_t kAccCols = kBN;             // fp32 columns per accumulator
constexpr uint32_t kTmemCols = 2 * kAccCols;   // two accumulators
constexpr int kGemmSmem = kStages * kStageBytes + 1024 + 1024;   // stages, control, alignment
constexpr long long kGemmWaitCycles = 4000000000ll;

// tcgen05 instruction descriptor, kind::f16: D fp32, A and B bf16, both
// K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

struct GemmCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort_flag;
  int last_split;   // epilogue: this block finishes the tile's split-K sum
};

constexpr int kEpilogueBar = 1;                 // named barrier of the 4 epilogue warps
constexpr int kPartialFloats = kBM * kBN;       // one split's fp32 tile [token][row]
constexpr int kMinSplitChunks = 8;              // K per split >= 8 stages (512 columns)
constexpr int kMaxSplits = 4;                   // the last block reads all splits' partials

__device__ __forceinline__ void epilogue_sync() {
  asm volatile("bar.sync %0, 128;" ::"n"(kEpilogueBar) : "memory");
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_arrive_one(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait; false when the block is aborting or the wait timed out.
__device__ __forceinline__ bool gemm_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kGemmWaitCycles) {
      *abort_flag = 1;
      atomicOr(status, kStatusWaitTimeout);
      return false;
    }
  }
}

// gemm_wait for warps that wait long (a whole tile) and must not take issue
// slots from the warps doing the work meanwhile: sleeps between polls.
__device__ __forceinline__ bool gemm_wait_idle(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                               unsigned* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(200);
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kGemmWaitCycles) {
      *abort_flag = 1;
      atomicOr(status, kStatusWaitTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// arrives once on `bar` when every tcgen05.mma this thread issued so far is complete
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
      : "memory");
}

__device__ __forceinline__ void tc_ld_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    prefill_gemm_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                        uint16_t* __restrict__ y, int m, int n, int k, int splits, float* __restrict__ partials,
                        unsigned* counters, unsigned* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;   // swizzle atoms need 1024-byte alignment
  GemmCtl* ctl = reinterpret_cast<GemmCtl*>(smem_raw + (sbase - raw) + kStages * kStageBytes);
  auto sa = [&](int s) { return sbase + (uint32_t)s * kStageBytes; };
  auto sb = [&](int s) { return sbase + (uint32_t)s * kStageBytes + kAStageBytes; };
  volatile int* abort_flag = &ctl->abort_flag;

  const int n_tiles = (n + kBM - 1) / kBM, m_tiles = (m + kBN - 1) / kBN;
  const int tiles = n_tiles * m_tiles, kch = k / kBK;
  const int units = tiles * splits;   // unit u: tile u / splits, K split u % splits
  auto k_range = [&](int u, int& kc0, int& kc1) {
    const int sp = u % splits;
    kc0 = (int)((long long)sp * kch / splits);
    kc1 = (int)((long long)(sp + 1) * kch / splits);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&ctl->full[s]), 1);    // TMA expect_tx arrival + bytes
      mbar_init(smem_addr(&ctl->empty[s]), 1);   // tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&ctl->acc_full[b]), 1);    // tcgen05.commit
      mbar_init(smem_addr(&ctl->acc_empty[b]), 4);   // one arrival per epilogue warp
    }
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&ctl->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  asm volatile("griddepcontrol.wait;" ::: "memory");   // x (and the dequantized W) are ready

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int it = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int tile = u / splits;
        const int nt = tile / m_tiles, mt = tile % m_tiles;
        int kc0, kc1;
        k_range(u, kc0, kc1);
        for (int kc = kc0; kc < kc1; ++kc, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (it >= kStages &&
              !gemm_wait(smem_addr(&ctl->empty[s]), ph ^ 1u, abort_flag, status))
            break;
          const uint32_t fb = smem_addr(&ctl->full[s]);
          mbar_arrive_expect_tx(fb, kStageBytes);
          tma_load_2d(sa(s), &wmap, kc * kBK, nt * kBM, fb);
          tma_load_2d(sb(s), &xmap, kc * kBK, mt * kBN, fb);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0, tcount = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x, ++tcount) {
        const int b = tcount & 1;
        const uint32_t aph = (uint32_t)(tcount >> 1) & 1u;
        if (tcount >= 2 && !gemm_wait(smem_addr(&ctl->acc_empty[b]), aph ^ 1u, abort_flag, status))
          break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)b * kAccCols;
        int kc0, kc1;
        k_range(u, kc0, kc1);
        for (int kc = kc0; kc < kc1; ++kc, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!gemm_wait(smem_addr(&ctl->full[s]), ph, abort_flag, status)) break;
          tc_fence_after();
          const uint64_t ad = sw128_desc(sa(s)), bd = sw128_desc(sb(s));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)   // 16 columns = 32 bytes = 2 descriptor units
            tc_mma(d, ad + 2u * (uint64_t)kk, bd + 2u * (uint64_t)kk, (kc > kc0 || kk > 0) ? 1u : 0u);
          tc_commit(smem_addr(&ctl->empty[s]));   // the stage is free once these MMAs are done
        }
        tc_commit(smem_addr(&ctl->acc_full[b]));
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;   // tensor-memory lane quarter of this warp
    int tcount = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++tcount) {
      const int tile = u / splits;
      const int nt = tile / m_tiles, mt = tile % m_tiles;
      const int b = tcount & 1;
      const uint32_t ph = (uint32_t)(tcount >> 1) & 1u;
      gemm_wait(smem_addr(&ctl->acc_full[b]), ph, abort_flag, status);
      epilogue_sync();          // all four warps leave together if any wait gave up
      if (*abort_flag) break;
      tc_fence_after();
      const int r = 32 * q + lane, row = nt * kBM + r;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)b * kAccCols;
      float* part = partials + (size_t)u * kPartialFloats;   // [token][row] of this split
#pragma unroll 1
      for (int j = 0; j < kBN / 32; ++j) {
        uint32_t v[32];
        tc_ld_x32(tbase + 32u * (uint32_t)j, v);
        tc_wait_ld();
        const int m0 = mt * kBN + 32 * j;
        if (splits > 1) {
#pragma unroll
          for (int i = 0; i < 32; ++i) __stcg(part + (32 * j + i) * kBM + r, __uint_as_float(v[i]));
        } else if (row < n) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (m0 + i < m) {
              const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[i]));
              y[(size_t)(m0 + i) * n + row] = *reinterpret_cast<const uint16_t*>(&h);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(smem_addr(&ctl->acc_empty[b]));
      if (splits > 1) {
        // publish this split; the last of the tile's splits adds them in order
        __threadfence();
        epilogue_sync();
        if (q == 0 && lane == 0) ctl->last_split = atomicAdd(counters + tile, 1u) == (unsigned)(splits - 1);
        epilogue_sync();
        if (ctl->last_split) {
          __threadfence();
          const float* base = partials + (size_t)tile * splits * kPartialFloats;
          if (row < n) {
            // 32 tokens at a time, so 32 loads of each split are in flight together
#pragma unroll 1
            for (int j0 = 0; j0 < kBN && mt * kBN + j0 < m; j0 += 32) {
              float acc[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
#pragma unroll 1
              for (int sp = 0; sp < splits; ++sp) {
                const float* src = base + (size_t)sp * kPartialFloats + j0 * kBM + r;
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] += __ldcg(src + i * kBM);
              }
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int mm = mt * kBN + j0 + i;
                if (mm < m) {
                  const __nv_bfloat16 h = __float2bfloat16_rn(acc[i]);
                  y[(size_t)mm * n + row] = *reinterpret_cast<const uint16_t*>(&h);
                }
              }
            }
          }
          epilogue_sync();
          if (q == 0 && lane == 0) counters[tile] = 0u;   // ready for the next call
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
}

// =============================================================================
// Fused prefill (any4): the weight tile is decoded straight into the GEMM's
// shared-memory stages, so every packed weight byte crosses HBM once and no
// bf16 copy of W is written or read back.
//
// Warps: 0 = TMA producer of the activation tiles, 1 = MMA issuer (and
// tensor-memory owner), 2-5 = epilogue, 6-13 = decoders. Decoder warp
// (p, h) expands half h of each 64-column stage of 32-row panel p of the
// 128-row tile: lane (g, t) holds the tables of rows g, g+8, g+16, g+24 as
// byte planes (regdecode.cuh), turns its row-pair index words (layout.cuh)
// into per-row selectors, decodes columns 16t + 8h .. 16t + 8h + 7 of each of
// its rows, scales them (one fma.rn.bf16x2 per pair: w_hat rounded once to
// bf16) and stores each row's 8 columns as one 16-byte run in the
// 128-byte-swizzled K-major layout the MMA descriptor expects (the layout a
// TMA load with SWIZZLE_128B writes). The decode is bound by the integer
// pipe (prmt at half rate), so two warps per panel keep each scheduler's
// pipe busy. Stage s is full when the TMA bytes of x have landed and all
// decoder warps have arrived.
constexpr int kFusedDecoders = 8;
constexpr int kFusedThreads = (6 + kFusedDecoders) * 32;
constexpr int kFusedStages = 4;

template <int BN>
struct FusedCfg {
  static constexpr int kBStage = BN * kBK * 2;
  static constexpr int kStage = kAStageBytes + kBStage;
  static constexpr uint32_t kTmem = 2 * BN;   // two accumulators (a power of two >= 32)
  static constexpr int kSmem = kFusedStages * kStage + 1024 + 1024;
  static constexpr uint32_t kIdescN = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((uint32_t)(kBM >> 4) << 24);
};

struct FusedCtl {
  uint64_t full[kFusedStages];
  uint64_t empty[kFusedStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort_flag;
  int last_split;
};

struct FusedParams {
  const uint8_t* packed;
  size_t w_off, lut_off, ab_off;
  int panels, kchunks, groups, g_shift;
};

template <int BN>
__device__ __forceinline__ void tc_mma_n(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(accumulate), "r"(FusedCfg<BN>::kIdescN)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int BN>
__global__ void __launch_bounds__(kFusedThreads, 1)
    prefill_fused_kernel(const __grid_constant__ CUtensorMap xmap, const FusedParams fp, uint16_t* __restrict__ y,
                         int m, int n, int k, int splits, float* __restrict__ partials, unsigned* counters,
                         unsigned* status) {
  using C = FusedCfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;   // swizzle atoms need 1024-byte alignment
  FusedCtl* ctl = reinterpret_cast<FusedCtl*>(smem_raw + (sbase - raw) + kFusedStages * C::kStage);
  auto sa = [&](int s) { return sbase + (uint32_t)s * C::kStage; };
  auto sb = [&](int s) { return sbase + (uint32_t)s * C::kStage + kAStageBytes; };
  volatile int* abort_flag = &ctl->abort_flag;

  const int n_tiles = (n + kBM - 1) / kBM, m_tiles = (m + BN - 1) / BN;
  const int tiles = n_tiles * m_tiles, kch = k / kBK;
  const int units = tiles * splits;   // unit u: tile u / splits, K split u % splits
  auto k_range = [&](int u, int& kc0, int& kc1) {
    const int sp = u % splits;
    kc0 = (int)((long long)sp * kch / splits);
    kc1 = (int)((long long)(sp + 1) * kch / splits);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFusedStages; ++s) {
      mbar_init(smem_addr(&ctl->full[s]), 1 + kFusedDecoders);   // TMA expect_tx + one per decoder warp
      mbar_init(smem_addr(&ctl->empty[s]), 1);                   // tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&ctl->acc_full[b]), 1);
      mbar_init(smem_addr(&ctl->acc_empty[b]), 4);
    }
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&ctl->tmem_base)),
                 "r"(C::kTmem)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp >= 6) {
    // ------------------------------------------------------------ decoders
    // The packed weight is immutable: decoding starts before the wait for
    // the previous kernel on the stream.
    const int p = (warp - 6) >> 1, half = (warp - 6) & 1, g = lane >> 2, t = lane & 3;
    const uint4* wsec = reinterpret_cast<const uint4*>(fp.packed + fp.w_off);
    const uint4* lsec = reinterpret_cast<const uint4*>(fp.packed + fp.lut_off);
    const uint4* asec = reinterpret_cast<const uint4*>(fp.packed + fp.ab_off);
    // this warp's 4 words of a chunk: steps 4h .. 4h+3 (half h of the chunk's
    // [half][lane][4 words] layout), columns 16t + 8h .. +7
    const int woff = 32 * half + lane;
    int it = 0;
    for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
      const int nt = (u / splits) / m_tiles;
      const int P = nt * (kBM / kPanelRows) + p;
      const bool live = P < fp.panels;   // the last tile may end before this panel
      int kc0, kc1;
      k_range(u, kc0, kc1);
      Planes T[4] = {};
      if (live) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {   // rows g, g+8, g+16, g+24 of the panel
          const uint4* row = lsec + ((size_t)P * kPanelRows + g + 8 * r) * 2;
          T[r] = to_planes(ld_nc_v4(row), ld_nc_v4(row + 1));
        }
      }
      // index words and scale record of chunk c (zeros past the tile's rows)
      auto words_of = [&](int c) {
        return live ? ld_stream_v4(wsec + ((size_t)P * fp.kchunks + c) * 64 + woff) : make_uint4(0u, 0u, 0u, 0u);
      };
      auto scales_of = [&](int c) {
        return live ? ld_nc_v4(asec + ((size_t)P * fp.groups + ((c * kBK) >> fp.g_shift)) * 8 + g)
                    : make_uint4(0u, 0u, 0u, 0u);
      };
      // one 64-column stage: decode, scale, store, publish
      auto stage = [&](int kc, const uint4& wa, const uint4& rc) -> bool {
        const int s = it % kFusedStages;
        const uint32_t ph = (uint32_t)(it / kFusedStages) & 1u;
        ++it;
        uint32_t al[4], be[4];
        scale_pairs(rc, al, be);
        if (it > kFusedStages && !gemm_wait(smem_addr(&ctl->empty[s]), ph ^ 1u, abort_flag, status)) return false;
        uint32_t o[4][4];   // [row][bf16 pair]: columns 16t + 8h + 2i, +1
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {   // k16 step 2h + jj: columns 16t + 8h + 4jj .. +3
          uint32_t t0, t1;
          rowpair_to_selectors(jj ? wa.z : wa.x, jj ? wa.w : wa.y, t0, t1);
          uint32_t a[4], b[4];
          decode8(T[0], T[1], t0, a);   // rows g, g+8
          decode8(T[2], T[3], t1, b);   // rows g+16, g+24
          o[0][2 * jj] = fma_bf16x2(a[0], al[0], be[0]);
          o[0][2 * jj + 1] = fma_bf16x2(a[2], al[0], be[0]);
          o[1][2 * jj] = fma_bf16x2(a[1], al[1], be[1]);
          o[1][2 * jj + 1] = fma_bf16x2(a[3], al[1], be[1]);
          o[2][2 * jj] = fma_bf16x2(b[0], al[2], be[2]);
          o[2][2 * jj + 1] = fma_bf16x2(b[2], al[2], be[2]);
          o[3][2 * jj] = fma_bf16x2(b[1], al[3], be[3]);
          o[3][2 * jj + 1] = fma_bf16x2(b[3], al[3], be[3]);
        }
        // tile rows 32p + {g, g+8, g+16, g+24}; row r's 16-byte chunk c goes
        // to chunk position c ^ (r & 7) = c ^ g (past the tile's rows the
        // tables, indices and scales are zero, so the values are too)
        const uint32_t dst = sa(s) + (uint32_t)(32 * p + g) * 128u + (uint32_t)(((2 * t + half) ^ g) * 16);
#pragma unroll
        for (int r = 0; r < 4; ++r) sts128(dst + (uint32_t)r * 8u * 128u, o[r][0], o[r][1], o[r][2], o[r][3]);
        fence_proxy_async_smem();   // the tensor core reads these stores
        __syncwarp();
        if (lane == 0) mbar_arrive_one(smem_addr(&ctl->full[s]));
        return true;
      };
      // Two chunks in flight, in alternating register slots: the loads of
      // chunk kc + 2 go out before chunk kc is decoded.
      uint4 w0 = words_of(kc0), r0 = scales_of(kc0);
      uint4 w1 = make_uint4(0u, 0u, 0u, 0u), r1 = w1;
      if (kc0 + 1 < kc1) { w1 = words_of(kc0 + 1); r1 = scales_of(kc0 + 1); }
      bool ok = true;
      for (int kc = kc0; kc < kc1 && ok; kc += 2) {
        const uint4 wa = w0, ra = r0;
        if (kc + 2 < kc1) { w0 = words_of(kc + 2); r0 = scales_of(kc + 2); }
        ok = stage(kc, wa, ra);
        if (ok && kc + 1 < kc1) {
          const uint4 wb = w1, rb = r1;
          if (kc + 3 < kc1) { w1 = words_of(kc + 3); r1 = scales_of(kc + 3); }
          ok = stage(kc + 1, wb, rb);
        }
      }
      if (!ok) break;
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    asm volatile("griddepcontrol.wait;" ::: "memory");   // x is ready
    if (lane == 0) {
      int it = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int mt = (u / splits) % m_tiles;
        int kc0, kc1;
        k_range(u, kc0, kc1);
        for (int kc = kc0; kc < kc1; ++kc, ++it) {
          const int s = it % kFusedStages;
          const uint32_t ph = (uint32_t)(it / kFusedStages) & 1u;
          if (it >= kFusedStages && !gemm_wait_idle(smem_addr(&ctl->empty[s]), ph ^ 1u, abort_flag, status)) break;
          const uint32_t fb = smem_addr(&ctl->full[s]);
          mbar_arrive_expect_tx(fb, C::kBStage);
          tma_load_2d(sb(s), &xmap, kc * kBK, mt * BN, fb);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0, tcount = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x, ++tcount) {
        const int b = tcount & 1;
        const uint32_t aph = (uint32_t)(tcount >> 1) & 1u;
        if (tcount >= 2 && !gemm_wait(smem_addr(&ctl->acc_empty[b]), aph ^ 1u, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)b * BN;
        int kc0, kc1;
        k_range(u, kc0, kc1);
        for (int kc = kc0; kc < kc1; ++kc, ++it) {
          const int s = it % kFusedStages;
          const uint32_t ph = (uint32_t)(it / kFusedStages) & 1u;
          if (!gemm_wait(smem_addr(&ctl->full[s]), ph, abort_flag, status)) break;
          tc_fence_after();
          const uint64_t ad = sw128_desc(sa(s)), bd = sw128_desc(sb(s));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_n<BN>(d, ad + 2u * (uint64_t)kk, bd + 2u * (uint64_t)kk, (kc > kc0 || kk > 0) ? 1u : 0u);
          tc_commit(smem_addr(&ctl->empty[s]));
        }
        tc_commit(smem_addr(&ctl->acc_full[b]));
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");   // y and the workspace are free
    const int q = warp & 3;
    int tcount = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++tcount) {
      const int tile = u / splits;
      const int nt = tile / m_tiles, mt = tile % m_tiles;
      const int b = tcount & 1;
      const uint32_t ph = (uint32_t)(tcount >> 1) & 1u;
      gemm_wait_idle(smem_addr(&ctl->acc_full[b]), ph, abort_flag, status);
      epilogue_sync();
      if (*abort_flag) break;
      tc_fence_after();
      const int r = 32 * q + lane, row = nt * kBM + r;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)b * BN;
      float* part = partials + (size_t)u * kPartialFloats;
#pragma unroll 1
      for (int j = 0; j < BN / 32; ++j) {
        uint32_t v[32];
        tc_ld_x32(tbase + 32u * (uint32_t)j, v);
        tc_wait_ld();
        const int m0 = mt * BN + 32 * j;
        if (splits > 1) {
#pragma unroll
          for (int i = 0; i < 32; ++i) __stcg(part + (32 * j + i) * kBM + r, __uint_as_float(v[i]));
        } else if (row < n) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (m0 + i < m) {
              const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[i]));
              y[(size_t)(m0 + i) * n + row] = *reinterpret_cast<const uint16_t*>(&h);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(smem_addr(&ctl->acc_empty[b]));
      if (splits > 1) {
        __threadfence();
        epilogue_sync();
        if (q == 0 && lane == 0) ctl->last_split = atomicAdd(counters + tile, 1u) == (unsigned)(splits - 1);
        epilogue_sync();
        if (ctl->last_split) {
          __threadfence();
          const float* base = partials + (size_t)tile * splits * kPartialFloats;
          if (row < n) {
#pragma unroll 1
            for (int j0 = 0; j0 < BN && mt * BN + j0 < m; j0 += 32) {
              float acc[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
#pragma unroll 1
              for (int sp = 0; sp < splits; ++sp) {
                const float* src = base + (size_t)sp * kPartialFloats + j0 * kBM + r;
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] += __ldcg(src + i * kBM);
              }
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int mm = mt * BN + j0 + i;
                if (mm < m) {
                  const __nv_bfloat16 h = __float2bfloat16_rn(acc[i]);
                  y[(size_t)mm * n + row] = *reinterpret_cast<const uint16_t*>(&h);
                }
              }
            }
          }
          epilogue_sync();
          if (q == 0 && lane == 0) counters[tile] = 0u;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmem) : "memory");
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

// rows x cols bf16 matrix (row-major), boxes of box_rows x 64 columns, 128-byte swizzle
bool encode_bf16_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t allow_gemm_smem() {
  static std::atomic<unsigned long long> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(prefill_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

template <int BN>
cudaError_t allow_fused_smem() {
  static std::atomic<unsigned long long> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(prefill_fused_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, FusedCfg<BN>::kSmem);
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

// Token tile of the fused path: the smallest of 64, 128, 256 that holds M
// (larger M loops over 256-token tiles).
int fused_bn(int m) { return m <= 64 ? 64 : m <= 128 ? 128 : 256; }

int tiles_for(const Layout& L, int m, int bn) { return ((L.n + kBM - 1) / kBM) * ((m + bn - 1) / bn); }

int splits_for(const Layout& L, int tiles, int num_sms) {
  const int kch = L.k / kBK;
  int s = tiles < num_sms ? num_sms / tiles : 1;
  const int smax = kch / kMinSplitChunks > 0 ? kch / kMinSplitChunks : 1;
  if (s > smax) s = smax;
  if (s > kMaxSplits) s = kMaxSplits;
  return s < 1 ? 1 : s;
}

// any4 prefill up to 512 tokens decodes into the GEMM's shared memory: it
// reads each packed weight once instead of writing and re-reading a bf16 copy
// of W. Beyond that the fused kernel would decode W once per 256-token tile,
// and the dequantize-once path is faster on B200 (measured: 14336x4096,
// M = 512: 82 vs 99 us; M = 1024: 155 vs 142 us). any3 / any2 always
// dequantize into the workspace first.
constexpr int kFusedMaxTokens = 512;
bool fused_path(const Layout& L, int m) { return L.bits == 4 && m <= kFusedMaxTokens; }

template <int BN>
cudaError_t launch_fused(const uint16_t* x, const uint8_t* packed, const Layout& L, int m, uint16_t* y,
                         void* workspace, int num_sms, cudaStream_t stream) {
  cudaError_t e = allow_fused_smem<BN>();
  if (e != cudaSuccess) return e;
  CUtensorMap xmap;
  if (!encode_bf16_map(&xmap, x, m, L.k, BN)) return cudaErrorInvalidValue;
  const int tiles = tiles_for(L, m, BN);
  const int splits = splits_for(L, tiles, num_sms);
  const int units = tiles * splits;
  const int grid = units < num_sms ? units : num_sms;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  FusedParams fp{};
  fp.packed = packed;
  fp.w_off = L.w_off; fp.lut_off = L.lut_off; fp.ab_off = L.ab_off;
  fp.panels = L.panels; fp.kchunks = L.kchunks; fp.groups = L.groups;
  fp.g_shift = 0;
  while ((1 << fp.g_shift) < L.g) ++fp.g_shift;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = FusedCfg<BN>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_fused_kernel<BN>, xmap, fp, y, m, L.n, L.k, splits,
                            reinterpret_cast<float*>(ws + kHeaderBytes), reinterpret_cast<unsigned*>(ws),
                            reinterpret_cast<unsigned*>(ws + kCountersBytes));
}

}  // namespace

size_t prefill_scratch_offset() { return kHeaderBytes; }

bool prefill_fused(const Layout& L, int m) { return fused_path(L, m); }

int prefill_splits(const Layout& L, int m, int num_sms) {
  const int tiles = ((L.n + kBM - 1) / kBM) * ((m + kBN - 1) / kBN);
  const int kch = L.k / kBK;
  int s = tiles < num_sms ? num_sms / tiles : 1;
  const int smax = kch / kMinSplitChunks > 0 ? kch / kMinSplitChunks : 1;
  if (s > smax) s = smax;
  if (s > kMaxSplits) s = kMaxSplits;
  return s < 1 ? 1 : s;
}

size_t prefill_partials_offset(const Layout& L) {
  return kHeaderBytes + align_up((size_t)L.n * L.k * 2, kAlign);
}

size_t prefill_workspace_bytes(const Layout& L, int m, int num_sms) {
  if (fused_path(L, m)) {
    const int tiles = tiles_for(L, m, fused_bn(m));
    const int splits = splits_for(L, tiles, num_sms);
    return kHeaderBytes + (splits > 1 ? (size_t)tiles * splits * kPartialFloats * sizeof(float) : 0);
  }
  const int splits = prefill_splits(L, m, num_sms);
  const int tiles = ((L.n + kBM - 1) / kBM) * ((m + kBN - 1) / kBN);
  const size_t partials = splits > 1 ? (size_t)tiles * splits * kPartialFloats * sizeof(float) : 0;
  return prefill_partials_offset(L) + partials;
}

cudaError_t launch_prefill(const uint16_t* x, const uint8_t* packed, const Layout& L, int m, uint16_t* y,
                           void* workspace, int num_sms, cudaStream_t stream) {
  if (fused_path(L, m)) {
    switch (fused_bn(m)) {
      case 64: return launch_fused<64>(x, packed, L, m, y, workspace, num_sms, stream);
      case 128: return launch_fused<128>(x, packed, L, m, y, workspace, num_sms, stream);
      default: return launch_fused<256>(x, packed, L, m, y, workspace, num_sms, stream);
    }
  }
  cudaError_t e = allow_gemm_smem();
  if (e != cudaSuccess) return e;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  uint16_t* what = reinterpret_cast<uint16_t*>(ws + prefill_scratch_offset());
  e = launch_dequant(packed, L, what, stream);   // bf16 W_hat, N x K
  if (e != cudaSuccess) return e;
  CUtensorMap wmap, xmap;
  if (!encode_bf16_map(&wmap, what, L.n, L.k, kBM) || !encode_bf16_map(&xmap, x, m, L.k, kBN))
    return cudaErrorInvalidValue;
  const int tiles = ((L.n + kBM - 1) / kBM) * ((m + kBN - 1) / kBN);
  const int splits = prefill_splits(L, m, num_sms);
  const int units = tiles * splits;
  const int grid = units < num_sms ? units : num_sms;
  unsigned* status = reinterpret_cast<unsigned*>(ws + kCountersBytes);
  unsigned* counters = reinterpret_cast<unsigned*>(ws);
  float* partials = reinterpret_cast<float*>(ws + prefill_partials_offset(L));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_gemm_kernel, wmap, xmap, y, m, L.n, L.k, splits, partials, counters,
                            status);
}

}  // namespace any4
