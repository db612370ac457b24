// any4_linear on B200 (sm_100a): y = x . W_hat^T with W stored as any4.
//
// Method (any4 explainer, 10100.com article 149119421): every row of W has its
// own table (LUT) of 16 bf16 values and every weight is a 4-bit index into it
// (section 2); each contiguous group of G columns has a scale alpha and an
// offset beta (section 2.1); w_hat = fma(alpha, LUT[idx], beta). tinygemm
// (section 3) keeps the table next to the arithmetic and runs batch 1-16 on
// the tensor cores. This kernel is built from B200 measurements:
//
//  * Contraction: mma.sync m16n8k16 (bf16 in, fp32 accumulate). For M <= 16
//    it consumes up to ~128 weights per clock per SM, where one tcgen05.mma of
//    128 x N x 16 costs ~198 cycles whatever N is (~10 weights per clock per
//    SM at this N), so the narrow-N path is the faster one for decode.
//  * Decode: a shared-memory load is the only per-lane gather on the SM. Each
//    index byte of the layout (layout.cuh) holds the indices of rows r and
//    r+16 at one column and selects one bf16 pair (LUT_r[lo], LUT_r+16[hi])
//    from a 256-entry row-pair table: one byte permute forms the address (the
//    tables sit at a 64 KB-aligned shared address, so the byte drops straight
//    into address bits 8..15) and one 32-bit load returns two weights. The
//    four lanes that share a row pair read four bank copies, so every
//    warp-wide lookup is conflict free whatever the indices are.
//  * alpha/beta: one bf16x2 fma per pair, with per-pair (alpha_r, alpha_r+16)
//    operands as stored, so w_hat is rounded once to bf16.
//  * Operands: for M <= 8 the four looked-up pairs are used as they are, as
//    one 16 x 16 tensor-core tile whose rows are the 16 row pairs; every token
//    gets two output columns whose activation operand is zero in the slot of
//    the other row of the pair, so the MMA itself separates the rows (no data
//    movement). For M > 8 byte permutes turn the pairs into the usual two
//    16-row tiles, which keeps one MMA per 8 tokens.
//  * Work split: a thread block (at most one per SM) owns a contiguous range
//    of (32-row panel, 64-column chunk) units: stream-K over all SMs when
//    panels outnumber them, one whole panel per block when they do not, and
//    a cluster of 2-8 blocks per panel (K slices) when whole panels would
//    leave most SMs idle. (Where a block would get only a few chunks,
//    plan_linear hands the shape to linear_small.cu or linear_regt.cu
//    instead, which skip this kernel's streaming structure.) For each panel its
//    consumer warps (16 for M <= 4, 12 for M <= 8, 8 for M <= 16: what the
//    register file and shared memory hold) build the 16 row-pair tables
//    (64 KB) once, then split the panel's chunks. A producer warp streams
//    every consumer warp's weights, four chunks (4 KB) per bulk copy, into
//    per-warp rings of full/empty mbarriers. Each consumer loads its
//    activation columns per chunk, one chunk ahead (for M <= 8 kept in L1
//    with evict_last), and alpha/beta per group (for M <= 8 once per group,
//    past L1). No block-wide barrier inside a panel.
//  * Reduction: a reducer warp sums the consumer warps' fp32 tiles in warp
//    order. A panel split between thread blocks is finished by the block
//    that holds its first unit, which processes it last: it waits (bounded)
//    for the other blocks' partials, published with a release increment when
//    they processed the panel first, and adds them in thread-block order, so
//    results are deterministic. Within a cluster the other ranks push their
//    partials into rank 0's shared memory (st.async onto its mbarrier)
//    instead, and rank 0 adds them in rank order.
//  * The SM's shared-memory/L1 data pipe (one 128-byte wavefront per clock)
//    bounds this decode: per chunk of a panel the lookups take 32 wavefronts,
//    the weight words about 17 (bulk-copy write plus read), the table build 8
//    at K = 4096, activation and alpha/beta loads the rest.
//  * any3 / any2 (BITS = 3, 2): the same kernel with a lane's row-pair codes
//    packed densely (layout.cuh); a code becomes a table address with a
//    funnel shift and one logic op, and the tables have 64 / 16 entries.
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.cuh"

namespace any4 {

namespace {

constexpr int kMinUnitsPerCta = 32;
// Weights stream in pieces of up to 4 chunks (4 KB), one bulk copy each: on
// B200 a bulk copy costs ~100+ cycles of issue in the producer warp whatever
// its size, so 1-2 KB copies cap the stream at 2-4 TB/s; 4 KB copies reach
// 6-7 TB/s.
constexpr int kPieceChunks = 4;
constexpr int kSlotBytes = kPieceChunks * kChunkBytes;
constexpr int kMiscBytes = 1024;                            // mbarriers and flags
constexpr uint32_t kTabAddr = 65536;         // shared-window address of the row-pair tables
constexpr uint32_t kTabBytes = 65536;        // 256 entries x 2 halves x 8 pairs x 4 copies x 4 B
constexpr uint32_t kHighAddr = kTabAddr + kTabBytes;   // ring overflow and warp tiles
constexpr uint32_t kMaxWindowBase = 8192;    // the dynamic window starts below this
constexpr long long kWaitLimitCycles = 4000000000ll;   // ~2 s: then the kernel records a timeout
constexpr int kConsumerBar = 1;              // named barrier of the consumer warps
constexpr int kMaxCluster = 8;               // thread blocks sharing one panel (portable cluster size)
constexpr int kMinClusterChunks = 16;        // chunks a block of such a cluster works on, at least
constexpr int kRegtMaxChunks = 16;           // chunks per block up to which linear_regt.cu decodes
constexpr int kSmallMaxTokens = 4;           // M up to which linear_small.cu takes the short splits
constexpr int kSmallWholeMaxChunks = 128;    // ... and whole panels of at most this many chunks

// MODE 0: M <= 4, MODE 1: M <= 8 (row-pair operands, one or two column tiles
// of 4 tokens); MODE 2: M <= 16 (row operands, two 8-token column tiles).
template <int MODE>
struct Cfg {
  static constexpr bool kTr = MODE == 2;
  static constexpr int kNt8 = MODE == 0 ? 1 : 2;                  // 8-column MMA tiles
  static constexpr int kNW = MODE == 0 ? 16 : MODE == 1 ? 12 : 8; // consumer warps
  static constexpr int kThreads = (kNW + 2) * 32;                 // + producer and reducer warps
  static constexpr int kNF = kTr ? 16 : 4 * kNt8;                 // fp32 results per lane
  static constexpr int kNS = MODE == 2 ? 3 : 2;                   // ring depth (pieces)
  static constexpr int kSlots = kNW * kNS;
  static constexpr int kTileBytes = kNW * 32 * kNF * 4;           // the warps' fp32 tiles of a panel
  // ring slots go below the tables while they fit (for the highest window
  // base), the rest above them, followed by the two buffers of warp tiles
  static constexpr int kLowSlotsMin = ((int)kTabAddr - (int)kMaxWindowBase - kMiscBytes) / kSlotBytes;
  static constexpr int kHighSlotsMax = kSlots > kLowSlotsMin ? kSlots - kLowSlotsMin : 0;
  // cluster rank 0 receives the other ranks' partial sums here
  static constexpr int kRecvBytes = (kMaxCluster - 1) * 32 * kNF * 4;
  static constexpr int kSmemBytes = (int)kHighAddr + kHighSlotsMax * kSlotBytes + 2 * kTileBytes + kRecvBytes;
  // everything below the tables, for a window that starts within 8 KB
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct Params {
  const uint16_t* x;
  const uint8_t* packed;
  uint16_t* y;
  float* partials;
  unsigned* counters;
  unsigned* status;
  int m, n, k;
  int kc, groups, g_shift;                  // chunks per panel, groups per row, log2(G)
  int ctas;
  int cluster;                              // thread blocks per panel (a cluster), or 1
  int x_vec32;                              // x is 32-byte aligned (M > 4: 256-bit activation loads)
  long long units;
  size_t w_off, lut_off, ab_off;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void consumer_sync(int threads) {
  asm volatile("bar.sync %0, %1;" ::"n"(kConsumerBar), "r"(threads) : "memory");
}

// Named barriers: 1 = consumer warps; 2 + b = "warp tiles of buffer b
// stored" (consumers arrive, the reducer waits); 4 + b = "buffer b read"
// (the reducer arrives, the consumers wait before reusing it).
__device__ __forceinline__ void named_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Thread block whose unit range [floor(c*U/C), floor((c+1)*U/C)) holds unit u.
__device__ __forceinline__ int cta_of_unit(long long u, long long U, int C) {
  if ((unsigned long long)U * (unsigned)C < (1ull << 32))
    return (int)(((unsigned)(u + 1) * (unsigned)C - 1u) / (unsigned)U);
  return (int)(((u + 1) * (long long)C - 1) / U);
}

// The chunks one consumer warp works on, in order: for every panel of the
// thread block (units [u_lo, u_hi)), the warp's share [c, cend) of the
// block's chunk range in that panel.
template <int NW>
struct ChunkCursor {
  int panel, plast, c, cend;
  long long u_lo, u_hi;
  int kc, w;
  __device__ void open() {
    const long long pu = (long long)panel * kc;
    const int a = (int)((u_lo > pu ? u_lo : pu) - pu);
    const int b = (int)((u_hi < pu + kc ? u_hi : pu + kc) - pu);
    c = a + (b - a) * w / NW;
    cend = a + (b - a) * (w + 1) / NW;
  }
  __device__ void settle() {   // move past empty ranges
    while (c >= cend && panel <= plast) {
      ++panel;
      if (panel <= plast) open();
    }
  }
  __device__ void start(int p0, int p1, long long lo, long long hi, int kc_, int w_) {
    panel = p0; plast = p1; u_lo = lo; u_hi = hi; kc = kc_; w = w_;
    open();
    settle();
  }
  __device__ bool valid() const { return panel <= plast; }
};

// Waits for phase `parity` of mbarrier `bar`, at most ~kWaitLimitCycles; after
// a timeout (or one seen earlier by this block) it returns without waiting.
__device__ __forceinline__ void wait_bar(uint32_t bar, uint32_t parity, volatile uint32_t* abort) {
  if (mbar_try_wait(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort = 1u;
      return;
    }
  }
}

// Rank 0 of a cluster waits for the other ranks' partials: every rank sends
// its partial even after a timeout of its own (then with whatever it summed),
// so this wait ends once their bytes have landed. It is bounded (twice the
// other waits, so a rank that gives up one of its own waits still gets to
// send) but, unlike wait_bar, not cut short by this block's abort flag: rank 0
// must not exit while another rank may still store into its shared memory.
__device__ __forceinline__ void wait_partials(uint32_t bar, volatile uint32_t* abort) {
  if (mbar_try_wait(bar, 0u)) return;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, 0u)) {
    if (clock64() - t0 > 2 * kWaitLimitCycles) {
      *abort = 1u;
      return;
    }
  }
}

// (token, row within the panel) of result i of lane `ln`.
template <int MODE>
__device__ __forceinline__ void out_pos(int ln, int i, int& token, int& row) {
  const int g = ln >> 2, t = ln & 3;
  if (!Cfg<MODE>::kTr) {
    const int h = i >> 2, q = i & 3;      // D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]
    token = 4 * h + t;
    row = g + (q == 1 ? 16 : q == 2 ? 8 : q == 3 ? 24 : 0);
  } else {
    const int tile = i >> 3, h = (i >> 2) & 1, q = i & 3;
    token = 8 * h + 2 * t + (q & 1);
    row = 16 * tile + g + 8 * (q >> 1);
  }
}

template <int MODE>
__device__ __forceinline__ void store_out(const Params& p, int P, int o, float v) {
  constexpr int NF = Cfg<MODE>::kNF;
  int token, row;
  out_pos<MODE>(o / NF, o % NF, token, row);
  const int n = P * kPanelRows + row;
  if (token < p.m && n < p.n) {
    const __nv_bfloat16 hv = __float2bfloat16_rn(v);
    p.y[(size_t)token * p.n + n] = *reinterpret_cast<const uint16_t*>(&hv);
  }
}

// Shared address of the row-pair table entry for code f (= 4s + q) of a lane's
// chunk words: 4 bits per index -> byte f of the words, dropped into address
// bits 8..15 by one byte permute; 3 and 2 bits -> the 2b-bit code at bit
// 2b*f of the lane's bit string, moved to bits 8.. by a (funnel) shift and
// merged with the lane's base by one logic op.
template <int BITS>
__device__ __forceinline__ uint32_t pair_addr(const uint32_t (&w)[8], int f, uint32_t base) {
  if (BITS == 4) return prmt(w[f >> 2], base, 0x7604u | ((uint32_t)(f & 3) << 4));
  const int bit = 2 * BITS * f, word = bit >> 5, off = bit & 31;
  uint32_t x;
  if (off + 2 * BITS <= 32)
    x = off >= 8 ? (w[word] >> (off - 8)) : (w[word] << (8 - off));
  else
    x = __funnelshift_r(w[word], w[word + 1], off - 8);
  return (x & (((1u << (2 * BITS)) - 1u) << 8)) | base;
}

template <int MODE, int BITS, bool XV8>
__global__ void __launch_bounds__(Cfg<MODE>::kThreads, 1) linear_kernel(const Params p) {
  using C = Cfg<MODE>;
  constexpr int kCB = kChunkBytes * BITS / 4;   // bytes per chunk: 1024, 768, 512
  constexpr int NS = C::kNS, NF = C::kNF, NW = C::kNW, NCT = NW * 32;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  // In a cluster launch the shared addresses of block rank r carry r in their
  // top byte (the block's window within the cluster's); every fixed address
  // below (tables at 64 KB, ring overflow at 128 KB) carries the same prefix.
  const uint32_t win = base & 0xFF000000u;
  const uint32_t tab = win | kTabAddr;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Shared window: [mbarriers, flags][ring slots][row-pair tables at 64 KB]
  // [remaining ring slots][two buffers of warp tiles][cluster partials]. The dynamic window
  // starts at a small fixed offset; if it ever starts higher than planned,
  // record it and leave before touching anything else.
  const uint32_t ring0 = base + kMiscBytes;
  const int n_low = min(C::kSlots, (int)((tab - ring0) / kSlotBytes));
  const uint32_t tiles_addr = (win | kHighAddr) + (uint32_t)(C::kSlots - n_low) * kSlotBytes;
  if (base - win > kMaxWindowBase ||
      tiles_addr + 2u * C::kTileBytes + C::kRecvBytes > base + (uint32_t)C::kSmemBytes) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) atomicOr(p.status, 2u);
    return;
  }
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + 1016);
  auto full_bar = [&](int w, int s) { return base + (uint32_t)(w * NS + s) * 16u; };
  auto empty_bar = [&](int w, int s) { return base + (uint32_t)(w * NS + s) * 16u + 8u; };
  auto slot_addr = [&](int w, int s) {
    const int i = w * NS + s;
    return i < n_low ? ring0 + (uint32_t)i * kSlotBytes : (win | kHighAddr) + (uint32_t)(i - n_low) * kSlotBytes;
  };
  float* tiles = reinterpret_cast<float*>(smem + (tiles_addr - base));   // [2][NW][NF / 4][32] float4
  // A panel split across a cluster of blocks (K slices): rank 0 finishes it
  // from the others' partials, [rank - 1][NF / 4][32] float4, which arrive as
  // transaction bytes on its receive mbarrier.
  const int csz = p.cluster;
  const int crank = (int)(blockIdx.x % (unsigned)csz);
  const uint32_t recv_addr = tiles_addr + 2u * C::kTileBytes;
  const uint32_t recv_bar = base + 960u;

  const long long U = p.units;
  const int kc = p.kc;
  // this block's units [u_lo, u_hi) and panels P0..P1; in 32-bit arithmetic
  // whenever it cannot overflow (a 64-bit division costs ~300 cycles, on the
  // critical path of every call)
  long long u_lo, u_hi;
  int P0, P1;
  if ((long long)p.ctas * kc == U) {   // one whole panel per block
    P0 = P1 = (int)blockIdx.x;
    u_lo = (long long)P0 * kc;
    u_hi = u_lo + kc;
  } else if ((unsigned long long)U * (unsigned)p.ctas < (1ull << 32)) {
    const unsigned uu = (unsigned)U, nc = (unsigned)p.ctas, b = blockIdx.x;
    const unsigned lo = b * uu / nc, hi = (b + 1) * uu / nc;
    u_lo = lo;
    u_hi = hi;
    P0 = (int)(lo / (unsigned)kc);
    P1 = (int)((hi - 1) / (unsigned)kc);
  } else {
    u_lo = (long long)blockIdx.x * U / p.ctas;
    u_hi = (long long)(blockIdx.x + 1) * U / p.ctas;
    P0 = (int)(u_lo / kc);
    P1 = (int)((u_hi - 1) / kc);
  }
  auto is_split = [&](int P) {
    const long long pu = (long long)P * kc;
    return !(pu >= u_lo && pu + kc <= u_hi);
  };

  // Row-pair modes keep the activations in L1 (evict_last) and stream the LUT
  // and alpha/beta past it, loading alpha/beta once per group: on B200 this
  // keeps the L1 misses, which cost several data-pipe wavefronts each, off the
  // activation loads.
  constexpr bool kRowPair = !C::kTr;

  // table build tasks: row pair brp (half, bg), high nibble bhi, low nibbles
  // 8*blh .. 8*blh+7; every entry goes to its four bank copies
  constexpr int kBuildPer = (512 + NCT - 1) / NCT;   // 512 tasks per panel
  // 3- and 2-bit tables: one task per (row pair, entry), 16 << 2b tasks; the
  // task's entry value (LUT_r[lo], LUT_r+16[hi]) is loaded a panel ahead
  constexpr int kSmallTasks = 16 << (2 * BITS);
  constexpr int kSmallPer = BITS == 4 ? 1 : (kSmallTasks + NCT - 1) / NCT;
  uint32_t sv[kSmallPer], snv[kSmallPer];
  auto load_small = [&](int P, uint32_t (&dv)[kSmallPer]) {
#pragma unroll
    for (int r = 0; r < kSmallPer; ++r) {
      const int task = tid + r * NCT;
      if (task >= kSmallTasks) break;
      const int brp = task & 15, e = task >> 4;
      const int br0 = (brp & 7) + 8 * (brp >> 3);
      const int lo = e & ((1 << BITS) - 1), hi = e >> BITS;
      const uint16_t* base_lut = reinterpret_cast<const uint16_t*>(p.packed + p.lut_off) + (size_t)P * kPanelRows * 16;
      dv[r] = ld_nc_u16(base_lut + br0 * 16 + lo) | (ld_nc_u16(base_lut + (br0 + 16) * 16 + hi) << 16);
    }
  };
  const uint16_t* lut = reinterpret_cast<const uint16_t*>(p.packed + p.lut_off);
  // this thread's LUT values of the panel being built (lw/lh) and of the
  // next one (nw/nh), loaded a full panel ahead
  uint4 lw[kBuildPer], nw[kBuildPer];
  uint32_t lh[kBuildPer], nh[kBuildPer];
  auto load_lut = [&](int P, uint4 (&dw)[kBuildPer], uint32_t (&dh)[kBuildPer]) {
#pragma unroll
    for (int r = 0; r < kBuildPer; ++r) {
      const int task = tid + r * NCT;
      if (task >= 512) break;
      const int brp = task & 15, bhi = (task >> 4) & 15, blh = task >> 8;
      const int br0 = (brp & 7) + 8 * (brp >> 3);
      if (kRowPair) {
        dw[r] = ld_stream_v4(lut + ((size_t)P * kPanelRows + br0) * 16 + 8 * blh);
        dh[r] = ld_stream_u16(lut + ((size_t)P * kPanelRows + br0 + 16) * 16 + bhi);
      } else {
        dw[r] = ld_nc_v4(lut + ((size_t)P * kPanelRows + br0) * 16 + 8 * blh);
        dh[r] = ld_nc_u16(lut + ((size_t)P * kPanelRows + br0 + 16) * 16 + bhi);
      }
    }
  };
  // the consumer warps' first LUT loads go out before the barrier setup
  if (warp < NW) {
    if (BITS == 4) {
      load_lut(P0, lw, lh);
      if (P0 < P1) load_lut(P0 + 1, nw, nh);
    } else {
      load_small(P0, sv);
      if (P0 < P1) load_small(P0 + 1, snv);
    }
  }

  if (tid == 0) *abort = 0u;
  if (tid < NW * NS) {
    mbar_init(full_bar(tid / NS, tid % NS), 1);
    mbar_init(empty_bar(tid / NS, tid % NS), 32);
  }
  const bool receiver = csz > 1 && crank == 0;
  if (tid == 0 && receiver) mbar_init(recv_bar, 1);
  fence_mbar_init();
  if (tid == 0 && receiver) mbar_arrive_expect_tx(recv_bar, (uint32_t)((csz - 1) * 32 * NF * 4));
  __syncthreads();
  if (csz > 1) cluster_sync_init();   // rank 0's receive barrier is armed before any rank sends
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // =========================== producer warp ===============================
  // Lane w < NW streams consumer warp w's pieces (up to two chunks of one
  // panel) in the order the warp uses them. It reads only the packed weight,
  // which is immutable, so it needs no grid-dependency wait: with
  // programmatic dependent launch it runs ahead while the previous kernel on
  // the stream finishes.
  if (warp == NW) {
    ChunkCursor<NW> cur;
    cur.start(P0, P1, u_lo, u_hi, kc, lane);
    if (lane >= NW) cur.panel = P1 + 1;   // lanes without a consumer warp
    const uint8_t* wbase = p.packed + p.w_off;
    int issued = 0;   // pieces issued so far; piece q uses slot q % NS for the (q / NS)-th time
    while (cur.valid()) {
      const int slot = issued % NS;
      const int n = min(kPieceChunks, cur.cend - cur.c);
      const uint32_t wbytes = (uint32_t)n * kCB;
      if (issued >= NS)   // the consumer's release of the slot's previous use
        wait_bar(empty_bar(lane, slot), (uint32_t)(issued / NS - 1) & 1u, abort);
      if (*abort) break;
      const uint32_t fb = full_bar(lane, slot), dst = slot_addr(lane, slot);
      mbar_arrive_expect_tx(fb, wbytes);
      bulk_g2s(dst, wbase + ((size_t)cur.panel * kc + cur.c) * kCB, wbytes, fb);
      ++issued;
      cur.c += n;
      cur.settle();
    }
    return;
  }

  // =========================== reducer warp ================================
  // Sums the consumer warps' fp32 tiles of each panel in warp order (a fixed
  // tree) and writes y. A panel split between thread blocks (stream-K) is
  // finished by the block that holds the panel's first unit; it processes
  // the panel last, while the other contributors process it first and
  // publish their partial sum at once (release-increment of the panel's
  // counter). The finisher collects their partials while its consumers still
  // work on the panel, adds them after its own sum in thread-block order
  // (deterministic) and resets the counter for the next call.
  if (warp == NW + 1) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // y, partials, counters
    for (int P = P0; P <= P1; ++P) {
      const int b = (P - P0) & 1;
      const bool split = is_split(P);
      const long long pu = (long long)P * kc;
      const bool finisher = split && pu >= u_lo;
      const bool clustered = csz > 1;   // split panels are finished within the cluster
      const int c_first = split ? cta_of_unit(pu, U, p.ctas) : 0;
      const int c_last = split ? cta_of_unit(pu + kc - 1, U, p.ctas) : 0;
      float other[NF];
#pragma unroll
      for (int i = 0; i < NF; ++i) other[i] = 0.0f;
      if (!clustered && finisher && c_last > c_first) {
        const unsigned need = (unsigned)(c_last - c_first);
        if (lane == 0 && ld_acquire(p.counters + P) < need) {
          const long long t0 = clock64();
          while (ld_acquire(p.counters + P) < need) {
            if (*abort) break;
            if (clock64() - t0 > kWaitLimitCycles) { *abort = 1u; break; }
          }
        }
        __syncwarp();
        (void)ld_acquire(p.counters + P);   // this lane's acquire of the publishers' stores
        for (int c = c_first + 1; c <= c_last; ++c) {
          const float* src = p.partials + ((size_t)c * 32 + lane) * NF;
#pragma unroll
          for (int i = 0; i < NF; ++i) other[i] += __ldcg(src + i);
        }
      }
      named_sync(2 + b, NCT + 32);   // tiles of panel P stored
      // tiles are [buffer][warp][NF / 4][lane] float4: lane-contiguous, so
      // every 128-bit load below is free of bank conflicts
      const float4* tb = reinterpret_cast<const float4*>(tiles) + (size_t)b * NW * (NF / 4) * 32 + lane;
      float v[NF];
#pragma unroll
      for (int i4 = 0; i4 < NF / 4; ++i4) {
        float4 t[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) t[w] = tb[((size_t)w * (NF / 4) + i4) * 32];
#pragma unroll
        for (int span = 1; span < NW; span *= 2)
#pragma unroll
          for (int w = 0; w + span < NW; w += 2 * span) {
            t[w].x += t[w + span].x;
            t[w].y += t[w + span].y;
            t[w].z += t[w + span].z;
            t[w].w += t[w + span].w;
          }
        v[4 * i4 + 0] = t[0].x;
        v[4 * i4 + 1] = t[0].y;
        v[4 * i4 + 2] = t[0].z;
        v[4 * i4 + 3] = t[0].w;
      }
      if (P + 2 <= P1) named_arrive(4 + b, NCT + 32);   // buffer b may be reused
      if (!split || finisher) {
        if (clustered && split) {   // the other ranks' partials, added in rank order
          wait_partials(recv_bar, abort);
          const float4* rb = reinterpret_cast<const float4*>(smem + (recv_addr - base)) + lane;
          for (int r = 1; r < csz; ++r) {
#pragma unroll
            for (int i4 = 0; i4 < NF / 4; ++i4) {
              const float4 q = rb[((size_t)(r - 1) * (NF / 4) + i4) * 32];
              other[4 * i4 + 0] += q.x;
              other[4 * i4 + 1] += q.y;
              other[4 * i4 + 2] += q.z;
              other[4 * i4 + 3] += q.w;
            }
          }
        }
#pragma unroll
        for (int i = 0; i < NF; ++i) store_out<MODE>(p, P, lane * NF + i, v[i] + other[i]);
        if (split && !clustered && lane == 0) p.counters[P] = 0u;   // ready for the next call
      } else if (clustered) {   // send this block's partial to rank 0
        const uint32_t bar0 = cluster_map(recv_bar, 0u);
#pragma unroll
        for (int i4 = 0; i4 < NF / 4; ++i4) {
          const uint32_t dst = recv_addr + (uint32_t)((((crank - 1) * (NF / 4) + i4) * 32 + lane) * 16);
          st_async_v4(cluster_map(dst, 0u), v[4 * i4], v[4 * i4 + 1], v[4 * i4 + 2], v[4 * i4 + 3], bar0);
        }
      } else {
        float* dst = p.partials + ((size_t)blockIdx.x * 32 + lane) * NF;
#pragma unroll
        for (int i = 0; i < NF; ++i) __stcg(dst + i, v[i]);
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add(p.counters + P, 1u);
      }
    }
    if (lane == 0 && *abort) atomicOr(p.status, kStatusWaitTimeout);
    return;
  }

  // =========================== consumer warps ==============================
  const int g = lane >> 2, t = lane & 3;

  // lookup address bases: byte b of a word goes to address bits 8..15
  const uint32_t baseA = tab | ((uint32_t)g << 4) | ((uint32_t)t << 2);   // pairs (g, g+16)
  const uint32_t baseB = baseA | 128u;                                         // pairs (g+8, g+24)

  // Activation operands. Tile h serves tokens 4h.. (row-pair mode: lane g
  // feeds output column g = 2j + p of token j, zero in the slot of the other
  // row of the pair) or 8h.. (row mode: lane g feeds token 8h+g). A lane whose
  // token is >= M reads token 0 (a cached line) and zeroes its operand.
  constexpr int NX = C::kTr ? 2 : C::kNt8;
  const uint16_t* xrow[NX];
  uint32_t selb0[NX], selb1[NX], xmask[NX];
#pragma unroll
  for (int h = 0; h < NX; ++h) {
    const int j = C::kTr ? 8 * h + g : 4 * h + (g >> 1);
    const bool ok = j < p.m;
    xrow[h] = p.x + (size_t)(ok ? j : 0) * p.k + 16 * t;
    selb0[h] = !ok ? 0x4444u : (g & 1) ? 0x1044u : 0x4410u;
    selb1[h] = !ok ? 0x4444u : (g & 1) ? 0x3244u : 0x4432u;
    xmask[h] = ok ? 0xffffffffu : 0u;
  }
  // Per chunk, loaded from L2 one chunk ahead: the activation words (word
  // s = 0..7 of tile h = component s & 3 of xn[h][s >> 2]; columns 16t + 2s, +1
  // of the chunk) and this lane's alpha/beta pairs of the chunk's group.
  const uint8_t* abase = p.packed + p.ab_off + 16 * g;
  uint4 xn[NX][2], scn;
  int last_grp = -1, pf_grp = -1;
  const int pf_lim = ((p.n + 31) >> 5) * p.groups;   // scale records in the packed weight
  ChunkCursor<NW> xc;   // the chunk whose operands load next
  xc.start(P0, P1, u_lo, u_hi, kc, warp);
  auto next_operands = [&]() {
    if (!xc.valid()) return;
    const int c = xc.c;
#pragma unroll
    for (int h = 0; h < NX; ++h) {
      const uint16_t* src = xrow[h] + (size_t)c * kChunkCols;
      if (XV8 && kRowPair) {   // one 32-byte request per lane (M <= 8: kept in L1)
        ld_keep_v8(src, xn[h][0], xn[h][1]);
      } else if (kRowPair) {
        xn[h][0] = ld_keep_v4(src);
        xn[h][1] = ld_keep_v4(src + 8);
      } else if (XV8) {   // one 32-byte request per lane (measured: gate/up 18.9 -> 17.9 us)
        ld_nc_v8(src, xn[h][0], xn[h][1]);
      } else {
        xn[h][0] = ld_nc_v4(src);
        xn[h][1] = ld_nc_v4(src + 8);
      }
    }
    const int grp = xc.panel * p.groups + ((c * kChunkCols) >> p.g_shift);
    if (!kRowPair) {
      scn = ld_nc_v4(abase + ((size_t)grp << 7));
      if (grp != pf_grp && grp + 1 < pf_lim) {   // the next group's record into L2 (measured: down
        pf_grp = grp;                            // 4096 x 14336 at M = 16, 17.0 -> 15.5 us)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(abase + ((size_t)(grp + 1) << 7)));
      }
    } else if (grp != last_grp) {   // a new group: its alpha/beta (read once, not kept in L1)
      scn = ld_stream_v4(abase + ((size_t)grp << 7));
      last_grp = grp;
    }
    ++xc.c;
    xc.settle();
  };

  // decode + contract one chunk (8 steps) from its weight words, alpha/beta
  // and activation words
  float acc[NF / 4][4];   // one m16n8 fp32 tile per 4 results
  auto chunk = [&](const uint4& wa, const uint4& wb, const uint4& sc, const uint32_t (&xw)[NX][8]) {
    const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    if (!C::kTr) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t a[4];
        a[0] = lds32(pair_addr<BITS>(w, 4 * s + 0, baseA));
        a[1] = lds32(pair_addr<BITS>(w, 4 * s + 1, baseB));
        a[2] = lds32(pair_addr<BITS>(w, 4 * s + 2, baseA));
        a[3] = lds32(pair_addr<BITS>(w, 4 * s + 3, baseB));
        a[0] = fma_bf16x2(a[0], sc.x, sc.y);
        a[2] = fma_bf16x2(a[2], sc.x, sc.y);
        a[1] = fma_bf16x2(a[1], sc.z, sc.w);
        a[3] = fma_bf16x2(a[3], sc.z, sc.w);
#pragma unroll
        for (int h = 0; h < NX; ++h)
          mma_m16n8k16(acc[h], a, prmt(xw[h][s], 0u, selb0[h]), prmt(xw[h][s], 0u, selb1[h]));
      }
    } else {
#pragma unroll
      for (int s = 0; s < 8; s += 2) {
        uint32_t e[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          e[u][0] = lds32(pair_addr<BITS>(w, 4 * (s + u) + 0, baseA));
          e[u][1] = lds32(pair_addr<BITS>(w, 4 * (s + u) + 1, baseB));
          e[u][2] = lds32(pair_addr<BITS>(w, 4 * (s + u) + 2, baseA));
          e[u][3] = lds32(pair_addr<BITS>(w, 4 * (s + u) + 3, baseB));
          e[u][0] = fma_bf16x2(e[u][0], sc.x, sc.y);
          e[u][2] = fma_bf16x2(e[u][2], sc.x, sc.y);
          e[u][1] = fma_bf16x2(e[u][1], sc.z, sc.w);
          e[u][3] = fma_bf16x2(e[u][3], sc.z, sc.w);
        }
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
          const uint32_t sel = tile ? 0x7632u : 0x5410u;
          const uint32_t a[4] = {prmt(e[0][0], e[0][2], sel), prmt(e[0][1], e[0][3], sel),
                                 prmt(e[1][0], e[1][2], sel), prmt(e[1][1], e[1][3], sel)};
#pragma unroll
          for (int h = 0; h < 2; ++h)
            mma_m16n8k16(acc[2 * tile + h], a, xw[h][s] & xmask[h], xw[h][s + 1] & xmask[h]);
        }
      }
    }
  };

  int q = 0;   // pieces consumed; piece q sits in slot q % NS, phase (q / NS) & 1

  for (int P = P0; P <= P1; ++P) {
    // ---- build the 16 row-pair tables of panel P
    if (BITS != 4) {
#pragma unroll
      for (int r = 0; r < kSmallPer; ++r) {
        const int task = tid + r * NCT;
        if (task >= kSmallTasks) break;
        const int brp = task & 15, e = task >> 4;
        const uint32_t bdst = tab + ((uint32_t)(brp >> 3) << 7) + ((uint32_t)(brp & 7) << 4);
        sts128(bdst + ((uint32_t)e << 8), sv[r], sv[r], sv[r], sv[r]);
      }
#pragma unroll
      for (int r = 0; r < kSmallPer; ++r) sv[r] = snv[r];
      if (P + 1 < P1) load_small(P + 2, snv);
    }
#pragma unroll
    for (int r = 0; r < kBuildPer; ++r) {
      const int task = tid + r * NCT;
      if (BITS != 4 || task >= 512) break;
      const int brp = task & 15, bhi = (task >> 4) & 15, blh = task >> 8;
      const uint32_t bdst = tab + ((uint32_t)(brp >> 3) << 7) + ((uint32_t)(brp & 7) << 4);
      const uint32_t L[4] = {lw[r].x, lw[r].y, lw[r].z, lw[r].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t e = (uint32_t)(8 * blh + i) | ((uint32_t)bhi << 4);
        const uint32_t v = prmt(L[i >> 1], lh[r], (i & 1) ? 0x5432u : 0x5410u);
        sts128(bdst + (e << 8), v, v, v, v);
      }
    }
    if (BITS == 4) {
#pragma unroll
      for (int r = 0; r < kBuildPer; ++r) { lw[r] = nw[r]; lh[r] = nh[r]; }
      if (P + 1 < P1) load_lut(P + 2, nw, nh);
    }
    if (P == P0) {
      // activations, y and the workspace are touched only from here on
      asm volatile("griddepcontrol.wait;" ::: "memory");
      next_operands();
    }
    consumer_sync(NCT);   // tables ready

#pragma unroll
    for (int i = 0; i < NF / 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

    int c0, c1;
    {
      ChunkCursor<NW> mine;
      mine.panel = P; mine.u_lo = u_lo; mine.u_hi = u_hi; mine.kc = kc; mine.w = warp;
      mine.open();
      c0 = mine.c; c1 = mine.cend;
    }
    // pieces of up to kPieceChunks chunks from the warp's ring, chunk by chunk
    for (int pc = c0; pc < c1; pc += kPieceChunks) {
      const int n = min(kPieceChunks, c1 - pc);
      const int slot = q % NS;
      const uint32_t sb = slot_addr(warp, slot) + 16u * lane;
      wait_bar(full_bar(warp, slot), (uint32_t)(q / NS) & 1u, abort);
      ++q;
      for (int cc = 0; cc < n; ++cc) {
        // this lane's words of the chunk: 8 (4 bits), 6 (3 bits) or 4 (2 bits)
        const uint4 wa = lds128(sb + (uint32_t)cc * kCB);
        uint4 wb = make_uint4(0u, 0u, 0u, 0u);
        if (BITS == 4) wb = lds128(sb + (uint32_t)cc * kCB + 512u);
        if (BITS == 3) {
          const uint2 w2 = lds64(sb - 8u * lane + (uint32_t)cc * kCB + 512u);
          wb.x = w2.x;
          wb.y = w2.y;
        }
        // release the slot once its last words are in registers
        if (cc == n - 1) mbar_arrive_after(empty_bar(warp, slot), wa.x, wb.x, 0u, 0u);
        uint32_t xw[NX][8];
#pragma unroll
        for (int h = 0; h < NX; ++h) {
          xw[h][0] = xn[h][0].x; xw[h][1] = xn[h][0].y; xw[h][2] = xn[h][0].z; xw[h][3] = xn[h][0].w;
          xw[h][4] = xn[h][1].x; xw[h][5] = xn[h][1].y; xw[h][6] = xn[h][1].z; xw[h][7] = xn[h][1].w;
        }
        const uint4 sc = scn;
        next_operands();   // the next chunk's activations and alpha/beta
        chunk(wa, wb, sc, xw);
      }
    }

    // ---- hand the warp tiles to the reducer warp (double-buffered)
    const int b = (P - P0) & 1;
    if (P - P0 >= 2) named_sync(4 + b, NCT + 32);   // the reducer is done with buffer b
    {
      float4* dst = reinterpret_cast<float4*>(tiles) + ((size_t)b * NW + warp) * (NF / 4) * 32 + lane;
#pragma unroll
      for (int i = 0; i < NF / 4; ++i) dst[(size_t)i * 32] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
    named_arrive(2 + b, NCT + 32);
    consumer_sync(NCT);   // every consumer is past its lookups: the tables are free
  }
  if (tid == 0 && *abort) atomicOr(p.status, kStatusWaitTimeout);
}

template <int MODE, int BITS>
cudaError_t allow_smem_mode() {
  cudaError_t e = cudaFuncSetAttribute(linear_kernel<MODE, BITS, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<MODE>::kSmemBytes);
  if (e == cudaSuccess && MODE >= 1)
    e = cudaFuncSetAttribute(linear_kernel<MODE, BITS, MODE >= 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<MODE>::kSmemBytes);
  return e;
}

template <int BITS>
cudaError_t allow_smem_bits() {
  cudaError_t e = allow_smem_mode<0, BITS>();
  if (e == cudaSuccess) e = allow_smem_mode<1, BITS>();
  if (e == cudaSuccess) e = allow_smem_mode<2, BITS>();
  return e;
}

cudaError_t allow_large_smem() {
  static std::atomic<unsigned long long> done_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_relaxed) & bit) return cudaSuccess;
  e = allow_smem_bits<4>();
  if (e == cudaSuccess) e = allow_smem_bits<3>();
  if (e == cudaSuccess) e = allow_smem_bits<2>();
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

template <int MODE, int BITS>
cudaError_t launch_mode(const Params& p, const LinearPlan& plan, cudaStream_t stream) {
  // programmatic dependent launch: this kernel's weight prologue may overlap the
  // tail of the previous kernel on the stream (see griddepcontrol in the kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.ctas);
  cfg.blockDim = dim3(Cfg<MODE>::kThreads);
  cfg.dynamicSmemBytes = Cfg<MODE>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)plan.cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = plan.cluster > 1 ? 2 : 1;
  // 256-bit activation loads: measured faster at M = 5..16 (M = 8 down
  // 4096 x 14336: 14.3 -> 13.9 us), no gain at M <= 4
  if (MODE >= 1 && p.x_vec32) return cudaLaunchKernelEx(&cfg, linear_kernel<MODE, BITS, MODE >= 1>, p);
  return cudaLaunchKernelEx(&cfg, linear_kernel<MODE, BITS, false>, p);
}

// How many clusters of `s` blocks of linear_kernel<MODE, BITS, false> the current
// device holds at once (0 if the query fails).
template <int MODE, int BITS>
int active_clusters(int s) {
  if (allow_large_smem() != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)s);
  cfg.blockDim = dim3(Cfg<MODE>::kThreads);
  cfg.dynamicSmemBytes = Cfg<MODE>::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)s;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, linear_kernel<MODE, BITS, false>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

template <int BITS>
int active_clusters_mode(int mode, int s) {
  return mode == 0 ? active_clusters<0, BITS>(s) : mode == 1 ? active_clusters<1, BITS>(s) : active_clusters<2, BITS>(s);
}

// Cached per device, mode, bit width and cluster size.
int max_active_clusters(int mode, int bits, int s) {
  static std::atomic<int>* const cache = [] {
    auto* c = new std::atomic<int>[64 * 3 * 3 * 4];
    for (int i = 0; i < 64 * 3 * 3 * 4; ++i) c[i].store(-1);
    return c;
  }();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int bi = bits == 4 ? 0 : bits == 3 ? 1 : 2;
  const int si = s == 2 ? 0 : s == 4 ? 1 : s == 8 ? 2 : 3;
  std::atomic<int>& slot = cache[((dev * 3 + mode) * 3 + bi) * 4 + si];
  int v = slot.load(std::memory_order_relaxed);
  if (v < 0) {
    v = bits == 4 ? active_clusters_mode<4>(mode, s) : bits == 3 ? active_clusters_mode<3>(mode, s)
                                                     : active_clusters_mode<2>(mode, s);
    slot.store(v, std::memory_order_relaxed);
  }
  return v;
}

template <int BITS>
cudaError_t launch_bits(const Params& p, const LinearPlan& plan, cudaStream_t stream) {
  switch (plan.mode) {
    case 0: return launch_mode<0, BITS>(p, plan, stream);
    case 1: return launch_mode<1, BITS>(p, plan, stream);
    default: return launch_mode<2, BITS>(p, plan, stream);
  }
}

}  // namespace

LinearPlan plan_linear(int m, const Layout& L, int num_sms) {
  LinearPlan pl{};
  if (m > 16) {   // prefill: dequantized W scratch + tensor-core GEMM
    pl.mode = 3;
    pl.workspace_bytes = prefill_workspace_bytes(L, m, num_sms);
    pl.ctas = num_sms;
    return pl;
  }
  pl.mode = m <= 4 ? 0 : m <= 8 ? 1 : 2;
  pl.nf = pl.mode == 0 ? 4 : pl.mode == 1 ? 8 : 16;
  pl.units = (long long)L.panels * L.kchunks;
  long long c;
  pl.cluster = 1;
  if (L.panels <= num_sms) {
    // one whole panel per thread block: no table built for a piece of a
    // panel and no split panel to finish (on B200 this is 1.3-1.5x faster
    // than spreading 128 panels over 148 blocks) ...
    c = L.panels;
    // ... and where that leaves SMs idle, a cluster of s blocks per panel,
    // each on a K slice of at least kMinClusterChunks chunks, finishing the
    // panel through distributed shared memory, when the device holds all
    // the clusters at once
    for (int s = kMaxCluster; s >= 2; s /= 2) {
      if ((long long)L.panels * s > num_sms || L.kchunks < s * kMinClusterChunks) continue;
      if (max_active_clusters(pl.mode, L.bits, s) < L.panels) continue;
      pl.cluster = s;
      c = (long long)L.panels * s;
      break;
    }
  } else {
    c = pl.units / kMinUnitsPerCta;
    if (c > num_sms) c = num_sms;
  }
  if (c < 1) c = 1;
  pl.ctas = (int)c;
  // a short K split over a cluster per panel (at most kRegtMaxChunks chunks
  // per block, at least one per warp): the fixed cost of this kernel's
  // streaming structure outweighs the decode, so for M = 5..16 the
  // register-table kernel takes it, on its own cluster split (measured on
  // B200: faster on such shapes, slower without a cluster or with idle warps).
  // For M <= 4 the same splits, and whole panels of up to
  // kSmallWholeMaxChunks chunks where this kernel would run whole panels
  // too, run the shared tables without the streaming structure
  // (linear_small.cu; measured on B200 at M = 1: k/v 3.70 -> 3.25 us, q/o
  // 4.64 -> 4.33 us, 4096 x 8192 7.12 -> 6.70 us, 4096 x 14336 equal; slower
  // than these kernels for M > 4).
  if (L.bits == 4 && L.panels <= num_sms) {
    const bool direct = m <= kSmallMaxTokens;
    const int warps = direct ? small_warps(m) : regt_warps(m);
    int s = 0;
    for (int q = direct ? small_max_cluster() : regt_max_cluster(); q >= 2; q /= 2) {   // each kernel's receive buffers
      if ((long long)L.panels * q <= num_sms && L.kchunks >= q * warps) {
        s = q;
        break;
      }
    }
    if (s > 0 && L.kchunks <= s * kRegtMaxChunks) {
      (direct ? pl.small : pl.regt) = true;
      pl.cluster = s;
      pl.ctas = L.panels * s;
    } else if (direct && pl.cluster == 1 && L.kchunks <= kSmallWholeMaxChunks) {   // whole panels here too
      pl.small = true;
      pl.cluster = 1;
      pl.ctas = L.panels;
    }
  }
  // partial sums are only used without clusters, by at most one block per
  // panel (whole panels) or per SM (stream-K); sized so that the workspace
  // does not depend on the cluster decision
  const long long pc = L.panels <= num_sms ? L.panels : c;
  pl.partials_bytes = (size_t)(pc < 1 ? 1 : pc) * 32 * pl.nf * sizeof(float);
  pl.workspace_bytes = kHeaderBytes + pl.partials_bytes;
  return pl;
}

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream) {
  if (plan.mode == 3) return launch_prefill(x, packed, L, m, y, workspace, plan.ctas, stream);
  if (plan.regt) return launch_linear_regt(x, packed, L, m, y, workspace, plan.cluster, stream);
  if (plan.small) return launch_linear_small(x, packed, L, m, y, workspace, plan.cluster, stream);
  cudaError_t e = allow_large_smem();
  if (e != cudaSuccess) return e;
  Params p{};
  p.x = x;
  p.packed = packed;
  p.y = y;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  p.counters = reinterpret_cast<unsigned*>(ws);
  p.status = reinterpret_cast<unsigned*>(ws + kCountersBytes);
  p.partials = reinterpret_cast<float*>(ws + kHeaderBytes);
  p.m = m; p.n = L.n; p.k = L.k;
  p.kc = L.kchunks; p.groups = L.groups;
  p.g_shift = 0;
  while ((1 << p.g_shift) < L.g) ++p.g_shift;
  p.ctas = plan.ctas;
  p.cluster = plan.cluster;
  p.x_vec32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;
  p.units = plan.units;
  p.w_off = L.w_off; p.lut_off = L.lut_off; p.ab_off = L.ab_off;
  switch (L.bits) {
    case 3: return launch_bits<3>(p, plan, stream);
    case 2: return launch_bits<2>(p, plan, stream);
    default: return launch_bits<4>(p, plan, stream);
  }
}

}  // namespace any4
