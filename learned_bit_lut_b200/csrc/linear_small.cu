// any4_linear, M <= 16, for shapes with few chunks per thread block: the
// shared row-pair tables of linear.cu without its streaming structure.
//
// Same decode as linear.cu (row-pair tables in shared memory: one byte
// permute forms the address, one 32-bit shared load returns two weights;
// explainer 10100.com article 149119421, sections 2-3), same contraction
// (mma.sync m16n8k16 after one fma.rn.bf16x2 per pair), but laid out for a
// block that owns only a short K slice of one panel:
//
//  * grid: one cluster of s blocks per 32-row panel (s = 1, 2, 4), each on a
//    contiguous K slice; every warp takes its own chunks of the slice;
//  * no producer warp and no ring: each warp loads its index words, scale
//    records and activations itself, one chunk ahead (the words and the
//    table entries before the grid-dependency wait: they are the immutable
//    packed weight);
//  * the block builds the panel's 64 KB row-pair table once (512 16-byte
//    stores), one barrier, then decodes;
//  * the warps' fp32 tiles are added in warp order in shared memory; ranks
//    1..s-1 send their sums to rank 0 over distributed shared memory
//    (st.async onto its mbarrier) and rank 0 adds them in rank order:
//    deterministic, no workspace traffic.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace any4 {

namespace {

constexpr int kSmallMaxCluster = 4;
constexpr uint32_t kSmallTab = 65536;                 // window address of the row-pair tables
constexpr uint32_t kSmallLow = 1024;                  // mbarrier area at the window base
constexpr uint32_t kSmallMaxBase = 8192;              // the dynamic window starts below this
constexpr int kSmallSmem = 2 * 65536;                 // covers the tables for any base below 64 KB
constexpr long long kSmallWaitCycles = 8000000000ll;  // ~4 s: then rank 0 records a timeout

// MODE 0: M <= 4, 1: M <= 8 (row-pair operands), 2: M <= 16 (row operands).
template <int MODE>
struct SmallCfg {
  static constexpr bool kTr = MODE == 2;
  static constexpr int kNt8 = MODE == 0 ? 1 : 2;
  static constexpr int kNW = MODE == 0 ? 16 : MODE == 1 ? 12 : 8;
  static constexpr int kThreads = kNW * 32;
  static constexpr int kNF = kTr ? 16 : 4 * kNt8;                  // fp32 results per lane
  static constexpr int kNX = kTr ? 2 : kNt8;                       // activation tiles
  static constexpr int kTileBytes = 32 * kNF * 4;                  // one warp's results
  static_assert(kSmallLow + (kNW + kSmallMaxCluster - 1) * kTileBytes + kSmallMaxBase <= kSmallTab,
                "tiles below the tables");
};

struct SmallParams {
  const uint16_t* x;
  const uint8_t* packed;
  uint16_t* y;
  unsigned* status;
  int m, n, k;
  int kc, groups, g_shift;
  int cluster;
  size_t w_off, lut_off, ab_off;
};

template <int MODE>
__global__ void __launch_bounds__(SmallCfg<MODE>::kThreads, 1) linear_small_kernel(const SmallParams p) {
  using C = SmallCfg<MODE>;
  constexpr int NW = C::kNW, NF = C::kNF, NX = C::kNX, NCT = NW * 32;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t win = base & 0xFF000000u;   // a cluster rank's window carries the rank in the top byte
  const uint32_t tab = win | kSmallTab;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int csz = p.cluster;
  const int crank = (int)(blockIdx.x % (unsigned)csz);
  const int P = (int)(blockIdx.x / (unsigned)csz);
  const bool receiver = csz > 1 && crank == 0;
  const uint32_t recv_bar = base;
  const uint32_t tiles = base + kSmallLow;                                 // [warp][NF/4][lane] float4
  const uint32_t recv = tiles + (uint32_t)(NW * C::kTileBytes);            // [rank-1][NF/4][lane] float4
  if (base - win > kSmallMaxBase) {   // the fixed table address would not be ours: record and leave
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) atomicOr(p.status, 2u);
    return;
  }

  // the next kernel on the stream may start launching (it waits for this
  // grid before it touches what this one writes)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- immutable inputs first: this thread's table-build entries, the
  // warp's first index words
  // 512 build tasks (pair slot, high nibble, low-nibble half), kPer per thread
  constexpr int kPer = (512 + NCT - 1) / NCT;
  const uint16_t* lut = reinterpret_cast<const uint16_t*>(p.packed + p.lut_off);
  uint4 lw[kPer];
  uint32_t lh[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int task = tid + r * NCT;
    lw[r] = make_uint4(0u, 0u, 0u, 0u);
    lh[r] = 0u;
    if (task < 512) {
      const int brp = task & 15, bhi = (task >> 4) & 15, blh = task >> 8;
      const int br0 = (brp & 7) + 8 * (brp >> 3);
      lw[r] = ld_stream_v4(lut + ((size_t)P * kPanelRows + br0) * 16 + 8 * blh);
      lh[r] = ld_stream_u16(lut + ((size_t)P * kPanelRows + br0 + 16) * 16 + bhi);
    }
  }
  const int s0 = (int)((long long)crank * p.kc / csz), s1 = (int)((long long)(crank + 1) * p.kc / csz);
  const int c0 = s0 + (int)((long long)(s1 - s0) * warp / NW);
  const int c1 = s0 + (int)((long long)(s1 - s0) * (warp + 1) / NW);
  const uint4* wsec = reinterpret_cast<const uint4*>(p.packed + p.w_off);
  auto words = [&](int c, uint4& a, uint4& b) {   // the lane's 8 words of chunk c ([half][lane][4 words])
    const uint4* src = wsec + ((size_t)P * p.kc + c) * 64 + lane;
    a = ld_stream_v4(src);
    b = ld_stream_v4(src + 32);
  };
  uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = wa;
  if (c0 < c1) words(c0, wa, wb);

  if (tid == 0 && receiver) {
    mbar_init(recv_bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(recv_bar, (uint32_t)((csz - 1) * C::kTileBytes));
  }

  // ---- the panel's 16 row-pair tables: entry e = lo | hi << 4 of pair
  // slot brp holds (LUT_r[lo], LUT_r+16[hi]) in its four bank copies
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int task = tid + r * NCT;
    if (task >= 512) break;
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
  __syncthreads();
  if (csz > 1) cluster_sync_init();   // rank 0's receive barrier is armed before any rank sends

  // ---- activations and scales (after the grid-dependency wait)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t baseA = tab | ((uint32_t)g << 4) | ((uint32_t)t << 2);   // pairs (g, g+16)
  const uint32_t baseB = baseA | 128u;                                         // pairs (g+8, g+24)
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
  const uint8_t* abase = p.packed + p.ab_off + 16 * g;
  auto operands = [&](int c, uint4 (&xn)[NX][2], uint4& sc) {
#pragma unroll
    for (int h = 0; h < NX; ++h) {
      const uint16_t* src = xrow[h] + (size_t)c * kChunkCols;
      xn[h][0] = ld_nc_v4(src);
      xn[h][1] = ld_nc_v4(src + 8);
    }
    sc = ld_nc_v4(abase + (((size_t)P * p.groups + ((c * kChunkCols) >> p.g_shift)) << 7));
  };
  uint4 xn[NX][2], scn = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int h = 0; h < NX; ++h) xn[h][0] = xn[h][1] = make_uint4(0u, 0u, 0u, 0u);
  if (c0 < c1) operands(c0, xn, scn);

  float acc[NF / 4][4];
#pragma unroll
  for (int i = 0; i < NF / 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

  for (int c = c0; c < c1; ++c) {
    const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    uint32_t xw[NX][8];
#pragma unroll
    for (int h = 0; h < NX; ++h) {
      xw[h][0] = xn[h][0].x; xw[h][1] = xn[h][0].y; xw[h][2] = xn[h][0].z; xw[h][3] = xn[h][0].w;
      xw[h][4] = xn[h][1].x; xw[h][5] = xn[h][1].y; xw[h][6] = xn[h][1].z; xw[h][7] = xn[h][1].w;
    }
    const uint4 sc = scn;
    if (c + 1 < c1) {   // the next chunk's loads go out before this one is decoded
      words(c + 1, wa, wb);
      operands(c + 1, xn, scn);
    }
    // byte f = 4s + q of the words -> address bits 8..15 (linear.cu)
    auto addr = [&](int f, uint32_t b) { return prmt(w[f >> 2], b, 0x7604u | ((uint32_t)(f & 3) << 4)); };
    if (!C::kTr) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t a[4];
        a[0] = lds32(addr(4 * s + 0, baseA));
        a[1] = lds32(addr(4 * s + 1, baseB));
        a[2] = lds32(addr(4 * s + 2, baseA));
        a[3] = lds32(addr(4 * s + 3, baseB));
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
          e[u][0] = lds32(addr(4 * (s + u) + 0, baseA));
          e[u][1] = lds32(addr(4 * (s + u) + 1, baseB));
          e[u][2] = lds32(addr(4 * (s + u) + 2, baseA));
          e[u][3] = lds32(addr(4 * (s + u) + 3, baseB));
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
  }

  // ---- block sum in warp order, then the cluster's sum in rank order
#pragma unroll
  for (int i = 0; i < NF / 4; ++i)
    sts128(tiles + (uint32_t)(((warp * (NF / 4) + i) * 32 + lane) * 16), __float_as_uint(acc[i][0]),
           __float_as_uint(acc[i][1]), __float_as_uint(acc[i][2]), __float_as_uint(acc[i][3]));
  __syncthreads();
  if (warp != 0) return;
  float v[NF];
#pragma unroll
  for (int i = 0; i < NF / 4; ++i) {
    uint4 q = lds128(tiles + (uint32_t)((i * 32 + lane) * 16));
    float sx = __uint_as_float(q.x), sy = __uint_as_float(q.y), sz = __uint_as_float(q.z), sw = __uint_as_float(q.w);
    for (int w2 = 1; w2 < NW; ++w2) {
      q = lds128(tiles + (uint32_t)(((w2 * (NF / 4) + i) * 32 + lane) * 16));
      sx += __uint_as_float(q.x); sy += __uint_as_float(q.y); sz += __uint_as_float(q.z); sw += __uint_as_float(q.w);
    }
    v[4 * i + 0] = sx; v[4 * i + 1] = sy; v[4 * i + 2] = sz; v[4 * i + 3] = sw;
  }
  if (csz > 1 && crank > 0) {   // send this block's sum to rank 0
    const uint32_t bar0 = cluster_map(recv_bar, 0u);
#pragma unroll
    for (int i = 0; i < NF / 4; ++i) {
      const uint32_t dst = recv + (uint32_t)((((crank - 1) * (NF / 4) + i) * 32 + lane) * 16);
      st_async_v4(cluster_map(dst, 0u), v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], bar0);
    }
    return;
  }
  if (receiver) {
    // the other ranks wait on nothing before they send, so this bound is a
    // safety net: rank 0 may not exit before their bytes land
    bool ok = mbar_try_wait(recv_bar, 0u);
    if (!ok) {
      const long long t0 = clock64();
      while (!(ok = mbar_try_wait(recv_bar, 0u)) && clock64() - t0 < kSmallWaitCycles) {
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.status, kStatusWaitTimeout);
      return;
    }
    for (int r = 1; r < csz; ++r)
#pragma unroll
      for (int i = 0; i < NF / 4; ++i) {
        const uint4 q = lds128(recv + (uint32_t)((((r - 1) * (NF / 4) + i) * 32 + lane) * 16));
        v[4 * i + 0] += __uint_as_float(q.x);
        v[4 * i + 1] += __uint_as_float(q.y);
        v[4 * i + 2] += __uint_as_float(q.z);
        v[4 * i + 3] += __uint_as_float(q.w);
      }
  }
  // result i of this lane: (token, row) as in linear.cu
#pragma unroll
  for (int i = 0; i < NF; ++i) {
    int token, row;
    if (!C::kTr) {
      const int h = i >> 2, q = i & 3;   // D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]
      token = 4 * h + t;
      row = g + (q == 1 ? 16 : q == 2 ? 8 : q == 3 ? 24 : 0);
    } else {
      const int tile = i >> 3, h = (i >> 2) & 1, q = i & 3;
      token = 8 * h + 2 * t + (q & 1);
      row = 16 * tile + g + 8 * (q >> 1);
    }
    const int nrow = P * kPanelRows + row;
    if (token < p.m && nrow < p.n) {
      const __nv_bfloat16 hv = __float2bfloat16_rn(v[i]);
      p.y[(size_t)token * p.n + nrow] = *reinterpret_cast<const uint16_t*>(&hv);
    }
  }
}

template <int MODE>
cudaError_t small_allow_smem() {
  return cudaFuncSetAttribute(linear_small_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmallSmem);
}

template <int MODE>
cudaError_t small_launch(const SmallParams& p, int blocks, int cluster, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(SmallCfg<MODE>::kThreads);
  cfg.dynamicSmemBytes = kSmallSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, linear_small_kernel<MODE>, p);
}

}  // namespace

int small_warps(int m) { return m <= 4 ? SmallCfg<0>::kNW : m <= 8 ? SmallCfg<1>::kNW : SmallCfg<2>::kNW; }
int small_max_cluster() { return kSmallMaxCluster; }

cudaError_t launch_linear_small(const uint16_t* x, const uint8_t* packed, const Layout& L, int m, uint16_t* y,
                                void* workspace, int cluster, cudaStream_t stream) {
  static bool ready[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!ready[dev]) {
    e = small_allow_smem<0>();
    if (e == cudaSuccess) e = small_allow_smem<1>();
    if (e == cudaSuccess) e = small_allow_smem<2>();
    if (e != cudaSuccess) return e;
    ready[dev] = true;
  }
  SmallParams p{};
  p.x = x;
  p.packed = packed;
  p.y = y;
  p.status = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(workspace) + kCountersBytes);
  p.m = m; p.n = L.n; p.k = L.k;
  p.kc = L.kchunks; p.groups = L.groups;
  p.g_shift = 0;
  while ((1 << p.g_shift) < L.g) ++p.g_shift;
  p.cluster = cluster;
  p.w_off = L.w_off; p.lut_off = L.lut_off; p.ab_off = L.ab_off;
  const int blocks = L.panels * cluster;
  if (m <= 4) return small_launch<0>(p, blocks, cluster, stream);
  if (m <= 8) return small_launch<1>(p, blocks, cluster, stream);
  return small_launch<2>(p, blocks, cluster, stream);
}

}  // namespace any4
