// any4_linear, M = 5..16, for shapes with few 32-row panels: row tables held
// in registers instead of shared memory.
//
// The explainer (10100.com, article 149119421, section 3) keeps each row's
// table in registers and decodes with native instructions. On B200 that
// decode is bound by the integer pipe (byte permutes at half rate), so the
// shared-table kernel (linear.cu) is faster wherever a warp streams many
// chunks of a panel. On shapes with few panels split over many thread blocks
// (the Llama K/V projections, 1024 x 4096) a warp sees only one or two
// chunks, and what a call then costs is its fixed work: building a 64 KB
// row-pair table per block and the block barriers around it. This kernel has
// none of it (for M <= 4, where the contraction is lighter, the shared tables
// with per-warp loads of linear_small.cu measured faster and take those
// shapes):
//
//  * grid: s thread blocks per panel (a thread-block cluster, s = 1, 2, 4), each
//    on a contiguous K slice; inside a block every warp takes its own chunks;
//  * decode: lane (g, t) loads its four rows' tables (g, g+8, g+16, g+24) as
//    byte planes (regdecode.cuh), turns its row-pair index words into per-row
//    selectors and decodes with byte permutes; w_hat = fma.rn.bf16x2(alpha,
//    LUT, beta) (rounded once to bf16), contracted with mma.sync m16n8k16
//    (fp32 accumulation), as in linear.cu;
//  * reduce: the block's warps add their fp32 tiles in warp order through
//    shared memory; the other ranks of the cluster send their block sums to
//    rank 0's shared memory (st.async, completing on its mbarrier) and rank 0
//    adds them in rank order and writes y: deterministic, no workspace.
//  * programmatic dependent launch: tables, scales and index words (the
//    immutable packed weight) are loaded before the grid-dependency wait; x
//    and y after it.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "regdecode.cuh"

namespace any4 {

namespace {

constexpr int kRegtMaxCluster = 4;   // 8-block clusters measured slower
constexpr long long kRegtWaitCycles = 8000000000ll;   // ~4 s: then rank 0 records a timeout

template <int NT8>
struct RegtCfg {
  static constexpr int kWarps = NT8 == 1 ? 16 : 8;    // <= 128 / 168 registers per thread
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTileBytes = 2 * NT8 * 32 * 16;   // one warp's fp32 tile: [u][h][lane] float4
  static constexpr int kSmem = 1024 + (kWarps + kRegtMaxCluster - 1) * kTileBytes;
};

struct RegtParams {
  const uint16_t* x;
  const uint8_t* packed;
  uint16_t* y;
  unsigned* status;
  int m, n, k;
  int kc, groups, g_shift;
  int cluster;   // thread blocks per panel
  size_t w_off, lut_off, ab_off;
};

template <int NT8>
__global__ void __launch_bounds__(RegtCfg<NT8>::kThreads, 1) linear_regt_kernel(const RegtParams p) {
  using C = RegtCfg<NT8>;
  constexpr int NW = C::kWarps;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int csz = p.cluster;
  const int crank = (int)(blockIdx.x % (unsigned)csz);
  const int P = (int)(blockIdx.x / (unsigned)csz);
  const uint32_t recv_bar = base;                  // rank 0: the other ranks' sums landed
  float4* tiles = reinterpret_cast<float4*>(smem + 1024);                    // [warp][u][h][lane]
  const uint32_t recv = base + 1024 + (uint32_t)(NW * C::kTileBytes);       // [rank-1][u][h][lane]
  const bool receiver = csz > 1 && crank == 0;

  if (tid == 0 && receiver) {
    mbar_init(recv_bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(recv_bar, (uint32_t)((csz - 1) * C::kTileBytes));
  }
  __syncthreads();
  if (csz > 1) cluster_sync_init();   // rank 0's receive barrier is armed before any rank sends
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // this warp's chunks: its share of the block's K slice of panel P
  const int s0 = (int)((long long)crank * p.kc / csz), s1 = (int)((long long)(crank + 1) * p.kc / csz);
  const int c0 = s0 + (int)((long long)(s1 - s0) * warp / NW);
  const int c1 = s0 + (int)((long long)(s1 - s0) * (warp + 1) / NW);

  // ---- immutable inputs first: tables, scales and index words
  const uint4* lsec = reinterpret_cast<const uint4*>(p.packed + p.lut_off);
  const uint4* wsec = reinterpret_cast<const uint4*>(p.packed + p.w_off);
  const uint4* asec = reinterpret_cast<const uint4*>(p.packed + p.ab_off);
  Planes T[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {   // rows g, g+8, g+16, g+24 of the panel
    const uint4* row = lsec + ((size_t)P * kPanelRows + g + 8 * r) * 2;
    T[r] = to_planes(ld_nc_v4(row), ld_nc_v4(row + 1));
  }
  auto words = [&](int c, uint4& a, uint4& b) {   // the lane's 8 words of chunk c ([half][lane][4 words])
    const uint4* src = wsec + ((size_t)P * p.kc + c) * 64 + lane;
    a = ld_stream_v4(src);
    b = ld_stream_v4(src + 32);
  };
  auto scales = [&](int c) { return ld_nc_v4(asec + ((size_t)P * p.groups + ((c * kChunkCols) >> p.g_shift)) * 8 + g); };
  uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = wa, rec = wa;
  if (c0 < c1) {
    words(c0, wa, wb);
    rec = scales(c0);
  }

  // ---- activations: lane (g, t) feeds token g (+8 for the second tile) with
  // columns 16t .. 16t+15 of each chunk; tokens >= M are zero
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const bool tok0 = g < p.m, tok1 = NT8 > 1 && g + 8 < p.m;
  const uint16_t* x0 = p.x + (size_t)(tok0 ? g : 0) * p.k + 16 * t;
  const uint16_t* x1 = p.x + (size_t)(tok1 ? g + 8 : 0) * p.k + 16 * t;
  auto load_x = [&](int c, uint4 (&xn)[NT8][2]) {
    const size_t off = (size_t)c * kChunkCols;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    xn[0][0] = tok0 ? ld_nc_v4(x0 + off) : z;
    xn[0][1] = tok0 ? ld_nc_v4(x0 + off + 8) : z;
    if (NT8 > 1) {
      xn[NT8 - 1][0] = tok1 ? ld_nc_v4(x1 + off) : z;
      xn[NT8 - 1][1] = tok1 ? ld_nc_v4(x1 + off + 8) : z;
    }
  };
  uint4 xn[NT8][2];
  if (c0 < c1) load_x(c0, xn);

  float acc[2][NT8][4];
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int h = 0; h < NT8; ++h) acc[u][h][0] = acc[u][h][1] = acc[u][h][2] = acc[u][h][3] = 0.0f;

  for (int c = c0; c < c1; ++c) {
    const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    uint32_t xw[NT8][8];
#pragma unroll
    for (int h = 0; h < NT8; ++h) {
      xw[h][0] = xn[h][0].x; xw[h][1] = xn[h][0].y; xw[h][2] = xn[h][0].z; xw[h][3] = xn[h][0].w;
      xw[h][4] = xn[h][1].x; xw[h][5] = xn[h][1].y; xw[h][6] = xn[h][1].z; xw[h][7] = xn[h][1].w;
    }
    uint32_t al[4], be[4];
    scale_pairs(rec, al, be);
    if (c + 1 < c1) {   // the next chunk's loads go out before this one is decoded
      words(c + 1, wa, wb);
      rec = scales(c + 1);
      load_x(c + 1, xn);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {   // k16 step j: columns 16t + 4j .. +3
      uint32_t t0, t1;
      rowpair_to_selectors(w[2 * j], w[2 * j + 1], t0, t1);
      uint32_t a[4], b[4];
      decode8(T[0], T[1], t0, a);   // tile 0: rows g, g+8
      decode8(T[2], T[3], t1, b);   // tile 1: rows g+16, g+24
      a[0] = fma_bf16x2(a[0], al[0], be[0]);
      a[2] = fma_bf16x2(a[2], al[0], be[0]);
      a[1] = fma_bf16x2(a[1], al[1], be[1]);
      a[3] = fma_bf16x2(a[3], al[1], be[1]);
      b[0] = fma_bf16x2(b[0], al[2], be[2]);
      b[2] = fma_bf16x2(b[2], al[2], be[2]);
      b[1] = fma_bf16x2(b[1], al[3], be[3]);
      b[3] = fma_bf16x2(b[3], al[3], be[3]);
#pragma unroll
      for (int h = 0; h < NT8; ++h) {
        mma_m16n8k16(acc[0][h], a, xw[h][2 * j], xw[h][2 * j + 1]);
        mma_m16n8k16(acc[1][h], b, xw[h][2 * j], xw[h][2 * j + 1]);
      }
    }
  }

  // ---- block sum in warp order, then the cluster's sum in rank order
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int h = 0; h < NT8; ++h)
      tiles[((warp * 2 + u) * NT8 + h) * 32 + lane] = make_float4(acc[u][h][0], acc[u][h][1], acc[u][h][2], acc[u][h][3]);
  __syncthreads();
  if (warp != 0) return;
  float v[2][NT8][4];
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int h = 0; h < NT8; ++h) {
      float4 sum = tiles[(u * NT8 + h) * 32 + lane];
      for (int w = 1; w < NW; ++w) {
        const float4 q = tiles[((w * 2 + u) * NT8 + h) * 32 + lane];
        sum.x += q.x; sum.y += q.y; sum.z += q.z; sum.w += q.w;
      }
      v[u][h][0] = sum.x; v[u][h][1] = sum.y; v[u][h][2] = sum.z; v[u][h][3] = sum.w;
    }
  if (csz > 1 && crank > 0) {   // send this block's sum to rank 0
    const uint32_t bar0 = cluster_map(recv_bar, 0u);
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int h = 0; h < NT8; ++h) {
        const uint32_t dst = recv + (uint32_t)(((((crank - 1) * 2 + u) * NT8 + h) * 32 + lane) * 16);
        st_async_v4(cluster_map(dst, 0u), v[u][h][0], v[u][h][1], v[u][h][2], v[u][h][3], bar0);
      }
    return;
  }
  if (receiver) {
    // every other rank sends; rank 0 may not exit before their bytes land.
    // The other ranks wait on nothing before they send (their loads and
    // decode only), so the bound is a safety net that a running cluster
    // never reaches: the cluster's blocks are co-scheduled.
    bool ok = mbar_try_wait(recv_bar, 0u);
    if (!ok) {
      const long long t0 = clock64();
      while (!(ok = mbar_try_wait(recv_bar, 0u)) && clock64() - t0 < kRegtWaitCycles) {
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.status, kStatusWaitTimeout);
      return;
    }
    const float4* rb = reinterpret_cast<const float4*>(smem + (recv - base));
    for (int r = 1; r < csz; ++r)
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int h = 0; h < NT8; ++h) {
          const float4 q = rb[((((r - 1) * 2 + u) * NT8 + h) * 32 + lane)];
          v[u][h][0] += q.x; v[u][h][1] += q.y; v[u][h][2] += q.z; v[u][h][3] += q.w;
        }
  }
  // D fragment: (row g, tokens 2t, 2t+1), (row g+8, tokens 2t, 2t+1) per tile
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int h = 0; h < NT8; ++h)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = P * kPanelRows + 16 * u + g + 8 * (q >> 1);
        const int tok = 8 * h + 2 * t + (q & 1);
        if (row < p.n && tok < p.m) {
          const __nv_bfloat16 hv = __float2bfloat16_rn(v[u][h][q]);
          p.y[(size_t)tok * p.n + row] = *reinterpret_cast<const uint16_t*>(&hv);
        }
      }
}

template <int NT8>
cudaError_t regt_allow_smem() {
  return cudaFuncSetAttribute(linear_regt_kernel<NT8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              RegtCfg<NT8>::kSmem);
}

}  // namespace

int regt_warps(int m) { return m <= 8 ? RegtCfg<1>::kWarps : RegtCfg<2>::kWarps; }
int regt_max_cluster() { return kRegtMaxCluster; }

cudaError_t launch_linear_regt(const uint16_t* x, const uint8_t* packed, const Layout& L, int m, uint16_t* y,
                               void* workspace, int cluster, cudaStream_t stream) {
  static bool ready[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!ready[dev]) {
    e = regt_allow_smem<1>();
    if (e == cudaSuccess) e = regt_allow_smem<2>();
    if (e != cudaSuccess) return e;
    ready[dev] = true;
  }
  RegtParams p{};
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(L.panels * cluster));
  cfg.blockDim = dim3(m <= 8 ? RegtCfg<1>::kThreads : RegtCfg<2>::kThreads);
  cfg.dynamicSmemBytes = m <= 8 ? RegtCfg<1>::kSmem : RegtCfg<2>::kSmem;
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
  return m <= 8 ? cudaLaunchKernelEx(&cfg, linear_regt_kernel<1>, p) : cudaLaunchKernelEx(&cfg, linear_regt_kernel<2>, p);
}

}  // namespace any4
