// Launchers of the any4 kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "device_ops.cuh"
#include "layout.cuh"

namespace any4 {

cudaError_t launch_pack(const uint8_t* idx_nib, const uint16_t* lut, const uint16_t* alpha,
                        const uint16_t* beta, const Layout& L, uint8_t* packed,
                        cudaStream_t stream);

// Pack with the same table in every row (fixed-table formats).
cudaError_t launch_pack_fixed(const uint8_t* idx_nib, const uint16_t (&lut)[16],
                              const uint16_t* alpha, const uint16_t* beta, const Layout& L,
                              uint8_t* packed, cudaStream_t stream);

// any4 quantizer (group scaling + weighted k-means), one thread per row.
cudaError_t launch_quantize(const uint16_t* w, const double* ex, int n, int k, int g, int bits,
                            int iters, uint8_t* idx_nib, uint16_t* lut, uint16_t* alpha,
                            uint16_t* beta, cudaStream_t stream);

// Keeps e for any4_last_cuda_error() on this host thread; returns ANY4_ECUDA.
int record_cuda_error(cudaError_t e);

// SM count of the current device, queried once per device and cached.
cudaError_t cached_sm_count(int* sms);

// The 16 bf16 values of a fixed-table format (any4_format); false if unknown.
bool format_table(int format, uint16_t (&lut)[16]);

cudaError_t launch_dequant(const uint8_t* packed, const Layout& L, uint16_t* w,
                           cudaStream_t stream);

// The workspace of any4_linear starts with a fixed header of arrival
// counters (one per possible 32-row panel, so the counters of every shape live
// in the same zero-filled header whatever the shape of earlier calls; sized for
// 16-row tiles, which leaves room), then a reserved 256-byte word area whose
// first word is the device status (0, or kStatusWaitTimeout when a kernel gave
// up waiting for one of its own copies), then the fp32 partial sums.
constexpr int kMaxTiles = kMaxRows / kTileRows;                 // 65536
constexpr size_t kCountersBytes = (size_t)kMaxTiles * sizeof(unsigned);
constexpr size_t kHeaderBytes = kCountersBytes + 256;
constexpr unsigned kStatusWaitTimeout = 1u;

// M > 16 (prefill): bf16 W_hat scratch at prefill_scratch_offset() of the
// workspace, then a tcgen05 GEMM (prefill.cu).
size_t prefill_scratch_offset();
bool prefill_fused(const Layout& L, int m);   // M > 16 decodes into the GEMM's shared memory
size_t prefill_workspace_bytes(const Layout& L, int m, int num_sms);
cudaError_t launch_prefill(const uint16_t* x, const uint8_t* packed, const Layout& L, int m, uint16_t* y,
                           void* workspace, int num_sms, cudaStream_t stream);

// Launch geometry of any4_linear for one shape on one device.
struct LinearPlan {
  int mode;             // 0: M <= 4, 1: M <= 8 (row-pair operands); 2: M <= 16 (row operands); 3: M > 16
  int nf;               // fp32 results per lane and panel
  long long units;      // panels x K/64 chunks
  int ctas;             // persistent thread blocks (one per SM at most)
  int cluster;          // thread blocks sharing one panel as a cluster (K slices), or 1
  bool regt;            // register-table kernel (linear_regt.cu) instead of linear.cu's
  bool small;           // shared-table kernel without streaming structure (linear_small.cu)
  size_t partials_bytes;
  size_t workspace_bytes;
};

LinearPlan plan_linear(int m, const Layout& L, int num_sms);

// M <= 16, any4, few chunks per thread block: row tables in registers, one
// cluster of `cluster` blocks per panel (linear_regt.cu).
int regt_warps(int m);
int regt_max_cluster();
cudaError_t launch_linear_regt(const uint16_t* x, const uint8_t* packed, const Layout& L, int m, uint16_t* y,
                               void* workspace, int cluster, cudaStream_t stream);

// M <= 16, any4, few chunks per thread block: the row-pair tables in shared
// memory, one cluster of `cluster` blocks per panel (linear_small.cu).
int small_warps(int m);
int small_max_cluster();
cudaError_t launch_linear_small(const uint16_t* x, const uint8_t* packed, const Layout& L, int m, uint16_t* y,
                                void* workspace, int cluster, cudaStream_t stream);

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream);

}  // namespace any4
