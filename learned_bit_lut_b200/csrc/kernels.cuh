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

cudaError_t launch_dequant(const uint8_t* packed, const Layout& L, uint16_t* w,
                           cudaStream_t stream);

// The workspace of any4_linear starts with a fixed header of arrival
// counters (one per possible 16-row tile, so the counters of every shape live
// in the same zero-filled header whatever the shape of earlier calls), then a
// reserved 256-byte word area, then the fp32 partial tiles.
constexpr int kMaxTiles = kMaxRows / kTileRows;                 // 65536
constexpr size_t kCountersBytes = (size_t)kMaxTiles * sizeof(unsigned);
constexpr size_t kHeaderBytes = kCountersBytes + 256;

// Launch geometry of any4_linear for one shape on one device.
struct LinearPlan {
  int nt;               // 8-token MMA column tiles: 1 for M <= 8, 2 for M <= 16
  long long atoms;      // 32-row blocks x K/64
  int ctas;             // persistent thread blocks
  size_t partials_bytes;
  size_t workspace_bytes;
};

LinearPlan plan_linear(int m, const Layout& L, int num_sms);

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream);

}  // namespace any4
