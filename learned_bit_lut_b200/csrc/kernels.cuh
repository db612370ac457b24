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

// The workspace of any4_linear starts with one arrival counter per possible
// 128-row tile, so the counters of every shape live in the same zero-filled
// header whatever the shape of earlier calls; then one error word; then the
// fp32 partial tiles.
constexpr int kMaxTiles = kMaxRows / kTileRows;                 // 8192
constexpr size_t kCountersBytes = (size_t)kMaxTiles * sizeof(unsigned);
constexpr size_t kHeaderBytes = kCountersBytes + 256;           // + error word, padded

// Launch geometry of any4_linear for one shape on one device.
struct LinearPlan {
  long long units;      // tiles * chunks (one unit = 128 rows x 64 columns)
  int ctas;             // persistent CTAs, one per SM at most
  size_t partials_bytes;
  size_t workspace_bytes;
};

LinearPlan plan_linear(int m, const Layout& L, int num_sms);

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream);

}  // namespace any4
