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

// Launch geometry of any4_linear for one shape on one device.
struct LinearPlan {
  int nt;               // n8 token tiles: 1 for M <= 8, 2 for M <= 16
  int warps;            // warps that receive atoms (each gets >= 1)
  int ctas;             // thread blocks
  long long atoms;      // (N/16) * (K/64)
  size_t counters_bytes;
  size_t partials_bytes;
  size_t workspace_bytes;
  size_t smem_bytes;    // dynamic shared memory per CTA
};

// The workspace starts with one arrival counter per possible 16-row tile, so
// the counters of every shape live in the same zero-initialised header
// whatever the shape of earlier calls; this bounds N at 16 * kMaxTiles rows.
constexpr int kMaxTiles = 65536;

LinearPlan plan_linear(int m, const Layout& L, int num_sms);

cudaError_t launch_linear(const uint16_t* x, const uint8_t* packed, const Layout& L, int m,
                          uint16_t* y, void* workspace, const LinearPlan& plan,
                          cudaStream_t stream);

}  // namespace any4
