// any4_linear_noalloc: the any4 linear layer for callers that cannot allocate
// device memory.
//
// Some callers never call cudaMalloc: code that runs as a plugin or operator
// inside a serving runtime that owns all device memory and hands a kernel only
// its input and output buffers, and latency-critical loops where cudaMalloc is
// banned because it can synchronize the device and take unbounded time. This
// entry point needs no workspace from them: the fp32 partial sums, arrival
// counters and status word of any4_linear live in a fixed array in this
// library's device memory instead.
//
// Costs and limits, stated for the user of this call:
//  * kNoAllocScratchBytes (8 MiB) of device memory is reserved on every GPU
//    that loads this library, for as long as the process runs.
//  * A shape whose plan needs more scratch than that is rejected with
//    ANY4_EWORKSPACE. The largest plan for M <= 16 is M = 9..16: a
//    256 KiB + 256 B header (arrival counters, status word) plus one partial
//    tile of 32 rows x 16 tokens in fp32 (2,048 bytes) per thread block, at
//    most one block per SM: 0.56 MB on a 148-SM B200, so every accepted shape
//    fits on any device with fewer than 3,900 SMs.
//  * All calls on a device share the one array and it keeps whatever the last
//    call left in it. Each call first clears the array's header (arrival
//    counters and status word) with an asynchronous memset on the caller's
//    stream (no allocation). Calls that may run at the same time on the GPU
//    (different streams without ordering between them) race on the array and
//    give wrong results: order them, or use any4_linear with separate
//    workspaces.
//  * A bounded wait that gives up inside the kernel sets the status word; it
//    is readable through any4_noalloc_status_word() until the next call on
//    that device clears it.
//  * The first call on a device (of either entry point below) looks up the
//    array's device address (cudaGetSymbolAddress, with that device current)
//    and caches it; make that first call before any stream capture on that
//    device.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/any4.h"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

// The scratch itself. In host code this name is only a handle for the runtime
// calls; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch on the current device, looked up once per
// device. Returns a cudaError_t.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" {

ANY4_API int any4_linear_noalloc(const uint16_t* x, const void* packed, int m, int n, int k,
                                 int group, uint16_t* y, any4_stream_t stream) {
  if (!x || !packed || !y) return ANY4_EINVAL;
  if (m < 1 || m > 16 || !any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(y, 4)) return ANY4_EALIGN;
  int sms = 0;
  cudaError_t e = any4::cached_sm_count(&sms);
  if (e != cudaSuccess) return any4::record_cuda_error(e);
  const any4::Layout L = any4::make_layout(n, k, group);
  const any4::LinearPlan plan = any4::plan_linear(m, L, sms);
  if (plan.workspace_bytes > kNoAllocScratchBytes) return ANY4_EWORKSPACE;
  void* scratch = nullptr;
  e = scratch_on_current_device(&scratch);
  // counters and status word start at zero for this call
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, any4::kHeaderBytes, (cudaStream_t)stream);
  if (e == cudaSuccess)
    e = any4::launch_linear(x, static_cast<const uint8_t*>(packed), L, m, y, scratch, plan,
                            (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : any4::record_cuda_error(e);
}

ANY4_API int any4_noalloc_status_word(const uint32_t** status) {
  if (!status) return ANY4_EINVAL;
  void* scratch = nullptr;
  const cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) return any4::record_cuda_error(e);
  *status = reinterpret_cast<const uint32_t*>(static_cast<uint8_t*>(scratch) + any4::kCountersBytes);
  return ANY4_OK;
}

}  // extern "C"
