// C ABI entry points (include/any4.h): argument checks, launch planning and
// error mapping. All compute happens in the kernels of pack_dequant.cu and
// linear.cu.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/any4.h"
#include "kernels.cuh"

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];   // per-device SM count cache (0 = unknown)

int fail_cuda(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return ANY4_ECUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

namespace any4 {
cudaError_t cached_sm_count(int* sms);
}

namespace {

// SM count of the current device (cached per device), or a negative status.
int current_sm_count(int* sms) {
  const cudaError_t e = any4::cached_sm_count(sms);
  return e == cudaSuccess ? ANY4_OK : fail_cuda(e);
}

}  // namespace

namespace any4 {
int record_cuda_error(cudaError_t e) { return fail_cuda(e); }

cudaError_t cached_sm_count(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = g_sm_count[dev].load(std::memory_order_relaxed);
    if (c > 0) {
      *sms = c;
      return cudaSuccess;
    }
  }
  int c = 0;
  e = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(c, std::memory_order_relaxed);
  *sms = c;
  return cudaSuccess;
}
}  // namespace any4

extern "C" {

size_t any4_packed_bytes(int n, int k, int group) {
  if (!any4::shape_ok(n, k, group)) return 0;
  return any4::make_layout(n, k, group).total;
}

int any4_pack(const uint8_t* idx_nib, const uint16_t* lut, const uint16_t* alpha,
              const uint16_t* beta, int n, int k, int group, void* packed, size_t packed_bytes,
              any4_stream_t stream) {
  if (!idx_nib || !lut || !alpha || !beta || !packed) return ANY4_EINVAL;
  if (!any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  if (!aligned(packed, 16)) return ANY4_EALIGN;
  const any4::Layout L = any4::make_layout(n, k, group);
  if (packed_bytes < L.total) return ANY4_EWORKSPACE;
  const cudaError_t e = any4::launch_pack(idx_nib, lut, alpha, beta, L,
                                          static_cast<uint8_t*>(packed), (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : fail_cuda(e);
}

int any4_dequant(const void* packed, int n, int k, int group, uint16_t* w, any4_stream_t stream) {
  if (!packed || !w) return ANY4_EINVAL;
  if (!any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  if (!aligned(packed, 16) || !aligned(w, 4)) return ANY4_EALIGN;
  const any4::Layout L = any4::make_layout(n, k, group);
  const cudaError_t e = any4::launch_dequant(static_cast<const uint8_t*>(packed), L, w,
                                             (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : fail_cuda(e);
}

size_t any4_linear_workspace_bytes(int m, int n, int k, int group) {
  if (m < 1 || m > any4::kMaxTokens || !any4::shape_ok(n, k, group)) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != ANY4_OK) return 0;
  return any4::plan_linear(m, any4::make_layout(n, k, group), sms).workspace_bytes;
}

size_t any4_linear_workspace_bytes_bits(int bits, int m, int n, int k, int group) {
  if (!any4::bits_ok(bits) || m < 1 || m > any4::kMaxTokens || !any4::shape_ok(n, k, group)) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != ANY4_OK) return 0;
  return any4::plan_linear(m, any4::make_layout(n, k, group, bits), sms).workspace_bytes;
}

int any4_linear_grid(int bits, int m, int n, int k, int group, int* blocks, int* cluster) {
  if (!blocks || !cluster) return ANY4_EINVAL;
  if (!any4::bits_ok(bits) || m < 1 || m > any4::kMaxTokens || !any4::shape_ok(n, k, group))
    return ANY4_ESHAPE;
  int sms = 0;
  const int st = current_sm_count(&sms);
  if (st != ANY4_OK) return st;
  const any4::LinearPlan plan = any4::plan_linear(m, any4::make_layout(n, k, group, bits), sms);
  *blocks = plan.ctas;
  *cluster = plan.mode == 3 ? 1 : plan.cluster;
  return ANY4_OK;
}

int any4_linear_kernel(int bits, int m, int n, int k, int group) {
  if (!any4::bits_ok(bits) || m < 1 || m > any4::kMaxTokens || !any4::shape_ok(n, k, group))
    return ANY4_ESHAPE;
  int sms = 0;
  const int st = current_sm_count(&sms);
  if (st != ANY4_OK) return st;
  const any4::Layout L = any4::make_layout(n, k, group, bits);
  const any4::LinearPlan plan = any4::plan_linear(m, L, sms);
  if (plan.mode == 3) return any4::prefill_fused(L, m) ? ANY4_KERNEL_PREFILL_FUSED : ANY4_KERNEL_PREFILL_GEMM;
  if (plan.small) return ANY4_KERNEL_SHARED_TABLES_DIRECT;
  return plan.regt ? ANY4_KERNEL_REGISTER_TABLES : ANY4_KERNEL_SHARED_TABLES;
}

int any4_linear(const uint16_t* x, const void* packed, int m, int n, int k, int group,
                uint16_t* y, void* workspace, size_t workspace_bytes, any4_stream_t stream) {
  if (!x || !packed || !y || !workspace) return ANY4_EINVAL;
  if (m < 1 || m > any4::kMaxTokens || !any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(y, 4) || !aligned(workspace, 16))
    return ANY4_EALIGN;
  int sms = 0;
  const int st = current_sm_count(&sms);
  if (st != ANY4_OK) return st;
  const any4::Layout L = any4::make_layout(n, k, group);
  const any4::LinearPlan plan = any4::plan_linear(m, L, sms);
  if (workspace_bytes < plan.workspace_bytes) return ANY4_EWORKSPACE;
  const cudaError_t e = any4::launch_linear(x, static_cast<const uint8_t*>(packed), L, m, y,
                                            workspace, plan, (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : fail_cuda(e);
}

size_t any4_packed_bytes_bits(int bits, int n, int k, int group) {
  if (!any4::bits_ok(bits) || !any4::shape_ok(n, k, group)) return 0;
  return any4::make_layout(n, k, group, bits).total;
}

int any4_pack_bits(int bits, const uint8_t* idx_nib, const uint16_t* lut, const uint16_t* alpha,
                   const uint16_t* beta, int n, int k, int group, void* packed, size_t packed_bytes,
                   any4_stream_t stream) {
  if (!idx_nib || !lut || !alpha || !beta || !packed) return ANY4_EINVAL;
  if (!any4::bits_ok(bits) || !any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  if (!aligned(packed, 16)) return ANY4_EALIGN;
  const any4::Layout L = any4::make_layout(n, k, group, bits);
  if (packed_bytes < L.total) return ANY4_EWORKSPACE;
  const cudaError_t e = any4::launch_pack(idx_nib, lut, alpha, beta, L,
                                          static_cast<uint8_t*>(packed), (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : fail_cuda(e);
}

int any4_dequant_bits(int bits, const void* packed, int n, int k, int group, uint16_t* w,
                      any4_stream_t stream) {
  if (!packed || !w) return ANY4_EINVAL;
  if (!any4::bits_ok(bits) || !any4::shape_ok(n, k, group)) return ANY4_ESHAPE;
  if (!aligned(packed, 16) || !aligned(w, 4)) return ANY4_EALIGN;
  const any4::Layout L = any4::make_layout(n, k, group, bits);
  const cudaError_t e = any4::launch_dequant(static_cast<const uint8_t*>(packed), L, w,
                                             (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : fail_cuda(e);
}

int any4_linear_bits(int bits, const uint16_t* x, const void* packed, int m, int n, int k, int group,
                     uint16_t* y, void* workspace, size_t workspace_bytes, any4_stream_t stream) {
  if (!x || !packed || !y || !workspace) return ANY4_EINVAL;
  if (!any4::bits_ok(bits) || m < 1 || m > any4::kMaxTokens || !any4::shape_ok(n, k, group))
    return ANY4_ESHAPE;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(y, 4) || !aligned(workspace, 16))
    return ANY4_EALIGN;
  int sms = 0;
  const int st = current_sm_count(&sms);
  if (st != ANY4_OK) return st;
  const any4::Layout L = any4::make_layout(n, k, group, bits);
  const any4::LinearPlan plan = any4::plan_linear(m, L, sms);
  if (workspace_bytes < plan.workspace_bytes) return ANY4_EWORKSPACE;
  const cudaError_t e = any4::launch_linear(x, static_cast<const uint8_t*>(packed), L, m, y,
                                            workspace, plan, (cudaStream_t)stream);
  return e == cudaSuccess ? ANY4_OK : fail_cuda(e);
}

const char* any4_strerror(int status) {
  switch (status) {
    case ANY4_OK: return "ANY4_OK: success";
    case ANY4_EINVAL: return "ANY4_EINVAL: null pointer or invalid size";
    case ANY4_EALIGN: return "ANY4_EALIGN: pointer misaligned";
    case ANY4_ESHAPE: return "ANY4_ESHAPE: M, N, K or group size not supported";
    case ANY4_EWORKSPACE: return "ANY4_EWORKSPACE: packed buffer or workspace too small";
    case ANY4_ECUDA: return "ANY4_ECUDA: CUDA runtime error (see any4_last_cuda_error)";
    default: return "unknown any4 status";
  }
}

int any4_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
