// Allocation-free variant of oq_linear.
//
// oq_linear needs device scratch between its two kernels: the activation codes, per-token
// scales and means that the rotate+quantize kernel writes and the GEMM reads. Normally the
// caller passes that scratch as `workspace`. Some callers cannot allocate it: plug-ins that run
// inside a host framework which owns all device memory and hands out no allocator, and
// latency-critical paths that may not call cudaMalloc (it can synchronise the device).
// oq_linear_static_scratch takes the scratch from a fixed array that lives in this module
// instead, so it allocates nothing.
//
// The array is a file-scope __device__ variable of OQ_STATIC_SCRATCH_BYTES. Every device that
// loads the library holds one copy until the process exits. In host code the variable's name
// is only a host-side stand-in, not a device address. So on the first call on each device
// (that device current) the address is fetched once with cudaGetSymbolAddress and cached.
// That first call should therefore come before any stream capture. The cached address belongs
// to the device's primary context: cudaDeviceReset (or another teardown of that context) makes
// it stale, so after one the entry point must not be called again in the process. All calls on
// a device share the one array: calls whose kernels overlap on the GPU (different streams, or
// several host threads) race on it and must be serialised by the caller. The array keeps the previous call's
// contents. Nothing in it has to start at zero: the GEMM reads only codes, scales and means that
// the rotate+quantize kernel of the same call has just written (rows past T are never read).
#include <mutex>

#include "oq_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = OQ_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device, looked up once per device.
oq_status static_scratch_address(void** out) {
  constexpr int kMaxDev = 64;
  static void* addr[kMaxDev] = {};
  static std::mutex mu;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return oq::cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDev) return oq::fail(OQ_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return oq::cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return OQ_OK;
}

}  // namespace

extern "C" oq_status oq_linear_static_scratch(const oq_plan* plan, const void* x_bf16,
                                              int64_t T, int64_t ldx, const uint8_t* w_packed,
                                              const float* w_scale, const float* w_rowsum,
                                              const void* bias_bf16, int64_t d_out,
                                              void* y_bf16, void* stream) {
  if (!plan) return oq::fail(OQ_ERR_INVALID_ARG, "NULL plan");
  if (T < 0) return oq::fail(OQ_ERR_INVALID_ARG, "T out of range");
  const size_t need = oq_linear_workspace_bytes(plan, T);
  if (need > kStaticScratchBytes)
    return oq::fail(OQ_ERR_INVALID_ARG,
                    "oq_linear_static_scratch: T=%lld needs %zu bytes of scratch but the static "
                    "buffer holds %zu; split the batch or call oq_linear with a workspace",
                    (long long)T, need, kStaticScratchBytes);
  void* scratch = nullptr;
  oq_status st = static_scratch_address(&scratch);
  if (st != OQ_OK) return st;
  return oq_linear(plan, x_bf16, T, ldx, w_packed, w_scale, w_rowsum, bias_bf16, d_out, y_bf16,
                   scratch, kStaticScratchBytes, stream);
}
