// Tensor-core peak microbenchmark: the roofline of the low-bit GEMMs, measured on this device
// by the same instruction the GEMMs issue.
//
// One CTA pair per two SMs (a cluster of two, as in the GEMM). The pair's leader issues `iters`
// groups of four back-to-back tcgen05.mma.cta_group::2 instructions, M = 256 (128 rows per
// CTA), N = 256, 128 bytes of K per group (kind::i8: K = 32 per instruction; kind::f16:
// K = 16), on operand tiles that stay in shared memory, into one TMEM accumulator. Nothing
// else runs: no loads, no conversion, no epilogue, so the time is the tensor pipe's own.
// The operands hold pseudo-random values (random int8, or fp16 of moderate magnitude), not
// zeros, so that the datapath toggles as it does on real data.
//
// Kind 2 (kind::i8, serialised) issues the same groups but commits each one to an mbarrier and
// waits for that arrive before issuing the next: its time per group minus kind 0's is the
// latency from the end of an MMA group to the completion seen by the issuing thread, the figure
// that sizes the GEMM's operand rings.
#include <algorithm>
#include <map>
#include <mutex>

#include "oq_internal.h"
#include "ptx.cuh"

namespace oq {
namespace {

constexpr int kPeakThreads = 128;
constexpr int kTile = 128 * 128;                  // one operand tile: 128 rows x 128 bytes
// A, B, alignment slack, barrier + TMEM slot, padded past half of an SM's shared memory so that
// exactly one CTA is resident per SM (the grid is one pair per two SMs)
constexpr int kPeakSmem = 150 * 1024;

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352du;
  x ^= x >> 15;
  x *= 0x846ca68bu;
  x ^= x >> 16;
  return x;
}

template <bool FP, bool SERIAL>
__global__ void __launch_bounds__(kPeakThreads, 1)
    k_mma_peak(int64_t iters, unsigned long long* err, unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + 2 * kTile);
  uint64_t* step = reinterpret_cast<uint64_t*>(smem + 2 * kTile + 16);   // serial kind
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + 2 * kTile + 8);
  const int tid = threadIdx.x;
  const uint32_t rank = dev::cluster_ctarank();

  // operands: A (128 rows of this CTA's M half) and B (this CTA's 128 rows of N)
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = tid; i < 2 * kTile / 4; i += kPeakThreads) {
    uint32_t r = mix32((uint32_t)i * 2654435761u + blockIdx.x * 97u + 1u);
    if constexpr (FP) {
      // two fp16 of magnitude in [2^-2, 2^2): random sign and mantissa, exponent 13..16
      const uint32_t e0 = 13u + (r & 3u), e1 = 13u + ((r >> 2) & 3u);
      r = (r & 0x83FF83FFu) | (e0 << 10) | (e1 << 26);
    }
    w[i] = r;
  }
  dev::fence_async_smem();
  if (tid == 0) {
    dev::mbar_init(dev::smem_u32(done), 1);
    dev::mbar_init(dev::smem_u32(step), 1);
    dev::fence_mbar_init_cluster();
  }
  if (tid < 32) {
    dev::tmem_alloc_pair(dev::smem_u32(tslot), 256);
    dev::tmem_relinquish_pair();
  }
  dev::tc_fence_before();
  dev::cluster_sync();
  dev::tc_fence_after();
  const uint32_t tmem = *tslot;

  if (rank == 0 && tid == 0) {
    constexpr uint32_t idesc = FP ? dev::idesc_f16(256, 256) : dev::idesc_i8(256, 256);
    const uint32_t a = dev::smem_u32(smem), b = dev::smem_u32(smem + kTile);
    for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = dev::sdesc_sw128(a + kk * 32);
        const uint64_t bd = dev::sdesc_sw128(b + kk * 32);
        if constexpr (FP)
          dev::mma_f16_pair(tmem, ad, bd, idesc, (it | kk) != 0);
        else
          dev::mma_i8_pair(tmem, ad, bd, idesc, (it | kk) != 0);
      }
      if constexpr (SERIAL) {   // the group's completion, seen by this thread
        dev::mma_commit_pair(dev::smem_u32(step));
        if (!dev::mbar_wait(dev::smem_u32(step), (uint32_t)(it & 1), err, kSitePeak, limit_ns))
          break;
      }
    }
    dev::mma_commit_pair(dev::smem_u32(done));   // arrives on both CTAs' barriers
  }
  if (tid == 0) dev::mbar_wait(dev::smem_u32(done), 0, err, kSitePeak, limit_ns);
  __syncwarp();
  dev::tc_fence_before();
  dev::cluster_sync();
  if (tid < 32) {
    dev::tc_fence_after();
    dev::tmem_dealloc_pair(tmem, 256);
  }
}

}  // namespace

oq_status launch_mma_peak(int kind, int64_t iters, int* pairs_out, cudaStream_t s) {
  const void* fn = kind == 0   ? reinterpret_cast<const void*>(&k_mma_peak<false, false>)
                   : kind == 1 ? reinterpret_cast<const void*>(&k_mma_peak<true, false>)
                               : reinterpret_cast<const void*>(&k_mma_peak<false, true>);
  cudaError_t e = allow_max_dynamic_smem(fn);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(mma_peak)");
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.blockDim = dim3(kPeakThreads);
  cfg.dynamicSmemBytes = kPeakSmem;
  cfg.gridDim = dim3(2 * (unsigned)std::max(nsm, 2));
  int pairs = 0;
  if (cudaOccupancyMaxActiveClusters(&pairs, fn, &cfg) != cudaSuccess || pairs <= 0) {
    cudaGetLastError();
    return fail(OQ_ERR_UNSUPPORTED, "mma_peak: no CTA pair fits");
  }
  // one pair per two SMs: a second resident pair on the same SMs would only share the pipe
  pairs = std::min(pairs, std::max(nsm / 2, 1));
  cfg.gridDim = dim3(2 * (unsigned)pairs);
  cfg.stream = s;
  unsigned long long* err = device_error_word();
  if (!err) return fail(OQ_ERR_CUDA, "device error word unavailable");
  const unsigned long long limit = kWaitLimitNs;
  e = kind == 0   ? cudaLaunchKernelEx(&cfg, &k_mma_peak<false, false>, iters, err, limit)
      : kind == 1 ? cudaLaunchKernelEx(&cfg, &k_mma_peak<true, false>, iters, err, limit)
                  : cudaLaunchKernelEx(&cfg, &k_mma_peak<false, true>, iters, err, limit);
  if (e != cudaSuccess) return cuda_fail(e, "launch mma_peak");
  if (pairs_out) *pairs_out = pairs;
  return OQ_OK;
}

}  // namespace oq

extern "C" oq_status oq_mma_peak_loop(int kind, int64_t iters, int* pairs_out, void* stream) {
  if (kind < 0 || kind > 2)
    return oq::fail(OQ_ERR_INVALID_ARG, "kind must be 0 (i8), 1 (f16) or 2 (i8, serialised)");
  // 2^16 groups of four MMAs take about 20 ms at the nominal rate (about 70 ms serialised), far
  // inside the 2 s bound on the completion wait (a wait that gave up must never be followed by the TMEM release while
  // MMAs still run)
  if (iters < 1 || iters > (int64_t)1 << 16)
    return oq::fail(OQ_ERR_INVALID_ARG, "iters out of [1, 2^16]");
  return oq::launch_mma_peak(kind, iters, pairs_out, static_cast<cudaStream_t>(stream));
}
