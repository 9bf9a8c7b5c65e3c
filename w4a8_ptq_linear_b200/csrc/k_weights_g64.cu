// Asymmetric grouped INT4 weights (CentriQ: Calibration-Free Quantization of Diffusion
// Transformers via Exact Mean Centering, §3 Eq. 2 and §4.3; App. B.2 for the stored codes).
//
// Offline step after the rotation: every row of the rotated weight W_R is cut into groups of 64
// consecutive columns; round to nearest sets the group's scale and shift from its minimum and
// maximum, both are stored in fp16, and the codes are taken against the stored grid:
//   sigma = fp16(max((max - min) / 15, 2^-14, |min| / 2^15)),  z = fp16(-min / sigma),
//   Q = clamp(rint(w / sigma + z), 0, 15),  stored nibble Q - 8 (= Q xor 8).
// The 2^-14 floor keeps the grid from collapsing (smallest normal fp16); the |min| / 2^15 floor
// keeps the stored shift |z| below 2^15 (1 + 2^-11), finite in fp16, for a nearly constant group
// far from zero. Every step is one float32 operation rounded to nearest.
//
// K order: the GEMM decodes INT4 activation codes into an operand that holds, within every four
// consecutive K positions, elements 0, 2, 1, 3 (it skips an interleave). The grouped weights are
// stored in that order too: stored position p holds column pi(p), pi swapping bits 0 and 1 of
// the position (an involution that stays inside each group of 64).
#include <cuda_fp16.h>

#include <algorithm>

#include "oq_internal.h"

namespace oq {
namespace {

constexpr int kGroup = 64;

// One warp per (row, group): lane l holds columns l and 32 + l of the group. Byte j of block b of
// the GEMM layout holds stored positions 32b + j (low nibble) and 32b + 16 + j (high nibble),
// i.e. columns 32b + pi(j) and 32b + 16 + pi(j).
__global__ void __launch_bounds__(256) k_quant_g64(const float* __restrict__ rot, int64_t n,
                                                   int d, uint8_t* __restrict__ w_packed,
                                                   uint32_t* __restrict__ w_sz,
                                                   float* __restrict__ w_scale) {
  const int lane = threadIdx.x & 31;
  const int groups = d / kGroup;
  const int64_t n_items = n * groups;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t item = warp0; item < n_items; item += n_warps) {
    const int64_t row = item / groups;
    const int g = (int)(item % groups);
    const float* src = rot + row * (int64_t)d + (int64_t)g * kGroup;
    const float w0 = src[lane], w1 = src[32 + lane];
    float lo = fminf(w0, w1), hi = fmaxf(w0, w1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const float s = fmaxf(fmaxf(__fdiv_rn(__fsub_rn(hi, lo), 15.f), 0x1p-14f),
                          fabsf(lo) * 0x1p-15f);   // exact: a power-of-two scale
    const __half s16 = __float2half_rn(s);
    const float sf = __half2float(s16);
    const __half z16 = __float2half_rn(__fdiv_rn(-lo, sf));
    const float zf = __half2float(z16);
    auto code = [&](float w) {
      const float v = rintf(__fadd_rn(__fdiv_rn(w, sf), zf));
      return (uint32_t)fminf(fmaxf(v, 0.f), 15.f) ^ 8u;   // nibble of Q - 8
    };
    const uint32_t c0 = code(w0), c1 = code(w1);
    const int j = lane & 15;
    const int pj = (j & ~3) | ((j & 1) << 1) | ((j >> 1) & 1);   // pi(j)
    const uint32_t lo0 = __shfl_sync(0xffffffffu, c0, pj);
    const uint32_t hi0 = __shfl_sync(0xffffffffu, c0, 16 + pj);
    const uint32_t lo1 = __shfl_sync(0xffffffffu, c1, pj);
    const uint32_t hi1 = __shfl_sync(0xffffffffu, c1, 16 + pj);
    const uint32_t byte = lane < 16 ? (lo0 | (hi0 << 4)) : (lo1 | (hi1 << 4));
    w_packed[row * (int64_t)(d / 2) + (int64_t)g * 32 + lane] = (uint8_t)byte;
    if (lane == 0) {
      w_sz[(int64_t)g * n + row] = (uint32_t)__half_as_ushort(s16) |
                                   ((uint32_t)__half_as_ushort(z16) << 16);
      if (g == 0) w_scale[row] = 1.f;   // per-row scale s_i, 1 under round to nearest
    }
  }
}

}  // namespace

oq_status launch_quant_g64(const float* rot, int64_t n, int d, uint8_t* w_packed, uint32_t* w_sz,
                           float* w_scale, cudaStream_t s) {
  if (n == 0) return OQ_OK;
  if (d % kGroup) return fail(OQ_ERR_INVALID_ARG, "grouped weights need d % 64 == 0");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "device query");
  const int64_t warps = n * (d / kGroup);
  const int64_t blocks = std::min<int64_t>((warps + 7) / 8, (int64_t)sms * 16);
  k_quant_g64<<<(unsigned)blocks, 256, 0, s>>>(rot, n, d, w_packed, w_sz, w_scale);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? OQ_OK : cuda_fail(e, "launch k_quant_g64");
}

}  // namespace oq
