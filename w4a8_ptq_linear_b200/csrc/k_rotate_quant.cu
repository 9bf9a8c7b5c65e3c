// Fused per-token center + RPBH rotation + scale + quantize (the activation path of CentriQ
// §4.2 and App. B.2; OrbitQuant PR #25 "Runtime work": the pre-rotation as one kernel).
//
// Design (HBM-bound; one token row = d bf16 values):
//  - Persistent CTAs. Each CTA walks tokens t = blockIdx.x, blockIdx.x + gridDim.x, ...; one
//    thread streams whole rows into shared memory with 1-D bulk copies (TMA), `nbuf` rows
//    ahead, each completing on its own mbarrier.
//  - Thread i owns E consecutive rotated positions [i*E, i*E + E). Its entries of the plan
//    table (permutation index | sign << 15, one uint16 per position and round) stay in
//    registers for the whole kernel.
//  - Round r: gather u_k = s_k * z[pi_k] from shared memory, then the Sylvester transform on
//    blocks of h: log2(E) butterfly stages inside the thread, then log2(h/E) stages across
//    lanes with shuffles (h <= 32 E, so a block never leaves its warp). The second round
//    gathers from an fp32 copy of the first round's output in shared memory.
//  - Centering uses the sum of the gathered values (a permutation keeps the sum), so the
//    mean costs one block reduction and no extra pass over the row.
//  - Per-token absmax (or sum of squares for Lloyd-Max) by warp shuffles + one block
//    reduction, then codes are written as packed int8 / nibbles with vector stores.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "oq_internal.h"
#include "ptx.cuh"

namespace oq {
namespace {

struct RqParams {
  const __nv_bfloat16* x;
  int64_t ldx, T;
  int d, hlog2, rounds, center, mode, nbuf, want_sum;
  const uint16_t* tab;
  void* codes;
  float* scale;
  float* mean;
  float* rotated;
  float* rowsum;
  float thr[16];
  float inv_norm;
  unsigned long long* err;
  unsigned long long limit_ns;
};

template <int E>
__device__ __forceinline__ void fwht_block(float (&v)[E], int lane, int hlog2) {
  const int h = 1 << hlog2;
#pragma unroll
  for (int len = 1; len < E; len <<= 1) {
    if (len >= h) break;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if (!(i & len)) {
        const float a = v[i], b = v[i | len];
        v[i] = a + b;
        v[i | len] = a - b;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    if (m * E >= h) break;
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ uint32_t tab_entry(const uint32_t* t, int i) {
  return (t[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu;
}

template <int E, int MAXT>
__global__ void __launch_bounds__(MAXT) k_rotate_quant(const RqParams p) {
  // The round-2 table stays in registers unless a 1024-thread block would spill it; then it
  // is read per token from the L1-resident plan table.
  constexpr bool kT1Regs = (E < 32) || (MAXT <= 256);
  extern __shared__ __align__(1024) uint8_t smem[];
  const int d = p.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int base = tid * E;
  const bool active = base < d;
  const uint32_t row_bytes = (uint32_t)d * 2u;
  const uint32_t row_stride = (row_bytes + 127u) & ~127u;
  uint8_t* rowbuf = smem;
  float* rbuf = reinterpret_cast<float*>(smem + (size_t)p.nbuf * row_stride);
  float* red = rbuf + (p.rounds == 2 ? d : 0);   // [0,32) sums, [32,64) max / sumsq
  float* thr = red + 64;
  uint64_t* bars = reinterpret_cast<uint64_t*>(thr + 16);

  // plan entries of my positions, two uint16 per register
  uint32_t t0[E / 2], t1[E / 2];
#pragma unroll
  for (int i = 0; i < E / 2; ++i) t0[i] = t1[i] = 0u;
  if (active) {
    const uint4* s0 = reinterpret_cast<const uint4*>(p.tab + base);
#pragma unroll
    for (int i = 0; i < E / 8; ++i) {
      const uint4 q = __ldg(s0 + i);
      t0[4 * i] = q.x; t0[4 * i + 1] = q.y; t0[4 * i + 2] = q.z; t0[4 * i + 3] = q.w;
    }
    if (kT1Regs && p.rounds == 2) {
      const uint4* s1 = reinterpret_cast<const uint4*>(p.tab + d + base);
#pragma unroll
      for (int i = 0; i < E / 8; ++i) {
        const uint4 q = __ldg(s1 + i);
        t1[4 * i] = q.x; t1[4 * i + 1] = q.y; t1[4 * i + 2] = q.z; t1[4 * i + 3] = q.w;
      }
    }
  }
  if (tid < 16) thr[tid] = p.thr[tid];
  if (tid == 0) {
    for (int b = 0; b < p.nbuf; ++b) dev::mbar_init(dev::smem_u32(&bars[b]), 1);
    dev::fence_mbar_init();
  }
  __syncthreads();

  const int64_t T = p.T;
  const int64_t G = gridDim.x;
  // thread 0 keeps the row loads nbuf tokens ahead
  if (tid == 0) {
    for (int b = 0; b < p.nbuf; ++b) {
      const int64_t tt = (int64_t)blockIdx.x + (int64_t)b * G;
      if (tt < T) {
        const uint32_t bar = dev::smem_u32(&bars[b]);
        dev::mbar_arrive_expect_tx(bar, row_bytes);
        dev::bulk_g2s(dev::smem_u32(rowbuf + (size_t)b * row_stride), p.x + tt * p.ldx,
                      row_bytes, bar);
      }
    }
  }

  int it = 0;
  bool aborted = false;
  for (int64_t t = blockIdx.x; t < T; t += G, ++it) {
    const int b = it % p.nbuf;
    const uint32_t parity = (uint32_t)(it / p.nbuf) & 1u;
    int fail = !dev::mbar_wait(dev::smem_u32(&bars[b]), parity, p.err, kSiteRqRow, p.limit_ns);

    // ---- round 1: gather from the bf16 row, apply signs --------------------------------
    float v[E];
    float psum = 0.f;
    const __nv_bfloat16* row =
        reinterpret_cast<const __nv_bfloat16*>(rowbuf + (size_t)b * row_stride);
#pragma unroll
    for (int i = 0; i < E; ++i) {
      float g = 0.f;
      const uint32_t e = tab_entry(t0, i);
      if (active && !fail) g = __bfloat162float(row[e & 0x7FFFu]);
      psum += g;
      v[i] = (e & 0x8000u) ? -g : g;
    }
    if (p.want_sum) {
      psum = warp_sum(psum);
      if (lane == 0) red[warp] = psum;
    }
    fail = __syncthreads_or(fail);
    if (fail) {
      aborted = true;
      break;
    }
    if (tid == 0) {  // row buffer b is free again
      const int64_t tn = t + (int64_t)p.nbuf * G;
      if (tn < T) {
        const uint32_t bar = dev::smem_u32(&bars[b]);
        dev::mbar_arrive_expect_tx(bar, row_bytes);
        dev::bulk_g2s(dev::smem_u32(rowbuf + (size_t)b * row_stride), p.x + tn * p.ldx,
                      row_bytes, bar);
      }
    }
    if (p.want_sum) {
      float s = 0.f;
      for (int w = 0; w < nwarps; ++w) s += red[w];
      if (p.center) {
        const float mu = s / (float)d;
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] -= (tab_entry(t0, i) & 0x8000u) ? -mu : mu;
        if (tid == 0) p.mean[t] = mu;
      }
      if (tid == 0 && p.rowsum) p.rowsum[t] = s;
    }
    fwht_block<E>(v, lane, p.hlog2);

    // ---- round 2: through an fp32 copy in shared memory --------------------------------
    if (p.rounds == 2) {
      if (active) {
        float4* dst = reinterpret_cast<float4*>(rbuf + base);
#pragma unroll
        for (int i = 0; i < E / 4; ++i)
          dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
      __syncthreads();
      if (!kT1Regs && active) {
        const uint4* s1 = reinterpret_cast<const uint4*>(p.tab + d + base);
#pragma unroll
        for (int i = 0; i < E / 8; ++i) {
          const uint4 q = __ldg(s1 + i);
          t1[4 * i] = q.x; t1[4 * i + 1] = q.y; t1[4 * i + 2] = q.z; t1[4 * i + 3] = q.w;
        }
      }
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const uint32_t e = tab_entry(t1, i);
        const float g = active ? rbuf[e & 0x7FFFu] : 0.f;
        v[i] = (e & 0x8000u) ? -g : g;
      }
      fwht_block<E>(v, lane, p.hlog2);
    }

    // ---- per-token statistic ---------------------------------------------------------------
    float stat = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      v[i] *= p.inv_norm;
      stat = (p.mode == kRqLloydMax) ? fmaf(v[i], v[i], stat) : fmaxf(stat, fabsf(v[i]));
    }
    stat = (p.mode == kRqLloydMax) ? warp_sum(stat) : warp_max(stat);
    if (lane == 0) red[32 + warp] = stat;
    __syncthreads();
    stat = 0.f;
    for (int w = 0; w < nwarps; ++w)
      stat = (p.mode == kRqLloydMax) ? stat + red[32 + w] : fmaxf(stat, red[32 + w]);

    if (p.rotated && active) {
      float4* dst = reinterpret_cast<float4*>(p.rotated + t * (int64_t)d + base);
#pragma unroll
      for (int i = 0; i < E / 4; ++i)
        dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }

    // ---- quantize + store ---------------------------------------------------------------------
    if (p.mode == kRqLloydMax) {
      const float sigma = fmaxf(sqrtf(stat / (float)d), 1e-10f);
      const float inv = 1.0f / sigma;
      if (tid == 0) p.scale[t] = sigma;
      if (active) {
        uint32_t packed[E / 8];
#pragma unroll
        for (int j = 0; j < E / 8; ++j) packed[j] = 0u;
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const float u = v[i] * inv;
          int c = (u > thr[7]) ? 8 : 0;
          c += (u > thr[c + 3]) ? 4 : 0;
          c += (u > thr[c + 1]) ? 2 : 0;
          c += (u > thr[c]) ? 1 : 0;
          packed[i >> 3] |= (uint32_t)c << ((i & 7) * 4);
        }
        uint8_t* dst = reinterpret_cast<uint8_t*>(p.codes) + t * (int64_t)(d / 2) + base / 2;
        if constexpr (E == 8) {
          *reinterpret_cast<uint32_t*>(dst) = packed[0];
        } else if constexpr (E == 16) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
        } else {
          *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
    } else {
      const float qmax = (p.mode == kRqInt8) ? 127.f : 7.f;
      const float a = fmaxf(stat, 1e-10f);
      const float r = qmax / a;
      if (tid == 0) p.scale[t] = a / qmax;
      if (active) {
        if (p.mode == kRqInt8) {
          uint32_t packed[E / 4];
#pragma unroll
          for (int j = 0; j < E / 4; ++j) packed[j] = 0u;
#pragma unroll
          for (int i = 0; i < E; ++i) {
            const float q = fminf(fmaxf(rintf(v[i] * r), -qmax), qmax);
            packed[i >> 2] |= ((uint32_t)(int32_t)q & 0xFFu) << ((i & 3) * 8);
          }
          uint8_t* dst = reinterpret_cast<uint8_t*>(p.codes) + t * (int64_t)d + base;
          if constexpr (E == 8) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
          } else {
#pragma unroll
            for (int j = 0; j < E / 16; ++j)
              reinterpret_cast<uint4*>(dst)[j] =
                  make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
        } else {
          uint32_t packed[E / 8];
#pragma unroll
          for (int j = 0; j < E / 8; ++j) packed[j] = 0u;
#pragma unroll
          for (int i = 0; i < E; ++i) {
            const float q = fminf(fmaxf(rintf(v[i] * r), -qmax), qmax);
            packed[i >> 3] |= ((uint32_t)(int32_t)q & 0xFu) << ((i & 7) * 4);
          }
          uint8_t* dst = reinterpret_cast<uint8_t*>(p.codes) + t * (int64_t)(d / 2) + base / 2;
          if constexpr (E == 8) {
            *reinterpret_cast<uint32_t*>(dst) = packed[0];
          } else if constexpr (E == 16) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
          } else {
            *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          }
        }
      }
    }
  }

  // After an abort, wait (bounded) for row loads this CTA still has in flight so that no
  // bulk copy lands in shared memory after the block has exited.
  if (aborted && tid == 0) {
    for (int k = 0; k < p.nbuf; ++k) {
      const int j = it + k;  // iteration whose load may be outstanding
      const int64_t tt = (int64_t)blockIdx.x + (int64_t)j * G;
      if (tt >= T) break;
      const int b = j % p.nbuf;
      dev::mbar_wait(dev::smem_u32(&bars[b]), (uint32_t)(j / p.nbuf) & 1u, p.err, kSiteRqDrain,
                     p.limit_ns);
    }
  }
}

template <int E, int MAXT>
void* rq_kernel() {
  return reinterpret_cast<void*>(&k_rotate_quant<E, MAXT>);
}

}  // namespace

oq_status launch_rotate_quant(const RqArgs& a, cudaStream_t s) {
  if (a.T == 0) return OQ_OK;
  int hlog2 = 0;
  while ((1 << hlog2) < a.h) ++hlog2;
  int E;
  if (a.h <= 256 && a.d <= 8192) E = 8;
  else if (a.h <= 512 && a.d <= 16384) E = 16;
  else E = 32;
  const int nthr = ((a.d / E + 31) / 32) * 32;

  int dev_id = 0;
  cudaError_t ce = cudaGetDevice(&dev_id);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  int nsm = 0, max_smem = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev_id);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev_id);

  const size_t row_stride = ((size_t)a.d * 2 + 127) & ~(size_t)127;
  const size_t fixed = (a.rounds == 2 ? (size_t)a.d * 4 : 0) + 64 * 4 + 16 * 4;
  int nbuf = 3;
  while (nbuf > 1 && fixed + nbuf * row_stride + nbuf * 8 > (size_t)max_smem / 2) --nbuf;
  const size_t smem = fixed + nbuf * row_stride + nbuf * 8;
  if (smem > (size_t)max_smem) return fail(OQ_ERR_UNSUPPORTED, "rotate_quant: d too large");

  void* fn = (E == 8)    ? rq_kernel<8, 1024>()
             : (E == 16) ? rq_kernel<16, 1024>()
             : (nthr <= 256) ? rq_kernel<32, 256>() : rq_kernel<32, 1024>();
  ce = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(rotate_quant)");
  int occ = 0;
  ce = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, nthr, smem);
  if (ce != cudaSuccess) return cuda_fail(ce, "occupancy(rotate_quant)");
  occ = std::max(occ, 1);
  const int64_t grid = std::min<int64_t>(a.T, (int64_t)nsm * occ);

  RqParams p{};
  p.x = reinterpret_cast<const __nv_bfloat16*>(a.x);
  p.ldx = a.ldx;
  p.T = a.T;
  p.d = a.d;
  p.hlog2 = hlog2;
  p.rounds = a.rounds;
  p.center = a.center;
  p.mode = a.mode;
  p.nbuf = nbuf;
  p.want_sum = (a.center || a.rowsum) ? 1 : 0;
  p.tab = a.tab;
  p.codes = a.codes;
  p.scale = a.scale;
  p.mean = a.mean;
  p.rotated = a.rotated;
  p.rowsum = a.rowsum;
  for (int i = 0; i < 15; ++i) p.thr[i] = a.thr[i];
  p.thr[15] = INFINITY;
  p.inv_norm = (float)std::pow(1.0 / std::sqrt((double)a.h), (double)a.rounds);
  p.err = device_error_word();
  if (!p.err) return fail(OQ_ERR_CUDA, "device error word unavailable");
  p.limit_ns = kWaitLimitNs;

  void* args[] = {&p};
  ce = cudaLaunchKernel(fn, dim3((unsigned)grid), dim3((unsigned)nthr), args, smem, s);
  if (ce != cudaSuccess) return cuda_fail(ce, "launch rotate_quant");
  return OQ_OK;
}

}  // namespace oq
