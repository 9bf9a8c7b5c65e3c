// Device code of the fused center + RPBH + scale + quantize kernels, shared by the standalone
// kernels (k_rotate_quant.cu) and the single-launch layer (k_linear_fused.cu). See
// k_rotate_quant.cu for the design.
#pragma once
#include <cuda_bf16.h>

#include "oq_internal.h"
#include "ptx.cuh"

namespace oq {

// Parameters of one launch of the rotate-quantize kernels (filled on the host by
// launch_rotate_quant, or by rq_pair_setup for a kernel that runs the two-token body inside).
struct RqParams {
  const uint16_t* x;   // bf16 bits
  int64_t ldx, T;
  int d, hlog2, center, mode, nbuf, want_sum, mask_smem;
  int wlayout;         // 4-bit absmax codes in the GEMM weight layout (see gemm_layout4)
  const float* thr8;   // 8-bit Lloyd-Max: 255 ascending thresholds (+ one pad), device
  int pct_r;           // percentile: order statistics needed from the top (2..6)
  float pct_frac;      // percentile: interpolation weight between ranks pct_r-1 and pct_r-2
  float pct_mult;      // percentile: gamma / Phi^-1((1 + rho) / 2)
  const uint16_t* tab;   // rounds x d entries in kernel order
  const uint4* smask;    // round-1 source signs: bit 15 / 31 of word j/2 flips channel j
  const uint4* slot;     // two-token kernel: byte offset of channel j's word, [j%8/4][j/8][j%4]
  int land_bytes;        // two-token kernel: bytes of one landing buffer
  const float4* ones;    // c' = unnormalised round-1 transform of the all-ones vector
  void* codes;
  float* scale;
  float* mean;
  float* rotated;
  float* rowsum;
  float2 cells[32];    // Lloyd-Max code cells (see lm_code)
  float inv_norm;
  unsigned long long* err;
  unsigned long long limit_ns;
};

// The two-token body's parameters for `a` without a launch: nthr threads and smem bytes of
// shared memory per unit. OQ_ERR_UNSUPPORTED if the width takes the single-token kernel.
oq_status rq_pair_setup(const RqArgs& a, RqParams& p, int& nthr, size_t& smem);

namespace {


constexpr int EP = 32;  // positions per thread



// ---- butterflies ------------------------------------------------------------------------------
// A thread's 32 values live in float2 v[16] (v[k] = elements 2k, 2k+1) so that butterflies
// whose partners sit in different pairs run as packed f32x2 operations.
// Stage over element-index bit `bit`: (a, b) -> (a + b, a - b).
template <int BIT>
__device__ __forceinline__ void stage(float2 (&v)[EP / 2]) {
  if constexpr (BIT == 0) {
#pragma unroll
    for (int k = 0; k < EP / 2; ++k) {
      const float a = v[k].x, b = v[k].y;
      v[k] = make_float2(a + b, a - b);
    }
  } else {
    constexpr int L = 1 << (BIT - 1);  // partner distance in pairs
    const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
    for (int k = 0; k < EP / 2; ++k) {
      if (!(k & L)) {
        const float2 a = v[k], b = v[k | L];
        v[k] = __fadd2_rn(a, b);
        v[k | L] = __ffma2_rn(b, m1, a);
      }
    }
  }
}

// butterfly stages over element-index bits [0, HI)
template <int HI>
__device__ __forceinline__ void reg_stages(float2 (&v)[EP / 2]) {
  if constexpr (HI > 0) stage<0>(v);
  if constexpr (HI > 1) stage<1>(v);
  if constexpr (HI > 2) stage<2>(v);
  if constexpr (HI > 3) stage<3>(v);
  if constexpr (HI > 4) stage<4>(v);
}

__device__ __forceinline__ float& el(float2 (&v)[EP / 2], int i) {
  return (i & 1) ? v[i >> 1].y : v[i >> 1].x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}
// max(a, b, c) in one instruction (three-input max.f32, sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
  return x;
}

__device__ __forceinline__ uint32_t entry(const uint32_t (&t)[EP / 2], int i) {
  return (i & 1) ? (t[i >> 1] >> 16) : (t[i >> 1] & 0xFFFFu);
}

__device__ __forceinline__ uint32_t byte_of(float f) { return __float_as_uint(f); }

// Lloyd-Max code of u = z / sigma, i.e. the number of thresholds below u. The 32 cells of width
// 1/4 over [-4, 4) hold at most one threshold each (the 16-level N(0,1) thresholds are more than
// 1/4 apart); cell j keeps (its threshold or +inf, the number of thresholds below the cell), so
// the code is that count plus one comparison. The cell index is floor(4u + 16): 4u + 15.5
// rounded to an integer by adding 2^23. The count is exact unless u lies within 2^-22 of a
// cell edge with a threshold between them, i.e. within 2^-22 of a decision boundary. Values
// outside [-4, 4) clamp to the end cells, which hold no threshold beyond their range.
__device__ __forceinline__ uint32_t lm_code(float u, const float2* cells) {
  int j = __float_as_int(fmaf(u, 4.f, 15.5f) + 8388608.f) - 0x4B000000;
  j = min(max(j, 0), 31);
  const float2 c = cells[j];
  return (uint32_t)__float_as_int(c.y) + (u > c.x ? 1u : 0u);
}

// Two's-complement bytes of a thread's 32 consecutive codes (w[k] = codes 4k..4k+3) -> one
// 16-byte group of the GEMM weight layout: byte j holds code j in its low nibble and code
// 16 + j in its high nibble.
__device__ __forceinline__ uint4 gemm_layout4(const uint32_t (&w)[8]) {
  uint32_t o[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) o[m] = (w[m] & 0x0F0F0F0Fu) | ((w[m + 4] << 4) & 0xF0F0F0F0u);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 8-bit Lloyd-Max code of u: the number of the 255 ascending thresholds strictly below u, by a
// branch-free binary search (the thresholds in shared memory; a tie goes to the lower code).
__device__ __forceinline__ uint32_t lm8_code(float u, const float* thr) {
  uint32_t lo = 0;
#pragma unroll
  for (uint32_t step = 128; step > 0; step >>= 1)
    if (thr[lo + step - 1] < u) lo += step;
  return lo;
}

// Block transform of the 32 values a thread holds, for h = 2^HLOG2 in one of three shapes.
template <int HLOG2>
__device__ __forceinline__ void block_transform(float2 (&v)[EP / 2], int lane, float* warp_tile) {
  if constexpr (HLOG2 <= 5) {
    // h <= 32: every block lies inside the thread
    reg_stages<HLOG2>(v);
  } else if constexpr (HLOG2 <= 7) {
    // h = 64 or 128: 5 stages in registers, then across 2 or 4 lanes
    reg_stages<5>(v);
#pragma unroll
    for (int m = 1; m < (1 << (HLOG2 - 5)); m <<= 1) {
      const float sg = (lane & m) ? -1.f : 1.f;
      const float2 sgn = make_float2(sg, sg);
#pragma unroll
      for (int k = 0; k < EP / 2; ++k) {
        const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, v[k].x, m),
                                     __shfl_xor_sync(0xffffffffu, v[k].y, m));
        v[k] = __ffma2_rn(v[k], sgn, o);  // lower lane: v + o; upper lane: o - v
      }
    }
  } else {
    // h = 256, 512, 1024: high bits in the strided arrangement, transpose, low bits
    constexpr int E2 = 1 << (HLOG2 - 5);
    reg_stages<HLOG2 - 5>(v);
    // Element i of lane (blk, kB) goes to row blk*E2 + ib, column kB + E2*ia of the tile,
    // stored at chunk (col/4) ^ g(row). With E2 >= 8 the chunk splits into a per-thread
    // part (kB/4 ^ G(blk)) and a per-register part ((E2/4)*ia ^ (ib & 7)), so every
    // address is a per-thread base plus one of 8 precomputed offsets and a constant.
    const int blk = lane / E2, kB = lane % E2;
    const int R = (kB >> 2) ^ ((blk * (E2 / 4)) & 7);
    float* tb = warp_tile + blk * E2 * 32 + (kB & 3);
    int off[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) off[c] = (R ^ c) << 2;
#pragma unroll
    for (int i = 0; i < EP; ++i) {
      const int ia = i / E2, ib = i % E2;
      const int ci = (((E2 / 4) * ia) ^ (ib & 7)) & 7;
      tb[ib * 32 + off[ci]] = el(v, i);
    }
    __syncwarp();
    const int g = (lane & 7) ^ (((lane / E2) * (E2 / 4)) & 7);
    const float* rb = warp_tile + lane * 32;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const float4 q = *reinterpret_cast<const float4*>(rb + ((m ^ g) << 2));
      v[2 * m] = make_float2(q.x, q.y);
      v[2 * m + 1] = make_float2(q.z, q.w);
    }
    __syncwarp();
    reg_stages<5>(v);
  }
}

template <int HLOG2, int MAXT, int ROUNDS>
__global__ void __launch_bounds__(MAXT, 1) k_rotate_quant(const RqParams p) {
  // Round-2 entries stay in registers unless a 1024-thread block would spill them.
  constexpr bool kT1Regs = (ROUNDS == 2) && (MAXT <= 256);
  extern __shared__ __align__(1024) uint8_t smem[];
  const int d = p.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int base = tid * EP;
  const bool active = base < d;
  const uint32_t row_bytes = (uint32_t)d * 2u;
  const uint32_t row_stride = (row_bytes + 127u) & ~127u;
  // With two rounds and h >= 256 the transpose tiles alias the fp32 round buffer: warp w's
  // tile is exactly the range of positions warp w writes into that buffer.
  constexpr int HMODE = HLOG2 <= 5 ? 0 : (HLOG2 <= 7 ? 1 : 2);
  constexpr bool kAlias = (ROUNDS == 2) && (HMODE == 2);
  uint8_t* rowbuf = smem;
  float* rbuf = reinterpret_cast<float*>(smem + (size_t)p.nbuf * row_stride);
  float* tbuf = kAlias ? rbuf : rbuf + (ROUNDS == 2 ? nwarps * 1024 : 0);
  float* red = tbuf + (HMODE == 2 ? nwarps * 1024 : 0);  // [0,32) sums, [32,64) statistic
  float2* cells = reinterpret_cast<float2*>(red + 64);     // 32 Lloyd-Max code cells
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 128);  // nbuf <= 3 barriers (16 floats)
  // round-1 sign masks, staged in shared memory when they fit beside the row buffers
  uint4* s_mask = reinterpret_cast<uint4*>(red + 144);
  float* warp_tile = tbuf + warp * 1024;

  uint32_t t0[EP / 2], t1[EP / 2];
#pragma unroll
  for (int i = 0; i < EP / 2; ++i) t0[i] = t1[i] = 0u;
  if (active) {
    const uint4* s0 = reinterpret_cast<const uint4*>(p.tab + base);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = __ldg(s0 + i);
      t0[4 * i] = q.x; t0[4 * i + 1] = q.y; t0[4 * i + 2] = q.z; t0[4 * i + 3] = q.w;
    }
    if constexpr (kT1Regs) {
      const uint4* s1 = reinterpret_cast<const uint4*>(p.tab + d + base);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 q = __ldg(s1 + i);
        t1[4 * i] = q.x; t1[4 * i + 1] = q.y; t1[4 * i + 2] = q.z; t1[4 * i + 3] = q.w;
      }
    }
  }
  if (tid < 32) cells[tid] = p.cells[tid];
  const uint4* mask = p.smask;
  if (p.mask_smem) {
    for (int c = tid; c < d / 8; c += blockDim.x) s_mask[c] = __ldg(p.smask + c);
    mask = s_mask;
  }
  if (tid == 0) {
    for (int b = 0; b < p.nbuf; ++b) dev::mbar_init(dev::smem_u32(&bars[b]), 1);
    dev::fence_mbar_init();
  }
  __syncthreads();

  const int64_t T = p.T;
  const int64_t G = gridDim.x;
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
    const bool take = active && !fail;

    // ---- source-side signs (and the row sum) in one coalesced pass ---------------------
    uint4* rowv = reinterpret_cast<uint4*>(rowbuf + (size_t)b * row_stride);
    const int nact = d / EP;          // threads that own positions; each takes 4 chunks
    float psum = 0.f;
    if (take) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int c = tid + m * nact;
        uint4 w = rowv[c];
        const uint4 mk = mask[c];
        if (p.want_sum) {
          psum += __uint_as_float(w.x << 16) + __uint_as_float(w.x & 0xFFFF0000u);
          psum += __uint_as_float(w.y << 16) + __uint_as_float(w.y & 0xFFFF0000u);
          psum += __uint_as_float(w.z << 16) + __uint_as_float(w.z & 0xFFFF0000u);
          psum += __uint_as_float(w.w << 16) + __uint_as_float(w.w & 0xFFFF0000u);
        }
        w.x ^= mk.x; w.y ^= mk.y; w.z ^= mk.z; w.w ^= mk.w;
        rowv[c] = w;
      }
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

    // ---- round 1: gather from the signed bf16 row ----------------------------------------
    float2 v[EP / 2];
    const uint16_t* row = reinterpret_cast<const uint16_t*>(rowbuf + (size_t)b * row_stride);
#pragma unroll
    for (int i = 0; i < EP; ++i) {
      const uint32_t ei = entry(t0, i);
      const uint32_t hb =
          active && OQ_IN_BOUNDS(ei < (uint32_t)d, p.err, kSiteBoundsRqRow) ? (uint32_t)row[ei] : 0u;
      el(v, i) = __uint_as_float(hb << 16);
    }
    float mu = 0.f;
    if (p.want_sum) {
      float sum = 0.f;
      for (int w = 0; w < nwarps; ++w) sum += red[w];
      mu = sum / (float)d;
      if (tid == 0) {
        if (p.center) p.mean[t] = mu;
        if (p.rowsum) p.rowsum[t] = sum;
      }
    }
    block_transform<HLOG2>(v, lane, warp_tile);
    if (p.center && active) {  // centered round = R(x) - mean * R(1)
      const float2 nm = make_float2(-mu, -mu);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float4 c1 = __ldg(p.ones + tid * 8 + m);
        v[2 * m] = __ffma2_rn(make_float2(c1.x, c1.y), nm, v[2 * m]);
        v[2 * m + 1] = __ffma2_rn(make_float2(c1.z, c1.w), nm, v[2 * m + 1]);
      }
    }

    // ---- round 2: through a swizzled fp32 copy in shared memory -------------------------
    if constexpr (ROUNDS == 2) {
      if (active) {
#pragma unroll
        for (int m = 0; m < 8; ++m)
          *reinterpret_cast<float4*>(&rbuf[base + ((m ^ (tid & 7)) << 2)]) =
              make_float4(v[2 * m].x, v[2 * m].y, v[2 * m + 1].x, v[2 * m + 1].y);
      }
      __syncthreads();
      if constexpr (!kT1Regs) {
        if (active) {
          const uint4* s1 = reinterpret_cast<const uint4*>(p.tab + d + base);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 q = __ldg(s1 + i);
            t1[4 * i] = q.x; t1[4 * i + 1] = q.y; t1[4 * i + 2] = q.z; t1[4 * i + 3] = q.w;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < EP; ++i) {
        const uint32_t e = entry(t1, i);
        const float g = active && OQ_IN_BOUNDS((e & 0x7FFFu) < (uint32_t)d, p.err,
                                               kSiteBoundsRqRound2)
                            ? rbuf[e & 0x7FFFu]
                            : 0.f;
        el(v, i) = __uint_as_float(__float_as_uint(g) ^ ((e & 0x8000u) << 16));
      }
      if constexpr (kAlias) __syncthreads();  // every warp is done reading the round buffer
      block_transform<HLOG2>(v, lane, warp_tile);
    }

    // ---- per-token statistic ------------------------------------------------------------
    const bool lm = p.mode == kRqLloydMax;
    float stat = 0.f;
    if (lm) {
#pragma unroll
      for (int i = 0; i < EP; ++i) stat = fmaf(el(v, i), el(v, i), stat);
    } else {
#pragma unroll
      for (int i = 0; i < EP; i += 2) stat = fmax3(stat, fabsf(el(v, i)), fabsf(el(v, i + 1)));
    }
    stat = lm ? warp_sum(stat) : warp_max(stat);
    if (lane == 0) red[32 + warp] = stat;
    __syncthreads();
    if (tid == 0) {  // every thread is past its gathers: row buffer b can be refilled
      const int64_t tn = t + (int64_t)p.nbuf * G;
      if (tn < T) {
        const uint32_t bar = dev::smem_u32(&bars[b]);
        dev::mbar_arrive_expect_tx(bar, row_bytes);
        dev::bulk_g2s(dev::smem_u32(rowbuf + (size_t)b * row_stride), p.x + tn * p.ldx,
                      row_bytes, bar);
      }
    }
    stat = 0.f;
    for (int w = 0; w < nwarps; ++w) stat = lm ? stat + red[32 + w] : fmaxf(stat, red[32 + w]);

    const float nrm = p.inv_norm;
    if (p.rotated && active) {
      float4* dst = reinterpret_cast<float4*>(p.rotated + t * (int64_t)d + base);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        dst[m] = make_float4(v[2 * m].x * nrm, v[2 * m].y * nrm, v[2 * m + 1].x * nrm,
                             v[2 * m + 1].y * nrm);
    }

    // ---- quantize + store --------------------------------------------------------------
    if (lm) {
      const float sigma = fmaxf(sqrtf(stat * nrm * nrm / (float)d), 1e-10f);
      const float mult = nrm * __frcp_rn(sigma);
      if (tid == 0) p.scale[t] = sigma;
      if (active) {
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < EP; ++i)
          packed[i >> 3] |= lm_code(el(v, i) * mult, cells) << ((i & 7) * 4);
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.codes) + t * (int64_t)(d / 2) +
                                  base / 2) = make_uint4(packed[0], packed[1], packed[2],
                                                         packed[3]);
      }
    } else {
      const float qmax = (p.mode == kRqInt8) ? 127.f : 7.f;
      const float a = fmaxf(stat * nrm, 1e-10f);
      const float mult = nrm * qmax * __frcp_rn(a);
      if (tid == 0) p.scale[t] = a / qmax;
      if (active) {
        // fma against 1.5 * 2^23 rounds half-to-even to an integer held in the low mantissa
        // bits; the low byte of each result is the two's-complement code
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 magic = make_float2(12582912.f, 12582912.f);
          const float2 mm = make_float2(mult, mult);
          const float2 r0 = __ffma2_rn(v[2 * k], mm, magic);
          const float2 r1 = __ffma2_rn(v[2 * k + 1], mm, magic);
          const uint32_t f0 = byte_of(r0.x), f1 = byte_of(r0.y);
          const uint32_t f2 = byte_of(r1.x), f3 = byte_of(r1.y);
          w[k] = __byte_perm(__byte_perm(f0, f1, 0x0040), __byte_perm(f2, f3, 0x0040), 0x5410);
        }
        if (p.mode == kRqInt8) {
          uint8_t* dst = reinterpret_cast<uint8_t*>(p.codes) + t * (int64_t)d + base;
          reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
          reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else if (p.wlayout) {
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.codes) + t * (int64_t)(d / 2) +
                                    base / 2) = gemm_layout4(w);
        } else {
          uint32_t n[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t a0 = w[2 * k] & 0x0F0F0F0Fu, a1 = w[2 * k + 1] & 0x0F0F0F0Fu;
            a0 |= a0 >> 4;   // byte 0: code0 | code1 << 4, byte 2: code2 | code3 << 4
            a1 |= a1 >> 4;
            n[k] = __byte_perm(a0, a1, 0x6420);
          }
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.codes) + t * (int64_t)(d / 2) +
                                    base / 2) = make_uint4(n[0], n[1], n[2], n[3]);
        }
      }
    }
  }

  // After an abort, wait (bounded) for row loads this CTA still has in flight so that no
  // bulk copy lands in shared memory after the block has exited.
  if (aborted && tid == 0) {
    for (int k = 0; k < p.nbuf; ++k) {
      const int j = it + k;
      const int64_t tt = (int64_t)blockIdx.x + (int64_t)j * G;
      if (tt >= T) break;
      dev::mbar_wait(dev::smem_u32(&bars[j % p.nbuf]), (uint32_t)(j / p.nbuf) & 1u, p.err,
                     kSiteRqDrain, p.limit_ns);
    }
  }
}


// ================================================================================================
// Two tokens per pass (widths up to 8192). Every value is a float2 holding the same rotated
// position of tokens A and B, so all butterflies, the centering and the rounding FMAs run as
// packed f32x2 operations, and one shared-memory gather fetches both tokens: a coalesced pass
// applies the source-side signs and interleaves the two bf16 rows into one 32-bit word per
// channel (A in the low half, B in the high half).
// ================================================================================================

// the two-token kernel's extra quantizer instantiation: 4-bit absmax codes in the GEMM layout
constexpr int kPairInt4W = 16;   // outside the RqMode values
static_assert(kPairInt4W > kRqPercentile2, "weight-layout mode must not alias a quantizer");
// the single launch's 4-bit quantizers (absmax, percentile): the same codes as kRqInt4 and
// kRqPercentile, stored one two's-complement byte per code (the INT8 layout) for its kind::i8
// split-K GEMM
constexpr int kPairInt4B = 17;
constexpr int kPairPct4B = 18;
// landing buffers of the two-token kernel (row pairs in flight per CTA)
constexpr int kPairNbuf = 1;

template <int BIT>
__device__ __forceinline__ void stage_pair(float2 (&v)[EP]) {
  constexpr int L = 1 << BIT;
  const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int k = 0; k < EP; ++k) {
    if (!(k & L)) {
      const float2 a = v[k], b = v[k | L];
      v[k] = __fadd2_rn(a, b);
      v[k | L] = __ffma2_rn(b, m1, a);
    }
  }
}

template <int HI>
__device__ __forceinline__ void reg_stages_pair(float2 (&v)[EP]) {
  if constexpr (HI > 0) stage_pair<0>(v);
  if constexpr (HI > 1) stage_pair<1>(v);
  if constexpr (HI > 2) stage_pair<2>(v);
  if constexpr (HI > 3) stage_pair<3>(v);
  if constexpr (HI > 4) stage_pair<4>(v);
}

// One component (C = 0: token A, 1: token B) of the strided -> consecutive warp transpose used
// for h >= 256 (same swizzle as the single-token kernel).
template <int HLOG2, int C>
__device__ __forceinline__ void transpose_component(float2 (&v)[EP], int lane, float* warp_tile) {
  constexpr int E2 = 1 << (HLOG2 - 5);
  const int blk = lane / E2, kB = lane % E2;
  const int R = (kB >> 2) ^ ((blk * (E2 / 4)) & 7);
  float* tb = warp_tile + blk * E2 * 32 + (kB & 3);
  int off[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) off[c] = (R ^ c) << 2;
#pragma unroll
  for (int i = 0; i < EP; ++i) {
    const int ia = i / E2, ib = i % E2;
    const int ci = (((E2 / 4) * ia) ^ (ib & 7)) & 7;
    tb[ib * 32 + off[ci]] = C ? v[i].y : v[i].x;
  }
  __syncwarp();
  const int g = (lane & 7) ^ (((lane / E2) * (E2 / 4)) & 7);
  const float* rb = warp_tile + lane * 32;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float4 q = *reinterpret_cast<const float4*>(rb + ((m ^ g) << 2));
    if (C) {
      v[4 * m].y = q.x; v[4 * m + 1].y = q.y; v[4 * m + 2].y = q.z; v[4 * m + 3].y = q.w;
    } else {
      v[4 * m].x = q.x; v[4 * m + 1].x = q.y; v[4 * m + 2].x = q.z; v[4 * m + 3].x = q.w;
    }
  }
  __syncwarp();
}

template <int HLOG2>
__device__ __forceinline__ void block_transform_pair(float2 (&v)[EP], int lane, float* warp_tile) {
  if constexpr (HLOG2 <= 5) {
    reg_stages_pair<HLOG2>(v);
  } else if constexpr (HLOG2 <= 7) {
    reg_stages_pair<5>(v);
#pragma unroll
    for (int m = 1; m < (1 << (HLOG2 - 5)); m <<= 1) {
      const float sg = (lane & m) ? -1.f : 1.f;
      const float2 sgn = make_float2(sg, sg);
#pragma unroll
      for (int k = 0; k < EP; ++k) {
        const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, v[k].x, m),
                                     __shfl_xor_sync(0xffffffffu, v[k].y, m));
        v[k] = __ffma2_rn(v[k], sgn, o);  // lower lane: v + o; upper lane: o - v
      }
    }
  } else {
    reg_stages_pair<HLOG2 - 5>(v);
    transpose_component<HLOG2, 0>(v, lane, warp_tile);
    transpose_component<HLOG2, 1>(v, lane, warp_tile);
    reg_stages_pair<5>(v);
  }
}

__device__ __forceinline__ float2 warp_sum_pair(float2 x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1)
    x = __fadd2_rn(x, make_float2(__shfl_xor_sync(0xffffffffu, x.x, m),
                                  __shfl_xor_sync(0xffffffffu, x.y, m)));
  return x;
}

// sum of the 8 bf16 values of chunk a (token A) and chunk b (token B), as a float2
__device__ __forceinline__ float2 chunk_sums(const uint4& a, const uint4& b) {
  float2 s = make_float2(0.f, 0.f);
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    s = __fadd2_rn(s, make_float2(__uint_as_float(wa[k] << 16), __uint_as_float(wb[k] << 16)));
    s = __fadd2_rn(s, make_float2(__uint_as_float(wa[k] & 0xFFFF0000u),
                                  __uint_as_float(wb[k] & 0xFFFF0000u)));
  }
  return s;
}

// a rounded value (1.5 * 2^23 + q) clipped to q in [-QM, QM] (exact: integers in this range)
template <int QM>
__device__ __forceinline__ float2 clamp_code(float2 r) {
  constexpr float lo = 12582912.f - QM, hi = 12582912.f + QM;
  return make_float2(fminf(fmaxf(r.x, lo), hi), fminf(fmaxf(r.y, lo), hi));
}

// low byte of every float of four rounded values, as one word
__device__ __forceinline__ uint32_t pack4(float a, float b, float c, float e) {
  return __byte_perm(__byte_perm(byte_of(a), byte_of(b), 0x0040),
                     __byte_perm(byte_of(c), byte_of(e), 0x0040), 0x5410);
}

// two's-complement bytes of 8 codes -> 8 nibbles (element 2j in the low nibble of byte j)
__device__ __forceinline__ uint32_t nibbles8(uint32_t w0, uint32_t w1) {
  uint32_t a0 = w0 & 0x0F0F0F0Fu, a1 = w1 & 0x0F0F0F0Fu;
  a0 |= a0 >> 4;
  a1 |= a1 >> 4;
  return __byte_perm(a0, a1, 0x6420);
}

// two's-complement bytes of 16 codes in -2..1 (four words, element 4k + i in byte i of word k)
// -> 16 two-bit fields, element e in bits 2e, 2e + 1
__device__ __forceinline__ uint32_t pairs16(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  uint32_t a[4] = {w0 & 0x03030303u, w1 & 0x03030303u, w2 & 0x03030303u, w3 & 0x03030303u};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    a[k] |= a[k] >> 6;    // byte 0: fields 0, 1; byte 2: fields 2, 3 (in its low nibble)
    a[k] |= a[k] >> 12;   // byte 0: fields 0-3
  }
  return __byte_perm(__byte_perm(a[0], a[1], 0x0040), __byte_perm(a[2], a[3], 0x0040), 0x5410);
}

// ---- percentile scale (CentriQ §4.2 "Scale and grid", App. B.3) ---------------------------
// The rho-quantile of |z| over the d positions, linear between the order statistics around
// position rho (d - 1), needs the R = d - floor(rho (d - 1)) largest magnitudes (R <= 6 for
// d <= 8192). Every thread keeps the R largest of its values in a descending list (one max/min
// insertion per value), the warp merges its lanes' lists by R rounds of max extraction, and
// every warp merges the warps' lists (through shared memory) the same way.

// insert x into the descending list m, keeping the R largest (a multiset: ties are kept)
template <int R>
__device__ __forceinline__ void topr_insert(float (&m)[R], float x) {
#pragma unroll
  for (int k = 0; k < R; ++k) {
    const float hi = fmaxf(m[k], x);
    x = fminf(m[k], x);
    m[k] = hi;
  }
}

// the R largest of the union of the lanes' descending lists, in every lane (out descending)
template <int R>
__device__ __forceinline__ void warp_topr(float (&m)[R], int lane, float (&out)[R]) {
#pragma unroll
  for (int k = 0; k < R; ++k) {
    const float top = warp_max(m[0]);
    const unsigned who = __ballot_sync(0xffffffffu, m[0] == top);
    const bool pop = lane == __ffs(who) - 1;   // exactly one lane gives up its head
#pragma unroll
    for (int j = 0; j < R - 1; ++j) m[j] = pop ? m[j + 1] : m[j];
    m[R - 1] = pop ? -1.f : m[R - 1];
    out[k] = top;
  }
}

// Phase 1 of the two tokens' percentile statistic: the warp's R largest |v| of token A (x) and
// token B (y), written to lists[warp][token][0..R) in shared memory.
template <int R>
__device__ __forceinline__ void pct_warp_lists(const float2 (&v)[EP], bool active, int lane,
                                               int warp, float* lists) {
  float ma[R], mb[R];
#pragma unroll
  for (int k = 0; k < R; ++k) ma[k] = mb[k] = -1.f;
  if (active) {
#pragma unroll
    for (int i = 0; i < EP; ++i) {
      topr_insert<R>(ma, fabsf(v[i].x));
      topr_insert<R>(mb, fabsf(v[i].y));
    }
  }
  float oa[R], ob[R];
  warp_topr<R>(ma, lane, oa);
  warp_topr<R>(mb, lane, ob);
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < R; ++k) {
      lists[(2 * warp) * R + k] = oa[k];
      lists[(2 * warp + 1) * R + k] = ob[k];
    }
  }
}

// Phase 2 (after a block barrier): the interpolated quantile of both tokens from every warp's
// lists; every warp computes the same result.
template <int R>
__device__ __forceinline__ float2 pct_quantiles(const float* lists, int nwarps, int lane,
                                                float frac) {
  float ma[R], mb[R];
#pragma unroll
  for (int k = 0; k < R; ++k) ma[k] = mb[k] = -1.f;
  // lane l takes list entries l and l + 32 of each token (nwarps * R <= 48)
#pragma unroll
  for (int rep = 0; rep < 2; ++rep) {
    const int e = lane + 32 * rep;
    if (e < nwarps * R) {
      const int w = e / R, k = e % R;
      topr_insert<R>(ma, lists[(2 * w) * R + k]);
      topr_insert<R>(mb, lists[(2 * w + 1) * R + k]);
    }
  }
  float oa[R], ob[R];
  warp_topr<R>(ma, lane, oa);
  warp_topr<R>(mb, lane, ob);
  // order statistic floor(pos) is rank R-1 from the top, floor(pos) + 1 is rank R-2
  return make_float2(fmaf(frac, oa[R - 2] - oa[R - 1], oa[R - 1]),
                     fmaf(frac, ob[R - 2] - ob[R - 1], ob[R - 1]));
}

// MODE: the quantizer (RqMode), or kPairInt4W for 4-bit absmax codes in the GEMM weight layout.
// One instantiation per quantizer keeps each kernel's code small.
// The kernel's body runs on threads 0 .. nthr - 1 of a block (the whole block when launched on
// its own, the first warps of the single-launch layer's CTAs), as unit `cta` of `ncta` over the
// token pairs, in the shared memory at `smem` (1024-byte aligned). Its block-wide barriers are
// the named barrier kRqBarrier over those nthr threads. With release_barriers the body ends by
// invalidating its mbarriers, so that the caller may reuse the shared memory.
constexpr uint32_t kRqBarrier = 1;

__device__ __forceinline__ int rq_sync_or(int pred, int nthr) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred), "r"(kRqBarrier), "r"(nthr)
      : "memory");
  return (int)r;
}

template <int HLOG2, int ROUNDS, int MODE>
__device__ __forceinline__ void rq_pair_body(const RqParams& p, uint8_t* smem, int cta, int ncta,
                                             int nthr, bool release_barriers) {
  const int d = p.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nthr >> 5;
  const int base = tid * EP;
  const int nact = d / EP;  // threads that own positions
  const bool active = tid < nact;
  const uint32_t row_bytes = (uint32_t)d * 2u;
  const uint32_t row_stride = (row_bytes + 127u) & ~127u;
  const size_t land_bytes = (size_t)p.land_bytes;
  // [kPairNbuf landing buffers: a pair of rows (A | B) each; while a pass runs, its own buffer also
  //  holds the warps' transpose tiles (h >= 256), so no barrier separates a warp's gather from
  //  its transposes] [interleaved words, bank-aware layout: nwarps x 4 KB]
  // [round buffer, two rounds only] [reductions, code cells, barriers, percentile lists,
  //  8-bit Lloyd-Max thresholds]
  uint8_t* land = smem;
  uint8_t* wbuf = smem + kPairNbuf * land_bytes;
  float2* rbuf = reinterpret_cast<float2*>(wbuf + nwarps * 4096);
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(rbuf) +
                                        (ROUNDS == 2 ? nwarps * 8192 : 0));
  // red: [0,16) sums, [16,32) statistic; then 32 Lloyd-Max code cells and the barriers
  float2* cells = reinterpret_cast<float2*>(red + 32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 96);
  float* pct_lists = red + 128;   // percentile: up to 8 warps x 2 tokens x 6 ranks
  float* s_thr8 = red + 224;      // 8-bit Lloyd-Max thresholds

  if (tid < 32) cells[tid] = p.cells[tid];
  if constexpr (MODE == kRqLloydMax8)
    for (int k = tid; k < 256; k += nthr) s_thr8[k] = __ldg(p.thr8 + k);
  if (tid == 0) {
    for (int b = 0; b < kPairNbuf; ++b) dev::mbar_init(dev::smem_u32(&bars[b]), 1);
    dev::fence_mbar_init();
  }
  dev::named_bar(kRqBarrier, nthr);

  const int64_t T = p.T;
  const int64_t NP = (T + 1) / 2;  // token pairs; an odd tail loads its one row twice
  const int64_t G = ncta;
  auto issue = [&](int b, int64_t q) {
    const int64_t ta = 2 * q, tb = (2 * q + 1 < T) ? 2 * q + 1 : 2 * q;
    const uint32_t bar = dev::smem_u32(&bars[b]);
    uint8_t* dst = land + (size_t)b * land_bytes;
    dev::mbar_arrive_expect_tx(bar, 2u * row_bytes);
    dev::bulk_g2s(dev::smem_u32(dst), p.x + ta * p.ldx, row_bytes, bar);
    dev::bulk_g2s(dev::smem_u32(dst + row_stride), p.x + tb * p.ldx, row_bytes, bar);
  };
  if (tid == 0)
    for (int b = 0; b < kPairNbuf; ++b)
      if ((int64_t)cta + (int64_t)b * G < NP) issue(b, (int64_t)cta + (int64_t)b * G);

  constexpr bool lm8 = MODE == kRqLloydMax8;
  constexpr bool lm = MODE == kRqLloydMax || lm8;   // RMS scale
  const float nrm = p.inv_norm;
  int it = 0;
  bool aborted = false;
  for (int64_t q = cta; q < NP; q += G, ++it) {
    const int b = it % kPairNbuf;
    uint8_t* lb = land + (size_t)b * land_bytes;
    float* warp_tile = reinterpret_cast<float*>(lb) + warp * 1024;
    const int64_t ta = 2 * q;
    const bool has_b = ta + 1 < T;
    // round-1 gather entries (byte offsets into the word buffer), L1-resident; loaded before
    // the wait so that their latency overlaps it
    uint32_t t0[EP / 2];
#pragma unroll
    for (int i = 0; i < EP / 2; ++i) t0[i] = 0u;
    if (active) {
      const uint4* s0 = reinterpret_cast<const uint4*>(p.tab + base);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(s0 + i);
        t0[4 * i] = w.x; t0[4 * i + 1] = w.y; t0[4 * i + 2] = w.z; t0[4 * i + 3] = w.w;
      }
    }
    // the interleave's sign masks and word offsets (L1-resident), also before the wait
    uint4 mks[4], sl0[4], sl1[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int c = active ? tid + m * nact : 0;
      mks[m] = __ldg(p.smask + c);
      sl0[m] = __ldg(p.slot + c);
      sl1[m] = __ldg(p.slot + d / 8 + c);
    }
    int fail = !dev::mbar_wait(dev::smem_u32(&bars[b]), (uint32_t)(it / kPairNbuf) & 1u, p.err,
                               kSiteRqRow, p.limit_ns);

    // ---- source-side signs, interleave A|B into the bank-aware word layout, row sums ------
    // Channel 8c + k of both tokens becomes one word (A low, B high) at the byte offset the
    // plan's slot table gives: the eight stores of a chunk, and the round-1 gathers below,
    // each touch 32 distinct banks across the warp.
    float2 psum = make_float2(0.f, 0.f);
    if (active && !fail) {
      const uint4* ra = reinterpret_cast<const uint4*>(lb);
      const uint4* rb = reinterpret_cast<const uint4*>(lb + row_stride);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int c = tid + m * nact;
        uint4 a = ra[c], bb = rb[c];
        const uint4 mk = mks[m], s0 = sl0[m], s1 = sl1[m];
        if (p.want_sum) psum = __fadd2_rn(psum, chunk_sums(a, bb));
        a.x ^= mk.x; a.y ^= mk.y; a.z ^= mk.z; a.w ^= mk.w;
        bb.x ^= mk.x; bb.y ^= mk.y; bb.z ^= mk.z; bb.w ^= mk.w;
#ifdef OQ_CHECKED
        {
          const uint32_t lim = (uint32_t)(nwarps * 4096 - 4);
          const uint32_t offs[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
          const uint32_t vals[8] = {__byte_perm(a.x, bb.x, 0x5410), __byte_perm(a.x, bb.x, 0x7632),
                                    __byte_perm(a.y, bb.y, 0x5410), __byte_perm(a.y, bb.y, 0x7632),
                                    __byte_perm(a.z, bb.z, 0x5410), __byte_perm(a.z, bb.z, 0x7632),
                                    __byte_perm(a.w, bb.w, 0x5410), __byte_perm(a.w, bb.w, 0x7632)};
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (OQ_IN_BOUNDS(offs[k] <= lim && (offs[k] & 3u) == 0u, p.err, kSiteBoundsPairSlot))
              *reinterpret_cast<uint32_t*>(wbuf + offs[k]) = vals[k];
        }
#else
        *reinterpret_cast<uint32_t*>(wbuf + s0.x) = __byte_perm(a.x, bb.x, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s0.y) = __byte_perm(a.x, bb.x, 0x7632);
        *reinterpret_cast<uint32_t*>(wbuf + s0.z) = __byte_perm(a.y, bb.y, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s0.w) = __byte_perm(a.y, bb.y, 0x7632);
        *reinterpret_cast<uint32_t*>(wbuf + s1.x) = __byte_perm(a.z, bb.z, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s1.y) = __byte_perm(a.z, bb.z, 0x7632);
        *reinterpret_cast<uint32_t*>(wbuf + s1.z) = __byte_perm(a.w, bb.w, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s1.w) = __byte_perm(a.w, bb.w, 0x7632);
#endif
      }
    }
    if (p.want_sum) {
      psum = warp_sum_pair(psum);
      if (lane == 0) { red[2 * warp] = psum.x; red[2 * warp + 1] = psum.y; }
    }
    fail = rq_sync_or(fail, nthr);
    if (fail) {
      aborted = true;
      break;
    }

    // ---- round 1: one gather for both tokens ---------------------------------------------
    float2 v[EP];
#pragma unroll
    for (int i = 0; i < EP; ++i) {
      const uint32_t ei = entry(t0, i);
      const uint32_t w =
          active && OQ_IN_BOUNDS(ei <= (uint32_t)(nwarps * 4096 - 4) && (ei & 3u) == 0u, p.err,
                                 kSiteBoundsPairGather)
              ? *reinterpret_cast<const uint32_t*>(wbuf + ei)
              : 0u;
      v[i] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
    float2 mu = make_float2(0.f, 0.f);
    if (p.want_sum) {
      float2 sum = make_float2(0.f, 0.f);
      for (int w = 0; w < nwarps; ++w) sum = __fadd2_rn(sum, make_float2(red[2 * w], red[2 * w + 1]));
      mu = make_float2(sum.x / (float)d, sum.y / (float)d);
      if (tid == 0) {
        if (p.center) { p.mean[ta] = mu.x; if (has_b) p.mean[ta + 1] = mu.y; }
        if (p.rowsum) { p.rowsum[ta] = sum.x; if (has_b) p.rowsum[ta + 1] = sum.y; }
      }
    }
    block_transform_pair<HLOG2>(v, lane, warp_tile);
    if (p.center && active) {  // centered round = R(x) - mean * R(1)
      const float2 nm = make_float2(-mu.x, -mu.y);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float4 c1 = __ldg(p.ones + tid * 8 + m);
        v[4 * m] = __ffma2_rn(make_float2(c1.x, c1.x), nm, v[4 * m]);
        v[4 * m + 1] = __ffma2_rn(make_float2(c1.y, c1.y), nm, v[4 * m + 1]);
        v[4 * m + 2] = __ffma2_rn(make_float2(c1.z, c1.z), nm, v[4 * m + 2]);
        v[4 * m + 3] = __ffma2_rn(make_float2(c1.w, c1.w), nm, v[4 * m + 3]);
      }
    }

    // ---- round 2: gather float2 pairs from the swizzled round buffer ----------------------
    if constexpr (ROUNDS == 2) {
      if (active) {
        float4* rv = reinterpret_cast<float4*>(rbuf) + tid * 16;
#pragma unroll
        for (int k = 0; k < 16; ++k)
          rv[k ^ (tid & 7)] = make_float4(v[2 * k].x, v[2 * k].y, v[2 * k + 1].x, v[2 * k + 1].y);
      }
      uint32_t t1[EP / 2];
#pragma unroll
      for (int i = 0; i < EP / 2; ++i) t1[i] = 0u;
      if (active) {
        const uint4* s1 = reinterpret_cast<const uint4*>(p.tab + d + base);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 w = __ldg(s1 + i);
          t1[4 * i] = w.x; t1[4 * i + 1] = w.y; t1[4 * i + 2] = w.z; t1[4 * i + 3] = w.w;
        }
      }
      dev::named_bar(kRqBarrier, nthr);
#pragma unroll
      for (int i = 0; i < EP; ++i) {
        const uint32_t e = entry(t1, i);
        const float2 g = active && OQ_IN_BOUNDS((e & 0x7FFFu) < (uint32_t)d, p.err,
                                                kSiteBoundsRqRound2)
                             ? rbuf[e & 0x7FFFu]
                             : make_float2(0.f, 0.f);
        const uint32_t sb = (e & 0x8000u) << 16;
        v[i] = make_float2(__uint_as_float(__float_as_uint(g.x) ^ sb),
                           __uint_as_float(__float_as_uint(g.y) ^ sb));
      }
      block_transform_pair<HLOG2>(v, lane, warp_tile);
    }

    // ---- per-token statistics --------------------------------------------------------------
    float2 st = make_float2(0.f, 0.f);
    constexpr bool pct = MODE == kRqPercentile || MODE == kRqPercentile2 || MODE == kPairPct4B;
    if constexpr (pct) {
      switch (p.pct_r) {
        case 2: pct_warp_lists<2>(v, active, lane, warp, pct_lists); break;
        case 3: pct_warp_lists<3>(v, active, lane, warp, pct_lists); break;
        case 4: pct_warp_lists<4>(v, active, lane, warp, pct_lists); break;
        case 5: pct_warp_lists<5>(v, active, lane, warp, pct_lists); break;
        default: pct_warp_lists<6>(v, active, lane, warp, pct_lists); break;
      }
    } else if constexpr (lm) {
#pragma unroll
      for (int i = 0; i < EP; ++i) st = __ffma2_rn(v[i], v[i], st);
      st = warp_sum_pair(st);
    } else {
#pragma unroll
      for (int i = 0; i < EP; i += 2) {
        st.x = fmax3(st.x, fabsf(v[i].x), fabsf(v[i + 1].x));
        st.y = fmax3(st.y, fabsf(v[i].y), fabsf(v[i + 1].y));
      }
      st.x = warp_max(st.x);
      st.y = warp_max(st.y);
    }
    if (lane == 0 && !pct) { red[16 + 2 * warp] = st.x; red[16 + 2 * warp + 1] = st.y; }
    dev::named_bar(kRqBarrier, nthr);
    // every thread is past its reads of landing buffer b (rows and transpose tiles): refill it
    if (tid == 0 && q + kPairNbuf * G < NP) issue(b, q + kPairNbuf * G);
    st = make_float2(0.f, 0.f);
    if constexpr (pct) {
      switch (p.pct_r) {
        case 2: st = pct_quantiles<2>(pct_lists, nwarps, lane, p.pct_frac); break;
        case 3: st = pct_quantiles<3>(pct_lists, nwarps, lane, p.pct_frac); break;
        case 4: st = pct_quantiles<4>(pct_lists, nwarps, lane, p.pct_frac); break;
        case 5: st = pct_quantiles<5>(pct_lists, nwarps, lane, p.pct_frac); break;
        default: st = pct_quantiles<6>(pct_lists, nwarps, lane, p.pct_frac); break;
      }
    } else {
      for (int w = 0; w < nwarps; ++w) {
        const float sa = red[16 + 2 * w], sb = red[16 + 2 * w + 1];
        st = lm ? make_float2(st.x + sa, st.y + sb) : make_float2(fmaxf(st.x, sa), fmaxf(st.y, sb));
      }
    }

    if (p.rotated && active) {
#pragma unroll
      for (int tk = 0; tk < 2; ++tk) {
        if (tk == 1 && !has_b) break;
        float4* dst = reinterpret_cast<float4*>(p.rotated + (ta + tk) * (int64_t)d + base);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float2 a0 = v[4 * m], a1 = v[4 * m + 1], a2 = v[4 * m + 2], a3 = v[4 * m + 3];
          dst[m] = tk ? make_float4(a0.y * nrm, a1.y * nrm, a2.y * nrm, a3.y * nrm)
                      : make_float4(a0.x * nrm, a1.x * nrm, a2.x * nrm, a3.x * nrm);
        }
      }
    }

    // ---- quantize + store ------------------------------------------------------------------
    uint8_t* codes = reinterpret_cast<uint8_t*>(p.codes);
    if constexpr (lm) {
      const float sa = fmaxf(sqrtf(st.x * nrm * nrm / (float)d), 1e-10f);
      const float sb = fmaxf(sqrtf(st.y * nrm * nrm / (float)d), 1e-10f);
      const float2 mult = make_float2(nrm * __frcp_rn(sa), nrm * __frcp_rn(sb));
      if (tid == 0) { p.scale[ta] = sa; if (has_b) p.scale[ta + 1] = sb; }
      if (lm8 && active) {
        // 8-bit codes: the number of the 255 thresholds below u, by binary search in shared
        // memory; one byte per code, 32 consecutive codes per thread and token
        uint32_t wa[8], wb[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint32_t ca[4], cb[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 u = __fmul2_rn(v[4 * k + e], mult);
            ca[e] = lm8_code(u.x, s_thr8);
            cb[e] = lm8_code(u.y, s_thr8);
          }
          wa[k] = ca[0] | (ca[1] << 8) | (ca[2] << 16) | (ca[3] << 24);
          wb[k] = cb[0] | (cb[1] << 8) | (cb[2] << 16) | (cb[3] << 24);
        }
        uint4* da = reinterpret_cast<uint4*>(codes + ta * (int64_t)d + base);
        da[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
        da[1] = make_uint4(wa[4], wa[5], wa[6], wa[7]);
        if (has_b) {
          uint4* db = reinterpret_cast<uint4*>(codes + (ta + 1) * (int64_t)d + base);
          db[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
          db[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
        }
      } else if (active) {
        uint32_t pa[4] = {0u, 0u, 0u, 0u}, pb[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < EP; ++i) {
          const float2 u = __fmul2_rn(v[i], mult);
          pa[i >> 3] |= lm_code(u.x, cells) << ((i & 7) * 4);
          pb[i >> 3] |= lm_code(u.y, cells) << ((i & 7) * 4);
        }
        *reinterpret_cast<uint4*>(codes + ta * (int64_t)(d / 2) + base / 2) =
            make_uint4(pa[0], pa[1], pa[2], pa[3]);
        if (has_b)
          *reinterpret_cast<uint4*>(codes + (ta + 1) * (int64_t)(d / 2) + base / 2) =
              make_uint4(pb[0], pb[1], pb[2], pb[3]);
      }
    } else {
      constexpr float qmax = (MODE == kRqInt8) ? 127.f : (MODE == kRqPercentile2 ? 1.f : 7.f);
      // range: absmax, or gamma * sigma_hat for the percentile scale (its quantile times
      // gamma / Phi^-1((1 + rho) / 2)); both floored at eps
      const float rs = pct ? p.pct_mult : 1.f;
      const float aa = fmaxf(st.x * nrm * rs, 1e-10f), ab = fmaxf(st.y * nrm * rs, 1e-10f);
      const float2 mult = make_float2(nrm * qmax * __frcp_rn(aa), nrm * qmax * __frcp_rn(ab));
      if (tid == 0) { p.scale[ta] = aa / qmax; if (has_b) p.scale[ta + 1] = ab / qmax; }
      if (active) {
        // fma against 1.5 * 2^23 rounds half-to-even to an integer held in the low mantissa
        // bits; the low byte of each result is the two's-complement code. The percentile range
        // can leave values past +-qmax: clamping the rounded value to magic +- qmax clips them
        const float2 magic = make_float2(12582912.f, 12582912.f);
        uint32_t wa[8], wb[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float2 r0 = __ffma2_rn(v[4 * k], mult, magic);
          float2 r1 = __ffma2_rn(v[4 * k + 1], mult, magic);
          float2 r2 = __ffma2_rn(v[4 * k + 2], mult, magic);
          float2 r3 = __ffma2_rn(v[4 * k + 3], mult, magic);
          if constexpr (pct) {
            constexpr int qm = MODE == kRqPercentile2 ? 1 : 7;
            r0 = clamp_code<qm>(r0); r1 = clamp_code<qm>(r1);
            r2 = clamp_code<qm>(r2); r3 = clamp_code<qm>(r3);
          }
          wa[k] = pack4(r0.x, r1.x, r2.x, r3.x);
          wb[k] = pack4(r0.y, r1.y, r2.y, r3.y);
        }
        if constexpr (MODE == kRqInt8 || MODE == kPairInt4B || MODE == kPairPct4B) {
          uint4* da = reinterpret_cast<uint4*>(codes + ta * (int64_t)d + base);
          da[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
          da[1] = make_uint4(wa[4], wa[5], wa[6], wa[7]);
          if (has_b) {
            uint4* db = reinterpret_cast<uint4*>(codes + (ta + 1) * (int64_t)d + base);
            db[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
            db[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
          }
        } else if constexpr (MODE == kRqPercentile2) {
          *reinterpret_cast<uint2*>(codes + ta * (int64_t)(d / 4) + base / 4) =
              make_uint2(pairs16(wa[0], wa[1], wa[2], wa[3]), pairs16(wa[4], wa[5], wa[6], wa[7]));
          if (has_b)
            *reinterpret_cast<uint2*>(codes + (ta + 1) * (int64_t)(d / 4) + base / 4) =
                make_uint2(pairs16(wb[0], wb[1], wb[2], wb[3]),
                           pairs16(wb[4], wb[5], wb[6], wb[7]));
        } else if constexpr (MODE == kPairInt4W) {
          *reinterpret_cast<uint4*>(codes + ta * (int64_t)(d / 2) + base / 2) = gemm_layout4(wa);
          if (has_b)
            *reinterpret_cast<uint4*>(codes + (ta + 1) * (int64_t)(d / 2) + base / 2) =
                gemm_layout4(wb);
        } else {
          *reinterpret_cast<uint4*>(codes + ta * (int64_t)(d / 2) + base / 2) =
              make_uint4(nibbles8(wa[0], wa[1]), nibbles8(wa[2], wa[3]), nibbles8(wa[4], wa[5]),
                         nibbles8(wa[6], wa[7]));
          if (has_b)
            *reinterpret_cast<uint4*>(codes + (ta + 1) * (int64_t)(d / 2) + base / 2) =
                make_uint4(nibbles8(wb[0], wb[1]), nibbles8(wb[2], wb[3]), nibbles8(wb[4], wb[5]),
                           nibbles8(wb[6], wb[7]));
        }
      }
    }
  }

  // After an abort, wait (bounded) for the row loads this CTA still has in flight, so that no
  // bulk copy lands in shared memory after the block has exited.
  if (aborted && tid == 0) {
    for (int k = 0; k < kPairNbuf; ++k) {
      const int j = it + k;
      if ((int64_t)cta + (int64_t)j * G >= NP) break;
      dev::mbar_wait(dev::smem_u32(&bars[j % kPairNbuf]), (uint32_t)(j / kPairNbuf) & 1u, p.err,
                     kSiteRqDrain, p.limit_ns);
    }
  }
  if (release_barriers) {
    dev::named_bar(kRqBarrier, nthr);   // every wait on the barriers has returned
    if (tid == 0)
      for (int b = 0; b < kPairNbuf; ++b) dev::mbar_inval(dev::smem_u32(&bars[b]));
  }
}

template <int HLOG2, int ROUNDS, int MODE>
__global__ void __launch_bounds__(256, 2) k_rotate_quant_pair(const RqParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  rq_pair_body<HLOG2, ROUNDS, MODE>(p, smem, (int)blockIdx.x, (int)gridDim.x, (int)blockDim.x,
                                    false);
}

}  // namespace
}  // namespace oq
