// Fused per-token center + RPBH rotation + scale + quantize (the activation path of CentriQ
// §4.2 and App. B.2; OrbitQuant PR #25 "Runtime work": the pre-rotation as one kernel).
//
// HBM-bound design; persistent CTAs of d/32 threads, every thread owning 32 rotated positions
// per round. Two kernel shapes share the building blocks below:
//  - k_rotate_quant_pair (d <= 8192): one pass handles two tokens. A 1-D bulk copy (TMA) lands
//    both bf16 rows in shared memory; one coalesced 16-byte pass applies the round-1 signs on
//    the source side (channel j takes the sign of the rotated position that gathers it) and
//    interleaves the rows into one 32-bit word per channel, so that one random gather per
//    position serves both tokens. Every value is then a float2 (token A, token B) and all
//    butterflies, the centering FMA and the rounding FMA run as packed f32x2 operations.
//  - k_rotate_quant (wider rows, up to 1024 threads): the same steps one token at a time, the
//    row streaming 1-3 rows ahead and the signs applied in place.
// Common steps:
//  - Gather entries (where the staged row keeps the source of each position) are laid out on
//    the host in the order the threads consume them.
//  - Block transform of size h = 2^L in three shapes:
//      h <= 32        the thread holds whole blocks: L register butterfly stages;
//      h = 64, 128    the thread holds 32 consecutive positions: 5 register stages, then
//                     1-2 stages across lanes by shuffles;
//      h >= 256       the gather fills a strided arrangement (the thread holds one column of
//                     a 32 x (h/32) view of its block), the high bits are transformed in
//                     registers, one swizzled, bank-conflict-free shared-memory transpose per
//                     warp (per token) brings 32 consecutive positions to each thread, and
//                     the low 5 bits are transformed in registers.
//  - A second round gathers from an fp32 copy of the first round's output, written in a
//    swizzled layout whose indices the host folded into the round-2 entries.
//  - Centering: the interleave / sign pass sums the row; since a round is linear, the centered
//    first round is R(x) - mean * R(1), with R(1) (unnormalised) a per-plan constant vector.
//  - Per-token absmax (or sum of squares for Lloyd-Max) by shuffles and one block reduction;
//    absmax codes are rounded with one FMA against 1.5 * 2^23 and packed with byte permutes
//    into 16-byte stores; Lloyd-Max codes come from a 32-cell table (lm_code).
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "oq_internal.h"
#include "ptx.cuh"

namespace oq {
namespace {

constexpr int EP = 32;  // positions per thread

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
      const uint32_t hb = active ? (uint32_t)row[entry(t0, i)] : 0u;
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
        const float g = active ? rbuf[e & 0x7FFFu] : 0.f;
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
constexpr int kPairInt4W = 5;
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

// a rounded value (1.5 * 2^23 + q) clipped to q in [-7, 7] (exact: integers in this range)
__device__ __forceinline__ float2 clamp_code(float2 r) {
  return make_float2(fminf(fmaxf(r.x, 12582905.f), 12582919.f),
                     fminf(fmaxf(r.y, 12582905.f), 12582919.f));
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
template <int HLOG2, int ROUNDS, int MODE>
__global__ void __launch_bounds__(256, 2) k_rotate_quant_pair(const RqParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int d = p.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
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
    for (int k = tid; k < 256; k += blockDim.x) s_thr8[k] = __ldg(p.thr8 + k);
  if (tid == 0) {
    for (int b = 0; b < kPairNbuf; ++b) dev::mbar_init(dev::smem_u32(&bars[b]), 1);
    dev::fence_mbar_init();
  }
  __syncthreads();

  const int64_t T = p.T;
  const int64_t NP = (T + 1) / 2;  // token pairs; an odd tail loads its one row twice
  const int64_t G = gridDim.x;
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
      if ((int64_t)blockIdx.x + (int64_t)b * G < NP) issue(b, (int64_t)blockIdx.x + (int64_t)b * G);

  constexpr bool lm8 = MODE == kRqLloydMax8;
  constexpr bool lm = MODE == kRqLloydMax || lm8;   // RMS scale
  const float nrm = p.inv_norm;
  int it = 0;
  bool aborted = false;
  for (int64_t q = blockIdx.x; q < NP; q += G, ++it) {
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
        *reinterpret_cast<uint32_t*>(wbuf + s0.x) = __byte_perm(a.x, bb.x, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s0.y) = __byte_perm(a.x, bb.x, 0x7632);
        *reinterpret_cast<uint32_t*>(wbuf + s0.z) = __byte_perm(a.y, bb.y, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s0.w) = __byte_perm(a.y, bb.y, 0x7632);
        *reinterpret_cast<uint32_t*>(wbuf + s1.x) = __byte_perm(a.z, bb.z, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s1.y) = __byte_perm(a.z, bb.z, 0x7632);
        *reinterpret_cast<uint32_t*>(wbuf + s1.z) = __byte_perm(a.w, bb.w, 0x5410);
        *reinterpret_cast<uint32_t*>(wbuf + s1.w) = __byte_perm(a.w, bb.w, 0x7632);
      }
    }
    if (p.want_sum) {
      psum = warp_sum_pair(psum);
      if (lane == 0) { red[2 * warp] = psum.x; red[2 * warp + 1] = psum.y; }
    }
    fail = __syncthreads_or(fail);
    if (fail) {
      aborted = true;
      break;
    }

    // ---- round 1: one gather for both tokens ---------------------------------------------
    float2 v[EP];
#pragma unroll
    for (int i = 0; i < EP; ++i) {
      const uint32_t w = active ? *reinterpret_cast<const uint32_t*>(wbuf + entry(t0, i)) : 0u;
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
      __syncthreads();
#pragma unroll
      for (int i = 0; i < EP; ++i) {
        const uint32_t e = entry(t1, i);
        const float2 g = active ? rbuf[e & 0x7FFFu] : make_float2(0.f, 0.f);
        const uint32_t sb = (e & 0x8000u) << 16;
        v[i] = make_float2(__uint_as_float(__float_as_uint(g.x) ^ sb),
                           __uint_as_float(__float_as_uint(g.y) ^ sb));
      }
      block_transform_pair<HLOG2>(v, lane, warp_tile);
    }

    // ---- per-token statistics --------------------------------------------------------------
    float2 st = make_float2(0.f, 0.f);
    constexpr bool pct = MODE == kRqPercentile;
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
    __syncthreads();
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
      constexpr float qmax = (MODE == kRqInt8) ? 127.f : 7.f;
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
            r0 = clamp_code(r0); r1 = clamp_code(r1); r2 = clamp_code(r2); r3 = clamp_code(r3);
          }
          wa[k] = pack4(r0.x, r1.x, r2.x, r3.x);
          wb[k] = pack4(r0.y, r1.y, r2.y, r3.y);
        }
        if constexpr (MODE == kRqInt8) {
          uint4* da = reinterpret_cast<uint4*>(codes + ta * (int64_t)d + base);
          da[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
          da[1] = make_uint4(wa[4], wa[5], wa[6], wa[7]);
          if (has_b) {
            uint4* db = reinterpret_cast<uint4*>(codes + (ta + 1) * (int64_t)d + base);
            db[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
            db[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
          }
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
      if ((int64_t)blockIdx.x + (int64_t)j * G >= NP) break;
      dev::mbar_wait(dev::smem_u32(&bars[j % kPairNbuf]), (uint32_t)(j / kPairNbuf) & 1u, p.err,
                     kSiteRqDrain, p.limit_ns);
    }
  }
}

struct LaunchCfg {
  void* fn = nullptr;
  int nthr = 0, nbuf = 0, grid_per_sm = 0, mask_smem = 0, pair = 0, land_bytes = 0;
  size_t smem = 0;
};

template <int HL, int MAXT, int R>
void* kern() {
  return reinterpret_cast<void*>(&k_rotate_quant<HL, MAXT, R>);
}

template <int MAXT, int R>
void* kern_h(int hlog2) {
  switch (hlog2) {
    case 0: return kern<0, MAXT, R>();
    case 1: return kern<1, MAXT, R>();
    case 2: return kern<2, MAXT, R>();
    case 3: return kern<3, MAXT, R>();
    case 4: return kern<4, MAXT, R>();
    case 5: return kern<5, MAXT, R>();
    case 6: return kern<6, MAXT, R>();
    case 7: return kern<7, MAXT, R>();
    case 8: return kern<8, MAXT, R>();
    case 9: return kern<9, MAXT, R>();
    default: return kern<10, MAXT, R>();
  }
}

void* pick_kernel(int hlog2, bool big, int rounds) {
  if (rounds == 1) return big ? kern_h<1024, 1>(hlog2) : kern_h<256, 1>(hlog2);
  return big ? kern_h<1024, 2>(hlog2) : kern_h<256, 2>(hlog2);
}

template <int HL, int R>
void* kern_pair(int mode) {
  switch (mode) {
    case kRqInt8: return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kRqInt8>);
    case kRqInt4: return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kRqInt4>);
    case kRqLloydMax: return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kRqLloydMax>);
    case kRqPercentile: return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kRqPercentile>);
    case kRqLloydMax8: return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kRqLloydMax8>);
    default: return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kPairInt4W>);
  }
}

template <int R>
void* kern_pair_h(int hlog2, int mode) {
  switch (hlog2) {
    case 0: return kern_pair<0, R>(mode);
    case 1: return kern_pair<1, R>(mode);
    case 2: return kern_pair<2, R>(mode);
    case 3: return kern_pair<3, R>(mode);
    case 4: return kern_pair<4, R>(mode);
    case 5: return kern_pair<5, R>(mode);
    case 6: return kern_pair<6, R>(mode);
    case 7: return kern_pair<7, R>(mode);
    case 8: return kern_pair<8, R>(mode);
    case 9: return kern_pair<9, R>(mode);
    default: return kern_pair<10, R>(mode);
  }
}

// widths up to kRqPairMaxD (at most 256 threads) run two tokens per pass
constexpr int kPairMaxD = kRqPairMaxD;

// CentriQ App. B.3 (Tab. 3): activation quantile rho and clip factor gamma*
constexpr double kPctRho = 0.9995;
constexpr double kPctGamma = 2.5591;

// Phi^-1(p) for the standard normal, by bisection on Phi(x) = erfc(-x / sqrt 2) / 2 (monotone)
double inv_normal_cdf(double prob) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < prob) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

}  // namespace

int rq_hmode(int h) { return h <= 32 ? 0 : (h <= 128 ? 1 : 2); }

// Position (within the row) that thread t, register i of the round's gather holds.
int64_t rq_gather_position(int h, int t, int i) {
  if (rq_hmode(h) < 2) return (int64_t)t * EP + i;
  const int E2 = h / 32;
  const int warp = t / 32, lane = t % 32;
  const int blk = lane / E2, kB = lane % E2, ia = i / E2, ib = i % E2;
  return (int64_t)warp * 1024 + (int64_t)blk * h + kB + E2 * ia + 32 * ib;
}

// Index in the swizzled round buffer at which rotated position p is stored: float2 slots
// swizzled in pairs of positions for the pair kernel, floats swizzled in fours otherwise.
int rq_round_buffer_index(int d, int p) {
  const int t = p / EP;
  if (d <= kPairMaxD) {
    const int k = (p % EP) / 2;
    return t * EP + (((k ^ (t & 7)) << 1) | (p & 1));
  }
  const int m = (p % EP) / 4;
  return t * EP + (((m ^ (t & 7)) << 2) | (p & 3));
}

oq_status launch_rotate_quant(const RqArgs& a, cudaStream_t s) {
  if (a.T == 0) return OQ_OK;
  int hlog2 = 0;
  while ((1 << hlog2) < a.h) ++hlog2;
  const int hmode = rq_hmode(a.h);
  const int active = a.d / EP;
  const int nthr = ((active + 31) / 32) * 32;
  const bool big = nthr > 256;

  int dev_id = 0;
  cudaError_t ce = cudaGetDevice(&dev_id);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");

  // launch shape per (device, d, h, rounds, quantizer), computed once
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int>, LaunchCfg> cache;
  const int lm8 = a.mode == kRqLloydMax8 ? 1 : 0;
  const int pmode = (a.mode == kRqInt4 && a.wlayout) ? kPairInt4W : a.mode;
  LaunchCfg cfg;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_tuple(dev_id, a.d, hlog2, a.rounds, pmode);
    auto itc = cache.find(key);
    if (itc != cache.end()) {
      cfg = itc->second;
    } else {
      int nsm = 0, max_smem = 0;
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev_id);
      cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev_id);
      const size_t row_stride = ((size_t)a.d * 2 + 127) & ~(size_t)127;
      if (a.d <= kPairMaxD) {
        // two landing buffers (each a row pair, and while its pass runs the warps' transpose
        // tiles), the interleaved words, the round buffer, then reductions + code cells +
        // barriers + percentile lists and, for 8-bit Lloyd-Max codes only, the 256 thresholds
        cfg.pair = 1;
        cfg.fn = a.rounds == 1 ? kern_pair_h<1>(hlog2, pmode) : kern_pair_h<2>(hlog2, pmode);
        cfg.nthr = nthr;
        ce = allow_max_dynamic_smem(cfg.fn);
        if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(rotate_quant)");
        cfg.nbuf = kPairNbuf;
        const size_t nw = (size_t)(nthr / 32);
        size_t land = 2 * row_stride;
        if (hmode == 2) land = std::max(land, nw * 4096);
        cfg.land_bytes = (int)((land + 127) & ~(size_t)127);
        cfg.smem = kPairNbuf * (size_t)cfg.land_bytes + nw * 4096 + (a.rounds == 2 ? nw * 8192 : 0) +
                   (size_t)(224 + (lm8 ? 256 : 0)) * 4;
        int best_occ = 0;
        ce = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&best_occ, cfg.fn, nthr, cfg.smem);
        if (ce != cudaSuccess) return cuda_fail(ce, "occupancy(rotate_quant)");
        cfg.grid_per_sm = std::max(best_occ, 1) * nsm;
        cache[key] = cfg;
      } else {
      // fp32 round buffer and transpose tiles (one region when both are needed), both sized
      // in whole warps of 1024 positions
      const size_t warps_bytes = (size_t)(nthr / 32) * 4096;
      // reductions, thresholds, barriers, then the sign masks (2 bytes per channel)
      size_t fixed = ((a.rounds == 2 || hmode == 2) ? warps_bytes : 0) + 144 * 4;
      const size_t mask_bytes = (size_t)a.d * 2;
      cfg.mask_smem = fixed + mask_bytes + row_stride <= (size_t)max_smem / 3;
      if (cfg.mask_smem) fixed += mask_bytes;
      int nbuf = 2;
      while (nbuf > 1 && fixed + nbuf * row_stride > (size_t)max_smem / 3) --nbuf;
      cfg.smem = fixed + nbuf * row_stride;
      if (cfg.smem > (size_t)max_smem) return fail(OQ_ERR_UNSUPPORTED, "rotate_quant: d too large");
      cfg.fn = pick_kernel(hlog2, big, a.rounds);
      cfg.nthr = nthr;
      cfg.nbuf = nbuf;
      ce = allow_max_dynamic_smem(cfg.fn);
      if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(rotate_quant)");
      int occ = 0;
      ce = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, cfg.fn, nthr, cfg.smem);
      if (ce != cudaSuccess) return cuda_fail(ce, "occupancy(rotate_quant)");
      cfg.grid_per_sm = std::max(occ, 1) * nsm;
      cache[key] = cfg;
      }
    }
  }
  const int64_t units = cfg.pair ? (a.T + 1) / 2 : a.T;
  const int64_t grid = std::min<int64_t>(units, (int64_t)cfg.grid_per_sm);

  RqParams p{};
  p.x = reinterpret_cast<const uint16_t*>(a.x);
  p.ldx = a.ldx;
  p.T = a.T;
  p.d = a.d;
  p.hlog2 = hlog2;
  p.center = a.center;
  p.mode = a.mode;
  p.nbuf = cfg.nbuf;
  p.want_sum = (a.center || a.rowsum) ? 1 : 0;
  p.mask_smem = cfg.mask_smem;
  p.wlayout = a.wlayout;
  p.thr8 = a.thr8;
  if (a.mode == kRqLloydMax8 && !cfg.pair)
    return fail(OQ_ERR_UNSUPPORTED, "8-bit Lloyd-Max codes support d <= %d", kPairMaxD);
  if (a.mode == kRqPercentile) {
    if (!cfg.pair) return fail(OQ_ERR_UNSUPPORTED, "percentile scale supports d <= %d", kPairMaxD);
    // linear interpolation between order statistics at pos = rho (d - 1) (ascending order):
    // ranks floor(pos) and floor(pos) + 1 are the (R-1)-th and (R-2)-th largest, R = d - floor(pos)
    const double pos = kPctRho * (double)(a.d - 1);
    const double lo = std::floor(pos);
    p.pct_r = a.d - (int)lo;
    p.pct_frac = (float)(pos - lo);
    p.pct_mult = (float)(kPctGamma / inv_normal_cdf(0.5 * (1.0 + kPctRho)));
    if (p.pct_r < 2 || p.pct_r > 6) return fail(OQ_ERR_UNSUPPORTED, "percentile rank out of range");
  }
  p.tab = a.tab;
  p.smask = reinterpret_cast<const uint4*>(a.smask);
  p.slot = reinterpret_cast<const uint4*>(a.slot);
  p.land_bytes = cfg.land_bytes;
  if (cfg.pair && !a.slot) return fail(OQ_ERR_INVALID_ARG, "rotate_quant: plan has no word layout");
  p.ones = reinterpret_cast<const float4*>(a.ones);
  p.codes = a.codes;
  p.scale = a.scale;
  p.mean = a.mean;
  p.rotated = a.rotated;
  p.rowsum = a.rowsum;
  if (a.mode == kRqLloydMax) {
    // cell j covers [-4 + j/4, -4 + (j+1)/4): its threshold (at most one) and the count below
    for (int j = 0; j < 32; ++j) {
      const float lo = -4.f + 0.25f * (float)j, hi = lo + 0.25f;
      int below = 0, inside = 0;
      float theta = INFINITY;
      for (int k = 0; k < 15; ++k) {
        if (a.thr[k] < lo) ++below;
        else if (a.thr[k] < hi) { theta = a.thr[k]; ++inside; }
      }
      if (inside > 1 || a.thr[0] < -4.f || a.thr[14] >= 4.f)
        return fail(OQ_ERR_UNSUPPORTED, "rotate_quant: codebook thresholds closer than 1/4");
      float below_bits;
      std::memcpy(&below_bits, &below, sizeof(float));   // the count, as the bits of .y
      p.cells[j] = make_float2(theta, below_bits);
    }
  }
  p.inv_norm = (float)std::pow(1.0 / std::sqrt((double)a.h), (double)a.rounds);
  p.err = device_error_word();
  if (!p.err) return fail(OQ_ERR_CUDA, "device error word unavailable");
  p.limit_ns = kWaitLimitNs;

  void* args[] = {&p};
  ce = cudaLaunchKernel(cfg.fn, dim3((unsigned)grid), dim3((unsigned)cfg.nthr), args, cfg.smem, s);
  if (ce != cudaSuccess) return cuda_fail(ce, "launch rotate_quant");
  return OQ_OK;
}

}  // namespace oq
