// Low-bit GEMM with the fused dequant epilogue, tcgen05 on sm_100a (CentriQ §4.2 Eq. 5 and
// App. B.2 Eq. 9: y_t = W_hat Q_a(R x_t^c) + mean_t w_1 + b, with the rank-1 term and the bias
// added in the GEMM epilogue; OrbitQuant PR #25: absmax INT8 activations at A8, Lloyd-Max
// codes below).
//
// Orientation: a tile is D[o, t] = sum_k W[o, k] X[t, k] for 128 output channels o (the MMA's
// M) and BN tokens t (the MMA's N). The weight operand is the one unpacked on chip, and the
// activation tile is shared through L2 by every channel tile of the same token range.
//
// Persistent CTAs (one per SM) walk the tiles in channel-fastest order. Warp roles (320 thr):
//   warp 0     producer: TMA loads of the packed weight tile and of the activation tile into
//              an S1-deep ring;
//   warp 1     TMEM owner and MMA issuer (one thread issues tcgen05.mma, 4 per 128-byte K
//              slice, into one of two TMEM accumulators of BN columns);
//   warps 2-5  converters: packed INT4 weights (and 4-bit activations) -> INT8 / FP16 in the
//              128-byte-swizzled K-major layout, into an S2-deep ring of operand tiles;
//   warps 6-9  epilogue: TMEM -> registers -> alpha_t s_w acc + mean_t w_1 + b -> bf16 ->
//              shared staging -> TMA store, 32 tokens at a time, double-buffered, while the
//              MMA already accumulates the next tile into the other TMEM buffer.
// Barriers: full[s] (TMA landed), xempty[s] (TMA slot free), wready[c] (operands converted),
// wfree[c] (MMA done with them), tfull[b] / tempty[b] (accumulator handoff). All waits are
// bounded; a wait that gives up records its site, sets an abort flag and the roles drain.
//
// Kinds:
//   A8       X int8 straight from TMA, W int4 -> int8; tcgen05.mma.kind::i8, exact int32.
//   A4       X int4 -> int8, W int4 -> int8; kind::i8.
//   LloydMax X code -> fp16 centroid (register table via prmt), W int4 -> fp16;
//            kind::f16 with fp32 accumulation.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "oq_internal.h"
#include "ptx.cuh"

namespace oq {
namespace {

constexpr int BM = 128;       // output channels per tile (MMA M)
constexpr int NCONV = 128;    // converter threads (warps 2-5)
constexpr int NEPI = 128;     // epilogue threads (warps 6-9)
constexpr int NTHREADS = 320;
constexpr int EPI_CHUNK = 32; // tokens per epilogue store

template <int KIND, int BN>
struct Cfg {
  static constexpr int BK = (KIND == kGemmLloydMax) ? 64 : 128;   // 128 bytes of K per stage
  static constexpr bool XPACK = KIND != kGemmA8;
  static constexpr int S1 = 4;                                     // TMA stages
  static constexpr int S2 = (KIND == kGemmLloydMax) ? 3 : 2;       // converted stages
  static constexpr int WT = BM * 128;                              // W operand tile
  static constexpr int XT = BN * 128;                              // X operand tile
  static constexpr int WP = BM * (BK / 2);                         // packed W per stage
  static constexpr int XP = BN * (BK / 2);                         // packed X per stage
  static constexpr int TMA_X = XPACK ? XP : XT;
  static constexpr int TMA_STAGE = TMA_X + WP;
  static constexpr int CONV_STAGE = WT + (XPACK ? XT : 0);
  static constexpr int OFF_TMA = 0;
  static constexpr int OFF_CONV = S1 * TMA_STAGE;
  static constexpr int OFF_OUT = OFF_CONV + S2 * CONV_STAGE;
  static constexpr int OUT_BYTES = 2 * EPI_CHUNK * BM * 2;         // two bf16 chunks or one acc
  static constexpr int OFF_TOK = OFF_OUT + OUT_BYTES;              // float2 (scale, mean) [BN]
  static constexpr int OFF_BAR = OFF_TOK + BN * 8;
  static constexpr int NBAR = 2 * S1 + 2 * S2 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;                // + slack for alignment
  static constexpr uint32_t TMA_BYTES = TMA_STAGE;
  static_assert(TMA_STAGE % 1024 == 0 && CONV_STAGE % 1024 == 0 && TMA_X % 1024 == 0,
                "operand tiles must stay 1024-byte aligned");
  static_assert(BN % EPI_CHUNK == 0 && BN % 16 == 0 && BN <= 256, "MMA N");
  static_assert(SMEM <= 232448, "shared memory");
};

struct GemmParams {
  const float* a_scale;
  const float* mean;
  const float* w_scale;
  const float* w_rowsum;
  const __nv_bfloat16* bias;
  int T, K, N;
  int out_acc;
  uint32_t lut[8];     // Lloyd-Max: fp16 low bytes (0-3) and high bytes (4-7) of c_0..c_15
  unsigned long long* err;
  unsigned long long limit_ns;
};

// ---- converters --------------------------------------------------------------------------
// prmt.b32 in its default mode: selector bit 3 replicates the sign of the chosen byte
// (CUDA's __byte_perm only honours the low 3 bits of each selector nibble).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 8 two's-complement nibbles (element 2j low, 2j+1 high in byte j) -> 8 int8.
__device__ __forceinline__ void nib8_to_i8(uint32_t w, uint32_t& o0, uint32_t& o1) {
  uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
  uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
  lo = (lo + 0x78787878u) ^ 0x80808080u;     // per-byte sign extension, no carries
  hi = (hi + 0x78787878u) ^ 0x80808080u;
  o0 = __byte_perm(lo, hi, 0x5140);
  o1 = __byte_perm(lo, hi, 0x7362);
}

// 8 two's-complement nibbles -> 8 fp16 (exact): (n ^ 8) | 0x6400 is the half 1024 + n + 8.
__device__ __forceinline__ void nib8_to_f16(uint32_t w, uint32_t (&o)[4]) {
  const uint32_t t = w ^ 0x88888888u;
  const uint32_t h0 = (t & 0x000F000Fu) | 0x64006400u;
  const uint32_t h1 = ((t >> 4) & 0x000F000Fu) | 0x64006400u;
  const uint32_t h2 = ((t >> 8) & 0x000F000Fu) | 0x64006400u;
  const uint32_t h3 = ((t >> 12) & 0x000F000Fu) | 0x64006400u;
  const uint32_t p[4] = {__byte_perm(h0, h1, 0x5410), __byte_perm(h2, h3, 0x5410),
                         __byte_perm(h0, h1, 0x7632), __byte_perm(h2, h3, 0x7632)};
  const __half2 bias = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 v = *reinterpret_cast<const __half2*>(&p[i]);
    v = __hsub2(v, bias);
    o[i] = *reinterpret_cast<uint32_t*>(&v);
  }
}

// 4 Lloyd-Max codes (nibbles of s, code 0 in bits 0-3) -> 4 fp16 centroids (2 words).
__device__ __forceinline__ void lm4_to_f16(uint32_t s, const uint32_t (&lut)[8], uint32_t& o0,
                                           uint32_t& o1) {
  const uint32_t s7 = s & 0x7777u;
  const uint32_t lo_a = __byte_perm(lut[0], lut[1], s7);
  const uint32_t lo_b = __byte_perm(lut[2], lut[3], s7);
  const uint32_t hi_a = __byte_perm(lut[4], lut[5], s7);
  const uint32_t hi_b = __byte_perm(lut[6], lut[7], s7);
  // byte j of m = 0xFF when bit 3 of code j is set (prmt sign-replicate mode)
  const uint32_t m = prmt(s << 4, s, 0xD9C8);
  const uint32_t lo = (lo_a & ~m) | (lo_b & m);
  const uint32_t hi = (hi_a & ~m) | (hi_b & m);
  o0 = __byte_perm(lo, hi, 0x5140);
  o1 = __byte_perm(lo, hi, 0x7362);
}

// Packed INT4 rows of 64 bytes -> int8 rows of 128 bytes in the 128-byte-swizzled layout
// (16-byte chunk c of row r at r * 128 + ((c ^ (r & 7)) << 4)). Thread ctid takes the
// 16-byte packed chunk q = ctid & 3 of rows ctid / 4 + 32 j; the swizzle phase r & 7 is the
// same for all j, so every address is a constant offset from a per-thread base.
template <int ROWS>
__device__ __forceinline__ void convert_i4_i8(const uint8_t* src, uint8_t* dst, int ctid) {
  const int r0 = ctid >> 2, q = ctid & 3;
  const uint8_t* s = src + r0 * 64 + q * 16;
  uint8_t* da = dst + r0 * 128 + (((2 * q) ^ (r0 & 7)) << 4);
  uint8_t* db = dst + r0 * 128 + (((2 * q + 1) ^ (r0 & 7)) << 4);
#pragma unroll
  for (int j = 0; j < ROWS / 32; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * 32 * 64);
    uint4 a, b;
    nib8_to_i8(in.x, a.x, a.y);
    nib8_to_i8(in.y, a.z, a.w);
    nib8_to_i8(in.z, b.x, b.y);
    nib8_to_i8(in.w, b.z, b.w);
    *reinterpret_cast<uint4*>(da + j * 32 * 128) = a;
    *reinterpret_cast<uint4*>(db + j * 32 * 128) = b;
  }
}

// Packed INT4 rows of 32 bytes (64 elements) -> fp16 rows of 128 bytes, swizzled.
template <int ROWS>
__device__ __forceinline__ void convert_i4_f16(const uint8_t* src, uint8_t* dst, int ctid) {
  const int r0 = ctid >> 1, q = ctid & 1;
  const uint8_t* s = src + r0 * 32 + q * 16;
  uint8_t* d = dst + r0 * 128;
  const int ph = r0 & 7;
#pragma unroll
  for (int j = 0; j < ROWS / 64; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * 64 * 32);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t o[4];
      nib8_to_f16(w[k], o);
      *reinterpret_cast<uint4*>(d + j * 64 * 128 + (((4 * q + k) ^ ph) << 4)) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Lloyd-Max code rows of 32 bytes (64 codes) -> fp16 centroid rows of 128 bytes, swizzled.
template <int ROWS>
__device__ __forceinline__ void convert_lm_f16(const uint8_t* src, uint8_t* dst, int ctid,
                                               const uint32_t (&lut)[8]) {
  const int r0 = ctid >> 1, q = ctid & 1;
  const uint8_t* s = src + r0 * 32 + q * 16;
  uint8_t* d = dst + r0 * 128;
  const int ph = r0 & 7;
#pragma unroll
  for (int j = 0; j < ROWS / 64; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * 64 * 32);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t o0, o1, o2, o3;
      lm4_to_f16(w[k] & 0xFFFFu, lut, o0, o1);
      lm4_to_f16(w[k] >> 16, lut, o2, o3);
      *reinterpret_cast<uint4*>(d + j * 64 * 128 + (((4 * q + k) ^ ph) << 4)) =
          make_uint4(o0, o1, o2, o3);
    }
  }
}

template <int KIND, int BN>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
           const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  using C = Cfg<KIND, BN>;
  constexpr int BK = C::BK, S1 = C::S1, S2 = C::S2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float2* s_tok = reinterpret_cast<float2*>(smem + C::OFF_TOK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);  // tmem, abort, epi flag
  volatile uint32_t* s_abort = s_misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_o = (p.N + BM - 1) / BM;
  const int n_tiles = n_o * ((p.T + BN - 1) / BN);
  const int nkb = (p.K + BK - 1) / BK;

  auto bar = [&](int i) { return dev::smem_u32(&bars[i]); };
  auto full_bar = [&](int s) { return bar(s); };
  auto xempty_bar = [&](int s) { return bar(S1 + s); };
  auto wready_bar = [&](int c) { return bar(2 * S1 + c); };
  auto wfree_bar = [&](int c) { return bar(2 * S1 + S2 + c); };
  auto tfull_bar = [&](int b) { return bar(2 * S1 + 2 * S2 + b); };
  auto tempty_bar = [&](int b) { return bar(2 * S1 + 2 * S2 + 2 + b); };
  const uint32_t drain_bar = bar(2 * S1 + 2 * S2 + 4);
  auto tma_stage = [&](int s) { return smem + C::OFF_TMA + s * C::TMA_STAGE; };
  auto conv_stage = [&](int c) { return smem + C::OFF_CONV + c * C::CONV_STAGE; };

  if (tid == 0) {
    for (int s = 0; s < S1; ++s) {
      dev::mbar_init(full_bar(s), 1);
      dev::mbar_init(xempty_bar(s), C::XPACK ? NCONV : 1);
    }
    for (int c = 0; c < S2; ++c) {
      dev::mbar_init(wready_bar(c), NCONV);
      dev::mbar_init(wfree_bar(c), 1);
    }
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(tfull_bar(b), 1);
      dev::mbar_init(tempty_bar(b), NEPI);
    }
    dev::mbar_init(drain_bar, 1);
    s_misc[1] = 0;
    dev::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    dev::prefetch_tmap(&tm_x);
    dev::prefetch_tmap(&tm_w);
    dev::prefetch_tmap(&tm_y);
  }
  if (warp == 1) {
    dev::tmem_alloc(dev::smem_u32(&s_misc[0]), 2 * BN);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = s_misc[0];

  auto give_up = [&]() { *s_abort = 1; };

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      uint32_t j = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        const int o0 = (tile % n_o) * BM, t0 = (tile / n_o) * BN;
        for (int kb = 0; kb < nkb; ++kb, ++j) {
          const int s = j % S1;
          if (*s_abort ||
              !dev::mbar_wait(xempty_bar(s), ((j / S1) & 1u) ^ 1u, p.err, kSiteGemmEmpty,
                              p.limit_ns)) {
            give_up();
            ok = false;
            break;
          }
          uint8_t* st = tma_stage(s);
          dev::mbar_arrive_expect_tx(full_bar(s), C::TMA_BYTES);
          dev::tma_load_2d(dev::smem_u32(st + C::TMA_X), &tm_w, kb * (BK / 2), o0, full_bar(s));
          dev::tma_load_2d(dev::smem_u32(st), &tm_x, C::XPACK ? kb * (BK / 2) : kb * BK, t0,
                           full_bar(s));
        }
      }
      if (!ok) {  // let the loads already issued land before the block can exit
        for (uint32_t i = (j >= (uint32_t)S1 ? j - S1 : 0); i < j; ++i)
          dev::mbar_wait(full_bar(i % S1), (i / S1) & 1u, p.err, kSiteGemmDrain, p.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc =
          (KIND == kGemmLloydMax) ? dev::idesc_f16(BM, BN) : dev::idesc_i8(BM, BN);
      uint32_t j = 0, it = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++it) {
        const int b = it & 1;
        if (*s_abort || !dev::mbar_wait(tempty_bar(b), ((it >> 1) & 1u) ^ 1u, p.err,
                                        kSiteGemmAccum, p.limit_ns)) {
          give_up();
          ok = false;
          break;
        }
        dev::tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(b * BN);
        for (int kb = 0; kb < nkb; ++kb, ++j) {
          const int s = j % S1, c = j % S2;
          bool w = !*s_abort &&
                   dev::mbar_wait(wready_bar(c), (j / S2) & 1u, p.err, kSiteGemmConv, p.limit_ns);
          if (w && !C::XPACK)
            w = dev::mbar_wait(full_bar(s), (j / S1) & 1u, p.err, kSiteGemmFull, p.limit_ns);
          if (!w) {
            give_up();
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t aw = dev::smem_u32(conv_stage(c));
          const uint32_t bx = C::XPACK ? dev::smem_u32(conv_stage(c) + C::WT)
                                       : dev::smem_u32(tma_stage(s));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = dev::sdesc_sw128(aw + kk * 32);
            const uint64_t bd = dev::sdesc_sw128(bx + kk * 32);
            if constexpr (KIND == kGemmLloydMax)
              dev::mma_f16(dt, ad, bd, idesc, (kb | kk) != 0);
            else
              dev::mma_i8(dt, ad, bd, idesc, (kb | kk) != 0);
          }
          issued = true;
          dev::mma_commit(wfree_bar(c));
          if (!C::XPACK) dev::mma_commit(xempty_bar(s));
        }
        if (!ok) break;
        dev::mma_commit(tfull_bar(b));
      }
      if (!ok && issued) {  // wait for the MMAs in flight before TMEM is freed
        dev::mma_commit(drain_bar);
        dev::mbar_wait(drain_bar, 0, p.err, kSiteGemmDrain, p.limit_ns);
      }
    }
  } else if (warp < 6) {
    // ---------------- converters ----------------
    const int ctid = tid - 64;
    uint32_t lut[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) lut[i] = p.lut[i];
    uint32_t j = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb, ++j) {
        const int s = j % S1, c = j % S2;
        bool w = !*s_abort &&
                 dev::mbar_wait(full_bar(s), (j / S1) & 1u, p.err, kSiteGemmFull, p.limit_ns);
        if (w)
          w = dev::mbar_wait(wfree_bar(c), ((j / S2) & 1u) ^ 1u, p.err, kSiteGemmConv,
                             p.limit_ns);
        if (!w) {
          give_up();
          ok = false;
          break;
        }
        const uint8_t* st = tma_stage(s);
        uint8_t* cv = conv_stage(c);
        if constexpr (KIND == kGemmLloydMax) {
          convert_i4_f16<BM>(st + C::TMA_X, cv, ctid);
          convert_lm_f16<BN>(st, cv + C::WT, ctid, lut);
        } else {
          convert_i4_i8<BM>(st + C::TMA_X, cv, ctid);
          if constexpr (KIND == kGemmA4) convert_i4_i8<BN>(st, cv + C::WT, ctid);
        }
        dev::fence_async_smem();
        dev::mbar_arrive(wready_bar(c));
        if (C::XPACK) dev::mbar_arrive(xempty_bar(s));
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int etid = tid - 192;          // 0..127
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const int o_local = q * 32 + lane;
    const bool leader = etid == 0;
    const int nbuf = p.out_acc ? 1 : 2;
    const int chunk_bytes = EPI_CHUNK * BM * (p.out_acc ? 4 : 2);
    uint8_t* stage_out = smem + C::OFF_OUT;
    uint32_t it = 0, g = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++it) {
      const int o0 = (tile % n_o) * BM, t0 = (tile / n_o) * BN;
      const int b = it & 1;
      const int o = o0 + o_local;
      const bool has_o = o < p.N;
      const float sw = has_o ? p.w_scale[o] : 0.f;
      const float w1 = (has_o && p.mean) ? p.w_rowsum[o] : 0.f;
      const float bb = (has_o && p.bias) ? __bfloat162float(p.bias[o]) : 0.f;
      for (int i = etid; i < BN; i += NEPI) {
        const int t = t0 + i;
        s_tok[i] = make_float2((t < p.T) ? p.a_scale[t] : 0.f,
                               (t < p.T && p.mean) ? p.mean[t] : 0.f);
      }
      // one thread waits for the accumulator; the verdict reaches all four warps through
      // shared memory behind a named barrier, so every later barrier is reached uniformly
      if (leader) {
        const bool ready = !*s_abort && dev::mbar_wait(tfull_bar(b), (it >> 1) & 1u, p.err,
                                                       kSiteGemmAccum, p.limit_ns);
        if (!ready) give_up();
        s_misc[2] = ready ? 1u : 0u;
      }
      dev::named_bar(1, NEPI);
      ok = *reinterpret_cast<volatile uint32_t*>(&s_misc[2]) != 0;
      if (ok) dev::tc_fence_after();
#pragma unroll 1
      for (int c = 0; ok && c < BN / EPI_CHUNK; ++c, ++g) {
        uint32_t r[32];
        dev::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN + c * EPI_CHUNK), r);
        dev::tmem_wait_ld();
        if (c == BN / EPI_CHUNK - 1) {  // accumulator fully read: hand it back to the MMA
          dev::tc_fence_before();
          dev::mbar_arrive(tempty_bar(b));
        }
        const int buf = (int)(g % (uint32_t)nbuf);
        if (g >= (uint32_t)nbuf) {  // the store that used this buffer must have read it
          if (leader) {
            if (nbuf == 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            else dev::bulk_wait_all_read();
          }
          dev::named_bar(1, NEPI);
        }
        uint8_t* ob = stage_out + buf * chunk_bytes;
        if (p.out_acc) {
          uint32_t* o32 = reinterpret_cast<uint32_t*>(ob);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) o32[jj * BM + o_local] = r[jj];
        } else {
          __nv_bfloat16* o16 = reinterpret_cast<__nv_bfloat16*>(ob);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float2 tk = s_tok[c * EPI_CHUNK + jj];
            const float acc = (KIND == kGemmLloydMax) ? __uint_as_float(r[jj])
                                                      : (float)(int32_t)r[jj];
            o16[jj * BM + o_local] = __float2bfloat16_rn(fmaf(acc, tk.x * sw, fmaf(tk.y, w1, bb)));
          }
        }
        dev::fence_async_smem();
        dev::named_bar(1, NEPI);
        if (leader) {
          dev::tma_store_2d(&tm_y, dev::smem_u32(ob), o0, t0 + c * EPI_CHUNK);
          dev::bulk_commit();
        }
      }
      dev::named_bar(1, NEPI);  // s_tok of this tile is no longer read
    }
    if (leader) dev::bulk_wait_all();
  }

  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, 2 * BN);
  }
}

// ---- host side ------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int KIND, int BN>
oq_status run(const GemmArgs& g, const GemmParams& p, cudaStream_t s) {
  using C = Cfg<KIND, BN>;
  constexpr int BK = C::BK;
  CUtensorMap tx, tw, ty;
  bool ok = true;
  if constexpr (C::XPACK)
    ok &= make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, (uint64_t)g.K / 2, (uint64_t)g.T,
                      (uint64_t)g.K / 2, BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    ok &= make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, (uint64_t)g.K, (uint64_t)g.T,
                      (uint64_t)g.K, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, (uint64_t)g.K / 2, (uint64_t)g.N,
                    (uint64_t)g.K / 2, BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
  const CUtensorMapDataType ydt =
      g.out_acc ? (KIND == kGemmLloydMax ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                         : CU_TENSOR_MAP_DATA_TYPE_INT32)
                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t ysz = g.out_acc ? 4 : 2;
  ok &= make_map_2d(&ty, ydt, g.out, (uint64_t)g.N, (uint64_t)g.T, (uint64_t)g.N * ysz, BM,
                    EPI_CHUNK, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return fail(OQ_ERR_CUDA, "cuTensorMapEncodeTiled failed or unavailable");

  auto kern = &k_gemm<KIND, BN>;
  const cudaError_t attr_err = allow_max_dynamic_smem(reinterpret_cast<const void*>(kern));
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(gemm)");
  const int64_t tiles = ((g.N + BM - 1) / BM) * ((g.T + BN - 1) / BN);
  const int grid = (int)std::min<int64_t>(tiles, sm_count());
  kern<<<grid, NTHREADS, C::SMEM, s>>>(tx, tw, ty, p);
  cudaError_t ce = cudaGetLastError();
  if (ce != cudaSuccess) return cuda_fail(ce, "launch gemm");
  return OQ_OK;
}

uint16_t f16_bits(float f) {
  const __half h = __float2half_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

}  // namespace

oq_status launch_gemm(const GemmArgs& g, cudaStream_t s) {
  if (g.T == 0) return OQ_OK;
  GemmParams p{};
  p.a_scale = g.a_scale;
  p.mean = g.mean;
  p.w_scale = g.w_scale;
  p.w_rowsum = g.w_rowsum;
  p.bias = reinterpret_cast<const __nv_bfloat16*>(g.bias);
  p.T = (int)g.T;
  p.K = (int)g.K;
  p.N = (int)g.N;
  p.out_acc = g.out_acc;
  if (g.kind == kGemmLloydMax) {
    uint8_t lo[16], hi[16];
    for (int i = 0; i < 16; ++i) {
      const uint16_t b = f16_bits(g.centroids[i]);
      lo[i] = (uint8_t)(b & 0xFF);
      hi[i] = (uint8_t)(b >> 8);
    }
    std::memcpy(&p.lut[0], lo, 16);
    std::memcpy(&p.lut[4], hi, 16);
  }
  p.err = device_error_word();
  if (!p.err) return fail(OQ_ERR_CUDA, "device error word unavailable");
  p.limit_ns = kWaitLimitNs;
  const bool small = g.T <= 128;
  switch (g.kind) {
    case kGemmA8: return small ? run<kGemmA8, 128>(g, p, s) : run<kGemmA8, 256>(g, p, s);
    case kGemmA4: return small ? run<kGemmA4, 128>(g, p, s) : run<kGemmA4, 256>(g, p, s);
    case kGemmLloydMax:
      return small ? run<kGemmLloydMax, 128>(g, p, s) : run<kGemmLloydMax, 256>(g, p, s);
    default: return fail(OQ_ERR_INVALID_ARG, "unknown GEMM kind");
  }
}

}  // namespace oq
