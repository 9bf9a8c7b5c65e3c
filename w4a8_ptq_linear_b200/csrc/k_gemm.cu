// Low-bit GEMM with the fused dequant epilogue, tcgen05 on sm_100a (CentriQ §4.2 Eq. 5 and
// App. B.2 Eq. 9: y_t = W_hat Q_a(R x_t^c) + mean_t w_1 + b, rank-1 term and bias fused into
// the epilogue; OrbitQuant PR #25: absmax INT8 activations at A8, Lloyd-Max codes below).
//
// Orientation: the CTA computes D[o, t] = sum_k W[o, k] X[t, k] for 128 output channels o
// (the MMA's M) and BN tokens t (the MMA's N), so the weight operand is the one that is
// unpacked on chip and the activation tile is shared by all channel tiles through L2.
//
// Warp roles (192 threads):
//   warps 0-3  converters: packed INT4 weights (and 4-bit activations) -> INT8 / FP16 in the
//              128-byte-swizzled K-major layout the tensor core reads; then the epilogue:
//              TMEM -> registers -> scale, rank-1, bias -> bf16 -> shared -> TMA store.
//   warp 4     producer: TMA loads of the packed weight tile and the activation tile.
//   warp 5     TMEM allocator and MMA issuer (one elected thread issues tcgen05.mma).
// Pipeline per stage s: full[s] (TMA landed) -> conv[s] (operands ready) -> empty[s]
// (tcgen05.commit after the stage's MMAs). All waits are bounded.
//
// Kinds:
//   A8       X int8 via TMA, W int4 -> int8; tcgen05.mma.kind::i8, exact int32 in TMEM.
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

constexpr int BM = 128;        // output channels per CTA (MMA M)
constexpr int NCONV = 128;     // converter / epilogue threads
constexpr int NTHREADS = 192;

template <int KIND> struct KTraits;
template <> struct KTraits<kGemmA8> {
  static constexpr int BK = 128;           // K elements per stage (128 bytes of int8)
  static constexpr bool X_PACKED = false;
  static constexpr int STAGES = 3;
};
template <> struct KTraits<kGemmA4> {
  static constexpr int BK = 128;
  static constexpr bool X_PACKED = true;
  static constexpr int STAGES = 3;
};
template <> struct KTraits<kGemmLloydMax> {
  static constexpr int BK = 64;            // 64 fp16 = 128 bytes
  static constexpr bool X_PACKED = true;
  static constexpr int STAGES = 3;
};

template <int KIND, int BN>
struct Layout {
  static constexpr int BK = KTraits<KIND>::BK;
  static constexpr int STAGES = KTraits<KIND>::STAGES;
  static constexpr int W_TILE = BM * 128;                   // swizzled operand bytes
  static constexpr int X_TILE = BN * 128;
  static constexpr int WP_TILE = BM * (BK / 2);             // packed staging bytes
  static constexpr int XP_TILE = KTraits<KIND>::X_PACKED ? BN * (BK / 2) : 0;
  static constexpr int STAGE = W_TILE + X_TILE + WP_TILE + XP_TILE;
  static constexpr int OFF_W = 0;
  static constexpr int OFF_X = W_TILE;
  static constexpr int OFF_WP = W_TILE + X_TILE;
  static constexpr int OFF_XP = OFF_WP + WP_TILE;
  static constexpr int PIPE = STAGES * STAGE;
  static constexpr int OUT_BYTES_MAX = BN * BM * 4;          // epilogue staging (aliases PIPE)
  static constexpr int MAIN = PIPE > OUT_BYTES_MAX ? PIPE : OUT_BYTES_MAX;
  // small region: per-token scale/mean, barriers, TMEM address, abort flag
  static constexpr int OFF_TOK = MAIN;
  static constexpr int OFF_BAR = OFF_TOK + 2 * BN * 4;
  static constexpr int NBARS = 3 * STAGES + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int TOTAL = OFF_MISC + 16;
  static constexpr int SMEM = TOTAL + 1024;                  // slack for 1024-B alignment
  static_assert(STAGE % 1024 == 0, "stage tiles must keep 1024-byte alignment");
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

// Address of 16-byte chunk `c` (0..7) of row `r` in a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint8_t* sw128(uint8_t* tile, int r, int c) {
  return tile + r * 128 + ((c ^ (r & 7)) << 4);
}

// Packed INT4 rows of 64 bytes (128 elements) -> int8 swizzled rows.
template <int ROWS>
__device__ __forceinline__ void convert_i4_i8(const uint8_t* src, uint8_t* dst, int ctid) {
#pragma unroll 4
  for (int c = ctid; c < ROWS * 4; c += NCONV) {
    const int r = c >> 2, q = c & 3;
    const uint4 in = *reinterpret_cast<const uint4*>(src + r * 64 + q * 16);
    uint4 a, b;
    nib8_to_i8(in.x, a.x, a.y);
    nib8_to_i8(in.y, a.z, a.w);
    nib8_to_i8(in.z, b.x, b.y);
    nib8_to_i8(in.w, b.z, b.w);
    *reinterpret_cast<uint4*>(sw128(dst, r, 2 * q)) = a;
    *reinterpret_cast<uint4*>(sw128(dst, r, 2 * q + 1)) = b;
  }
}

// Packed INT4 rows of 32 bytes (64 elements) -> fp16 swizzled rows.
template <int ROWS>
__device__ __forceinline__ void convert_i4_f16(const uint8_t* src, uint8_t* dst, int ctid) {
#pragma unroll 2
  for (int c = ctid; c < ROWS * 2; c += NCONV) {
    const int r = c >> 1, q = c & 1;
    const uint4 in = *reinterpret_cast<const uint4*>(src + r * 32 + q * 16);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t o[4];
      nib8_to_f16(w[j], o);
      *reinterpret_cast<uint4*>(sw128(dst, r, 4 * q + j)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Lloyd-Max code rows of 32 bytes (64 codes) -> fp16 centroid swizzled rows.
template <int ROWS>
__device__ __forceinline__ void convert_lm_f16(const uint8_t* src, uint8_t* dst, int ctid,
                                               const uint32_t (&lut)[8]) {
#pragma unroll 2
  for (int c = ctid; c < ROWS * 2; c += NCONV) {
    const int r = c >> 1, q = c & 1;
    const uint4 in = *reinterpret_cast<const uint4*>(src + r * 32 + q * 16);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t o0, o1, o2, o3;
      lm4_to_f16(w[j] & 0xFFFFu, lut, o0, o1);
      lm4_to_f16(w[j] >> 16, lut, o2, o3);
      *reinterpret_cast<uint4*>(sw128(dst, r, 4 * q + j)) = make_uint4(o0, o1, o2, o3);
    }
  }
}

template <int KIND, int BN>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
           const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  using L = Layout<KIND, BN>;
  constexpr int BK = L::BK;
  constexpr int STAGES = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* s_tok_scale = reinterpret_cast<float*>(smem + L::OFF_TOK);
  float* s_tok_mean = s_tok_scale + BN;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);  // [0] tmem, [1] abort
  volatile uint32_t* s_abort = s_misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int o0 = blockIdx.x * BM;
  const int t0 = blockIdx.y * BN;
  const int nkb = (p.K + BK - 1) / BK;

  auto full_bar = [&](int s) { return dev::smem_u32(&bars[s]); };
  auto conv_bar = [&](int s) { return dev::smem_u32(&bars[STAGES + s]); };
  auto empty_bar = [&](int s) { return dev::smem_u32(&bars[2 * STAGES + s]); };
  const uint32_t accum_bar = dev::smem_u32(&bars[3 * STAGES]);
  const uint32_t drain_bar = dev::smem_u32(&bars[3 * STAGES + 1]);

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      dev::mbar_init(full_bar(s), 1);
      dev::mbar_init(conv_bar(s), NCONV);
      dev::mbar_init(empty_bar(s), 1);
    }
    dev::mbar_init(accum_bar, 1);
    dev::mbar_init(drain_bar, 1);
    s_misc[1] = 0;
    dev::fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    dev::prefetch_tmap(&tm_x);
    dev::prefetch_tmap(&tm_w);
    dev::prefetch_tmap(&tm_y);
  }
  if (warp == 5) {
    dev::tmem_alloc(dev::smem_u32(&s_misc[0]), BN);
    dev::tmem_relinquish();
  }
  // per-token scale and mean of this tile (zero outside [0, T))
  for (int i = tid; i < BN; i += NTHREADS) {
    const int t = t0 + i;
    s_tok_scale[i] = (t < p.T) ? p.a_scale[t] : 0.f;
    s_tok_mean[i] = (t < p.T && p.mean) ? p.mean[t] : 0.f;
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = s_misc[0];

  if (warp == 4) {
    // ---------------- producer ----------------
    if (lane == 0) {
      constexpr uint32_t bytes =
          (uint32_t)(L::WP_TILE + (KTraits<KIND>::X_PACKED ? L::XP_TILE : L::X_TILE));
      int kb = 0;
      for (; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t par = ((uint32_t)(kb / STAGES) & 1u) ^ 1u;
        if (*s_abort) break;
        if (!dev::mbar_wait(empty_bar(s), par, p.err, kSiteGemmEmpty, p.limit_ns)) {
          *s_abort = 1;
          break;
        }
        uint8_t* st = smem + s * L::STAGE;
        dev::mbar_arrive_expect_tx(full_bar(s), bytes);
        dev::tma_load_2d(dev::smem_u32(st + L::OFF_WP), &tm_w, kb * (BK / 2), o0, full_bar(s));
        if constexpr (KTraits<KIND>::X_PACKED) {
          dev::tma_load_2d(dev::smem_u32(st + L::OFF_XP), &tm_x, kb * (BK / 2), t0, full_bar(s));
        } else {
          dev::tma_load_2d(dev::smem_u32(st + L::OFF_X), &tm_x, kb * BK, t0, full_bar(s));
        }
      }
      if (*s_abort) {
        // drain: wait (bounded) for the loads of the last issued stages to land
        for (int j = std::max(0, kb - STAGES); j < kb; ++j)
          dev::mbar_wait(full_bar(j % STAGES), (uint32_t)(j / STAGES) & 1u, p.err, kSiteGemmDrain,
                         p.limit_ns);
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc =
          (KIND == kGemmLloydMax) ? dev::idesc_f16(BM, BN) : dev::idesc_i8(BM, BN);
      bool issued_any = false;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        if (*s_abort) break;
        if (!dev::mbar_wait(conv_bar(s), (uint32_t)(kb / STAGES) & 1u, p.err, kSiteGemmConv,
                            p.limit_ns)) {
          *s_abort = 1;
          break;
        }
        dev::tc_fence_after();
        uint8_t* st = smem + s * L::STAGE;
        const uint32_t aw = dev::smem_u32(st + L::OFF_W);
        const uint32_t bx = dev::smem_u32(st + L::OFF_X);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = dev::sdesc_sw128(aw + kk * 32);
          const uint64_t bd = dev::sdesc_sw128(bx + kk * 32);
          if constexpr (KIND == kGemmLloydMax)
            dev::mma_f16(tmem, ad, bd, idesc, (kb | kk) != 0);
          else
            dev::mma_i8(tmem, ad, bd, idesc, (kb | kk) != 0);
        }
        issued_any = true;
        dev::mma_commit(empty_bar(s));
      }
      if (!*s_abort) {
        dev::mma_commit(accum_bar);
      } else if (issued_any) {
        dev::mma_commit(drain_bar);
        dev::mbar_wait(drain_bar, 0, p.err, kSiteGemmDrain, p.limit_ns);
      }
    }
  } else {
    // ---------------- converters (warps 0-3) ----------------
    const int ctid = tid;  // 0..127
    uint32_t lut[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) lut[i] = p.lut[i];
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % STAGES;
      if (*s_abort) break;
      if (!dev::mbar_wait(full_bar(s), (uint32_t)(kb / STAGES) & 1u, p.err, kSiteGemmFull,
                          p.limit_ns)) {
        *s_abort = 1;
        break;
      }
      uint8_t* st = smem + s * L::STAGE;
      if constexpr (KIND == kGemmLloydMax) {
        convert_i4_f16<BM>(st + L::OFF_WP, st + L::OFF_W, ctid);
        convert_lm_f16<BN>(st + L::OFF_XP, st + L::OFF_X, ctid, lut);
      } else {
        convert_i4_i8<BM>(st + L::OFF_WP, st + L::OFF_W, ctid);
        if constexpr (KIND == kGemmA4) convert_i4_i8<BN>(st + L::OFF_XP, st + L::OFF_X, ctid);
      }
      dev::fence_async_smem();
      dev::mbar_arrive(conv_bar(s));
    }

    // ---------------- epilogue ----------------
    const int q = warp;                 // TMEM lane quarter 0..3
    const int o_local = q * 32 + lane;  // output channel within the tile
    const int o = o0 + o_local;
    bool ok = !*s_abort;
    if (ok && !dev::mbar_wait(accum_bar, 0, p.err, kSiteGemmAccum, p.limit_ns)) {
      *s_abort = 1;
      ok = false;
    }
    dev::tc_fence_after();
    const bool has_o = o < p.N;
    const float sw = has_o ? p.w_scale[o] : 0.f;
    const float w1 = (has_o && p.mean) ? p.w_rowsum[o] : 0.f;
    const float b = (has_o && p.bias) ? __bfloat162float(p.bias[o]) : 0.f;
    if (ok) {
      uint8_t* out = smem;  // pipeline stages are idle once the accumulator is complete
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        dev::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), r);
        dev::tmem_wait_ld();
        if (p.out_acc) {
          uint32_t* o32 = reinterpret_cast<uint32_t*>(out);
#pragma unroll
          for (int j = 0; j < 32; ++j) o32[(c * 32 + j) * BM + o_local] = r[j];
        } else {
          __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(out);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tl = c * 32 + j;
            const float acc = (KIND == kGemmLloydMax) ? __uint_as_float(r[j])
                                                      : (float)(int32_t)r[j];
            const float y = fmaf(acc, s_tok_scale[tl] * sw, fmaf(s_tok_mean[tl], w1, b));
            ob[tl * BM + o_local] = __float2bfloat16_rn(y);
          }
        }
      }
      dev::fence_async_smem();
      dev::named_bar(1, NCONV);
      if (tid == 0) {
        dev::tma_store_2d(&tm_y, dev::smem_u32(out), o0, t0);
        dev::bulk_commit();
        dev::bulk_wait_all_read();
      }
    }
    dev::tc_fence_before();
  }

  __syncthreads();
  if (warp == 5) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, BN);
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

template <int KIND, int BN>
oq_status run(const GemmArgs& g, const GemmParams& p, cudaStream_t s) {
  using L = Layout<KIND, BN>;
  constexpr int BK = L::BK;
  CUtensorMap tx, tw, ty;
  bool ok = true;
  if constexpr (KTraits<KIND>::X_PACKED)
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
  ok &= make_map_2d(&ty, ydt, g.out, (uint64_t)g.N, (uint64_t)g.T, (uint64_t)g.N * ysz, BM, BN,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return fail(OQ_ERR_CUDA, "cuTensorMapEncodeTiled failed or unavailable");

  auto kern = &k_gemm<KIND, BN>;
  cudaError_t ce =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(gemm)");
  const dim3 grid((unsigned)((g.N + BM - 1) / BM), (unsigned)((g.T + BN - 1) / BN));
  kern<<<grid, NTHREADS, L::SMEM, s>>>(tx, tw, ty, p);
  ce = cudaGetLastError();
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
