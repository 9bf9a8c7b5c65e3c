// The whole layer in one launch for small token counts: center + RPBH + quantize and the
// integer GEMM with its epilogue, for INT8 absmax or INT4 (absmax, percentile) activations
// against per-channel INT4 weights. INT4 codes are written one byte per code, so that every
// kind runs the same kind::i8 GEMM on them (their integer sums are those of the 4-bit GEMM).
//
// CentriQ App. B.2 runs the activation path as a prologue of its INT4 GEMM: the token tile is
// loaded once, centered, rotated and quantized with one scale per token, then multiplied. The
// per-token scale needs the whole rotated token, and at the DiT widths a tile of whole tokens
// does not fit on chip beside the GEMM's operands, so here the prologue is a phase of the same
// kernel instead of a stage of every tile:
//
//   phase A  every CTA rotates and quantizes its share of the token pairs with the two-token
//            body of the standalone kernel (rq_device.cuh), writing codes (one byte each),
//            scales and means;
//            meanwhile the CTA's remaining warps widen its slice of the packed INT4 weights
//            (which do not depend on phase A) into the tensor-core layout in shared memory;
//   grid     one grid-wide barrier (a cooperative launch, so every CTA is resident) publishes
//            the codes; they are read back from L2 by TMA while still resident there;
//   phase B  split-K GEMM: a cluster of S CTAs owns one 128-channel tile, CTA r of the cluster
//            its K blocks [r ks, (r + 1) ks), all T <= 256 tokens at once (MMA M = 128
//            channels, N = T rounded up to 32, kind::i8 into TMEM), the code tiles streaming
//            through a ring of ns stages. Each CTA moves its int32 partial sums to shared
//            memory; after a cluster barrier CTA r adds the S partials of its share of the
//            tokens through distributed shared memory and applies the epilogue of CentriQ
//            Eq. 5 / Eq. 9.
//
// Integer partial sums add exactly in any order, and the epilogue takes the same float steps
// as the two-kernel path (scale alpha_t * s_w / 16, offset mean_t * w_1 + b, one fused
// multiply-add, one rounding to bf16), so both paths return the same bits. For INT4 codes the
// two-kernel path's GEMM widens both operands (sums of 256 w x, scale s_w / 256) where this one
// widens the weights only (16 w x, s_w / 16): the factors are exact powers of two, so the
// product that enters the fused multiply-add, and hence the result, is the same.
//
// With FUSED = false the same kernel is the split-K W4A8 GEMM alone for up to 256 tokens
// (phase B on codes an earlier launch wrote): an ordinary cluster launch, no grid barrier.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cooperative_groups.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "oq_internal.h"
#include "ptx.cuh"
#include "rq_device.cuh"

namespace oq {

bool tma_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                CUtensorMapSwizzle sw);

namespace {

constexpr int FT = 256;           // threads per CTA
constexpr int FM = 128;           // output channels per cluster (MMA M)
constexpr int FWT = FM * 128;     // widened weight bytes of one K block (128 rows x 128 B)
constexpr int kFusedMaxT = kFusedMaxTokens;   // tokens of one launch at most
constexpr int kFusedMaxS = 8;     // CTAs per cluster at most (portable cluster size)
constexpr int kFusedMaxNs = 8;    // code-tile stages at most
constexpr int kTokUnroll = 4;     // tokens per warp in flight in the cluster reduction

struct FusedParams {
  RqParams rq;                    // phase A: codes int8 [T, K], scale [T], mean [T]
  const uint8_t* w;               // packed INT4 weights [N, K/2], GEMM layout
  const float* w_scale;
  const float* w_rowsum;          // null without centering
  const __nv_bfloat16* bias;      // may be null
  __nv_bfloat16* y;               // [T, N]
  int T, K, N, npad, ks, nkb, ns, rq_threads;
  int off_u, off_bar, off_tok;    // shared-memory offsets: union region, barriers, token scales
  unsigned long long* err;
  unsigned long long limit_ns;
};

// This CTA's weight tile, widened in place. At launch one TMA load per K block k brings the
// packed rows (GEMM layout, 64 bytes = 128 elements per row) into the upper half of the K
// block's 16 KB of widened weights; here they become int8 rows of 16 w in the 128-byte-swizzled
// K-major layout of the MMA's A operand (as the GEMM's converters), written over the whole
// 16 KB. Each of the nt participating threads (t = 0 .. nt - 1) first reads its packed groups
// of the K block into registers, then, after a named barrier over the nt threads, writes them
// widened, so that no write overtakes a read of the same block. Rows past N arrive as zeros.
constexpr uint32_t kWidenBarrier = 2;
constexpr int kWidenMaxItems = 4;   // packed 16-byte groups per thread and K block (nt >= 128)
static_assert(FM * 4 <= kWidenMaxItems * (FT / 2), "widening threads: at least half the block");
static_assert((2 * kFusedMaxNs + 2) * 8 + 8 <= 256, "barriers and misc fit their 256 bytes");

__device__ __forceinline__ void widen_weights(uint8_t* ww, int nk, int t, int nt) {
  for (int k = 0; k < nk; ++k) {
    uint8_t* blk = ww + k * FWT;
    const uint8_t* packed = blk + FWT / 2;
    uint4 in[kWidenMaxItems];
#pragma unroll
    for (int j = 0; j < kWidenMaxItems; ++j) {
      const int i = t + j * nt;   // group q = i & 3 of row i >> 2
      if (i < FM * 4) in[j] = *reinterpret_cast<const uint4*>(packed + i * 16);
    }
    dev::named_bar(kWidenBarrier, nt);
#pragma unroll
    for (int j = 0; j < kWidenMaxItems; ++j) {
      const int i = t + j * nt;
      if (i >= FM * 4) break;
      const int row = i >> 2, q = i & 3;
      const uint4 v = in[j];
      const uint4 lo = make_uint4((v.x << 4) & 0xF0F0F0F0u, (v.y << 4) & 0xF0F0F0F0u,
                                  (v.z << 4) & 0xF0F0F0F0u, (v.w << 4) & 0xF0F0F0F0u);
      const uint4 hi = make_uint4(v.x & 0xF0F0F0F0u, v.y & 0xF0F0F0F0u, v.z & 0xF0F0F0F0u,
                                  v.w & 0xF0F0F0F0u);
      uint8_t* dst = blk + row * 128;
      *reinterpret_cast<uint4*>(dst + (((2 * q) ^ (row & 7)) << 4)) = lo;
      *reinterpret_cast<uint4*>(dst + (((2 * q + 1) ^ (row & 7)) << 4)) = hi;
    }
  }
}

// FUSED = false: the GEMM alone (phase B) on codes, scales and means a previous launch wrote;
// no grid barrier, no cooperative launch; every thread widens the weights once they land.
// MODE: phase A's quantizer (kRqInt8, kPairInt4B or kPairPct4B).
template <int HLOG2, int ROUNDS, bool FUSED, int MODE>
__global__ void __launch_bounds__(FT, 1)
    k_linear_fused(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ww = smem;                          // widened weights, ks K blocks
  uint8_t* u = smem + p.off_u;                 // phase A scratch | X tiles | partial sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  // bars: full[ns], empty[ns], done, wfull; then the TMEM base and the abort flag
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 2 * kFusedMaxNs + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = (int)dev::cluster_nctarank();
  const int r = (int)dev::cluster_ctarank();
  const int o0 = ((int)blockIdx.x / S) * FM;   // the cluster's channel tile
  const int kb0 = r * p.ks;
  const int nk = max(0, min(p.nkb, kb0 + p.ks) - kb0);
  const int npad = p.npad;
  const int ns = p.ns;
  auto full = [&](int st) { return dev::smem_u32(&bars[st]); };
  auto empty = [&](int st) { return dev::smem_u32(&bars[kFusedMaxNs + st]); };
  const uint32_t done = dev::smem_u32(&bars[2 * kFusedMaxNs]);
  const uint32_t wfull = dev::smem_u32(&bars[2 * kFusedMaxNs + 1]);
  const int stage_bytes = npad * 128;

  if (tid == 0) {
    for (int st = 0; st < ns; ++st) {
      dev::mbar_init(full(st), 1);
      dev::mbar_init(empty(st), 1);
    }
    dev::mbar_init(done, 1);
    dev::mbar_init(wfull, 1);
    misc[1] = 0u;
    dev::fence_mbar_init();
    dev::prefetch_tmap(&tm_x);
    // the packed weights do not depend on phase A: their loads fly while it runs
    dev::mbar_arrive_expect_tx(wfull, (uint32_t)(nk * (FWT / 2)));
    for (int k = 0; k < nk; ++k)
      dev::tma_load_2d(dev::smem_u32(ww + k * FWT + FWT / 2), &tm_w, (kb0 + k) * 64, o0, wfull);
  }
  if (warp == 1) {
    dev::tmem_alloc(dev::smem_u32(&misc[0]), kFusedMaxT);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = misc[0];

  // ---- phase A: rotate-quantize the token pairs; widen this CTA's weights ------------------
  const int nrq = FUSED ? p.rq_threads : 0;
  if constexpr (FUSED)
    if (tid < nrq)
      rq_pair_body<HLOG2, ROUNDS, MODE>(p.rq, u, (int)blockIdx.x, (int)gridDim.x, nrq, true);
  // the widening threads: the four or more warps phase A leaves idle, else all after phase A;
  // their first thread waits for the packed weights, the others meet it at the named barrier
  const int w0 = FT - nrq >= FT / 2 ? nrq : 0;
  if (tid >= w0) {
    if (tid == w0 && nk > 0 && !dev::mbar_wait(wfull, 0, p.err, kSiteFusedLoad, p.limit_ns))
      misc[1] = 1u;
    dev::named_bar(kWidenBarrier, FT - w0);
    widen_weights(ww, nk, tid - w0, FT - w0);
  }
  // this thread's generic shared-memory writes (widened weights, phase A scratch) are ordered
  // before the tensor core's reads and the TMA writes that follow the barrier below
  dev::fence_async_smem();
  if constexpr (FUSED) {
    // every CTA's codes, scales and means are written (the grid barrier orders them before
    // what follows in every CTA)
    cooperative_groups::this_grid().sync();
  } else {
    __syncthreads();   // the widened weights, before the MMA thread reads them
  }

  // ---- phase B: split-K GEMM ---------------------------------------------------------------
  int issued = 0;   // code tiles this CTA's producer issued (thread 0)
  if (tid == 0 && nk > 0) {
    if constexpr (FUSED) dev::fence_async_global();   // the codes acquired above, before TMA
    for (int k = 0; k < nk; ++k) {
      const int st = k % ns;
      if (k >= ns && !dev::mbar_wait(empty(st), (uint32_t)((k / ns) - 1) & 1u, p.err,
                                     kSiteGemmEmpty, p.limit_ns)) {
        misc[1] = 1u;
        break;
      }
      if (*reinterpret_cast<volatile uint32_t*>(&misc[1]) != 0u) break;
      if (!OQ_IN_BOUNDS((st + 1) * stage_bytes <= p.off_bar - p.off_u, p.err, kSiteBoundsFused)) {
        misc[1] = 1u;
        break;
      }
      dev::mbar_arrive_expect_tx(full(st), (uint32_t)stage_bytes);
      dev::tma_load_2d(dev::smem_u32(u + st * stage_bytes), &tm_x, (kb0 + k) * 128, 0, full(st));
      issued = k + 1;
    }
  }
  if (warp == 1 && lane == 0) {
    const uint32_t idesc = dev::idesc_i8(FM, npad);
    for (int k = 0; k < nk; ++k) {
      const int st = k % ns;
      if (!dev::mbar_wait(full(st), (uint32_t)(k / ns) & 1u, p.err, kSiteFusedLoad,
                          p.limit_ns)) {
        misc[1] = 1u;
        break;
      }
      dev::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = dev::sdesc_sw128(dev::smem_u32(ww + k * FWT) + kk * 32);
        const uint64_t bd = dev::sdesc_sw128(dev::smem_u32(u + st * stage_bytes) + kk * 32);
        dev::mma_i8(tmem, ad, bd, idesc, (k | kk) != 0);
      }
      dev::mma_commit(empty(st));   // the stage is free once these MMAs have read it
    }
    dev::mma_commit(done);   // arrives once every MMA issued above has completed
  }

  // This CTA's share of the tokens for the reduction: [t0, t1).
  const int tps = (p.T + S - 1) / S;
  const int t0 = min(p.T, r * tps), t1 = min(p.T, t0 + tps);
  // their scales and means (written by other CTAs in phase A, ordered by the grid barrier),
  // read at L2 while the MMAs run; the cluster barrier below publishes them to the CTA
  float2* s_tok = reinterpret_cast<float2*>(smem + p.off_tok);
  for (int t = t0 + tid; t < t1; t += FT)
    if (OQ_IN_BOUNDS(t - t0 < kFusedMaxT, p.err, kSiteBoundsFused))
      s_tok[t - t0] = make_float2(__ldcg(p.rq.scale + t), p.rq.mean ? __ldcg(p.rq.mean + t) : 0.f);

  // ---- partial sums: TMEM -> shared memory (int32 [npad tokens][128 channels]) -------------
  // A token's 128 partial sums are 512 contiguous bytes, so that the reduction below reads
  // whole rows from the other CTAs' shared memory; the stores of a warp (32 channels of one
  // token) are 128 contiguous bytes.
  {
    bool ok = true;
    if (lane == 0) ok = dev::mbar_wait(done, 0, p.err, kSiteFusedMma, p.limit_ns);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    dev::tc_fence_after();
    const bool valid = ok && nk > 0 && *reinterpret_cast<volatile uint32_t*>(&misc[1]) == 0u;
    int32_t* part = reinterpret_cast<int32_t*>(u);   // the code tiles are consumed
    const int q = warp & 3, o_local = q * 32 + lane;   // TMEM lane quarter of this warp
    const bool fits = OQ_IN_BOUNDS(npad * FM * 4 <= p.off_bar - p.off_u, p.err, kSiteBoundsFused);
    for (int c = warp >> 2; fits && c < npad / 32; c += 2) {
      uint32_t v[32];
      dev::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), v);
      dev::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) part[(c * 32 + j) * FM + o_local] = valid ? (int32_t)v[j] : 0;
    }
  }
  dev::tc_fence_before();
  __syncwarp();
  dev::cluster_sync();   // every CTA's partial sums are in its shared memory

  // ---- cluster reduction and epilogue ------------------------------------------------------
  // Thread: four consecutive channels of one token per item, the S partial sums of the
  // cluster's CTAs loaded together; a warp reads one token's whole row from each CTA and
  // writes 256 contiguous bytes of y. y = bf16(acc * (alpha_t s_w / 16) + (mean_t w_1 + b)).
  {
    const int c4 = lane * 4;
    const int o = o0 + c4;
    const bool has = o < p.N;   // N % 16 == 0: the four channels lie all inside or all outside
    float sw[4], w1[4], bb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sw[i] = has ? p.w_scale[o + i] * (1.f / 16.f) : 0.f;   // 1/16: the widened weights
      w1[i] = (has && p.w_rowsum) ? p.w_rowsum[o + i] : 0.f;
      bb[i] = (has && p.bias) ? __bfloat162float(p.bias[o + i]) : 0.f;
    }
    const uint32_t part0 = dev::smem_u32(u) + (uint32_t)(c4 * 4);
    uint32_t peer[kFusedMaxS];
#pragma unroll
    for (int sr = 0; sr < kFusedMaxS; ++sr)
      peer[sr] = sr < S ? dev::map_to_cta(part0, (uint32_t)sr) : 0u;
    const bool fits = OQ_IN_BOUNDS(t1 <= npad && t1 - t0 <= kFusedMaxT, p.err, kSiteBoundsFused);
    // kTokUnroll tokens per warp and iteration: their S x kTokUnroll remote loads are all in
    // flight together (a remote load takes about as long as the rest of the iteration)
    for (int tb = t0 + warp; fits && tb < t1; tb += kTokUnroll * (FT / 32)) {
      uint4 v[kTokUnroll][kFusedMaxS];
#pragma unroll
      for (int uu = 0; uu < kTokUnroll; ++uu) {
        const int t = tb + uu * (FT / 32);
        const uint32_t off = (uint32_t)(t * FM * 4);
#pragma unroll
        for (int sr = 0; sr < kFusedMaxS; ++sr)
          if (sr < S && t < t1) v[uu][sr] = dev::ld_cluster_v4(peer[sr] + off);
      }
#pragma unroll
      for (int uu = 0; uu < kTokUnroll; ++uu) {
        const int t = tb + uu * (FT / 32);
        if (t >= t1) break;
        int32_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int sr = 0; sr < kFusedMaxS; ++sr)
          if (sr < S) {
            acc[0] += (int32_t)v[uu][sr].x; acc[1] += (int32_t)v[uu][sr].y;
            acc[2] += (int32_t)v[uu][sr].z; acc[3] += (int32_t)v[uu][sr].w;
          }
        const float2 tk = s_tok[t - t0];
        uint32_t yb[2];
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
          const float2 s2 = __fmul2_rn(make_float2(tk.x, tk.x), make_float2(sw[i], sw[i + 1]));
          const float2 c2 = __ffma2_rn(make_float2(tk.y, tk.y), make_float2(w1[i], w1[i + 1]),
                                       make_float2(bb[i], bb[i + 1]));
          const float2 a2 = make_float2((float)acc[i], (float)acc[i + 1]);
          const __nv_bfloat162 yv = __float22bfloat162_rn(__ffma2_rn(a2, s2, c2));
          yb[i / 2] = *reinterpret_cast<const uint32_t*>(&yv);
        }
        if (has)
          *reinterpret_cast<uint2*>(p.y + (int64_t)t * p.N + o) = make_uint2(yb[0], yb[1]);
      }
    }
  }
  __syncwarp();
  dev::cluster_sync();   // no CTA leaves while another still reads its partial sums

  // after an abort, loads already issued may still land: wait for them (bounded) before the
  // block exits (a stage's barrier is at most one phase past its last issued load)
  if (tid == 0 && misc[1] != 0u) {
    for (int k = max(0, issued - ns); k < issued; ++k)
      dev::mbar_wait(full(k % ns), (uint32_t)(k / ns) & 1u, p.err, kSiteGemmDrain, p.limit_ns);
    if (nk > 0) dev::mbar_wait(wfull, 0, p.err, kSiteGemmDrain, p.limit_ns);
  }
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, kFusedMaxT);
  }
}

template <int HL, int R, int M>
const void* fused_kern() {
  return reinterpret_cast<const void*>(&k_linear_fused<HL, R, true, M>);
}

template <int R, int M>
const void* fused_kern_h(int hlog2) {
  switch (hlog2) {
    case 0: return fused_kern<0, R, M>();
    case 1: return fused_kern<1, R, M>();
    case 2: return fused_kern<2, R, M>();
    case 3: return fused_kern<3, R, M>();
    case 4: return fused_kern<4, R, M>();
    case 5: return fused_kern<5, R, M>();
    case 6: return fused_kern<6, R, M>();
    case 7: return fused_kern<7, R, M>();
    case 8: return fused_kern<8, R, M>();
    case 9: return fused_kern<9, R, M>();
    default: return fused_kern<10, R, M>();
  }
}

template <int M>
const void* fused_kern_m(int rounds, int hlog2) {
  return rounds == 1 ? fused_kern_h<1, M>(hlog2) : fused_kern_h<2, M>(hlog2);
}

// Shared memory of a launch: widened weights, the union region, barriers, alignment slack.
struct FusedShape {
  int ks = 0, S = 0, ns = 0, off_u = 0, off_bar = 0, off_tok = 0;
  size_t smem = 0;
};

// ks K blocks per CTA: the widened weights, then the union of the phase A scratch, the partial
// sums and as many code-tile stages (up to ks) as the shared memory leaves room for; ns = 0 if
// not even one stage fits.
FusedShape fused_shape(int ks, int nkb, int npad, size_t rq_smem, size_t max_smem) {
  FusedShape f;
  f.ks = ks;
  f.S = (nkb + ks - 1) / ks;
  f.off_u = ks * FWT;
  // barriers and misc (256 B), the token scales and means (8 B a token), alignment slack
  const size_t tail = 256 + 8 * kFusedMaxT + 1024;
  const size_t stage = (size_t)npad * 128;
  const size_t fixed = std::max(rq_smem, (size_t)npad * FM * 4);
  const size_t room = max_smem > f.off_u + tail ? max_smem - f.off_u - tail : 0;
  int ns = std::min(std::min(ks, kFusedMaxNs), (int)(room / stage));
  size_t uz = std::max(fixed, (size_t)ns * stage);
  uz = (uz + 1023) & ~(size_t)1023;
  if (uz > room) ns = 0;
  f.ns = ns;
  f.off_bar = f.off_u + (int)uz;
  f.off_tok = f.off_bar + 256;
  f.smem = (size_t)f.off_bar + tail;
  return f;
}

// Shape, tensor maps and launch of the kernel `fn` (the single launch, or with
// cooperative = false the GEMM alone) for T tokens, K x N weights; p holds everything else.
oq_status launch_shaped(const void* fn, bool cooperative, FusedParams& p, const void* codes,
                        const uint8_t* w, int64_t T, int64_t K, int64_t N, size_t rq_smem,
                        cudaStream_t s) {
  cudaError_t ce = allow_max_dynamic_smem(fn);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaFuncSetAttribute(linear_fused)");
  int dev = 0, max_smem = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int npad = ((int)T + 31) / 32 * 32;
  const int nkb = (int)(K / 128);
  const int n_o = (int)((N + FM - 1) / FM);

  // The smallest K share per CTA (most CTAs) whose cluster fits the portable size and whose
  // shared memory fits; for the single launch its clusters must also all be resident at once
  // (the grid barrier needs that). Computed once per (device, kernel, T rounded, K, N).
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int, int, int, size_t>, FusedShape> cache;
  FusedShape f;
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, fn, npad, nkb, n_o, rq_smem);
    auto it = cache.find(key);
    if (it != cache.end()) {
      f = it->second;
    } else {
      for (int ks = (nkb + kFusedMaxS - 1) / kFusedMaxS; ks <= nkb; ++ks) {
        const FusedShape c = fused_shape(ks, nkb, npad, rq_smem, (size_t)max_smem);
        if (c.ns < 1 || c.smem > (size_t)max_smem) break;   // only grows with ks
        if ((c.S - 1) * ks >= nkb) continue;          // a CTA would get no K block
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(n_o * c.S));
        cfg.blockDim = dim3(FT);
        cfg.dynamicSmemBytes = c.smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)c.S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, fn, &cfg) != cudaSuccess) {
          cudaGetLastError();
          nclusters = 0;
        }
        // the GEMM alone needs no co-residency: any size that launches at all will do, but
        // the clusters that fit at once bound its parallelism the same way
        if (nclusters >= n_o) {
          f = c;
          break;
        }
      }
      cache[key] = f;
    }
  }
  if (f.ks == 0)
    return fail(OQ_ERR_UNSUPPORTED, "single-launch layer: %d channel tiles do not fit at once",
                n_o);

  CUtensorMap tx, tw;
  if (!tma_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, (uint64_t)K, (uint64_t)T,
                  (uint64_t)K, 128, (uint32_t)npad, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tma_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)K / 2, (uint64_t)N,
                  (uint64_t)K / 2, 64, FM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return fail(OQ_ERR_CUDA, "cuTensorMapEncodeTiled failed or unavailable");
  p.T = (int)T;
  p.K = (int)K;
  p.N = (int)N;
  p.npad = npad;
  p.ks = f.ks;
  p.ns = f.ns;
  p.nkb = nkb;
  p.off_u = f.off_u;
  p.off_bar = f.off_bar;
  p.off_tok = f.off_tok;
  p.err = device_error_word();
  if (!p.err) return fail(OQ_ERR_CUDA, "device error word unavailable");
  p.limit_ns = kWaitLimitNs;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(n_o * f.S));
  cfg.blockDim = dim3(FT);
  cfg.dynamicSmemBytes = f.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)f.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 2 : 1;
  void* args[] = {&tx, &tw, &p};
  ce = cudaLaunchKernelExC(&cfg, fn, args);
  if (ce == cudaErrorCooperativeLaunchTooLarge) {
    // the device cannot hold every CTA at once right now (e.g. a partitioned or shared GPU):
    // nothing was launched, and the caller takes the two-kernel path
    cudaGetLastError();
    return fail(OQ_ERR_UNSUPPORTED, "single-launch layer: the grid does not fit at once");
  }
  if (ce != cudaSuccess) return cuda_fail(ce, "launch linear_fused");
  return OQ_OK;
}

}  // namespace

oq_status launch_linear_fused(const FusedArgs& a, cudaStream_t s) {
  if (a.T <= 0 || a.T > kFusedMaxT)
    return fail(OQ_ERR_UNSUPPORTED, "single-launch layer: T must be in [1, %d]", kFusedMaxT);
  if (a.rq.mode != kRqInt8 && a.rq.mode != kRqInt4 && a.rq.mode != kRqPercentile)
    return fail(OQ_ERR_UNSUPPORTED,
                "single-launch layer: INT8 absmax, INT4 absmax or INT4 percentile activations");
  if (a.N % 16 || a.K % 128)
    return fail(OQ_ERR_UNSUPPORTED, "single-launch layer: d_in %% 128 == 0, d_out %% 16 == 0");
  FusedParams p{};
  int rq_threads = 0;
  size_t rq_smem = 0;
  oq_status st = rq_pair_setup(a.rq, p.rq, rq_threads, rq_smem);
  if (st != OQ_OK) return st;
  if (rq_threads > FT) return fail(OQ_ERR_UNSUPPORTED, "single-launch layer: d too large");
  int hlog2 = 0;
  while ((1 << hlog2) < a.rq.h) ++hlog2;
  const void* fn = a.rq.mode == kRqInt8 ? fused_kern_m<kRqInt8>(a.rq.rounds, hlog2)
                   : a.rq.mode == kRqInt4 ? fused_kern_m<kPairInt4B>(a.rq.rounds, hlog2)
                                          : fused_kern_m<kPairPct4B>(a.rq.rounds, hlog2);
  p.w = a.w;
  p.w_scale = a.w_scale;
  p.w_rowsum = a.w_rowsum;
  p.bias = reinterpret_cast<const __nv_bfloat16*>(a.bias);
  p.y = reinterpret_cast<__nv_bfloat16*>(a.y);
  p.rq_threads = rq_threads;
  return launch_shaped(fn, true, p, a.rq.codes, a.w, a.T, a.K, a.N, rq_smem, s);
}

oq_status launch_gemm_splitk(const GemmArgs& g, cudaStream_t s) {
  if (g.kind != kGemmA8 || g.out_acc || g.T < 1 || g.T > kFusedMaxT || g.N % 16 || g.K % 128)
    return fail(OQ_ERR_UNSUPPORTED, "split-K GEMM: W4A8, bf16 output, T <= %d", kFusedMaxT);
  FusedParams p{};
  p.rq.scale = const_cast<float*>(g.a_scale);
  p.rq.mean = const_cast<float*>(g.mean);
  p.w = g.w;
  p.w_scale = g.w_scale;
  p.w_rowsum = g.mean ? g.w_rowsum : nullptr;
  p.bias = reinterpret_cast<const __nv_bfloat16*>(g.bias);
  p.y = reinterpret_cast<__nv_bfloat16*>(g.out);
  p.rq_threads = 0;
  const void* fn = reinterpret_cast<const void*>(&k_linear_fused<0, 1, false, kRqInt8>);
  return launch_shaped(fn, false, p, g.a, g.w, g.T, g.K, g.N, 0, s);
}

}  // namespace oq
