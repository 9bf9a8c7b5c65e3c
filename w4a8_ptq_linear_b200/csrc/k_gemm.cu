// Low-bit GEMM with the fused dequant epilogue, tcgen05 on sm_100a (CentriQ §4.2 Eq. 5 and
// App. B.2 Eq. 9: y_t = W_hat Q_a(R x_t^c) + mean_t w_1 + b, with the rank-1 term and the bias
// added in the GEMM epilogue; OrbitQuant PR #25: absmax INT8 activations at A8, Lloyd-Max
// codes below).
//
// Orientation: a tile is D[o, t] = sum_k W[o, k] X[t, k] for 128 output channels o per CTA (the
// MMA's M) and N tokens t (the MMA's N). The weight operand is the one unpacked on chip, and
// the activation tile is shared through L2 by every channel tile of the same token range.
//
// Two shapes (template CG):
//   CG = 1  one CTA per tile of 128 channels x N <= 128 tokens (small token counts);
//   CG = 2  a cluster of two CTAs on neighbouring SMs computes 256 channels x N <= 256 tokens
//           with tcgen05.mma.cta_group::2 (M = 256): each CTA stages and unpacks its own 128
//           weight rows and half of the activation rows, and the pair's leader issues the MMAs,
//           whose completions are multicast to both CTAs. Every activation byte that crosses L2
//           and shared memory then feeds 256 channels instead of 128.
//
// Schedule: persistent CTAs (pairs) take the tiles round robin in channel-tile-fastest order,
// so that the pairs running at the same time share activation rows through L2. Tiles are 256
// (CG = 2) or 128 (CG = 1) tokens wide; only the last token tile of a ragged T is narrower,
// and its MMAs run with an N cut to the next multiple of 32.
//
// Warp roles (608 thr; the warp numbers are those of the 4-bit kinds, INT8 activations move
// the producers to warps 5 and 9 and the converters to 0, 2-4, 6-8, 10):
//   warp 0     packed-operand producer: TMA loads of the packed weight tile (and, for 4-bit
//              activations, the packed activation rows) into an SP-deep ring that the
//              converters release as soon as they have unpacked it;
//   warp 1     TMEM owner and MMA issuer (one thread of the pair's leader issues tcgen05.mma,
//              4 per 128-byte K slice, into one of two TMEM accumulators of up to 256 columns);
//   warp 2     activation producer (INT8 activations only): TMA loads of the activation rows
//              (boxes of 16 rows, exactly the tile's width) into an SX-deep ring that only the
//              MMA releases;
//   warps 3-10 converters: packed INT4 weights (and 4-bit activations) -> INT8 / FP16 in the
//              128-byte-swizzled K-major layout, into an S2-deep ring of operand tiles; two
//              groups of four warps take alternate K blocks, so that the hand-off latency of
//              one block (barrier wait, proxy fence, arrive) overlaps the other's work;
//   warps 11-18 epilogue: TMEM -> registers -> alpha_t s_w acc + mean_t w_1 + b -> bf16 ->
//              coalesced global stores (each warp writes 32 consecutive channels of a token),
//              while the MMA already accumulates the next tile into the other TMEM buffer.
// Barriers: xfull/xempty (activation ring), pfull/pempty (packed ring), wready/wfree
// (converted operands), tfull/tempty (accumulators). With CG = 2 the barriers the MMA waits on
// (xfull, wready, tempty) are the leader's: the peer's activation loads complete on the
// leader's xfull, and its converter and epilogue warps arrive there remotely. All waits are
// bounded; a wait that gives up records its site, sets an abort flag and the roles drain.
//
// Integer widening. The weights arrive in the GEMM layout of the prepared weights: in every
// 16-byte group of a row, byte j holds element j in its low nibble and element 16 + j in its
// high nibble. A two's-complement nibble moved to the high half of a byte is the int8 16 n,
// so a group widens to two 16-byte int8 chunks with one shift and two masks per word. The
// 4-bit activations (element 2j low, 2j + 1 high in byte j) widen the same way plus two byte
// permutes. A 2-bit code moved to the top two bits of a byte is the int8 64 c. The products
// are then 16, 256 or 1024 times the true ones; the int32 sums stay exact (|16 * 127 * 7| K
// and |1024 * 7| K stay below 2^31 for K <= 32768) and the epilogue folds 1/16, 1/256 or
// 1/1024 into its scale, which is exact in floating point.
//
// Kinds:
//   A8       X int8 straight from TMA, W int4 -> 16 W int8; tcgen05.mma.kind::i8, exact int32.
//   A4       X int4 -> 16 X int8, W int4 -> 16 W int8; kind::i8.
//   A2       X 2-bit -> 64 X int8 (four codes per byte), W as A4; kind::i8.
//   LloydMax X code -> fp16 centroid (register table via prmt), W int4 -> 16 W fp16 (exact);
//            kind::f16 with fp32 accumulation.
//   LloydMax8 X 8-bit code -> fp16 centroid through a 256-entry table in shared memory, W as
//            LloydMax; kind::f16.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>

#include "oq_internal.h"
#include "ptx.cuh"

namespace oq {
namespace {

constexpr int BM = 128;       // output channels per CTA (MMA M per CTA)
constexpr int CH = 32;        // tokens per schedule chunk (MMA N granularity)
constexpr int NCONV = 256;    // converter threads (warps 3-10)
constexpr int NGROUP = 2;     // converter groups; group g converts the k-blocks j = g mod NGROUP
constexpr int NCG = NCONV / NGROUP;  // threads per converter group
constexpr int CONV0 = 96;     // threads before the epilogue that are not converters
constexpr int NEPI = 256;     // epilogue threads (warps 11-18), two per TMEM lane quarter
constexpr int EPW = NEPI / 128;               // epilogue warps per TMEM lane quarter
constexpr int EPI0 = CONV0 + NCONV;  // first epilogue thread
constexpr int NTHREADS = EPI0 + NEPI;

constexpr int kMaxPairs = 160;   // CTA pairs a balanced schedule describes at most

template <int KIND, int CG>
struct Cfg {
  static constexpr bool FP = KIND == kGemmLloydMax || KIND == kGemmLloydMax8 ||
                             KIND == kGemmG64;                       // kind::f16
  static constexpr bool X4F = KIND == kGemmLloydMax || KIND == kGemmG64;  // 4-bit codes -> fp16
  static constexpr int BK = FP ? 64 : 128;                          // 128 bytes of K per stage
  static constexpr bool XPACK = KIND != kGemmA8;
  static constexpr int XB =                                          // activation bytes per row
      KIND == kGemmLloydMax8 ? BK : (KIND == kGemmA2 ? BK / 4 : BK / 2);
  static constexpr int BNMAX = 128 * CG;                           // tokens per tile, at most
  static constexpr int MAXCH = BNMAX / CH;                         // chunks per tile, at most
  static constexpr int XR = 128;                                   // activation rows per CTA
  // Ring depths. Loads from L2 take a few thousand cycles, so the packed ring, which the
  // converters free only after unpacking, must cover that latency at the MMA's pace.
  static constexpr int SX = XPACK ? 0 : (CG == 2 ? 5 : 4);         // activation ring (A8)
  static constexpr int SP = CG == 1 ? 4 : (X4F ? 8 : 6);
  static constexpr int S2 =
      (KIND == kGemmA4 || KIND == kGemmA2) ? (CG == 2 ? 3 : 2) : (CG == 2 ? 4 : 3);
  static constexpr int WT = BM * 128;                              // W operand tile
  static constexpr int XT = XR * 128;                              // X operand tile (this CTA)
  static constexpr int WP = BM * (BK / 2);                         // packed W per stage
  static constexpr int XP = XPACK ? XR * XB : 0;                   // staged X per stage
  static constexpr int P_STAGE = XP + WP;                          // [Xp][Wp]
  static constexpr int CONV_STAGE = WT + (XPACK ? XT : 0);         // [W][X]
  static constexpr int OFF_X = 0;
  static constexpr int OFF_P = OFF_X + SX * XT;
  static constexpr int OFF_CONV = OFF_P + SP * P_STAGE;
  static constexpr int OFF_STG = OFF_CONV + S2 * CONV_STAGE;       // epilogue staging tiles
  static constexpr int STG = 32 * 32 * 2;                          // bf16 [32 tokens][32 ch]
  static constexpr int OFF_TOK = OFF_STG + (NEPI / 32) * STG;      // float2 (scale, mean)
  static constexpr int OFF_BAR = OFF_TOK + BNMAX * 8;
  static constexpr int NBAR = 2 * SX + 2 * SP + 2 * S2 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_LUT8 = OFF_MISC + 16;                   // 8-bit code -> fp16 table
  static constexpr int SMEM = OFF_LUT8 + (KIND == kGemmLloydMax8 ? 512 : 0) + 1024;
  // 1/16 per widened INT4 operand and 1/64 per widened 2-bit one (see "Integer widening"); the
  // grouped weights are decoded to their real values and the activation codes to plain integers
  static constexpr float ACC_SCALE =
      KIND == kGemmA4 ? 1.f / 256.f
                      : (KIND == kGemmA2 ? 1.f / 1024.f : (KIND == kGemmG64 ? 1.f : 1.f / 16.f));
  static constexpr int ACC_SHIFT = KIND == kGemmA4 ? 8 : (KIND == kGemmA2 ? 10 : 4);
  static_assert(XT % 1024 == 0 && P_STAGE % 1024 == 0 && CONV_STAGE % 1024 == 0 &&
                XP % 1024 == 0, "operand tiles must stay 1024-byte aligned");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(NGROUP <= S2, "a converter group may run at most one ring phase ahead");
};

struct GemmParams {
  const float* a_scale;
  const float* mean;
  const float* w_scale;
  const float* w_rowsum;
  const __nv_bfloat16* bias;
  void* out;
  int T, K, N;
  int out_acc;
  uint32_t lut[8];     // Lloyd-Max: fp16 low bytes (0-3) and high bytes (4-7) of c_0..c_15
  uint32_t lut8[128];  // 8-bit Lloyd-Max: fp16 centroids c_0..c_255, two per word
  const uint32_t* w_sz;  // grouped weights: [K/64][N] words, fp16 sigma (low half), z (high)
  unsigned long long* err;
  unsigned long long limit_ns;
  // balanced schedules: CTA pair u takes the flattened (channel tile, 32-token chunk) range
  // [sched[u], sched[u + 1])
  int sched[kMaxPairs + 1];
};

// ---- schedule ----------------------------------------------------------------------------------
// The tiles of one CTA (pair), round robin over the grid in channel-tile-fastest order, so that
// the pairs running at the same time share activation rows through L2. A tile is 256 (or 128)
// tokens of one channel tile; only the last token tile of a ragged T is narrower, and its MMAs
// run with the narrower N. Every role walks the same sequence.
template <int MAXCH>
struct TileIter {
  int tile, n_tiles, step, n_o, cpm;
  __device__ TileIter(int T, int n_o_, int unit_index, int n_units) {
    cpm = (T + CH - 1) / CH;
    n_o = n_o_;
    n_tiles = n_o * ((cpm + MAXCH - 1) / MAXCH);
    tile = unit_index;
    step = n_units;
  }
  // channel tile m, first token t0, chunks of 32 tokens nch of the next tile
  __device__ bool next(int& m, int& t0, int& nch) {
    if (tile >= n_tiles) return false;
    m = tile % n_o;
    const int tt = tile / n_o;
    t0 = tt * MAXCH * CH;
    nch = min(MAXCH, cpm - tt * MAXCH);
    tile += step;
    return true;
  }
};

// ---- converters --------------------------------------------------------------------------
// prmt.b32 in its default mode: selector bit 3 replicates the sign of the chosen byte
// (CUDA's __byte_perm only honours the low 3 bits of each selector nibble).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 8 two's-complement nibbles (element 2j low, 2j+1 high in byte j) -> 8 int8 of 16 n.
__device__ __forceinline__ void nib8_to_i8x16(uint32_t w, uint32_t& o0, uint32_t& o1) {
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;   // 16 * even elements
  const uint32_t hi = w & 0xF0F0F0F0u;          // 16 * odd elements
  o0 = __byte_perm(lo, hi, 0x5140);
  o1 = __byte_perm(lo, hi, 0x7362);
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

// Weight rows in the GEMM layout (64 packed bytes = 128 elements per stage) -> int8 rows of
// 128 bytes in the 128-byte-swizzled layout (16-byte chunk c of row r at
// r * 128 + ((c ^ (r & 7)) << 4)). Thread ctid of a group takes packed group q = ctid & 3 of
// rows ctid / 4 + (NCG / 4) j: its low nibbles are chunk 2q, its high nibbles chunk 2q + 1.
// The swizzle phase r & 7 is the same for all j, so every address is a constant offset from a
// per-thread base.
__device__ __forceinline__ void convert_w_i8(const uint8_t* src, uint8_t* dst, int ctid) {
  constexpr int RSTEP = NCG / 4;     // rows covered by one pass of the group's threads
  const int r0 = ctid >> 2, q = ctid & 3;
  const uint8_t* s = src + r0 * 64 + q * 16;
  uint8_t* da = dst + r0 * 128 + (((2 * q) ^ (r0 & 7)) << 4);
  uint8_t* db = dst + r0 * 128 + (((2 * q + 1) ^ (r0 & 7)) << 4);
#pragma unroll
  for (int j = 0; j < BM / RSTEP; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * RSTEP * 64);
    const uint4 lo = make_uint4((in.x << 4) & 0xF0F0F0F0u, (in.y << 4) & 0xF0F0F0F0u,
                                (in.z << 4) & 0xF0F0F0F0u, (in.w << 4) & 0xF0F0F0F0u);
    const uint4 hi = make_uint4(in.x & 0xF0F0F0F0u, in.y & 0xF0F0F0F0u, in.z & 0xF0F0F0F0u,
                                in.w & 0xF0F0F0F0u);
    *reinterpret_cast<uint4*>(da + j * RSTEP * 128) = lo;
    *reinterpret_cast<uint4*>(db + j * RSTEP * 128) = hi;
  }
}

// 4-bit activation rows (natural nibble order, 64 packed bytes per stage) -> int8 rows, the
// first `rows` rows (rounded up to a pass of the group).
__device__ __forceinline__ void convert_x_i8(const uint8_t* src, uint8_t* dst, int ctid, int rows) {
  constexpr int RSTEP = NCG / 4;
  const int r0 = ctid >> 2, q = ctid & 3;
  const uint8_t* s = src + r0 * 64 + q * 16;
  uint8_t* da = dst + r0 * 128 + (((2 * q) ^ (r0 & 7)) << 4);
  uint8_t* db = dst + r0 * 128 + (((2 * q + 1) ^ (r0 & 7)) << 4);
#pragma unroll 1
  for (int j = 0; j * RSTEP < rows; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * RSTEP * 64);
    uint4 a, b;
    nib8_to_i8x16(in.x, a.x, a.y);
    nib8_to_i8x16(in.y, a.z, a.w);
    nib8_to_i8x16(in.z, b.x, b.y);
    nib8_to_i8x16(in.w, b.z, b.w);
    *reinterpret_cast<uint4*>(da + j * RSTEP * 128) = a;
    *reinterpret_cast<uint4*>(db + j * RSTEP * 128) = b;
  }
}

// 2-bit activation rows (element e in bits 2e, 2e + 1 of a 32-bit word, two's complement; 32
// packed bytes = 128 codes per stage) -> int8 rows of 64 times the codes, swizzled as in
// convert_w_i8, the
// first `rows` rows (rounded up to a pass of the group). Thread ctid takes packed bytes
// 8q .. 8q + 7 (q = ctid & 3) of its rows: codes 32q .. 32q + 31, chunks 2q and 2q + 1.
__device__ __forceinline__ void pairs16_to_i8x64(uint32_t w, uint4& o) {
  // field i of every byte moved to that byte's top two bits: 64 times element 4j + i in byte j
  const uint32_t a0 = (w << 6) & 0xC0C0C0C0u, a1 = (w << 4) & 0xC0C0C0C0u;
  const uint32_t a2 = (w << 2) & 0xC0C0C0C0u, a3 = w & 0xC0C0C0C0u;
  const uint32_t l01 = __byte_perm(a0, a1, 0x5140), h01 = __byte_perm(a0, a1, 0x7362);
  const uint32_t l23 = __byte_perm(a2, a3, 0x5140), h23 = __byte_perm(a2, a3, 0x7362);
  o = make_uint4(__byte_perm(l01, l23, 0x5410), __byte_perm(l01, l23, 0x7632),
                 __byte_perm(h01, h23, 0x5410), __byte_perm(h01, h23, 0x7632));
}

__device__ __forceinline__ void convert_x2_i8(const uint8_t* src, uint8_t* dst, int ctid,
                                              int rows) {
  constexpr int RSTEP = NCG / 4;
  const int r0 = ctid >> 2, q = ctid & 3;
  const uint8_t* s = src + r0 * 32 + q * 8;
  uint8_t* da = dst + r0 * 128 + (((2 * q) ^ (r0 & 7)) << 4);
  uint8_t* db = dst + r0 * 128 + (((2 * q + 1) ^ (r0 & 7)) << 4);
#pragma unroll 1
  for (int j = 0; j * RSTEP < rows; ++j) {
    const uint2 in = *reinterpret_cast<const uint2*>(s + j * RSTEP * 32);
    uint4 a, b;
    pairs16_to_i8x64(in.x, a);
    pairs16_to_i8x64(in.y, b);
    *reinterpret_cast<uint4*>(da + j * RSTEP * 128) = a;
    *reinterpret_cast<uint4*>(db + j * RSTEP * 128) = b;
  }
}

// Half-precision lane pairs of 16 n from two bytes of a GEMM-layout word (bytes b0, b1 moved
// to the low byte of each 16-bit lane by prmt): the low nibble n gives the half
// 1024 + (n + 8) (n xor 8 is n + 8), scaled by 16 and shifted by FMA; the high nibble gives
// 1024 + 16 (n + 8) directly. Both results are exact.
__device__ __forceinline__ void w_pair_f16(uint32_t x, uint32_t& lo16, uint32_t& hi16) {
  const uint32_t l = (x & 0x000F000Fu) ^ 0x64086408u;
  const uint32_t h = (x & 0x00F000F0u) ^ 0x64806480u;
  const __half2 sixteen = __halves2half2(__ushort_as_half(0x4C00), __ushort_as_half(0x4C00));
  const __half2 off_l = __halves2half2(__ushort_as_half(0xF408), __ushort_as_half(0xF408));
  const __half2 off_h = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
  __half2 vl = __hfma2(*reinterpret_cast<const __half2*>(&l), sixteen, off_l);  // 16 v - 16512
  __half2 vh = __hsub2(*reinterpret_cast<const __half2*>(&h), off_h);           // v - 1152
  lo16 = *reinterpret_cast<uint32_t*>(&vl);
  hi16 = *reinterpret_cast<uint32_t*>(&vh);
}

// Weight rows in the GEMM layout (32 packed bytes = 64 elements per stage) -> fp16 rows of 128
// bytes (16 n), swizzled. Thread ctid takes packed group q = ctid & 1 of its rows: chunks
// 4q, 4q + 1 hold its low nibbles (elements 0-15 of the group), 4q + 2, 4q + 3 its high ones.
__device__ __forceinline__ void convert_w_f16(const uint8_t* src, uint8_t* dst, int ctid) {
  constexpr int RSTEP = NCG / 2;
  const int r0 = ctid >> 1, q = ctid & 1;
  const uint8_t* s = src + r0 * 32 + q * 16;
  uint8_t* d = dst + r0 * 128;
  const int ph = r0 & 7;
#pragma unroll
  for (int j = 0; j < BM / RSTEP; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * RSTEP * 32);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t P[4][2], Q[4][2];   // [word][byte pair]: low-nibble and high-nibble lanes
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      w_pair_f16(__byte_perm(w[m], 0u, 0x4140), P[m][0], Q[m][0]);
      w_pair_f16(__byte_perm(w[m], 0u, 0x4342), P[m][1], Q[m][1]);
    }
    uint8_t* row = d + j * RSTEP * 128;
    *reinterpret_cast<uint4*>(row + (((4 * q + 0) ^ ph) << 4)) =
        make_uint4(P[0][0], P[0][1], P[1][0], P[1][1]);
    *reinterpret_cast<uint4*>(row + (((4 * q + 1) ^ ph) << 4)) =
        make_uint4(P[2][0], P[2][1], P[3][0], P[3][1]);
    *reinterpret_cast<uint4*>(row + (((4 * q + 2) ^ ph) << 4)) =
        make_uint4(Q[0][0], Q[0][1], Q[1][0], Q[1][1]);
    *reinterpret_cast<uint4*>(row + (((4 * q + 3) ^ ph) << 4)) =
        make_uint4(Q[2][0], Q[2][1], Q[3][0], Q[3][1]);
  }
}

// Grouped asymmetric weights (CentriQ §4.3 and App. B.2): the stored nibble is n = Q - 8
// (two's complement), and row o of group g reconstructs as sigma (Q - z) = sigma n + m with
// m = -sigma (z - 8), the zero-point correction sigma z' taken into the operand. Both nibbles
// are first decoded exactly to n (1024 + (n + 8) - 1032; (1024 + 16 (n + 8)) / 16 - 72), then
// one fused multiply-add per lane pair rounds sigma n + m to fp16 once.
__device__ __forceinline__ void nib_pair_f16(uint32_t x, __half2& nl, __half2& nh) {
  const uint32_t l = (x & 0x000F000Fu) ^ 0x64086408u;
  const uint32_t h = (x & 0x00F000F0u) ^ 0x64806480u;
  const __half2 off_l = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
  const __half2 sixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
  const __half2 off_h = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
  nl = __hsub2(*reinterpret_cast<const __half2*>(&l), off_l);             // low nibbles
  nh = __hfma2(*reinterpret_cast<const __half2*>(&h), sixteenth, off_h);  // high nibbles
}

__device__ __forceinline__ void wg_pair_f16(uint32_t x, __half2 sg, __half2 mg, uint32_t& lo16,
                                            uint32_t& hi16) {
  __half2 nl, nh;
  nib_pair_f16(x, nl, nh);
  __half2 vl = __hfma2(nl, sg, mg);
  __half2 vh = __hfma2(nh, sg, mg);
  lo16 = *reinterpret_cast<uint32_t*>(&vl);
  hi16 = *reinterpret_cast<uint32_t*>(&vh);
}

// (sigma, z) word of one row and group -> the broadcast pairs (sigma, sigma) and (m, m),
// m = -sigma (z - 8) formed in fp32 (z - 8 exact) and rounded to fp16 once more.
__device__ __forceinline__ void group_consts(uint32_t sz, __half2& sg, __half2& mg) {
  const __half s = __ushort_as_half((unsigned short)(sz & 0xFFFFu));
  const __half z = __ushort_as_half((unsigned short)(sz >> 16));
  const float sf = __half2float(s);
  const float mf = sf * (8.f - __half2float(z));
  sg = __halves2half2(s, s);
  const __half m = __float2half_rn(mf);
  mg = __halves2half2(m, m);
}

// Grouped weight rows in the GEMM layout (one group of 64 per stage) -> fp16 rows of the real
// weights, swizzled as in convert_w_f16; sz0, sz1 are the (sigma, z) words of the thread's rows
// ctid / 2 and ctid / 2 + NCG / 2 for this group.
__device__ __forceinline__ void convert_wg_f16(const uint8_t* src, uint8_t* dst, int ctid,
                                               uint32_t sz0, uint32_t sz1) {
  constexpr int RSTEP = NCG / 2;
  static_assert(BM / RSTEP == 2, "two weight rows per converter thread");
  const int r0 = ctid >> 1, q = ctid & 1;
  const uint8_t* s = src + r0 * 32 + q * 16;
  uint8_t* d = dst + r0 * 128;
  const int ph = r0 & 7;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    __half2 sg, mg;
    group_consts(j == 0 ? sz0 : sz1, sg, mg);
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * RSTEP * 32);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t P[4][2], Q[4][2];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      wg_pair_f16(__byte_perm(w[m], 0u, 0x4140), sg, mg, P[m][0], Q[m][0]);
      wg_pair_f16(__byte_perm(w[m], 0u, 0x4342), sg, mg, P[m][1], Q[m][1]);
    }
    uint8_t* row = d + j * RSTEP * 128;
    *reinterpret_cast<uint4*>(row + (((4 * q + 0) ^ ph) << 4)) =
        make_uint4(P[0][0], P[0][1], P[1][0], P[1][1]);
    *reinterpret_cast<uint4*>(row + (((4 * q + 1) ^ ph) << 4)) =
        make_uint4(P[2][0], P[2][1], P[3][0], P[3][1]);
    *reinterpret_cast<uint4*>(row + (((4 * q + 2) ^ ph) << 4)) =
        make_uint4(Q[0][0], Q[0][1], Q[1][0], Q[1][1]);
    *reinterpret_cast<uint4*>(row + (((4 * q + 3) ^ ph) << 4)) =
        make_uint4(Q[2][0], Q[2][1], Q[3][0], Q[3][1]);
  }
}

// INT4 activation code rows (natural nibble order, 32 bytes = 64 codes per stage) -> fp16
// integer rows of 128 bytes, swizzled as in convert_lm_f16; the first `rows` rows (rounded up to
// a pass of the group). Bytes j, j + 1 of a word decode exactly as in nib_pair_f16 to the lane
// pairs (e_2j, e_2j+2) and (e_2j+1, e_2j+3), which are stored as they come: within every four
// consecutive K positions the operand holds elements 0, 2, 1, 3. The grouped weights are stored
// offline in the same K order, so the products pair up and the sum is unchanged.
__device__ __forceinline__ void convert_x4_f16(const uint8_t* src, uint8_t* dst, int ctid,
                                               int rows) {
  constexpr int RSTEP = NCG / 2;
  const int r0 = ctid >> 1, q = ctid & 1;
  const uint8_t* s = src + r0 * 32 + q * 16;
  uint8_t* d = dst + r0 * 128;
  const int ph = r0 & 7;
#pragma unroll 1
  for (int j = 0; j * RSTEP < rows; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * RSTEP * 32);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t o[4];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        __half2 nl, nh;
        nib_pair_f16(__byte_perm(w[k], 0u, hb ? 0x4342 : 0x4140), nl, nh);
        o[2 * hb] = *reinterpret_cast<uint32_t*>(&nl);
        o[2 * hb + 1] = *reinterpret_cast<uint32_t*>(&nh);
      }
      *reinterpret_cast<uint4*>(d + j * RSTEP * 128 + (((4 * q + k) ^ ph) << 4)) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Lloyd-Max code rows of 32 bytes (64 codes) -> fp16 centroid rows of 128 bytes, swizzled; the
// first `rows` rows (rounded up to a pass of the group).
__device__ __forceinline__ void convert_lm_f16(const uint8_t* src, uint8_t* dst, int ctid,
                                               const uint32_t (&lut)[8], int rows) {
  constexpr int RSTEP = NCG / 2;
  const int r0 = ctid >> 1, q = ctid & 1;
  const uint8_t* s = src + r0 * 32 + q * 16;
  uint8_t* d = dst + r0 * 128;
  const int ph = r0 & 7;
#pragma unroll 1
  for (int j = 0; j * RSTEP < rows; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * RSTEP * 32);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t o0, o1, o2, o3;
      lm4_to_f16(w[k] & 0xFFFFu, lut, o0, o1);
      lm4_to_f16(w[k] >> 16, lut, o2, o3);
      *reinterpret_cast<uint4*>(d + j * RSTEP * 128 + (((4 * q + k) ^ ph) << 4)) =
          make_uint4(o0, o1, o2, o3);
    }
  }
}

// 8-bit Lloyd-Max code rows (64 codes per stage) -> fp16 centroid rows of 128 bytes, swizzled,
// through a 256-entry table in shared memory; the first `rows` rows (rounded up to a pass).
// Thread ctid takes 16 codes (16-byte group q = ctid & 3) of its rows: chunks 2q and 2q + 1.
__device__ __forceinline__ void convert_lm8_f16(const uint8_t* src, uint8_t* dst, int ctid,
                                                const uint16_t* lut, int rows) {
  constexpr int RSTEP = NCG / 4;
  const int r0 = ctid >> 2, q = ctid & 3;
  const uint8_t* s = src + r0 * 64 + q * 16;
  uint8_t* da = dst + r0 * 128 + (((2 * q) ^ (r0 & 7)) << 4);
  uint8_t* db = dst + r0 * 128 + (((2 * q + 1) ^ (r0 & 7)) << 4);
#pragma unroll 1
  for (int j = 0; j * RSTEP < rows; ++j) {
    const uint4 in = *reinterpret_cast<const uint4*>(s + j * RSTEP * 64);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = (uint32_t)lut[w[k] & 0xFF] | ((uint32_t)lut[(w[k] >> 8) & 0xFF] << 16);
      o[2 * k + 1] = (uint32_t)lut[(w[k] >> 16) & 0xFF] | ((uint32_t)lut[w[k] >> 24] << 16);
    }
    *reinterpret_cast<uint4*>(da + j * RSTEP * 128) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(db + j * RSTEP * 128) = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// First K block of a tile. Tiles that run at the same time and share an activation range
// (neighbouring channel tiles) start their K loops at different blocks, so that they do not all
// request the same L2 lines at the same moment. Integer accumulation is exact in any order.
__device__ __forceinline__ int k_rotation(int m, int nkb) {
  return (int)(((unsigned)m * 7u) % (unsigned)nkb);
}

template <int KIND, int CG>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
           const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  using C = Cfg<KIND, CG>;
  constexpr int BK = C::BK, SX = C::SX, SP = C::SP, S2 = C::S2, MAXCH = C::MAXCH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float2* s_tok = reinterpret_cast<float2*>(smem + C::OFF_TOK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);  // tmem, abort, epi flag
  volatile uint32_t* s_abort = s_misc + 1;
  const uint16_t* s_lut8 = reinterpret_cast<const uint16_t*>(smem + C::OFF_LUT8);
  if constexpr (KIND == kGemmLloydMax8)
    for (int i = threadIdx.x; i < 128; i += blockDim.x)
      reinterpret_cast<uint32_t*>(smem + C::OFF_LUT8)[i] = p.lut8[i];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = (CG == 2) ? dev::cluster_ctarank() : 0u;  // 0 = the pair's leader
  constexpr int UNIT = BM * CG;                                    // channels per tile
  const int n_o = (p.N + UNIT - 1) / UNIT;
  const int nkb = (p.K + BK - 1) / BK;
  const int unit_index = (int)blockIdx.x / CG, n_units = (int)gridDim.x / CG;
  auto tiles = [&]() { return TileIter<MAXCH>(p.T, n_o, unit_index, n_units); };

  auto bar = [&](int i) { return dev::smem_u32(&bars[i]); };
  auto xfull_bar = [&](int s) { return bar(s); };
  auto xempty_bar = [&](int s) { return bar(SX + s); };
  auto pfull_bar = [&](int s) { return bar(2 * SX + s); };
  auto pempty_bar = [&](int s) { return bar(2 * SX + SP + s); };
  auto wready_bar = [&](int c) { return bar(2 * SX + 2 * SP + c); };
  auto wfree_bar = [&](int c) { return bar(2 * SX + 2 * SP + S2 + c); };
  auto tfull_bar = [&](int b) { return bar(2 * SX + 2 * SP + 2 * S2 + b); };
  auto tempty_bar = [&](int b) { return bar(2 * SX + 2 * SP + 2 * S2 + 2 + b); };
  const uint32_t drain_bar = bar(2 * SX + 2 * SP + 2 * S2 + 4);
  auto x_stage = [&](int s) { return smem + C::OFF_X + s * C::XT; };
  auto p_stage = [&](int s) { return smem + C::OFF_P + s * C::P_STAGE; };
  auto conv_stage = [&](int c) { return smem + C::OFF_CONV + c * C::CONV_STAGE; };
  // the leader's copy of one of this CTA's barriers, as a cluster address
  auto lead = [&](uint32_t a) { return CG == 2 ? dev::map_to_cta(a, 0) : a; };
  // arrive on the leader's copy of a barrier (a plain local arrive when CG = 1)
  auto arrive_lead = [&](uint32_t a) {
    if constexpr (CG == 2)
      dev::mbar_arrive_cluster(lead(a));
    else
      dev::mbar_arrive(a);
  };

  if (tid == 0) {
    for (int s = 0; s < SX; ++s) {
      dev::mbar_init(xfull_bar(s), 1);
      dev::mbar_init(xempty_bar(s), 1);
    }
    for (int s = 0; s < SP; ++s) {
      dev::mbar_init(pfull_bar(s), 1);
      dev::mbar_init(pempty_bar(s), NCG / 32);   // one arrive per converter warp
    }
    for (int c = 0; c < S2; ++c) {
      dev::mbar_init(wready_bar(c), CG * (NCG / 32));   // one arrive per converter warp
      dev::mbar_init(wfree_bar(c), 1);
    }
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(tfull_bar(b), 1);
      dev::mbar_init(tempty_bar(b), CG * (NEPI / 32));  // one arrive per epilogue warp
    }
    dev::mbar_init(drain_bar, 1);
    s_misc[1] = 0;
    if constexpr (CG == 2)
      dev::fence_mbar_init_cluster();
    else
      dev::fence_mbar_init();
  }
  // Warp roles. A warp's scheduler is warp % 4. With INT8 activations (light unpacking) the
  // single MMA thread (warp 1) shares its scheduler only with the two TMA producers (warps 5
  // and 9) and the two epilogue warps that must read TMEM lane quarter 1, while the eight
  // converter warps (0, 2-4, 6-8, 10) use the other three schedulers. The 4-bit kinds unpack
  // both operands and keep their converters (warps 3-10) on all four schedulers.
  constexpr bool MMA_ALONE = KIND == kGemmA8;
  constexpr int W_MMA = 1, W_PROD_P = MMA_ALONE ? 5 : 0, W_PROD_X = MMA_ALONE ? 9 : 2;
  constexpr int W_EPI0 = EPI0 / 32;
  const bool is_conv = warp < W_EPI0 && warp != W_MMA && warp != W_PROD_P && warp != W_PROD_X;
  const int conv_idx = warp - (warp > W_MMA) - (warp > W_PROD_P) - (warp > W_PROD_X);
  if (warp == W_PROD_P && lane == 0) {
    dev::prefetch_tmap(&tm_x);
    dev::prefetch_tmap(&tm_w);
  }
  if (warp == W_EPI0 && lane == 0 && !p.out_acc) dev::prefetch_tmap(&tm_y);
  if (warp == 1) {
    if constexpr (CG == 2) {
      dev::tmem_alloc_pair(dev::smem_u32(&s_misc[0]), 2 * C::BNMAX);
      dev::tmem_relinquish_pair();
    } else {
      dev::tmem_alloc(dev::smem_u32(&s_misc[0]), 2 * C::BNMAX);
      dev::tmem_relinquish();
    }
  }
  dev::tc_fence_before();
  if constexpr (CG == 2)
    dev::cluster_sync();  // barrier inits of both CTAs visible before any remote arrive
  else
    __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = s_misc[0];

  auto give_up = [&]() { *s_abort = 1; };

  if (warp == W_PROD_P || warp == W_PROD_X) {
    // ---------------- producers ----------------
    // W_PROD_P: packed ring (W, and X for 4-bit activations); W_PROD_X: INT8 activation ring
    const bool packed_role = warp == W_PROD_P;
    if (lane == 0 && (packed_role || SX > 0)) {
      const int ns = packed_role ? SP : SX;
      uint32_t j = 0;
      bool ok = true;
      auto it = tiles();
      int m, t0, nch;
      while (ok && it.next(m, t0, nch)) {
        const int o0 = m * UNIT + (int)rank * BM;          // this CTA's weight rows
        // this CTA's activation rows start at x0; one box brings XR rows (a narrower last
        // tile reads rows past it, or past T as zeros, that its MMAs do not use)
        const int x0 = t0 + (int)rank * (nch * CH / CG);
        const int krot = k_rotation(m, nkb);
        for (int step = 0; step < nkb; ++step, ++j) {
          const int kb = (step + krot) % nkb;
          const int s = j % ns;
          const uint32_t empty_b = packed_role ? pempty_bar(s) : xempty_bar(s);
          const uint32_t full_b = packed_role ? pfull_bar(s) : xfull_bar(s);
          if (*s_abort || !dev::mbar_wait(empty_b, ((j / ns) & 1u) ^ 1u, p.err, kSiteGemmEmpty,
                                          p.limit_ns)) {
            give_up();
            ok = false;
            break;
          }
          if (packed_role) {
            uint8_t* st = p_stage(s);
            dev::mbar_arrive_expect_tx(full_b, (uint32_t)C::P_STAGE);
            dev::tma_load_2d(dev::smem_u32(st + C::XP), &tm_w, kb * (BK / 2), o0, full_b);
            if constexpr (C::XPACK)
              dev::tma_load_2d(dev::smem_u32(st), &tm_x, kb * C::XB, x0, full_b);
          } else if constexpr (CG == 2) {
            // both halves complete on the leader's barrier, which expects the bytes of both
            if (rank == 0) dev::mbar_arrive_expect_tx(full_b, (uint32_t)(2 * C::XT));
            dev::tma_load_2d_pair(dev::smem_u32(x_stage(s)), &tm_x, kb * BK, x0, lead(full_b));
          } else {
            dev::mbar_arrive_expect_tx(full_b, (uint32_t)C::XT);
            dev::tma_load_2d(dev::smem_u32(x_stage(s)), &tm_x, kb * BK, x0, full_b);
          }
        }
      }
      // let the loads already issued land before the block can exit (activation loads of a
      // pair complete on the leader's barriers, so only the leader can watch them)
      if (!ok && (packed_role || rank == 0)) {
        for (uint32_t i = (j >= (uint32_t)ns ? j - ns : 0); i < j; ++i)
          dev::mbar_wait(packed_role ? pfull_bar(i % ns) : xfull_bar(i % ns), (i / ns) & 1u, p.err,
                         kSiteGemmDrain, p.limit_ns);
      }
    }
  } else if (warp == W_MMA) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && rank == 0) {
      auto commit = [&](uint32_t bar) {
        if constexpr (CG == 2)
          dev::mma_commit_pair(bar);
        else
          dev::mma_commit(bar);
      };
      uint32_t j = 0, it_n = 0;
      bool ok = true, issued = false;
      auto it = tiles();
      int m, t0, nch;
      for (; ok && it.next(m, t0, nch); ++it_n) {
        const uint32_t idesc = C::FP ? dev::idesc_f16(UNIT, nch * CH)
                                                       : dev::idesc_i8(UNIT, nch * CH);
        const int b = it_n & 1;
        if (*s_abort || !dev::mbar_wait(tempty_bar(b), ((it_n >> 1) & 1u) ^ 1u, p.err,
                                        kSiteGemmAccum, p.limit_ns)) {
          give_up();
          ok = false;
          break;
        }
        dev::tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(b * C::BNMAX);
        for (int step = 0; step < nkb; ++step, ++j) {
          const int c = j % S2;
          const int sx = SX > 0 ? (int)(j % (uint32_t)(SX > 0 ? SX : 1)) : 0;
          bool w = !*s_abort &&
                   dev::mbar_wait(wready_bar(c), (j / S2) & 1u, p.err, kSiteGemmConv, p.limit_ns);
          if constexpr (!C::XPACK) {
            if (w)
              w = dev::mbar_wait(xfull_bar(sx), (j / SX) & 1u, p.err, kSiteGemmFull, p.limit_ns);
          }
          if (!w) {
            give_up();
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t aw = dev::smem_u32(conv_stage(c));
          const uint32_t bx = C::XPACK ? dev::smem_u32(conv_stage(c) + C::WT)
                                       : dev::smem_u32(x_stage(sx));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = dev::sdesc_sw128(aw + kk * 32);
            const uint64_t bd = dev::sdesc_sw128(bx + kk * 32);
            if constexpr (CG == 2) {
              if constexpr (C::FP)
                dev::mma_f16_pair(dt, ad, bd, idesc, (step | kk) != 0);
              else
                dev::mma_i8_pair(dt, ad, bd, idesc, (step | kk) != 0);
            } else {
              if constexpr (C::FP)
                dev::mma_f16(dt, ad, bd, idesc, (step | kk) != 0);
              else
                dev::mma_i8(dt, ad, bd, idesc, (step | kk) != 0);
            }
          }
          issued = true;
          commit(wfree_bar(c));
          if constexpr (!C::XPACK) commit(xempty_bar(sx));
        }
        if (!ok) break;
        commit(tfull_bar(b));
      }
      if (!ok && issued) {  // wait for the MMAs in flight before TMEM is freed
        commit(drain_bar);
        dev::mbar_wait(drain_bar, 0, p.err, kSiteGemmDrain, p.limit_ns);
      }
    }
  } else if (is_conv) {
    // ---------------- converters ----------------
    const int cid = conv_idx * 32 + lane;   // 0 .. NCONV - 1
    const int grp = cid / NCG, ctid = cid % NCG;
    uint32_t lut[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) lut[i] = p.lut[i];
    uint32_t j = 0;
    bool ok = true;
    auto it = tiles();
    int m, t0, nch;
    while (ok && it.next(m, t0, nch)) {
      const int rows = nch * CH / CG;   // activation rows of this CTA
      const int krot = k_rotation(m, nkb);
      for (int step = 0; step < nkb; ++step, ++j) {
        if ((int)(j % NGROUP) != grp) continue;
        const int s = j % SP, c = j % S2;
        uint32_t sz0 = 0u, sz1 = 0u;   // grouped weights: this k block's (sigma, z) words
        if constexpr (KIND == kGemmG64) {
          const int kb = (step + krot) % nkb;
          const int o = m * UNIT + (int)rank * BM + (ctid >> 1);
          const uint32_t* src = p.w_sz + (size_t)kb * (size_t)p.N;
          if (o < p.N) sz0 = __ldg(src + o);
          if (o + NCG / 2 < p.N) sz1 = __ldg(src + o + NCG / 2);
        }
        bool w = !*s_abort &&
                 dev::mbar_wait(pfull_bar(s), (j / SP) & 1u, p.err, kSiteGemmFull, p.limit_ns);
        if (w)
          w = dev::mbar_wait(wfree_bar(c), ((j / S2) & 1u) ^ 1u, p.err, kSiteGemmConv,
                             p.limit_ns);
        w = __all_sync(0xffffffffu, w);  // one verdict per warp: its lanes meet in __syncwarp
        if (!w) {
          give_up();
          ok = false;
          break;
        }
        const uint8_t* st = p_stage(s);
        uint8_t* cv = conv_stage(c);
        if constexpr (KIND == kGemmLloydMax) {
          convert_w_f16(st + C::XP, cv, ctid);
          convert_lm_f16(st, cv + C::WT, ctid, lut, rows);
        } else if constexpr (KIND == kGemmG64) {
          convert_wg_f16(st + C::XP, cv, ctid, sz0, sz1);
          convert_x4_f16(st, cv + C::WT, ctid, rows);
        } else if constexpr (KIND == kGemmLloydMax8) {
          convert_w_f16(st + C::XP, cv, ctid);
          convert_lm8_f16(st, cv + C::WT, ctid, s_lut8, rows);
        } else {
          convert_w_i8(st + C::XP, cv, ctid);
          if constexpr (KIND == kGemmA4) convert_x_i8(st, cv + C::WT, ctid, rows);
          if constexpr (KIND == kGemmA2) convert_x2_i8(st, cv + C::WT, ctid, rows);
        }
        dev::fence_async_smem();  // this thread's tiles -> visible to the tensor cores
        __syncwarp();             // the warp's reads of the packed stage and writes are done
        if (lane == 0) {
          dev::mbar_arrive(pempty_bar(s));
          arrive_lead(wready_bar(c));
        }
      }
    }
  } else {
    // ---------------- epilogue ----------------
    // Thread (lane quarter q, lane) owns output channel o; a 32-column TMEM load gives it 32
    // consecutive tokens of that channel. For each token the 32 lanes of a warp store 32
    // consecutive channels, i.e. 64 (bf16) or 128 (raw accumulator) contiguous bytes. The
    // EPW warps of a lane quarter take the tile's 32-column chunks in turn.
    const int etid = tid - EPI0;         // 0..NEPI-1
    uint8_t* stg = smem + C::OFF_STG + (warp - W_EPI0) * C::STG;
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const int half = etid >> 7;          // index among the warps of the quarter
    const int o_local = q * 32 + lane;
    const bool ep_lead = etid == 0;
    uint32_t it_n = 0;
    bool ok = true;
    auto it = tiles();
    int m, t0, nch;
    for (; ok && it.next(m, t0, nch); ++it_n) {
      const int o0 = m * UNIT + (int)rank * BM;
      const int b = it_n & 1;
      const int o = o0 + o_local;
      const bool has_o = o < p.N;
      const float sw = has_o ? p.w_scale[o] * C::ACC_SCALE : 0.f;
      const float w1 = (has_o && p.mean) ? p.w_rowsum[o] : 0.f;
      const float bb = (has_o && p.bias) ? __bfloat162float(p.bias[o]) : 0.f;
      const int ncols = nch * CH;
      for (int i = etid; i < ncols; i += NEPI) {
        const int t = t0 + i;
        s_tok[i] = make_float2((t < p.T) ? p.a_scale[t] : 0.f,
                               (t < p.T && p.mean) ? p.mean[t] : 0.f);
      }
      // one thread waits for the accumulator; the verdict reaches all epilogue warps through
      // shared memory behind a named barrier, so every later barrier is reached uniformly
      if (ep_lead) {
        const bool ready = !*s_abort && dev::mbar_wait(tfull_bar(b), (it_n >> 1) & 1u, p.err,
                                                       kSiteGemmAccum, p.limit_ns);
        if (!ready) give_up();
        s_misc[2] = ready ? 1u : 0u;
      }
      dev::named_bar(1, NEPI);
      ok = *reinterpret_cast<volatile uint32_t*>(&s_misc[2]) != 0;
      if (ok) dev::tc_fence_after();
      const int t_end = min(ncols, p.T - t0);   // tokens of this tile inside [0, T)
      const int nmine = (nch - half + EPW - 1) / EPW;   // chunks half, half + EPW, ...
      if (ok && nmine == 0) {
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_lead(tempty_bar(b));
      }
#pragma unroll 1
      for (int cc = 0; ok && cc < nmine; ++cc) {
        const int c = half + cc * EPW;   // 32-column chunk of the tile
        uint32_t r[32];
        dev::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::BNMAX + c * 32), r);
        dev::tmem_wait_ld();
        if (cc == nmine - 1) {  // this warp's part of the accumulator is read
          dev::tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_lead(tempty_bar(b));
        }
        if (o0 + q * 32 >= p.N) continue;    // this warp's channels all lie past N
        const int n_valid = t_end - c * 32;   // tokens of this chunk inside [0, T)
        if (p.out_acc) {
          if constexpr (C::FP) {
            float* dst = reinterpret_cast<float*>(p.out) + (int64_t)(t0 + c * 32) * p.N + o;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (has_o && jj < n_valid) dst[(int64_t)jj * p.N] = __uint_as_float(r[jj]) * C::ACC_SCALE;
          } else {
            int32_t* dst = reinterpret_cast<int32_t*>(p.out) + (int64_t)(t0 + c * 32) * p.N + o;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (has_o && jj < n_valid) dst[(int64_t)jj * p.N] = (int32_t)r[jj] >> C::ACC_SHIFT;
          }
        } else {
          // two tokens at a time as f32x2: y = acc * (alpha_t s_w) + (mean_t w_1 + b), into
          // this warp's staging tile [32 tokens][32 channels]; one TMA store writes the tile
          // (the store clips tokens past T and channels past N)
          const float4* tk4 = reinterpret_cast<const float4*>(s_tok + c * 32);
          const float2 sw2 = make_float2(sw, sw), w12 = make_float2(w1, w1);
          const float2 bb2 = make_float2(bb, bb);
          uint32_t yb[16];
#pragma unroll
          for (int jj = 0; jj < 32; jj += 2) {
            const float4 tk = tk4[jj / 2];    // (alpha, mean) of tokens jj and jj + 1
            const float2 s2 = __fmul2_rn(make_float2(tk.x, tk.z), sw2);
            const float2 c2 = __ffma2_rn(make_float2(tk.y, tk.w), w12, bb2);
            const float2 a2 = C::FP
                                  ? make_float2(__uint_as_float(r[jj]), __uint_as_float(r[jj + 1]))
                                  : make_float2((float)(int32_t)r[jj], (float)(int32_t)r[jj + 1]);
            const __nv_bfloat162 y = __float22bfloat162_rn(__ffma2_rn(a2, s2, c2));
            yb[jj / 2] = *reinterpret_cast<const uint32_t*>(&y);
          }
          if (lane == 0) dev::bulk_wait_all_read();   // the previous store has read the tile
          __syncwarp();
#pragma unroll
          for (int jj = 0; jj < 32; jj += 2) {
            *reinterpret_cast<uint16_t*>(stg + jj * 64 + lane * 2) = (uint16_t)(yb[jj / 2] & 0xFFFFu);
            *reinterpret_cast<uint16_t*>(stg + (jj + 1) * 64 + lane * 2) = (uint16_t)(yb[jj / 2] >> 16);
          }
          dev::fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            dev::tma_store_2d(&tm_y, dev::smem_u32(stg), o0 + q * 32, t0 + c * 32);
            dev::bulk_commit();
          }
        }
      }
      dev::named_bar(1, NEPI);  // s_tok of this tile is no longer read
    }
    if (lane == 0) dev::bulk_wait_all();   // this warp's output stores are complete
  }

  dev::tc_fence_before();
  if constexpr (CG == 2)
    dev::cluster_sync();  // no MMA, remote arrive or TMEM read of either CTA is still pending
  else
    __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    if constexpr (CG == 2)
      dev::tmem_dealloc_pair(tmem, 2 * C::BNMAX);
    else
      dev::tmem_dealloc(tmem, 2 * C::BNMAX);
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

// Clusters of two CTAs that can be resident at once for a kernel and its shared memory (0 if
// the query fails), computed once per kernel and device.
int active_pairs_n(const void* kern, size_t smem, int nthreads) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({kern, dev});
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * (unsigned)sm_count());
  cfg.blockDim = dim3((unsigned)nthreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[{kern, dev}] = n;
  return n;
}

int active_pairs(const void* kern, size_t smem) { return active_pairs_n(kern, smem, NTHREADS); }

template <int KIND, int CG>
oq_status run(const GemmArgs& g, const GemmParams& p, cudaStream_t s) {
  using C = Cfg<KIND, CG>;
  constexpr int BK = C::BK;
  CUtensorMap tx, tw, ty;
  bool ok = true;
  if (!g.out_acc)
    ok &= make_map_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.out, (uint64_t)g.N, (uint64_t)g.T,
                      (uint64_t)g.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    std::memset(&ty, 0, sizeof(ty));
  if constexpr (C::XPACK) {
    const uint64_t xrow = (uint64_t)g.K * C::XB / BK;   // activation bytes per token
    ok &= make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, xrow, (uint64_t)g.T, xrow, C::XB,
                      C::XR, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  else
    ok &= make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, (uint64_t)g.K, (uint64_t)g.T,
                      (uint64_t)g.K, BK, C::XR, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.w, (uint64_t)g.K / 2, (uint64_t)g.N,
                    (uint64_t)g.K / 2, BK / 2, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return fail(OQ_ERR_CUDA, "cuTensorMapEncodeTiled failed or unavailable");

  auto kern = &k_gemm<KIND, CG>;
  const cudaError_t attr_err = allow_max_dynamic_smem(reinterpret_cast<const void*>(kern));
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(gemm)");
  // tiles of 128 * CG tokens of one channel tile; no more CTAs (pairs) than tiles
  const int64_t tiles = ((g.N + BM * CG - 1) / (BM * CG)) * ((g.T + 128 * CG - 1) / (128 * CG));
  if constexpr (CG == 1) {
    const int grid = (int)std::min<int64_t>(tiles, sm_count());
    kern<<<grid, NTHREADS, C::SMEM, s>>>(tx, tw, ty, p);
  } else {
    const int pairs = active_pairs(reinterpret_cast<const void*>(kern), C::SMEM);
    if (pairs <= 0) return fail(OQ_ERR_UNSUPPORTED, "gemm: no CTA pair fits on this device");
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(2 * std::min<int64_t>(tiles, pairs)));
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, tx, tw, ty, p);
    if (le != cudaSuccess) return cuda_fail(le, "launch gemm (CTA pairs)");
  }
  cudaError_t ce = cudaGetLastError();
  if (ce != cudaSuccess) return cuda_fail(ce, "launch gemm");
  return OQ_OK;
}

// ---- balanced schedule of the CTA-pair GEMM -----------------------------------------------------
namespace ta {
constexpr int MAXCH = 256 / CH;      // 32-token chunks per tile at most

// The tiles of one CTA pair: its range [sched[u], sched[u + 1]) of the flattened (channel tile,
// chunk) space, cut at channel tile boundaries and into as-even-as-possible tiles of at most
// MAXCH chunks. Every role of the pair walks the same sequence.
struct RangeIter {
  int cpm, cur, end;
  __device__ RangeIter(int T, const int* sched, int unit) {
    cpm = (T + CH - 1) / CH;
    cur = sched[unit];
    end = sched[unit + 1];
  }
  __device__ bool next(int& m, int& t0, int& nch) {
    if (cur >= end) return false;
    m = cur / cpm;
    const int tc = cur - m * cpm;
    const int run = min(end, (m + 1) * cpm) - cur;     // chunks left in this channel tile
    const int ntiles = (run + MAXCH - 1) / MAXCH;
    nch = (run + ntiles - 1) / ntiles;
    t0 = tc * CH;
    cur += nch;
    return true;
  }
};
}  // namespace ta

// ================================================================================================
// W4A8 with the widened weights in shared memory and double-buffered accumulators (CTA pairs,
// T > 128). The variant the W4A8 layer runs.
//
// The converter warps load the packed INT4 weights of each 128-byte K block straight from L2
// (the prepared weights stay L2-resident) into registers, widen them to the int8 16 n and store
// them into a stage of widened weights in the 128-byte-swizzled K-major layout the MMA reads.
// There is no shared-memory ring of packed weights: its space goes to deeper rings. The loads
// of a K block are issued before the converter waits for its stage to be free, and that wait
// (the converters run ahead of the MMA) hides the L2 latency.
//
// Pipeline depth. The completion of an MMA reaches an mbarrier (tcgen05.commit) several hundred
// nanoseconds after the tensor pipe finishes it, and a stage is refilled only after that
// arrive. SK = 3 stages of two 128-byte K blocks of widened weights and activations (1.7 us of
// MMA work at N = 256) keep the pipe fed. The single MMA thread pays a fixed cost per stage
// (its wait, fence and commit), so a stage carries two K blocks: eight MMAs per wait. TMEM
// holds two accumulators of 256 columns, so the epilogue of one tile overlaps the next tile's
// MMAs.
//
// Schedule: every CTA pair takes a contiguous range of the (channel tile, 32-token chunk) space,
// cut into tiles of at most 256 tokens; the host chooses the ranges so that the largest
// per-pair cost (chunks plus a fixed cost per tile) is as small as possible (balance_ranges).
//
// Warps: 1 TMEM owner + MMA issuer, 5 activation producer, eight converters in two groups of
// four that take every other stage (two stages convert at once: a conversion is bound by the
// latency of its L2 loads, the stores and the hand-off, not by its work), 12-19 epilogue (two
// per TMEM lane quarter), 9 and 11 idle.
// A warp's scheduler is warp % 4: the single MMA thread shares its scheduler only with the
// producer and the two epilogue warps of lane quarter 1; the converters (warps 0, 2-4, 6-8, 10)
// use the other three schedulers, so that their work never delays an MMA issue.
namespace sa {
constexpr int BN = 256;              // tokens per tile at most (MMA N)
constexpr int XR = BN / 2;           // activation rows per CTA and stage
constexpr int KSUB = 2;              // 128-byte K blocks per stage
constexpr int SK = 3;                // stages: widened weights and activations
constexpr int WT = BM * 128;         // widened weight bytes of one K block
constexpr int XT = XR * 128;         // activation bytes of one K block (this CTA's rows)
constexpr int WS = KSUB * WT, XS = KSUB * XT;   // stage bytes
constexpr int TCOLS = 2 * BN;        // two accumulators
constexpr int STG = 32 * 32 * 2;     // bf16 [32 tokens][32 channels] staging tile per warp
constexpr int OFF_W = 0;
constexpr int OFF_X = OFF_W + SK * WS;
constexpr int OFF_STG = OFF_X + SK * XS;
constexpr int OFF_TOK = OFF_STG + (NEPI / 32) * STG;
constexpr int OFF_BAR = OFF_TOK + BN * 8;
constexpr int NBAR = 2 * SK + 4 + 1;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM = OFF_MISC + 16 + 1024;
constexpr int NTHR = 640;
constexpr int W_PROD_X = 5, W_MMA = 1, W_EPI0 = 12;
constexpr int CONV_GROUPS = 2;       // converter groups (of four warps); group g takes stages g mod 2
// converter index (0..7) of a warp, -1 for the other roles
__device__ __forceinline__ int conv_index(int w) {
  switch (w) {
    case 0: return 0; case 2: return 1; case 3: return 2; case 4: return 3;
    case 6: return 4; case 7: return 5; case 8: return 6; case 10: return 7;
    default: return -1;
  }
}
static_assert(WT % 1024 == 0 && XT % 1024 == 0 && OFF_X % 1024 == 0, "stage alignment");
static_assert(SMEM <= 232448, "shared memory");
static_assert(NTHR == (W_EPI0 * 32 + NEPI), "warp roles");
}  // namespace sa

// A walk over one CTA pair's K blocks in the order every role processes them.
struct KWalk {
  ta::RangeIter rit;
  int m = 0, t0 = 0, nch = 0, step = 0, nkb;
  bool live;
  __device__ KWalk(int T, const int* sched, int unit, int nkb_)
      : rit(T, sched, unit), nkb(nkb_) {
    live = rit.next(m, t0, nch);
  }
  __device__ void advance() {
    if (live && ++step == nkb) {
      step = 0;
      live = rit.next(m, t0, nch);
    }
  }
};

__global__ void __launch_bounds__(sa::NTHR, 1)
    k_gemm_a8s(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
               const uint8_t* __restrict__ wpk, const GemmParams p) {
  using namespace sa;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float2* s_tok = reinterpret_cast<float2*>(smem + OFF_TOK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(smem + OFF_MISC);  // tmem, abort, epi flag
  volatile uint32_t* s_abort = s_misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = dev::cluster_ctarank();   // 0 = the pair's leader
  constexpr int UNIT = 2 * BM;                     // channels per tile
  const int nkb = (p.K + 127) / 128;
  const int nst = (nkb + KSUB - 1) / KSUB;        // stages per tile (a K loop)
  const int unit_index = (int)blockIdx.x / 2;
  auto tiles = [&]() { return ta::RangeIter(p.T, p.sched, unit_index); };

  // ready[s]: stage s is in place, i.e. both activation halves of its K blocks landed (TMA
  // bytes on the leader's barrier, armed by the leader's producer) and the converter warps of
  // both CTAs stored its widened weights: one wait per stage for the MMA thread
  auto bar = [&](int i) { return dev::smem_u32(&bars[i]); };
  auto ready_bar = [&](int s) { return bar(s); };
  auto kfree_bar = [&](int s) { return bar(SK + s); };        // stage s consumed by the MMAs
  auto tfull_bar = [&](int b) { return bar(2 * SK + b); };
  auto tempty_bar = [&](int b) { return bar(2 * SK + 2 + b); };
  const uint32_t drain_bar = bar(2 * SK + 4);
  auto w_stage = [&](int s) { return smem + OFF_W + s * WS; };
  auto x_stage = [&](int s) { return smem + OFF_X + s * XS; };
  auto lead = [&](uint32_t a) { return dev::map_to_cta(a, 0); };

  if (tid == 0) {
    for (int s = 0; s < SK; ++s) {
      // the leader's producer + the converter warps of a group in each CTA
      dev::mbar_init(ready_bar(s), 1 + 2 * (8 / CONV_GROUPS));
      dev::mbar_init(kfree_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(tfull_bar(b), 1);
      dev::mbar_init(tempty_bar(b), 2 * (NEPI / 32));
    }
    dev::mbar_init(drain_bar, 1);
    s_misc[1] = 0;
    dev::fence_mbar_init_cluster();
  }
  if (warp == W_PROD_X && lane == 0) dev::prefetch_tmap(&tm_x);
  if (warp == W_EPI0 && lane == 0 && !p.out_acc) dev::prefetch_tmap(&tm_y);
  if (warp == W_MMA) {
    dev::tmem_alloc_pair(dev::smem_u32(&s_misc[0]), TCOLS);
    dev::tmem_relinquish_pair();
  }
  dev::tc_fence_before();
  dev::cluster_sync();   // barrier inits of both CTAs visible before any remote arrive
  dev::tc_fence_after();
  const uint32_t tmem = s_misc[0];
  auto give_up = [&]() { *s_abort = 1; };

  if (warp == W_PROD_X) {
    // ---------------- activation producer ----------------
    if (lane == 0) {
      uint32_t j = 0;
      bool ok = true;
      auto it = tiles();
      int m, t0, nch;
      while (ok && it.next(m, t0, nch)) {
        const int x0 = t0 + (int)rank * (nch * CH / 2);      // this CTA's activation rows
        const int krot = k_rotation(m, nst);
        for (int step = 0; step < nst; ++step, ++j) {
          const int kb0 = ((step + krot) % nst) * KSUB;        // first K block of the stage
          const int s = j % SK;
          if (!dev::mbar_wait(kfree_bar(s), ((j / SK) & 1u) ^ 1u, p.err, kSiteGemmEmpty,
                              p.limit_ns) || *s_abort) {
            give_up();
            ok = false;
            break;
          }
          // both halves complete on the leader's barrier, which expects the bytes of both; a K
          // block past the end of K (an odd count) lands as zeros and still counts its bytes
          if (rank == 0) dev::mbar_arrive_expect_tx(ready_bar(s), (uint32_t)(2 * XS));
#pragma unroll
          for (int u = 0; u < KSUB; ++u)
            dev::tma_load_2d_pair(dev::smem_u32(x_stage(s) + u * XT), &tm_x, (kb0 + u) * 128, x0,
                                  lead(ready_bar(s)));
        }
      }
      // after an abort the landed bytes of the loads in flight can no longer be told apart from
      // the converters' arrivals: wait (bounded) for the stages' completions, which also covers
      // the bytes; a stage whose converter arrivals never come gives up at the time limit
      if (!ok && rank == 0) {
        for (uint32_t i = (j >= (uint32_t)SK ? j - SK : 0); i < j; ++i)
          dev::mbar_wait(ready_bar(i % SK), (i / SK) & 1u, p.err, kSiteGemmDrain, p.limit_ns);
      }
    }
  } else if (warp == W_MMA) {
    // ---------------- MMA issuer (the leader's lane 0) ----------------
    if (lane == 0 && rank == 0) {
      uint32_t j = 0, it_n = 0;
      bool ok = true, issued = false;
      auto it = tiles();
      int m, t0, nch;
      for (; ok && it.next(m, t0, nch); ++it_n) {
        const uint32_t idesc = dev::idesc_i8(UNIT, nch * CH);
        const int b = it_n & 1;
        if (!dev::mbar_wait(tempty_bar(b), ((it_n >> 1) & 1u) ^ 1u, p.err, kSiteGemmAccum,
                            p.limit_ns) || *s_abort) {
          give_up();
          ok = false;
          break;
        }
        dev::tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(b * BN);
        // one wait, one fence and one commit per stage of KSUB K blocks (4 KSUB MMAs): the
        // single issuing thread's fixed cost per wait is what sets the pace, not the tensor pipe
        const int krot = k_rotation(m, nst);
        for (int step = 0; step < nst; ++step, ++j) {
          const int c = j % SK;
          const int kb0 = ((step + krot) % nst) * KSUB;
          if (!dev::mbar_wait(ready_bar(c), (j / SK) & 1u, p.err, kSiteGemmFull, p.limit_ns)) {
            give_up();
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t aw = dev::smem_u32(w_stage(c)), bx = dev::smem_u32(x_stage(c));
#pragma unroll
          for (int u = 0; u < KSUB; ++u) {
            if (kb0 + u >= nkb) break;   // past the end of K: zeros, nothing to add
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              dev::mma_i8_pair(dt, dev::sdesc_sw128(aw + u * WT + kk * 32),
                               dev::sdesc_sw128(bx + u * XT + kk * 32), idesc,
                               (step | u | kk) != 0);
          }
          issued = true;
          dev::mma_commit_pair(kfree_bar(c));
        }
        if (!ok) break;
        dev::mma_commit_pair(tfull_bar(b));
      }
      if (!ok && issued) {  // wait for the MMAs in flight before TMEM is freed
        dev::mma_commit_pair(drain_bar);
        dev::mbar_wait(drain_bar, 0, p.err, kSiteGemmDrain, p.limit_ns);
      }
    }
  } else if (conv_index(warp) >= 0) {
    // ---------------- converters: packed weights (L2) -> int8 16 n -> shared memory -------
    // Group g (four warps) takes the stages j = g, g + CONV_GROUPS, ... Thread ctid of a group
    // takes 16-byte packed group q = ctid & 3 of rows r0 + 32 i (r0 = ctid >> 2, i = 0..3) in
    // each K block of the stage: its low nibbles become chunk 2q and its high nibbles chunk
    // 2q + 1 of the row's 128 widened bytes, stored at chunk index ^ (row & 7) (the 128-byte
    // swizzle), the same for every i. All loads of the stage are issued before the wait for a
    // free stage.
    constexpr int NCG_A = 32 * (8 / CONV_GROUPS), RS = NCG_A / 4, NRI = BM / RS;
    const int grp = conv_index(warp) / (8 / CONV_GROUPS);
    const int ctid = (conv_index(warp) % (8 / CONV_GROUPS)) * 32 + lane;
    const int r0 = ctid >> 2, q = ctid & 3;
    const int ph = r0 & 7;
    const int64_t kbytes = p.K / 2;                  // packed bytes per weight row
    static_assert(RS % 8 == 0, "rows of a thread share the swizzle phase");
    KWalk wk(p.T, p.sched, unit_index, nst);
    for (int g = 0; g < grp; ++g) wk.advance();
    bool ok = true;
    for (uint32_t j = (uint32_t)grp; ok && wk.live; j += CONV_GROUPS) {
      const int kb0 = ((wk.step + k_rotation(wk.m, nst)) % nst) * KSUB;
      const int o0 = wk.m * UNIT + (int)rank * BM;
      uint4 in[KSUB][NRI];
#pragma unroll
      for (int u = 0; u < KSUB; ++u) {
        const int64_t col = (int64_t)(kb0 + u) * 64 + q * 16;
#pragma unroll
        for (int i = 0; i < NRI; ++i) {
          const int o = o0 + r0 + RS * i;
          in[u][i] = (o < p.N && col < kbytes)
                         ? __ldg(reinterpret_cast<const uint4*>(wpk + (int64_t)o * kbytes + col))
                         : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      const int c = j % SK;
      bool w = dev::mbar_wait(kfree_bar(c), ((j / SK) & 1u) ^ 1u, p.err, kSiteGemmConv,
                              p.limit_ns) && !*s_abort;
      w = __all_sync(0xffffffffu, w);
      if (!w) {
        give_up();
        ok = false;
        break;
      }
#pragma unroll
      for (int u = 0; u < KSUB; ++u) {
        uint8_t* dst = w_stage(c) + u * WT;
#pragma unroll
        for (int i = 0; i < NRI; ++i) {
          uint8_t* rowp = dst + (r0 + RS * i) * 128;
          const uint4 v = in[u][i];
          *reinterpret_cast<uint4*>(rowp + (((2 * q) ^ ph) << 4)) =
              make_uint4((v.x << 4) & 0xF0F0F0F0u, (v.y << 4) & 0xF0F0F0F0u,
                         (v.z << 4) & 0xF0F0F0F0u, (v.w << 4) & 0xF0F0F0F0u);
          *reinterpret_cast<uint4*>(rowp + (((2 * q + 1) ^ ph) << 4)) =
              make_uint4(v.x & 0xF0F0F0F0u, v.y & 0xF0F0F0F0u, v.z & 0xF0F0F0F0u,
                         v.w & 0xF0F0F0F0u);
        }
      }
      dev::fence_async_smem();   // this thread's stores -> visible to the tensor cores
      __syncwarp();
      if (lane == 0) dev::mbar_arrive_cluster(lead(ready_bar(c)));
      for (int g = 0; g < CONV_GROUPS; ++g) wk.advance();
    }
  } else if (warp >= W_EPI0) {
    // ---------------- epilogue ----------------
    const int etid = tid - W_EPI0 * 32;
    uint8_t* stg = smem + OFF_STG + (warp - W_EPI0) * STG;
    const int q = warp & 3;
    const int half = (warp - W_EPI0) >> 2;
    const int o_local = q * 32 + lane;
    const bool ep_lead = etid == 0;
    uint32_t it_n = 0;
    bool ok = true;
    auto it = tiles();
    int m, t0, nch;
    for (; ok && it.next(m, t0, nch); ++it_n) {
      const int o0 = m * UNIT + (int)rank * BM;
      const int b = it_n & 1;
      const int o = o0 + o_local;
      const bool has_o = o < p.N;
      const float sw = has_o ? p.w_scale[o] * (1.f / 16.f) : 0.f;
      const float w1 = (has_o && p.mean) ? p.w_rowsum[o] : 0.f;
      const float bb = (has_o && p.bias) ? __bfloat162float(p.bias[o]) : 0.f;
      const int ncols = nch * CH;
      for (int i = etid; i < ncols; i += NEPI) {
        const int t = t0 + i;
        s_tok[i] = make_float2((t < p.T) ? p.a_scale[t] : 0.f,
                               (t < p.T && p.mean) ? p.mean[t] : 0.f);
      }
      if (ep_lead) {
        const bool ready = dev::mbar_wait(tfull_bar(b), (it_n >> 1) & 1u, p.err,
                                          kSiteGemmAccum, p.limit_ns) && !*s_abort;
        if (!ready) give_up();
        s_misc[2] = ready ? 1u : 0u;
      }
      dev::named_bar(1, NEPI);
      ok = *reinterpret_cast<volatile uint32_t*>(&s_misc[2]) != 0;
      if (ok) dev::tc_fence_after();
      const int t_end = min(ncols, p.T - t0);
      const int nmine = (nch - half + EPW - 1) / EPW;
      if (ok && nmine == 0) {
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive_cluster(lead(tempty_bar(b)));
      }
#pragma unroll 1
      for (int cc = 0; ok && cc < nmine; ++cc) {
        const int c = half + cc * EPW;
        uint32_t r[32];
        dev::tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN + c * 32), r);
        dev::tmem_wait_ld();
        if (cc == nmine - 1) {
          dev::tc_fence_before();
          __syncwarp();
          if (lane == 0) dev::mbar_arrive_cluster(lead(tempty_bar(b)));
        }
        if (o0 + q * 32 >= p.N) continue;
        const int n_valid = t_end - c * 32;
        if (p.out_acc) {
          int32_t* dst = reinterpret_cast<int32_t*>(p.out) + (int64_t)(t0 + c * 32) * p.N + o;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (has_o && jj < n_valid) dst[(int64_t)jj * p.N] = (int32_t)r[jj] >> 4;
        } else {
          const float4* tk4 = reinterpret_cast<const float4*>(s_tok + c * 32);
          const float2 sw2 = make_float2(sw, sw), w12 = make_float2(w1, w1);
          const float2 bb2 = make_float2(bb, bb);
          uint32_t yb[16];
#pragma unroll
          for (int jj = 0; jj < 32; jj += 2) {
            const float4 tk = tk4[jj / 2];
            const float2 s2 = __fmul2_rn(make_float2(tk.x, tk.z), sw2);
            const float2 c2 = __ffma2_rn(make_float2(tk.y, tk.w), w12, bb2);
            const float2 a2 = make_float2((float)(int32_t)r[jj], (float)(int32_t)r[jj + 1]);
            const __nv_bfloat162 y = __float22bfloat162_rn(__ffma2_rn(a2, s2, c2));
            yb[jj / 2] = *reinterpret_cast<const uint32_t*>(&y);
          }
          if (lane == 0) dev::bulk_wait_all_read();
          __syncwarp();
#pragma unroll
          for (int jj = 0; jj < 32; jj += 2) {
            *reinterpret_cast<uint16_t*>(stg + jj * 64 + lane * 2) = (uint16_t)(yb[jj / 2] & 0xFFFFu);
            *reinterpret_cast<uint16_t*>(stg + (jj + 1) * 64 + lane * 2) = (uint16_t)(yb[jj / 2] >> 16);
          }
          dev::fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            dev::tma_store_2d(&tm_y, dev::smem_u32(stg), o0 + q * 32, t0 + c * 32);
            dev::bulk_commit();
          }
        }
      }
      dev::named_bar(1, NEPI);   // s_tok of this tile is no longer read
    }
    if (lane == 0) dev::bulk_wait_all();
  }

  dev::tc_fence_before();
  dev::cluster_sync();  // no MMA, remote arrive or TMEM access of either CTA is still pending
  if (warp == W_MMA) {
    dev::tc_fence_after();
    dev::tmem_dealloc_pair(tmem, TCOLS);
  }
}

// The CTA pairs' ranges of the flattened (channel tile, 32-token chunk) space. A range costs
// its chunks plus kTileCost for every tile it is cut into (at most maxch chunks, never across a
// channel tile): a tile's K loop costs nearly the same whatever its width (measured: the issue
// loop, not the tensor pipe, sets the time per K block), so the tile count dominates and a cut
// that would add a narrow tile is avoided. The largest cost over the pairs is minimised by
// bisection on a bound C with a greedy cover that stretches every range while its cost stays
// within C. Computed once per shape.
constexpr int kTileCost = 8;

void balance_ranges(int n_o, int cpm, int pairs, int maxch, int* starts) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int>, std::vector<int>> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(n_o, cpm, pairs, maxch);
  auto it = cache.find(key);
  if (it == cache.end()) {
    const int64_t total = (int64_t)n_o * cpm;
    // cost of [a, b): chunks + kTileCost * tiles, tiles counted per channel-tile piece
    auto cover = [&](int64_t cmax, std::vector<int>* out) {
      int64_t pos = 0;
      for (int u = 0; u < pairs; ++u) {
        if (out) (*out)[u] = (int)pos;
        int64_t cost = 0, end = pos;
        while (end < total) {
          // extend by one chunk: a new tile starts at a channel-tile boundary or after maxch
          // chunks of the current piece
          const int64_t m = end / cpm, piece_start = std::max(pos, m * cpm);
          const int64_t len = end - piece_start;            // chunks of this piece so far
          const int64_t add = 1 + ((len % maxch == 0) ? kTileCost : 0);
          if (cost + add > cmax) break;
          cost += add;
          ++end;
        }
        pos = end;
      }
      if (out) (*out)[pairs] = (int)total;
      return pos >= total;
    };
    int64_t lo = 1 + kTileCost, hi = total + kTileCost * (total + maxch - 1) / maxch + 1;
    while (lo < hi) {
      const int64_t mid = (lo + hi) / 2;
      if (cover(mid, nullptr)) hi = mid; else lo = mid + 1;
    }
    std::vector<int> v((size_t)pairs + 1);
    cover(lo, &v);
    it = cache.emplace(key, std::move(v)).first;
  }
  std::copy(it->second.begin(), it->second.end(), starts);
}

oq_status run_a8s(const GemmArgs& g, const GemmParams& p_in, cudaStream_t s) {
  using namespace sa;
  GemmParams p = p_in;
  CUtensorMap tx, ty;
  bool ok = true;
  if (!g.out_acc)
    ok &= make_map_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.out, (uint64_t)g.N, (uint64_t)g.T,
                      (uint64_t)g.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    std::memset(&ty, 0, sizeof(ty));
  ok &= make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.a, (uint64_t)g.K, (uint64_t)g.T,
                    (uint64_t)g.K, 128, XR, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return fail(OQ_ERR_CUDA, "cuTensorMapEncodeTiled failed or unavailable");
  auto kern = &k_gemm_a8s;
  const cudaError_t attr_err = allow_max_dynamic_smem(reinterpret_cast<const void*>(kern));
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(gemm_a8s)");
  int pairs = active_pairs_n(reinterpret_cast<const void*>(kern), SMEM, NTHR);
  if (pairs <= 0) return fail(OQ_ERR_UNSUPPORTED, "gemm: no CTA pair fits on this device");
  const int n_o = (int)((g.N + 2 * BM - 1) / (2 * BM));
  const int cpm = (int)((g.T + CH - 1) / CH);
  const int64_t chunks = (int64_t)n_o * cpm;
  pairs = (int)std::min<int64_t>(std::min<int64_t>(chunks, pairs), kMaxPairs);
  balance_ranges(n_o, cpm, pairs, BN / CH, p.sched);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(NTHR);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint8_t* wpk = g.w;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, tx, ty, wpk, p);
  if (le != cudaSuccess) return cuda_fail(le, "launch gemm_a8s");
  return OQ_OK;
}

uint16_t f16_bits(float f) {
  const __half h = __float2half_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

}  // namespace

bool tma_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                CUtensorMapSwizzle sw) {
  return make_map_2d(m, dt, base, inner, outer, row_bytes, box_inner, box_outer, sw);
}

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
  p.out = g.out;
  p.w_sz = g.w_sz;
  if (g.kind == kGemmLloydMax8)
    for (int i = 0; i < 128; ++i)
      p.lut8[i] = (uint32_t)f16_bits(g.centroids8[2 * i]) |
                  ((uint32_t)f16_bits(g.centroids8[2 * i + 1]) << 16);
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
  // up to 128 tokens: single CTAs on 128-channel tiles; beyond: CTA pairs on 256 channels
  const bool small = g.T <= 128;
  // W4A8 with a bf16 result and up to 256 tokens: the split-K cluster GEMM, which spreads
  // the K loop over the whole device instead of one tile per channel block
  if (g.kind == kGemmA8 && !g.out_acc && g.T <= 256) {
    const oq_status st = launch_gemm_splitk(g, s);
    if (st != OQ_ERR_UNSUPPORTED) return st;
  }
  switch (g.kind) {
    case kGemmA8: return small ? run<kGemmA8, 1>(g, p, s) : run_a8s(g, p, s);
    case kGemmA4: return small ? run<kGemmA4, 1>(g, p, s) : run<kGemmA4, 2>(g, p, s);
    case kGemmA2:
      if (g.K % 64) return fail(OQ_ERR_INVALID_ARG, "2-bit activations need K %% 64 == 0");
      return small ? run<kGemmA2, 1>(g, p, s) : run<kGemmA2, 2>(g, p, s);
    case kGemmLloydMax:
      return small ? run<kGemmLloydMax, 1>(g, p, s) : run<kGemmLloydMax, 2>(g, p, s);
    case kGemmLloydMax8:
      return small ? run<kGemmLloydMax8, 1>(g, p, s) : run<kGemmLloydMax8, 2>(g, p, s);
    case kGemmG64:
      if (g.K % 64 || !g.w_sz) return fail(OQ_ERR_INVALID_ARG, "grouped weights need K % 64 == 0");
      return small ? run<kGemmG64, 1>(g, p, s) : run<kGemmG64, 2>(g, p, s);
    default: return fail(OQ_ERR_INVALID_ARG, "unknown GEMM kind");
  }
}

}  // namespace oq
