// Internal declarations shared by the host glue and the kernel translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/oq.h"

struct oq_plan {
  int d = 0, h = 0, rounds = 0, center = 0;
  oq_act_kind act = OQ_ACT_INT8_ABSMAX;
  uint64_t seed = 0;
  int device = -1;
  std::vector<int8_t> signs;    // rounds * d
  std::vector<int32_t> perm;    // rounds * d
  uint16_t* d_tab = nullptr;    // device: rounds * d gather entries in kernel order,
                                // source index (| (sign < 0) << 15 in round 2)
  uint32_t* d_smask = nullptr;  // device: d/2 words, round-1 sign of channel j at bit 15 / 31
  uint32_t* d_slot = nullptr;   // device (d <= 8192): byte offset of channel j's word,
                                // laid out [j % 8 / 4][j / 8][j % 4]
  float* d_ones = nullptr;      // device: d floats, unnormalised round-1 transform of ones
  double cb_c[16] = {}, cb_t[15] = {};
  double cb8_c[256] = {}, cb8_t[255] = {};   // 8-bit Lloyd-Max codebook
  float* d_thr8 = nullptr;      // device: its 255 thresholds (fp32) + one pad
};

namespace oq {

// ---- host tables -------------------------------------------------------------------------
uint64_t splitmix64_at(uint64_t key, uint64_t i);
void rpbh_round_tables(int d, int round, uint64_t seed, int8_t* signs, int32_t* perm);
void lloyd_max_newton(double c16[16], double t15[15]);
// 16-level Lloyd-Max codebook of the width-d post-rotation marginal (d >= 4)
void lloyd_max_newton_width(int d, double c16[16], double t15[15]);
// 256-level N(0,1) Lloyd-Max codebook (8-bit Lloyd-Max activations)
void lloyd_max_newton_256(double c256[256], double t255[255]);

// ---- launch helpers ----------------------------------------------------------------------
// Raises a kernel's dynamic shared-memory ceiling to the device's opt-in maximum, once per
// (device, kernel). The ceiling is a per-function attribute, so it must not depend on the
// size of any one launch.
cudaError_t allow_max_dynamic_smem(const void* fn);

// ---- errors ------------------------------------------------------------------------------
oq_status fail(oq_status s, const char* fmt, ...);
oq_status cuda_fail(cudaError_t e, const char* what);
// Device address of the error word of the current device (set up once per device).
unsigned long long* device_error_word();

// Device-side wait limit (nanoseconds of %globaltimer) for every bounded wait.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Site codes written into the error word (bits 32..47) by a wait that gave up.
enum : uint32_t {
  kSiteRqRow = 1,          // rotate-quantize: row load
  kSiteRqDrain = 2,        // rotate-quantize: drain of a row load after an abort
  kSiteGemmEmpty = 16,     // GEMM producer: stage free
  kSiteGemmFull = 17,      // GEMM converter: stage loaded
  kSiteGemmConv = 18,      // GEMM MMA: stage converted
  kSiteGemmAccum = 19,     // GEMM epilogue: accumulator ready
  kSiteGemmDrain = 20,     // GEMM: drain after an abort
  kSitePeak = 21,          // tensor-core peak loop: completion of the MMAs
  kSiteFusedLoad = 22,     // single-launch layer: activation codes loaded
  kSiteFusedMma = 23,      // single-launch layer: partial sums complete
  kSiteDebug = 99,         // oq_debug_wait_timeout
  // checked builds (-DOQ_CHECKED): an index outside its buffer (sites >= kSiteBounds)
  kSiteBounds = 0x100,
  kSiteBoundsRqRow = 0x101,      // single-token kernel: round-1 gather from the staged row
  kSiteBoundsRqRound2 = 0x102,   // round-2 gather from the round buffer
  kSiteBoundsPairSlot = 0x103,   // two-token kernel: interleave store into the word buffer
  kSiteBoundsPairGather = 0x104, // two-token kernel: round-1 gather from the word buffer
  kSiteBoundsFused = 0x120       // single-launch layer: ring stage, partial sums, token share
};

// ---- rotate + quantize ---------------------------------------------------------------------
enum RqMode : int { kRqInt8 = 0, kRqInt4 = 1, kRqLloydMax = 2, kRqPercentile = 3,
                     kRqLloydMax8 = 4, kRqPercentile2 = 5 };

struct RqArgs {
  const void* x = nullptr;   // bf16 [T, ldx]
  int64_t ldx = 0, T = 0;
  int d = 0, h = 0, rounds = 0, center = 0, mode = 0;
  const uint16_t* tab = nullptr;  // rounds * d
  const uint32_t* smask = nullptr;  // d/2 words: round-1 signs moved to the source channels
  const uint32_t* slot = nullptr;   // d <= kRqPairMaxD: byte offsets of the channels' words
  const float* ones = nullptr;      // d floats: unnormalised round-1 transform of all ones
  void* codes = nullptr;
  float* scale = nullptr;
  float* mean = nullptr;     // written when center (or when rowsum is wanted: see rowsum)
  float* rotated = nullptr;  // optional [T, d]
  float* rowsum = nullptr;   // optional [T]: sum of the row before centering/rotation
  float thr[15] = {};        // Lloyd-Max thresholds (fp32)
  int wlayout = 0;           // kRqInt4 only: write the codes in the GEMM weight layout
  const float* thr8 = nullptr;  // kRqLloydMax8: 256 floats (255 thresholds + pad), device
};
oq_status launch_rotate_quant(const RqArgs& a, cudaStream_t s);
// Kernel-order gather table helpers: the row position thread t, register i gathers in a
// round, where the staged input row keeps channel j, and where the fp32 round buffer keeps
// rotated position p (the last two depend on which kernel shape width d uses).
int64_t rq_gather_position(int h, int t, int i);
int rq_round_buffer_index(int d, int p);
// Widths up to this run the two-token kernel; wider rows the single-token kernel.
constexpr int kRqPairMaxD = 8192;
// tokens of one single-launch layer call at most (its MMA N and TMEM columns)
constexpr int kFusedMaxTokens = 256;
// Two-token kernel: the word (32-bit slot of the interleaved row) of every channel, chosen so
// that the interleave stores and the round-1 gathers of a warp are free of bank conflicts
// (a 32-colour edge colouring of the bipartite store-group / gather-group multigraph).
std::vector<int> pair_word_layout(int d, int h, const int32_t* perm0);

// ---- GEMM ----------------------------------------------------------------------------------
// kGemmG64: INT4 codes (decoded to fp16 integers) against asymmetric g = 64 weights
// dequantized to fp16 per (row, group) in the converters
enum GemmKind : int { kGemmA8 = 0, kGemmA4 = 1, kGemmLloydMax = 2, kGemmLloydMax8 = 3, kGemmG64 = 4,
                      kGemmA2 = 5 };

struct GemmArgs {
  int kind = kGemmA8;
  const void* a = nullptr;          // int8 [T, K] or uint8 [T, K/2]
  const float* a_scale = nullptr;
  const float* mean = nullptr;      // may be null
  const uint8_t* w = nullptr;       // uint8 [N, K/2]
  const float* w_scale = nullptr;
  const float* w_rowsum = nullptr;  // may be null when mean is null
  const void* bias = nullptr;       // bf16 [N] or null
  int64_t T = 0, K = 0, N = 0;
  int out_acc = 0;
  void* out = nullptr;
  float centroids[16] = {};
  float centroids8[256] = {};   // kGemmLloydMax8
  const uint32_t* w_sz = nullptr;  // kGemmG64: [K/64][N] words, fp16 sigma (low), z (high)
};
oq_status launch_gemm(const GemmArgs& g, cudaStream_t s);

// The whole layer in one launch (T <= 256; INT8 absmax, INT4 absmax or INT4 percentile
// activations, rq.mode kRqInt8 / kRqInt4 / kRqPercentile; per-channel weights): rotate-quantize
// into rq.codes / rq.scale / rq.mean, then the GEMM and epilogue into y.
struct FusedArgs {
  RqArgs rq;                        // the activation path, codes int8 [T, K] (one byte per
                                    // code for every kind) in the workspace
  const uint8_t* w = nullptr;       // uint8 [N, K/2], GEMM layout
  const float* w_scale = nullptr;
  const float* w_rowsum = nullptr;  // null unless the plan centers
  const void* bias = nullptr;       // bf16 [N] or null
  void* y = nullptr;                // bf16 [T, N]
  int64_t T = 0, K = 0, N = 0;
};
oq_status launch_linear_fused(const FusedArgs& a, cudaStream_t s);
// The same kernel's split-K GEMM alone (W4A8, bf16 output, 1 <= T <= 256) on codes a previous
// launch wrote; OQ_ERR_UNSUPPORTED (nothing launched) outside that or when it does not fit.
oq_status launch_gemm_splitk(const GemmArgs& g, cudaStream_t s);

// oq_prepare_weights that also writes the rotated rows (float [n_out, d]) to `rot` (if not null)
oq_status oq_prepare_weights_rotated(const oq_plan* plan, const void* w_bf16, int64_t n_out,
                                     int64_t ldw, uint8_t* w_packed, float* w_scale,
                                     float* w_rowsum, float* rot, cudaStream_t stream);

// Grouped asymmetric INT4 weights from rotated fp32 rows [n, d] (d % 64 == 0): codes Q - 8 in
// the GEMM layout, (sigma, z) fp16 words [d/64][n], per-row scale 1.
oq_status launch_quant_g64(const float* rot, int64_t n, int d, uint8_t* w_packed, uint32_t* w_sz,
                           float* w_scale, cudaStream_t s);

oq_status launch_debug_wait(unsigned long long timeout_ns, cudaStream_t s);

// Tensor-core peak loop (kind 0: kind::i8, 1: kind::f16); *pairs_out = CTA pairs launched.
oq_status launch_mma_peak(int kind, int64_t iters, int* pairs_out, cudaStream_t s);

}  // namespace oq
