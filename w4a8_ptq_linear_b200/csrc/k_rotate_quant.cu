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

#include "rq_device.cuh"

namespace oq {
namespace {

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
    case kRqPercentile2:
      return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kRqPercentile2>);
    case kPairInt4W: return reinterpret_cast<void*>(&k_rotate_quant_pair<HL, R, kPairInt4W>);
    default: return nullptr;
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

// The launch shape of `a` (per device, width, block, rounds and quantizer; computed once).
static oq_status rq_config(const RqArgs& a, LaunchCfg& cfg) {
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
        if (!cfg.fn) return fail(OQ_ERR_INVALID_ARG, "rotate_quant: unknown quantizer %d", pmode);
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
  return OQ_OK;
}

// The kernel parameters of `a` for launch shape `cfg`.
static oq_status rq_fill(const RqArgs& a, const LaunchCfg& cfg, RqParams& p) {
  int hlog2 = 0;
  while ((1 << hlog2) < a.h) ++hlog2;
  p = RqParams{};
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
  if (a.mode == kRqPercentile || a.mode == kRqPercentile2) {
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
  return OQ_OK;
}

oq_status launch_rotate_quant(const RqArgs& a, cudaStream_t s) {
  if (a.T == 0) return OQ_OK;
  LaunchCfg cfg;
  oq_status st = rq_config(a, cfg);
  if (st != OQ_OK) return st;
  RqParams p;
  st = rq_fill(a, cfg, p);
  if (st != OQ_OK) return st;
  const int64_t units = cfg.pair ? (a.T + 1) / 2 : a.T;
  const int64_t grid = std::min<int64_t>(units, (int64_t)cfg.grid_per_sm);
  void* args[] = {&p};
  const cudaError_t ce =
      cudaLaunchKernel(cfg.fn, dim3((unsigned)grid), dim3((unsigned)cfg.nthr), args, cfg.smem, s);
  if (ce != cudaSuccess) return cuda_fail(ce, "launch rotate_quant");
  return OQ_OK;
}

oq_status rq_pair_setup(const RqArgs& a, RqParams& p, int& nthr, size_t& smem) {
  LaunchCfg cfg;
  oq_status st = rq_config(a, cfg);
  if (st != OQ_OK) return st;
  if (!cfg.pair) return fail(OQ_ERR_UNSUPPORTED, "the two-token body supports d <= %d", kPairMaxD);
  st = rq_fill(a, cfg, p);
  if (st != OQ_OK) return st;
  nthr = cfg.nthr;
  smem = cfg.smem;
  return OQ_OK;
}

}  // namespace oq
