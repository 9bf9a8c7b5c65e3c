// C ABI of the rotated, quantized linear layer (declarations and contracts: include/oq.h).
// Host-side validation, plan lifecycle, the device error word and dispatch to the kernels.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "oq_internal.h"
#include "ptx.cuh"

// Device error word: first bounded wait that gives up writes (1 << 63 | site << 32 | block).
__device__ unsigned long long g_oq_error_word;

namespace oq {

static thread_local char g_last_error[512] = "";

oq_status fail(oq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

oq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(OQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

unsigned long long* device_error_word() {
  constexpr int kMaxDev = 64;
  static unsigned long long* ptrs[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_oq_error_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned long long*>(p);
  }
  return ptrs[dev];
}

cudaError_t allow_max_dynamic_smem(const void* fn) {
  static std::mutex mu;
  static std::vector<std::pair<int, const void*>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& d : done)
    if (d.first == dev && d.second == fn) return cudaSuccess;
  int max_smem = 0;
  e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa{};
  e = cudaFuncGetAttributes(&fa, fn);
  if (e != cudaSuccess) return e;
  // the ceiling covers dynamic shared memory only; static shared memory comes on top
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           max_smem - (int)fa.sharedSizeBytes);
  if (e == cudaSuccess) done.emplace_back(dev, fn);
  return e;
}

namespace {

__global__ void k_debug_wait(unsigned long long* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    dev::mbar_init(dev::smem_u32(&bar), 1);
    dev::fence_mbar_init();
    // nothing ever arrives: the wait must give up by itself
    dev::mbar_wait(dev::smem_u32(&bar), 0, err, kSiteDebug, limit_ns);
  }
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

oq_status check_plan_device(const oq_plan* p) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != p->device)
    return fail(OQ_ERR_INVALID_ARG, "plan belongs to device %d, current device is %d",
                p->device, dev);
  return OQ_OK;
}

oq_status check_gemm_args(const void* a, const float* a_scale, const float* mean,
                          const uint8_t* w, const float* w_scale, const float* w_rowsum,
                          const void* bias, int64_t T, int64_t K, int64_t N, int out_kind,
                          const void* out) {
  if (T < 0 || T > 0x7FFFFFFF) return fail(OQ_ERR_INVALID_ARG, "T=%lld out of range", (long long)T);
  if (K < 32 || K > 32768 || K % 32)
    return fail(OQ_ERR_INVALID_ARG, "d_in=%lld must be a multiple of 32 in [32, 32768]",
                (long long)K);
  if (N < 16 || N > (1 << 24) || N % 16)
    return fail(OQ_ERR_INVALID_ARG, "d_out=%lld must be a positive multiple of 16",
                (long long)N);
  if (out_kind != OQ_OUT_BF16 && out_kind != OQ_OUT_ACC)
    return fail(OQ_ERR_INVALID_ARG, "unknown out_kind %d", out_kind);
  if (!w || !w_scale || !out) return fail(OQ_ERR_INVALID_ARG, "NULL weight/scale/out pointer");
  if (T > 0 && (!a || !a_scale)) return fail(OQ_ERR_INVALID_ARG, "NULL activation pointer");
  if (mean && !w_rowsum) return fail(OQ_ERR_INVALID_ARG, "mean given without w_rowsum");
  if ((T > 0 && !aligned16(a)) || !aligned16(w) || !aligned16(out))
    return fail(OQ_ERR_MISALIGNED, "activation, weight and output must be 16-byte aligned");
  (void)bias;
  return OQ_OK;
}

}  // namespace
}  // namespace oq

using namespace oq;

extern "C" {

const char* oq_status_string(oq_status s) {
  switch (s) {
    case OQ_OK: return "OQ_OK";
    case OQ_ERR_INVALID_ARG: return "OQ_ERR_INVALID_ARG";
    case OQ_ERR_UNSUPPORTED: return "OQ_ERR_UNSUPPORTED";
    case OQ_ERR_MISALIGNED: return "OQ_ERR_MISALIGNED";
    case OQ_ERR_CUDA: return "OQ_ERR_CUDA";
    case OQ_ERR_DEVICE_TIMEOUT: return "OQ_ERR_DEVICE_TIMEOUT";
    case OQ_ERR_NOMEM: return "OQ_ERR_NOMEM";
  }
  return "OQ_STATUS_UNKNOWN";
}

const char* oq_last_error(void) { return g_last_error; }

oq_status oq_device_status(int clear, uint64_t* code_out) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned long long* w = device_error_word();
  if (!w) return fail(OQ_ERR_CUDA, "device error word unavailable");
  unsigned long long v = 0;
  e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (code_out) *code_out = v;
  if (clear && v) {
    e = cudaMemset(w, 0, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  }
  const unsigned site = (unsigned)((v >> 32) & 0xFFFF);
  if (v && site >= kSiteBounds)
    return fail(OQ_ERR_INVALID_ARG, "index out of range (checked build): site %#x block %u", site,
                (unsigned)(v & 0xFFFFFFFFu));
  if (v) return fail(OQ_ERR_DEVICE_TIMEOUT, "device wait gave up: site %u block %u", site,
                     (unsigned)(v & 0xFFFFFFFFu));
  return OQ_OK;
}

int oq_default_block(int d) {
  if (d <= 0) return 0;
  int h = d & -d;
  return h > 1024 ? 1024 : h;
}

int oq_default_rounds(int h) { return h < 512 ? 2 : 1; }

oq_status oq_rpbh_tables(int d, int round, uint64_t seed, int8_t* signs_host,
                         int32_t* perm_host) {
  if (d <= 0 || d > 32768) return fail(OQ_ERR_INVALID_ARG, "d=%d out of range", d);
  if (round < 0) return fail(OQ_ERR_INVALID_ARG, "round must be >= 0");
  if (!signs_host || !perm_host) return fail(OQ_ERR_INVALID_ARG, "NULL output");
  rpbh_round_tables(d, round, seed, signs_host, perm_host);
  return OQ_OK;
}

oq_status oq_lloyd_max_codebook(double* centroids16_host, double* thresholds15_host) {
  if (!centroids16_host || !thresholds15_host) return fail(OQ_ERR_INVALID_ARG, "NULL output");
  lloyd_max_newton(centroids16_host, thresholds15_host);
  return OQ_OK;
}

oq_status oq_lloyd_max_codebook_8bit(double* centroids256_host, double* thresholds255_host) {
  if (!centroids256_host || !thresholds255_host) return fail(OQ_ERR_INVALID_ARG, "NULL output");
  lloyd_max_newton_256(centroids256_host, thresholds255_host);
  return OQ_OK;
}

oq_status oq_lloyd_max_codebook_width(int d, double* centroids16_host,
                                      double* thresholds15_host) {
  if (!centroids16_host || !thresholds15_host) return fail(OQ_ERR_INVALID_ARG, "NULL output");
  if (d < 32 || d > 32768) return fail(OQ_ERR_INVALID_ARG, "d=%d outside [32, 32768]", d);
  lloyd_max_newton_width(d, centroids16_host, thresholds15_host);
  return OQ_OK;
}

oq_status oq_plan_create(oq_plan** out, int d, int h, int rounds, uint64_t seed, int center,
                         oq_act_kind act) {
  if (!out) return fail(OQ_ERR_INVALID_ARG, "NULL plan output");
  *out = nullptr;
  if (d < 32 || d > 32768 || d % 32)
    return fail(OQ_ERR_INVALID_ARG, "d=%d must be a multiple of 32 in [32, 32768]", d);
  if (!pow2(h) || h > 1024 || d % h)
    return fail(OQ_ERR_INVALID_ARG, "h=%d must be a power of two <= 1024 dividing d=%d", h, d);
  if (rounds != 1 && rounds != 2) return fail(OQ_ERR_INVALID_ARG, "rounds=%d not in {1,2}", rounds);
  if (act != OQ_ACT_INT8_ABSMAX && act != OQ_ACT_INT4_ABSMAX && act != OQ_ACT_INT4_LLOYDMAX &&
      act != OQ_ACT_INT4_PERCENTILE && act != OQ_ACT_INT4_LLOYDMAX_WIDTH &&
      act != OQ_ACT_INT8_LLOYDMAX && act != OQ_ACT_INT2_PERCENTILE)
    return fail(OQ_ERR_INVALID_ARG, "unknown activation kind %d", (int)act);
  if (act == OQ_ACT_INT4_PERCENTILE && d > 8192)
    return fail(OQ_ERR_UNSUPPORTED, "the percentile scale supports d <= 8192 (d=%d)", d);
  if (act == OQ_ACT_INT8_LLOYDMAX && d > 8192)
    return fail(OQ_ERR_UNSUPPORTED, "8-bit Lloyd-Max codes support d <= 8192 (d=%d)", d);
  if (act == OQ_ACT_INT2_PERCENTILE && (d > 8192 || d % 64))
    return fail(d % 64 ? OQ_ERR_INVALID_ARG : OQ_ERR_UNSUPPORTED,
                "2-bit activations need d %% 64 == 0 and d <= 8192 (d=%d)", d);
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(OQ_ERR_UNSUPPORTED, "needs an sm_100 device (found sm_%d%d)", major, minor);

  oq_plan* p = new (std::nothrow) oq_plan();
  if (!p) return fail(OQ_ERR_NOMEM, "plan allocation");
  p->d = d; p->h = h; p->rounds = rounds; p->center = center ? 1 : 0; p->act = act;
  p->seed = seed; p->device = dev;
  p->signs.resize((size_t)rounds * d);
  p->perm.resize((size_t)rounds * d);
  // Gather entries in the order the rotate-quantize kernel consumes them: thread t, register
  // i of round r reads rotated position q = rq_gather_position(h, t, i), i.e. source index
  // perm_r[q] with sign signs_r[q]. Round 1 reads the staged row, so the index is where the
  // kernel keeps that channel; round 2 reads the fp32 round buffer, so the index is where
  // that buffer keeps position perm_r[q].
  std::vector<uint16_t> tab((size_t)rounds * d);
  for (int r = 0; r < rounds; ++r)
    rpbh_round_tables(d, r, seed, p->signs.data() + (size_t)r * d, p->perm.data() + (size_t)r * d);
  // Two-token kernel (d <= kRqPairMaxD): the interleaved row keeps channel j in word word[j]
  // (bank-conflict-free stores and gathers); round-1 entries are byte offsets of those words.
  // The single-token kernel reads the bf16 row as it is: entry = channel index.
  const bool pair = d <= kRqPairMaxD;
  std::vector<int> word;
  if (pair) {
    word = pair_word_layout(d, h, p->perm.data());
    if (word.size() != (size_t)d) {
      delete p;
      return fail(OQ_ERR_UNSUPPORTED, "word layout failed for d=%d h=%d", d, h);
    }
  }
  std::vector<uint32_t> slot(pair ? (size_t)d : 0);
  for (int j = 0; pair && j < d; ++j)
    slot[((size_t)((j % 8) / 4) * (d / 8) + j / 8) * 4 + j % 4] = 4u * (uint32_t)word[(size_t)j];
  for (int r = 0; r < rounds; ++r) {
    const int8_t* sg = p->signs.data() + (size_t)r * d;
    const int32_t* pm = p->perm.data() + (size_t)r * d;
    for (int t = 0; t < d / 32; ++t) {
      for (int i = 0; i < 32; ++i) {
        const int64_t q = rq_gather_position(h, t, i);
        // round 1 carries no sign: it is applied to the source channel (see below)
        const int src = (r == 0) ? (pair ? 4 * word[(size_t)pm[q]] : pm[q])
                                 : (rq_round_buffer_index(d, pm[q]) | (sg[q] < 0 ? 0x8000 : 0));
        tab[(size_t)r * d + (size_t)t * 32 + i] = (uint16_t)src;
      }
    }
  }
  // Round-1 signs moved to the source side: channel pm[i] takes sign sg[i] (the rotated
  // position that gathers it). Bit 15 (even channel) / 31 (odd channel) of word j/2.
  std::vector<uint32_t> smask((size_t)d / 2, 0u);
  for (int i = 0; i < d; ++i)
    if (p->signs[i] < 0) smask[p->perm[i] / 2] |= 1u << (15 + 16 * (p->perm[i] & 1));
  // c' = unnormalised round-1 transform of the all-ones vector = block Hadamard of the signs
  std::vector<float> ones((size_t)d);
  {
    std::vector<int32_t> v(p->signs.begin(), p->signs.begin() + d);
    for (int blk = 0; blk < d; blk += h)
      for (int len = 1; len < h; len <<= 1)
        for (int i = blk; i < blk + h; ++i)
          if (!((i - blk) & len)) {
            const int32_t a0 = v[i], b0 = v[i + len];
            v[i] = a0 + b0;
            v[i + len] = a0 - b0;
          }
    for (int i = 0; i < d; ++i) ones[i] = (float)v[i];
  }
  if (act == OQ_ACT_INT4_LLOYDMAX_WIDTH)
    lloyd_max_newton_width(d, p->cb_c, p->cb_t);
  else
    lloyd_max_newton(p->cb_c, p->cb_t);
  if (act == OQ_ACT_INT8_LLOYDMAX) lloyd_max_newton_256(p->cb8_c, p->cb8_t);
  auto release = [&]() {
    if (p->d_tab) cudaFree(p->d_tab);
    if (p->d_smask) cudaFree(p->d_smask);
    if (p->d_slot) cudaFree(p->d_slot);
    if (p->d_ones) cudaFree(p->d_ones);
    if (p->d_thr8) cudaFree(p->d_thr8);
    delete p;
  };
  if (cudaMalloc(&p->d_tab, tab.size() * sizeof(uint16_t)) != cudaSuccess ||
      cudaMalloc(&p->d_smask, smask.size() * sizeof(uint32_t)) != cudaSuccess ||
      cudaMalloc(&p->d_ones, ones.size() * sizeof(float)) != cudaSuccess ||
      (pair && cudaMalloc(&p->d_slot, slot.size() * sizeof(uint32_t)) != cudaSuccess)) {
    release();
    return fail(OQ_ERR_NOMEM, "cudaMalloc plan tables");
  }
  e = cudaMemcpy(p->d_tab, tab.data(), tab.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_smask, smask.data(), smask.size() * sizeof(uint32_t),
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_ones, ones.data(), ones.size() * sizeof(float), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && pair)
    e = cudaMemcpy(p->d_slot, slot.data(), slot.size() * sizeof(uint32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && act == OQ_ACT_INT8_LLOYDMAX) {
    float thr[256];
    for (int k = 0; k < 255; ++k) thr[k] = (float)p->cb8_t[k];
    thr[255] = INFINITY;
    e = cudaMalloc(&p->d_thr8, sizeof(thr));
    if (e == cudaSuccess) e = cudaMemcpy(p->d_thr8, thr, sizeof(thr), cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    release();
    return cuda_fail(e, "upload plan tables");
  }
  if (!device_error_word()) {
    release();
    return fail(OQ_ERR_CUDA, "device error word unavailable");
  }
  *out = p;
  return OQ_OK;
}

void oq_plan_destroy(oq_plan* plan) {
  if (!plan) return;
  if (plan->d_tab || plan->d_smask || plan->d_ones || plan->d_thr8 || plan->d_slot) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != plan->device) cudaSetDevice(plan->device);
    if (plan->d_tab) cudaFree(plan->d_tab);
    if (plan->d_smask) cudaFree(plan->d_smask);
    if (plan->d_slot) cudaFree(plan->d_slot);
    if (plan->d_ones) cudaFree(plan->d_ones);
    if (plan->d_thr8) cudaFree(plan->d_thr8);
    if (cur != plan->device && cur >= 0) cudaSetDevice(cur);
  }
  delete plan;
}

oq_status oq_plan_get_rpbh(const oq_plan* plan, int round, int8_t* signs_host,
                           int32_t* perm_host) {
  if (!plan || !signs_host || !perm_host) return fail(OQ_ERR_INVALID_ARG, "NULL argument");
  if (round < 0 || round >= plan->rounds) return fail(OQ_ERR_INVALID_ARG, "round out of range");
  std::memcpy(signs_host, plan->signs.data() + (size_t)round * plan->d, plan->d);
  std::memcpy(perm_host, plan->perm.data() + (size_t)round * plan->d, plan->d * sizeof(int32_t));
  return OQ_OK;
}

oq_status oq_debug_pair_layout(int d, int h, uint64_t seed, int32_t* word_host) {
  if (!word_host) return fail(OQ_ERR_INVALID_ARG, "NULL output");
  if (d < 32 || d > kRqPairMaxD || d % 32 || !pow2(h) || h > 1024 || d % h)
    return fail(OQ_ERR_INVALID_ARG, "d=%d h=%d outside the two-token kernel's range", d, h);
  std::vector<int8_t> sg((size_t)d);
  std::vector<int32_t> pm((size_t)d);
  rpbh_round_tables(d, 0, seed, sg.data(), pm.data());
  const std::vector<int> word = pair_word_layout(d, h, pm.data());
  if (word.size() != (size_t)d) return fail(OQ_ERR_UNSUPPORTED, "word layout failed");
  for (int j = 0; j < d; ++j) word_host[j] = word[(size_t)j];
  return OQ_OK;
}

oq_status oq_plan_get_codebook(const oq_plan* plan, int levels, double* centroids_host,
                               double* thresholds_host) {
  if (!plan || !centroids_host || !thresholds_host)
    return fail(OQ_ERR_INVALID_ARG, "NULL argument");
  int have = 0;
  if (plan->act == OQ_ACT_INT4_LLOYDMAX || plan->act == OQ_ACT_INT4_LLOYDMAX_WIDTH) have = 16;
  if (plan->act == OQ_ACT_INT8_LLOYDMAX) have = 256;
  if (have == 0)
    return fail(OQ_ERR_INVALID_ARG, "the plan's activation kind (%d) uses no codebook",
                (int)plan->act);
  if (levels != have)
    return fail(OQ_ERR_INVALID_ARG, "the plan's codebook has %d levels, not %d", have, levels);
  const double* c = have == 16 ? plan->cb_c : plan->cb8_c;
  const double* t = have == 16 ? plan->cb_t : plan->cb8_t;
  std::memcpy(centroids_host, c, sizeof(double) * (size_t)have);
  std::memcpy(thresholds_host, t, sizeof(double) * (size_t)(have - 1));
  return OQ_OK;
}

static oq_status rotate_quantize_impl(const oq_plan* plan, const void* x, int64_t T, int64_t ldx,
                                      void* codes, float* scale, float* mean, float* rotated,
                                      float* rowsum, int mode, int center, int wlayout,
                                      cudaStream_t s) {
  RqArgs a;
  a.x = x; a.ldx = ldx; a.T = T; a.d = plan->d; a.h = plan->h; a.rounds = plan->rounds;
  a.center = center; a.mode = mode; a.tab = plan->d_tab; a.smask = plan->d_smask;
  a.slot = plan->d_slot;
  a.ones = plan->d_ones; a.codes = codes; a.scale = scale;
  a.mean = mean; a.rotated = rotated; a.rowsum = rowsum; a.wlayout = wlayout;
  a.thr8 = plan->d_thr8;
  for (int i = 0; i < 15; ++i) a.thr[i] = (float)plan->cb_t[i];
  return launch_rotate_quant(a, s);
}

oq_status oq_rotate_quantize(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                             void* codes, float* scale, float* mean, float* rotated_f32,
                             void* stream) {
  if (!plan) return fail(OQ_ERR_INVALID_ARG, "NULL plan");
  if (T < 0 || T > 0x7FFFFFFF) return fail(OQ_ERR_INVALID_ARG, "T out of range");
  if (ldx < plan->d || (ldx * 2) % 16) return fail(OQ_ERR_MISALIGNED, "ldx must be >= d and a multiple of 8");
  if (T > 0 && (!x_bf16 || !codes || !scale)) return fail(OQ_ERR_INVALID_ARG, "NULL x/codes/scale");
  if (T > 0 && plan->center && !mean) return fail(OQ_ERR_INVALID_ARG, "centering plan needs mean");
  if ((x_bf16 && !aligned16(x_bf16)) || (codes && !aligned16(codes)) ||
      (rotated_f32 && !aligned16(rotated_f32)))
    return fail(OQ_ERR_MISALIGNED, "x, codes and rotated must be 16-byte aligned");
  oq_status st = check_plan_device(plan);
  if (st != OQ_OK) return st;
  const int mode = plan->act == OQ_ACT_INT8_ABSMAX       ? kRqInt8
                   : plan->act == OQ_ACT_INT4_ABSMAX     ? kRqInt4
                   : plan->act == OQ_ACT_INT4_PERCENTILE ? kRqPercentile
                   : plan->act == OQ_ACT_INT2_PERCENTILE ? kRqPercentile2
                   : plan->act == OQ_ACT_INT8_LLOYDMAX   ? kRqLloydMax8
                                                         : kRqLloydMax;   // either codebook
  return rotate_quantize_impl(plan, x_bf16, T, ldx, codes, scale, plan->center ? mean : nullptr,
                              rotated_f32, nullptr, mode, plan->center, 0,
                              static_cast<cudaStream_t>(stream));
}

oq_status oq_prepare_weights(const oq_plan* plan, const void* w_bf16, int64_t n_out, int64_t ldw,
                             uint8_t* w_packed, float* w_scale, float* w_rowsum, void* stream) {
  return oq_prepare_weights_rotated(plan, w_bf16, n_out, ldw, w_packed, w_scale, w_rowsum,
                                    nullptr, static_cast<cudaStream_t>(stream));
}
}  // extern "C"

namespace oq {
// oq_prepare_weights, optionally keeping the rotated rows (float [n_out, d]) in `rot`
oq_status oq_prepare_weights_rotated(const oq_plan* plan, const void* w_bf16, int64_t n_out,
                                     int64_t ldw, uint8_t* w_packed, float* w_scale,
                                     float* w_rowsum, float* rot, cudaStream_t stream) {
  if (!plan) return fail(OQ_ERR_INVALID_ARG, "NULL plan");
  if (n_out < 0 || n_out > 0x7FFFFFFF) return fail(OQ_ERR_INVALID_ARG, "n_out out of range");
  if (ldw < plan->d || (ldw * 2) % 16) return fail(OQ_ERR_MISALIGNED, "ldw must be >= d and a multiple of 8");
  if (n_out > 0 && (!w_bf16 || !w_packed || !w_scale || !w_rowsum))
    return fail(OQ_ERR_INVALID_ARG, "NULL weight argument");
  if ((w_bf16 && !aligned16(w_bf16)) || (w_packed && !aligned16(w_packed)))
    return fail(OQ_ERR_MISALIGNED, "w and w_packed must be 16-byte aligned");
  oq_status st = check_plan_device(plan);
  if (st != OQ_OK) return st;
  return rotate_quantize_impl(plan, w_bf16, n_out, ldw, w_packed, w_scale, nullptr, rot,
                              w_rowsum, kRqInt4, 0, 1, stream);
}
}  // namespace oq

extern "C" {


oq_status oq_prepare_weights_g64(const oq_plan* plan, const void* w_bf16, int64_t n_out,
                                 int64_t ldw, uint8_t* w_packed, uint32_t* w_sz, float* w_scale,
                                 float* w_rowsum, void* stream) {
  if (!plan) return fail(OQ_ERR_INVALID_ARG, "NULL plan");
  if (plan->d % 64) return fail(OQ_ERR_INVALID_ARG, "grouped weights need d %% 64 == 0");
  if (n_out < 0 || n_out > 0x7FFFFFFF) return fail(OQ_ERR_INVALID_ARG, "n_out out of range");
  if (n_out > 0 && !w_sz) return fail(OQ_ERR_INVALID_ARG, "NULL w_sz");
  if (n_out == 0) return OQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* rot = nullptr;
  cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&rot),
                                  (size_t)n_out * (size_t)plan->d * sizeof(float), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(rotated weights)");
  // the rotation (and w_1) of oq_prepare_weights; its per-channel codes and scales are
  // overwritten by the grouped quantizer below
  oq_status st = oq_prepare_weights_rotated(plan, w_bf16, n_out, ldw, w_packed, w_scale,
                                            w_rowsum, rot, s);
  if (st == OQ_OK) st = launch_quant_g64(rot, n_out, plan->d, w_packed, w_sz, w_scale, s);
  e = cudaFreeAsync(rot, s);
  if (st == OQ_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(rotated weights)");
  return st;
}

oq_status oq_gemm_w4a4_g64(oq_act_kind kind, const uint8_t* a_packed, const float* a_scale,
                           const float* mean, const uint8_t* w_packed, const uint32_t* w_sz,
                           const float* w_scale, const float* w_rowsum, const void* bias_bf16,
                           int64_t T, int64_t d_in, int64_t d_out, oq_out_kind out_kind,
                           void* out, void* stream) {
  if (kind != OQ_ACT_INT4_ABSMAX && kind != OQ_ACT_INT4_PERCENTILE)
    return fail(OQ_ERR_INVALID_ARG, "grouped weights take INT4_ABSMAX or INT4_PERCENTILE codes");
  if (d_in % 64) return fail(OQ_ERR_INVALID_ARG, "grouped weights need d_in %% 64 == 0");
  if (!w_sz) return fail(OQ_ERR_INVALID_ARG, "NULL w_sz");
  oq_status st = check_gemm_args(a_packed, a_scale, mean, w_packed, w_scale, w_rowsum, bias_bf16,
                                 T, d_in, d_out, (int)out_kind, out);
  if (st != OQ_OK) return st;
  GemmArgs g;
  g.kind = kGemmG64; g.a = a_packed; g.a_scale = a_scale; g.mean = mean; g.w = w_packed;
  g.w_sz = w_sz; g.w_scale = w_scale; g.w_rowsum = w_rowsum; g.bias = bias_bf16; g.T = T;
  g.K = d_in; g.N = d_out; g.out_acc = out_kind == OQ_OUT_ACC; g.out = out;
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

oq_status oq_gemm_w4a8(const int8_t* a, const float* a_scale, const float* mean,
                       const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                       const void* bias_bf16, int64_t T, int64_t d_in, int64_t d_out,
                       oq_out_kind out_kind, void* out, void* stream) {
  oq_status st = check_gemm_args(a, a_scale, mean, w_packed, w_scale, w_rowsum, bias_bf16, T,
                                 d_in, d_out, (int)out_kind, out);
  if (st != OQ_OK) return st;
  GemmArgs g;
  g.kind = kGemmA8; g.a = a; g.a_scale = a_scale; g.mean = mean; g.w = w_packed;
  g.w_scale = w_scale; g.w_rowsum = w_rowsum; g.bias = bias_bf16; g.T = T; g.K = d_in;
  g.N = d_out; g.out_acc = out_kind == OQ_OUT_ACC; g.out = out;
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

oq_status oq_gemm_w4a4(const oq_plan* plan, oq_act_kind kind, const uint8_t* a_packed,
                       const float* a_scale, const float* mean, const uint8_t* w_packed,
                       const float* w_scale, const float* w_rowsum, const void* bias_bf16,
                       int64_t T, int64_t d_in, int64_t d_out, oq_out_kind out_kind, void* out,
                       void* stream) {
  if (kind != OQ_ACT_INT4_ABSMAX && kind != OQ_ACT_INT4_LLOYDMAX &&
      kind != OQ_ACT_INT4_PERCENTILE && kind != OQ_ACT_INT4_LLOYDMAX_WIDTH)
    return fail(OQ_ERR_INVALID_ARG,
                "oq_gemm_w4a4 takes INT4_ABSMAX, INT4_PERCENTILE or a Lloyd-Max kind");
  const bool lm = kind == OQ_ACT_INT4_LLOYDMAX || kind == OQ_ACT_INT4_LLOYDMAX_WIDTH;
  if (lm && !plan)
    return fail(OQ_ERR_INVALID_ARG, "Lloyd-Max GEMM needs the plan's codebook");
  oq_status st = check_gemm_args(a_packed, a_scale, mean, w_packed, w_scale, w_rowsum, bias_bf16,
                                 T, d_in, d_out, (int)out_kind, out);
  if (st != OQ_OK) return st;
  GemmArgs g;
  g.kind = lm ? kGemmLloydMax : kGemmA4;   // percentile codes run through the A4 GEMM
  g.a = a_packed; g.a_scale = a_scale; g.mean = mean; g.w = w_packed; g.w_scale = w_scale;
  g.w_rowsum = w_rowsum; g.bias = bias_bf16; g.T = T; g.K = d_in; g.N = d_out;
  g.out_acc = out_kind == OQ_OUT_ACC; g.out = out;
  if (plan)
    for (int i = 0; i < 16; ++i) g.centroids[i] = (float)plan->cb_c[i];
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

oq_status oq_gemm_w4a2(const uint8_t* a_packed, const float* a_scale, const float* mean,
                       const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                       const void* bias_bf16, int64_t T, int64_t d_in, int64_t d_out,
                       oq_out_kind out_kind, void* out, void* stream) {
  if (d_in % 64) return fail(OQ_ERR_INVALID_ARG, "2-bit activations need d_in %% 64 == 0");
  oq_status st = check_gemm_args(a_packed, a_scale, mean, w_packed, w_scale, w_rowsum, bias_bf16,
                                 T, d_in, d_out, (int)out_kind, out);
  if (st != OQ_OK) return st;
  GemmArgs g;
  g.kind = kGemmA2; g.a = a_packed; g.a_scale = a_scale; g.mean = mean; g.w = w_packed;
  g.w_scale = w_scale; g.w_rowsum = w_rowsum; g.bias = bias_bf16; g.T = T; g.K = d_in;
  g.N = d_out; g.out_acc = out_kind == OQ_OUT_ACC; g.out = out;
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

oq_status oq_gemm_w4a8_lloydmax(const oq_plan* plan, const uint8_t* codes, const float* sigma,
                                const float* mean, const uint8_t* w_packed, const float* w_scale,
                                const float* w_rowsum, const void* bias_bf16, int64_t T,
                                int64_t d_in, int64_t d_out, oq_out_kind out_kind, void* out,
                                void* stream) {
  if (!plan || plan->act != OQ_ACT_INT8_LLOYDMAX)
    return fail(OQ_ERR_INVALID_ARG, "the 8-bit Lloyd-Max GEMM needs an INT8_LLOYDMAX plan");
  oq_status st = check_gemm_args(codes, sigma, mean, w_packed, w_scale, w_rowsum, bias_bf16, T,
                                 d_in, d_out, (int)out_kind, out);
  if (st != OQ_OK) return st;
  GemmArgs g;
  g.kind = kGemmLloydMax8;
  g.a = codes; g.a_scale = sigma; g.mean = mean; g.w = w_packed; g.w_scale = w_scale;
  g.w_rowsum = w_rowsum; g.bias = bias_bf16; g.T = T; g.K = d_in; g.N = d_out;
  g.out_acc = out_kind == OQ_OUT_ACC; g.out = out;
  for (int i = 0; i < 256; ++i) g.centroids8[i] = (float)plan->cb8_c[i];
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

static size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }
// one byte per code (A8 absmax and 8-bit Lloyd-Max) or two codes per byte
static bool codes8(const oq_plan* plan) {
  return plan->act == OQ_ACT_INT8_ABSMAX || plan->act == OQ_ACT_INT8_LLOYDMAX;
}

// bytes of one token's codes: d (8-bit kinds), d / 2 (4-bit) or d / 4 (2-bit)
static size_t code_row_bytes(const oq_plan* plan) {
  if (codes8(plan)) return (size_t)plan->d;
  return plan->act == OQ_ACT_INT2_PERCENTILE ? (size_t)plan->d / 4 : (size_t)plan->d / 2;
}

// the activation kinds the single-launch layer takes (it writes their codes one byte each)
static bool fused_kind(const oq_plan* plan) {
  return plan->act == OQ_ACT_INT8_ABSMAX || plan->act == OQ_ACT_INT4_ABSMAX ||
         plan->act == OQ_ACT_INT4_PERCENTILE;
}

// bytes of oq_linear's code region for T tokens: one byte per code wherever the single launch
// may run, the kind's own rows otherwise
static size_t linear_code_bytes(const oq_plan* plan, int64_t T) {
  if (fused_kind(plan) && T >= 1 && T <= kFusedMaxTokens) return (size_t)T * (size_t)plan->d;
  return (size_t)T * code_row_bytes(plan);
}

size_t oq_linear_workspace_bytes(const oq_plan* plan, int64_t T) {
  if (!plan || T < 0) return 0;
  return round256(linear_code_bytes(plan, T)) + 2 * round256((size_t)T * 4);
}

oq_status oq_linear(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                    const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                    const void* bias_bf16, int64_t d_out, void* y_bf16, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!plan) return fail(OQ_ERR_INVALID_ARG, "NULL plan");
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, "T out of range");
  const size_t need = oq_linear_workspace_bytes(plan, T);
  if (T > 0 && (!workspace || workspace_bytes < need))
    return fail(OQ_ERR_INVALID_ARG, "workspace too small: need %zu bytes", need);
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(OQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if (plan->center && !w_rowsum) return fail(OQ_ERR_INVALID_ARG, "centering needs w_rowsum");
  // Up to 256 tokens of an INT8 absmax or INT4 (absmax, percentile) layer run as one launch
  // where the device holds all of its clusters at once (same results bit for bit); otherwise
  // the two kernels below.
  if (fused_kind(plan) && T >= 1 && T <= kFusedMaxTokens && plan->d <= kRqPairMaxD &&
      plan->d % 128 == 0 && d_out % 16 == 0) {
    const oq_status fs = oq_linear_fused(plan, x_bf16, T, ldx, w_packed, w_scale, w_rowsum,
                                         bias_bf16, d_out, y_bf16, workspace, workspace_bytes,
                                         stream);
    if (fs != OQ_ERR_UNSUPPORTED) return fs;
  }
  const size_t code_bytes = linear_code_bytes(plan, T);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* codes = ws;
  float* scale = reinterpret_cast<float*>(ws + round256(code_bytes));
  float* mean = reinterpret_cast<float*>(ws + round256(code_bytes) + round256((size_t)T * 4));
  oq_status st = oq_rotate_quantize(plan, x_bf16, T, ldx, codes, scale, mean, nullptr, stream);
  if (st != OQ_OK) return st;
  const float* m = plan->center ? mean : nullptr;
  if (plan->act == OQ_ACT_INT8_ABSMAX)
    return oq_gemm_w4a8(static_cast<const int8_t*>(codes), scale, m, w_packed, w_scale, w_rowsum,
                        bias_bf16, T, plan->d, d_out, OQ_OUT_BF16, y_bf16, stream);
  if (plan->act == OQ_ACT_INT8_LLOYDMAX)
    return oq_gemm_w4a8_lloydmax(plan, static_cast<const uint8_t*>(codes), scale, m, w_packed,
                                 w_scale, w_rowsum, bias_bf16, T, plan->d, d_out, OQ_OUT_BF16,
                                 y_bf16, stream);
  if (plan->act == OQ_ACT_INT2_PERCENTILE)
    return oq_gemm_w4a2(static_cast<const uint8_t*>(codes), scale, m, w_packed, w_scale,
                        w_rowsum, bias_bf16, T, plan->d, d_out, OQ_OUT_BF16, y_bf16, stream);
  return oq_gemm_w4a4(plan, plan->act, static_cast<const uint8_t*>(codes), scale, m, w_packed,
                      w_scale, w_rowsum, bias_bf16, T, plan->d, d_out, OQ_OUT_BF16, y_bf16,
                      stream);
}

oq_status oq_linear_fused(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                          const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                          const void* bias_bf16, int64_t d_out, void* y_bf16, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!plan) return fail(OQ_ERR_INVALID_ARG, "NULL plan");
  if (!fused_kind(plan))
    return fail(OQ_ERR_UNSUPPORTED,
                "the single-launch layer takes INT8_ABSMAX, INT4_ABSMAX or INT4_PERCENTILE plans");
  if (T < 1 || T > kFusedMaxTokens)
    return fail(OQ_ERR_UNSUPPORTED, "the single-launch layer takes 1 <= T <= 256");
  const size_t need = oq_linear_workspace_bytes(plan, T);
  if (!workspace || workspace_bytes < need)
    return fail(OQ_ERR_INVALID_ARG, "workspace too small: need %zu bytes", need);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(OQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if (plan->center && !w_rowsum) return fail(OQ_ERR_INVALID_ARG, "centering needs w_rowsum");
  if (ldx < plan->d || (ldx * 2) % 16) return fail(OQ_ERR_MISALIGNED, "ldx must be >= d and a multiple of 8");
  if (!x_bf16 || !aligned16(x_bf16)) return fail(OQ_ERR_MISALIGNED, "x must be 16-byte aligned");
  oq_status st = check_gemm_args(workspace, reinterpret_cast<const float*>(workspace), nullptr,
                                 w_packed, w_scale, w_rowsum, bias_bf16, T, plan->d, d_out,
                                 OQ_OUT_BF16, y_bf16);
  if (st != OQ_OK) return st;
  st = check_plan_device(plan);
  if (st != OQ_OK) return st;
  const size_t code_bytes = linear_code_bytes(plan, T);   // T * d: one byte per code
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  FusedArgs f;
  RqArgs& a = f.rq;
  a.x = x_bf16; a.ldx = ldx; a.T = T; a.d = plan->d; a.h = plan->h; a.rounds = plan->rounds;
  a.center = plan->center;
  a.mode = plan->act == OQ_ACT_INT8_ABSMAX   ? kRqInt8
           : plan->act == OQ_ACT_INT4_ABSMAX ? kRqInt4
                                             : kRqPercentile;
  a.tab = plan->d_tab; a.smask = plan->d_smask;
  a.slot = plan->d_slot; a.ones = plan->d_ones; a.codes = ws;
  a.scale = reinterpret_cast<float*>(ws + round256(code_bytes));
  a.mean = plan->center ? reinterpret_cast<float*>(ws + round256(code_bytes) +
                                                   round256((size_t)T * 4))
                        : nullptr;
  f.w = w_packed; f.w_scale = w_scale; f.w_rowsum = plan->center ? w_rowsum : nullptr;
  f.bias = bias_bf16; f.y = y_bf16; f.T = T; f.K = plan->d; f.N = d_out;
  return launch_linear_fused(f, static_cast<cudaStream_t>(stream));
}

oq_status oq_linear_g64(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                        const uint8_t* w_packed, const uint32_t* w_sz, const float* w_scale,
                        const float* w_rowsum, const void* bias_bf16, int64_t d_out,
                        void* y_bf16, void* workspace, size_t workspace_bytes, void* stream) {
  if (!plan) return fail(OQ_ERR_INVALID_ARG, "NULL plan");
  if (plan->act != OQ_ACT_INT4_ABSMAX && plan->act != OQ_ACT_INT4_PERCENTILE)
    return fail(OQ_ERR_INVALID_ARG, "grouped weights need an INT4_ABSMAX or INT4_PERCENTILE plan");
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, "T out of range");
  const size_t need = oq_linear_workspace_bytes(plan, T);
  if (T > 0 && (!workspace || workspace_bytes < need))
    return fail(OQ_ERR_INVALID_ARG, "workspace too small: need %zu bytes", need);
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(OQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if (plan->center && !w_rowsum) return fail(OQ_ERR_INVALID_ARG, "centering needs w_rowsum");
  const size_t code_bytes = (size_t)T * (plan->d / 2);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* scale = reinterpret_cast<float*>(ws + round256(code_bytes));
  float* mean = reinterpret_cast<float*>(ws + round256(code_bytes) + round256((size_t)T * 4));
  oq_status st = oq_rotate_quantize(plan, x_bf16, T, ldx, ws, scale, mean, nullptr, stream);
  if (st != OQ_OK) return st;
  return oq_gemm_w4a4_g64(plan->act, ws, scale, plan->center ? mean : nullptr, w_packed, w_sz,
                          w_scale, w_rowsum, bias_bf16, T, plan->d, d_out, OQ_OUT_BF16, y_bf16,
                          stream);
}

oq_status oq_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull)
    return fail(OQ_ERR_INVALID_ARG, "timeout_ns must be in (0, 1e10]");
  unsigned long long* w = device_error_word();
  if (!w) return fail(OQ_ERR_CUDA, "device error word unavailable");
  k_debug_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(w, timeout_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch debug wait");
  return OQ_OK;
}

}  // extern "C"
