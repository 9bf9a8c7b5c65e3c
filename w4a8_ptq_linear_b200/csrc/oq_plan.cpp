// Host-side plan tables: RPBH signs/permutations and the N(0,1) Lloyd-Max codebook.
//
// RPBH (OrbitQuant PR #25 "Default changes"; FLUX.1-schnell-OrbitQuant-W4A4 model card,
// "Quantization": rotation rpbh, rotation seed 0): the pages give no generator, so the
// tables follow a fixed, documented rule built on SplitMix64 (Steele, Lea and Flood,
// OOPSLA 2014) in counter form. The rule is stated in include/oq.h (oq_rpbh_tables).
//
// Lloyd-Max (OrbitQuant PR #25: codebook v3 is solved with Newton's method): the 16-level
// quantizer of N(0,1) satisfies, for every cell k with edges (tau_{k-1}, tau_k),
//     c_k = E[X | tau_{k-1} < X < tau_k],   tau_k = (c_k + c_{k+1}) / 2.
// By odd symmetry tau_7 = 0 and only c_8..c_15 are unknown; Newton's method solves the
// 8 centroid equations with the thresholds eliminated, using the analytic Jacobian.
#include "oq_internal.h"

#include <algorithm>
#include <cmath>
#include <utility>
#include <vector>

namespace oq {

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t splitmix64_at(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1ull) * 0x9E3779B97F4A7C15ull);
}

void rpbh_round_tables(int d, int round, uint64_t seed, int8_t* signs, int32_t* perm) {
  const uint64_t k_sign = splitmix64_at(seed, 2ull * (uint64_t)round);
  const uint64_t k_perm = splitmix64_at(seed, 2ull * (uint64_t)round + 1ull);
  std::vector<std::pair<uint64_t, int32_t>> keyed((size_t)d);
  for (int i = 0; i < d; ++i) {
    signs[i] = (splitmix64_at(k_sign, (uint64_t)i) >> 63) ? (int8_t)-1 : (int8_t)1;
    keyed[(size_t)i] = {splitmix64_at(k_perm, (uint64_t)i), i};
  }
  std::sort(keyed.begin(), keyed.end());  // by key, then by index
  for (int i = 0; i < d; ++i) perm[i] = keyed[(size_t)i].second;
}

// ---- Lloyd-Max ---------------------------------------------------------------------------

static double pdf(double x) { return std::exp(-0.5 * x * x) * 0.39894228040143267794; }

// P(a < X < b) for 0 <= a < b <= inf, from the upper tails (no cancellation).
static double cell_prob_pos(double a, double b) {
  const double ta = 0.5 * std::erfc(a * 0.70710678118654752440);
  const double tb = std::isinf(b) ? 0.0 : 0.5 * std::erfc(b * 0.70710678118654752440);
  return ta - tb;
}

void lloyd_max_newton(double c16[16], double t15[15]) {
  // unknowns c[j] = c_{8+j}, j = 0..7; edges e_j = tau_{7+j}: e_0 = 0, e_j = (c_{j-1}+c_j)/2
  double c[8];
  for (int j = 0; j < 8; ++j) c[j] = 0.15 + 0.33 * j;
  for (int it = 0; it < 100; ++it) {
    double a[8], b[8], p[8], g[8], F[8];
    for (int j = 0; j < 8; ++j) {
      a[j] = (j == 0) ? 0.0 : 0.5 * (c[j - 1] + c[j]);
      b[j] = (j == 7) ? INFINITY : 0.5 * (c[j] + c[j + 1]);
      p[j] = cell_prob_pos(a[j], b[j]);
      const double pb = std::isinf(b[j]) ? 0.0 : pdf(b[j]);
      g[j] = (pdf(a[j]) - pb) / p[j];
      F[j] = c[j] - g[j];
    }
    // Jacobian: dg/da = pdf(a)(g - a)/P, dg/db = pdf(b)(b - g)/P, da/dc = db/dc = 1/2
    double J[8][9];
    for (int j = 0; j < 8; ++j) {
      for (int k = 0; k < 8; ++k) J[j][k] = (j == k) ? 1.0 : 0.0;
      const double dga = (j == 0) ? 0.0 : pdf(a[j]) * (g[j] - a[j]) / p[j];
      const double dgb = (j == 7) ? 0.0 : pdf(b[j]) * (b[j] - g[j]) / p[j];
      if (j > 0) { J[j][j - 1] -= 0.5 * dga; J[j][j] -= 0.5 * dga; }
      if (j < 7) { J[j][j] -= 0.5 * dgb; J[j][j + 1] -= 0.5 * dgb; }
      J[j][8] = -F[j];
    }
    // Gaussian elimination with partial pivoting
    for (int col = 0; col < 8; ++col) {
      int piv = col;
      for (int r = col + 1; r < 8; ++r)
        if (std::fabs(J[r][col]) > std::fabs(J[piv][col])) piv = r;
      for (int k = 0; k < 9; ++k) std::swap(J[col][k], J[piv][k]);
      for (int r = col + 1; r < 8; ++r) {
        const double f = J[r][col] / J[col][col];
        for (int k = col; k < 9; ++k) J[r][k] -= f * J[col][k];
      }
    }
    double dx[8];
    for (int r = 7; r >= 0; --r) {
      double s = J[r][8];
      for (int k = r + 1; k < 8; ++k) s -= J[r][k] * dx[k];
      dx[r] = s / J[r][r];
    }
    double step = 0.0;
    for (int j = 0; j < 8; ++j) { c[j] += dx[j]; step = std::fmax(step, std::fabs(dx[j])); }
    if (step < 1e-15) break;
  }
  for (int j = 0; j < 8; ++j) { c16[8 + j] = c[j]; c16[7 - j] = -c[j]; }
  for (int k = 0; k < 15; ++k) t15[k] = 0.5 * (c16[k] + c16[k + 1]);
  t15[7] = 0.0;
}

// ---- per-width Lloyd-Max -------------------------------------------------------------------
// OrbitQuant PR #25 solves one codebook per width d (codebook v3). The quantized variable is a
// coordinate of the token normalised to unit RMS after the rotation; for a uniformly random
// direction it is y = sqrt(d) u_1, u uniform on the sphere S^(d-1), with density
//     f_d(y) = c_d (1 - y^2 / d)^((d - 3) / 2),  c_d = Gamma(d/2) / (sqrt(pi d) Gamma((d-1)/2)),
// on |y| < sqrt(d) (the N(0,1) limit as d grows). Its first moment over a cell is closed form,
// int_a^b y f_d = m(a) - m(b) with m(t) = c_d d / (d - 1) (1 - t^2 / d)^((d - 1) / 2); cell
// probabilities are integrated numerically (composite Simpson, steps of 1/2048).
namespace {
struct SphereMarginal {
  double d, r, log_c;
  explicit SphereMarginal(int dd)
      : d((double)dd), r(std::sqrt((double)dd)),
        log_c(std::lgamma(0.5 * dd) - 0.5 * std::log(3.14159265358979323846 * dd) -
              std::lgamma(0.5 * (dd - 1))) {}
  double pdf(double y) const {
    const double q = y * y / d;
    return q < 1.0 ? std::exp(log_c + 0.5 * (d - 3.0) * std::log1p(-q)) : 0.0;
  }
  double tail_moment(double t) const {   // int_t^r y f_d(y) dy, t >= 0
    const double q = t * t / d;
    return q < 1.0 ? std::exp(log_c + 0.5 * (d - 1.0) * std::log1p(-q)) * d / (d - 1.0) : 0.0;
  }
  double cell_prob(double a, double b) const {   // 0 <= a < b; f_d < 1e-40 beyond 16
    b = std::min(b, std::min(r, 16.0));
    if (b <= a) return 0.0;
    int n = (int)std::ceil((b - a) * 2048.0);
    n += n & 1;
    if (n < 2) n = 2;
    const double h = (b - a) / n;
    double sum = pdf(a) + pdf(b);
    for (int i = 1; i < n; ++i) sum += pdf(a + i * h) * ((i & 1) ? 4.0 : 2.0);
    return sum * h / 3.0;
  }
};
}  // namespace

void lloyd_max_newton_width(int d, double c16[16], double t15[15]) {
  const SphereMarginal f(d);
  double c[8];
  for (int j = 0; j < 8; ++j) c[j] = 0.15 + 0.3 * j;
  for (int it = 0; it < 100; ++it) {
    double a[8], b[8], p[8], g[8], F[8];
    for (int j = 0; j < 8; ++j) {
      a[j] = (j == 0) ? 0.0 : 0.5 * (c[j - 1] + c[j]);
      b[j] = (j == 7) ? f.r : 0.5 * (c[j] + c[j + 1]);
      p[j] = f.cell_prob(a[j], b[j]);
      g[j] = (f.tail_moment(a[j]) - f.tail_moment(b[j])) / p[j];
      F[j] = c[j] - g[j];
    }
    // Jacobian: dg/da = f(a)(g - a)/P, dg/db = f(b)(b - g)/P, da/dc = db/dc = 1/2
    double J[8][9];
    for (int j = 0; j < 8; ++j) {
      for (int k = 0; k < 8; ++k) J[j][k] = (j == k) ? 1.0 : 0.0;
      const double dga = (j == 0) ? 0.0 : f.pdf(a[j]) * (g[j] - a[j]) / p[j];
      const double dgb = (j == 7) ? 0.0 : f.pdf(b[j]) * (b[j] - g[j]) / p[j];
      if (j > 0) { J[j][j - 1] -= 0.5 * dga; J[j][j] -= 0.5 * dga; }
      if (j < 7) { J[j][j] -= 0.5 * dgb; J[j][j + 1] -= 0.5 * dgb; }
      J[j][8] = -F[j];
    }
    for (int col = 0; col < 8; ++col) {
      int piv = col;
      for (int rr = col + 1; rr < 8; ++rr)
        if (std::fabs(J[rr][col]) > std::fabs(J[piv][col])) piv = rr;
      for (int k = 0; k < 9; ++k) std::swap(J[col][k], J[piv][k]);
      for (int rr = col + 1; rr < 8; ++rr) {
        const double m = J[rr][col] / J[col][col];
        for (int k = col; k < 9; ++k) J[rr][k] -= m * J[col][k];
      }
    }
    double dx[8];
    for (int rr = 7; rr >= 0; --rr) {
      double sum = J[rr][8];
      for (int k = rr + 1; k < 8; ++k) sum -= J[rr][k] * dx[k];
      dx[rr] = sum / J[rr][rr];
    }
    double step = 0.0;
    for (int j = 0; j < 8; ++j) { c[j] += dx[j]; step = std::fmax(step, std::fabs(dx[j])); }
    if (step < 1e-15) break;
  }
  for (int j = 0; j < 8; ++j) { c16[8 + j] = c[j]; c16[7 - j] = -c[j]; }
  for (int k = 0; k < 15; ++k) t15[k] = 0.5 * (c16[k] + c16[k + 1]);
  t15[7] = 0.0;
}

// ---- 256-level N(0,1) Lloyd-Max ----------------------------------------------------------------
// The same centroid conditions with 128 unknowns (the positive centroids); the Jacobian is
// tridiagonal and solved by the Thomas algorithm. The start is the high-resolution
// (Panter-Dite) point density, proportional to phi^(1/3), i.e. quantiles of N(0, 3).
static double inv_phi(double prob) {   // Phi^-1 by bisection on erfc
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * std::erfc(-mid * 0.70710678118654752440) < prob) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

void lloyd_max_newton_256(double c256[256], double t255[255]) {
  constexpr int H = 128;
  double c[H];
  for (int j = 0; j < H; ++j) c[j] = std::sqrt(3.0) * inv_phi((H + j + 0.5) / (2.0 * H));
  for (int it = 0; it < 200; ++it) {
    double a[H], b[H], p[H], g[H], F[H], lo[H], di[H], up[H];
    for (int j = 0; j < H; ++j) {
      a[j] = (j == 0) ? 0.0 : 0.5 * (c[j - 1] + c[j]);
      b[j] = (j == H - 1) ? INFINITY : 0.5 * (c[j] + c[j + 1]);
      p[j] = cell_prob_pos(a[j], b[j]);
      const double pb = std::isinf(b[j]) ? 0.0 : pdf(b[j]);
      g[j] = (pdf(a[j]) - pb) / p[j];
      F[j] = c[j] - g[j];
    }
    for (int j = 0; j < H; ++j) {
      const double dga = (j == 0) ? 0.0 : pdf(a[j]) * (g[j] - a[j]) / p[j];
      const double dgb = (j == H - 1) ? 0.0 : pdf(b[j]) * (b[j] - g[j]) / p[j];
      lo[j] = -0.5 * dga;
      di[j] = 1.0 - 0.5 * dga - 0.5 * dgb;
      up[j] = -0.5 * dgb;
    }
    // Thomas algorithm for J dx = -F
    double cp[H], dp[H], dx[H];
    cp[0] = up[0] / di[0];
    dp[0] = -F[0] / di[0];
    for (int j = 1; j < H; ++j) {
      const double m = di[j] - lo[j] * cp[j - 1];
      cp[j] = up[j] / m;
      dp[j] = (-F[j] - lo[j] * dp[j - 1]) / m;
    }
    dx[H - 1] = dp[H - 1];
    for (int j = H - 2; j >= 0; --j) dx[j] = dp[j] - cp[j] * dx[j + 1];
    double step = 0.0;
    for (int j = 0; j < H; ++j) { c[j] += dx[j]; step = std::fmax(step, std::fabs(dx[j])); }
    if (step < 1e-15) break;
  }
  for (int j = 0; j < H; ++j) { c256[H + j] = c[j]; c256[H - 1 - j] = -c[j]; }
  for (int k = 0; k < 255; ++k) t255[k] = 0.5 * (c256[k] + c256[k + 1]);
  t255[H - 1] = 0.0;
}

}  // namespace oq

namespace oq {

// Bank-aware word layout of the two-token kernel's interleaved row (widths d <= 8192).
//
// The interleave pass stores one 32-bit word per channel (both tokens' bf16 values) and the
// round-1 gather loads one word per rotated position. Each warp-wide store instruction writes
// a fixed set of channels (a "store group": thread t stores channels 8c + k, c = t + m nact,
// for chunk m and k = 0..7), and each warp-wide gather instruction reads the channels of a
// fixed set of rotated positions (a "gather group": register i of the warp's 32 lanes). A
// channel lies in exactly one group of each kind, so the channels are the edges of a bipartite
// multigraph between store groups and gather groups in which every node has degree <= 32.
// By Koenig's edge-colouring theorem its edges can be coloured with 32 colours so that no two
// edges at a node share a colour; with colour = shared-memory bank, every store and every
// gather instruction then touches 32 distinct banks (no bank conflict). The colouring is built
// edge by edge: an edge takes a colour free at both ends, or, when the free colours a (at the
// store end) and b (at the gather end) differ, the a/b alternating path from the gather end is
// recoloured first (in a bipartite graph it cannot reach the store end).
// The word of channel ch is then 32 * store_group(ch) + colour(ch): unique, since the channels
// of one store group have distinct colours.
std::vector<int> pair_word_layout(int d, int h, const int32_t* perm0) {
  const int nact = d / 32;                       // threads that own positions
  const int nwarps = (nact + 31) / 32;
  const int ng = nwarps * 32;                    // groups of each kind
  std::vector<int> wg((size_t)d), rg((size_t)d, -1);
  for (int ch = 0; ch < d; ++ch) {
    const int c = ch / 8, k = ch % 8;
    const int t = c % nact, m = c / nact;       // thread t, chunk m
    wg[(size_t)ch] = ((t / 32) * 4 + m) * 8 + k;
  }
  for (int t = 0; t < nact; ++t)
    for (int i = 0; i < 32; ++i) {
      const int64_t q = rq_gather_position(h, t, i);
      rg[(size_t)perm0[q]] = (t / 32) * 32 + i;
    }
  std::vector<int> at_w((size_t)ng * 32, -1), at_r((size_t)ng * 32, -1), col((size_t)d, -1);
  auto free_at = [&](const std::vector<int>& at, int node) {
    for (int c = 0; c < 32; ++c)
      if (at[(size_t)node * 32 + c] < 0) return c;
    return -1;
  };
  std::vector<int> path;
  for (int ch = 0; ch < d; ++ch) {
    const int u = wg[(size_t)ch], v = rg[(size_t)ch];
    const int a = free_at(at_w, u), b = free_at(at_r, v);
    if (a < 0 || b < 0) return {};              // degree above 32: cannot happen
    if (at_r[(size_t)v * 32 + a] >= 0) {
      // flip the a/b path that starts at v with its a-edge
      path.clear();
      int node = v, c = a;
      bool on_gather_side = true;
      while (true) {
        const std::vector<int>& at = on_gather_side ? at_r : at_w;
        const int e = at[(size_t)node * 32 + c];
        if (e < 0) break;
        path.push_back(e);
        node = on_gather_side ? wg[(size_t)e] : rg[(size_t)e];
        on_gather_side = !on_gather_side;
        c = (c == a) ? b : a;
      }
      for (int e : path) {                       // clear, then recolour swapped
        at_w[(size_t)wg[(size_t)e] * 32 + col[(size_t)e]] = -1;
        at_r[(size_t)rg[(size_t)e] * 32 + col[(size_t)e]] = -1;
      }
      for (int e : path) {
        col[(size_t)e] = (col[(size_t)e] == a) ? b : a;
        at_w[(size_t)wg[(size_t)e] * 32 + col[(size_t)e]] = e;
        at_r[(size_t)rg[(size_t)e] * 32 + col[(size_t)e]] = e;
      }
    }
    col[(size_t)ch] = a;
    at_w[(size_t)u * 32 + a] = ch;
    at_r[(size_t)v * 32 + a] = ch;
  }
  std::vector<int> word((size_t)d);
  for (int ch = 0; ch < d; ++ch) word[(size_t)ch] = 32 * wg[(size_t)ch] + col[(size_t)ch];
  return word;
}

}  // namespace oq
