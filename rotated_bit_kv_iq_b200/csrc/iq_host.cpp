// Host-side pieces of libiq: the Lloyd-Max codebook and the seeded rotation parameters.
//
// Codebook -- "压缩与速度的博弈——TurboQuant 和 RotorQuant 的真相" (zhichai.net), section
// "Lloyd-Max 最优量化": the optimal scalar quantiser for the known coordinate law is found
// offline by Lloyd's alternation (cells at midpoints, levels at cell means) and applied at
// run time by lookup; section "Beta 分布的魔力": that law is N(0, 1/d) for rotated unit
// vectors, i.e. the N(0,1) quantiser divided by sqrt(d); section "K 和 V 的非对称需求": K and V
// may use different widths (2, 3 or 4 bits here).  Computed here once per width and process in
// double precision from the closed-form Gaussian cell moments.
//
// Rotation parameters -- RotaryQuant abstract (arXiv 2608.08081): 256 stored parameters per
// head for the block-diagonal SO(4) stage; "压缩与速度的博弈" (zhichai.net), section "三种变体",
// and "RotorQuant" (sd114.wiki), section "1. 绕过蝴蝶网络": 128 parameters for one quaternion per
// block of 4 or one Givens rotation per pair.  The pages publish no values; this library draws
// every quaternion uniformly from the unit 3-sphere (Marsaglia 1972) and every Givens pair
// uniformly from the unit circle (a disc point by rejection, normalised), from a splitmix64
// counter stream (S. Vigna's splitmix64.c output function) keyed by
// (variant, seed, layer, head, block, side).  Only IEEE add/multiply/divide/sqrt are used,
// compiled without contraction, so the result is the same on every conforming platform.
#include <cmath>
#include <cstdint>

#include "iq_internal.h"

namespace iq {

static double phi(double x) { return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI); }
static double Phi(double x) {
  if (x == -INFINITY) return 0.0;
  if (x == INFINITY) return 1.0;
  return 0.5 * std::erfc(-x / std::sqrt(2.0));
}

Codebook compute_codebook(int bits) {
  // 2^bits levels; start from the means of equal-probability cells (edges by bisection).
  const int n = 1 << bits;
  double edges[17];
  edges[0] = -INFINITY;
  edges[n] = INFINITY;
  for (int k = 1; k < n; ++k) {
    double lo = -10.0, hi = 10.0;
    for (int it = 0; it < 200; ++it) {
      double mid = 0.5 * (lo + hi);
      if (Phi(mid) < double(k) / n) lo = mid; else hi = mid;
    }
    edges[k] = 0.5 * (lo + hi);
  }
  double c[16];
  for (int k = 0; k < n; ++k) c[k] = (phi(edges[k]) - phi(edges[k + 1])) / (Phi(edges[k + 1]) - Phi(edges[k]));
  for (int it = 0; it < 200000; ++it) {
    double e[17];
    e[0] = -INFINITY;
    e[n] = INFINITY;
    for (int k = 1; k < n; ++k) e[k] = 0.5 * (c[k - 1] + c[k]);
    double nc[16], delta = 0.0;
    for (int k = 0; k < n; ++k) nc[k] = (phi(e[k]) - phi(e[k + 1])) / (Phi(e[k + 1]) - Phi(e[k]));
    for (int k = 0; k < n; ++k) {  // the Gaussian is symmetric: keep the levels odd-symmetric
      double v = 0.5 * (nc[k] - nc[n - 1 - k]);
      delta = std::fmax(delta, std::fabs(v - c[k]));
      c[k] = v;
    }
    if (delta < 1e-15) break;
  }
  Codebook cb;
  cb.bits = bits;
  for (int k = 0; k < n; ++k) cb.level[k] = c[k];
  for (int k = 0; k < n - 1; ++k) cb.bound[k] = 0.5 * (c[k] + c[k + 1]);
  return cb;
}

// ---------------------------------------------------------------- seeded quaternions
static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
static const uint64_t kGolden = 0x9E3779B97F4A7C15ull;

struct Stream {
  uint64_t key, i;
  Stream(uint64_t seed, uint64_t sid) : key(mix64(seed + kGolden) ^ mix64(sid + 2 * kGolden)), i(0) {}
  double uniform() {  // top 53 bits of the i-th output, scaled to [0, 1)
    ++i;
    uint64_t r = mix64(key + i * kGolden);
    return double(r >> 11) * (1.0 / 9007199254740992.0);
  }
};

// Stream of one quaternion (rot ROT_ISO: block, side 0 = qL / 1 = qR; ROT_QUAT: block, side 0)
// or one Givens pair (ROT_PLANAR: pair index as the block, side 0).
static uint64_t stream_id(uint64_t rot, uint64_t layer, uint64_t head, uint64_t block, uint64_t side) {
  return ((((rot * 65536ull + layer) * 65536ull + head) * 64ull + block) * 2ull + side);
}

void unit_quaternion(uint64_t seed, uint64_t sid, double q[4]) {
  Stream st(seed, sid);
  double x1, x2, s1, x3, x4, s2;
  for (;;) {
    x1 = 2.0 * st.uniform() - 1.0;
    x2 = 2.0 * st.uniform() - 1.0;
    s1 = x1 * x1 + x2 * x2;
    if (s1 < 1.0) break;
  }
  for (;;) {
    x3 = 2.0 * st.uniform() - 1.0;
    x4 = 2.0 * st.uniform() - 1.0;
    s2 = x3 * x3 + x4 * x4;
    if (s2 > 0.0 && s2 < 1.0) break;
  }
  double t = std::sqrt((1.0 - s1) / s2);
  q[0] = x1;
  q[1] = x2;
  q[2] = x3 * t;
  q[3] = x4 * t;
}

// A uniform point on the unit circle: a point of the open unit disc without its centre
// (rejection), divided by its length.
static void unit_circle(uint64_t seed, uint64_t sid, double cs[2]) {
  Stream st(seed, sid);
  double x, y, r2;
  for (;;) {
    x = 2.0 * st.uniform() - 1.0;
    y = 2.0 * st.uniform() - 1.0;
    r2 = x * x + y * y;
    if (r2 > 0.0 && r2 < 1.0) break;
  }
  const double r = std::sqrt(r2);
  cs[0] = x / r;
  cs[1] = y / r;
}

void init_rotation_params(uint64_t seed, int rot, int n_layers, int n_kv_heads, float* out) {
  const int pph = params_per_head(rot);
  for (int l = 0; l < n_layers; ++l)
    for (int h = 0; h < n_kv_heads; ++h) {
      float* dst = out + ((size_t)l * n_kv_heads + h) * pph;
      if (rot == ROT_ISO) {
        for (int k = 0; k < 32; ++k)
          for (int side = 0; side < 2; ++side) {
            double q[4];
            unit_quaternion(seed, stream_id(0, l, h, k, side), q);
            for (int i = 0; i < 4; ++i) dst[(k * 2 + side) * 4 + i] = (float)q[i];
          }
      } else if (rot == ROT_QUAT) {
        for (int k = 0; k < 32; ++k) {
          double q[4];
          unit_quaternion(seed, stream_id(1, l, h, k, 0), q);
          for (int i = 0; i < 4; ++i) dst[k * 4 + i] = (float)q[i];
        }
      } else {
        for (int i = 0; i < 64; ++i) {
          double cs[2];
          unit_circle(seed, stream_id(2, l, h, i, 0), cs);
          dst[2 * i] = (float)cs[0];
          dst[2 * i + 1] = (float)cs[1];
        }
      }
    }
}

}  // namespace iq
