// RoPE / YaRN cos-sin tables (one elementwise kernel).
//
// Plain RoPE pairs element i with i + d/2 (rotate_half, MiniMind "Attention
// 前向传播" section 3) and rotates the pair by t * theta_i, theta_i =
// base^(-2i/d).  YaRN frequencies follow the NTK-by-parts reading of the
// parameters listed in the Megatron-LM MLA guide (MLA 专属参数详解): a linear
// ramp between the correction dimensions of beta_fast and beta_slow blends
// theta_i (kept) with theta_i / s (interpolated), and the table magnitude is
// m(s, mscale) / m(s, mscale_all_dim) with m(s, a) = 0.1 a ln s + 1.
#include <cmath>

#include "internal.h"

namespace mla {
namespace {

struct RopeK {
  double log_base;    // ln(base)
  double factor;      // s (1 for plain)
  double lo, hi;      // ramp end points (yarn); lo >= d when no ramp
  double mag;
  int d, half, max_pos;
  int mode;           // 0 none, 1 plain, 2 yarn
};

__global__ void rope_tables_kernel(RopeK k, float* __restrict__ cos_out,
                                   float* __restrict__ sin_out) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)k.max_pos * k.half;
  if (idx >= total) return;
  const int t = (int)(idx / k.half);
  const int i = (int)(idx % k.half);
  double c = 1.0, s = 0.0;
  if (k.mode != 0) {
    double theta = exp(-2.0 * (double)i / (double)k.d * k.log_base);
    if (k.mode == 2) {
      double r = ((double)i - k.lo) / (k.hi - k.lo);
      r = r < 0.0 ? 0.0 : (r > 1.0 ? 1.0 : r);
      theta = (1.0 - r) * theta + r * (theta / k.factor);
    }
    const double ang = (double)t * theta;
    sincos(ang, &s, &c);
    c *= k.mag;
    s *= k.mag;
  }
  const int64_t row = (int64_t)t * k.d;
  cos_out[row + i] = (float)c;
  cos_out[row + i + k.half] = (float)c;
  sin_out[row + i] = (float)s;
  sin_out[row + i + k.half] = (float)s;
}

double yarn_m(double s, double a) { return s <= 1.0 ? 1.0 : 0.1 * a * std::log(s) + 1.0; }

}  // namespace

cudaError_t launch_rope_tables(const mla_config& cfg, int max_pos, float* cos,
                               float* sin, cudaStream_t st) {
  RopeK k{};
  k.d = cfg.qk_rope_head_dim;
  k.half = k.d / 2;
  k.max_pos = max_pos;
  k.mode = cfg.rope_type;
  k.log_base = std::log(cfg.rope_theta);
  k.factor = cfg.rope_factor;
  k.mag = 1.0;
  k.lo = 0.0;
  k.hi = 1.0;
  if (cfg.rope_type == MLA_ROPE_YARN) {
    const double d = k.d, L = cfg.original_max_position_embeddings;
    auto corr = [&](double b) {
      return d * std::log(L / (b * 2.0 * M_PI)) / (2.0 * k.log_base);
    };
    double lo = std::max(std::floor(corr(cfg.beta_fast)), 0.0);
    double hi = std::min(std::ceil(corr(cfg.beta_slow)), d - 1.0);
    if (lo == hi) hi += 0.001;
    k.lo = lo;
    k.hi = hi;
    k.mag = yarn_m(cfg.rope_factor, cfg.rope_mscale) /
            yarn_m(cfg.rope_factor, cfg.rope_mscale_all_dim);
  }
  const int64_t total = (int64_t)max_pos * k.half;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  rope_tables_kernel<<<(unsigned)blocks, threads, 0, st>>>(k, cos, sin);
  count_launches();
  return cudaGetLastError();
}

}  // namespace mla
