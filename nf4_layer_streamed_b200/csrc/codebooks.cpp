// Code tables of the double-quantised NF4 format, built on the host from the
// published constructions.  "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §2.4: the NF4
// table (16 fp32) and the nested table (256 fp32) are constant for every weight,
// so one resident copy is shared and the shard records their hash.
//
// NF4 (QLoRA, Dettmers et al. 2023, §3): normal quantiles taken asymmetrically so
// that 0 is exact.  8 positive values at probabilities delta + i (1/2 - delta)/8,
// 7 negative ones at delta + i (1/2 - delta)/7 (negated), plus 0; all divided by
// the largest.  delta = ((1 - 1/30) + (1 - 1/32)) / 2.  The quantile function is
// evaluated by bisection on Phi(x) = erfc(-x / sqrt 2) / 2 in double precision.
//
// Nested 8-bit table: signed dynamic tree quantisation (Dettmers 2016).  For
// decade level i = 0..6 with scale 10^(i-6), the 2^i midpoints of an even split
// of [0.1, 1] into 2^i intervals, with both signs; plus 0 and 1.  Sorted.
//
// Both tables are computed in double precision and rounded once to fp32.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace nf4ls {

namespace {

double normal_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double normal_quantile(double p) {
  double lo = -10.0, hi = 10.0;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (normal_cdf(mid) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

uint64_t fnv1a(const uint8_t* data, size_t n, uint64_t h) {
  for (size_t i = 0; i < n; ++i) {
    h ^= data[i];
    h *= 0x100000001B3ull;
  }
  return h;
}

void build(Codebooks* cb) {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  std::vector<double> pos, neg;
  const double step8 = (0.5 - delta) / 8.0, step7 = (0.5 - delta) / 7.0;
  for (int i = 0; i < 8; ++i) pos.push_back(normal_quantile(delta + i * step8));
  for (int i = 0; i < 7; ++i) neg.push_back(-normal_quantile(delta + i * step7));
  const double top = pos[0];
  std::vector<double> v;
  for (double x : pos) v.push_back(x / top);
  v.push_back(0.0);
  for (double x : neg) v.push_back(x / top);
  std::sort(v.begin(), v.end());
  for (int i = 0; i < 16; ++i) cb->nf4[i] = static_cast<float>(v[i]);

  static const double decades[7] = {1e-6, 1e-5, 1e-4, 1e-3, 1e-2, 1e-1, 1.0};
  std::vector<double> c{0.0, 1.0};
  for (int i = 0; i < 7; ++i) {
    const int n = 1 << i;
    const double step = 0.9 / n;
    for (int j = 0; j < n; ++j) {
      const double b0 = 0.1 + j * step, b1 = 0.1 + (j + 1) * step;
      const double mid = (b0 + b1) / 2.0;
      c.push_back(decades[i] * mid);
      c.push_back(-decades[i] * mid);
    }
  }
  std::sort(c.begin(), c.end());
  for (int i = 0; i < 256; ++i) cb->code8[i] = static_cast<float>(c[i]);

  for (int i = 0; i < 15; ++i)
    cb->mid4[i] = static_cast<float>(((double)cb->nf4[i] + (double)cb->nf4[i + 1]) / 2.0);
  for (int i = 0; i < 255; ++i)
    cb->mid8[i] = static_cast<float>(((double)cb->code8[i] + (double)cb->code8[i + 1]) / 2.0);
  cb->zero4 = cb->zero8 = -1;
  for (int i = 0; i < 16; ++i)
    if (cb->nf4[i] == 0.0f) cb->zero4 = i;
  for (int i = 0; i < 256; ++i)
    if (cb->code8[i] == 0.0f) cb->zero8 = i;

  uint64_t h = 0xCBF29CE484222325ull;
  h = fnv1a(reinterpret_cast<const uint8_t*>(cb->nf4), sizeof(cb->nf4), h);
  h = fnv1a(reinterpret_cast<const uint8_t*>(cb->code8), sizeof(cb->code8), h);
  cb->hash = h;
}

}  // namespace

const Codebooks& codebooks() {
  static Codebooks cb;
  static std::once_flag once;
  std::call_once(once, [] { build(&cb); });
  return cb;
}

}  // namespace nf4ls

extern "C" int nf4ls_codebooks(float nf4_host[16], float code8_host[256], uint64_t* hash) {
  const nf4ls::Codebooks& cb = nf4ls::codebooks();
  if (nf4_host) std::memcpy(nf4_host, cb.nf4, sizeof(cb.nf4));
  if (code8_host) std::memcpy(code8_host, cb.code8, sizeof(cb.code8));
  if (hash) *hash = cb.hash;
  return NF4LS_OK;
}
