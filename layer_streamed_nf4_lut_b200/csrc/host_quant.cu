// Host-side NF4 quantiser: the same format and the same decisions as the device quantiser in
// quant.cu, for callers that hand the library float32 weights in host memory (the base model
// never has to be on the GPU in float32: the pages keep it in CPU RAM and feed the GPU one
// quantised layer at a time, rug.gal radar "Soup ... layer streaming", "En detalle").
//
// Format, per tensor of n row-major elements: blocks of 64; absmax m; code = argmin_j |w/m - c_j|
// in float64 with the lowest index on ties (m = 0: the code of 0.0); element 2i in the low nibble
// of byte i; mean = float32(sequential float64 sum of m / nb); per group of 256 blocks s2 =
// float32(max |m - mean| / 127) (1 if 0), q8 = clamp(round-half-even((m - mean) / s2), +-127) in
// float64.  Every decision is taken in IEEE float64 on exact inputs, so this code and the GPU
// kernels give the same bytes.
#include "../../include/soup.h"
#include "internal.h"

#include <algorithm>
#include <cmath>
#include <thread>
#include <vector>

const soup::LUT16& soup_codebook_lut();

namespace soup {

namespace {

int worker_count(int requested, long long units) {
  int n = requested;
  if (n <= 0) {
    const unsigned hc = std::thread::hardware_concurrency();
    n = hc ? static_cast<int>(hc) : 1;
  }
  n = std::min(n, 64);
  if (units < n) n = static_cast<int>(std::max(1ll, units));
  return n;
}

// Runs f(lo, hi) over [0, units) split into `workers` contiguous ranges.
template <class F>
void parallel_ranges(long long units, int workers, F&& f) {
  if (workers <= 1) {
    f(0ll, units);
    return;
  }
  std::vector<std::thread> th;
  th.reserve(workers);
  for (int t = 0; t < workers; ++t) {
    const long long lo = units * t / workers, hi = units * (t + 1) / workers;
    th.emplace_back([&f, lo, hi] { f(lo, hi); });
  }
  for (auto& x : th) x.join();
}

int nearest_code(float w, double m, const double (&c)[16]) {
  const double r = static_cast<double>(w) / m;
  int best = 0;
  double bd = std::fabs(r - c[0]);
  for (int j = 1; j < 16; ++j) {
    const double d = std::fabs(r - c[j]);
    if (d < bd) {
      bd = d;
      best = j;
    }
  }
  return best;
}

}  // namespace

int host_nf4_quantize(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales, float* mean,
                      int threads) {
  if (!w || n <= 0 || !codes || !q8 || !scales || !mean) return SOUP_ERR_INVALID_ARG;
  const LUT16& lut = soup_codebook_lut();
  double c[16];
  int zero_code = 0;
  for (int j = 0; j < 16; ++j) {
    c[j] = static_cast<double>(lut.v[j]);
    if (lut.v[j] == 0.f) zero_code = j;
  }
  const long long nb = (n + 63) / 64, ng = (nb + 255) / 256;
  std::vector<float> absmax(static_cast<size_t>(nb));
  // codes and absmax, block by block
  parallel_ranges(nb, worker_count(threads, nb), [&](long long lo, long long hi) {
    for (long long b = lo; b < hi; ++b) {
      const long long e0 = b * 64, e1 = std::min(n, e0 + 64);
      float m = 0.f;
      for (long long e = e0; e < e1; ++e) m = std::max(m, std::fabs(w[e]));
      absmax[b] = m;
      const double md = static_cast<double>(m);
      for (long long e = e0; e < e1; e += 2) {
        const int lo4 = m > 0.f ? nearest_code(w[e], md, c) : zero_code;
        int hi4 = 0;
        if (e + 1 < e1) hi4 = m > 0.f ? nearest_code(w[e + 1], md, c) : zero_code;
        codes[e >> 1] = static_cast<uint8_t>(lo4 | (hi4 << 4));
      }
    }
  });
  // mean: sequential float64 sum in block order
  double acc = 0.0;
  for (long long b = 0; b < nb; ++b) acc += static_cast<double>(absmax[b]);
  const float mu_f = static_cast<float>(acc / static_cast<double>(nb));
  *mean = mu_f;
  const double mu = static_cast<double>(mu_f);
  // double quantisation, group by group
  parallel_ranges(ng, worker_count(threads, ng), [&](long long lo, long long hi) {
    for (long long g = lo; g < hi; ++g) {
      const long long b0 = g * 256, b1 = std::min(nb, b0 + 256);
      double amax = 0.0;
      for (long long b = b0; b < b1; ++b) amax = std::max(amax, std::fabs(static_cast<double>(absmax[b]) - mu));
      const float s2 = amax > 0.0 ? static_cast<float>(amax / 127.0) : 1.0f;
      scales[g] = s2;
      const double s2d = static_cast<double>(s2);
      for (long long b = b0; b < b1; ++b) {
        double q = std::nearbyint((static_cast<double>(absmax[b]) - mu) / s2d);  // ties to even
        q = std::min(127.0, std::max(-127.0, q));
        q8[b] = static_cast<int8_t>(q);
      }
    }
  });
  return SOUP_OK;
}

}  // namespace soup

extern "C" soup_status soup_nf4_quantize_host(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales,
                                              float* mean, int n_threads) {
  try {
    return soup::host_nf4_quantize(w, n, codes, q8, scales, mean, n_threads);
  } catch (...) {
    return SOUP_ERR_OOM;
  }
}
