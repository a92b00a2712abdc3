// Host-side codebook construction (nsn_build_codebook_host in include/nsn.h).
//
// "NSNQuant: A Double Normalization Approach ...", technical summary,
// Metodologia 3: the single global codebook is initialised by k-means on
// synthetic standard-normal data; the README's "Codebook tuning" builds the
// 2-bit codebook over absolute values (--abs).
//
// The same passage: the k-means codebook is then fine-tuned to minimise the
// cosine distance between vectors and their quantized versions
// (nsn_build_codebook_cosine_host; the README's "--method learned").
//
// Standard normals: Philox4x64-10 counter-based generator (Salmon, Moraes, Dror,
// Shaw, SC'11) + Box-Muller transform (Box & Muller, 1958); stream layout in nsn.h.

#include <cmath>
#include <cstdint>
#include <vector>

#include <cuda_fp16.h>

#include "nsn.h"

namespace {

constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ull;
constexpr uint64_t kM1 = 0xCA5A826395121157ull;
constexpr uint64_t kW0 = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kW1 = 0xBB67AE8584CAA73Bull;
constexpr uint64_t kStreamKey1 = 0x4E534E51ull;

struct Block4 {
  uint64_t w[4];
};

Block4 philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3, uint64_t k0, uint64_t k1) {
  for (int r = 0; r < 10; ++r) {
    const unsigned __int128 p0 = (unsigned __int128)kM0 * c0;
    const unsigned __int128 p1 = (unsigned __int128)kM1 * c2;
    const uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
    const uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
    const uint64_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    k0 += kW0;
    k1 += kW1;
  }
  return Block4{{c0, c1, c2, c3}};
}

double uniform_open(uint64_t w) { return ((double)(w >> 12) + 0.5) * 0x1.0p-52; }

void normal_stream(uint64_t seed, size_t count, double* out) {
  const double two_pi = 2.0 * M_PI;
  for (size_t j = 0; 4 * j < count; ++j) {
    const Block4 b = philox4x64_10(j, 0, 0, 0, seed, kStreamKey1);
    double z[4];
    for (int pr = 0; pr < 2; ++pr) {
      const double ua = uniform_open(b.w[2 * pr]), ub = uniform_open(b.w[2 * pr + 1]);
      const double r = std::sqrt(-2.0 * std::log(ua));
      z[2 * pr] = r * std::cos(two_pi * ub);
      z[2 * pr + 1] = r * std::sin(two_pi * ub);
    }
    for (int i = 0; i < 4 && 4 * j + i < count; ++i) out[4 * j + i] = z[i];
  }
}

// Lloyd k-means from the first k samples (ties to the lowest centroid, empty
// clusters keep their centroid); `label` receives the last assignment.
void assign(const std::vector<double>& x, const std::vector<double>& cent, size_t n, size_t k, size_t d,
            std::vector<int32_t>& label) {
  for (size_t i = 0; i < n; ++i) {
    const double* xi = &x[i * d];
    double best = INFINITY;
    int32_t bi = 0;
    for (size_t c = 0; c < k; ++c) {
      const double* cc = &cent[c * d];
      double s = 0.0;
      for (size_t e = 0; e < d; ++e) {
        const double df = xi[e] - cc[e];
        s += df * df;
      }
      if (s < best) {
        best = s;
        bi = (int32_t)c;
      }
    }
    label[i] = bi;
  }
}

void kmeans(const std::vector<double>& x, std::vector<double>& cent, size_t n, size_t k, size_t d, int iters) {
  std::vector<double> sums(k * d);
  std::vector<int64_t> counts(k);
  std::vector<int32_t> label(n);
  for (int it = 0; it < iters; ++it) {
    assign(x, cent, n, k, d, label);
    std::fill(sums.begin(), sums.end(), 0.0);
    std::fill(counts.begin(), counts.end(), 0);
    for (size_t i = 0; i < n; ++i) {
      const size_t c = (size_t)label[i];
      counts[c] += 1;
      for (size_t e = 0; e < d; ++e) sums[c * d + e] += x[i * d + e];
    }
    for (size_t c = 0; c < k; ++c)
      if (counts[c] > 0)
        for (size_t e = 0; e < d; ++e) cent[c * d + e] = sums[c * d + e] / (double)counts[c];
  }
}

// Cosine fine-tuning.  With the samples assigned to their nearest codeword (as
// the quantizer assigns), codeword c is turned to the direction that maximises
// the summed cosine with its members -- the normalised sum of their unit
// vectors -- and given the least-squares length along it, the mean projection
// of its members.  Codewords without members, with a zero direction sum or a
// non-positive mean projection are kept.
void cosine_finetune(const std::vector<double>& x, std::vector<double>& cent, size_t n, size_t k, size_t d,
                     int iters) {
  std::vector<double> unit(n * d);
  for (size_t i = 0; i < n; ++i) {
    double ss = 0.0;
    for (size_t e = 0; e < d; ++e) ss += x[i * d + e] * x[i * d + e];
    const double nr = std::sqrt(ss);
    for (size_t e = 0; e < d; ++e) unit[i * d + e] = nr > 0.0 ? x[i * d + e] / nr : 0.0;
  }
  std::vector<double> dir(k * d), proj(k);
  std::vector<int64_t> counts(k);
  std::vector<int32_t> label(n);
  for (int it = 0; it < iters; ++it) {
    assign(x, cent, n, k, d, label);
    std::fill(dir.begin(), dir.end(), 0.0);
    std::fill(counts.begin(), counts.end(), 0);
    for (size_t i = 0; i < n; ++i) {
      const size_t c = (size_t)label[i];
      counts[c] += 1;
      for (size_t e = 0; e < d; ++e) dir[c * d + e] += unit[i * d + e];
    }
    for (size_t c = 0; c < k; ++c) {
      double ss = 0.0;
      for (size_t e = 0; e < d; ++e) ss += dir[c * d + e] * dir[c * d + e];
      const double nr = std::sqrt(ss);
      for (size_t e = 0; e < d; ++e) dir[c * d + e] = nr > 0.0 ? dir[c * d + e] / nr : 0.0;
    }
    std::fill(proj.begin(), proj.end(), 0.0);
    for (size_t i = 0; i < n; ++i) {
      const size_t c = (size_t)label[i];
      double p = 0.0;
      for (size_t e = 0; e < d; ++e) p += x[i * d + e] * dir[c * d + e];
      proj[c] += p;
    }
    for (size_t c = 0; c < k; ++c) {
      if (counts[c] == 0) continue;
      const double len = proj[c] / (double)counts[c];
      if (!(len > 0.0)) continue;
      for (size_t e = 0; e < d; ++e) cent[c * d + e] = dir[c * d + e] * len;
    }
  }
}

std::vector<double> samples(uint64_t seed, size_t n, size_t d, int abs_mode) {
  std::vector<double> x(n * d);
  normal_stream(seed, n * d, x.data());
  if (abs_mode)
    for (double& v : x) v = std::fabs(v);
  return x;
}

void store_f16(const std::vector<double>& cent, size_t count, float* out) {
  for (size_t i = 0; i < count; ++i) out[i] = __half2float(__double2half(cent[i]));
}

}  // namespace

extern "C" nsn_status nsn_build_codebook_host(uint64_t seed, int n_samples, int n_codes, int dim, int abs_mode,
                                              int iters, float* out) {
  if (!out || n_codes <= 0 || dim <= 0 || n_samples < n_codes || iters < 0) return NSN_ERR_INVALID_ARG;
  const size_t n = (size_t)n_samples, k = (size_t)n_codes, d = (size_t)dim;
  const std::vector<double> x = samples(seed, n, d, abs_mode);
  std::vector<double> cent(x.begin(), x.begin() + k * d);  // first n_codes samples
  kmeans(x, cent, n, k, d, iters);
  store_f16(cent, k * d, out);
  return NSN_OK;
}

extern "C" nsn_status nsn_build_codebook_cosine_host(uint64_t seed, int n_samples, int n_codes, int dim,
                                                     int abs_mode, int kmeans_iters, int cosine_iters, float* out) {
  if (!out || n_codes <= 0 || dim <= 0 || n_samples < n_codes || kmeans_iters < 0 || cosine_iters < 0)
    return NSN_ERR_INVALID_ARG;
  const size_t n = (size_t)n_samples, k = (size_t)n_codes, d = (size_t)dim;
  const std::vector<double> x = samples(seed, n, d, abs_mode);
  std::vector<double> cent(x.begin(), x.begin() + k * d);
  kmeans(x, cent, n, k, d, kmeans_iters);
  cosine_finetune(x, cent, n, k, d, cosine_iters);
  store_f16(cent, k * d, out);
  return NSN_OK;
}

// Double quantization of the codebook entries ([TS] Metodologia 3: the codebook
// entries are stored in 4 bits as well): 16 uniform levels between the
// fp16-rounded min and max of all entries, level = round-half-even((x - lo) /
// step) clamped to 0..15, step = (hi - lo) / 15; each entry becomes the fp16
// rounding of lo + level * step, so the quantizer and the fp16 decode read the
// same values.
extern "C" nsn_status nsn_codebook_4bit_host(float* codebook, int n_values) {
  if (!codebook || n_values <= 0) return NSN_ERR_INVALID_ARG;
  double mn = INFINITY, mx = -INFINITY;
  for (int i = 0; i < n_values; ++i) {
    mn = std::fmin(mn, (double)codebook[i]);
    mx = std::fmax(mx, (double)codebook[i]);
  }
  const double lo = (double)__half2float(__double2half(mn));
  const double hi = (double)__half2float(__double2half(mx));
  const double step = (hi - lo) / 15.0;
  for (int i = 0; i < n_values; ++i) {
    double level = 0.0;
    if (step > 0.0) level = std::fmin(15.0, std::fmax(0.0, std::nearbyint(((double)codebook[i] - lo) / step)));
    codebook[i] = __half2float(__double2half(lo + level * step));
  }
  return NSN_OK;
}
