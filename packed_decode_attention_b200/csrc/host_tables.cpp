// Host-side tables.  Each routine follows a published definition:
//  * Lloyd-Max quantiser for N(0,1): Lloyd (1957/1982), Max (1960) -- the
//    scalar codebook of TurboQuant-MSE (arXiv 2504.19874), the encoder the
//    Block-GTQ pages build on;
//  * Haar rotation: SplitMix64 (Steele et al. 2014) -> Box-Muller (1958) ->
//    Householder QR with Mezzadri's (2007) sign fix;
//  * greedy marginal-gain bit allocation: the Block-GTQ abstract assigns
//    integer widths one greedy step at a time by their marginal gain.
#include "host_tables.h"

#include <algorithm>
#include <cmath>
#include <cstring>

namespace bgtq {

const double kDistortion[kMaxBits + 1] = {1.0, 0.363380, 0.117482, 0.034548, 0.009497};

namespace {

double gauss_pdf(double x) {
  if (std::isinf(x)) return 0.0;
  return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
}

double gauss_cdf(double x) {
  if (x == INFINITY) return 1.0;
  return 0.5 * (1.0 + std::erf(x / std::sqrt(2.0)));
}

// Mean of N(0,1) restricted to (a, b).
double truncated_mean(double a, double b) {
  return (gauss_pdf(a) - gauss_pdf(b)) / (gauss_cdf(b) - gauss_cdf(a));
}

// Positive half of the symmetric codebook, ascending.  Alternates the
// nearest-neighbour (midpoint) and centroid (conditional mean) conditions
// until no level moves by more than 1e-15.
std::vector<double> positive_levels(int bits) {
  const int half = 1 << (bits - 1);
  std::vector<double> c(half);
  if (half == 1) {
    c[0] = truncated_mean(0.0, INFINITY);
    return c;
  }
  for (int k = 0; k < half; ++k) c[k] = (k + 0.5) * 4.0 / half;
  std::vector<double> edge(half + 1), next(half);
  for (int it = 0; it < 100000; ++it) {
    edge[0] = 0.0;
    for (int k = 1; k < half; ++k) edge[k] = 0.5 * (c[k - 1] + c[k]);
    edge[half] = INFINITY;
    double moved = 0.0;
    for (int k = 0; k < half; ++k) {
      next[k] = truncated_mean(edge[k], edge[k + 1]);
      moved = std::max(moved, std::fabs(next[k] - c[k]));
    }
    c = next;
    if (moved <= 1e-15) break;
  }
  return c;
}

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

}  // namespace

// Round a double to the nearest binary16 value (ties to even), returned as a
// double; normal range only (the codebook levels lie in [0.12, 2.8]).
double round_to_fp16(double x) {
  if (x == 0.0) return 0.0;
  int e = 0;
  const double m = std::frexp(x, &e);            // x = m * 2^e, 0.5 <= |m| < 1
  const double q = std::nearbyint(std::ldexp(m, 11));  // 11 significant bits, to nearest even
  return std::ldexp(q, e - 11);
}

void lloyd_max_codebook(int bits, std::vector<float>* centroids, std::vector<float>* thresholds) {
  const std::vector<double> pos = positive_levels(bits);
  const int half = static_cast<int>(pos.size());
  std::vector<double> all(2 * half);
  for (int k = 0; k < half; ++k) {
    all[half + k] = round_to_fp16(pos[k]);
    all[half - 1 - k] = -round_to_fp16(pos[k]);
  }
  centroids->resize(2 * half);
  thresholds->resize(2 * half - 1);
  for (int k = 0; k < 2 * half; ++k) (*centroids)[k] = static_cast<float>(all[k]);
  // midpoints of binary16 values are exact in float32
  for (int k = 0; k + 1 < 2 * half; ++k) (*thresholds)[k] = static_cast<float>(0.5 * (all[k] + all[k + 1]));
}

uint64_t SplitMix64::next() {
  state += kGamma;
  return mix64(state);
}

double SplitMix64::uniform() { return static_cast<double>(next() >> 11) * (1.0 / 9007199254740992.0); }

uint64_t rotation_key(uint64_t seed, uint64_t layer, uint64_t head, uint64_t kind, uint64_t width) {
  uint64_t key = seed;
  const uint64_t fields[4] = {layer, head, kind, width};
  for (uint64_t f : fields) key = SplitMix64(key ^ f).next();
  return key;
}

std::vector<double> haar_rotation(int d, uint64_t key) {
  // Gaussian matrix, row-major, filled two entries per uniform pair.
  std::vector<double> a(static_cast<size_t>(d) * d);
  SplitMix64 gen(key);
  size_t filled = 0;
  while (filled < a.size()) {
    const double u1 = 1.0 - gen.uniform();
    const double u2 = gen.uniform();
    const double r = std::sqrt(-2.0 * std::log(u1));
    const double th = 2.0 * M_PI * u2;
    a[filled++] = r * std::cos(th);
    if (filled < a.size()) a[filled++] = r * std::sin(th);
  }
  // Householder QR: R = H_{d-1} ... H_0 A, A = Q R with Q = H_0 ... H_{d-1}.
  std::vector<double> R = a;
  std::vector<std::vector<double>> vs(d);
  std::vector<double> rdiag(d, 0.0);
  for (int k = 0; k < d; ++k) {
    double norm2 = 0.0;
    for (int i = k; i < d; ++i) norm2 += R[i * d + k] * R[i * d + k];
    const double norm = std::sqrt(norm2);
    if (norm == 0.0) {
      rdiag[k] = 0.0;
      continue;
    }
    const double x0 = R[k * d + k];
    const double alpha = (x0 >= 0.0) ? -norm : norm;
    std::vector<double> v(d - k);
    for (int i = k; i < d; ++i) v[i - k] = R[i * d + k];
    v[0] -= alpha;
    double vv = 0.0;
    for (double x : v) vv += x * x;
    if (vv == 0.0) {
      rdiag[k] = x0;
      continue;
    }
    for (int j = k; j < d; ++j) {
      double s = 0.0;
      for (int i = k; i < d; ++i) s += v[i - k] * R[i * d + j];
      const double f = 2.0 * s / vv;
      for (int i = k; i < d; ++i) R[i * d + j] -= f * v[i - k];
    }
    rdiag[k] = R[k * d + k];
    vs[k] = std::move(v);
  }
  std::vector<double> Q(static_cast<size_t>(d) * d, 0.0);
  for (int i = 0; i < d; ++i) Q[i * d + i] = 1.0;
  for (int k = d - 1; k >= 0; --k) {
    if (vs[k].empty()) continue;
    const std::vector<double>& v = vs[k];
    double vv = 0.0;
    for (double x : v) vv += x * x;
    for (int j = 0; j < d; ++j) {
      double s = 0.0;
      for (int i = k; i < d; ++i) s += v[i - k] * Q[i * d + j];
      const double f = 2.0 * s / vv;
      for (int i = k; i < d; ++i) Q[i * d + j] -= f * v[i - k];
    }
  }
  for (int k = 0; k < d; ++k) {
    if (rdiag[k] < 0.0)
      for (int i = 0; i < d; ++i) Q[i * d + k] = -Q[i * d + k];
  }
  return Q;
}

double u128_to_double(uint64_t lo, uint64_t hi) {
  if (hi == 0) {
    // 64-bit path, rounded by hand the same way as the 128-bit one below.
    if (lo == 0) return 0.0;
  }
  // Position of the top set bit (0..127).
  int top = hi ? 64 + 63 - __builtin_clzll(hi) : 63 - __builtin_clzll(lo);
  if (top < 53) return static_cast<double>(lo);  // exact
  const int drop = top - 52;                      // bits below the 53-bit mantissa
  // mantissa = value >> drop; rest = value & ((1 << drop) - 1)
  unsigned __int128 v = (static_cast<unsigned __int128>(hi) << 64) | lo;
  unsigned __int128 mant = v >> drop;
  unsigned __int128 rest = v - (mant << drop);
  unsigned __int128 halfway = static_cast<unsigned __int128>(1) << (drop - 1);
  if (rest > halfway || (rest == halfway && (mant & 1))) mant += 1;
  // mant <= 2^53 here; ldexp is exact.
  return std::ldexp(static_cast<double>(static_cast<uint64_t>(mant)), drop);
}

std::vector<int> greedy_allocate(const double* scores, int avg_bits, int b_min, int b_max) {
  std::vector<int> w(kBlocks, b_min);
  int left = avg_bits * kBlocks - b_min * kBlocks;
  while (left > 0) {
    int best = -1;
    double best_gain = 0.0;
    for (int j = 0; j < kBlocks; ++j) {
      if (w[j] >= b_max) continue;
      const double gain = scores[j] * (kDistortion[w[j]] - kDistortion[w[j] + 1]);
      if (best < 0 || gain > best_gain) {
        best = j;
        best_gain = gain;
      }
    }
    w[best] += 1;
    --left;
  }
  return w;
}

void block_dims(int j, int pairing, int* a, int* b) {
  if (pairing == 0) {
    *a = j;
    *b = j + kBlocks;
  } else {
    *a = 2 * j;
    *b = 2 * j + 1;
  }
}

GroupLayout build_layout(const int* block_widths, int pairing) {
  int dim_width[kHeadDim];
  for (int j = 0; j < kBlocks; ++j) {
    int a, b;
    block_dims(j, pairing, &a, &b);
    dim_width[a] = block_widths[j];
    dim_width[b] = block_widths[j];
  }
  GroupLayout L;
  std::memset(L.perm, 0, sizeof(L.perm));
  int pos = 0, bit = 0;
  for (int width = kMaxBits; width >= 1; --width) {
    int count = 0;
    for (int d = 0; d < kHeadDim; ++d) count += (dim_width[d] == width);
    if (count == 0) continue;
    const int g = L.n_groups++;
    L.width[g] = width;
    L.size[g] = count;
    L.start[g] = pos;
    L.bitoff[g] = bit;
    for (int d = 0; d < kHeadDim; ++d)
      if (dim_width[d] == width) L.perm[pos++] = d;
    bit += count * width;
  }
  L.n_positions = pos;
  // Width-0 dims take the remaining positions (never stored or read).
  for (int d = 0; d < kHeadDim; ++d)
    if (dim_width[d] == 0) L.perm[pos++] = d;
  return L;
}

}  // namespace bgtq
