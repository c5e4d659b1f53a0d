// Host-side table construction for the Block-GTQ library: Lloyd-Max
// codebooks, Haar rotations, exact-score greedy allocation, group layouts.
#pragma once
#include <cstdint>
#include <vector>

namespace bgtq {

constexpr int kHeadDim = 128;
constexpr int kBlocks = kHeadDim / 2;
constexpr int kMaxBits = 4;
constexpr int kMaxGroups = 4;

// N(0,1) Lloyd-Max mean-squared errors used as the greedy's distortion
// model (six-digit constants, index = width).
extern const double kDistortion[kMaxBits + 1];

// Codebook of 2^bits levels: the double Lloyd-Max levels rounded once to
// binary16 (held as exact floats) and the 2^bits-1 exact midpoints.
void lloyd_max_codebook(int bits, std::vector<float>* centroids, std::vector<float>* thresholds);

// SplitMix64 (Steele, Lea, Flood 2014).
struct SplitMix64 {
  uint64_t state;
  explicit SplitMix64(uint64_t s) : state(s) {}
  uint64_t next();
  double uniform();  // [0, 1), 53 bits
};

uint64_t rotation_key(uint64_t seed, uint64_t layer, uint64_t head, uint64_t kind, uint64_t width);

// Haar orthogonal d x d matrix (row-major, double): Box-Muller normals from
// the key's SplitMix64 stream, Householder QR, columns signed so R's
// diagonal is positive (Mezzadri 2007).
std::vector<double> haar_rotation(int d, uint64_t key);

// Correctly rounded (to nearest, ties to even) conversion of an unsigned
// 128-bit integer given as (lo, hi) to double.
double u128_to_double(uint64_t lo, uint64_t hi);

// Greedy marginal-gain allocation over kBlocks scores; returns widths.
std::vector<int> greedy_allocate(const double* scores, int avg_bits, int b_min, int b_max);

// Dims of RoPE block j: pairing 0 -> (j, j+64), 1 -> (2j, 2j+1).
void block_dims(int j, int pairing, int* a, int* b);

struct GroupLayout {
  int n_groups = 0;
  int width[kMaxGroups] = {0, 0, 0, 0};
  int size[kMaxGroups] = {0, 0, 0, 0};
  int start[kMaxGroups] = {0, 0, 0, 0};    // first record position
  int bitoff[kMaxGroups] = {0, 0, 0, 0};   // first bit in the record
  int perm[kHeadDim];                      // record position -> original dim
  int n_positions = 0;                     // positions with width > 0
};

// Groups of equal width, widest first, dims ascending inside; width-0
// blocks are left out of the record.
GroupLayout build_layout(const int* block_widths, int pairing);

}  // namespace bgtq
