// Host-side generation of the Gaussian JL matrices S and S_out.
//
// QJL summary (atlas.scime.ai), Approach: keys are multiplied by a random
// Gaussian JL matrix. Entries are i.i.d. N(0,1), drawn as follows:
//   * SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): output n of the stream
//     `seed` is mix64(seed + n * 0x9E3779B97F4A7C15), where mix64 is
//     xor-shift 30, multiply 0xBF58476D1CE4E5B9, xor-shift 27, multiply
//     0x94D049BB133111EB, xor-shift 31.
//   * uniform in (0,1): ((x >> 12) + 1/2) * 2^-52.
//   * Box-Muller, cosine branch: sqrt(-2 ln u1) * cos(2 pi u2), with u1, u2
//     from outputs offset + 2e + 1 and offset + 2e + 2 for row-major element e.
//   * rounded to the nearest bfloat16, ties to even.
#include <cmath>
#include <cstring>

#include "qjl_internal.cuh"

namespace qjl {

static inline uint64_t splitmix64_output(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline double open_unit(uint64_t x) { return (static_cast<double>(x >> 12) + 0.5) * 0x1p-52; }

// Nearest bfloat16 to a double (ties to even), for finite values in bf16's normal range.
static inline uint16_t bf16_bits_nearest(double v) {
  uint64_t b;
  std::memcpy(&b, &v, sizeof b);
  const uint64_t low = (1ull << 45) - 1;  // fraction bits that bf16 drops
  b = (b + ((1ull << 44) - 1) + ((b >> 45) & 1ull)) & ~low;
  double r;
  std::memcpy(&r, &b, sizeof r);
  const float f = static_cast<float>(r);  // exact: r has at most 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  return static_cast<uint16_t>(u >> 16);
}

void sketch_fill_host(uint64_t seed, uint64_t counter_offset, int rows, int d, uint16_t* out) {
  const double two_pi = 6.283185307179586;
  const uint64_t n = static_cast<uint64_t>(rows) * static_cast<uint64_t>(d);
  for (uint64_t e = 0; e < n; ++e) {
    const double u1 = open_unit(splitmix64_output(seed, counter_offset + 2 * e + 1));
    const double u2 = open_unit(splitmix64_output(seed, counter_offset + 2 * e + 2));
    const double g = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
    out[e] = bf16_bits_nearest(g);
  }
}

}  // namespace qjl
