// Host check of msa::exp2_fma (block_sparse_long_exp_b200/csrc/msa_exp2.cuh):
// the function is plain fp32 arithmetic with explicitly rounded operations,
// so its host build gives the device results bit for bit.  Compared with
// exp2 in double precision over every 64th float of [-125, 10], a seeded
// uniform sample of [-125, 10], the floats next to every integer and half
// integer of [-125, 10], and the special inputs.  Prints the largest relative
// error; exits non-zero when a check fails.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <limits>

#include "msa_exp2.cuh"

static double worst = 0.0;
static float worst_x = 0.0f;
static long checked = 0, failures = 0;
static const double kBound = 7.6e-5;

static float from_bits(uint32_t u) { float x; std::memcpy(&x, &u, 4); return x; }
static uint32_t to_bits(float x) { uint32_t u; std::memcpy(&u, &x, 4); return u; }

static void check(float x) {
  const double ref = std::exp2((double)x);
  const float got = msa::exp2_fma(x);
  const double rel = std::fabs((double)got / ref - 1.0);
  ++checked;
  if (!(rel <= kBound) || !std::isnormal(got)) {
    if (failures++ < 10) std::printf("FAIL x=%.9g got=%.9g ref=%.9g rel=%.3e\n", x, got, ref, rel);
  }
  if (rel > worst) { worst = rel; worst_x = x; }
}

int main() {
  // every 64th float of [-125, 0] and of [0, 10]
  for (uint32_t u = 0x80000000u; u <= to_bits(-125.0f); u += 64) check(from_bits(u));
  for (uint32_t u = 0; u <= to_bits(10.0f); u += 64) check(from_bits(u));
  // seeded uniform sample of [-125, 10] (64-bit LCG, top 24 bits)
  uint64_t s = 0x9E3779B97F4A7C15ull;
  for (int i = 0; i < 4000000; ++i) {
    s = s * 6364136223846793005ull + 1442695040888963407ull;
    const float u = (float)(s >> 40) * (1.0f / 16777216.0f);
    check(-125.0f + 135.0f * u);
  }
  // around integers and half integers (the rounding step's ties and edges)
  for (int k = -250; k <= 20; ++k) {
    const float c = 0.5f * (float)k;
    uint32_t b = to_bits(c);
    for (int d = -4; d <= 4; ++d) {
      const float x = (c == 0.0f) ? from_bits((d < 0 ? 0x80000000u : 0u) + (uint32_t)std::abs(d))
                                  : from_bits(b + (uint32_t)d);
      if (x >= -125.0f && x <= 10.0f) check(x);
    }
  }
  check(127.0f);
  check(-125.0f);
  // below the domain: exactly zero
  const float inf = std::numeric_limits<float>::infinity();
  const float zeros[] = {-inf, std::nextafter(-125.0f, -inf), -126.0f, -1e30f, std::nanf("")};
  for (float x : zeros) {
    ++checked;
    if (msa::exp2_fma(x) != 0.0f || std::signbit(msa::exp2_fma(x))) {
      ++failures;
      std::printf("FAIL x=%.9g should give +0, got %.9g\n", x, msa::exp2_fma(x));
    }
  }
  std::printf("checked %ld inputs, %ld failures, largest relative error %.4e at x=%.9g\n", checked, failures,
              worst, worst_x);
  return failures == 0 ? 0 : 1;
}
