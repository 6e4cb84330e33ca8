// Host check of FastDiv (common.cuh): n / d by multiply-high and shift must
// equal the integer quotient for every divisor 1..5000, on the small
// numerators where rounding errors would show first, on random numerators
// up to 2^31 - 1 and on 2^31 - 1 itself.  Exit status 0 when all agree.
#include <algorithm>
using std::min;
#include <cstdio>
#include <random>

#include "common.cuh"

int main() {
  std::mt19937_64 rng(12345);
  long long bad = 0, tests = 0;
  for (uint32_t d = 1; d <= 5000; ++d) {
    const FastDiv f = make_fastdiv(d);
    for (uint32_t n = 0; n < 3 * d + 3; ++n, ++tests)
      if (fdiv(n, f) != n / d) ++bad;
    for (int k = 0; k < 400; ++k, ++tests) {
      const uint32_t n = k == 0 ? 0x7fffffffu : (uint32_t)(rng() & 0x7fffffffu);
      if (fdiv(n, f) != n / d) ++bad;
    }
  }
  std::printf("fastdiv: %lld cases, %lld wrong\n", tests, bad);
  return bad != 0;
}
