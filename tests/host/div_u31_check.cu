// Host check of the launch-time divisor constants of the few-token product
// kernels (make_div_u31 in few_token.cuh): for every divisor tested, the
// multiply-high-and-shift quotient equals n / d for numerators across
// [0, 2^31).  Built and run by tests/test_host_div.py; needs no GPU.
#include <cstdint>
#include <cstdio>
#include <random>

#include "few_token.cuh"

static uint32_t quotient(const qlora::DivU31 &v, uint32_t n) {
  // the device form: __umulhi(n, mul) >> shr, with mul = 0 meaning d = 1
  return v.mul ? (uint32_t)(((uint64_t)n * v.mul) >> 32) >> v.shr : n;
}

int main() {
  std::mt19937_64 rng(12345);
  uint64_t checked = 0, bad = 0;
  auto check_divisor = [&](uint32_t d) {
    const qlora::DivU31 v = qlora::make_div_u31(d);
    auto one = [&](uint32_t n) {
      ++checked;
      if (quotient(v, n) != n / d && bad++ < 10) printf("bad n=%u d=%u\n", n, d);
    };
    for (uint32_t n : {0u, 1u, d - 1, d, d + 1, 0x7FFFFFFEu, 0x7FFFFFFFu}) one(n);
    for (uint64_t k : {1ull, 2ull, 3ull, 1000ull, 0x7FFFFFFFull / d})
      for (int64_t e = -1; e <= 1; ++e) {
        const int64_t n = (int64_t)(k * d) + e;
        if (n >= 0 && n < 0x80000000ll) one((uint32_t)n);
      }
    for (int i = 0; i < 64; ++i) one((uint32_t)(rng() & 0x7FFFFFFFu));
  };
  for (uint32_t d = 1; d <= 70000; ++d) check_divisor(d);
  for (int k = 1; k < 31; ++k)
    for (int e = -1; e <= 1; ++e) check_divisor((uint32_t)((1u << k) + e));
  for (int i = 0; i < 20000; ++i) check_divisor(1 + (uint32_t)(rng() % 0x7FFFFFFFu));
  printf("checked %llu quotients, %llu wrong\n", (unsigned long long)checked, (unsigned long long)bad);
  return bad ? 1 : 0;
}
