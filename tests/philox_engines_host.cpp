// Two independent host implementations of Philox4x32-10 (Salmon et al.,
// SC'11), used only by the tests as outside checks of the oracle's generator:
//   - cuda::std::philox4x32 from libcudacxx, the C++26 standard engine
//     (philox_engine<uint_fast32_t, 32, 4, 10, 0xCD9E8D57, 0x9E3779B9,
//     0xD2511F53, 0xBB67AE85>), driven through its public interface only;
//   - at::Philox4_32 from PyTorch's ATen headers.
// Compiled by the tests with the host compiler.  Reads lines
// "c0 c1 c2 c3 k0 k1" (decimal) on stdin and prints, for each, the four words
// of each engine ("std w0 w1 w2 w3" and "torch w0 w1 w2 w3") in call order.
#include <cstdint>
#include <cstdio>

#ifdef WITH_STD_ENGINE
#include <cuda/std/__random/philox_engine.h>
#endif
#ifdef WITH_TORCH_ENGINE
#include <ATen/core/PhiloxRNGEngine.h>
#endif

#ifdef WITH_STD_ENGINE
// A seed sequence whose generate() yields the two key words (seeding the
// standard engine from a sequence sets key word i from its i-th 32-bit value).
struct KeyWords {
  using result_type = uint32_t;
  uint32_t k0, k1;
  template <class It>
  void generate(It b, It e) {
    uint32_t v[2] = {k0, k1};
    for (int i = 0; b != e; ++b, ++i) *b = i < 2 ? v[i] : 0u;
  }
};
#endif

int main() {
  unsigned long c0, c1, c2, c3, k0, k1;
  while (scanf("%lu %lu %lu %lu %lu %lu", &c0, &c1, &c2, &c3, &k0, &k1) == 6) {
    uint32_t w[4];
#ifdef WITH_STD_ENGINE
    {
      KeyWords ks{(uint32_t)k0, (uint32_t)k1};
      cuda::std::philox4x32 e(ks);
      // set_counter takes the counter with the most significant word first
      e.set_counter({(uint32_t)c3, (uint32_t)c2, (uint32_t)c1, (uint32_t)c0});
      for (int i = 0; i < 4; ++i) w[i] = (uint32_t)e();
      printf("std %u %u %u %u\n", w[0], w[1], w[2], w[3]);
    }
#endif
#ifdef WITH_TORCH_ENGINE
    {
      // key = seed; counter words 2, 3 = subsequence; words 0, 1 = offset
      at::Philox4_32 e((uint64_t)k0 | ((uint64_t)k1 << 32), (uint64_t)c2 | ((uint64_t)c3 << 32),
                       (uint64_t)c0 | ((uint64_t)c1 << 32));
      for (int i = 0; i < 4; ++i) w[i] = e();
      printf("torch %u %u %u %u\n", w[0], w[1], w[2], w[3]);
    }
#endif
  }
  return 0;
}
