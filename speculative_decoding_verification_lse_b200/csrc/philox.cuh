// philox.cuh -- Philox4x32-10 on the device.
//
// Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
// (SC'11): a 4x32-bit counter is passed through ten rounds of a multiply-xor
// S-box.  Each round multiplies counter words 0 and 2 by two fixed odd
// constants, keeps both halves of the 64-bit products, and mixes the high
// halves with counter words 1 and 3 and the round key.  The 2x32-bit key is
// advanced by a Weyl sequence (the golden ratio and sqrt(3)-1 in 32-bit fixed
// point) between rounds.
#pragma once
#include <stdint.h>

namespace sv {

constexpr uint32_t kPhiloxMulA = 0xD2511F53u;  // multiplies counter word 0
constexpr uint32_t kPhiloxMulB = 0xCD9E8D57u;  // multiplies counter word 2
constexpr uint32_t kWeylA = 0x9E3779B9u;
constexpr uint32_t kWeylB = 0xBB67AE85u;

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const unsigned long long pa = (unsigned long long)kPhiloxMulA * c.x;
    const unsigned long long pb = (unsigned long long)kPhiloxMulB * c.z;
    uint4 n;
    n.x = (uint32_t)(pb >> 32) ^ c.y ^ k0;
    n.y = (uint32_t)pb;
    n.z = (uint32_t)(pa >> 32) ^ c.w ^ k1;
    n.w = (uint32_t)pa;
    c = n;
    k0 += kWeylA;
    k1 += kWeylB;
  }
  return c;
}

// The accept uniform of position d of request g: top 24 bits of word 0 at
// counter (d, g, 0, 0), times 2^-24 (exact in single precision).
__device__ __forceinline__ uint32_t accept_word(uint64_t seed, uint32_t g, uint32_t d) {
  return philox4x32_10(make_uint4(d, g, 0u, 0u), (uint32_t)seed, (uint32_t)(seed >> 32)).x;
}

// The four race words of tokens 4i..4i+3 of request g: counter (i, g, 1, 0).
__device__ __forceinline__ uint4 race_words(uint64_t seed, uint32_t g, uint32_t i) {
  return philox4x32_10(make_uint4(i, g, 1u, 0u), (uint32_t)seed, (uint32_t)(seed >> 32));
}

}  // namespace sv
