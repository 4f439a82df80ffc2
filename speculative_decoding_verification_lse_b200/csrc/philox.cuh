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

// Full 64-bit product of two 32-bit words.
__device__ __forceinline__ unsigned long long mul_wide(uint32_t a, uint32_t b) {
  unsigned long long r;
  asm("mul.wide.u32 %0, %1, %2;" : "=l"(r) : "r"(a), "r"(b));
  return r;
}

// The ten round keys of one seed (warp-uniform; computed once per work item).
struct PhiloxKey {
  uint32_t k0[10], k1[10];
};

__device__ __forceinline__ PhiloxKey philox_key(uint64_t seed) {
  PhiloxKey K;
  uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    K.k0[r] = a;
    K.k1[r] = b;
    a += kWeylA;
    b += kWeylB;
  }
  return K;
}

__device__ __forceinline__ void philox_round(uint4& c, uint32_t k0, uint32_t k1) {
  const unsigned long long pa = mul_wide(kPhiloxMulA, c.x);
  const unsigned long long pb = mul_wide(kPhiloxMulB, c.z);
  c = make_uint4((uint32_t)(pb >> 32) ^ c.y ^ k0, (uint32_t)pb, (uint32_t)(pa >> 32) ^ c.w ^ k1,
                 (uint32_t)pa);
}

// The race words of counter (i, g, 1, 0) for many i and one request g.  Words 2
// and 3 of the counter are constants, so round 1 needs one per-thread product
// instead of two, and so does round 2 (its first product is the same for every
// i); the rest of the rounds are the published ones.
struct RaceStream {
  PhiloxKey K;
  uint32_t i0;    // counter of the row's first four tokens (vocabulary offset / 4)
  uint32_t x1;    // round-1 word 0: hi(B*1) ^ g ^ k0[0] = g ^ k0[0]
  uint32_t y2c;   // round-2 word 0 term: lo(B*1) ^ k0[1] = B ^ k0[1]
  uint32_t z2c;   // round-2 word 2 term: hi(A*x1) ^ k1[1]
  uint32_t w2;    // round-2 word 3: lo(A*x1)
};

__device__ __forceinline__ RaceStream race_stream(uint64_t seed, uint32_t g, uint32_t i0 = 0) {
  RaceStream R;
  R.K = philox_key(seed);
  R.i0 = i0;
  R.x1 = g ^ R.K.k0[0];
  R.y2c = kPhiloxMulB ^ R.K.k0[1];
  const unsigned long long pa = (unsigned long long)kPhiloxMulA * R.x1;
  R.z2c = (uint32_t)(pa >> 32) ^ R.K.k1[1];
  R.w2 = (uint32_t)pa;
  return R;
}

__device__ __forceinline__ uint4 race_words_fast(const RaceStream& R, uint32_t i) {
  i += R.i0;
  // round 1 on (i, g, 1, 0)
  const unsigned long long pa = mul_wide(kPhiloxMulA, i);
  const uint32_t z1 = (uint32_t)(pa >> 32) ^ R.K.k1[0];
  const uint32_t w1 = (uint32_t)pa;
  // round 2 on (x1, lo(B), z1, w1)
  const unsigned long long pb = mul_wide(kPhiloxMulB, z1);
  uint4 c = make_uint4((uint32_t)(pb >> 32) ^ R.y2c, (uint32_t)pb, w1 ^ R.z2c, R.w2);
#pragma unroll
  for (int r = 2; r < 10; ++r) philox_round(c, R.K.k0[r], R.K.k1[r]);
  return c;
}

}  // namespace sv
