// Philox-4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC'11): ten rounds of two
// 32x32->64-bit products (multipliers 0xD2511F53, 0xCD9E8D57), with the key
// bumped by the Weyl constants 0x9E3779B9, 0xBB67AE85 before every round but
// the first.  A round maps (c0, c1, c2, c3) to
// (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0)).
#pragma once

#include <stdint.h>

namespace qg {

struct PhiloxKey {
  uint32_t k0, k1;
};

__device__ __forceinline__ void philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                              PhiloxKey key, uint32_t (&out)[4]) {
  uint32_t k0 = key.k0, k1 = key.k1;
#pragma unroll
  for (int rnd = 0; rnd < 10; ++rnd) {
    if (rnd) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ k0;
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ k1;
    c1 = static_cast<uint32_t>(p1);
    c3 = static_cast<uint32_t>(p0);
    c0 = n0;
    c2 = n2;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

// The ten round keys of a key, formed once and reused by many calls.
struct PhiloxRoundKeys {
  uint32_t k0[10], k1[10];
};

__device__ __forceinline__ PhiloxRoundKeys philox_round_keys(PhiloxKey key) {
  PhiloxRoundKeys rk;
#pragma unroll
  for (int rnd = 0; rnd < 10; ++rnd) {
    rk.k0[rnd] = key.k0 + static_cast<uint32_t>(rnd) * 0x9E3779B9u;
    rk.k1[rnd] = key.k1 + static_cast<uint32_t>(rnd) * 0xBB67AE85u;
  }
  return rk;
}

// The same generator with precomputed round keys.
__device__ __forceinline__ void philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                              const PhiloxRoundKeys& rk, uint32_t (&out)[4]) {
#pragma unroll
  for (int rnd = 0; rnd < 10; ++rnd) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ rk.k0[rnd];
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ rk.k1[rnd];
    c1 = static_cast<uint32_t>(p1);
    c3 = static_cast<uint32_t>(p0);
    c0 = n0;
    c2 = n2;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

}  // namespace qg
