// keys.cuh -- order-preserving 32-bit keys of fp32 scores, shared by the
// top-k selection and the indexer's candidate lists.
#pragma once
#include <stdint.h>

namespace dsa {

// Larger float -> larger unsigned key; -0.0 is folded into +0.0, so the two
// zeros are one key (the selection treats them as equal scores).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose key is u (inverse of order_key on the keys it produces):
// x >= key_float(order_key(y)) exactly when order_key(x) >= order_key(y).
__device__ __forceinline__ float key_float(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

}  // namespace dsa
