// Widening of 2-bit ternary weight codes (00 = 0, 01 = +1, 11 = -1, code i of
// a word at bits 2i .. 2i+1) to int8, shared by the widening kernel and the
// small-M forward kernel that reads packed weights directly.
#pragma once

#include <cstdint>

namespace hbl {
namespace tern {

// Eight 2-bit fields (the low 16 bits of w) -> eight nibbles, field i in
// nibble i: three shift-or-mask steps.
__device__ __forceinline__ uint32_t spread_fields(uint32_t w) {
  uint32_t y = w & 0xffffu;
  y = (y | (y << 8)) & 0x00ff00ffu;
  y = (y | (y << 4)) & 0x0f0f0f0fu;
  y = (y | (y << 2)) & 0x33333333u;
  return y;
}

// 2-bit code -> int8 byte by a byte-permute lookup: the table's bytes are
// 00 -> 0x00, 01 -> 0x01, 10 -> 0x00 (unused pattern), 11 -> 0xFF (-1).
__device__ __forceinline__ uint4 widen16(uint32_t w) {
  constexpr uint32_t kLut = 0xff000100u;
  const uint32_t lo = spread_fields(w), hi = spread_fields(w >> 16);
  return make_uint4(__byte_perm(kLut, 0u, lo & 0xffffu), __byte_perm(kLut, 0u, lo >> 16),
                    __byte_perm(kLut, 0u, hi & 0xffffu), __byte_perm(kLut, 0u, hi >> 16));
}

}  // namespace tern
}  // namespace hbl
