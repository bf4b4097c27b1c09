// decode_frag.cuh -- shared-memory loads and the exact nibble conversion that
// feed the decode kernel's warp MMAs: Q4_0 nibbles become f16 values holding
// nibble - 8 (f16 has 11 significant bits, so every nibble - 8 is exact).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace kvq {
namespace frag {

// Nibbles at bits 0-3 and 16-19 of w -> half2 (u - 8); bits 4-7 and 20-23 -> half2 (u - 8).
__device__ __forceinline__ uint32_t nib_lo(uint32_t w)
{
    const uint32_t x = (w & 0x000F000Fu) | 0x64006400u;  // 1024 + u
    const __half2 c = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));  // 1032
    return ptx::h2_bits(__hsub2(ptx::bits_h2(x), c));
}

__device__ __forceinline__ uint32_t nib_hi(uint32_t w)
{
    const uint32_t x = (w & 0x00F000F0u) | 0x64006400u;  // 1024 + 16u
    const __half2 s = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));  // 1/16
    const __half2 c = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));  // -72
    return ptx::h2_bits(__hfma2(ptx::bits_h2(x), s, c));
}

__device__ __forceinline__ uint32_t lds16(const uint8_t *p)
{
    return *reinterpret_cast<const uint16_t *>(p);
}

__device__ __forceinline__ uint32_t lds32(const uint8_t *p)
{
    return *reinterpret_cast<const uint32_t *>(p);
}

}  // namespace frag
}  // namespace kvq
