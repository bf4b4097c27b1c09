// decode_frag.cuh -- shared-memory loads and exact conversions that feed the
// decode kernels' warp MMAs: int8 Q8_0 bytes and Q4_0 nibbles become f16
// values holding the same integers (f16 has 11 significant bits, so every
// int8 and every nibble - 8 is exact).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace kvq {
namespace frag {

// Four int8 in a u32 -> two half2 holding the exact integers:
// (0x64 << 8 | (b ^ 0x80)) is the f16 1152 + b.
__device__ __forceinline__ void s8x4_to_h2x2(uint32_t w, uint32_t &h01, uint32_t &h23)
{
    w ^= 0x80808080u;
    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
    h01 = ptx::h2_bits(__hsub2(ptx::bits_h2(ptx::prmt(w, 0x64646464u, 0x5140)), bias));
    h23 = ptx::h2_bits(__hsub2(ptx::bits_h2(ptx::prmt(w, 0x64646464u, 0x7362)), bias));
}

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

// The four K bytes [p, p+4) of a k-step; 4-byte aligned exactly when `aligned`
// (a constant once the block loop is unrolled).
__device__ __forceinline__ uint32_t k_word(const uint8_t *p, bool aligned)
{
    if (aligned)
        return lds32(p);
    return ptx::prmt(lds16(p), lds16(p + 2), 0x5410);
}

}  // namespace frag
}  // namespace kvq
