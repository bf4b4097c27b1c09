// quant.cuh -- one warp quantizes one 32-element block (Q8_0 or Q4_0).
//
// Used by the append and quantize kernels.  Every
// arithmetic step is an explicitly rounded fp32 operation (__fdiv_rn,
// __fmul_rn, __fadd_rn), so the blocks do not depend on the compiler's
// multiply-add contraction and are bit-identical wherever these run.
// Definitions: see quant.cu.
#pragma once

#include "common.cuh"

namespace kvq {

// The fp16 scale is converted by every lane (outside any lane-divergent
// branch) and lane 0 stores it as one 16-bit word; blocks start at even byte
// offsets (34*b, 18*b) of a 2-byte aligned buffer.  A byte-wise store of a
// value converted inside the lane-0 branch was observed to write 0 into the
// low byte on sm_100a; the bit-exact tests against the oracle caught it.
__device__ __forceinline__ unsigned short d_bits(float d)
{
    return __half_as_ushort(__float2half_rn(d));
}

__device__ __forceinline__ void store_d(uint8_t *blk, unsigned short h)
{
    *reinterpret_cast<unsigned short *>(blk) = h;
}

// Lane `lane` holds x = element `lane` of the block that starts at `blk`.
__device__ __forceinline__ void warp_quant_q8_0(float x, uint8_t *blk, int lane)
{
    float amax = fabsf(x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float d = __fdiv_rn(amax, 127.0f);
    const float id = (d != 0.0f) ? __fdiv_rn(1.0f, d) : 0.0f;
    const int q = (int)roundf(__fmul_rn(x, id));
    const unsigned short h = d_bits(d);
    blk[2 + lane] = (uint8_t)(int8_t)q;
    if (lane == 0)
        store_d(blk, h);
}

__device__ __forceinline__ void warp_quant_q4_0(float x, uint8_t *blk, int lane)
{
    // first index of the largest |x|: larger magnitude wins, ties go to the lower lane
    float a = fabsf(x);
    int idx = lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float a2 = __shfl_xor_sync(0xffffffffu, a, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
        if (a2 > a || (a2 == a && i2 < idx)) {
            a = a2;
            idx = i2;
        }
    }
    const float xm = __shfl_sync(0xffffffffu, x, idx);
    const float m = (a > 0.0f) ? xm : 0.0f;  // an all-zero block keeps m = +0
    const float d = __fdiv_rn(m, -8.0f);
    const float id = (d != 0.0f) ? __fdiv_rn(1.0f, d) : 0.0f;
    const float s = __fadd_rn(__fmul_rn(x, id), 8.5f);
    int u = (int)truncf(s);
    u = u > 15 ? 15 : u;
    const int u_hi = __shfl_down_sync(0xffffffffu, u, 16);
    const unsigned short h = d_bits(d);
    if (lane < 16)
        blk[2 + lane] = (uint8_t)(u | (u_hi << 4));
    if (lane == 0)
        store_d(blk, h);
}

}  // namespace kvq
