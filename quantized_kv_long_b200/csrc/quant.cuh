// quant.cuh -- one warp quantizes one block (32-element Q8_0 or Q4_0, or
// 128-element OSCAR2).
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
// offsets (34*b, 18*b, 36*b) of a 2-byte aligned buffer.  A byte-wise store of a
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

// The value and element index of the first extreme element of the block: the
// smallest (MIN) or largest value, the lowest element index among equal values
// (so a block holding both -0 and +0 takes the sign of the first).  Lane `lane`
// holds elements lane + 32 k, k = 0..3.
template <bool MIN>
__device__ __forceinline__ float first_extreme(const float (&x)[4], int lane)
{
    float v = x[0];
    int idx = lane;
#pragma unroll
    for (int k = 1; k < 4; ++k)
        if (MIN ? x[k] < v : x[k] > v) {  // strict: the lower index wins a tie
            v = x[k];
            idx = lane + 32 * k;
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
        if ((MIN ? v2 < v : v2 > v) || (v2 == v && i2 < idx)) {
            v = v2;
            idx = i2;
        }
    }
    return v;
}

// OSCAR2: lane `lane` holds x[k] = element lane + 32 k of the 128-element block
// at `blk` (4-byte aligned) and writes code byte `lane`:
//   mn, mx = first min / max; d = (mx - mn)/3; id = d ? 1/d : 0;
//   u = min(3, trunc((x - mn)*id + 0.5)); byte j = u_j | u_{j+32} << 2 | ...;
//   fp16(d) and fp16(mn) in bytes 0-3.
__device__ __forceinline__ void warp_quant_oscar2(const float (&x)[4], uint8_t *blk, int lane)
{
    const float mn = first_extreme<true>(x, lane);
    const float mx = first_extreme<false>(x, lane);
    const float d = __fdiv_rn(__fsub_rn(mx, mn), 3.0f);
    const float id = (d != 0.0f) ? __fdiv_rn(1.0f, d) : 0.0f;
    int byte = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        int u = (int)truncf(__fadd_rn(__fmul_rn(__fsub_rn(x[k], mn), id), 0.5f));
        u = u > 3 ? 3 : u;
        byte |= u << (2 * k);
    }
    const unsigned short hd = d_bits(d), hm = d_bits(mn);
    blk[4 + lane] = (uint8_t)byte;
    if (lane == 0) {
        store_d(blk, hd);
        store_d(blk + 2, hm);
    }
}

}  // namespace kvq
