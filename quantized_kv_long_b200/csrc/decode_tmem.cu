// decode_tmem.cu -- split-KV GQA decode attention at head_dim 256 for up to
// 24 query rows per KV head (T <= 4 query tokens x 6 query heads), with
// Q K^T on the tcgen05 tensor cores over keys staged in tensor memory and
// P V on warp MMAs, one persistent CTA per SM.
//
// What it computes (speculative-decoding paragraph of the RX 9070 XT
// KV-streaming page: paged decode attention over a verify batch; "Known
// Issues Fixed" of the OSCAR2 page: the softmax max covers complete scores;
// GQA section of the KV-cache guide): per (layer, KV head, chunk) -- one
// "unit" -- the chunk partial o = sum_j p_j v^_j / l and lse = m + ln l of
// every query row, with s_j = scale * sum_b d_b * sum_i q_i k_ij, and the
// same exact arithmetic as the other decode kernels:
//  * int8 K and f16 q multiply exactly; each 32-element block's sum is
//    accumulated in fp32 by the tensor core and scaled by its fp32 d_b;
//  * P = 2^(s - m) enters P V as two f16 parts (residual ~2^-22 relative),
//    and the per-key d_v through the exact two-part product
//    hi = RN(P_hi d), lo = fma(P_hi, d, -hi) + P_lo d.
//
// Why this shape (B200): with 24 rows, the nine legacy warp MMAs per key of
// an all-mma.sync decode need about the tensor-pipe time that reading the
// key's 416 bytes takes at full HBM speed, on top of ~100 other
// instructions per key.  Here Q K^T moves to tcgen05: A = the key tile in
// TMEM (keys = M = the 128 TMEM lanes, written by tcgen05.st from the
// thread that owns the key, so the f16 tile never passes through shared
// memory), B = Q^T in shared memory.  Blocks are paired: one MMA of N = 16 NT
// (48 for 24 rows) computes the sums of two blocks side by side, with Q^T
// block-diagonal (each N-row holds one block's 32 dims and zeros over the
// other's), so the per-block accumulators of a 128-key tile take 4 * 48
// TMEM columns and two of them fit beside one key tile: the MMAs of a tile
// never wait for the softmax of the tile before.  P V stays on mma.sync,
// where d_v can enter the B operand per key.
//
// Work: the grid is one CTA per SM; CTA i takes units i, i + grid, ...,
// and all roles stream the tiles of consecutive units without a break.
// A tile is 128 keys: 34,816 B of K head-rows and 18,432 B of V head-rows,
// each one contiguous 16-byte-aligned range of the head-major cache.
// Warp roles (28 warps):
//  * K copy (warp 0) and V copy (warp 3): lane 0 runs a ring of raw K
//    (resp. V) tiles with cp.async.bulk, completion on mbarriers; K slots
//    free once converted, V slots once P V is done;
//  * MMA (warp 1): one elected lane of the converged warp issues the
//    tcgen05.mma and commits;
//  * Q loader (warp 2): Q^T of the next unit with cp.async into the other
//    of two 128-byte-swizzled buffers;
//  * 8 convert warps, one key per thread (warp pairs split the 8 blocks):
//    int8 -> f16 into the key's TMEM lane, and d_k * scale * log2 e as fp32
//    for the softmax;
//  * 8 softmax warps, one key per thread, 12 (4 NT) rows each: S = sum_b
//    d_b acc_b from TMEM with packed f32x2 FMAs, masks, a running max per
//    row shared by the eight warps (lazy: a reducing barrier per tile tells
//    whether any score exceeds it by more than TAU; only then do the warps
//    exchange tile maxima and move it to the exact maximum, recording the
//    tile's rescale), P = 2^(s - m) as P_hi + P_lo stored [key][row] f16;
//  * 8 value warps, Q4_0 block b each: O^T += V^T (P d_v)^T on mma.sync
//    m16n8k16 over the tile's 8 groups of 16 keys, B fragments of P read
//    with ldmatrix.trans.
// Every warp waits and arrives with all its lanes (no lane-divergent
// hand-offs).  Every wait is bounded (about one second of wall time); one
// that runs out sets the device status word and the roles fall through; the
// copy warps and the MMA warp wait (bounded) for their copies and MMAs
// before the CTA frees TMEM.
#include <atomic>

#include "common.cuh"
#include "decode_frag.cuh"
#include "ptx.cuh"

namespace kvq {

namespace {

using namespace frag;

constexpr int HD = 256;                      // head_dim of this kernel
constexpr int KROW = 272, VROW = 144;        // head-row bytes at head_dim 256
constexpr int TOK = 128;                     // keys per tile: the MMA's M, the TMEM lanes
constexpr int NGRP = TOK / 16;               // 16-key groups of a tile for P V
constexpr int NSK = 2, NSV = 3;              // raw K / V tiles in the rings
constexpr int NP = 2;                        // P slots between softmax and value warps
constexpr int STAGE_K = TOK * KROW;          // 34,816
constexpr int STAGE_V = TOK * VROW;          // 18,432
constexpr int DKROW = 48;                    // bytes per key of a d_k slot (8 floats + pad)
constexpr int DKBUF = TOK * DKROW;

constexpr int W_KCOPY = 0, W_MMA = 1, W_QLOAD = 2, W_VCOPY = 3;
constexpr int W_CONV = 4, W_SOFT = 12, W_VAL = 20;
constexpr int N_CONV = 8, N_SOFT = 8, N_VAL = 8;
constexpr int WARPS = 28, THREADS = 32 * WARPS;
constexpr int BAR_SOFT = 1;                  // named barrier of the softmax warps
constexpr int REG_CTL = 64, REG_CONV = 56, REG_SOFT = 80, REG_VAL = 80;  // registers per thread
static_assert(128 * (REG_CTL + 2 * REG_CONV + 2 * REG_SOFT + 2 * REG_VAL) <= THREADS * 72,
              "register split within the launch's 72 per thread");

constexpr uint64_t WAIT_NS = 1000000000ull;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float TAU = 8.0f;                  // lazy-max slack (log2 units): p <= 2^8
constexpr float M_INIT = -1.0e30f;           // "no score yet", finite: ex2(s - M_INIT) is defined

template <int NT>
struct Cfg {
    static constexpr int NR = 8 * NT;            // query rows (padded)
    static constexpr int RH = 4 * NT;            // rows per softmax half
    static constexpr int NQP = 4 * RH;           // MMA N of a block pair
    static constexpr int PROW = 2 * NR;          // bytes per key of one P part
    static constexpr int PPART = TOK * PROW;
    static constexpr int PSLOT = 2 * PPART;      // P_hi then P_lo
    static constexpr int QPAIR = NQP * 128;      // Q^T of a block pair: [NQP N-rows][128 B]
    static constexpr int QBUF = 4 * QPAIR;
    // tensor memory: two S buffers of 4 pairs x NQP columns, then the f16 key tile
    static constexpr uint32_t COL_S = 0, SBUF = 4 * NQP, COL_K = 2 * SBUF;
    static constexpr uint32_t TMEM_COLS = COL_K + 128 <= 256 ? 256 : 512;
    // shared memory, from a 1024-aligned base
    static constexpr int OFF_Q = 0;                              // [2][QBUF]
    static constexpr int OFF_RK = OFF_Q + 2 * QBUF;              // [NSK][STAGE_K]
    static constexpr int OFF_RV = OFF_RK + NSK * STAGE_K;        // [NSV][STAGE_V]
    static constexpr int OFF_DK = OFF_RV + NSV * STAGE_V;        // [2][DKBUF]
    static constexpr int OFF_P = OFF_DK + 2 * DKBUF;             // [NP][PSLOT]
    static constexpr int OFF_HEAD = OFF_P + NP * PSLOT;
    static_assert(COL_K + 128 <= 512, "tensor memory columns");
    static_assert(QPAIR % 1024 == 0 && OFF_RK % 16 == 0 && OFF_RV % 16 == 0 &&
                      OFF_DK % 16 == 0 && OFF_P % 16 == 0 && OFF_HEAD % 8 == 0,
                  "operand alignment");
};

// Barrier arrival counts: warps arrive with all 32 lanes.
constexpr uint32_t ALL = 32;

struct Head {
    uint64_t kfull[NSK], kfree[NSK];      // raw K landed / converted
    uint64_t vfull[NSV], vfree[NSV];      // raw V landed / P V done
    uint64_t kbfull, kbfree;              // f16 K tile in TMEM written / its MMAs done
    uint64_t dkfull[2], dkfree[2];        // scaled d_k of a tile written / read
    uint64_t sfull[2], sfree[2];          // S buffer of a tile complete / read by the softmax
    uint64_t pfull[NP], pfree[NP];        // P of a tile written / read by the value warps
    uint64_t qfull[2], qfree[2];          // Q^T of a unit loaded / its last MMA done
    uint64_t lfull[2], lfree[2];          // per-row sums and max of a unit published / read
    uint64_t drain, never;
    float alpha[NP][24];                  // per tile: rescale of O per row when `changed`
    int changed[NP];
    float tmx[4][24];                     // per-quarter tile maxima of a running-max update
    float fl[2][4][24];                   // per unit: per-quarter sums
    float fm[2][24];                      // per unit: final running max
    uint32_t tmem_base;
    int abort;
};

template <int NT>
constexpr int smem_bytes()
{
    return Cfg<NT>::OFF_HEAD + (int)sizeof(Head) + 1024;  // + alignment slack
}
static_assert(smem_bytes<3>() <= 232448, "dynamic shared memory per block");

// A unit: (layer, KV head, chunk) and its key range.
struct Unit {
    int layer, h, c, n_tok, n_tiles;
    int64_t c0;
};

__device__ __forceinline__ Unit unit_of(const DecodeArgs &a, int u, int C)
{
    Unit x;
    x.c = u % C;
    x.h = (u / C) % a.n_kv_heads;
    x.layer = u / (C * a.n_kv_heads);
    x.c0 = (int64_t)x.c * a.chunk;
    x.n_tok = (int)((x.c0 + a.chunk < a.n_kv ? x.c0 + a.chunk : a.n_kv) - x.c0);
    x.n_tiles = (x.n_tok + TOK - 1) / TOK;
    return x;
}

// The dynamic shared memory of the kernel, from a 1024-aligned base.
__device__ __forceinline__ uint8_t *smem_base()
{
    extern __shared__ __align__(1024) uint8_t dt_raw[];
    return dt_raw + ((1024u - (ptx::smem_u32(dt_raw) & 1023u)) & 1023u);
}

// Bounded wait of the whole warp (every lane tests the barrier; the result is
// made uniform).  false (abort flag and status word set) when it ran out or the
// CTA aborted.
__device__ __forceinline__ bool wait_slow(uint64_t *bar, uint32_t parity, volatile int *abort,
                                       unsigned int *status)
{
    const bool ok = ptx::mbar_wait_bounded(bar, parity, abort, WAIT_NS);
    if (!ok && !*abort) {
        *abort = 1;
        report_timeout(status);
    }
    return ok;
}

__device__ __forceinline__ bool wwait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                      unsigned int *status)
{
    bool ok = ptx::mbar_try_wait(bar, parity);
    if (!ok)
        ok = wait_slow(bar, parity, abort, status);
    return __all_sync(0xffffffffu, ok);
}

// Named barrier that also returns the OR of `pred` over the `threads` threads
// taking it (whole warps).
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t threads, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}

// a += b * c on a pair of fp32 values with one packed instruction
__device__ __forceinline__ void ffma2(float &a0, float &a1, float b, float c0, float c1)
{
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%0, %1};\n\t"
        "mov.b64 rb, {%2, %2};\n\t"
        "mov.b64 rc, {%3, %4};\n\t"
        "fma.rn.f32x2 ra, rb, rc, ra;\n\t"
        "mov.b64 {%0, %1}, ra;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(b), "f"(c0), "f"(c1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                              uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Warp-collective: thread t reads TMEM lane (lane base + t), 8 consecutive columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

// Converts this thread's key's four Q8_0 blocks 4 HH .. 4 HH + 3 (raw head-row
// at `row`) to f16 in TMEM columns [col + 16 b, col + 16 b + 16) and returns
// their fp32 scales d_b * dscale.  int8 -> f16 is exact: (0x64 << 8 | (q ^ 0x80))
// is the f16 1152 + q.
template <int HH>
__device__ __forceinline__ float4 convert_key(const uint8_t *row, uint32_t taddr, float dscale)
{
    constexpr int BASE = 128 * HH;  // first byte loaded: 16-byte chunk 8 HH
    uint32_t w[36];
#pragma unroll
    for (int i = 0; i < 9; ++i) {
        const uint4 v = *reinterpret_cast<const uint4 *>(row + BASE + 16 * i);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
    }
    float dsc[4];
#pragma unroll
    for (int bi = 0; bi < 4; ++bi) {
        const int rel = 34 * (4 * HH + bi) - BASE;  // block start, relative to BASE
        const uint32_t dw = w[rel >> 2];
        const uint32_t d16 = (rel & 2) ? (dw >> 16) : (dw & 0xFFFFu);
        dsc[bi] = __half2float(__ushort_as_half((unsigned short)d16)) * dscale;
    }
#pragma unroll
    for (int i = 0; i < 36; ++i)
        w[i] ^= 0x80808080u;
    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152
#pragma unroll
    for (int bi = 0; bi < 4; ++bi) {
        const int rel = 34 * (4 * HH + bi) - BASE + 2;  // first q byte
        uint32_t r[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int off = rel + 2 * e;  // bytes off, off + 1: elements 2e, 2e + 1
            const uint32_t src = w[off >> 2];
            const uint32_t sel = (off & 2) ? 0x4342u : 0x4140u;  // [b, 0x64, b+1, 0x64]
            const uint32_t x = ptx::prmt(src, 0x64646464u, sel);
            r[e] = ptx::h2_bits(__hsub2(ptx::bits_h2(x), bias));
        }
        ptx::tmem_st16(taddr + 16 * (4 * HH + bi), r);
    }
    return make_float4(dsc[0], dsc[1], dsc[2], dsc[3]);
}

// P V of one group of 16 keys for the value warp of block b:
// O^T += V^T (P d_v)^T, A = the block's nibbles (exact f16 integers u - 8),
// B = P d_v as two f16 parts.  CHECK: keys >= valid hold stale bytes (scale 0).
template <int NT, bool CHECK>
__device__ __forceinline__ void pv_group(float (&o)[2][NT][4], const uint8_t *vb, uint32_t pa,
                                         int valid, int g, int cq)
{
    uint32_t d0 = lds16(vb), d1 = lds16(vb + VROW);
    uint32_t d2 = lds16(vb + 8 * VROW), d3 = lds16(vb + 9 * VROW);
    if (CHECK) {
        if (2 * cq >= valid) d0 = 0;
        if (2 * cq + 1 >= valid) d1 = 0;
        if (2 * cq + 8 >= valid) d2 = 0;
        if (2 * cq + 9 >= valid) d3 = 0;
    }
    const __half2 dA = ptx::bits_h2(ptx::prmt(d0, d1, 0x5410));
    const __half2 dB = ptx::bits_h2(ptx::prmt(d2, d3, 0x5410));
    const uint32_t x0 = lds16(vb + 2 + 2 * g), x1 = lds16(vb + VROW + 2 + 2 * g);
    const uint32_t x2 = lds16(vb + 8 * VROW + 2 + 2 * g);
    const uint32_t x3 = lds16(vb + 9 * VROW + 2 + 2 * g);
    const uint32_t wA0 = ptx::prmt(x0, x1, 0x0400);  // byte 2g of keys 2c, 2c+1
    const uint32_t wA1 = ptx::prmt(x0, x1, 0x0501);  // byte 2g+1
    const uint32_t wB0 = ptx::prmt(x2, x3, 0x0400);  // keys 2c+8, 2c+9
    const uint32_t wB1 = ptx::prmt(x2, x3, 0x0501);
    const uint32_t alo[4] = {nib_lo(wA0), nib_lo(wA1), nib_lo(wB0), nib_lo(wB1)};
    const uint32_t ahi[4] = {nib_hi(wA0), nib_hi(wA1), nib_hi(wB0), nib_hi(wB1)};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        uint32_t ph[2], pl[2];
        ldsm_x4_trans(pa + 16 * nt, ph[0], ph[1], pl[0], pl[1]);
        // P d_v as hi + lo without loss: hi = RN(P_hi d), the exact product
        // error fma(P_hi, d, -hi), plus P_lo d
        uint32_t bh[2], bl[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const __half2 d = k == 0 ? dA : dB;
            const __half2 a_hi = ptx::bits_h2(ph[k]);
            const __half2 hi = __hmul2_rn(a_hi, d);
            const __half2 err = __hfma2(a_hi, d, __hneg2(hi));
            bh[k] = ptx::h2_bits(hi);
            bl[k] = ptx::h2_bits(__hfma2(ptx::bits_h2(pl[k]), d, err));
        }
        ptx::mma_f16_16816(o[0][nt], alo, bh[0], bh[1], o[0][nt]);
        ptx::mma_f16_16816(o[0][nt], alo, bl[0], bl[1], o[0][nt]);
        ptx::mma_f16_16816(o[1][nt], ahi, bh[0], bh[1], o[1][nt]);
        ptx::mma_f16_16816(o[1][nt], ahi, bl[0], bl[1], o[1][nt]);
    }
}

// ---------------------------------------------------------------- roles
// Each role derives what it needs from the parameters, threadIdx and shared
// memory after its register budget is set.

template <int NT>
__device__ __forceinline__ void role_copy(const DecodeArgs &a, bool is_k)
{
    using CF = Cfg<NT>;
    uint8_t *smem = smem_base();
    Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
    volatile int *abort = &hd.abort;
    const int C = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int units = a.n_layers * a.n_kv_heads * C;
    const int NS = is_k ? NSK : NSV;
    const int ROW = is_k ? KROW : VROW;
    uint64_t *full = is_k ? hd.kfull : hd.vfull;
    uint64_t *freeb = is_k ? hd.kfree : hd.vfree;
    uint8_t *ring = smem + (is_k ? CF::OFF_RK : CF::OFF_RV);
    const int stage = TOK * ROW;
    if (is_k && a.test_timeout) {
        // test hook: wait on a barrier that nothing completes
        if (!ptx::mbar_wait_bounded(&hd.never, 0, abort, WAIT_NS) && !*abort) {
            *abort = 1;
            report_timeout(a.status);
        }
    }
    int it = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < units && !stop; u += gridDim.x) {
        const Unit un = unit_of(a, u, C);
        const int64_t cap = a.layers.cap[un.layer];
        const uint8_t *src = (is_k ? a.layers.k[un.layer] : a.layers.v[un.layer]) +
                             ((int64_t)un.h * cap + un.c0) * ROW;
        for (int i = 0; i < un.n_tiles; ++i, ++it) {
            const int slot = it % NS;
            if (it >= NS &&
                !ptx::mbar_wait_bounded(&freeb[slot], ((it / NS) - 1) & 1, abort, WAIT_NS)) {
                if (!*abort) {
                    *abort = 1;
                    report_timeout(a.status);
                }
                stop = true;
                break;
            }
            if (*abort) {
                stop = true;
                break;
            }
            const int rows = min(TOK, un.n_tok - i * TOK);
            ptx::mbar_arrive_expect_tx(&full[slot], rows * ROW);
            ptx::bulk_g2s(ring + slot * stage, src + (int64_t)i * stage, rows * ROW, &full[slot]);
        }
    }
    // every issued copy has landed before the CTA exits (bounded, without the
    // abort short-cut)
    int none = 0;
    for (int t = (it > NS ? it - NS : 0); t < it; ++t)
        if (!ptx::mbar_wait_bounded(&full[t % NS], (t / NS) & 1, &none, WAIT_NS))
            report_timeout(a.status);
}

// Q^T of each unit: pair p's tile is [NQP N-rows][128 B] (dims 64 p .. 64 p + 63),
// 128-byte swizzle.  N-row n = (r / RH) 2 RH + parity RH + r % RH holds query
// row r's 32 dims of block 2p + parity (bytes 64 parity .. +64) and zeros over
// the other block's; query row r = t G + gq.
template <int NT>
__device__ __forceinline__ void role_qload(const DecodeArgs &a)
{
    using CF = Cfg<NT>;
    constexpr int RH = CF::RH;
    uint8_t *smem = smem_base();
    Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
    volatile int *abort = &hd.abort;
    const int lane = threadIdx.x & 31;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;
    const int C = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int units = a.n_layers * a.n_kv_heads * C;
    int ui = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++ui) {
        const int qb = ui & 1;
        if (ui >= 2 && !wwait(&hd.qfree[qb], ((ui >> 1) - 1) & 1, abort, a.status))
            break;
        if (*abort)
            break;
        const Unit un = unit_of(a, u, C);
        const __half *qbase = a.q + (int64_t)un.layer * a.T * a.n_q_heads * HD;
        uint8_t *qs = smem + CF::OFF_Q + qb * CF::QBUF;
        for (int e = lane; e < R * 32; e += 32) {
            const int r = e >> 5, b = (e >> 2) & 7, c4 = e & 3;  // 16-byte chunk c4 of block b
            const int p = b >> 1, par = b & 1;
            const int n = (r / RH) * 2 * RH + par * RH + r % RH;
            const int ch = 4 * par + c4;  // 16-byte chunk within the N-row
            const int t = r / G, gq = r % G;
            const __half *src =
                qbase + ((int64_t)t * a.n_q_heads + un.h * G + gq) * HD + 32 * b + 8 * c4;
            cp_async16(ptx::smem_u32(qs + p * CF::QPAIR + n * 128 + ((ch ^ (n & 7)) << 4)), src);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&hd.qfull[qb]);
    }
}

template <int NT>
__device__ __forceinline__ void role_mma(const DecodeArgs &a)
{
    using CF = Cfg<NT>;
    uint8_t *smem = smem_base();
    Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
    volatile int *abort = &hd.abort;
    const int lane = threadIdx.x & 31;
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(&hd.tmem_base);
    const int C = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int units = a.n_layers * a.n_kv_heads * C;
    // converged: the whole warp waits; one elected lane issues (a tcgen05.mma issued
    // inside a lane-divergent branch costs ~45 cycles to issue)
    const uint32_t leader = ptx::elect_one();
    const uint32_t idesc = ptx::idesc_f16_f32(TOK, CF::NQP, false, false);
    const uint64_t dq0 = ptx::smem_desc_sw128(smem + CF::OFF_Q, 16, 1024);
    bool ok = true;
    int it = 0, ui = 0;
    for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++ui) {
        const int qb = ui & 1;
        if (!(ok = wwait(&hd.qfull[qb], (ui >> 1) & 1, abort, a.status)))
            break;
        const int n_tiles = unit_of(a, u, C).n_tiles;
        const uint64_t dq = dq0 + (uint64_t)((qb * CF::QBUF) >> 4);
        for (int i = 0; i < n_tiles; ++i, ++it) {
            const int sb = it & 1;
            // the key tile of tile it, and S buffer sb read by the softmax of tile it - 2
            if (!(ok = wwait(&hd.kbfull, it & 1, abort, a.status)))
                break;
            if (it >= 2 && !(ok = wwait(&hd.sfree[sb], ((it >> 1) - 1) & 1, abort, a.status)))
                break;
            ptx::tc_fence_after();
            if (leader) {
#pragma unroll
                for (int p = 0; p < 4; ++p)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)  // dims 64 p + 16 ks .. +16
                        ptx::umma_f16_ts(tbase + CF::COL_S + CF::SBUF * sb + CF::NQP * p,
                                         tbase + CF::COL_K + 32 * p + 8 * ks,
                                         dq + (uint64_t)((p * CF::QPAIR + 32 * ks) >> 4), idesc,
                                         ks > 0);
                ptx::umma_commit(&hd.sfull[sb]);
                ptx::umma_commit(&hd.kbfree);
            }
            __syncwarp();
        }
        if (!ok)
            break;
        if (leader)
            ptx::umma_commit(&hd.qfree[qb]);
        __syncwarp();
    }
    // every issued MMA has finished before TMEM is freed: one commit tracks them all
    if (leader)
        ptx::umma_commit(&hd.drain);
    __syncwarp();
    if (lane == 0) {
        int none = 0;
        if (!ptx::mbar_wait_bounded(&hd.drain, 0, &none, WAIT_NS))
            report_timeout(a.status);
    }
    __syncwarp();
}

template <int NT>
__device__ __forceinline__ void role_conv(const DecodeArgs &a)
{
    using CF = Cfg<NT>;
    uint8_t *smem = smem_base();
    Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
    volatile int *abort = &hd.abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(&hd.tmem_base);
    const int C = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int units = a.n_layers * a.n_kv_heads * C;
    const int quad = warp & 3, hh = (warp - W_CONV) >> 2;
    const int key = 32 * quad + lane;
    const uint32_t taddr = tbase + ((uint32_t)(32 * quad) << 16) + CF::COL_K;
    const float dscale = a.scale * LOG2E;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
        const int n_tok = unit_of(a, u, C).n_tok;
        for (int i = 0; i * TOK < n_tok; ++i, ++it) {
            const int slot = it % NSK, ds = it & 1;
            // raw K landed; the key tile's MMAs of tile it - 1 and the d_k slot's reader
            // (softmax of tile it - 2) are done
            ok = wwait(&hd.kfull[slot], (it / NSK) & 1, abort, a.status);
            if (ok && it >= 1)
                ok = wwait(&hd.kbfree, (it - 1) & 1, abort, a.status);
            if (ok && it >= 2)
                ok = wwait(&hd.dkfree[ds], ((it >> 1) - 1) & 1, abort, a.status);
            if (!ok)
                break;
            ptx::tc_fence_after();
            const uint8_t *row = smem + CF::OFF_RK + slot * STAGE_K + key * KROW;
            float4 dsc = hh == 0 ? convert_key<0>(row, taddr, dscale)
                                 : convert_key<1>(row, taddr, dscale);
            if (key >= n_tok - i * TOK)  // past the chunk end: stale bytes, scale 0
                dsc = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(smem + CF::OFF_DK + ds * DKBUF + key * DKROW + 16 * hh) = dsc;
            ptx::mbar_arrive(&hd.kfree[slot]);
            ptx::mbar_arrive(&hd.dkfull[ds]);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&hd.kbfull);
        }
    }
}

template <int NT>
__device__ __forceinline__ void role_soft(const DecodeArgs &a)
{
    using CF = Cfg<NT>;
    constexpr int NR = CF::NR, RH = CF::RH;
    uint8_t *smem = smem_base();
    Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
    volatile int *abort = &hd.abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(&hd.tmem_base);
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;
    const int C = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int units = a.n_layers * a.n_kv_heads * C;
    const int quad = warp & 3, rh = (warp - W_SOFT) >> 2;
    const int key = 32 * quad + lane;  // = its TMEM lane
    const int r0 = RH * rh;            // first query row of this warp
    // pair p of S buffer sb: this warp's rows of block 2p at columns [2 RH rh, +RH),
    // of block 2p+1 at [2 RH rh + RH, +RH)
    const uint32_t taddr = tbase + ((uint32_t)(32 * quad) << 16) + CF::COL_S + 2 * RH * rh;
    float m[RH], l[RH];
    bool aborted = false;
    int it = 0, ui = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++ui) {
        const Unit un = unit_of(a, u, C);
#pragma unroll
        for (int r = 0; r < RH; ++r) {
            m[r] = M_INIT;
            l[r] = 0.0f;
        }
        for (int i = 0; i < un.n_tiles; ++i, ++it) {
            const int ds = it & 1, sb = it & 1, ps = it % NP;
            if (!aborted)
                aborted = !wwait(&hd.dkfull[ds], (it >> 1) & 1, abort, a.status);
            float dk[8];
            {
                const uint8_t *dp = smem + CF::OFF_DK + ds * DKBUF + key * DKROW;
                const float4 d0 = *reinterpret_cast<const float4 *>(dp);
                const float4 d1 = *reinterpret_cast<const float4 *>(dp + 16);
                dk[0] = d0.x; dk[1] = d0.y; dk[2] = d0.z; dk[3] = d0.w;
                dk[4] = d1.x; dk[5] = d1.y; dk[6] = d1.z; dk[7] = d1.w;
            }
            ptx::mbar_arrive(&hd.dkfree[ds]);
            float sv[RH];
#pragma unroll
            for (int r = 0; r < RH; ++r)
                sv[r] = 0.0f;
            if (!aborted)
                aborted = !wwait(&hd.sfull[sb], (it >> 1) & 1, abort, a.status);
            if (!aborted) {
                ptx::tc_fence_after();
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    uint32_t x[2 * RH];
#pragma unroll
                    for (int c8 = 0; c8 < 2 * RH / 8; ++c8) {
                        uint32_t y[8];
                        tmem_ld8(taddr + CF::SBUF * sb + CF::NQP * p + 8 * c8, y);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            x[8 * c8 + k] = y[k];
                    }
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int r = 0; r + 1 < RH; r += 2) {
                        ffma2(sv[r], sv[r + 1], dk[2 * p], __uint_as_float(x[r]),
                              __uint_as_float(x[r + 1]));
                        ffma2(sv[r], sv[r + 1], dk[2 * p + 1], __uint_as_float(x[RH + r]),
                              __uint_as_float(x[RH + r + 1]));
                    }
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&hd.sfree[sb]);
            // ---- masks: keys past the chunk end, the verify batch's causal rows,
            //      padded rows
            const int j = i * TOK + key;  // key index in the chunk
            const bool edge = (i + 1) * TOK > un.n_tok ||
                              un.c0 + (int64_t)(i + 1) * TOK - 1 > a.vis_last || R < NR;
            if (aborted || edge) {
                // token t sees keys <= vis_last + t: visible iff kk <= t
                const int64_t kk = un.c0 + j - a.vis_last;
#pragma unroll
                for (int r = 0; r < RH; ++r) {
                    const int rr = r0 + r;
                    const bool vis = !aborted && j < un.n_tok && rr < R && kk <= rr / G;
                    if (!vis)
                        sv[r] = -INFINITY;
                }
            }
            // the P slot (and its rescale record) is free once the value warps are done
            // with tile it - NP
            if (!aborted && it >= NP)
                aborted = !wwait(&hd.pfree[ps], ((it / NP) - 1) & 1, abort, a.status);
            // ---- running max shared by the eight warps
            float tmax = sv[0] - m[0];
#pragma unroll
            for (int r = 1; r < RH; ++r)
                tmax = fmaxf(tmax, sv[r] - m[r]);
            const bool any = named_bar_or(BAR_SOFT, 32 * N_SOFT, tmax > TAU);
            if (any) {
#pragma unroll
                for (int r = 0; r < RH; ++r) {
                    float v = sv[r];
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                    if (lane == 0)
                        hd.tmx[quad][r0 + r] = v;
                }
                ptx::named_bar_sync(BAR_SOFT, 32 * N_SOFT);
#pragma unroll
                for (int r = 0; r < RH; ++r) {
                    const int rr = r0 + r;
                    const float v = fmaxf(fmaxf(hd.tmx[0][rr], hd.tmx[1][rr]),
                                          fmaxf(hd.tmx[2][rr], hd.tmx[3][rr]));
                    const float mn = fmaxf(m[r], v);
                    const float al = ptx::ex2(m[r] - mn);
                    m[r] = mn;
                    l[r] *= al;
                    if (quad == 0 && lane == 0)
                        hd.alpha[ps][rr] = al;
                }
            }
            if (warp == W_SOFT && lane == 0)
                hd.changed[ps] = any ? 1 : 0;
            // ---- P = P_hi + P_lo, [key][row] f16 per part
            uint32_t ph[RH / 2], pl[RH / 2];
#pragma unroll
            for (int r = 0; r < RH; r += 2) {
                const float p0 = ptx::ex2(sv[r] - m[r]);
                const float p1 = ptx::ex2(sv[r + 1] - m[r + 1]);
                l[r] += p0;
                l[r + 1] += p1;
                // hi: p with its low 13 mantissa bits cleared (11 significant bits,
                // exact in f16 for p >= 2^-14); lo: the exact fp32 remainder, rounded
                const float h0 = __uint_as_float(__float_as_uint(p0) & 0xFFFFE000u);
                const float h1 = __uint_as_float(__float_as_uint(p1) & 0xFFFFE000u);
                ph[r / 2] = ptx::h2_bits(__floats2half2_rn(h0, h1));
                pl[r / 2] = ptx::h2_bits(__floats2half2_rn(p0 - h0, p1 - h1));
            }
            uint8_t *pslot = smem + CF::OFF_P + ps * CF::PSLOT + key * CF::PROW + 2 * r0;
            if constexpr (NT == 3) {
                if (rh == 0) {
                    *reinterpret_cast<uint4 *>(pslot) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
                    *reinterpret_cast<uint2 *>(pslot + 16) = make_uint2(ph[4], ph[5]);
                    *reinterpret_cast<uint4 *>(pslot + CF::PPART) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
                    *reinterpret_cast<uint2 *>(pslot + CF::PPART + 16) = make_uint2(pl[4], pl[5]);
                } else {
                    *reinterpret_cast<uint2 *>(pslot) = make_uint2(ph[0], ph[1]);
                    *reinterpret_cast<uint4 *>(pslot + 8) = make_uint4(ph[2], ph[3], ph[4], ph[5]);
                    *reinterpret_cast<uint2 *>(pslot + CF::PPART) = make_uint2(pl[0], pl[1]);
                    *reinterpret_cast<uint4 *>(pslot + CF::PPART + 8) = make_uint4(pl[2], pl[3], pl[4], pl[5]);
                }
            } else if constexpr (NT == 2) {
                *reinterpret_cast<uint4 *>(pslot) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
                *reinterpret_cast<uint4 *>(pslot + CF::PPART) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
            } else {
                *reinterpret_cast<uint2 *>(pslot) = make_uint2(ph[0], ph[1]);
                *reinterpret_cast<uint2 *>(pslot + CF::PPART) = make_uint2(pl[0], pl[1]);
            }
            ptx::mbar_arrive(&hd.pfull[ps]);
        }
        // ---- end of the unit: per-row sums over the warp's 32 keys, and the max
        const int lb = ui & 1;
        if (!aborted && ui >= 2)
            aborted = !wwait(&hd.lfree[lb], ((ui >> 1) - 1) & 1, abort, a.status);
#pragma unroll
        for (int r = 0; r < RH; ++r) {
            float v = l[r];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            if (lane == 0) {
                hd.fl[lb][quad][r0 + r] = v;
                if (quad == 0)
                    hd.fm[lb][r0 + r] = m[r];
            }
        }
        ptx::mbar_arrive(&hd.lfull[lb]);
    }
}

template <int NT>
__device__ __forceinline__ void role_val(const DecodeArgs &a)
{
    using CF = Cfg<NT>;
    uint8_t *smem = smem_base();
    Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
    volatile int *abort = &hd.abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;
    const int C = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int units = a.n_layers * a.n_kv_heads * C;
    const int b = warp - W_VAL;  // Q4_0 block b: head dims [32b, 32b + 32)
    const int g = lane >> 2, cq = lane & 3;
    const int Hq = a.n_q_heads;
    // ldmatrix row address of this lane: matrix lane/8 = (part, key half), row lane%8
    const int lm = lane >> 3;
    const uint32_t p_lane = ptx::smem_u32(smem + CF::OFF_P) + (lm >> 1) * CF::PPART +
                            (8 * (lm & 1) + (lane & 7)) * CF::PROW;
    float o[2][NT][4];
    bool ok = true;
    int it = 0, ui = 0;
    for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++ui) {
        const Unit un = unit_of(a, u, C);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    o[mt][nt][k] = 0.0f;
        for (int i = 0; i < un.n_tiles; ++i, ++it) {
            const int vs = it % NSV, ps = it % NP;
            ok = wwait(&hd.vfull[vs], (it / NSV) & 1, abort, a.status) &&
                 wwait(&hd.pfull[ps], (it / NP) & 1, abort, a.status);
            if (!ok)
                break;
            if (hd.changed[ps]) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const float al = hd.alpha[ps][nt * 8 + 2 * cq + k];
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            o[mt][nt][k] *= al;
                            o[mt][nt][2 + k] *= al;
                        }
                    }
            }
            // ---- O^T += V^T (P d_v)^T over the tile's groups, this warp's block
            const uint8_t *v0 = smem + CF::OFF_RV + vs * STAGE_V + (2 * cq) * VROW + 18 * b;
            const uint32_t pbase = p_lane + ps * CF::PSLOT;
            const int rows = min(TOK, un.n_tok - i * TOK);
            if (rows == TOK) {
#pragma unroll 2
                for (int w = 0; w < NGRP; ++w)
                    pv_group<NT, false>(o, v0 + (16 * w) * VROW, pbase + 16 * w * CF::PROW, 16, g,
                                        cq);
            } else {
                for (int w = 0; 16 * w < rows; ++w)
                    pv_group<NT, true>(o, v0 + (16 * w) * VROW, pbase + 16 * w * CF::PROW,
                                       rows - 16 * w, g, cq);
            }
            ptx::mbar_arrive(&hd.pfree[ps]);
            ptx::mbar_arrive(&hd.vfree[vs]);
        }
        if (!ok)
            break;
        // ---- end of the unit: the chunk partial of every live row
        const int lb = ui & 1;
        if (!(ok = wwait(&hd.lfull[lb], (ui >> 1) & 1, abort, a.status)))
            break;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int col = nt * 8 + 2 * cq + k;
                if (col >= R)
                    continue;
                const float L = hd.fl[lb][0][col] + hd.fl[lb][1][col] + hd.fl[lb][2][col] +
                                hd.fl[lb][3][col];
                const float f = L > 0.0f ? 1.0f / L : 0.0f;
                const int t = col / G, gq = col % G;
                const int64_t row = ((int64_t)un.layer * a.T + t) * Hq + un.h * G + gq;
                float *dst = a.out_part + (row * C + un.c) * HD + 32 * b + 2 * g;
                *reinterpret_cast<float2 *>(dst) = make_float2(o[0][nt][k] * f, o[0][nt][2 + k] * f);
                *reinterpret_cast<float2 *>(dst + 16) =
                    make_float2(o[1][nt][k] * f, o[1][nt][2 + k] * f);
                if (b == 0 && g == 0)
                    a.lse_part[row * C + un.c] =
                        L > 0.0f ? (hd.fm[lb][col] + log2f(L)) * LN2 : -INFINITY;
            }
        ptx::mbar_arrive(&hd.lfree[lb]);
    }
}

template <int NT>
__global__ void __launch_bounds__(THREADS, 1) decode_tmem_kernel(const DecodeArgs a)
{
    using CF = Cfg<NT>;
    {
        uint8_t *smem = smem_base();
        Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
        if (threadIdx.x == 0) {
            for (int i = 0; i < NSK; ++i) {
                ptx::mbar_init(&hd.kfull[i], 1);
                ptx::mbar_init(&hd.kfree[i], ALL * N_CONV);
            }
            for (int i = 0; i < NSV; ++i) {
                ptx::mbar_init(&hd.vfull[i], 1);
                ptx::mbar_init(&hd.vfree[i], ALL * N_VAL);
            }
            ptx::mbar_init(&hd.kbfull, ALL * N_CONV);
            ptx::mbar_init(&hd.kbfree, 1);
            for (int i = 0; i < 2; ++i) {
                ptx::mbar_init(&hd.dkfull[i], ALL * N_CONV);
                ptx::mbar_init(&hd.dkfree[i], ALL * N_SOFT);
                ptx::mbar_init(&hd.sfull[i], 1);
                ptx::mbar_init(&hd.sfree[i], ALL * N_SOFT);
                ptx::mbar_init(&hd.qfull[i], ALL);
                ptx::mbar_init(&hd.qfree[i], 1);
                ptx::mbar_init(&hd.lfull[i], ALL * N_SOFT);
                ptx::mbar_init(&hd.lfree[i], ALL * N_VAL);
            }
            for (int i = 0; i < NP; ++i) {
                ptx::mbar_init(&hd.pfull[i], ALL * N_SOFT);
                ptx::mbar_init(&hd.pfree[i], ALL * N_VAL);
            }
            ptx::mbar_init(&hd.drain, 1);
            ptx::mbar_init(&hd.never, 1);
            hd.abort = 0;
            ptx::fence_mbar_init();
        }
        // both Q^T buffers start as zeros: the block-diagonal halves and the N-rows
        // without a query row stay zero
        for (int i = threadIdx.x; i < 2 * CF::QBUF / 16; i += THREADS)
            reinterpret_cast<uint4 *>(smem + CF::OFF_Q)[i] = make_uint4(0u, 0u, 0u, 0u);
        ptx::fence_proxy_async_smem();
        if ((threadIdx.x >> 5) == W_MMA) {
            ptx::tmem_alloc(&hd.tmem_base, CF::TMEM_COLS);
            ptx::tmem_relinquish();
        }
        ptx::tc_fence_before();
    }
    __syncthreads();
    ptx::tc_fence_after();
    // Registers per warpgroup (launched with 72 per thread, 64,512 in all): each
    // role's branch first sets its budget -- the copy / MMA / Q warps and the convert
    // warps give registers up, the softmax and value warps take more.
    const int warp = threadIdx.x >> 5;
    if (warp < W_CONV) {
        ptx::setmaxnreg_dec<REG_CTL>();
        if (warp == W_KCOPY || warp == W_VCOPY) {
            if ((threadIdx.x & 31) == 0)
                role_copy<NT>(a, warp == W_KCOPY);
            __syncwarp();
        } else if (warp == W_QLOAD) {
            role_qload<NT>(a);
        } else {
            role_mma<NT>(a);
        }
    } else if (warp < W_SOFT) {
        ptx::setmaxnreg_dec<REG_CONV>();
        role_conv<NT>(a);
    } else if (warp < W_VAL) {
        ptx::setmaxnreg_inc<REG_SOFT>();
        role_soft<NT>(a);
    } else {
        ptx::setmaxnreg_inc<REG_VAL>();
        role_val<NT>(a);
    }
    ptx::tc_fence_before();
    __syncthreads();  // every role is past its last tile; copies and MMAs are done
    if ((threadIdx.x >> 5) == W_MMA) {
        ptx::tc_fence_after();
        uint8_t *smem = smem_base();
        Head &hd = *reinterpret_cast<Head *>(smem + CF::OFF_HEAD);
        ptx::tmem_dealloc(*reinterpret_cast<volatile uint32_t *>(&hd.tmem_base), CF::TMEM_COLS);
    }
}

// Per-device one-time launch set-up: the shared-memory attribute and the SM count.
std::atomic<int> g_sms[MAX_DEVICES];

template <int NT>
bool launch_nt(const DecodeArgs &a, cudaStream_t s)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES)
        return false;
    static std::atomic<int> smem_set[MAX_DEVICES];
    if (!ensure_smem(reinterpret_cast<const void *>(decode_tmem_kernel<NT>), smem_set,
                     smem_bytes<NT>()))
        return false;
    int sms = g_sms[dev].load(std::memory_order_acquire);
    if (sms == 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            sms < 1)
            return false;
        g_sms[dev].store(sms, std::memory_order_release);
    }
    const int64_t C = (a.n_kv + a.chunk - 1) / a.chunk;
    const int64_t units = (int64_t)a.n_layers * a.n_kv_heads * C;
    if (units >= (1ll << 31))
        return false;
    const int grid = (int)(units < sms ? units : sms);
    decode_tmem_kernel<NT><<<grid, THREADS, smem_bytes<NT>(), s>>>(a);
    return true;
}

}  // namespace

// The decode at head_dim 256 with the default block formats and up to 24 rows
// per KV head.
bool launch_decode_tmem(const DecodeArgs &a, cudaStream_t s)
{
    const int rows = (a.n_q_heads / a.n_kv_heads) * a.T;
    const int nt = (rows + 7) / 8;
    if (nt == 1)
        return launch_nt<1>(a, s);
    if (nt == 2)
        return launch_nt<2>(a, s);
    if (nt == 3)
        return launch_nt<3>(a, s);
    return false;
}

}  // namespace kvq
