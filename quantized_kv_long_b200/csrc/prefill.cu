// prefill.cu -- chunked prefill attention over the Q8_0/Q4_0 cache.
//
// What it computes ("Online Log-Sum-Exp prefill & pipelined prefetch" of the
// RX 9070 XT KV-streaming page: prefill computed chunk by chunk over streamed
// pages of keys with the log-sum-exp accumulated online): T new query tokens
// per layer, appended at rows [n_cached, n_cached + T), attend to keys
// j <= n_cached + t (query token t); GQA: query head g reads KV head g / G.
// out = sum_j p_j v^_j / l and lse = m + ln l over all visible keys, with the
// online (running max, running sum) merge carried across pages of keys
// inside the kernel.
//
// Kernels:
//  * prefill_tc_kernel -- the tensor-core path (tcgen05, TMEM) for rows that
//    see at least PF_MIN_KEYS keys (Q8_0 K / Q4_0 V at head_dim 256).  One CTA
//    per (128 query rows of one KV head's group, (layer, KV head) pair); rows
//    are (token, q head) pairs.  Per tile of 32 keys, in the variant that
//    dequantizes in the CTA (PRE = false):
//      - a producer thread bulk-copies the tile's raw Q8_0 K head-rows (32 x
//        272 B) and Q4_0 V head-rows (32 x 144 B) into a 4-slot staging ring,
//        so that three tiles of copies are in flight while one is dequantized;
//      - 8 dequant warps (one (key, block) unit of K and one of V per thread)
//        turn them into f16 tiles in shared memory with 128-byte swizzle:
//        K^ = d * q as an exact two-part f16 sum (K^hi = RN_f16(d q),
//        K^lo = fma(d, q, -K^hi)), K-major (keys x head_dim), and
//        V^ = RN_f16(d * (u - 8)) MN-major (keys x head_dim), zeros past the
//        end; three slots of each;
//      - the MMA warp (warp-converged; one elected lane issues) runs
//        tcgen05.mma: S = Q K^hi^T + Q K^lo^T (A = Q held in tensor memory,
//        M = 128, N = 32, K = 256, twice) into one of 4 S slots in TMEM --
//        exact products, so the logits carry only fp32 rounding -- then
//        O += P V^ (A = P in TMEM, written over its S slot; N = 256, K = 32)
//        into the fp32 O accumulator in TMEM (256 columns).  A slot is
//        rewritten four tiles later, once that tile's PV has finished, so the
//        tensor pipe never waits for its own last PV;
//      - 4 softmax warps own one query row per thread (its TMEM lane): they
//        read S, apply the causal mask, keep a lazy running max (moves only
//        when a score exceeds it by 8 in log2 units, with an exact rescale of
//        O in TMEM) and write P = 2^(s - m) as f16 back into the slot.
//    With a workspace (PRE = true) prefill_expand_kernel first writes every
//    tile of a (layer, KV head) pair once as its three swizzled f16 images into
//    the pair's slab; the tensor-core kernel then bulk-copies the images into 4
//    slots (no dequant warps).  A workspace of fewer slabs than pairs is used in
//    chunks of pairs through its two halves, alternating between the caller's
//    stream and a second one (launch_prefill).
//    V^ and P carry one f16 rounding each (relative 2^-11).  These errors are
//    independent per key and average over the visible keys, but a row whose
//    softmax is peaked (a large query component on an x8 outlier channel) can
//    give one key a large share of the weight at a few thousand keys, and one
//    f16 rounding of |v^| ~ 20 is ~1e-2; a rounded K^ would move that key's
//    logit by ~2e-3 (why K^ is split exactly).  Measured max-abs error of this
//    path against the oracle (96 sampled rows, N(0,1) K/V with x8 outlier
//    channels): 4.7e-4 at 4,352 keys, 2.2e-4 at 16,384, 9.1e-5 at 65,536,
//    8.8e-5 at 262,144 (tolerance 2e-3).  Rows that see fewer than
//    PF_MIN_KEYS = 16,384 keys take the exact kernel.
//  * prefill_exact_kernel -- CUDA cores, fp32 with per-block scaling (the
//    same arithmetic as the general decode kernel), templated on both block
//    formats, for rows that see fewer than PF_MIN_KEYS keys, for every other
//    format pair and head_dim, and for calls that ask for per-page partials
//    (a page is a short context, where the f16 rounding above misses the
//    tolerance: measured 4.0-5.2e-3).
// Every mbarrier wait is bounded; a wait that runs out records
// KVQ_ERR_TIMEOUT in the status word and the roles fall through, waiting
// (bounded) for their own copies and MMAs before the CTA frees TMEM and exits.
#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace kvq {

namespace {

constexpr int PF_MIN_KEYS = 16384;
constexpr int BM = 128, BN = 32, HD = 256;
constexpr int KROW = 272, VROW = 144;
constexpr int RAW_K = BN * KROW, RAW_V = BN * VROW, RAW_BYTES = RAW_K + RAW_V;  // 13,312 B
constexpr int TILE_H = BN * HD * 2;  // one f16 tile of 32 keys x 256 dims: 16 KB
constexpr int NR = 4;  // raw staging slots (bulk copies in flight ahead of the dequant)
// f16 K^hi / K^lo / V^ tile slots: 3 beside the raw staging ring, 4 when the tiles
// come expanded from the workspace (no raw ring, and one more tile of copy lead)
template <bool PRE> constexpr int nb() { return PRE ? 4 : 3; }
constexpr int NB_MAX = 4;
constexpr int NS = 4;  // S / P slots in tensor memory
constexpr int N_SOFT = 4, N_DEQ = 8;
// roles: softmax warps, dequant warps (none when the f16 tiles were expanded into
// the workspace beforehand), the producer warp, the MMA warp
template <bool PRE> constexpr int n_deq() { return PRE ? 0 : N_DEQ; }
// softmax warps: one per TMEM lane quadrant, each with all 32 keys of a tile (P
// overwrites the tile's scores in tensor memory, so a warp that shared a quadrant
// would need a per-tile barrier before writing it; measured slower)
template <bool PRE> constexpr int n_soft() { return N_SOFT; }
template <bool PRE> constexpr int w_prod() { return n_soft<PRE>() + n_deq<PRE>(); }
template <bool PRE> constexpr int w_mma() { return w_prod<PRE>() + 1; }
template <bool PRE> constexpr int pf_threads() { return (w_mma<PRE>() + 1) * 32; }  // 14 / 6 warps
constexpr int TILE3 = 3 * TILE_H;  // one key tile's K^hi, K^lo, V^ in the workspace: 48 KB
constexpr uint64_t WAIT_NS = 1000000000ull;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float TAU = 8.0f;
constexpr float M_INIT = -1.0e30f;
// tensor-memory columns: O (fp32, 256), Q (f16 pairs, 128), S slot s at COL_S0 + BN s
// (P of that tile, f16 pairs, is written over the first BN / 2 columns of its slot)
constexpr uint32_t COL_O = 0, COL_Q = 256, COL_S0 = 384;
static_assert(COL_S0 + NS * BN <= 512, "tensor-memory columns");
static_assert(BN * 8 == N_DEQ * 32, "one K unit and one V unit per dequant thread and tile");
// The MMA warp waits only for k_full(j) and p_full(j - 1) per tile, and k_full(j)
// must imply that the PV of tile j - NS (which read the S/P slot the QK^T of tile j
// rewrites) is done.  PVs finish in order.
//  - Dequant warps: k_full(j) completes after every dequant warp has finished V^ of
//    tile j - 1 (program order in each warp), which waited for the PV of tile
//    j - 1 - NB; so k_full(j) covers v_full(j - 1) too.  Needs NB + 1 <= NS.
//  - Expanded tiles: the producer copies tile j after the PV of tile j - NB is done.
//    Needs NB <= NS.
static_assert(nb<false>() + 1 <= NS && nb<true>() <= NS, "k_full(j): the PV of tile j - NS");

struct PfSmemHead {
    uint64_t raw_full[NR], raw_free[NR], k_full[NB_MAX], v_full[NB_MAX], s_full[NS], p_full[NS],
        pv_done[NS], q_ready;
    uint64_t mma_drain;              // one commit after the last MMA: all of them are done
    uint64_t never;                  // test hook: a barrier that nothing completes
    uint32_t tmem_base;
    int abort;
};
// layout: [K^hi NB x 16K][K^lo NB x 16K][V^ NB x 16K][raw NR x 13,312 (dequant warps
// only)][head], base 1024-aligned
template <bool PRE> constexpr int off_head()
{
    return 3 * nb<PRE>() * TILE_H + (PRE ? 0 : NR * RAW_BYTES);
}
template <bool PRE> constexpr int pf_smem()
{
    return off_head<PRE>() + (int)sizeof(PfSmemHead) + 1024;  // + alignment slack
}
static_assert(pf_smem<false>() <= 232448 && pf_smem<true>() <= 232448,
              "dynamic shared memory per block");

// slot and phase parity of tile t in a ring of S slots
__device__ __forceinline__ int slot(int t, int S) { return t % S; }
__device__ __forceinline__ uint32_t par(int t, int S) { return (uint32_t)(t / S) & 1u; }

// byte offset of (row, dim) in a [BN rows x 256 dims] f16 tile stored as four
// 1024-aligned column blocks of [BN rows x 128 B] with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw_off(int row, int dim)
{
    const int c16 = (dim >> 3) & 7;
    return (uint32_t)((dim >> 6) * (BN * 128) + row * 128 + ((c16 ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t lds32(const uint8_t *p) { return *reinterpret_cast<const uint32_t *>(p); }
__device__ __forceinline__ uint32_t lds16(const uint8_t *p) { return *reinterpret_cast<const uint16_t *>(p); }

__device__ __forceinline__ __half2 dup_h(uint32_t d16)
{
    return ptx::bits_h2(d16 | (d16 << 16));
}

// four int8 -> d * q as an exact two-part f16 sum: x = RN(d q) (two half2) and
// r = d q - x = fma(d, q, -x) (exact: q has 8 significant bits, d 11)
__device__ __forceinline__ void k4(uint32_t w, __half2 d2, uint32_t (&x)[2], uint32_t (&r)[2])
{
    w ^= 0x80808080u;
    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
    const __half2 a = __hsub2(ptx::bits_h2(ptx::prmt(w, 0x64646464u, 0x5140)), bias);
    const __half2 b = __hsub2(ptx::bits_h2(ptx::prmt(w, 0x64646464u, 0x7362)), bias);
    const __half2 xa = __hmul2_rn(a, d2), xb = __hmul2_rn(b, d2);
    x[0] = ptx::h2_bits(xa);
    x[1] = ptx::h2_bits(xb);
    r[0] = ptx::h2_bits(__hfma2(a, d2, __hneg2(xa)));
    r[1] = ptx::h2_bits(__hfma2(b, d2, __hneg2(xb)));
}

// two Q4_0 bytes (at bits 0-7 and 16-23 of x) -> low-nibble and high-nibble half2, times d
__device__ __forceinline__ void v2(uint32_t x, __half2 d2, uint32_t &lo, uint32_t &hi)
{
    const __half2 c1032 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
    const __half2 s16 = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
    const __half2 c72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
    const __half2 a = __hsub2(ptx::bits_h2((x & 0x000F000Fu) | 0x64006400u), c1032);
    const __half2 b = __hfma2(ptx::bits_h2((x & 0x00F000F0u) | 0x64006400u), s16, c72);
    lo = ptx::h2_bits(__hmul2_rn(a, d2));
    hi = ptx::h2_bits(__hmul2_rn(b, d2));
}

__device__ __forceinline__ void sts128(uint8_t *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}

// Dequant of one (key r, 32-element block bk) unit of a raw tile into the f16
// tiles (offsets off[m4] of dims 32 bk + 8 m4 of key r, from sw_off); keys past
// the end (in = false) are written as zeros so that 0-weight products stay 0.
// K: rk = raw Q8_0 head-rows (KROW bytes each) -> K^hi, K^lo (exact two-part).
__device__ __forceinline__ void dequant_k_unit(const uint8_t *rk, int r, int bk, bool in,
                                               const uint32_t (&off)[4], uint8_t *kh, uint8_t *kl)
{
    if (in) {
        // ---- K block: d (fp16) + 32 int8
        const uint8_t *src = rk + r * KROW + 34 * bk;
        uint32_t w[8];
        uint32_t d16;
        if ((bk & 1) == 0) {  // block starts 4-byte aligned: d, q0, q1 | ...
            uint32_t x[9];
#pragma unroll
            for (int q = 0; q < 9; ++q)
                x[q] = lds32(src + 4 * q);
            d16 = x[0] & 0xFFFFu;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                w[q] = ptx::prmt(x[q], x[q + 1], 0x5432);
        } else {              // qs start 4-byte aligned
            d16 = lds16(src);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                w[q] = lds32(src + 2 + 4 * q);
        }
        const __half2 d2 = dup_h(d16);
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4) {
            uint32_t x0[2], x1[2], r0[2], r1[2];
            k4(w[2 * m4], d2, x0, r0);
            k4(w[2 * m4 + 1], d2, x1, r1);
            sts128(kh + off[m4], x0[0], x0[1], x1[0], x1[1]);
            sts128(kl + off[m4], r0[0], r0[1], r1[0], r1[1]);
        }
    } else {
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4) {
            sts128(kh + off[m4], 0u, 0u, 0u, 0u);
            sts128(kl + off[m4], 0u, 0u, 0u, 0u);
        }
    }
}

// V: rv = raw Q4_0 head-rows (VROW bytes each) -> V^.
__device__ __forceinline__ void dequant_v_unit(const uint8_t *rv, int r, int bk, bool in,
                                               const uint32_t (&off)[4], uint8_t *vh)
{
    if (in) {
        // ---- V block: d (fp16) + 16 bytes of nibbles
        const uint8_t *vsrc = rv + r * VROW + 18 * bk;
        uint32_t vw[4];
        uint32_t d16;
        if ((bk & 1) == 0) {
            uint32_t x[5];
#pragma unroll
            for (int q = 0; q < 5; ++q)
                x[q] = lds32(vsrc + 4 * q);
            d16 = x[0] & 0xFFFFu;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                vw[q] = ptx::prmt(x[q], x[q + 1], 0x5432);
        } else {
            d16 = lds16(vsrc);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                vw[q] = lds32(vsrc + 2 + 4 * q);
        }
        const __half2 dv = dup_h(d16);
        // byte j of the block: element j (low nibble), element j + 16 (high)
        uint32_t lo[8], hi[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            v2(ptx::prmt(vw[q], 0u, 0x4140), dv, lo[2 * q], hi[2 * q]);          // bytes 0, 1
            v2(ptx::prmt(vw[q], 0u, 0x4342), dv, lo[2 * q + 1], hi[2 * q + 1]);  // bytes 2, 3
        }
        sts128(vh + off[0], lo[0], lo[1], lo[2], lo[3]);
        sts128(vh + off[1], lo[4], lo[5], lo[6], lo[7]);
        sts128(vh + off[2], hi[0], hi[1], hi[2], hi[3]);
        sts128(vh + off[3], hi[4], hi[5], hi[6], hi[7]);
    } else {
        // keys past the end: zero V so that 0-weight products stay 0
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4)
            sts128(vh + off[m4], 0u, 0u, 0u, 0u);
    }
}

template <bool PRE>
__global__ void __launch_bounds__(pf_threads<PRE>(), 1) prefill_tc_kernel(const PrefillArgs a, int row0)
{
    extern __shared__ __align__(1024) uint8_t pf_raw[];
    uint8_t *smem = pf_raw + ((1024u - (ptx::smem_u32(pf_raw) & 1023u)) & 1023u);
    constexpr int NB = nb<PRE>();
    constexpr int OFF_KH = 0, OFF_KL = NB * TILE_H, OFF_VH = 2 * NB * TILE_H;
    constexpr int OFF_RAW = 3 * NB * TILE_H, OFF_HEAD = off_head<PRE>();
    PfSmemHead &hd = *reinterpret_cast<PfSmemHead *>(smem + OFF_HEAD);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int rows_total = a.T * G;
    // (layer, KV head) pair of this CTA; `slab` indexes its key tiles in the workspace
    const int slab = blockIdx.y + blockIdx.z * gridDim.y;
    const int pair = a.pair0 + slab;
    const int h = pair % a.n_kv_heads, layer = pair / a.n_kv_heads;
    const int R0 = row0 + blockIdx.x * BM;                 // first row of this tile
    const int r_last = min(R0 + BM, rows_total) - 1;
    const int64_t n_keys = a.n_cached + r_last / G + 1;    // keys any row of the tile sees
    const int ntiles = (int)((n_keys + BN - 1) / BN);
    const int64_t cap = a.layers.cap[layer];
    const uint8_t *kg = a.layers.k[layer] + (int64_t)h * cap * KROW;
    const uint8_t *vg = a.layers.v[layer] + (int64_t)h * cap * VROW;
    volatile int *abort = &hd.abort;
    // test hook: the first CTA's producer waits on a barrier that nothing completes
    const bool hook_wait = a.test_timeout && blockIdx.x == 0 && pair == 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NR; ++i) {
            ptx::mbar_init(&hd.raw_full[i], 1);
            ptx::mbar_init(&hd.raw_free[i], N_DEQ);
        }
        for (int i = 0; i < NB; ++i) {
            ptx::mbar_init(&hd.k_full[i], PRE ? 1 : N_DEQ);  // PRE: one copy of the whole tile
            ptx::mbar_init(&hd.v_full[i], N_DEQ);
        }
        for (int i = 0; i < NS; ++i) {
            ptx::mbar_init(&hd.s_full[i], 1);
            ptx::mbar_init(&hd.p_full[i], n_soft<PRE>());
            ptx::mbar_init(&hd.pv_done[i], 1);
        }
        ptx::mbar_init(&hd.q_ready, n_soft<PRE>());
        ptx::mbar_init(&hd.mma_drain, 1);
        ptx::mbar_init(&hd.never, 1);
        hd.abort = 0;
        ptx::fence_mbar_init();
    }
    constexpr int W_PROD = w_prod<PRE>(), W_MMA = w_mma<PRE>();
    if (warp == W_MMA) {
        ptx::tmem_alloc(&hd.tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tbase = hd.tmem_base;
    auto fail = [&]() {
        if (!*abort) {
            *abort = 1;
            report_timeout(a.status);
        }
    };
    // warp-wide bounded wait: lane 0 waits, the result is broadcast
    auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
        bool ok = true;
        if (lane == 0)
            ok = ptx::mbar_wait_bounded(bar, parity, abort, WAIT_NS);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };

    if (warp < n_soft<PRE>()) {
        // ================================================================ softmax
        // Warp quad owns the query rows of TMEM lane quadrant quad (one row per thread)
        // and all 32 keys of every tile: it reads the tile's scores, then writes P over
        // them.  Each 8-key group g of a tile has its own running sum l_g; l = (l_0 +
        // l_1) + (l_2 + l_3) at the end.
        const int quad = warp & 3;
        const int i = quad * 32 + lane;   // query row of this thread = its TMEM lane
        const int gr = R0 + i;
        const bool live = gr <= r_last;
        const int t = live ? gr / G : 0, gq = live ? gr % G : 0;
        const int64_t lim = a.n_cached + t;  // last visible key
        const uint32_t lane_addr = tbase + ((uint32_t)(quad * 32) << 16);
        {   // Q row -> TMEM columns [COL_Q, COL_Q + 128): two f16 per column, lower dim low
            const uint4 *qp = reinterpret_cast<const uint4 *>(
                a.q + (((int64_t)layer * a.T + t) * a.n_q_heads + (int64_t)h * G + gq) * HD);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t r[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 x = live ? qp[c * 4 + v] : make_uint4(0u, 0u, 0u, 0u);
                    r[4 * v + 0] = x.x;
                    r[4 * v + 1] = x.y;
                    r[4 * v + 2] = x.z;
                    r[4 * v + 3] = x.w;
                }
                ptx::tmem_st16(lane_addr + COL_Q + 16 * c, r);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&hd.q_ready);
        }
        const float sl2 = a.scale * LOG2E;
        float m = M_INIT, l[4];             // l[g]: running sum of 8-key group g
#pragma unroll
        for (int k = 0; k < 4; ++k)
            l[k] = 0.0f;
        const int64_t row_out = ((int64_t)layer * a.T + t) * a.n_q_heads + (int64_t)h * G + gq;
        // out = O / l and lse = (m + log2 l) ln 2 of this thread's row into dsto / dstl,
        // once the PV of tile `last` is done.  false: a wait ran out.
        auto emit = [&](int last, float *dsto, float *dstl) -> bool {
            if (!wwait(&hd.pv_done[slot(last, NS)], par(last, NS)))
                return false;
            const float lt = (l[0] + l[1]) + (l[2] + l[3]);
            ptx::tc_fence_after();
            const float inv = lt > 0.0f ? 1.0f / lt : 0.0f;
            float4 *op = reinterpret_cast<float4 *>(dsto);
            for (int c = 0; c < 16; ++c) {
                uint32_t r[16];
                ptx::tmem_ld16(lane_addr + COL_O + 16 * c, r);
                ptx::tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        op[c * 4 + v] = make_float4(__uint_as_float(r[4 * v]) * inv,
                                                    __uint_as_float(r[4 * v + 1]) * inv,
                                                    __uint_as_float(r[4 * v + 2]) * inv,
                                                    __uint_as_float(r[4 * v + 3]) * inv);
                }
            }
            if (live)
                *dstl = lt > 0.0f ? (m + log2f(lt)) * LN2 : -INFINITY;
            return true;
        };
        bool ok = true;
        for (int j = 0; ok && j < ntiles; ++j) {
            const int sb = slot(j, NS);
            const uint32_t scol = COL_S0 + BN * sb;
            if (!wwait(&hd.s_full[sb], par(j, NS))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            // every warp reads the whole tile's 32 scores (keys in order)
            float sc[BN];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                uint32_t r[16];
                ptx::tmem_ld16(lane_addr + scol + 16 * k, r);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    sc[16 * k + e] = __uint_as_float(r[e]);
            }
            ptx::tmem_wait_ld();
            const int64_t kj0 = (int64_t)j * BN;
            if (kj0 + BN - 1 > lim) {  // causal edge / end of the keys
#pragma unroll
                for (int e = 0; e < BN; ++e)
                    if (kj0 + e > lim)
                        sc[e] = -INFINITY;
            }
            float mx8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                mx8[e] = fmaxf(fmaxf(sc[e], sc[e + 8]), fmaxf(sc[e + 16], sc[e + 24]));
            // scaling is monotonic: the max of the scaled scores
            const float mx = sl2 * fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            float alpha = 1.0f;
            if (mx > m + TAU) {  // lazy running max: moves only by more than TAU
                alpha = ptx::ex2(m - mx);
                m = mx;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    l[k] *= alpha;
            }
            // rescale this warp's columns of O (rare): the whole warp takes part once any
            // lane needs it, after the PV of the previous tile has finished
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                if (!wwait(&hd.pv_done[slot(j - 1, NS)], par(j - 1, NS))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (int c = 0; c < 16; ++c) {
                    uint32_t r[16];
                    ptx::tmem_ld16(lane_addr + COL_O + 16 * c, r);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                    ptx::tmem_st16(lane_addr + COL_O + 16 * c, r);
                }
                ptx::tmem_wait_st();
            }
            // P = 2^(s scale - m) in f16 (keys 2e, 2e + 1 of the tile in column e of this S
            // slot), and each 8-key group's sum ((p0 + p1) + (p2 + p3)) + ((p4 + p5) +
            // (p6 + p7))
            uint32_t pk[16];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float pr[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float p0 = ptx::ex2(fmaf(sc[8 * k + 2 * e], sl2, -m));
                    const float p1 = ptx::ex2(fmaf(sc[8 * k + 2 * e + 1], sl2, -m));
                    pr[e] = p0 + p1;
                    pk[4 * k + e] = ptx::h2_bits(__floats2half2_rn(p0, p1));
                }
                l[k] += (pr[0] + pr[1]) + (pr[2] + pr[3]);
            }
            ptx::tmem_st16(lane_addr + scol, pk);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&hd.p_full[sb]);
        }
        if (!ok && lane == 0)
            fail();
        // ---- epilogue: out = O / l, lse = (m + log2 l) ln 2, l = l[0] + l[1]
        if (ok && !*abort && !emit(ntiles - 1, a.out + row_out * HD, a.lse + row_out) &&
            lane == 0)
            fail();
    } else if (warp < W_PROD) {
        // ================================================================ dequant
        // Each of the 256 dequant threads owns one (key r, block bk) unit of every
        // tile, for K and for V.  A warp takes 8 keys x 4 blocks of one parity
        // (bk = p, p+2, p+4, p+6): the even/odd alignment branch is uniform across
        // the warp, the 8 lanes of each quarter-warp store 8 different keys of one
        // block (8 different bank groups after the swizzle), and the raw 32-bit
        // loads (rows 68 words apart, blocks 17 words apart) hit 32 different banks.
        const int dt = threadIdx.x - N_SOFT * 32;  // 0..255
        const int grp = dt >> 5, ln = dt & 31;
        const int r = (grp % (BN / 8)) * 8 + (ln & 7), bk = grp / (BN / 8) + 2 * (ln >> 3);
        uint32_t off[4];  // swizzled offsets of dims 32 bk + 8 m4 of key r in an f16 tile
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4)
            off[m4] = sw_off(r, 32 * bk + 8 * m4);
        for (int j = 0; j < ntiles; ++j) {
            const int rb = slot(j, NR), kb = slot(j, NB);
            // raw tile j has landed; K^ slot kb is free once the QK^T of tile j - NB is done
            if (!wwait(&hd.raw_full[rb], par(j, NR)) ||
                (j >= NB && !wwait(&hd.s_full[slot(j - NB, NS)], par(j - NB, NS)))) {
                if (lane == 0)
                    fail();
                break;
            }
            const bool in = r < (int)min((int64_t)BN, n_keys - (int64_t)j * BN);
            const uint8_t *rk = smem + OFF_RAW + rb * RAW_BYTES;
            const uint8_t *rv = rk + RAW_K;
            uint8_t *kh = smem + OFF_KH + kb * TILE_H;
            uint8_t *kl = smem + OFF_KL + kb * TILE_H;
            uint8_t *vh = smem + OFF_VH + kb * TILE_H;
            dequant_k_unit(rk, r, bk, in, off, kh, kl);
            ptx::fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&hd.k_full[kb]);
            // V^ slot kb is free once the PV of tile j - NB is done
            if (j >= NB && !wwait(&hd.pv_done[slot(j - NB, NS)], par(j - NB, NS))) {
                if (lane == 0)
                    fail();
                break;
            }
            dequant_v_unit(rv, r, bk, in, off, vh);
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&hd.raw_free[rb]);
                ptx::mbar_arrive(&hd.v_full[kb]);
            }
        }
    } else if (warp == W_PROD && PRE) {
        // ================================================================ copies (PRE)
        // The f16 tiles were expanded into the workspace: tile j of (layer, h) is one
        // 48 KB image of the three slots.  Slot kb is free once the QK^T (K^) and the
        // PV (V^) of tile j - NB are done; one transaction barrier covers the tile.
        if (lane == 0 && hook_wait && !ptx::mbar_wait_bounded(&hd.never, 0, abort, WAIT_NS))
            fail();
        if (lane == 0) {
            const int tiles_total = (int)((a.n_cached + a.T + BN - 1) / BN);
            const uint8_t *wsb = static_cast<const uint8_t *>(a.workspace) +
                                 (int64_t)slab * tiles_total * TILE3;
            int issued = 0;
            for (int j = 0; j < ntiles; ++j) {
                const int kb = slot(j, NB);
                if (*abort || (j >= NB && (!ptx::mbar_wait_bounded(&hd.s_full[slot(j - NB, NS)],
                                                                   par(j - NB, NS), abort, WAIT_NS) ||
                                           !ptx::mbar_wait_bounded(&hd.pv_done[slot(j - NB, NS)],
                                                                   par(j - NB, NS), abort, WAIT_NS)))) {
                    fail();
                    break;
                }
                const uint8_t *src = wsb + (int64_t)j * TILE3;
                ptx::mbar_arrive_expect_tx(&hd.k_full[kb], TILE3);
                ptx::bulk_g2s(smem + OFF_KH + kb * TILE_H, src, TILE_H, &hd.k_full[kb]);
                ptx::bulk_g2s(smem + OFF_KL + kb * TILE_H, src + TILE_H, TILE_H, &hd.k_full[kb]);
                ptx::bulk_g2s(smem + OFF_VH + kb * TILE_H, src + 2 * TILE_H, TILE_H, &hd.k_full[kb]);
                issued = j + 1;
            }
            // no copy may still be landing when the CTA exits
            int none = 0;
            for (int j = (issued > NB ? issued - NB : 0); j < issued; ++j)
                if (!ptx::mbar_wait_bounded(&hd.k_full[slot(j, NB)], par(j, NB), &none, WAIT_NS))
                    report_timeout(a.status);
        }
    } else if (warp == W_PROD) {
        // ================================================================ copies
        if (lane == 0 && hook_wait && !ptx::mbar_wait_bounded(&hd.never, 0, abort, WAIT_NS))
            fail();
        if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < ntiles; ++j) {
                const int rb = slot(j, NR);
                // raw slot rb is free once every dequant warp is done with tile j - NR
                if (*abort || (j >= NR && !ptx::mbar_wait_bounded(&hd.raw_free[rb], par(j - NR, NR),
                                                                   abort, WAIT_NS))) {
                    fail();
                    break;
                }
                const int rows = (int)min((int64_t)BN, n_keys - (int64_t)j * BN);
                uint8_t *dst = smem + OFF_RAW + rb * RAW_BYTES;
                ptx::mbar_arrive_expect_tx(&hd.raw_full[rb], rows * (KROW + VROW));
                ptx::bulk_g2s(dst, kg + (int64_t)j * RAW_K, rows * KROW, &hd.raw_full[rb]);
                ptx::bulk_g2s(dst + RAW_K, vg + (int64_t)j * RAW_V, rows * VROW, &hd.raw_full[rb]);
                issued = j + 1;
            }
            // no copy may still be landing when the CTA exits
            int none = 0;
            for (int j = (issued > NR ? issued - NR : 0); j < issued; ++j)
                if (!ptx::mbar_wait_bounded(&hd.raw_full[slot(j, NR)], par(j, NR), &none, WAIT_NS))
                    report_timeout(a.status);
        }
    } else {
        // ================================================================ MMA issue
        // The whole warp runs this loop (descriptors stay warp-uniform); the
        // elected lane issues every MMA and commit, so all tcgen05 work of the
        // CTA comes from one thread and each commit covers what came before.
        const uint32_t leader = ptx::elect_one();
        // the MMA warp's waits: every lane tests the barrier without blocking (no
        // lane-divergent branch, no broadcast), bounded in time and by the abort flag
        auto mwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            if (ptx::mbar_test(bar, parity))
                return true;
            const uint64_t t0 = ptx::globaltimer_ns();
            for (;;) {
                if (ptx::mbar_test(bar, parity))
                    return true;
                if (*abort || ptx::globaltimer_ns() - t0 > WAIT_NS)
                    return false;
            }
        };
        const uint32_t id_qk = ptx::idesc_f16_f32(BM, BN, false, false);
        const uint32_t id_pv = ptx::idesc_f16_f32(BM, HD, false, true);
        // descriptors of slot 0; slots and k-steps add to the start-address field
        // (16-byte units; every tile lies inside one 256 KB window)
        const uint64_t dk_hi0 = ptx::smem_desc_sw128(smem + OFF_KH, 16, 1024);
        const uint64_t dk_lo0 = ptx::smem_desc_sw128(smem + OFF_KL, 16, 1024);
        const uint64_t dv0 = ptx::smem_desc_sw128(smem + OFF_VH, BN * 128, 1024);
        bool ok = wwait(&hd.q_ready, 0);
        // PV of tile jj, issued after the QK^T of tile jj + 1: V^ is ready once
        // k_full(jj + 1) has completed (see NS above); the last tile has no successor
        // and waits for v_full itself
        auto issue_pv = [&](int jj) -> bool {
            const int vb = slot(jj, NB), sb = slot(jj, NS);
            if ((!PRE && jj == ntiles - 1 && !mwait(&hd.v_full[vb], par(jj, NB))) ||
                !mwait(&hd.p_full[sb], par(jj, NS)))
                return false;
            ptx::tc_fence_after();
            if (leader) {
                const uint64_t dv = dv0 + (uint64_t)((vb * TILE_H) >> 4);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    ptx::umma_f16_ts(tbase + COL_O, tbase + COL_S0 + BN * sb + 8 * kk,
                                     dv + (uint64_t)((kk * 2 * 1024) >> 4), id_pv, jj > 0 || kk > 0);
                ptx::umma_commit(&hd.pv_done[sb]);
            }
            __syncwarp();
            return true;
        };
        for (int j = 0; ok && j < ntiles; ++j) {
            const int kb = slot(j, NB), sb = slot(j, NS);
            // K^ of tile j is ready, and (see NS above) the PV of tile j - NS that read
            // S/P slot sb is done
            ok = mwait(&hd.k_full[kb], par(j, NB));
            if (!ok)
                break;
            ptx::tc_fence_after();
            if (leader) {
                // S = Q K^hi^T + Q K^lo^T: exact products of q and d*q_int, fp32 sums
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint64_t dk = (part ? dk_lo0 : dk_hi0) + (uint64_t)((kb * TILE_H) >> 4);
#pragma unroll
                    for (int ks = 0; ks < HD / 16; ++ks)
                        ptx::umma_f16_ts(tbase + COL_S0 + BN * sb, tbase + COL_Q + 8 * ks,
                                         dk + (uint64_t)(((ks >> 2) * (BN * 128) + (ks & 3) * 32) >> 4),
                                         id_qk, part > 0 || ks > 0);
                }
                ptx::umma_commit(&hd.s_full[sb]);
            }
            __syncwarp();
            if (j >= 1)
                ok = issue_pv(j - 1);
        }
        if (ok)
            ok = issue_pv(ntiles - 1);
        if (!ok && lane == 0)
            fail();
        // every issued MMA has finished before TMEM is freed, also after a failed wait:
        // one commit tracks all earlier tcgen05 operations of the issuing thread
        if (leader)
            ptx::umma_commit(&hd.mma_drain);
        __syncwarp();
        if (lane == 0) {
            int none = 0;
            if (!ptx::mbar_wait_bounded(&hd.mma_drain, 0, &none, WAIT_NS))
                report_timeout(a.status);
        }
        __syncwarp();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, 512);
    }
}

// ---------------------------------------------------------------------------
// Expansion of the f16 tiles into the workspace, once per call: one CTA per
// (key tile, KV head, layer) copies the tile's raw rows in, dequantizes them with
// the same unit routines as the dequant warps (so the tiles are bit-identical),
// and stores the 48 KB image of the three slots (K^hi, K^lo, V^, 128-byte
// swizzle) with one bulk copy.  The prefill kernel then bulk-copies each tile
// straight into its slots: every row tile of a KV head reads the same keys, and
// this turns 96 dequantizations of a key tile (prefill262k) into one.
constexpr int EXP_THREADS = N_DEQ * 32;  // one K unit and one V unit per thread
constexpr int EXP_SMEM = TILE3 + RAW_BYTES + 16 + 1024;

__global__ void __launch_bounds__(EXP_THREADS) prefill_expand_kernel(const PrefillArgs a,
                                                                     int tiles_total)
{
    extern __shared__ __align__(1024) uint8_t ex_raw_sm[];
    uint8_t *smem = ex_raw_sm + ((1024u - (ptx::smem_u32(ex_raw_sm) & 1023u)) & 1023u);
    uint8_t *kh = smem, *kl = smem + TILE_H, *vh = smem + 2 * TILE_H;
    uint8_t *rk = smem + TILE3, *rv = rk + RAW_K;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + TILE3 + RAW_BYTES);
    __shared__ int ok_s;
    const int t = blockIdx.x;
    const int slab = blockIdx.y + blockIdx.z * gridDim.y;  // as in prefill_tc_kernel
    const int pair = a.pair0 + slab;
    const int h = pair % a.n_kv_heads, layer = pair / a.n_kv_heads;
    const int64_t n_keys = a.n_cached + a.T;
    const int rows = (int)min((int64_t)BN, n_keys - (int64_t)t * BN);
    const int64_t cap = a.layers.cap[layer];
    if (threadIdx.x == 0 && a.test_timeout && t == 0 && pair == 0) {
        // test hook: a bounded wait on a barrier that nothing completes, before any copy
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
        int none = 0;
        if (!ptx::mbar_wait_bounded(bar, 0, &none, WAIT_NS))
            report_timeout(a.status);
        ok_s = 0;
    }
    if (a.test_timeout && t == 0 && pair == 0) {
        __syncthreads();
        return;
    }
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
        ptx::mbar_arrive_expect_tx(bar, rows * (KROW + VROW));
        ptx::bulk_g2s(rk, a.layers.k[layer] + ((int64_t)h * cap + (int64_t)t * BN) * KROW,
                      rows * KROW, bar);
        ptx::bulk_g2s(rv, a.layers.v[layer] + ((int64_t)h * cap + (int64_t)t * BN) * VROW,
                      rows * VROW, bar);
        int none = 0;
        ok_s = ptx::mbar_wait_bounded(bar, 0, &none, WAIT_NS) ? 1 : 0;
        if (!ok_s)
            report_timeout(a.status);
    }
    __syncthreads();
    if (!ok_s)
        return;  // the copy timed out (recorded); it was waited for as long as allowed
    const int grp = threadIdx.x >> 5, ln = threadIdx.x & 31;
    const int r = (grp % (BN / 8)) * 8 + (ln & 7), bk = grp / (BN / 8) + 2 * (ln >> 3);
    uint32_t off[4];
#pragma unroll
    for (int m4 = 0; m4 < 4; ++m4)
        off[m4] = sw_off(r, 32 * bk + 8 * m4);
    dequant_k_unit(rk, r, bk, r < rows, off, kh, kl);
    dequant_v_unit(rv, r, bk, r < rows, off, vh);
    ptx::fence_proxy_async_smem();  // generic-proxy writes -> the bulk store reads them
    __syncthreads();
    if (threadIdx.x == 0) {
        uint8_t *dst = static_cast<uint8_t *>(a.workspace) +
                       ((int64_t)slab * tiles_total + t) * TILE3;
        ptx::bulk_s2g(dst, smem, TILE3);
        ptx::bulk_commit();
        ptx::bulk_wait_read0();  // the shared memory stays valid until it has been read
    }
}

// ---------------------------------------------------------------------------
// Exact path for short visible ranges: one CTA per (token block, KV head,
// layer); rows (t, g) of TB tokens; keys in tiles of 64 with an online
// softmax in fp32; per-block K scale applied to each block's fp32 dot product.
constexpr int EX_THREADS = 256, EX_TILE = 64;

template <int KT, int VT>
__global__ void __launch_bounds__(EX_THREADS) prefill_exact_kernel(const PrefillArgs a, int tb_tok,
                                                                   int t_end)
{
    extern __shared__ float ex_sm[];
    const int G = a.n_q_heads / a.n_kv_heads;
    constexpr int KE = block_elems(KT), VE = block_elems(VT);  // elements per block
    const int D = a.head_dim, nb = D / KE;
    const int t0 = blockIdx.x * tb_tok;
    const int ntok = min(tb_tok, t_end - t0);
    const int R = ntok * G;
    const int h = blockIdx.y, layer = blockIdx.z;
    float *q_s = ex_sm;                 // [R][D]
    float *acc = q_s + R * D;           // [R][D]
    float *p_s = acc + R * D;           // [R][TILE]
    float *m_s = p_s + R * EX_TILE;
    float *l_s = m_s + R;
    float *al_s = l_s + R;
    const int64_t krow = row_bytes(KT, D), vrow = row_bytes(VT, D);
    const uint8_t *kb = a.layers.k[layer] + (int64_t)h * a.layers.cap[layer] * krow;
    const uint8_t *vb = a.layers.v[layer] + (int64_t)h * a.layers.cap[layer] * vrow;
    for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
        const int r = p / D, i = p % D;
        const int t = t0 + r / G, g = r % G;
        q_s[p] = __half2float(a.q[(((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g) * D + i]);
        acc[p] = 0.0f;
    }
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        m_s[r] = -INFINITY;
        l_s[r] = 0.0f;
    }
    __syncthreads();
    const int64_t kend = a.n_cached + t0 + ntok;  // keys the last token sees
    const bool PG = a.page_out != nullptr;  // per-page partials (see prefill_tc_kernel)
    const int n_pages = (int)((a.n_cached + a.T + a.page - 1) / a.page);
    // the partial of page pg of every row: out = acc / l, lse = m + ln l (0, -inf if
    // the row saw nothing of it)
    auto write_page = [&](int pg) {
        for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
            const int r = p / D, i = p % D;
            const int t = t0 + r / G, g = r % G;
            const int64_t row = ((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g;
            const float l = l_s[r];
            a.page_out[(row * n_pages + pg) * D + i] = (l > 0.0f) ? acc[p] / l : 0.0f;
            if (i == 0)
                a.page_lse[row * n_pages + pg] = (l > 0.0f) ? m_s[r] + logf(l) : -INFINITY;
        }
    };
    for (int64_t j0 = 0; j0 < kend; j0 += EX_TILE) {
        if (PG && j0 > 0 && j0 % a.page == 0) {
            // page boundary: write the previous page, restart the (max, sum, acc)
            write_page((int)(j0 / a.page) - 1);
            __syncthreads();
            for (int p = threadIdx.x; p < R * D; p += blockDim.x)
                acc[p] = 0.0f;
            for (int r = threadIdx.x; r < R; r += blockDim.x) {
                m_s[r] = -INFINITY;
                l_s[r] = 0.0f;
            }
            __syncthreads();
        }
        for (int p = threadIdx.x; p < R * EX_TILE; p += blockDim.x) {
            const int r = p / EX_TILE, jj = p % EX_TILE;
            const int64_t j = j0 + jj;
            const int t = t0 + r / G;
            float s = -INFINITY;
            if (j <= a.n_cached + t) {
                const uint8_t *kr = kb + j * krow;
                const float *qr = q_s + r * D;
                float tot = 0.0f;
                for (int bq = 0; bq < nb; ++bq) {
                    const uint8_t *blk = kr + bq * block_bytes(KT);
                    float part = 0.0f, qsum = 0.0f;
                    for (int i = 0; i < KE; ++i) {
                        part += qr[bq * KE + i] * (float)block_int<KT>(blk, i);
                        if (KT == KVQ_TYPE_OSCAR2)
                            qsum += qr[bq * KE + i];
                    }
                    tot += block_d(blk) * part;
                    if (KT == KVQ_TYPE_OSCAR2)  // q . (d u + m) = d (q . u) + m sum(q)
                        tot += block_m<KT>(blk) * qsum;
                }
                s = a.scale * tot;
            }
            p_s[p] = s;
        }
        __syncthreads();
        for (int r = threadIdx.x; r < R; r += blockDim.x) {
            float mt = -INFINITY;
            for (int jj = 0; jj < EX_TILE; ++jj)
                mt = fmaxf(mt, p_s[r * EX_TILE + jj]);
            const float m_old = m_s[r], m_new = fmaxf(m_old, mt);
            float alpha = 1.0f, sum = 0.0f;
            if (m_new != -INFINITY) {
                alpha = (m_old == -INFINITY) ? 0.0f : expf(m_old - m_new);
                for (int jj = 0; jj < EX_TILE; ++jj) {
                    const float s = p_s[r * EX_TILE + jj];
                    const float pw = (s == -INFINITY) ? 0.0f : expf(s - m_new);
                    p_s[r * EX_TILE + jj] = pw;
                    sum += pw;
                }
            } else {
                for (int jj = 0; jj < EX_TILE; ++jj)
                    p_s[r * EX_TILE + jj] = 0.0f;
            }
            l_s[r] = l_s[r] * alpha + sum;
            m_s[r] = m_new;
            al_s[r] = alpha;
        }
        __syncthreads();
        for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
            const int r = p / D, i = p % D;
            const int bq = i / VE, ii = i % VE;
            float o = acc[p] * al_s[r];
            for (int jj = 0; jj < EX_TILE; ++jj) {
                const float pw = p_s[r * EX_TILE + jj];
                if (pw == 0.0f)
                    continue;
                const uint8_t *blk = vb + (j0 + jj) * vrow + bq * block_bytes(VT);
                o += pw * (block_d(blk) * (float)block_int<VT>(blk, ii) + block_m<VT>(blk));
            }
            acc[p] = o;
        }
        __syncthreads();
    }
    if (PG) {
        const int pl = (int)((kend - 1) / a.page);  // the page of the last key read
        write_page(pl);
        // pages past the keys of this block: nothing visible
        for (int pg = pl + 1; pg < n_pages; ++pg)
            for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
                const int r = p / D, i = p % D;
                const int t = t0 + r / G, g = r % G;
                const int64_t row = ((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g;
                a.page_out[(row * n_pages + pg) * D + i] = 0.0f;
                if (i == 0)
                    a.page_lse[row * n_pages + pg] = -INFINITY;
            }
        return;
    }
    for (int p = threadIdx.x; p < R * D; p += blockDim.x) {
        const int r = p / D, i = p % D;
        const int t = t0 + r / G, g = r % G;
        const int64_t row = ((int64_t)layer * a.T + t) * a.n_q_heads + h * G + g;
        const float l = l_s[r];
        a.out[row * D + i] = (l > 0.0f) ? acc[p] / l : 0.0f;
        if (i == 0)
            a.lse[row] = (l > 0.0f) ? m_s[r] + logf(l) : -INFINITY;
    }
}

}  // namespace

size_t prefill_workspace_bytes(int, int, int, int, int) { return 0; }

size_t prefill_expand_bytes(int n_layers, int n_kv_heads, int head_dim, int64_t n_keys)
{
    if (head_dim != HD || n_layers < 1 || n_kv_heads < 1 || n_keys < 1)
        return 0;
    return (size_t)n_layers * n_kv_heads * (size_t)((n_keys + BN - 1) / BN) * TILE3;
}

size_t prefill_slab_bytes(int head_dim, int64_t n_keys)
{
    return prefill_expand_bytes(1, 1, head_dim, n_keys);
}

bool prefill_supported(int n_q_heads, int n_kv_heads, int head_dim)
{
    const int G = n_q_heads / n_kv_heads;
    return G >= 1 && G <= 32 && head_dim >= 32 && head_dim <= 512 && head_dim % 32 == 0;
}

namespace {

// A second stream and two events per device for the double-buffered expansion;
// the mutex keeps one call's fork and join (which reuse the events) together.
struct ForkStream {
    std::mutex mu;
    cudaStream_t s2 = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
ForkStream g_fork[MAX_DEVICES];

template <int KT, int VT>
void launch_exact(const PrefillArgs &a, dim3 grid, size_t smem, int tb, int t_end, cudaStream_t s)
{
    static std::atomic<int> smem_ex[MAX_DEVICES];
    ensure_smem(reinterpret_cast<const void *>(prefill_exact_kernel<KT, VT>), smem_ex, (int)smem);
    prefill_exact_kernel<KT, VT><<<grid, EX_THREADS, smem, s>>>(a, tb, t_end);
}

// Expansion and tensor-core attention of the pairs [p0, p0 + np) with their key
// tiles at `ws` (np slabs).
void expand_and_attend(PrefillArgs a, int p0, int np, void *ws, int tiles_total, int row0,
                       int rows, cudaStream_t s)
{
    a.pair0 = p0;
    a.workspace = ws;
    dim3 egrid((unsigned)tiles_total, (unsigned)np, 1);
    dim3 grid((unsigned)((rows + BM - 1) / BM), (unsigned)np, 1);
    prefill_expand_kernel<<<egrid, EXP_THREADS, EXP_SMEM, s>>>(a, tiles_total);
    prefill_tc_kernel<true><<<grid, pf_threads<true>(), pf_smem<true>(), s>>>(a, row0);
}

}  // namespace

bool launch_prefill(const PrefillArgs &a_in, cudaStream_t s)
{
    PrefillArgs a = a_in;
    a.pair0 = 0;
    const int G = a.n_q_heads / a.n_kv_heads;
    // tokens whose rows see fewer than PF_MIN_KEYS keys take the exact kernel; so do
    // all rows when per-page partials are asked for (a page is a short context, where
    // the tensor-core path's f16 rounding of V^ and P is not within the tolerance)
    int64_t t_split = PF_MIN_KEYS - 1 - a.n_cached;
    t_split = t_split < 0 ? 0 : (t_split > a.T ? a.T : t_split);
    if (a.page_out)
        t_split = a.T;
    // the tensor-core path is built for head_dim 256 and Q8_0 K / Q4_0 V
    if (a.head_dim != HD || a.k_type != KVQ_TYPE_Q8_0 || a.v_type != KVQ_TYPE_Q4_0)
        t_split = a.T;
    if (t_split > 0) {
        const int tb = max(1, 32 / G);
        const size_t smem = sizeof(float) * ((size_t)2 * tb * G * a.head_dim +
                                             (size_t)tb * G * EX_TILE + 3 * (size_t)tb * G);
        dim3 grid((unsigned)((t_split + tb - 1) / tb), a.n_kv_heads, a.n_layers);
        launch_for_types(a.k_type, a.v_type, [&](auto kt, auto vt) {
            launch_exact<decltype(kt)::value, decltype(vt)::value>(a, grid, smem, tb,
                                                                   (int)t_split, s);
            return true;
        });
    }
    if (t_split == a.T)
        return true;
    const bool pre = a.workspace != nullptr;
    static std::atomic<int> smem_tc[2][MAX_DEVICES], smem_exp[MAX_DEVICES];
    if (pre) {
        ensure_smem(reinterpret_cast<const void *>(prefill_tc_kernel<true>), smem_tc[1],
                    pf_smem<true>());
        ensure_smem(reinterpret_cast<const void *>(prefill_expand_kernel), smem_exp, EXP_SMEM);
    } else {
        ensure_smem(reinterpret_cast<const void *>(prefill_tc_kernel<false>), smem_tc[0],
                    pf_smem<false>());
    }
    const int row0 = (int)t_split * G;
    const int rows = a.T * G - row0;
    if (!pre) {
        dim3 grid((unsigned)((rows + BM - 1) / BM), a.n_kv_heads, a.n_layers);
        prefill_tc_kernel<false><<<grid, pf_threads<false>(), pf_smem<false>(), s>>>(a, row0);
        return true;
    }
    // With a workspace (the caller checked that it holds at least one slab): every
    // (layer, KV head) pair's key tiles are expanded once into a slab of it, then read
    // by all row tiles of the pair.  If every pair has a slab, one expansion and one
    // attention launch cover the call.  Otherwise the pairs go in chunks through two
    // halves of the workspace, alternating between the caller's stream and a second
    // one, so that a chunk's expansion and the start of its attention overlap the end
    // of the previous chunk's attention.
    const int tiles_total = (int)((a.n_cached + a.T + BN - 1) / BN);
    const size_t slab = (size_t)tiles_total * TILE3;
    const int pairs = a.n_layers * a.n_kv_heads;
    const int64_t slots = (int64_t)(a.ws_bytes / slab);
    if (slots >= pairs) {
        dim3 egrid((unsigned)tiles_total, a.n_kv_heads, a.n_layers);
        dim3 grid((unsigned)((rows + BM - 1) / BM), a.n_kv_heads, a.n_layers);
        prefill_expand_kernel<<<egrid, EXP_THREADS, EXP_SMEM, s>>>(a, tiles_total);
        prefill_tc_kernel<true><<<grid, pf_threads<true>(), pf_smem<true>(), s>>>(a, row0);
        return true;
    }
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES)
        return false;
    ForkStream &f = g_fork[dev];
    std::lock_guard<std::mutex> lock(f.mu);
    if (slots >= 2 && !f.s2) {
        if (cudaStreamCreateWithFlags(&f.s2, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&f.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&f.join, cudaEventDisableTiming) != cudaSuccess)
            return false;
    }
    if (slots < 2) {  // one slab: the pairs one at a time on the caller's stream
        for (int p = 0; p < pairs; ++p)
            expand_and_attend(a, p, 1, ws, tiles_total, row0, rows, s);
        return true;
    }
    const int chunk = (int)(slots / 2);
    if (cudaEventRecord(f.fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(f.s2, f.fork, 0) != cudaSuccess)
        return false;
    for (int p0 = 0, i = 0; p0 < pairs; p0 += chunk, ++i) {
        const int np = min(chunk, pairs - p0);
        expand_and_attend(a, p0, np, ws + (size_t)(i & 1) * chunk * slab, tiles_total, row0,
                          rows, (i & 1) ? f.s2 : s);
    }
    return cudaEventRecord(f.join, f.s2) == cudaSuccess &&
           cudaStreamWaitEvent(s, f.join, 0) == cudaSuccess;
}

}  // namespace kvq
