// decode.cu -- split-KV GQA decode attention over the Q8_0/Q4_0 cache,
// tiled for sm_100a, and the dispatch between it and the general kernel.
//
// What it computes (speculative-decoding paragraph of the RX 9070 XT
// KV-streaming page: paged decode attention over a verify batch; "Known
// Issues Fixed" of the OSCAR2 page: the softmax max covers complete scores;
// GQA section of the KV-cache guide): for every (layer, KV head h, chunk c of
// `chunk` keys) and every row r = t*G + g (query head h*G + g of token t),
// s_j = scale * sum_b d_b * sum_i q_i k_ij over the keys j of the chunk with
// j <= n_kv - T + t, and the chunk partial o = sum_j p_j v^_j / l,
// lse = m + ln l.
//
// Layout of the work (head_dim 256, up to 24 rows = G*T):
//  * one CTA per (layer, KV head, chunk) of NPAIR warp pairs (8 for up to 8
//    rows, 6 for up to 16: PairCfg); thread 0 also
//    issues the copies: a prologue of NS stages, then each stage's slot is
//    refilled as soon as every warp has released it;
//  * the chunk streams in stages of 16*NPAIR tokens -- that many K head-rows
//    (272 B each) and V head-rows (144 B each), each one contiguous 16-byte-
//    aligned range of the head-major cache -- with cp.async.bulk into a ring
//    of NS shared-memory stages, completion tracked by mbarriers;
//  * pair p owns tokens [16p, 16p+16) of every stage; warp 2p+hf of the pair
//    owns head_dim half hf (Q8_0/Q4_0 blocks 4hf..4hf+3) of both contractions;
//  * S^T = K Q^T on mma.sync m16n8k16 (rows = 16 tokens, columns = 8 query
//    rows).  The contraction index is permuted inside each 16-dim step so
//    that a thread's four K bytes are contiguous (one 32-bit shared load for
//    odd blocks, which start 4-byte aligned); Q's B-fragments live in shared
//    memory in the same order.  int8 K converts to f16 exactly, q is f16, each
//    32-element block's product is accumulated in fp32 and scaled by its fp32
//    d_b (times scale*log2 e): only fp32 rounding separates S from exact.  The
//    two halves' partial S are exchanged through shared memory;
//  * online softmax per query row in base 2 with a lazy running max: it moves
//    (exactly, with the rescale of O and l) only when a score exceeds it by
//    more than TAU = 8, so p <= 2^8 -- harmless in fp32 and f16 -- and the
//    cross-lane max and the rescale are almost never executed after the
//    first tile.  The max then covers complete scores;
//  * O^T += V^T P^T on mma.sync (rows = 16 head dims, columns = 8 query
//    rows): Q4_0 nibbles become (u - 8) in f16 exactly; P is split into two
//    f16 parts (P_hi + P_lo, ~2^-22 relative) that reach the B-operand layout
//    with movmatrix.trans, and the token's fp16 d_v enters through an exact
//    two-part product (hi = RN(P_hi d), lo = fma(P_hi, d, -hi) + P_lo d), so
//    each block costs two MMAs per tile but the PV side carries no fp16
//    rounding of P: a single fp16 rounding of a dominant weight would cost
//    up to |v^| * 2^-11, about 1.5e-2 on the x8 outlier channels;
//  * at the end the pairs' (m, l, O) merge through shared memory and the
//    chunk partial (out, lse) is written.
// Every mbarrier wait is bounded (about one second of wall time); a wait that
// runs out sets the device status word and the CTA falls through without
// hanging, after waiting (bounded) for its own copies in flight.
#include "common.cuh"
#include "merge.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "decode_frag.cuh"

namespace kvq {

bool launch_decode_simple(const DecodeArgs &a, cudaStream_t s);
bool launch_decode_split(const DecodeArgs &a, cudaStream_t s);
bool launch_decode_tmem(const DecodeArgs &a, cudaStream_t s);

namespace {

using namespace frag;

constexpr int KROW = 272, VROW = 144;         // head-row bytes at head_dim 256
// Launch shape per number of n-tiles of rows: with one n-tile (up to 8 rows) a
// warp's O^T takes 32 registers, so 8 warp pairs fit the register file (and a
// 3-stage ring of 128-token stages the shared memory); with two, 6 pairs and a
// 4-stage ring of 96-token stages.
template <int NT>
struct PairCfg {
    static constexpr int NPAIR = NT == 1 ? 8 : 6;  // warp pairs per CTA
    static constexpr int WARPS = 2 * NPAIR;
    static constexpr int THREADS = 32 * WARPS;
    static constexpr int TOK = 16 * NPAIR;         // tokens per stage
    static constexpr int NS = NT == 1 ? 3 : 4;     // stages in the ring
    static constexpr int STAGE_K = TOK * KROW;
    static constexpr int STAGE_V = TOK * VROW;
    static constexpr int STAGE_BYTES = STAGE_K + STAGE_V;
};
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float TAU = 8.0f;                   // lazy-max slack (log2 units)
constexpr float M_INIT = -1.0e30f;            // "no score yet", finite: ex2(s - M_INIT) stays defined

template <int NT>
struct __align__(16) DecodeSmem {
    using C = PairCfg<NT>;
    uint8_t ring[C::NS][C::STAGE_BYTES];
    float4 xs[C::NPAIR][2][2][NT][32];  // partial S exchange [pair][parity][half][n-tile][lane]
    uint2 qf[2][8][NT][32];             // Q^T B-fragments [half][k-step][n-tile][lane]
    float pm[C::NPAIR][32], pl[C::NPAIR][32];
    float red[C::NPAIR][2];  // fused step: per-group reduction slots of the merge
    uint64_t full[C::NS], empty[C::NS], never;
    int abort;
    int last;             // fused step: this CTA is the last of its (layer, KV head)
};

template <int NT, bool FUSED>
__global__ void __launch_bounds__(PairCfg<NT>::THREADS, 1) decode_tc_kernel(const DecodeArgs a)
{
    using Cfg = PairCfg<NT>;
    constexpr int NPAIR = Cfg::NPAIR, WARPS = Cfg::WARPS, THREADS = Cfg::THREADS, TOK = Cfg::TOK,
                  NS = Cfg::NS, STAGE_K = Cfg::STAGE_K, STAGE_V = Cfg::STAGE_V,
                  STAGE_BYTES = Cfg::STAGE_BYTES;
    // fused step: chunks whose merge weights fit in the ring, per 64-thread group
    constexpr int FUSED_SMEM_CHUNKS = (int)(NS * STAGE_BYTES / (NPAIR * sizeof(float)));
    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecodeSmem<NT> &sm = *reinterpret_cast<DecodeSmem<NT> *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.n_q_heads / a.n_kv_heads;
    const int R = G * a.T;  // live query rows (<= NT*8)
    const int C = (int)((a.n_kv + a.chunk - 1) / a.chunk);
    const int c = blockIdx.x % C;
    const int h = (blockIdx.x / C) % a.n_kv_heads;
    const int layer = blockIdx.x / (C * a.n_kv_heads);
    const int64_t c0 = (int64_t)c * a.chunk;
    const int n_tok = (int)((c0 + a.chunk < a.n_kv ? c0 + a.chunk : a.n_kv) - c0);
    const int n_stages = (n_tok + TOK - 1) / TOK;
    const int64_t cap = a.layers.cap[layer];
    const uint8_t *kg = a.layers.k[layer] + ((int64_t)h * cap + c0) * KROW;
    const uint8_t *vg = a.layers.v[layer] + ((int64_t)h * cap + c0) * VROW;

    // one stage's K and V rows into its ring slot (one thread; the slot is free)
    auto copy_stage = [&](int st) {
        const int slot = st % NS;
        const int rows = min(TOK, n_tok - st * TOK);
        ptx::mbar_arrive_expect_tx(&sm.full[slot], rows * (KROW + VROW));
        ptx::bulk_g2s(sm.ring[slot], kg + (int64_t)st * STAGE_K, rows * KROW, &sm.full[slot]);
        ptx::bulk_g2s(sm.ring[slot] + STAGE_K, vg + (int64_t)st * STAGE_V, rows * VROW,
                      &sm.full[slot]);
    };
    // unless this chunk holds rows that the fused step appends first, the first stages
    // are requested before anything else, so that their latency overlaps the set-up
    const bool appends_here = FUSED && c0 + n_tok > a.n_kv - a.T;
    const int early = appends_here ? 0 : min(NS, n_stages);
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            ptx::mbar_init(&sm.full[i], 1);
            ptx::mbar_init(&sm.empty[i], WARPS);
        }
        ptx::mbar_init(&sm.never, 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
        for (int st = 0; st < early; ++st)
            copy_stage(st);
    }
    // Q^T B-fragments: entry (hf, ks, nt, lane) holds q[row nt*8 + lane/4] dims
    // 128 hf + 16 ks + 4 (lane%4) .. +3 (the permuted k order; zero for padded rows)
    {
        const __half *qbase = a.q + (int64_t)layer * a.T * a.n_q_heads * 256;
        for (int e = threadIdx.x; e < 2 * 8 * NT * 32; e += THREADS) {
            const int ln = e & 31, nt = (e >> 5) % NT, ks = (e / (32 * NT)) & 7;
            const int hf2 = e / (32 * NT * 8);
            const int r = nt * 8 + (ln >> 2);
            uint2 v = make_uint2(0u, 0u);
            if (r < R) {
                const int t = r / G, gq = r % G;
                v = *reinterpret_cast<const uint2 *>(
                    qbase + ((int64_t)t * a.n_q_heads + h * G + gq) * 256 + hf2 * 128 + ks * 16 +
                    4 * (ln & 3));
            }
            sm.qf[hf2][ks][nt][ln] = v;
        }
    }
    if (FUSED) {
        // append: the new rows [n_kv - T, n_kv) that fall in this chunk are quantized here,
        // before any copy of the chunk is issued (no other CTA reads them); one warp
        // per 32-element block, K blocks 0..7 then V blocks 0..7 of each row
        const int64_t j_lo = max(c0, a.n_kv - a.T), j_hi = c0 + n_tok;
        const int tasks = j_hi > j_lo ? (int)(j_hi - j_lo) * 16 : 0;
        uint8_t *kw = const_cast<uint8_t *>(a.layers.k[layer]);
        uint8_t *vw = const_cast<uint8_t *>(a.layers.v[layer]);
        for (int task = threadIdx.x >> 5; task < tasks; task += WARPS) {
            const int64_t j = j_lo + task / 16;
            const int blk = task % 16, b = blk & 7;
            const int tok = (int)(j - (a.n_kv - a.T));
            const int64_t src = (((int64_t)layer * a.T + tok) * a.n_kv_heads + h) * 256 + b * QK +
                                (threadIdx.x & 31);
            const int64_t row = (int64_t)h * cap + j;
            if (blk < 8)
                warp_quant_q8_0(a.k_new[src], kw + row * KROW + b * Q8_0_BYTES, threadIdx.x & 31);
            else
                warp_quant_q4_0(a.v_new[src], vw + row * VROW + b * Q4_0_BYTES, threadIdx.x & 31);
        }
        // the blocks just written are read next by bulk copies (the async proxy)
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncthreads();
    volatile int *abort = &sm.abort;

    const int g = lane >> 2, cq = lane & 3;
    const int pair = warp >> 1, hf = warp & 1;
    float o[8][NT][4];  // O^T of this warp's 128 dims (8 m-tiles) x NT n-tiles
    float m2[NT][2], l2[NT][2];

    // ---------------------------------------------------------------- copies
    // thread 0 issues stage st into slot st % NS once the slot's consumers
    // released it (empty) and its previous copy landed (full); false on timeout
    auto issue = [&](int st) -> bool {
        const int slot = st % NS;
        const uint32_t round = st / NS;
        if (st >= NS &&
            (!ptx::mbar_wait_bounded(&sm.empty[slot], (round - 1) & 1, abort, WAIT_LIMIT_NS) ||
             !ptx::mbar_wait_bounded(&sm.full[slot], (round - 1) & 1, abort, WAIT_LIMIT_NS)))
            return false;
        copy_stage(st);
        return true;
    };
    int issued = threadIdx.x == 0 ? early : 0;
    if (threadIdx.x == 0)
        for (; issued < NS && issued < n_stages; ++issued)
            issue(issued);

    const float dscale = a.scale * LOG2E;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                o[mt][nt][i] = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            m2[nt][k] = M_INIT;
            l2[nt][k] = 0.0f;
        }
    if (a.test_timeout && lane == 0) {
        // test hook: wait on a barrier that nothing completes
        if (!ptx::mbar_wait_bounded(&sm.never, 0, abort, WAIT_LIMIT_NS)) {
            *abort = 1;
            report_timeout(a.status);
        }
    }
    __syncwarp();

    int par = 0;
    bool aborted = false;
    for (int s = 0; s < n_stages; ++s) {
        const int slot = s % NS;
        if (!aborted) {
            bool ok = true;
            if (lane == 0)
                ok = ptx::mbar_wait_bounded(&sm.full[slot], (s / NS) & 1, abort, WAIT_LIMIT_NS);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                if (lane == 0 && !*abort) {
                    *abort = 1;
                    report_timeout(a.status);
                }
                aborted = true;
            }
        }
        const int valid = min(16, n_tok - s * TOK - 16 * pair);  // tokens of this pair's tile
        // both warps of a pair see the same `valid`, so both take the exchange barrier
        if (valid > 0) {
            const uint8_t *ks = sm.ring[slot] + (16 * pair) * KROW;
            const uint8_t *vs = sm.ring[slot] + STAGE_K + (16 * pair) * VROW;
            const int j0 = s * TOK + 16 * pair;  // key of token 0, relative to c0
            float sacc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    sacc[nt][i] = 0.0f;
            if (!aborted) {
                // ---- S^T partial over this warp's 4 blocks, exact per-block scale
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    const int b = 4 * hf + bb;  // parity of b is the parity of bb
                    const uint8_t *r0 = ks + g * KROW + 34 * b;
                    const uint8_t *r1 = r0 + 8 * KROW;
                    const float dk0 = __half2float(__ushort_as_half((unsigned short)lds16(r0))) * dscale;
                    const float dk1 = __half2float(__ushort_as_half((unsigned short)lds16(r1))) * dscale;
                    float blk[NT][4];
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        const int off = 2 + 16 * s2 + 4 * cq;
                        uint32_t af[4];
                        s8x4_to_h2x2(k_word(r0 + off, (bb & 1) != 0), af[0], af[2]);
                        s8x4_to_h2x2(k_word(r1 + off, (bb & 1) != 0), af[1], af[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint2 qb = sm.qf[hf][2 * bb + s2][nt][lane];
                            if (s2 == 0) {
                                const float z[4] = {0.f, 0.f, 0.f, 0.f};
                                ptx::mma_f16_16816(blk[nt], af, qb.x, qb.y, z);
                            } else {
                                ptx::mma_f16_16816(blk[nt], af, qb.x, qb.y, blk[nt]);
                            }
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        sacc[nt][0] = fmaf(dk0, blk[nt][0], sacc[nt][0]);
                        sacc[nt][1] = fmaf(dk0, blk[nt][1], sacc[nt][1]);
                        sacc[nt][2] = fmaf(dk1, blk[nt][2], sacc[nt][2]);
                        sacc[nt][3] = fmaf(dk1, blk[nt][3], sacc[nt][3]);
                    }
                }
            }
            // ---- exchange partial S with the other half of the pair
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                sm.xs[pair][par][hf][nt][lane] =
                    make_float4(sacc[nt][0], sacc[nt][1], sacc[nt][2], sacc[nt][3]);
            ptx::named_bar_sync(1 + pair, 64);
            float sv[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float4 x = sm.xs[pair][par][hf ^ 1][nt][lane];
                sv[nt][0] = sacc[nt][0] + x.x;
                sv[nt][1] = sacc[nt][1] + x.y;
                sv[nt][2] = sacc[nt][2] + x.z;
                sv[nt][3] = sacc[nt][3] + x.w;
            }
            par ^= 1;

            if (!aborted) {
                // ---- mask (ragged tail of the chunk, causal rows of the verify batch,
                //      padded rows)
                const bool need_mask = valid < 16 || c0 + j0 + 15 > a.n_kv - a.T;
                if (need_mask) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int tt = g + 8 * (i >> 1);
                            const int r = nt * 8 + 2 * cq + (i & 1);
                            const bool vis = tt < valid && r < R &&
                                             c0 + j0 + tt <= a.n_kv - a.T + r / G;
                            if (!vis)
                                sv[nt][i] = -INFINITY;
                        }
                }
                // ---- online softmax (base 2), lazy running max
                float tmax[NT][2];
                bool up = false;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        tmax[nt][k] = fmaxf(sv[nt][k], sv[nt][2 + k]);
                        up |= tmax[nt][k] > m2[nt][k] + TAU;
                    }
                if (__any_sync(0xffffffffu, up)) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            float v = tmax[nt][k];
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                            const float mn = fmaxf(m2[nt][k], v);
                            const float al = ptx::ex2(m2[nt][k] - mn);
                            m2[nt][k] = mn;
                            l2[nt][k] *= al;
#pragma unroll
                            for (int mt = 0; mt < 8; ++mt) {
                                o[mt][nt][k] *= al;
                                o[mt][nt][2 + k] *= al;
                            }
                        }
                }
                // P = P_hi + P_lo (two f16 parts, residual ~2^-22 relative), moved to the
                // B-operand layout (tokens along k) with movmatrix.trans
                uint32_t ph[NT][2], pl[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float p[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        p[i] = ptx::ex2(sv[nt][i] - m2[nt][i & 1]);
                    l2[nt][0] += p[0] + p[2];
                    l2[nt][1] += p[1] + p[3];
                    const __half2 h01 = __floats2half2_rn(p[0], p[1]);
                    const __half2 h23 = __floats2half2_rn(p[2], p[3]);
                    const __half2 r01 = __floats2half2_rn(p[0] - __low2float(h01),
                                                          p[1] - __high2float(h01));
                    const __half2 r23 = __floats2half2_rn(p[2] - __low2float(h23),
                                                          p[3] - __high2float(h23));
                    ph[nt][0] = ptx::movmatrix_trans(ptx::h2_bits(h01));
                    ph[nt][1] = ptx::movmatrix_trans(ptx::h2_bits(h23));
                    pl[nt][0] = ptx::movmatrix_trans(ptx::h2_bits(r01));
                    pl[nt][1] = ptx::movmatrix_trans(ptx::h2_bits(r23));
                }
                // ---- O^T += V^T (P d_v)^T over this warp's 4 blocks
                const uint8_t *v0 = vs + (2 * cq) * VROW;  // tokens 2c, 2c+1, 2c+8, 2c+9
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) {
                    const int b = 4 * hf + bb;
                    const uint8_t *vb = v0 + 18 * b;
                    uint32_t d0 = lds16(vb), d1 = lds16(vb + VROW);
                    uint32_t d2 = lds16(vb + 8 * VROW), d3 = lds16(vb + 9 * VROW);
                    if (valid < 16) {  // tokens past the chunk end may hold stale bytes
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
                    const uint32_t wA0 = ptx::prmt(x0, x1, 0x0400);  // byte 2g of tokens 2c, 2c+1
                    const uint32_t wA1 = ptx::prmt(x0, x1, 0x0501);  // byte 2g+1
                    const uint32_t wB0 = ptx::prmt(x2, x3, 0x0400);  // tokens 2c+8, 2c+9
                    const uint32_t wB1 = ptx::prmt(x2, x3, 0x0501);
                    const uint32_t alo[4] = {nib_lo(wA0), nib_lo(wA1), nib_lo(wB0), nib_lo(wB1)};
                    const uint32_t ahi[4] = {nib_hi(wA0), nib_hi(wA1), nib_hi(wB0), nib_hi(wB1)};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        // P d_v as hi + lo without loss: hi = RN(P_hi d), the exact
                        // product error fma(P_hi, d, -hi), plus P_lo d
                        uint32_t bh[2], bl[2];
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            const __half2 d = k == 0 ? dA : dB;
                            const __half2 a_hi = ptx::bits_h2(ph[nt][k]);
                            const __half2 hi = __hmul2_rn(a_hi, d);
                            const __half2 err = __hfma2(a_hi, d, __hneg2(hi));
                            bh[k] = ptx::h2_bits(hi);
                            bl[k] = ptx::h2_bits(__hfma2(ptx::bits_h2(pl[nt][k]), d, err));
                        }
                        ptx::mma_f16_16816(o[2 * bb][nt], alo, bh[0], bh[1], o[2 * bb][nt]);
                        ptx::mma_f16_16816(o[2 * bb][nt], alo, bl[0], bl[1], o[2 * bb][nt]);
                        ptx::mma_f16_16816(o[2 * bb + 1][nt], ahi, bh[0], bh[1], o[2 * bb + 1][nt]);
                        ptx::mma_f16_16816(o[2 * bb + 1][nt], ahi, bl[0], bl[1], o[2 * bb + 1][nt]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            ptx::mbar_arrive(&sm.empty[slot]);
        if (threadIdx.x == 0 && issued < n_stages && !*abort) {
            if (issue(issued)) {
                ++issued;
            } else if (!*abort) {
                *abort = 1;
                report_timeout(a.status);
            }
        }
    }
    // per-row sums over the 8 lanes that share a column
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            float v = l2[nt][k];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            l2[nt][k] = v;
        }
    if (hf == 0 && g == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                sm.pm[pair][nt * 8 + 2 * cq + k] = m2[nt][k];
                sm.pl[pair][nt * 8 + 2 * cq + k] = l2[nt][k];
            }
    }
    if (threadIdx.x == 0) {
        // drain: every issued copy has landed before the ring is reused or freed
        // (bounded, without the abort short-cut)
        int no_abort = 0;
        for (int st = (issued > NS ? issued - NS : 0); st < issued; ++st)
            if (!ptx::mbar_wait_bounded(&sm.full[st % NS], (st / NS) & 1, &no_abort,
                                        WAIT_LIMIT_NS))
                report_timeout(a.status);
    }
    __syncthreads();  // ring consumed and drained; pair stats visible

    // ---------------------------------------------------------------- merge pairs
    constexpr int NCOL = NT * 8;
    static_assert(sizeof(float) * NPAIR * NCOL * 256 <= sizeof(uint8_t) * NS * STAGE_BYTES,
                  "merge buffer must fit in the ring");
    float *obuf = reinterpret_cast<float *>(sm.ring);  // [NPAIR][NCOL][256]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int col = nt * 8 + 2 * cq + k;
            float M = M_INIT;
#pragma unroll
            for (int p = 0; p < NPAIR; ++p)
                M = fmaxf(M, sm.pm[p][col]);
            float L = 0.0f;
#pragma unroll
            for (int p = 0; p < NPAIR; ++p)
                L += sm.pl[p][col] * ptx::ex2(sm.pm[p][col] - M);
            const float f = (L > 0.0f) ? ptx::ex2(m2[nt][k] - M) / L : 0.0f;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int b = 4 * hf + (mt >> 1);
                const int dbase = 32 * b + ((mt & 1) ? 16 : 0) + 2 * g;
                obuf[(pair * NCOL + col) * 256 + dbase] = o[mt][nt][k] * f;
                obuf[(pair * NCOL + col) * 256 + dbase + 1] = o[mt][nt][2 + k] * f;
            }
        }
    __syncthreads();
    const int Hq = a.n_q_heads;
    for (int idx = threadIdx.x; idx < R * 256; idx += THREADS) {
        const int col = idx >> 8, dim = idx & 255;
        float v = 0.0f;
#pragma unroll
        for (int p = 0; p < NPAIR; ++p)
            v += obuf[(p * NCOL + col) * 256 + dim];
        const int t = col / G, gq = col % G;
        const int64_t row = ((int64_t)layer * a.T + t) * Hq + h * G + gq;
        a.out_part[(row * C + c) * 256 + dim] = v;
    }
    for (int col = threadIdx.x; col < R; col += THREADS) {
        float M = M_INIT;
        for (int p = 0; p < NPAIR; ++p)
            M = fmaxf(M, sm.pm[p][col]);
        float L = 0.0f;
        for (int p = 0; p < NPAIR; ++p)
            L += sm.pl[p][col] * ptx::ex2(sm.pm[p][col] - M);
        const int t = col / G, gq = col % G;
        const int64_t row = ((int64_t)layer * a.T + t) * Hq + h * G + gq;
        a.lse_part[row * C + c] = (L > 0.0f) ? (M + log2f(L)) * LN2 : -INFINITY;
    }
    if (FUSED) {
        // the last CTA of this (layer, KV head) to finish merges the chunk partials of its
        // rows, read through L2.  Release: the barrier orders every thread's partial
        // writes before thread 0's device-scope fence and count; acquire: the last CTA's
        // thread 0 fences after seeing the count, and the barrier passes that on.
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            const bool last =
                atomicAdd(&a.counters[layer * a.n_kv_heads + h], 1u) == (unsigned)(C - 1);
            if (last)
                __threadfence();
            sm.last = last;
        }
        __syncthreads();
        if (sm.last) {
            const int grp = threadIdx.x >> 6, t64 = threadIdx.x & 63;  // group = warp pair
            float *w_s = C <= FUSED_SMEM_CHUNKS ? reinterpret_cast<float *>(sm.ring) + grp * C
                                                : nullptr;
            for (int col = grp; col < R; col += NPAIR) {
                const int t = col / G, gq = col % G;
                const int64_t row = ((int64_t)layer * a.T + t) * Hq + h * G + gq;
                merge_row<true>(a.out_part + row * C * 256, a.lse_part + row * C, C, 256,
                                a.out + row * 256, a.lse + row, w_s, sm.red[grp], t64,
                                [grp] { ptx::named_bar_sync(1 + grp, 64); });
            }
        }
    }
}

template <int NT, bool FUSED>
bool launch_tc(const DecodeArgs &a, cudaStream_t s)
{
    const size_t smem = sizeof(DecodeSmem<NT>);
    static bool attr_set[64] = {};  // the attribute belongs to the function on each device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return false;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(decode_tc_kernel<NT, FUSED>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return false;
        attr_set[dev] = true;
    }
    const int64_t C = (a.n_kv + a.chunk - 1) / a.chunk;
    const int64_t grid = (int64_t)a.n_layers * a.n_kv_heads * C;
    if (grid >= (1ll << 31))
        return false;
    decode_tc_kernel<NT, FUSED><<<(unsigned)grid, PairCfg<NT>::THREADS, smem, s>>>(a);
    return true;
}

}  // namespace

bool decode_tc_supported(const DecodeArgs &a)
{
    const int rows = (a.n_q_heads / a.n_kv_heads) * a.T;
    return a.head_dim == 256 && rows <= 24 && a.k_type == KVQ_TYPE_Q8_0 &&
           a.v_type == KVQ_TYPE_Q4_0;
}

bool launch_decode(const DecodeArgs &a, cudaStream_t s)
{
    if (a.counters) {  // fused step: tiled kernel only
        if (!decode_tc_supported(a))
            return false;
        const int nt = ((a.n_q_heads / a.n_kv_heads) * a.T + 7) / 8;
        if (nt == 1)
            return launch_tc<1, true>(a, s);
        if (nt == 2)
            return launch_tc<2, true>(a, s);
        return launch_decode_split(a, s);
    }
    if (!a.force_simple && decode_tc_supported(a))
        return launch_decode_tmem(a, s);
    return launch_decode_simple(a, s);
}

}  // namespace kvq
