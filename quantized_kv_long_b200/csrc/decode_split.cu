// decode_split.cu -- split-KV GQA decode attention for the 24-row verify
// batch (T = 4 query tokens x 6 query heads per KV head, head_dim 256) with
// the work split by role: score warps and value warps.
//
// What it computes is what decode.cu's kernel computes (speculative-decoding
// paragraph of the RX 9070 XT KV-streaming page: paged decode attention over a
// verify batch; "Known Issues Fixed" of the OSCAR2 page: the softmax max
// covers complete scores; GQA section of the KV-cache guide): per (layer, KV
// head, chunk) the chunk partial o = sum_j p_j v^_j / l and lse = m + ln l of
// every row, s_j = scale * sum_b d_b * sum_i q_i k_ij, with the same exact
// arithmetic (per-block fp32 K scaling, two-part P, exact two-part P d_v).
// decode.cu's pair kernel splits head_dim between the two warps of a pair,
// which then both run the softmax of the same 16 tokens; here each step runs
// once.  Measured on the 262,144-key verify step it is ~4 % faster; with one
// query token (6 rows) it is ~5 % slower, so launch_decode uses it for three
// n-tiles of rows only.
//
// Layout of the work:
//  * one CTA per (layer, KV head, chunk) with three warp roles: a copy warp,
//    NSW = 6 score warps and NOW = 8 value warps;
//  * the chunk streams in stages of 16*NSW tokens -- that many K head-rows
//    (272 B each) and V head-rows (144 B each), each one contiguous 16-byte-
//    aligned range of the head-major cache -- with cp.async.bulk into a ring
//    of NS shared-memory stages, completion tracked by mbarriers; the copy
//    warp refills a slot once every score and value warp has released it;
//  * score warp w owns tokens [16w, 16w+16) of every stage, over all of
//    head_dim: S^T = K Q^T on mma.sync m16n8k16 (rows = 16 tokens, columns =
//    8 query rows), in the permuted k order of decode_frag.cuh, each 32-element
//    block's product accumulated in fp32 and scaled by its fp32 d_b (times
//    scale*log2 e);
//  * online softmax per query row in base 2 with one running max per row
//    shared by the score warps, lazy: once per stage a barrier that also ORs
//    a flag tells whether any score exceeds it by more than TAU = 8; only then
//    do the warps exchange their tile maxima and move it (to the exact
//    maximum), recording the stage's rescale factor.  So p <= 2^8 and the max
//    covers complete scores;
//  * P is split into two f16 parts (P_hi + P_lo, ~2^-22 relative), moved to
//    the B-operand layout with movmatrix.trans and handed to the value warps
//    through NP shared-memory slots;
//  * value warp b owns Q4_0 block b (head dims 32b..32b+31) of every token:
//    O^T += V^T P^T on mma.sync (rows = 16 head dims, columns = 8 query rows)
//    with the token's fp16 d_v entering through the exact two-part product
//    (hi = RN(P_hi d), lo = fma(P_hi, d, -hi) + P_lo d).  It applies a
//    stage's rescale to O before the stage's PV;
//  * at the end the value warps divide by the sum of the score warps' l and
//    write the chunk partial (out, lse); the fused step then merges as in
//    decode.cu.
// Every mbarrier wait is bounded (about one second of wall time); a wait that
// runs out sets the device status word and the CTA falls through without
// hanging, after the copy warp waited (bounded) for its copies in flight.
#include "common.cuh"
#include "decode_frag.cuh"
#include "merge.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace kvq {

namespace {

using namespace frag;

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

constexpr int NSW = 6;                        // score warps (QK^T + softmax, 16 tokens each)
constexpr int NOW = 8;                        // value warps (PV, one 32-dim block each)
constexpr int PROD = NSW + NOW;               // the copy warp
constexpr int WARPS = NSW + NOW + 1;
constexpr int THREADS = 32 * WARPS;
constexpr int TOK = 16 * NSW;                 // tokens per stage
constexpr int NS = 4;                         // stages in the copy ring
constexpr int NP = 2;                         // P slots between score and value warps
constexpr int KROW = 272, VROW = 144;         // head-row bytes at head_dim 256
constexpr int STAGE_K = TOK * KROW;
constexpr int STAGE_V = TOK * VROW;
constexpr int STAGE_BYTES = STAGE_K + STAGE_V;
constexpr int BAR_S = 1;                      // named barrier of the score warps
constexpr int NGRP = (NSW + NOW) / 2;         // fused step: 64-thread merge groups
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float TAU = 8.0f;                   // lazy-max slack (log2 units)
constexpr float M_INIT = -1.0e30f;            // "no score yet", finite: ex2(s - M_INIT) stays defined

template <int NT>
struct __align__(16) DecodeSmem {
    uint8_t ring[NS][STAGE_BYTES];
    uint2 qf[16][NT][32];            // Q^T B-fragments [k-step][n-tile][lane]
    uint4 pf[NP][NSW][NT][32];       // P^T B-fragments (hi, hi, lo, lo) [slot][tile][n-tile][lane]
    float alpha[NP][NT * 8];         // per stage: rescale of O per row when `changed`
    int changed[NP];
    float tmx[NSW][NT * 8];          // tile maxima of a running-max update
    float fm[NT * 8];                // final running max per row
    float fl[NSW][NT * 8];           // final per-warp sums per row
    float red[NGRP][2];              // fused step: per-group reduction slots of the merge
    uint64_t full[NS], empty[NS], pfull[NP], pempty[NP], never;
    int abort;
    int last;                        // fused step: this CTA is the last of its (layer, KV head)
};
// fused step: chunks whose merge weights fit in the ring, per 64-thread group
constexpr int FUSED_SMEM_CHUNKS = (int)(NS * STAGE_BYTES / (NGRP * sizeof(float)));

// Bounded wait of one lane, broadcast to the warp; false (and the CTA's abort
// flag and the status word set) when it ran out.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          unsigned int *status, int lane)
{
    bool ok = true;
    if (lane == 0)
        ok = ptx::mbar_wait_bounded(bar, parity, abort, WAIT_LIMIT_NS);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok && lane == 0 && !*abort) {
        *abort = 1;
        report_timeout(status);
    }
    __syncwarp();
    return ok;
}

template <int NT, bool FUSED>
__global__ void __launch_bounds__(THREADS, 1) decode_split_kernel(const DecodeArgs a)
{
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
            ptx::mbar_init(&sm.empty[i], NSW + NOW);
        }
        for (int i = 0; i < NP; ++i) {
            ptx::mbar_init(&sm.pfull[i], NSW);
            ptx::mbar_init(&sm.pempty[i], NOW);
        }
        ptx::mbar_init(&sm.never, 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
        for (int st = 0; st < early; ++st)
            copy_stage(st);
    }
    // Q^T B-fragments: entry (ks, nt, lane) holds q[row nt*8 + lane/4] dims
    // 16 ks + 4 (lane%4) .. +3 (the permuted k order; zero for padded rows)
    {
        const __half *qbase = a.q + (int64_t)layer * a.T * a.n_q_heads * 256;
        for (int e = threadIdx.x; e < 16 * NT * 32; e += THREADS) {
            const int ln = e & 31, nt = (e >> 5) % NT, ks = e / (32 * NT);
            const int r = nt * 8 + (ln >> 2);
            uint2 v = make_uint2(0u, 0u);
            if (r < R) {
                const int t = r / G, gq = r % G;
                v = *reinterpret_cast<const uint2 *>(
                    qbase + ((int64_t)t * a.n_q_heads + h * G + gq) * 256 + ks * 16 + 4 * (ln & 3));
            }
            sm.qf[ks][nt][ln] = v;
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
        for (int task = warp; task < tasks; task += WARPS) {
            const int64_t j = j_lo + task / 16;
            const int blk = task % 16, b = blk & 7;
            const int tok = (int)(j - (a.n_kv - a.T));
            const int64_t src =
                (((int64_t)layer * a.T + tok) * a.n_kv_heads + h) * 256 + b * QK + lane;
            const int64_t row = (int64_t)h * cap + j;
            if (blk < 8)
                warp_quant_q8_0(a.k_new[src], kw + row * KROW + b * Q8_0_BYTES, lane);
            else
                warp_quant_q4_0(a.v_new[src], vw + row * VROW + b * Q4_0_BYTES, lane);
        }
        // the blocks just written are read next by bulk copies (the async proxy)
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncthreads();
    volatile int *abort = &sm.abort;
    const int g = lane >> 2, cq = lane & 3;

    if (a.test_timeout && lane == 0) {
        // test hook: wait on a barrier that nothing completes
        if (!ptx::mbar_wait_bounded(&sm.never, 0, abort, WAIT_LIMIT_NS)) {
            *abort = 1;
            report_timeout(a.status);
        }
    }
    __syncwarp();

    float o[2][NT][4];  // value warps: O^T of the warp's block (2 m-tiles) x NT n-tiles
    if (warp == PROD) {
        // ------------------------------------------------------------ copies
        if (lane == 0) {
            int issued = early;
            for (int st = early; st < n_stages; ++st) {
                const int slot = st % NS;
                const uint32_t round = st / NS;
                // refill once every warp released the slot and its previous copy landed
                if (st >= NS &&
                    (!ptx::mbar_wait_bounded(&sm.empty[slot], (round - 1) & 1, abort, WAIT_LIMIT_NS) ||
                     !ptx::mbar_wait_bounded(&sm.full[slot], (round - 1) & 1, abort, WAIT_LIMIT_NS))) {
                    if (!*abort) {
                        *abort = 1;
                        report_timeout(a.status);
                    }
                    break;
                }
                if (*abort)
                    break;
                copy_stage(st);
                ++issued;
            }
            // drain: every issued copy has landed before the ring is reused or freed
            // (bounded, without the abort short-cut)
            int no_abort = 0;
            for (int st = (issued > NS ? issued - NS : 0); st < issued; ++st)
                if (!ptx::mbar_wait_bounded(&sm.full[st % NS], (st / NS) & 1, &no_abort,
                                            WAIT_LIMIT_NS))
                    report_timeout(a.status);
        }
    } else if (warp < NSW) {
        // ------------------------------------------------------------ score warp w
        const int w = warp;
        const float dscale = a.scale * LOG2E;
        float m2[NT][2], l2[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                m2[nt][k] = M_INIT;
                l2[nt][k] = 0.0f;
            }
        bool aborted = false;
        for (int s = 0; s < n_stages; ++s) {
            const int slot = s % NS, ps = s % NP;
            const int valid = min(16, n_tok - s * TOK - 16 * w);  // tokens of this warp's tile
            if (!aborted)
                aborted = !warp_wait(&sm.full[slot], (s / NS) & 1, abort, a.status, lane);
            float sv[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    sv[nt][i] = -INFINITY;
            if (valid > 0 && !aborted) {
                // ---- S^T of the tile over all 8 blocks, exact per-block scale
                const uint8_t *ks = sm.ring[slot] + (16 * w) * KROW;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        sv[nt][i] = 0.0f;
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const uint8_t *r0 = ks + g * KROW + 34 * b;
                    const uint8_t *r1 = r0 + 8 * KROW;
                    const float dk0 = __half2float(__ushort_as_half((unsigned short)lds16(r0))) * dscale;
                    const float dk1 = __half2float(__ushort_as_half((unsigned short)lds16(r1))) * dscale;
                    float blk[NT][4];
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        const int off = 2 + 16 * s2 + 4 * cq;
                        uint32_t af[4];
                        s8x4_to_h2x2(k_word(r0 + off, (b & 1) != 0), af[0], af[2]);
                        s8x4_to_h2x2(k_word(r1 + off, (b & 1) != 0), af[1], af[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint2 qb = sm.qf[2 * b + s2][nt][lane];
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
                        sv[nt][0] = fmaf(dk0, blk[nt][0], sv[nt][0]);
                        sv[nt][1] = fmaf(dk0, blk[nt][1], sv[nt][1]);
                        sv[nt][2] = fmaf(dk1, blk[nt][2], sv[nt][2]);
                        sv[nt][3] = fmaf(dk1, blk[nt][3], sv[nt][3]);
                    }
                }
                // ---- mask (ragged tail of the chunk, causal rows of the verify batch,
                //      padded rows)
                const int j0 = s * TOK + 16 * w;  // key of token 0, relative to c0
                if (valid < 16 || c0 + j0 + 15 > a.n_kv - a.T) {
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
            }
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&sm.empty[slot]);  // this warp is done with the slot's K rows

            // ---- running max shared by the score warps (lazy: it moves only when a
            //      score exceeds it by more than TAU; then to the exact maximum)
            float tmax[NT][2];
            bool up = false;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    tmax[nt][k] = fmaxf(sv[nt][k], sv[nt][2 + k]);
                    up |= tmax[nt][k] > m2[nt][k] + TAU;
                }
            const bool any = named_bar_or(BAR_S, NSW * 32, up);
            float alk[NT][2] = {};
            if (any) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        float v = tmax[nt][k];
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                        if (g == 0)
                            sm.tmx[w][nt * 8 + 2 * cq + k] = v;
                    }
                ptx::named_bar_sync(BAR_S, NSW * 32);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int row = nt * 8 + 2 * cq + k;
                        float v = sm.tmx[0][row];
#pragma unroll
                        for (int w2 = 1; w2 < NSW; ++w2)
                            v = fmaxf(v, sm.tmx[w2][row]);
                        const float mn = fmaxf(m2[nt][k], v);
                        alk[nt][k] = ptx::ex2(m2[nt][k] - mn);
                        m2[nt][k] = mn;
                        l2[nt][k] *= alk[nt][k];
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
                const __half2 r01 =
                    __floats2half2_rn(p[0] - __low2float(h01), p[1] - __high2float(h01));
                const __half2 r23 =
                    __floats2half2_rn(p[2] - __low2float(h23), p[3] - __high2float(h23));
                ph[nt][0] = ptx::movmatrix_trans(ptx::h2_bits(h01));
                ph[nt][1] = ptx::movmatrix_trans(ptx::h2_bits(h23));
                pl[nt][0] = ptx::movmatrix_trans(ptx::h2_bits(r01));
                pl[nt][1] = ptx::movmatrix_trans(ptx::h2_bits(r23));
            }
            // ---- hand P (and the stage's rescale) to the value warps
            if (!aborted && s >= NP)
                aborted = !warp_wait(&sm.pempty[ps], ((s / NP) - 1) & 1, abort, a.status, lane);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                sm.pf[ps][w][nt][lane] = make_uint4(ph[nt][0], ph[nt][1], pl[nt][0], pl[nt][1]);
            if (w == 0) {
                if (lane == 0)
                    sm.changed[ps] = any ? 1 : 0;
                if (any && g == 0) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int k = 0; k < 2; ++k)
                            sm.alpha[ps][nt * 8 + 2 * cq + k] = alk[nt][k];
                }
            }
            __syncwarp();
            if (lane == 0)
                ptx::mbar_arrive(&sm.pfull[ps]);
        }
        // per-row sums over the 8 lanes that share a row
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                float v = l2[nt][k];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                if (g == 0) {
                    sm.fl[w][nt * 8 + 2 * cq + k] = v;
                    if (w == 0)
                        sm.fm[nt * 8 + 2 * cq + k] = m2[nt][k];
                }
            }
    } else {
        // ------------------------------------------------------------ value warp
        const int b = warp - NSW;  // Q4_0 block b: head dims [32b, 32b + 32)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    o[mt][nt][i] = 0.0f;
        bool aborted = false;
        for (int s = 0; s < n_stages; ++s) {
            const int slot = s % NS, ps = s % NP;
            if (!aborted)
                aborted = !warp_wait(&sm.full[slot], (s / NS) & 1, abort, a.status, lane) ||
                          !warp_wait(&sm.pfull[ps], (s / NP) & 1, abort, a.status, lane);
            if (!aborted) {
                if (sm.changed[ps]) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            const float al = sm.alpha[ps][nt * 8 + 2 * cq + k];
#pragma unroll
                            for (int mt = 0; mt < 2; ++mt) {
                                o[mt][nt][k] *= al;
                                o[mt][nt][2 + k] *= al;
                            }
                        }
                }
                // ---- O^T += V^T (P d_v)^T over the stage's tiles, this warp's block
                const uint8_t *v0 = sm.ring[slot] + STAGE_K + (2 * cq) * VROW + 18 * b;
#pragma unroll
                for (int w = 0; w < NSW; ++w) {
                    const int valid = min(16, n_tok - s * TOK - 16 * w);
                    if (valid <= 0)
                        break;
                    const uint8_t *vb = v0 + (16 * w) * VROW;  // tokens 2c, 2c+1, 2c+8, 2c+9
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
                        const uint4 pf = sm.pf[ps][w][nt][lane];
                        const uint32_t ph[2] = {pf.x, pf.y}, pl[2] = {pf.z, pf.w};
                        // P d_v as hi + lo without loss: hi = RN(P_hi d), the exact
                        // product error fma(P_hi, d, -hi), plus P_lo d
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
            }
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(&sm.pempty[ps]);
                ptx::mbar_arrive(&sm.empty[slot]);
            }
        }
    }
    __syncthreads();  // copies drained; per-warp sums and the final max visible

    // ---------------------------------------------------------------- chunk partial
    const int Hq = a.n_q_heads;
    if (warp >= NSW && warp < PROD) {
        const int b = warp - NSW;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int col = nt * 8 + 2 * cq + k;
                if (col >= R)
                    continue;
                float L = 0.0f;
#pragma unroll
                for (int w = 0; w < NSW; ++w)
                    L += sm.fl[w][col];
                const float f = L > 0.0f ? 1.0f / L : 0.0f;
                const int t = col / G, gq = col % G;
                const int64_t row = ((int64_t)layer * a.T + t) * Hq + h * G + gq;
                float *dst = a.out_part + (row * C + c) * 256 + 32 * b + 2 * g;
                *reinterpret_cast<float2 *>(dst) = make_float2(o[0][nt][k] * f, o[0][nt][2 + k] * f);
                *reinterpret_cast<float2 *>(dst + 16) =
                    make_float2(o[1][nt][k] * f, o[1][nt][2 + k] * f);
                if (b == 0 && g == 0)
                    a.lse_part[row * C + c] =
                        L > 0.0f ? (sm.fm[col] + log2f(L)) * LN2 : -INFINITY;
            }
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
        if (sm.last && threadIdx.x < NGRP * 64) {
            const int grp = threadIdx.x >> 6, t64 = threadIdx.x & 63;
            float *w_s = C <= FUSED_SMEM_CHUNKS ? reinterpret_cast<float *>(sm.ring) + grp * C
                                                : nullptr;
            for (int col = grp; col < R; col += NGRP) {
                const int t = col / G, gq = col % G;
                const int64_t row = ((int64_t)layer * a.T + t) * Hq + h * G + gq;
                merge_row<true>(a.out_part + row * C * 256, a.lse_part + row * C, C, 256,
                                a.out + row * 256, a.lse + row, w_s, sm.red[grp], t64,
                                [grp] { ptx::named_bar_sync(2 + grp, 64); });
            }
        }
    }
}

template <bool FUSED>
bool launch_split(const DecodeArgs &a, cudaStream_t s)
{
    constexpr int NT = 3;
    const size_t smem = sizeof(DecodeSmem<NT>);
    static bool attr_set[64] = {};  // the attribute belongs to the function on each device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return false;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(decode_split_kernel<NT, FUSED>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return false;
        attr_set[dev] = true;
    }
    const int64_t C = (a.n_kv + a.chunk - 1) / a.chunk;
    const int64_t grid = (int64_t)a.n_layers * a.n_kv_heads * C;
    if (grid >= (1ll << 31))
        return false;
    decode_split_kernel<NT, FUSED><<<(unsigned)grid, THREADS, smem, s>>>(a);
    return true;
}

}  // namespace

// The shapes decode_tc_supported accepts with 17..24 rows (three n-tiles).
bool launch_decode_split(const DecodeArgs &a, cudaStream_t s)
{
    return a.counters ? launch_split<true>(a, s) : launch_split<false>(a, s);
}

}  // namespace kvq
