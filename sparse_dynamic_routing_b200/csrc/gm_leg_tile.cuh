// gm_leg_tile.cuh - leg sparsification and its backward, one thread per leg row.
//
// Same definition and arithmetic as gm_leg.cuh ("Graph Machine: Towards Better Pretraining
// via Edges", ai.info summary, "Methodology in Plain English", referral paragraph: the stored
// edges are mixed into a pair of legs and each leg is sparsified), with a division of work
// that spends far fewer instructions when k is a power of two up to 16, s0 is 2 or 4 and
// both leg budgets are at most SM.
//
// A warp owns TPW = 16 / K consecutive tokens, i.e. 32 leg rows (token, leg, h), one per lane.
//  Staging (whole warp, per token): the token's k*s0 stored edges are grouped by target once
//    (__match_any_sync over the active ones) into a compact list of 16-byte group records
//    (target, first member's channel and weight, mask of the later members) in shared
//    memory, beside the stored weights and both legs' [k, k] coefficients.
//  Rows (one per lane): walk the token's groups; a group's merged weight is the fp32 sum, in
//    ascending candidate order, of fl32(M[h, c] * w) over its members, started from 0.0f.
//    Adding +0 to a non-negative float and adding x to 0 are exact, so members whose product
//    is zero change nothing and the sum equals the reference sum over the nonzero products
//    only, started from the first. Groups with a positive weight enter a sorted register
//    list of the SM heaviest (weight desc, then target asc); the first s_L are written,
//    padded with (0, 0.0f).
//  Backward: the same selection, then each kept group's members receive g * M[h, c] (into a
//    per-row shared-memory line of the token's candidates) and the row's coefficient
//    gradients g * w (into its own shared-memory line); a final pass sums the candidate
//    lines over the token's rows in a fixed order. Deterministic, no atomics.
#pragma once

#include "gm_common.cuh"
#include "gm_leg.cuh"

namespace gm {

template <int K, int S0> struct LegTileGeom {
    static constexpr int NC = K * S0;   // stored edges (candidates) per token
    static constexpr int RPT = 2 * K;   // leg rows per token
    static constexpr int TPW = 32 / RPT;
    static constexpr int MP = K + 1;    // padded coefficient row (bank spread across rows)
    static_assert(NC <= 32 && RPT <= 32 && 32 % RPT == 0, "unsupported leg tile shape");
};

// One target group of a token: its first member inline (most groups have no other), the
// later members as a mask.
struct __align__(16) LegGroup {
    int32_t t;       // target
    int32_t ch;      // stored channel of the first member
    float w;         // stored weight of the first member
    unsigned more;   // later members (bit c = stored edge c)
};

template <int K, int S0> struct LegTok {
    using Geo = LegTileGeom<K, S0>;
    LegGroup grp[Geo::NC];      // groups in order of first member
    unsigned gm[Geo::NC];       // all members of each group
    float w[Geo::NC];           // stored weights (0 when inactive)
    float mix[2][K][Geo::MP];   // both legs' coefficients, [leg][h][c]
    int ng;                     // number of groups
};

// Stage one token into shared memory (whole warp; tok < tokens is warp-uniform).
template <int K, int S0>
__device__ __forceinline__ void leg_stage(const LegArgs &a, uint32_t tok, int lane, LegTok<K, S0> &S)
{
    constexpr int NC = K * S0;
    int32_t t = 0;
    float w = 0.0f;
    if (lane < NC) {
        t = __ldg(a.e_idx + (size_t)tok * NC + lane);
        w = __ldg(a.e_w + (size_t)tok * NC + lane);
    }
    bool act = w > 0.0f;
    if (act && (t < 0 || t >= a.n)) {
        raise_index_error();
        act = false;
    }
    const unsigned amask = __ballot_sync(FULL, act);
    const unsigned same = __match_any_sync(FULL, act ? t : -1) & amask;
    const bool leader = act && (__ffs(same) - 1 == lane);
    const unsigned lmask = __ballot_sync(FULL, leader);
    if (leader) {
        const int gi = __popc(lmask & ((1u << lane) - 1u));
        S.grp[gi] = LegGroup{t, lane / S0, w, same & ~(1u << lane)};
        S.gm[gi] = same;
    }
    if (lane < NC) S.w[lane] = act ? w : 0.0f;
    if (lane == 0) S.ng = __popc(lmask);
    const float *m1 = a.mix1 + (size_t)tok * a.mix_stride;
    const float *m2 = a.mix2 + (size_t)tok * a.mix_stride;
#pragma unroll
    for (int e = lane; e < 2 * K * K; e += 32) {
        const int leg = e / (K * K), rem = e - leg * (K * K);
        const int h = rem / K, c = rem - h * K;
        S.mix[leg][h][c] = __ldg((leg == 0 ? m1 : m2) + rem);
    }
}

// Sorted insertion into the register list of the SM heaviest groups.
template <int SM>
__device__ __forceinline__ void leg_insert(float W, int32_t t, int g, float (&bw)[SM],
                                           int32_t (&bt)[SM], int (&bg)[SM])
{
    if (W > bw[SM - 1] || (W == bw[SM - 1] && t < bt[SM - 1])) {
        bw[SM - 1] = W;
        bt[SM - 1] = t;
        bg[SM - 1] = g;
#pragma unroll
        for (int x = SM - 1; x > 0; --x) {
            const bool up = bw[x] > bw[x - 1] || (bw[x] == bw[x - 1] && bt[x] < bt[x - 1]);
            const float fw = bw[x];
            const int32_t ft = bt[x];
            const int fg = bg[x];
            bw[x] = up ? bw[x - 1] : bw[x];
            bt[x] = up ? bt[x - 1] : bt[x];
            bg[x] = up ? bg[x - 1] : bg[x];
            bw[x - 1] = up ? fw : bw[x - 1];
            bt[x - 1] = up ? ft : bt[x - 1];
            bg[x - 1] = up ? fg : bg[x - 1];
        }
    }
}

// Merge and select one leg row (leg, h) of a staged token.
template <int K, int S0, int SM>
__device__ __forceinline__ void leg_row_select(const LegTok<K, S0> &S, int leg, int h,
                                               float (&bw)[SM], int32_t (&bt)[SM], int (&bg)[SM])
{
#pragma unroll
    for (int x = 0; x < SM; ++x) {
        bw[x] = 0.0f;
        bt[x] = 0;
        bg[x] = -1;
    }
    const float *mrow = S.mix[leg][h];
    const int ng = S.ng;
    for (int g = 0; g < ng; ++g) {
        const LegGroup G = S.grp[g];
        // 0 + x is exact, so starting from the first product equals starting from 0.0f
        float W = __fmul_rn(mrow[G.ch], G.w);
        unsigned mask = G.more;
        while (mask) {
            const int c = __ffs(mask) - 1;
            mask &= mask - 1;
            W = __fadd_rn(W, __fmul_rn(mrow[c / S0], S.w[c]));
        }
        if (W > 0.0f) leg_insert<SM>(W, G.t, g, bw, bt, bg);
    }
}

template <int K, int S0, int SM, int WPB>
__global__ void __launch_bounds__(WPB * 32) leg_fwd_tile_kernel(LegArgs a)
{
    using Geo = LegTileGeom<K, S0>;
    __shared__ LegTok<K, S0> sm[WPB][Geo::TPW];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t tok0 = (blockIdx.x * WPB + wid) * Geo::TPW;
    if (tok0 >= a.tokens) return;  // warp-uniform
#pragma unroll
    for (int tt = 0; tt < Geo::TPW; ++tt)
        if (tok0 + tt < a.tokens) leg_stage<K, S0>(a, tok0 + tt, lane, sm[wid][tt]);
    __syncwarp();

    const int tt = lane / Geo::RPT, r = lane - tt * Geo::RPT;
    const int leg = r / K, h = r - leg * K;
    const uint32_t tok = tok0 + tt;
    if (tok >= a.tokens) return;  // no warp-wide operation below
    float bw[SM];
    int32_t bt[SM];
    int bg[SM];
    leg_row_select<K, S0, SM>(sm[wid][tt], leg, h, bw, bt, bg);
    const int sl = leg == 0 ? a.s2 : a.s3;
    int32_t *oi = (leg == 0 ? a.a1_idx : a.a2_idx) + ((size_t)tok * K + h) * sl;
    float *ow = (leg == 0 ? a.a1_w : a.a2_w) + ((size_t)tok * K + h) * sl;
#pragma unroll
    for (int x = 0; x < SM; ++x) {
        if (x < sl) {
            oi[x] = bt[x];  // (0, 0.0f) where fewer groups than slots
            ow[x] = bw[x];
        }
    }
}

template <int K, int S0> struct LegBwdTok {
    using Geo = LegTileGeom<K, S0>;
    float contrib[Geo::RPT][Geo::NC + 1];  // per row: g * M[h, c] of each kept member c
    float dm[Geo::RPT][K];                 // per row: its coefficient gradients
};

template <int K, int S0, int SM, int WPB>
__global__ void __launch_bounds__(WPB * 32) leg_bwd_tile_kernel(LegArgs a)
{
    using Geo = LegTileGeom<K, S0>;
    constexpr int NC = Geo::NC;
    __shared__ LegTok<K, S0> sm[WPB][Geo::TPW];
    __shared__ LegBwdTok<K, S0> sb[WPB][Geo::TPW];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t tok0 = (blockIdx.x * WPB + wid) * Geo::TPW;
    if (tok0 >= a.tokens) return;  // warp-uniform
#pragma unroll
    for (int tt = 0; tt < Geo::TPW; ++tt)
        if (tok0 + tt < a.tokens) leg_stage<K, S0>(a, tok0 + tt, lane, sm[wid][tt]);
    __syncwarp();

    {
        const int tt = lane / Geo::RPT, r = lane - tt * Geo::RPT;
        const int leg = r / K, h = r - leg * K;
        const uint32_t tok = tok0 + tt;
        if (tok < a.tokens) {
            const LegTok<K, S0> &S = sm[wid][tt];
            LegBwdTok<K, S0> &B = sb[wid][tt];
#pragma unroll
            for (int c = 0; c < NC; ++c) B.contrib[r][c] = 0.0f;
#pragma unroll
            for (int c = 0; c < K; ++c) B.dm[r][c] = 0.0f;
            float bw[SM];
            int32_t bt[SM];
            int bg[SM];
            leg_row_select<K, S0, SM>(S, leg, h, bw, bt, bg);
            const int sl = leg == 0 ? a.s2 : a.s3;
            const float *g = (leg == 0 ? a.g1 : a.g2) + ((size_t)tok * K + h) * sl;
            const float *mrow = S.mix[leg][h];
#pragma unroll
            for (int x = 0; x < SM; ++x) {
                if (x < sl && bg[x] >= 0) {
                    const float gr = __ldg(g + x);
                    // every active member of the kept group, also one whose product was zero
                    unsigned mask = S.gm[bg[x]];
                    while (mask) {
                        const int c = __ffs(mask) - 1;
                        mask &= mask - 1;
                        B.contrib[r][c] = gr * mrow[c / S0];
                        B.dm[r][c / S0] += gr * S.w[c];
                    }
                }
            }
        }
    }
    __syncwarp();

#pragma unroll
    for (int tt = 0; tt < Geo::TPW; ++tt) {
        const uint32_t tok = tok0 + tt;
        if (tok >= a.tokens) break;  // warp-uniform
        const LegBwdTok<K, S0> &B = sb[wid][tt];
        if (lane < NC) {  // dE.w[c]: rows in order leg 1 h = 0..K-1, then leg 2
            float s = 0.0f;
#pragma unroll
            for (int r = 0; r < Geo::RPT; ++r) s += B.contrib[r][lane];
            float *p = a.dew + (size_t)tok * NC + lane;
            *p = a.accumulate ? *p + s : s;
        }
#pragma unroll
        for (int e = lane; e < 2 * K * K; e += 32) {
            const int r = e / K, c = e - r * K;  // row r = leg * K + h
            const int leg = r / K, h = r - leg * K;
            float *p = (leg == 0 ? a.dmix1 : a.dmix2) + (size_t)tok * K * K + h * K + c;
            *p = a.accumulate ? *p + B.dm[r][c] : B.dm[r][c];
        }
    }
}

}  // namespace gm
