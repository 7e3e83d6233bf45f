// gm_leg.cuh - leg sparsification in front of the referral, and its backward.
//
// "Graph Machine: Towards Better Pretraining via Edges" (ai.info summary), "Methodology in
// Plain English", referral paragraph: before the two-hop composition the stored edges are
// mixed into a pair of legs and each leg is sparsified; "Main Findings", bullet on more
// edges: the mixing is full across the k edge channels (its cost grows as k^2). For token
// (b, i), leg L in {1, 2} and leg channel h, every stored edge (c, a) of the token is a
// candidate with target E.idx[b,i,c,a] and weight fl32(M_L[b,i,h,c] * E.w[b,i,c,a]);
// candidates reaching the same target are summed in ascending c*s0 + a, and the s_L heaviest
// targets are kept (weight descending, then target ascending), padded with (0, 0.0f). This is
// the referral's own sparsify applied to a different candidate set.
//
// Work decomposition: one warp per token, lane = stored edge (c, a) (k*s0 <= 32). The stored
// edges are loaded once and grouped by target once (__match_any_sync); each of the 2k
// (leg, channel) rows then only multiplies by its coefficient, merges its duplicates and runs
// s_L rounds of warp max-reductions. The backward recomputes the same selection and keeps
// every output of a token in its warp: dE.w summed over (h, leg) in registers, dM by a
// fixed-order segment sum over each channel's s0 lanes. No atomics; deterministic.
#pragma once

#include "gm_common.cuh"

namespace gm {

struct LegArgs {
    const int32_t *e_idx;  // [tokens, k, s0]
    const float *e_w;
    const float *mix1;     // [tokens, k, k] at token stride mix_stride (k*k, or 0 = shared)
    const float *mix2;
    uint32_t mix_stride;
    int32_t *a1_idx;       // [tokens, k, s2]
    float *a1_w;
    int32_t *a2_idx;       // [tokens, k, s3]
    float *a2_w;
    const float *g1;       // backward: [tokens, k, s2], [tokens, k, s3]
    const float *g2;
    float *dew;            // backward: [tokens, k, s0]
    float *dmix1;          // backward: [tokens, k, k]
    float *dmix2;
    int accumulate;
    int k, s0, s2, s3, n;
    uint32_t tokens;
};

// The stored edge of this lane and its target group among the active lanes.
struct LegLane {
    int32_t t;       // target (valid when act)
    float w;         // stored weight (0 when not act)
    int c;           // stored channel of this lane
    bool act;        // active and in range
    unsigned same;   // lanes whose active edge has the same target (0 for inactive lanes)
};

__device__ __forceinline__ LegLane leg_lane(const LegArgs &a, uint32_t tok, int lane)
{
    const int nc = a.k * a.s0;
    LegLane L;
    L.c = lane / a.s0;
    L.t = 0;
    L.w = 0.0f;
    if (lane < nc) {
        L.t = __ldg(a.e_idx + (size_t)tok * nc + lane);
        L.w = __ldg(a.e_w + (size_t)tok * nc + lane);
    }
    L.act = L.w > 0.0f;
    if (L.act && (L.t < 0 || L.t >= a.n)) {
        raise_index_error();
        L.act = false;
    }
    if (!L.act) L.w = 0.0f;
    const unsigned amask = __ballot_sync(FULL, L.act);
    L.same = __match_any_sync(FULL, L.act ? L.t : -1) & amask;
    return L;
}

// A small per-token array (one leg's [k, k] coefficients, or one leg's [k, s] gradients),
// cached across the warp: with at most 64 elements lane l holds elements l and 32 + l in
// registers, loaded before any row is processed so the token's loads overlap; element e is
// then two shuffles away. Larger arrays read through L1.
struct TokCache {
    const float *p;
    float r0, r1;
    bool regs;
    __device__ __forceinline__ void load(const float *base, int kk, int lane)
    {
        p = base;
        regs = kk <= 64;
        r0 = regs && lane < kk ? __ldg(base + lane) : 0.0f;
        r1 = regs && lane + 32 < kk ? __ldg(base + 32 + lane) : 0.0f;
    }
    // element e (per lane; lanes with use == false get 0, but every lane takes part)
    __device__ __forceinline__ float get(int e, bool use) const
    {
        if (regs) {  // warp-uniform
            const float a = __shfl_sync(FULL, r0, e & 31);
            const float b = __shfl_sync(FULL, r1, e & 31);
            return use ? (e < 32 ? a : b) : 0.0f;
        }
        return use ? __ldg(p + e) : 0.0f;
    }
};

// Merge the nonzero products u of one (leg, channel) row by target, in ascending lane order,
// and return this lane's selection key (nonzero only on each target's first lane).
__device__ __forceinline__ void leg_merge(const LegLane &L, float u, int lane, unsigned &key_hi,
                                          unsigned &key_lo)
{
    const bool cand = u != 0.0f;
    const unsigned cmask = __ballot_sync(FULL, cand);
    const unsigned grp = L.same & cmask;
    const bool leader = cand && (__ffs(grp) - 1 == lane);
    float W = u;
    unsigned followers = __ballot_sync(FULL, cand && !leader);
    while (followers) {  // duplicates only; ascending lane order
        const int src = __ffs(followers) - 1;
        followers &= followers - 1;
        const float v = __shfl_sync(FULL, u, src);
        if (leader && ((grp >> src) & 1u)) W = __fadd_rn(W, v);
    }
    key_hi = leader ? __float_as_uint(W) : 0u;  // W > 0: its bits order like its value
    key_lo = leader ? ~(unsigned)L.t : 0u;       // larger key = smaller target
}

template <int WPB>
__global__ void __launch_bounds__(WPB * 32) leg_fwd_kernel(LegArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t tok = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (tok >= a.tokens) return;  // warp-uniform
    TokCache M[2];
    M[0].load(a.mix1 + (size_t)tok * a.mix_stride, a.k * a.k, lane);
    M[1].load(a.mix2 + (size_t)tok * a.mix_stride, a.k * a.k, lane);
    const LegLane L = leg_lane(a, tok, lane);

#pragma unroll
    for (int leg = 0; leg < 2; ++leg) {
        const int sl = leg == 0 ? a.s2 : a.s3;
        int32_t *oi = leg == 0 ? a.a1_idx : a.a2_idx;
        float *ow = leg == 0 ? a.a1_w : a.a2_w;
        for (int h = 0; h < a.k; ++h) {
            const float m = M[leg].get(h * a.k + L.c, L.act);
            const float u = L.act ? __fmul_rn(m, L.w) : 0.0f;
            unsigned key_hi, key_lo;
            leg_merge(L, u, lane, key_hi, key_lo);
            int32_t my_t = 0;
            float my_w = 0.0f;
            for (int r = 0; r < sl; ++r) {
                const unsigned mh = __reduce_max_sync(FULL, key_hi);
                if (mh == 0u) break;  // warp-uniform: the remaining slots are padding
                const unsigned ml = __reduce_max_sync(FULL, key_hi == mh ? key_lo : 0u);
                if (lane == r) {
                    my_t = (int32_t)~ml;
                    my_w = __uint_as_float(mh);
                }
                if (key_hi == mh && key_lo == ml) key_hi = key_lo = 0u;
            }
            if (lane < sl) {
                const size_t o = ((size_t)tok * a.k + h) * sl + lane;
                oi[o] = my_t;
                ow[o] = my_w;
            }
        }
    }
}

template <int WPB>
__global__ void __launch_bounds__(WPB * 32) leg_bwd_kernel(LegArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t tok = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (tok >= a.tokens) return;  // warp-uniform
    TokCache M[2];
    M[0].load(a.mix1 + (size_t)tok * a.mix_stride, a.k * a.k, lane);
    M[1].load(a.mix2 + (size_t)tok * a.mix_stride, a.k * a.k, lane);
    const LegLane L = leg_lane(a, tok, lane);
    const int nc = a.k * a.s0;
    const bool head = lane < nc && lane == L.c * a.s0;  // first lane of its stored channel

    TokCache G[2];
    G[0].load(a.g1 + (size_t)tok * a.k * a.s2, a.k * a.s2, lane);
    G[1].load(a.g2 + (size_t)tok * a.k * a.s3, a.k * a.s3, lane);

    float dew = 0.0f;
#pragma unroll
    for (int leg = 0; leg < 2; ++leg) {
        const int sl = leg == 0 ? a.s2 : a.s3;
        float *dmix = (leg == 0 ? a.dmix1 : a.dmix2) + (size_t)tok * a.k * a.k;
        for (int h = 0; h < a.k; ++h) {
            const float m = M[leg].get(h * a.k + L.c, L.act);
            const float u = L.act ? __fmul_rn(m, L.w) : 0.0f;
            unsigned key_hi, key_lo;
            leg_merge(L, u, lane, key_hi, key_lo);
            // kept slot of this lane's target; every active lane reaching a kept target takes
            // part in the derivative, also one whose own product was zero
            int slot = -1;
            for (int r = 0; r < sl; ++r) {
                const unsigned mh = __reduce_max_sync(FULL, key_hi);
                if (mh == 0u) break;
                const unsigned ml = __reduce_max_sync(FULL, key_hi == mh ? key_lo : 0u);
                if (L.act && (int32_t)~ml == L.t) slot = r;
                if (key_hi == mh && key_lo == ml) key_hi = key_lo = 0u;
            }
            const float gr = G[leg].get(h * sl + (slot >= 0 ? slot : 0), slot >= 0);
            dew = fmaf(gr, m, dew);
            // dM[h, c] = sum over the channel's s0 lanes, ascending a
            const float x = gr * L.w;
            float acc = x;
            for (int e = 1; e < a.s0; ++e) acc += __shfl_down_sync(FULL, x, e);
            if (head) {
                float *p = dmix + h * a.k + L.c;
                *p = a.accumulate ? *p + acc : acc;
            }
        }
    }
    if (lane < nc) {
        float *p = a.dew + (size_t)tok * nc + lane;
        *p = a.accumulate ? *p + dew : dew;
    }
}

}  // namespace gm
