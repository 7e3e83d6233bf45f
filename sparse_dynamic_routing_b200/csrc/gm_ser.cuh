// gm_ser.cuh - sparse edge referral (SER), one warp per edge row (b, i, h).
//
// "Graph Machine: Towards Better Pretraining via Edges" (ai.info summary), "Key
// Contributions" item 3 and "Methodology in Plain English", referral paragraph:
// A' = Sparsify_s1(A1 A2). Lane c < s2*s3 owns candidate c = a*s3 + e, i.e. the two-hop
// path i -> j = A1.idx[a] -> t = A2[j].idx[e] with weight fl32(A1.w[a] * A2[j].w[e]). With
// refresh edges F ("Methodology in Plain English", referral paragraph, last sentence), lane
// s2*s3 + f owns refresh slot f with its own weight: A' = Sparsify_s1(A1 A2 + F).
// Duplicates are merged with __match_any_sync: the lowest lane of each group of equal
// targets sums the group's weights in ascending lane (= candidate) order with __fadd_rn.
// Top-s1 is s1 rounds of a two-stage warp max (REDUX) on the key (weight bits, ~index):
// positive fp32 values order like their bit patterns, and ~t = 0xffffffff - t makes the
// smaller index win a tie. Products and sums use the _rn intrinsics so that nvcc cannot fuse
// them into FMAs; the result is bit-identical to the plain sequential definition.
#pragma once

#include "gm_common.cuh"

// Legs of a multi-step referral after the first one (the pages' models use 3 or 4 legs).
#ifndef GM_MAX_CHAIN
#define GM_MAX_CHAIN 7
#endif

namespace gm {

struct SerArgs {
    const int32_t *a1_idx;
    const float *a1_w;
    const int32_t *a2_idx;
    const float *a2_w;
    int32_t *out_idx;
    float *out_w;
    int s1, s2, s3;
    int n, k;
    uint32_t rows;  // B * n * k
    RowMap map;     // heads = k
    // refresh edges [rows, sf] joining the candidates after the two-hop paths (sf = 0: none)
    const int32_t *f_idx;
    const float *f_w;
    int sf;
    // multi-step referral: legs 3.. of the chain B_{m+1} = Sparsify(B_m A_{m+1}) (leg 2 is
    // a2), nchain of them; intermediates are cut to s_mid slots, the last step to s1
    const int32_t *chain_idx[GM_MAX_CHAIN - 1];
    const float *chain_w[GM_MAX_CHAIN - 1];
    int nchain;
    int s_mid;
};

// ---- one referral step of one row, one candidate per lane ----------------------------------
//
// The first leg of the row is held by the warp (lane a < s_in holds slot a: target j_l,
// weight w1_l); the second leg is [rows, s3] at (leg_idx, leg_w), channel h of the same
// sequence; lanes s_in*s3 .. s_in*s3 + sf - 1 hold the row's refresh slots, if any.

struct ReferCand {
    int32_t t;    // candidate target (valid when u != 0)
    float u;      // candidate weight (0: no candidate)
    float w1;     // first-leg weight of a path candidate
    float w2;     // second-leg weight of a path candidate
    size_t r2;    // second-leg element of a path candidate
    bool path;    // lane < s_in * s3
    bool refresh; // refresh slot lane - s_in * s3
};

__device__ __forceinline__ ReferCand refer_candidates(int32_t j_l, float w1_l, int s_in,
                                                      const int32_t *leg_idx, const float *leg_w,
                                                      int s3, const int32_t *f_idx,
                                                      const float *f_w, int sf, uint32_t row,
                                                      int n, int k, uint32_t seq_base,
                                                      uint32_t h, int lane)
{
    const int nc = s_in * s3;
    const int ca = lane / s3;          // first-leg slot of this lane's candidate
    const int ce = lane - ca * s3;     // second-leg slot
    const int32_t j = __shfl_sync(FULL, j_l, ca);
    ReferCand c;
    c.w1 = __shfl_sync(FULL, w1_l, ca);
    c.u = 0.0f;
    c.w2 = 0.0f;
    c.t = 0;
    c.r2 = 0;
    c.path = lane < nc;
    c.refresh = lane >= nc && lane < nc + sf;
    bool act = c.path && c.w1 > 0.0f;
    if (act && (j < 0 || j >= n)) {
        if (ce == 0) raise_index_error();  // once per active first-leg slot
        act = false;
    }
    if (act) {
        c.r2 = ((size_t)(seq_base + (uint32_t)j) * k + h) * s3 + ce;
        c.w2 = __ldg(leg_w + c.r2);
        const int32_t t2 = __ldg(leg_idx + c.r2);
        if (c.w2 > 0.0f) {
            if (t2 < 0 || t2 >= n) {
                raise_index_error();
            } else {
                c.u = __fmul_rn(c.w1, c.w2);
                c.t = t2;
            }
        }
    }
    if (c.refresh) {
        const size_t rf = (size_t)row * sf + (lane - nc);
        const float wf = __ldg(f_w + rf);
        const int32_t tf = __ldg(f_idx + rf);
        if (wf > 0.0f) {
            if (tf < 0 || tf >= n) {
                raise_index_error();
            } else {
                c.u = wf;
                c.t = tf;
            }
        }
    }
    return c;
}

// Merge: equal targets form a group whose lowest lane (the leader) accumulates the other
// members in ascending lane order (only non-leading members need a shuffle). Returns the
// lane's selection key (weight bits, ~target), nonzero on leaders only.
__device__ __forceinline__ void refer_merge(const ReferCand &c, int lane, unsigned &key_hi,
                                            unsigned &key_lo)
{
    const bool cand = c.u != 0.0f;
    const unsigned cmask = __ballot_sync(FULL, cand);
    const unsigned grp = __match_any_sync(FULL, cand ? c.t : -1) & cmask;
    const bool leader = cand && (__ffs(grp) - 1 == lane);
    float W = c.u;
    unsigned followers = __ballot_sync(FULL, cand && !leader);
    while (followers) {  // warp-uniform loop, usually empty
        const int src = __ffs(followers) - 1;
        followers &= followers - 1;
        const float v = __shfl_sync(FULL, c.u, src);
        if (leader && ((grp >> src) & 1u)) W = __fadd_rn(W, v);
    }
    key_hi = leader ? __float_as_uint(W) : 0u;
    key_lo = leader ? ~(unsigned)c.t : 0u;
}

// Top-s_out by (weight desc, index asc). Lane r < s_out receives the r-th kept (t, W),
// others (0, 0.0f); every candidate lane whose target was kept receives its slot and W.
__device__ __forceinline__ void refer_select(const ReferCand &c, unsigned key_hi, unsigned key_lo,
                                             int s_out, int lane, int32_t &t_out, float &w_out,
                                             int &slot, float &slot_w)
{
    t_out = 0;
    w_out = 0.0f;
    slot = -1;
    slot_w = 0.0f;
    const bool cand = c.u != 0.0f;
    for (int r = 0; r < s_out; ++r) {
        const unsigned mh = __reduce_max_sync(FULL, key_hi);
        if (mh == 0u) break;  // warp-uniform: no candidate left, the rest stays padding
        const unsigned ml = __reduce_max_sync(FULL, key_hi == mh ? key_lo : 0u);
        if (lane == r) {
            t_out = (int32_t)~ml;
            w_out = __uint_as_float(mh);
        }
        if (cand && (int32_t)~ml == c.t) {
            slot = r;
            slot_w = __uint_as_float(mh);
        }
        if (key_hi == mh && key_lo == ml) key_hi = key_lo = 0u;
    }
}

// Referral of one edge row. On return lane r < s1 holds the r-th kept (t, W); other lanes
// (and slots beyond the number of distinct targets) hold (0, 0.0f). Must be called by all
// 32 lanes of the warp. `seq_base` = b*n and `h` = channel of `row`.
__device__ __forceinline__ void ser_row(const SerArgs &a, uint32_t row, uint32_t seq_base,
                                        uint32_t h, int lane, int32_t &t_out, float &w_out)
{
    // first leg: lane a < s2 reads slot a of row i
    int32_t j_l = 0;
    float w1_l = 0.0f;
    if (lane < a.s2) {
        j_l = __ldg(a.a1_idx + (size_t)row * a.s2 + lane);
        w1_l = __ldg(a.a1_w + (size_t)row * a.s2 + lane);
    }
    const ReferCand c = refer_candidates(j_l, w1_l, a.s2, a.a2_idx, a.a2_w, a.s3, a.f_idx, a.f_w,
                                         a.sf, row, a.n, a.k, seq_base, h, lane);
    unsigned key_hi, key_lo;
    refer_merge(c, lane, key_hi, key_lo);
    int slot;
    float slot_w;
    refer_select(c, key_hi, key_lo, a.s1, lane, t_out, w_out, slot, slot_w);
}

template <int WPB>
__global__ void __launch_bounds__(WPB * 32) ser_kernel(SerArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t row = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (row >= a.rows) return;  // warp-uniform
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t t;
    float w;
    ser_row(a, row, seq_base, h, lane, t, w);
    if (lane < a.s1) {
        a.out_idx[(size_t)row * a.s1 + lane] = t;
        a.out_w[(size_t)row * a.s1 + lane] = w;
    }
}

}  // namespace gm
