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
};

// Referral of one edge row. On return lane r < s1 holds the r-th kept (t, W); other lanes
// (and slots beyond the number of distinct targets) hold (0, 0.0f). Must be called by all
// 32 lanes of the warp. `seq_base` = b*n and `h` = channel of `row`.
__device__ __forceinline__ void ser_row(const SerArgs &a, uint32_t row, uint32_t seq_base,
                                        uint32_t h, int lane, int32_t &t_out, float &w_out)
{
    const int nc = a.s2 * a.s3;

    // first leg: lane a < s2 reads slot a of row i
    int32_t j_l = 0;
    float w1_l = 0.0f;
    if (lane < a.s2) {
        j_l = __ldg(a.a1_idx + (size_t)row * a.s2 + lane);
        w1_l = __ldg(a.a1_w + (size_t)row * a.s2 + lane);
    }
    const int ca = lane / a.s3;          // first-leg slot of this lane's candidate
    const int ce = lane - ca * a.s3;     // second-leg slot
    const int32_t j = __shfl_sync(FULL, j_l, ca);
    const float w1 = __shfl_sync(FULL, w1_l, ca);

    // second leg: lane c reads slot e of row j (same channel h)
    float u = 0.0f;
    int32_t t = 0;
    bool act = lane < nc && w1 > 0.0f;
    if (act && (j < 0 || j >= a.n)) {
        if (ce == 0) raise_index_error();  // once per active first-leg slot
        act = false;
    }
    if (act) {
        const size_t r2 = ((size_t)(seq_base + (uint32_t)j) * a.k + h) * a.s3 + ce;
        const float w2 = __ldg(a.a2_w + r2);
        const int32_t t2 = __ldg(a.a2_idx + r2);
        if (w2 > 0.0f) {
            if (t2 < 0 || t2 >= a.n) {
                raise_index_error();
            } else {
                u = __fmul_rn(w1, w2);
                t = t2;
            }
        }
    }
    // refresh lanes nc <= lane < nc + sf: candidate nc + f is refresh slot f with its own weight
    if (lane >= nc && lane < nc + a.sf) {
        const size_t rf = (size_t)row * a.sf + (lane - nc);
        const float wf = __ldg(a.f_w + rf);
        const int32_t tf = __ldg(a.f_idx + rf);
        if (wf > 0.0f) {
            if (tf < 0 || tf >= a.n) {
                raise_index_error();
            } else {
                u = wf;
                t = tf;
            }
        }
    }
    const bool cand = u != 0.0f;

    // merge: equal targets form a group whose lowest lane (the leader) accumulates the
    // other members in ascending lane order. Only non-leading members need a shuffle.
    const unsigned cmask = __ballot_sync(FULL, cand);
    const unsigned grp = __match_any_sync(FULL, cand ? t : -1) & cmask;
    const bool leader = cand && (__ffs(grp) - 1 == lane);
    float W = u;
    unsigned followers = __ballot_sync(FULL, cand && !leader);
    while (followers) {  // warp-uniform loop, usually empty
        const int src = __ffs(followers) - 1;
        followers &= followers - 1;
        const float v = __shfl_sync(FULL, u, src);
        if (leader && ((grp >> src) & 1u)) W = __fadd_rn(W, v);
    }

    // top-s1 by (weight desc, index asc)
    unsigned key_hi = leader ? __float_as_uint(W) : 0u;
    unsigned key_lo = leader ? ~(unsigned)t : 0u;
    t_out = 0;
    w_out = 0.0f;
    for (int r = 0; r < a.s1; ++r) {
        const unsigned mh = __reduce_max_sync(FULL, key_hi);
        if (mh == 0u) break;  // warp-uniform: no candidate left, the rest stays padding
        const unsigned ml = __reduce_max_sync(FULL, key_hi == mh ? key_lo : 0u);
        if (lane == r) {
            t_out = (int32_t)~ml;
            w_out = __uint_as_float(mh);
        }
        if (key_hi == mh && key_lo == ml) key_hi = key_lo = 0u;
    }
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
