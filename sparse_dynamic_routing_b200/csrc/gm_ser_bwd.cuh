// gm_ser_bwd.cuh - backward pass of sparse edge referral (SER).
//
// "Graph Machine: Towards Better Pretraining via Edges" (ai.info summary), "Methodology in
// Plain English", referral paragraph: the hard top-s selection keeps the budget and only the
// retained weights get gradients; indices get none. With the kept merged weights
// W_r = sum over the candidates c reaching target t_r of w1[a_c] * w2[j_c][e_c], an upstream
// gradient g_r on W_r (or on ln W_r, then g_r / W_r) gives
//     dw1[row][a]  += g_r * w2[j_a][e]        for every kept candidate (a, e) of the row
//     dw2[j_a][e]  += g_r * w1[row][a]        (the second-leg row is shared by many rows)
// One warp per edge row: the referral is recomputed exactly as ser_row does (same lanes,
// same fp32 operations, same selection), each candidate lane finds its kept slot, the
// first-leg gradient of slot a is summed in ascending e by lane a (deterministic), and the
// second-leg gradients are scatter-added with fp32 atomics.
#pragma once

#include "gm_common.cuh"
#include "gm_fused_tile.cuh"
#include "gm_ser.cuh"

namespace gm {

struct SerBwdArgs {
    SerArgs f;           // legs, sizes and row map of the forward (outputs unused)
    const float *gout;   // [rows, s1]
    int grad_is_log;
    float *dw1;          // [rows, s2]
    float *dw2;          // [rows, s3]
    int accumulate;
    float *dfw;          // [rows, sf] when the forward had refresh edges
};

template <int WPB>
__global__ void __launch_bounds__(WPB * 32) ser_bwd_kernel(SerBwdArgs b)
{
    const SerArgs &a = b.f;
    const int lane = threadIdx.x & 31;
    const uint32_t row = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (row >= a.rows) return;  // warp-uniform
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    const int nc = a.s2 * a.s3;

    // ---- forward recompute (ser_row's arithmetic, keeping the per-lane candidate) ----------
    int32_t j_l = 0;
    float w1_l = 0.0f;
    if (lane < a.s2) {
        j_l = __ldg(a.a1_idx + (size_t)row * a.s2 + lane);
        w1_l = __ldg(a.a1_w + (size_t)row * a.s2 + lane);
    }
    const int ca = lane / a.s3, ce = lane - ca * a.s3;
    const int32_t j = __shfl_sync(FULL, j_l, ca);
    const float w1 = __shfl_sync(FULL, w1_l, ca);
    float u = 0.0f, w2 = 0.0f;
    int32_t t = 0;
    size_t r2 = 0;
    bool act = lane < nc && w1 > 0.0f;
    if (act && (j < 0 || j >= a.n)) {
        if (ce == 0) raise_index_error();
        act = false;
    }
    if (act) {
        r2 = ((size_t)(seq_base + (uint32_t)j) * a.k + h) * a.s3 + ce;
        w2 = __ldg(a.a2_w + r2);
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
    const bool refresh = lane >= nc && lane < nc + a.sf;  // refresh slot lane - nc
    if (refresh) {
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
    const unsigned cmask = __ballot_sync(FULL, cand);
    const unsigned grp = __match_any_sync(FULL, cand ? t : -1) & cmask;
    const bool leader = cand && (__ffs(grp) - 1 == lane);
    float W = u;
    unsigned followers = __ballot_sync(FULL, cand && !leader);
    while (followers) {
        const int src = __ffs(followers) - 1;
        followers &= followers - 1;
        const float v = __shfl_sync(FULL, u, src);
        if (leader && ((grp >> src) & 1u)) W = __fadd_rn(W, v);
    }
    unsigned key_hi = leader ? __float_as_uint(W) : 0u;
    unsigned key_lo = leader ? ~(unsigned)t : 0u;

    // ---- selection, and each candidate's kept slot ------------------------------------------
    int slot = -1;       // kept slot of this lane's candidate (-1: not kept)
    float slot_w = 0.0f;  // its merged weight
    for (int r = 0; r < a.s1; ++r) {
        const unsigned mh = __reduce_max_sync(FULL, key_hi);
        if (mh == 0u) break;  // warp-uniform
        const unsigned ml = __reduce_max_sync(FULL, key_hi == mh ? key_lo : 0u);
        if (cand && (int32_t)~ml == t) {
            slot = r;
            slot_w = __uint_as_float(mh);
        }
        if (key_hi == mh && key_lo == ml) key_hi = key_lo = 0u;
    }
    float g = 0.0f;
    if (slot >= 0) {
        g = __ldg(b.gout + (size_t)row * a.s1 + slot);
        if (b.grad_is_log) g = g / slot_w;
    }

    // ---- first leg: lane a sums its s3 candidates in ascending e --------------------------------
    const float c1 = slot >= 0 ? g * w2 : 0.0f;
    float d1 = 0.0f;
    for (int e = 0; e < a.s3; ++e) {
        const float v = __shfl_sync(FULL, c1, (lane * a.s3 + e) & 31);
        d1 += v;
    }
    if (lane < a.s2) {
        float *p = b.dw1 + (size_t)row * a.s2 + lane;
        *p = b.accumulate ? *p + d1 : d1;
    }
    // ---- second leg: scatter to the shared second-leg rows ----------------------------------------
    if (slot >= 0 && lane < nc) atomicAdd(b.dw2 + r2, g * w1);
    // ---- refresh slots: d W / d w_f = 1 -------------------------------------------------------------
    if (refresh) {
        float *p = b.dfw + (size_t)row * a.sf + (lane - nc);
        *p = b.accumulate ? *p + g : g;
    }
}

// The same backward, one thread per edge row, for small exact budgets (S2, S3; s1 <= S1M):
// the referral is recomputed in registers exactly as the fused forward's per-thread referral
// (same products, pairwise merge in ascending candidate order, arg-max selection), each
// candidate finds the kept slot of its target, the first-leg gradient of slot a is summed
// in ascending e, and the second-leg gradients are scatter-added with fp32 atomics. It
// spends a fraction of the warp-per-row kernel's instructions when the budgets are 2 or 4.
template <int S2, int S3, int S1M, int WPB>
__global__ void __launch_bounds__(WPB * 32) ser_bwd_thread_kernel(SerBwdArgs b)
{
    constexpr int NC = S2 * S3;
    const SerArgs &a = b.f;
    const uint32_t row = blockIdx.x * (WPB * 32) + threadIdx.x;
    if (row >= a.rows) return;  // no warp-wide operation below
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t j[S2];
    float w1[S2];
    ld_vec<S2>(a.a1_idx + (size_t)row * S2, j);
    ld_vec<S2>(a.a1_w + (size_t)row * S2, w1);

    int32_t ct[NC];
    float cu[NC], w2c[NC];
    size_t r2[S2];
#pragma unroll
    for (int x = 0; x < S2; ++x) {
        bool act = w1[x] > 0.0f;
        if (act && (j[x] < 0 || j[x] >= a.n)) {
            raise_index_error();
            act = false;
        }
        int32_t t2[S3];
        float w2[S3];
#pragma unroll
        for (int e = 0; e < S3; ++e) {
            t2[e] = 0;
            w2[e] = 0.0f;
        }
        r2[x] = act ? ((size_t)(seq_base + (uint32_t)j[x]) * a.k + h) * S3 : 0;
        if (act) {
            ld_vec<S3>(a.a2_idx + r2[x], t2);
            ld_vec<S3>(a.a2_w + r2[x], w2);
        }
#pragma unroll
        for (int e = 0; e < S3; ++e) {
            bool v = w2[e] > 0.0f;
            if (v && (t2[e] < 0 || t2[e] >= a.n)) {
                raise_index_error();
                v = false;
            }
            ct[x * S3 + e] = t2[e];
            cu[x * S3 + e] = v ? __fmul_rn(w1[x], w2[e]) : 0.0f;
            w2c[x * S3 + e] = w2[e];
        }
    }
    bool cand[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) cand[c] = cu[c] != 0.0f;
    merge_pairs<0, NC>(ct, cu);
    // selection (weight desc, target asc) and the upstream gradient of each kept slot
    int32_t kt[S1M];
    float kg[S1M];
#pragma unroll
    for (int r = 0; r < S1M; ++r) {
        float bw = 0.0f;
        int32_t bt = 0;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const bool better = cu[c] > bw || (cu[c] == bw && cu[c] > 0.0f && ct[c] < bt);
            bw = better ? cu[c] : bw;
            bt = better ? ct[c] : bt;
        }
#pragma unroll
        for (int c = 0; c < NC; ++c) cu[c] = (cu[c] == bw && ct[c] == bt) ? 0.0f : cu[c];
        const bool keep = r < a.s1 && bw > 0.0f;
        float g = keep ? __ldg(b.gout + (size_t)row * a.s1 + r) : 0.0f;
        if (b.grad_is_log) g = keep ? g / bw : 0.0f;
        kt[r] = keep ? bt : -1;  // -1 never equals a valid target
        kg[r] = g;
    }
    // per candidate: the gradient of its kept target (0 if cut)
    float gc[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        float g = 0.0f;
#pragma unroll
        for (int r = 0; r < S1M; ++r) g = (cand[c] && ct[c] == kt[r]) ? kg[r] : g;
        gc[c] = g;
    }
#pragma unroll
    for (int x = 0; x < S2; ++x) {
        float d1 = 0.0f;
#pragma unroll
        for (int e = 0; e < S3; ++e) d1 += gc[x * S3 + e] * w2c[x * S3 + e];
        float *p = b.dw1 + (size_t)row * S2 + x;
        *p = b.accumulate ? *p + d1 : d1;
#pragma unroll
        for (int e = 0; e < S3; ++e)
            if (gc[x * S3 + e] != 0.0f) atomicAdd(b.dw2 + r2[x] + e, gc[x * S3 + e] * w1[x]);
    }
}

}  // namespace gm
