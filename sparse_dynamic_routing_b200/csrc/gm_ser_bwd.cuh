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

// Backward of one referral step of one row (the candidates, merge and selection of
// refer_candidates / refer_merge / refer_select, recomputed). Lane r < s_out holds g_r, the
// upstream gradient of kept slot r (of ln W_r when grad_is_log). Returns, on lane a < s_in,
// the gradient of first-leg slot a (its candidates' terms summed in ascending e), scatter-adds
// the second-leg gradients into dleg with fp32 atomics, and gives refresh lanes g of their
// target in g_refresh.
__device__ __forceinline__ float refer_step_backward(const ReferCand &c, unsigned key_hi,
                                                     unsigned key_lo, int s_in, int s3, int s_out,
                                                     float g_l, int grad_is_log, float *dleg,
                                                     int lane, float &g_refresh)
{
    int32_t t_out;
    float w_out;
    int slot;
    float slot_w;
    refer_select(c, key_hi, key_lo, s_out, lane, t_out, w_out, slot, slot_w);
    const float gs = __shfl_sync(FULL, g_l, slot >= 0 ? slot : 0);
    float g = 0.0f;
    if (slot >= 0) g = grad_is_log ? gs / slot_w : gs;
    // first leg: lane a sums its s3 candidates in ascending e (each product and add rounded
    // once, as in ser_bwd_thread_kernel, so both kernels give the same bits)
    const float c1 = slot >= 0 ? __fmul_rn(g, c.w2) : 0.0f;
    float d1 = 0.0f;
    for (int e = 0; e < s3; ++e) {
        const float v = __shfl_sync(FULL, c1, (lane * s3 + e) & 31);
        d1 = __fadd_rn(d1, v);
    }
    // second leg: scatter to the shared second-leg rows
    if (slot >= 0 && c.path) atomicAdd(dleg + c.r2, __fmul_rn(g, c.w1));
    g_refresh = c.refresh ? g : 0.0f;
    return lane < s_in ? d1 : 0.0f;
}

template <int WPB>
__global__ void __launch_bounds__(WPB * 32) ser_bwd_kernel(SerBwdArgs b)
{
    pdl_wait();  // the zeroed leg gradients (launched after the zero-fill)
    const SerArgs &a = b.f;
    const int lane = threadIdx.x & 31;
    const uint32_t row = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (row >= a.rows) return;  // warp-uniform
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t j_l = 0;
    float w1_l = 0.0f, g_l = 0.0f;
    if (lane < a.s2) {
        j_l = __ldg(a.a1_idx + (size_t)row * a.s2 + lane);
        w1_l = __ldg(a.a1_w + (size_t)row * a.s2 + lane);
    }
    if (lane < a.s1) g_l = __ldg(b.gout + (size_t)row * a.s1 + lane);
    const ReferCand c = refer_candidates(j_l, w1_l, a.s2, a.a2_idx, a.a2_w, a.s3, a.f_idx, a.f_w,
                                         a.sf, row, a.n, a.k, seq_base, h, lane);
    unsigned key_hi, key_lo;
    refer_merge(c, lane, key_hi, key_lo);
    float g_refresh;
    const float d1 = refer_step_backward(c, key_hi, key_lo, a.s2, a.s3, a.s1, g_l, b.grad_is_log,
                                         b.dw2, lane, g_refresh);
    if (lane < a.s2) {
        float *p = b.dw1 + (size_t)row * a.s2 + lane;
        *p = b.accumulate ? *p + d1 : d1;
    }
    // refresh slots: d W / d w_f = 1
    if (c.refresh) {
        float *p = b.dfw + (size_t)row * a.sf + (lane - a.s2 * a.s3);
        *p = b.accumulate ? *p + g_refresh : g_refresh;
    }
}

// Backward of one referral step of one row by one thread. The step's candidates are
// recomputed from the first leg (j, w1) [S_IN] and the second-leg rows at (leg_idx, leg_w)
// [S3 each] (then the row's SF refresh slots when SF > 0), merged and selected exactly as
// refer_thread does (the kept set, s_keep <= S_OUT slots); with g[r] the upstream gradient of
// kept slot r (of ln W_r when is_log), each candidate reaching a kept target passes it on:
// d1[a] = sum over e of g * w2 (ascending e, each product and add rounded once), g * w1 is
// added to the second-leg weight (fp32 atomics into dleg), and refresh slot f gets gf[f] = g.
template <int S_IN, int S3, int S_OUT, int SF = 0>
__device__ __forceinline__ void refer_thread_backward(const SerArgs &a, uint32_t row, uint32_t seq_base,
                                                      uint32_t h, const int32_t (&j)[S_IN],
                                                      const float (&w1)[S_IN], const int32_t *leg_idx,
                                                      const float *leg_w, int s_keep,
                                                      const float (&g)[S_OUT], bool is_log, float *dleg,
                                                      float (&d1)[S_IN], float (&gf)[SF > 0 ? SF : 1])
{
    constexpr int NP2 = S_IN * S3, NC = NP2 + SF;  // SF refresh slots after the paths
    int32_t ct[NC];
    float cu[NC], w2c[NC];
    size_t r2[S_IN];
#pragma unroll
    for (int x = 0; x < S_IN; ++x) {
        bool act = w1[x] > 0.0f;
        if (act && (uint32_t)j[x] >= (uint32_t)a.n) {
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
            ld_vec<S3>(leg_idx + r2[x], t2);
            ld_vec<S3>(leg_w + r2[x], w2);
        }
#pragma unroll
        for (int e = 0; e < S3; ++e) {
            bool v = w2[e] > 0.0f;
            if (v && (uint32_t)t2[e] >= (uint32_t)a.n) {
                raise_index_error();
                v = false;
            }
            const float u = v ? __fmul_rn(w1[x], w2[e]) : 0.0f;
            ct[x * S3 + e] = u != 0.0f ? t2[e] : no_target(x * S3 + e);
            cu[x * S3 + e] = u;
            w2c[x * S3 + e] = w2[e];
        }
    }
    if constexpr (SF > 0) {
        int32_t tf[SF];
        float wf[SF];
        ld_vec<SF>(a.f_idx + (size_t)row * SF, tf);
        ld_vec<SF>(a.f_w + (size_t)row * SF, wf);
#pragma unroll
        for (int f = 0; f < SF; ++f) {
            bool v = wf[f] > 0.0f;
            if (v && (uint32_t)tf[f] >= (uint32_t)a.n) {
                raise_index_error();
                v = false;
            }
            ct[NP2 + f] = v ? tf[f] : no_target(NP2 + f);
            cu[NP2 + f] = v ? wf[f] : 0.0f;
        }
    }
    bool cand[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) cand[c] = cu[c] != 0.0f;
    merge_pairs<0, NC>(ct, cu);
    // selection (weight desc, target asc) and the upstream gradient of each kept slot
    int32_t kt[S_OUT];
    float kg[S_OUT];
#pragma unroll
    for (int r = 0; r < S_OUT; ++r) {
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
        const bool keep = r < s_keep && bw > 0.0f;
        float gr = keep ? g[r] : 0.0f;
        if (is_log) gr = keep ? gr / bw : 0.0f;
        kt[r] = keep ? bt : -1;  // -1 never equals a valid target
        kg[r] = gr;
    }
    // per candidate: the gradient of its kept target (0 if cut)
    float gc[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        float gg = 0.0f;
#pragma unroll
        for (int r = 0; r < S_OUT; ++r) gg = (cand[c] && ct[c] == kt[r]) ? kg[r] : gg;
        gc[c] = gg;
    }
#pragma unroll
    for (int x = 0; x < S_IN; ++x) {
        float acc = 0.0f;
#pragma unroll
        for (int e = 0; e < S3; ++e) acc = __fadd_rn(acc, __fmul_rn(gc[x * S3 + e], w2c[x * S3 + e]));
        d1[x] = acc;
#pragma unroll
        for (int e = 0; e < S3; ++e)
            if (gc[x * S3 + e] != 0.0f) atomicAdd(dleg + r2[x] + e, __fmul_rn(gc[x * S3 + e], w1[x]));
    }
    if constexpr (SF > 0) {
#pragma unroll
        for (int f = 0; f < SF; ++f) gf[f] = gc[NP2 + f];
    }
}

// The same backward as ser_bwd_kernel, one thread per edge row, for small exact budgets (S2,
// S3; s1 <= S1M), through refer_thread_backward: the referral is recomputed in registers
// exactly as the fused forward's per-thread referral (same products, pairwise merge in
// ascending candidate order, selection by weight then target), and the gradients flow as in
// the warp kernel. It spends a fraction of the warp-per-row kernel's instructions when the
// budgets are 2 or 4.
//
// The dispatch picks this kernel or ser_bwd_kernel by shape and alignment alone, so the two
// must agree bit for bit: the candidate products (__fmul_rn), the merge in ascending candidate
// order (merge_pairs here and refer_thread in gm_fused_tile.cuh; __match_any_sync groups
// summed from their first lane in refer_merge), the selection (weight descending, then target
// ascending, zero weights never kept), g / W for a log-weight gradient, and the first-leg sums
// (g * w2 rounded, then added in ascending e). Only dw2, summed by atomics, varies in order.
template <int S2, int S3, int S1M, int WPB, int SF = 0>
__global__ void __launch_bounds__(WPB * 32) ser_bwd_thread_kernel(SerBwdArgs b)
{
    pdl_wait();  // the zeroed leg gradients (launched after the zero-fill)
    const SerArgs &a = b.f;
    const uint32_t row = blockIdx.x * (WPB * 32) + threadIdx.x;
    if (row >= a.rows) return;  // no warp-wide operation below
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t j[S2];
    float w1[S2];
    ld_vec<S2>(a.a1_idx + (size_t)row * S2, j);
    ld_vec<S2>(a.a1_w + (size_t)row * S2, w1);
    float g[S1M];
#pragma unroll
    for (int r = 0; r < S1M; ++r) g[r] = r < a.s1 ? __ldg(b.gout + (size_t)row * a.s1 + r) : 0.0f;
    float d1[S2], gf[SF > 0 ? SF : 1];
    refer_thread_backward<S2, S3, S1M, SF>(a, row, seq_base, h, j, w1, a.a2_idx, a.a2_w, a.s1, g,
                                           b.grad_is_log != 0, b.dw2, d1, gf);
#pragma unroll
    for (int x = 0; x < S2; ++x) {
        float *p = b.dw1 + (size_t)row * S2 + x;
        *p = b.accumulate ? *p + d1[x] : d1[x];
    }
    if constexpr (SF > 0) {  // refresh slots: d W / d w_f = 1
#pragma unroll
        for (int f = 0; f < SF; ++f) {
            float *p = b.dfw + (size_t)row * SF + f;
            *p = b.accumulate ? *p + gf[f] : gf[f];
        }
    }
}

}  // namespace gm
