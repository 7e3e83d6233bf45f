// gm_ser_chain.cuh - multi-step referral: a chain of referral steps inside one layer.
//
// "Graph Machine: Towards Better Pretraining via Edges" (ai.info summary), "Key Contributions"
// item 2: the soft sparse adjacency matrix is raised to the l-th power and the result is
// sparsified; "Main Findings", bullet on referral: models with 3 and 4 referral legs (R3,
// R4). With legs A1 (s2 slots), A2 .. Al (s3 slots each, channel h reads channel h):
//     B_1 = A1,   B_{m+1} = Sparsify(B_m A_{m+1}),   A' = B_l
// every intermediate cut to s_mid slots and the last to s1; each step is the referral of
// gm_ser.cuh (same candidates, fp32 order and selection), applied to the row's previous
// result, which the warp keeps in registers: no intermediate is written.
//
// One warp per edge row. The backward recomputes the chain, keeping each step's first leg in
// registers, then runs the steps in reverse: each step's first-leg gradient (summed in a
// fixed order) is the upstream gradient of the previous step's kept weights, and each leg's
// gradient is scatter-added with fp32 atomics. For budgets s2 = s3 = s_mid of 2 or 4 the
// backward also runs one thread per row (ser_chain_bwd_thread_kernel), with the same results
// (the per-thread referral steps agree bit for bit with the warp ones).
#pragma once

#include "gm_common.cuh"
#include "gm_ser.cuh"
#include "gm_ser_bwd.cuh"

namespace gm {

__device__ __forceinline__ const int32_t *chain_leg_idx(const SerArgs &a, int m)
{
    return m == 0 ? a.a2_idx : a.chain_idx[m - 1];
}
__device__ __forceinline__ const float *chain_leg_w(const SerArgs &a, int m)
{
    return m == 0 ? a.a2_w : a.chain_w[m - 1];
}

struct ChainBwdArgs {
    SerArgs f;
    const float *gout;                // [rows, s1]
    int grad_is_log;
    float *dw1;                       // [rows, s2]
    float *dleg[GM_MAX_CHAIN];        // [rows, s3] per leg, zeroed (or accumulated into)
    int accumulate;
};

// NL = number of legs after A1 (1 + nchain).
template <int NL, int WPB>
__global__ void __launch_bounds__(WPB * 32) ser_chain_kernel(SerArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t row = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (row >= a.rows) return;  // warp-uniform
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t j_l = 0;
    float w_l = 0.0f;
    if (lane < a.s2) {
        j_l = __ldg(a.a1_idx + (size_t)row * a.s2 + lane);
        w_l = __ldg(a.a1_w + (size_t)row * a.s2 + lane);
    }
    int s_in = a.s2;
#pragma unroll
    for (int m = 0; m < NL; ++m) {
        const int s_out = m == NL - 1 ? a.s1 : a.s_mid;
        const ReferCand c = refer_candidates(j_l, w_l, s_in, chain_leg_idx(a, m), chain_leg_w(a, m),
                                             a.s3, nullptr, nullptr, 0, row, a.n, a.k, seq_base, h,
                                             lane);
        unsigned key_hi, key_lo;
        refer_merge(c, lane, key_hi, key_lo);
        int slot;
        float slot_w;
        refer_select(c, key_hi, key_lo, s_out, lane, j_l, w_l, slot, slot_w);
        s_in = s_out;
    }
    if (lane < a.s1) {
        a.out_idx[(size_t)row * a.s1 + lane] = j_l;
        a.out_w[(size_t)row * a.s1 + lane] = w_l;
    }
}

template <int NL, int WPB>
__global__ void __launch_bounds__(WPB * 32) ser_chain_bwd_kernel(ChainBwdArgs b)
{
    const SerArgs &a = b.f;
    const int lane = threadIdx.x & 31;
    const uint32_t row = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (row >= a.rows) return;  // warp-uniform
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    // forward: the first leg of every step, held by the lanes
    int32_t jm[NL];
    float wm[NL];
    jm[0] = 0;
    wm[0] = 0.0f;
    if (lane < a.s2) {
        jm[0] = __ldg(a.a1_idx + (size_t)row * a.s2 + lane);
        wm[0] = __ldg(a.a1_w + (size_t)row * a.s2 + lane);
    }
#pragma unroll
    for (int m = 0; m + 1 < NL; ++m) {
        const int s_in = m == 0 ? a.s2 : a.s_mid;
        const ReferCand c = refer_candidates(jm[m], wm[m], s_in, chain_leg_idx(a, m), chain_leg_w(a, m),
                                             a.s3, nullptr, nullptr, 0, row, a.n, a.k, seq_base, h,
                                             lane);
        unsigned key_hi, key_lo;
        refer_merge(c, lane, key_hi, key_lo);
        int slot;
        float slot_w;
        refer_select(c, key_hi, key_lo, a.s_mid, lane, jm[m + 1], wm[m + 1], slot, slot_w);
    }
    // backward through the steps
    float g_l = lane < a.s1 ? __ldg(b.gout + (size_t)row * a.s1 + lane) : 0.0f;
#pragma unroll
    for (int m = NL - 1; m >= 0; --m) {
        const int s_in = m == 0 ? a.s2 : a.s_mid;
        const int s_out = m == NL - 1 ? a.s1 : a.s_mid;
        const ReferCand c = refer_candidates(jm[m], wm[m], s_in, chain_leg_idx(a, m), chain_leg_w(a, m),
                                             a.s3, nullptr, nullptr, 0, row, a.n, a.k, seq_base, h,
                                             lane);
        unsigned key_hi, key_lo;
        refer_merge(c, lane, key_hi, key_lo);
        float g_refresh;
        g_l = refer_step_backward(c, key_hi, key_lo, s_in, a.s3, s_out, g_l,
                                  m == NL - 1 ? b.grad_is_log : 0, b.dleg[m], lane, g_refresh);
    }
    if (lane < a.s2) {
        float *p = b.dw1 + (size_t)row * a.s2 + lane;
        *p = b.accumulate ? *p + g_l : g_l;
    }
}

// The chain backward one thread per edge row, for budgets S = s2 = s3 = s_mid in {2, 4} and
// s1 <= 4: the chain is recomputed step by step with refer_thread (each step's first leg kept
// in registers), then refer_thread_backward runs the steps in reverse, the first-leg gradient
// of step m being the upstream gradient of step m - 1's kept weights.
template <int S, int NL, int WPB>
__global__ void __launch_bounds__(WPB * 32) ser_chain_bwd_thread_kernel(ChainBwdArgs b)
{
    constexpr int S1M = 4;
    const SerArgs &a = b.f;
    const uint32_t row = blockIdx.x * (WPB * 32) + threadIdx.x;
    if (row >= a.rows) return;  // no warp-wide operation below
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t jm[NL][S];
    float wm[NL][S];
    ld_vec<S>(a.a1_idx + (size_t)row * S, jm[0]);
    ld_vec<S>(a.a1_w + (size_t)row * S, wm[0]);
#pragma unroll
    for (int m = 0; m + 1 < NL; ++m)
        refer_thread<S, S, S>(a, row, seq_base, h, jm[m], wm[m], chain_leg_idx(a, m), chain_leg_w(a, m), S,
                              jm[m + 1], wm[m + 1]);
    float g1[S1M];
#pragma unroll
    for (int r = 0; r < S1M; ++r) g1[r] = r < a.s1 ? __ldg(b.gout + (size_t)row * a.s1 + r) : 0.0f;
    float d1[S], unused[1];
    refer_thread_backward<S, S, S1M>(a, row, seq_base, h, jm[NL - 1], wm[NL - 1], chain_leg_idx(a, NL - 1),
                                     chain_leg_w(a, NL - 1), a.s1, g1, b.grad_is_log != 0, b.dleg[NL - 1],
                                     d1, unused);
#pragma unroll
    for (int m = NL - 2; m >= 0; --m) {
        float g[S];
#pragma unroll
        for (int x = 0; x < S; ++x) g[x] = d1[x];
        refer_thread_backward<S, S, S>(a, row, seq_base, h, jm[m], wm[m], chain_leg_idx(a, m), chain_leg_w(a, m),
                                       S, g, false, b.dleg[m], d1, unused);
    }
#pragma unroll
    for (int x = 0; x < S; ++x) {
        float *p = b.dw1 + (size_t)row * S + x;
        *p = b.accumulate ? *p + d1[x] : d1[x];
    }
}

}  // namespace gm
