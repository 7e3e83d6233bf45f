// gm_sea.cuh - sparse edge attention (SEA) forward and the fused SER -> SEA forward.
//
// "Graph Machine: Towards Better Pretraining via Edges" (ai.info summary), "Key
// Contributions" item 3 and "Methodology in Plain English", SEA paragraph: the edge indices
// pick which positions supply keys and values, and each entry's score is the scaled
// query-key product plus the log of the edge weight (a product of experts), followed by a
// softmax over the entries and a weighted sum of V.
//
// One warp per (b, i, KV head h). The K/V rows of the s slots are gathered once, as
// 16-byte chunks, and shared by the G query heads of the group (GQA). Scores are kept in
// the log2 domain (z2 = z * log2 e) so the softmax uses exp2. Slots go in batches of four:
// all K and V loads of a batch are issued before any is used, the batch's scores are
// computed together, and the running max / sum / accumulator are rescaled once per batch
// (never for the first batch, so s <= 4 needs no rescaling at all).
#pragma once

#include "gm_common.cuh"
#include "gm_ser.cuh"

namespace gm {

struct SeaArgs {
    const void *q, *k, *v;
    const int32_t *idx;
    const float *w;
    void *o;
    float *lse;
    int s, n, hkv;
    float scale;
    uint32_t rows;  // B * n * hkv
    RowMap map;     // heads = hkv
};

constexpr int SEA_BATCH = 4;

// Query rows of one edge row, prefetched as raw 16-byte chunks (issued before the edges are
// known so the load overlaps the edge fetch / the referral step).
template <typename T, int D, int G>
__device__ __forceinline__ void load_q(const void *q, uint32_t row, int lane, uint4 (&qraw)[Geom<T, D, G>::NI])
{
    using Gm = Geom<T, D, G>;
    const int c = lane % Gm::C, seg = lane / Gm::C;
#pragma unroll
    for (int it = 0; it < Gm::NI; ++it) {
        const int g = it * Gm::RPI + seg;
        qraw[it] = make_uint4(0, 0, 0, 0);
        if (g < G)
            qraw[it] = ld16_stream(static_cast<const T *>(q) + ((size_t)row * G + g) * D + c * Gm::VEC);
    }
}

// Attention of one edge row. Lane j < s holds slot j's (t_l, w_l); other lanes hold w = 0.
template <typename T, int D, int G>
__device__ __forceinline__ void sea_row(const SeaArgs &a, uint32_t row, uint32_t seq_base, uint32_t h,
                                        int lane, int32_t t_l, float w_l,
                                        const uint4 (&qraw)[Geom<T, D, G>::NI])
{
    using Gm = Geom<T, D, G>;
    constexpr int VEC = Gm::VEC, NI = Gm::NI, C = Gm::C, RPI = Gm::RPI;
    const int c = lane % C, seg = lane / C;
    const T *K = static_cast<const T *>(a.k);
    const T *V = static_cast<const T *>(a.v);
    const float sl2 = a.scale * LOG2E;

    float2 q2[NI][VEC / 2];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        float f[VEC];
        unpack<T>(qraw[it], f);
#pragma unroll
        for (int x = 0; x < VEC / 2; ++x) q2[it][x] = make_float2(f[2 * x], f[2 * x + 1]);
    }

    float m[NI], l[NI], acc[NI][VEC];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        m[it] = -INFINITY;
        l[it] = 0.0f;
#pragma unroll
        for (int x = 0; x < VEC; ++x) acc[it][x] = 0.0f;
    }

    for (int j0 = 0; j0 < a.s; j0 += SEA_BATCH) {
        bool on[SEA_BATCH];
        float lw2[SEA_BATCH];
        uint4 kr[SEA_BATCH], vr[SEA_BATCH];
        bool any = false;
#pragma unroll
        for (int jj = 0; jj < SEA_BATCH; ++jj) {
            const int j = j0 + jj;
            const int32_t t = __shfl_sync(FULL, t_l, j & 31);
            const float w = __shfl_sync(FULL, w_l, j & 31);
            on[jj] = j < a.s && w > 0.0f;  // warp-uniform
            if (on[jj] && (t < 0 || t >= a.n)) {
                if (lane == 0) raise_index_error();
                on[jj] = false;
            }
            lw2[jj] = lg2(w);
            kr[jj] = vr[jj] = make_uint4(0, 0, 0, 0);
            if (on[jj]) {
                const size_t off = ((size_t)(seq_base + (uint32_t)t) * a.hkv + h) * D + c * VEC;
                kr[jj] = ld16(K + off);
                vr[jj] = ld16(V + off);
            }
            any |= on[jj];
        }
        if (!any) continue;  // warp-uniform

        float z[NI][SEA_BATCH];
#pragma unroll
        for (int jj = 0; jj < SEA_BATCH; ++jj) {
            float kf[VEC];
            unpack<T>(kr[jj], kf);
#pragma unroll
            for (int it = 0; it < NI; ++it) {
                const float dot = chunk_dot<VEC / 2>(q2[it], kf);
                z[it][jj] = on[jj] ? fmaf(seg_sum<C>(dot), sl2, lw2[jj]) : -INFINITY;
            }
        }
#pragma unroll
        for (int it = 0; it < NI; ++it) {
            float mb = z[it][0];
#pragma unroll
            for (int jj = 1; jj < SEA_BATCH; ++jj) mb = fmaxf(mb, z[it][jj]);
            const float mn = fmaxf(m[it], mb);  // finite: the batch has an active slot
            float p[SEA_BATCH];
            float ps = 0.0f;
#pragma unroll
            for (int jj = 0; jj < SEA_BATCH; ++jj) {
                p[jj] = ex2(z[it][jj] - mn);  // 0 for inactive slots (z = -inf)
                ps += p[jj];
            }
            if (j0 > 0) {  // rescale what earlier batches accumulated
                const float alpha = ex2(m[it] - mn);
                l[it] *= alpha;
#pragma unroll
                for (int x = 0; x < VEC; ++x) acc[it][x] *= alpha;
            }
            l[it] += ps;
            m[it] = mn;
#pragma unroll
            for (int jj = 0; jj < SEA_BATCH; ++jj) {
                if (!on[jj]) continue;  // warp-uniform
                float vf[VEC];
                unpack<T>(vr[jj], vf);
#pragma unroll
                for (int x = 0; x < VEC; ++x) acc[it][x] = fmaf(p[jj], vf[x], acc[it][x]);
            }
        }
    }

    T *O = static_cast<T *>(a.o);
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        const int g = it * RPI + seg;
        if (g >= G) continue;
        const bool nonempty = l[it] > 0.0f;
        const float inv = nonempty ? __frcp_rn(l[it]) : 0.0f;
        float of[VEC];
#pragma unroll
        for (int x = 0; x < VEC; ++x) of[x] = acc[it][x] * inv;
        *reinterpret_cast<uint4 *>(O + ((size_t)row * G + g) * D + c * VEC) = pack<T>(of);
        if (a.lse != nullptr && c == 0)
            a.lse[(size_t)row * G + g] = nonempty ? (m[it] + lg2(l[it])) * LN2 : -INFINITY;
    }
}

template <typename T, int D, int G, int WPB>
__global__ void __launch_bounds__(WPB * 32, GM_FWD_MINB) sea_fwd_kernel(SeaArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t row = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (row >= a.rows) return;  // warp-uniform
    uint4 qraw[Geom<T, D, G>::NI];
    load_q<T, D, G>(a.q, row, lane, qraw);
    int32_t t_l = 0;
    float w_l = 0.0f;
    if (lane < a.s) {
        t_l = __ldg(a.idx + (size_t)row * a.s + lane);
        w_l = __ldg(a.w + (size_t)row * a.s + lane);
    }
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    sea_row<T, D, G>(a, row, seq_base, h, lane, t_l, w_l, qraw);
}

// Fused SER -> SEA: the referral result stays in registers (lane r holds slot r) and feeds
// the attention directly; it is stored once for the next layer and never read back.
template <typename T, int D, int G, int WPB>
__global__ void __launch_bounds__(WPB * 32, GM_FWD_MINB) ser_sea_fwd_kernel(SerArgs sa, SeaArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint32_t row = blockIdx.x * WPB + (threadIdx.x >> 5);
    if (row >= a.rows) return;  // warp-uniform
    uint4 qraw[Geom<T, D, G>::NI];
    load_q<T, D, G>(a.q, row, lane, qraw);
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t t_l;
    float w_l;
    ser_row(sa, row, seq_base, h, lane, t_l, w_l);
    if (sa.out_idx != nullptr && lane < sa.s1) {
        sa.out_idx[(size_t)row * sa.s1 + lane] = t_l;
        sa.out_w[(size_t)row * sa.s1 + lane] = w_l;
    }
    sea_row<T, D, G>(a, row, seq_base, h, lane, t_l, w_l, qraw);
}

}  // namespace gm
