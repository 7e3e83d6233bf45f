// gm_sea_bwd.cuh - backward pass of sparse edge attention.
//
// The derivative of the SEA forward ("Graph Machine: Towards Better Pretraining via Edges",
// ai.info summary, "Key Contributions" item 3); indices get no gradient and the log edge
// weights do ("Methodology in Plain English", referral paragraph).
//
// One warp per (b, i, KV head h), recomputing the forward from q, K, V and the edges: the
// K rows are read anyway for dq, so no forward state (o, lse) is read back. With
// e_j = exp(z_j - m), l = sum e_j and dp_j = <dO, V[t_j]>:
//   D   = sum_j p_j dp_j                    = (sum_j e_j dp_j) / l
//   dq  = scale * sum_j p_j (dp_j - D) K_j  = scale / l * (sum_j e_j dp_j K_j - D sum_j e_j K_j)
// so one streaming pass over the slots (pass A, batches of four with an online max as in
// the forward) yields dq; the per-slot scores z_j and dp_j go to shared memory, and pass B
// turns them into dz_j = p_j (dp_j - D) for the scatter-adds dK[t_j] += scale dz_j q and
// dV[t_j] += p_j dO (16-byte vector fp32 atomics, summed over the query-head group first)
// and for dlogw_j = sum over the group of dz_j.
//
// When the group's rows exactly fill the warp in two segments (G = 2, C = 16: bf16
// head_dim 128), the segments split the scatter: segment 0 adds dK, segment 1 adds dV, and
// each fetches the other segment's q (resp. dO) chunk once per row, so a slot costs two
// shuffles instead of a cross-segment reduction of every element.
#pragma once

#include "gm_common.cuh"

namespace gm {

struct SeaBwdArgs {
    const void *q, *k, *v, *dout;
    const int32_t *idx;
    const float *w;
    float *dq, *dk, *dv, *dlogw;
    // gather mode only (see gm_bwd_gather.cuh): each edge's rank inside its target's bucket,
    // the bucket offsets, and the sorted record array; unused by the atomic path
    const int32_t *rank;
    const int32_t *off;
    int32_t *srec;
    int s, n, hkv;
    float scale;
    int accumulate;
    uint32_t rows;  // B * n * hkv
    RowMap map;     // heads = hkv
    // fused referral backward (tile row pass with SB > 0): A' = Sparsify_s(A1 A2) was the
    // referral's output; the gradient of ln A'.w that this backward computes flows on to the
    // legs' weights (dw1 [rows, SB] stored, dw2 [rows, SB] scatter-added)
    const int32_t *a1_idx, *a2_idx;
    const float *a1_w, *a2_w;
    float *dw1, *dw2;
};

__device__ __forceinline__ void red_add4(float *p, float a, float b, float c, float d)
{
    atomicAdd(reinterpret_cast<float4 *>(p), make_float4(a, b, c, d));
}

template <typename T, int D, int G, int WPB>
__global__ void __launch_bounds__(WPB * 32, GM_BWD_MINB) sea_bwd_kernel(SeaBwdArgs a)
{
    using Gm = Geom<T, D, G>;
    constexpr int VEC = Gm::VEC, NI = Gm::NI, C = Gm::C, RPI = Gm::RPI;
    constexpr bool PAIR = (G == 2 && RPI == 2 && NI == 1);  // the two-segment split
    __shared__ float sh_z[WPB][G][32];
    __shared__ float sh_dp[WPB][G][32];

    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t row = blockIdx.x * WPB + wid;
    if (row >= a.rows) return;  // warp-uniform
    const int c = lane % C, seg = lane / C;
    const T *Q = static_cast<const T *>(a.q);
    const T *K = static_cast<const T *>(a.k);
    const T *V = static_cast<const T *>(a.v);
    const T *GO = static_cast<const T *>(a.dout);
    const float sl2 = a.scale * LOG2E;

    uint4 qr[NI], gr[NI];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        const int g = it * RPI + seg;
        qr[it] = gr[it] = make_uint4(0, 0, 0, 0);
        if (g < G) {
            qr[it] = ld16_stream(Q + ((size_t)row * G + g) * D + c * VEC);
            gr[it] = ld16_stream(GO + ((size_t)row * G + g) * D + c * VEC);
        }
    }
    int32_t t_l = 0;
    float w_l = 0.0f;
    if (lane < a.s) {
        t_l = __ldg(a.idx + (size_t)row * a.s + lane);
        w_l = __ldg(a.w + (size_t)row * a.s + lane);
    }
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    float qf[NI][VEC], gf[NI][VEC];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        unpack<T>(qr[it], qf[it]);
        unpack<T>(gr[it], gf[it]);
    }

    // ---- pass A: scores, softmax statistics and the two dq accumulators ------------------
    float m[NI], l[NI], sdp[NI], Ak[NI][VEC], Bk[NI][VEC];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        m[it] = -INFINITY;
        l[it] = sdp[it] = 0.0f;
#pragma unroll
        for (int x = 0; x < VEC; ++x) Ak[it][x] = Bk[it][x] = 0.0f;
    }
    unsigned active = 0;  // bit j: slot j active (warp-uniform)
    for (int j0 = 0; j0 < a.s; j0 += 4) {
        bool on[4];
        float lw2[4];
        uint4 kr[4], vr[4];
        bool any = false;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = j0 + jj;
            const int32_t t = __shfl_sync(FULL, t_l, j & 31);
            const float w = __shfl_sync(FULL, w_l, j & 31);
            on[jj] = j < a.s && w > 0.0f;
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
                active |= 1u << j;
            }
            any |= on[jj];
        }
        if (!any) continue;  // warp-uniform

        float z[NI][4], dp[NI][4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            float kf[VEC], vf[VEC];
            unpack<T>(kr[jj], kf);
            unpack<T>(vr[jj], vf);
#pragma unroll
            for (int it = 0; it < NI; ++it) {
                float sk = 0.0f, sv = 0.0f;
#pragma unroll
                for (int x = 0; x < VEC; ++x) {
                    sk = fmaf(qf[it][x], kf[x], sk);
                    sv = fmaf(gf[it][x], vf[x], sv);
                }
                z[it][jj] = -INFINITY;
                dp[it][jj] = 0.0f;
                if (on[jj]) {  // warp-uniform
                    z[it][jj] = fmaf(seg_sum<C>(sk), sl2, lw2[jj]);
                    dp[it][jj] = seg_sum<C>(sv);
                    const int g = it * RPI + seg;
                    if (c == 0 && g < G) {
                        sh_z[wid][g][j0 + jj] = z[it][jj];
                        sh_dp[wid][g][j0 + jj] = dp[it][jj];
                    }
                }
            }
        }
#pragma unroll
        for (int it = 0; it < NI; ++it) {
            float mb = z[it][0];
#pragma unroll
            for (int jj = 1; jj < 4; ++jj) mb = fmaxf(mb, z[it][jj]);
            const float mn = fmaxf(m[it], mb);
            if (j0 > 0) {
                const float alpha = ex2(m[it] - mn);
                l[it] *= alpha;
                sdp[it] *= alpha;
#pragma unroll
                for (int x = 0; x < VEC; ++x) {
                    Ak[it][x] *= alpha;
                    Bk[it][x] *= alpha;
                }
            }
            m[it] = mn;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                if (!on[jj]) continue;  // warp-uniform
                float kf[VEC];
                unpack<T>(kr[jj], kf);
                const float e = ex2(z[it][jj] - mn);
                const float edp = e * dp[it][jj];
                l[it] += e;
                sdp[it] += edp;
#pragma unroll
                for (int x = 0; x < VEC; ++x) {
                    Ak[it][x] = fmaf(edp, kf[x], Ak[it][x]);
                    Bk[it][x] = fmaf(e, kf[x], Bk[it][x]);
                }
            }
        }
    }

    // dq = scale / l * (Ak - D Bk), D = sdp / l
    float Dd[NI], inv[NI];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        const int g = it * RPI + seg;
        inv[it] = l[it] > 0.0f ? __frcp_rn(l[it]) : 0.0f;
        Dd[it] = sdp[it] * inv[it];
        if (g >= G) continue;
        float *dqp = a.dq + ((size_t)row * G + g) * D + c * VEC;
        const float f = a.scale * inv[it];
#pragma unroll
        for (int x = 0; x < VEC; x += 4) {
            float4 r;
            r.x = f * fmaf(-Dd[it], Bk[it][x + 0], Ak[it][x + 0]);
            r.y = f * fmaf(-Dd[it], Bk[it][x + 1], Ak[it][x + 1]);
            r.z = f * fmaf(-Dd[it], Bk[it][x + 2], Ak[it][x + 2]);
            r.w = f * fmaf(-Dd[it], Bk[it][x + 3], Ak[it][x + 3]);
            if (a.accumulate) {
                const float4 o = *reinterpret_cast<const float4 *>(dqp + x);
                r.x += o.x; r.y += o.y; r.z += o.z; r.w += o.w;
            }
            *reinterpret_cast<float4 *>(dqp + x) = r;
        }
    }
    __syncwarp();

    // ---- pass B: per-slot gradients, summed over the query-head group, scattered ---------
    float my_dlw = 0.0f;
    if constexpr (PAIR) {
        // segment 0 needs the other head's q, segment 1 the other head's dO
        float xf[VEC];
        {
            const uint4 send = seg == 0 ? gr[0] : qr[0];
            uint4 recv;
            recv.x = __shfl_xor_sync(FULL, send.x, C);
            recv.y = __shfl_xor_sync(FULL, send.y, C);
            recv.z = __shfl_xor_sync(FULL, send.z, C);
            recv.w = __shfl_xor_sync(FULL, send.w, C);
            unpack<T>(recv, xf);
        }
        float ownf[VEC];
#pragma unroll
        for (int x = 0; x < VEC; ++x) ownf[x] = seg == 0 ? qf[0][x] : gf[0][x];
        for (int j = 0; j < a.s; ++j) {
            if (!((active >> j) & 1u)) continue;  // warp-uniform
            const int32_t t = __shfl_sync(FULL, t_l, j);
            const float p = ex2(sh_z[wid][seg][j] - m[0]) * inv[0];
            const float dz = p * (sh_dp[wid][seg][j] - Dd[0]);
            // segment 0 gets the other head's dz, segment 1 the other head's p
            const float other = __shfl_xor_sync(FULL, seg == 0 ? p : dz, C);
            const float dz_sum = dz + __shfl_xor_sync(FULL, dz, C);
            if (lane == j) my_dlw = dz_sum;
            // seg 0: scale * (dz_own q_own + dz_other q_other); seg 1: p_own dO_own + p_other dO_other
            const float fo = seg == 0 ? a.scale * dz : p;
            const float fx = seg == 0 ? a.scale * other : other;
            float part[VEC];
#pragma unroll
            for (int x = 0; x < VEC; ++x) part[x] = fmaf(fo, ownf[x], fx * xf[x]);
            float *dst = (seg == 0 ? a.dk : a.dv) +
                         ((size_t)(seq_base + (uint32_t)t) * a.hkv + h) * D + c * VEC;
#pragma unroll
            for (int x = 0; x < VEC; x += 4) red_add4(dst + x, part[x], part[x + 1], part[x + 2], part[x + 3]);
        }
    } else {
        for (int j = 0; j < a.s; ++j) {
            if (!((active >> j) & 1u)) continue;  // warp-uniform
            const int32_t t = __shfl_sync(FULL, t_l, j);
            float pk[VEC], pv[VEC];
#pragma unroll
            for (int x = 0; x < VEC; ++x) pk[x] = pv[x] = 0.0f;
            float dzs = 0.0f;
#pragma unroll
            for (int it = 0; it < NI; ++it) {
                const int g = it * RPI + seg;
                if (g >= G) continue;
                const float p = ex2(sh_z[wid][g][j] - m[it]) * inv[it];
                const float dz = p * (sh_dp[wid][g][j] - Dd[it]);
                dzs += dz;
                const float sdz = a.scale * dz;
#pragma unroll
                for (int x = 0; x < VEC; ++x) {
                    pk[x] = fmaf(sdz, qf[it][x], pk[x]);
                    pv[x] = fmaf(p, gf[it][x], pv[x]);
                }
            }
            // each segment holds a partial over its query heads: combine across segments
#pragma unroll
            for (int x = 0; x < VEC; ++x) {
                pk[x] = cross_seg_sum<C>(pk[x]);
                pv[x] = cross_seg_sum<C>(pv[x]);
            }
            // dz is uniform inside a segment: count it once per segment (lane c == 0)
            float part = c == 0 ? dzs : 0.0f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(FULL, part, off);
            if (lane == j) my_dlw = part;

            const size_t off = ((size_t)(seq_base + (uint32_t)t) * a.hkv + h) * D + c * VEC;
            if (RPI == 1 || seg == 0) {
#pragma unroll
                for (int x = 0; x < VEC; x += 4)
                    red_add4(a.dk + off + x, pk[x], pk[x + 1], pk[x + 2], pk[x + 3]);
            }
            if (RPI == 1 || seg == 1) {
#pragma unroll
                for (int x = 0; x < VEC; x += 4)
                    red_add4(a.dv + off + x, pv[x], pv[x + 1], pv[x + 2], pv[x + 3]);
            }
        }
    }
    if (lane < a.s) {
        float *p = a.dlogw + (size_t)row * a.s + lane;
        *p = a.accumulate ? *p + my_dlw : my_dlw;
    }
}

// dk = dv = 0 before a non-accumulating backward (count = elements of each, multiple of 4).
__global__ void zero2_kernel(float4 *a, float4 *b, int64_t count4)
{
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count4;
         i += (int64_t)gridDim.x * blockDim.x) {
        a[i] = z;
        b[i] = z;
    }
}

}  // namespace gm
