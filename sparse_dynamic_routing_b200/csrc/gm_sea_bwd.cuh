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
// so one streaming pass over the slots (pass A, online max as in the forward) yields dq; the
// per-slot scores z_j and dp_j go to shared memory, and pass B turns them into
// dz_j = p_j (dp_j - D) for the scatter-adds dK[t_j] += scale dz_j q and dV[t_j] += p_j dO
// (16-byte vector fp32 atomics, summed over the query-head group first) and for
// dlogw_j = sum over the group of dz_j.
#pragma once

#include "gm_common.cuh"

namespace gm {

struct SeaBwdArgs {
    const void *q, *k, *v, *dout;
    const int32_t *idx;
    const float *w;
    float *dq, *dk, *dv, *dlogw;
    int s, n, hkv;
    float scale;
    int accumulate;
    int64_t rows;  // B * n * hkv
};

__device__ __forceinline__ void red_add4(float *p, float a, float b, float c, float d)
{
    atomicAdd(reinterpret_cast<float4 *>(p), make_float4(a, b, c, d));
}

template <typename T, int D, int G, int WPB>
__global__ void __launch_bounds__(WPB * 32) sea_bwd_kernel(SeaBwdArgs a)
{
    using Gm = Geom<T, D, G>;
    constexpr int VEC = Gm::VEC, NI = Gm::NI, C = Gm::C, RPI = Gm::RPI;
    __shared__ float sh_z[WPB][G][32];
    __shared__ float sh_dp[WPB][G][32];

    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * WPB + wid;
    if (row >= a.rows) return;  // warp-uniform
    const int c = lane % C, seg = lane / C;
    const int h = (int)(row % a.hkv);
    const int64_t seq_base = (row / a.hkv) / a.n * a.n;
    const T *Q = static_cast<const T *>(a.q);
    const T *K = static_cast<const T *>(a.k);
    const T *V = static_cast<const T *>(a.v);
    const T *GO = static_cast<const T *>(a.dout);
    const float sl2 = a.scale * LOG2E;

    float qf[NI][VEC], gf[NI][VEC];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        const int g = it * RPI + seg;
        uint4 qr = make_uint4(0, 0, 0, 0), gr = make_uint4(0, 0, 0, 0);
        if (g < G) {
            qr = ld16_stream(Q + (row * G + g) * D + c * VEC);
            gr = ld16_stream(GO + (row * G + g) * D + c * VEC);
        }
        unpack<T>(qr, qf[it]);
        unpack<T>(gr, gf[it]);
    }
    int32_t t_l = 0;
    float w_l = 0.0f;
    if (lane < a.s) {
        t_l = __ldg(a.idx + row * a.s + lane);
        w_l = __ldg(a.w + row * a.s + lane);
    }

    // ---- pass A: scores, online softmax statistics and the two dq accumulators ----------
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
            lw2[jj] = on[jj] ? log2f(w) : 0.0f;
            kr[jj] = vr[jj] = make_uint4(0, 0, 0, 0);
            if (on[jj]) {
                const int64_t off = ((seq_base + t) * a.hkv + h) * D + c * VEC;
                kr[jj] = ld16(K + off);
                vr[jj] = ld16(V + off);
                active |= 1u << j;
            }
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            if (!on[jj]) continue;  // warp-uniform
            float kf[VEC], vf[VEC];
            unpack<T>(kr[jj], kf);
            unpack<T>(vr[jj], vf);
#pragma unroll
            for (int it = 0; it < NI; ++it) {
                float dk = 0.0f, dv = 0.0f;
#pragma unroll
                for (int x = 0; x < VEC; ++x) {
                    dk = fmaf(qf[it][x], kf[x], dk);
                    dv = fmaf(gf[it][x], vf[x], dv);
                }
                const float z = seg_sum<C>(dk) * sl2 + lw2[jj];
                const float dp = seg_sum<C>(dv);
                const int g = it * RPI + seg;
                if (c == 0 && g < G) {
                    sh_z[wid][g][j0 + jj] = z;
                    sh_dp[wid][g][j0 + jj] = dp;
                }
                const float mn = fmaxf(m[it], z);
                const float alpha = exp2f(m[it] - mn);
                const float e = exp2f(z - mn);
                l[it] = l[it] * alpha + e;
                sdp[it] = sdp[it] * alpha + e * dp;
                const float edp = e * dp;
#pragma unroll
                for (int x = 0; x < VEC; ++x) {
                    Ak[it][x] = fmaf(edp, kf[x], Ak[it][x] * alpha);
                    Bk[it][x] = fmaf(e, kf[x], Bk[it][x] * alpha);
                }
                m[it] = mn;
            }
        }
    }

    // dq = scale / l * (Ak - D Bk), D = sdp / l
    float Dd[NI], inv[NI];
#pragma unroll
    for (int it = 0; it < NI; ++it) {
        const int g = it * RPI + seg;
        inv[it] = l[it] > 0.0f ? 1.0f / l[it] : 0.0f;
        Dd[it] = sdp[it] * inv[it];
        if (g >= G) continue;
        float *dqp = a.dq + (row * G + g) * D + c * VEC;
        const float f = a.scale * inv[it];
#pragma unroll
        for (int x = 0; x < VEC; x += 4) {
            float4 r;
            r.x = f * (Ak[it][x + 0] - Dd[it] * Bk[it][x + 0]);
            r.y = f * (Ak[it][x + 1] - Dd[it] * Bk[it][x + 1]);
            r.z = f * (Ak[it][x + 2] - Dd[it] * Bk[it][x + 2]);
            r.w = f * (Ak[it][x + 3] - Dd[it] * Bk[it][x + 3]);
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
            const float p = exp2f(sh_z[wid][g][j] - m[it]) * inv[it];
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

        const int64_t off = ((seq_base + t) * a.hkv + h) * D + c * VEC;
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
    if (lane < a.s) {
        float *p = a.dlogw + row * a.s + lane;
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
