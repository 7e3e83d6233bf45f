// gm_bwd_tile.cuh - SEA backward, tiled for small edge budgets (s <= 4, head_dim 64/128).
//
// Same mathematics as sea_bwd_kernel (gm_sea_bwd.cuh); the work division of the tiled
// forward (gm_fused_tile.cuh): a warp owns tiles of 32 consecutive edge rows (the last
// round's shorter); phase 1 loads the tile's edges one thread per row into shared memory;
// phase 2 processes RPW rows per pass with C lanes per row, each lane owning one 16-byte
// chunk of every feature row for all G query heads, with its K and V chunks staged by the
// lane itself via cp.async P passes ahead and its q and dO chunks read into registers one
// pass ahead. Per row and query head, with z_j = scale q.k_j + ln w_j, p = softmax(z),
// dp_j = dO.v_j, D = sum_j p_j dp_j and dz_j = p_j (dp_j - D):
//   dq          = scale sum_j dz_j k_j                       (stored)
//   dK[t_j]    += scale sum_heads dz_j q                     (GATHER = false: 16-byte fp32
//   dV[t_j]    += sum_heads p_j dO                            vector atomics)
//   dlogw[j]    = sum_heads dz_j                             (stored)
// With GATHER = true the two scatter-adds are not done here: the kernel writes each active
// edge's record (target row, source row, scale dz_g, p_g) at its place in its target's
// bucket (the bucket offset plus the rank the count pass gave the edge), and the gather pass
// of gm_bwd_gather.cuh forms dK and dV. With SB > 0 a third phase runs the referral backward
// of the tile's rows (ser_backward_row).
// Every shuffle runs on all 32 lanes (slots padded to S1M and masked after the reduction).
#pragma once

#include "gm_bwd_gather.cuh"
#include "gm_common.cuh"
#include "gm_fused_tile.cuh"
#include "gm_sea_bwd.cuh"

namespace gm {

template <typename T, int D, int G, int S1M> struct BwdTileGeom {
    static constexpr int VEC = Vec<T>::N;
    static constexpr int C = D / VEC;
    static constexpr int RPW = 32 / C;
    static constexpr int NPASS = 32 / RPW;
    static constexpr int ROW = D * (int)sizeof(T);
    // per row: the K and V rows of the S1M slots (q and dO go straight to registers)
    static constexpr int RK = 0, RV = S1M * ROW;
    static constexpr int RBYTES = RV + S1M * ROW;
    static constexpr int STAGE = RPW * RBYTES;
    static_assert(C >= 2 && C <= 16 && (C & (C - 1)) == 0, "two or more rows per warp pass");
};

// Resident blocks per SM the tile kernel is compiled for: caps registers at 65536 / (32 * WPB *
// MINB). Four blocks (128 registers, no spills) measured faster than five (96 registers with
// spills) for the gather row pass; the atomic row pass keeps four too.
#ifndef GM_BWD_TILE_MINB
#define GM_BWD_TILE_MINB 4
#endif

// Shared memory per warp of the tile row pass: the edge tile (K/V row, log2 w per slot), with
// the fused referral backward (SB > 0) also each slot's target, weight and d ln w, in gather
// mode each slot's record position; then the P stages.
template <int S1M, int SB, bool GATHER> __host__ __device__ constexpr int bwd_tile_bytes()
{
    return 32 * S1M * ((SB > 0 ? 20 : 8) + (GATHER ? 4 : 0));
}

// Referral backward of one edge row by one thread, fused after the attention backward of its
// tile: the forward kept (kt[r], kw[r]) (index, weight > 0) of A' = Sparsify(A1 A2); g[r] is
// the gradient of ln kw[r]. Each two-hop candidate (a, e) whose product fl32(w1 w2) is nonzero
// and whose target was kept passes g / W to dw1[a] (times w2, summed in ascending e, each
// product and add rounded once, as ser_bwd_thread_kernel) and to dw2 of its second-leg slot
// (times w1, fp32 atomics).
template <int SB, int S1M>
__device__ __forceinline__ void ser_backward_row(const SeaBwdArgs &a, uint32_t row, uint32_t seq_base, uint32_t h,
                                                 const int32_t (&kt)[S1M], const float (&kw)[S1M],
                                                 const float (&gl)[S1M])
{
    float kg[S1M];
#pragma unroll
    for (int r = 0; r < S1M; ++r) kg[r] = kw[r] > 0.0f ? gl[r] / kw[r] : 0.0f;
    int32_t j[SB];
    float w1[SB];
    ld_vec<SB>(a.a1_idx + (size_t)row * SB, j);
    ld_vec<SB>(a.a1_w + (size_t)row * SB, w1);
#pragma unroll
    for (int x = 0; x < SB; ++x) {
        bool act = w1[x] > 0.0f;
        if (act && (uint32_t)j[x] >= (uint32_t)a.n) {
            raise_index_error();
            act = false;
        }
        int32_t t2[SB];
        float w2[SB];
#pragma unroll
        for (int e = 0; e < SB; ++e) {
            t2[e] = 0;
            w2[e] = 0.0f;
        }
        const size_t r2 = act ? ((size_t)(seq_base + (uint32_t)j[x]) * a.hkv + h) * SB : 0;
        if (act) {
            ld_vec<SB>(a.a2_idx + r2, t2);
            ld_vec<SB>(a.a2_w + r2, w2);
        }
        float d1 = 0.0f;
#pragma unroll
        for (int e = 0; e < SB; ++e) {
            bool v = w2[e] > 0.0f;
            if (v && (uint32_t)t2[e] >= (uint32_t)a.n) {
                raise_index_error();
                v = false;
            }
            const bool cand = v && __fmul_rn(w1[x], w2[e]) != 0.0f;
            float g = 0.0f;
#pragma unroll
            for (int r = 0; r < S1M; ++r) g = (cand && t2[e] == kt[r] && kw[r] > 0.0f) ? kg[r] : g;
            d1 = __fadd_rn(d1, __fmul_rn(g, w2[e]));
            if (g != 0.0f) atomicAdd(a.dw2 + r2 + e, __fmul_rn(g, w1[x]));
        }
        float *p = a.dw1 + (size_t)row * SB + x;
        *p = a.accumulate ? *p + d1 : d1;
    }
}

template <typename T, int D, int G, int S1M, int P, int WPB, bool GATHER, int SB = 0>
__global__ void __launch_bounds__(WPB * 32, GATHER ? GM_BWD_TILE_MINB : 4) sea_bwd_tile_kernel(SeaBwdArgs a)
{
    pdl_wait();  // the bucket offsets and ranks (gather mode), when launched after the scan
    pdl_trigger();
    using TG = BwdTileGeom<T, D, G, S1M>;
    constexpr int VEC = TG::VEC, C = TG::C, RPW = TG::RPW, NP = VEC / 2;
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    constexpr int TILE_BYTES = bwd_tile_bytes<S1M, SB, GATHER>();
    char *wbase = smem + (size_t)wid * (TILE_BYTES + P * TG::STAGE);
    int32_t *tile_t = reinterpret_cast<int32_t *>(wbase);
    float *tile_lw = reinterpret_cast<float *>(wbase + 32 * S1M * 4);
    // fused referral backward: raw targets, weights and d ln w of the tile's slots
    int32_t *tile_tt = reinterpret_cast<int32_t *>(wbase + 32 * S1M * 8);
    float *tile_w = reinterpret_cast<float *>(wbase + 32 * S1M * 12);
    float *tile_g = reinterpret_cast<float *>(wbase + 32 * S1M * 16);
    // gather mode: where each active slot's record goes (off[target] + the edge's rank)
    int32_t *tile_pos = reinterpret_cast<int32_t *>(wbase + 32 * S1M * (SB > 0 ? 20 : 8));
    char *stages = wbase + TILE_BYTES;

    const uint32_t rows = a.rows;
    const uint32_t W = gridDim.x * WPB;
    const int rr = lane / C, c = lane % C;
    const float sl2 = a.scale * LOG2E;
    // this lane's chunk of K/V row 0: a gathered row's chunk is one wide multiply-add away
    const char *kbase = static_cast<const char *>(a.k) + (size_t)c * 16;
    const char *vbase = static_cast<const char *>(a.v) + (size_t)c * 16;

    // rounds of one 32-row tile per warp, the remainder split evenly over the warps (as in
    // the forward tile kernel)
    const uint32_t gw = blockIdx.x * WPB + wid;
    const uint32_t full = rows / (W * 32);
    const uint32_t rem = rows - full * W * 32;
    const uint32_t per = (rem + W - 1) / W;
    const uint32_t nround = full + (rem > 0 ? 1u : 0u);
    for (uint32_t round = 0; round < nround; ++round) {
        uint32_t r0, rend;
        if (round < full) {
            r0 = (round * W + gw) * 32;
            rend = r0 + 32;
        } else {
            r0 = full * W * 32 + gw * per;
            if (r0 >= rows) break;  // warp-uniform
            rend = min(r0 + per, rows);
        }
        const int npass = (int)((rend - r0 + RPW - 1) / RPW);  // warp-uniform, <= 32 / RPW

        // ---- phase 1: the tile's edges, one thread per row ----------------------------------
        {
            const uint32_t row = r0 + lane;
            // slots are stored as K/V rows ((b*n + t)*hkv + h): phase 2 issues its copies and
            // keys its records without decomposing the row again
            uint32_t seq_base = 0, h = 0;
            if (row < rend) a.map.split(row, seq_base, h);
#pragma unroll
            for (int r = 0; r < S1M; ++r) {
                int32_t t = 0;
                float lw = -INFINITY;
                if (row < rend && r < a.s) {
                    const float w = __ldg(a.w + (size_t)row * a.s + r);
                    const int32_t ti = __ldg(a.idx + (size_t)row * a.s + r);
                    if (w > 0.0f) {
                        if ((uint32_t)ti >= (uint32_t)a.n) {
                            raise_index_error();
                        } else {
                            t = ti;
                            lw = lg2(w);
                        }
                    }
                }
                const uint32_t key = (seq_base + (uint32_t)t) * (uint32_t)a.hkv + h;
                tile_t[lane * S1M + r] = (int32_t)key;
                tile_lw[lane * S1M + r] = lw;
                if constexpr (GATHER) {  // the count pass applied the same activity test
                    // the record's place, and in bit 31 whether its target is hot (its bucket
                    // holds more than GATHER_HOT records; the gather pass splits those)
                    int32_t pos = -1;
                    if (lw != -INFINITY) {
                        const int32_t o0 = __ldg(a.off + key), o1 = __ldg(a.off + key + 1);
                        pos = o0 + __ldg(a.rank + (size_t)row * a.s + r);
                        if (o1 - o0 > GATHER_HOT) pos |= (int32_t)0x80000000u;
                    }
                    tile_pos[lane * S1M + r] = pos;
                }
                if constexpr (SB > 0) {
                    tile_tt[lane * S1M + r] = t;
                    tile_w[lane * S1M + r] = lw == -INFINITY ? 0.0f : __ldg(a.w + (size_t)row * a.s + r);
                    tile_g[lane * S1M + r] = 0.0f;
                }
            }
        }
        __syncwarp();

        // ---- phase 2 ----------------------------------------------------------------------------
        auto issue = [&](int pass) {
            if (pass < npass) {
                const int lr = pass * RPW + rr;
                const uint32_t row = r0 + lr;
                char *st = stages + (pass % P) * TG::STAGE + rr * TG::RBYTES;
                // every slot is copied; an inactive one (or a row past the end) reads nothing
                // and gets zeros, so no branch and no stale data
                float lwv[S1M];
                int32_t tv[S1M];
                ld_tile<S1M>(tile_lw + lr * S1M, lwv);
                ld_tile<S1M>(tile_t + lr * S1M, tv);
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    const bool live = row < rend && lwv[jj] != -INFINITY;
                    const size_t off = (size_t)(live ? (uint32_t)tv[jj] : 0u) * TG::ROW;
                    cp_async16_zfill(st + TG::RK + jj * TG::ROW + c * 16, kbase + off, live);
                    cp_async16_zfill(st + TG::RV + jj * TG::ROW + c * 16, vbase + off, live);
                }
            }
            cp_async_commit();
        };
        // q and dO chunks of a pass in registers, read one pass ahead (a pass's compute covers
        // the loads; without them in shared memory more warps are resident)
        auto load_qg = [&](int pass, uint4 (&qv)[G], uint4 (&gv)[G]) {
            const uint32_t row = r0 + pass * RPW + rr;
            const bool ok = pass < npass && row < rend;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const size_t off = (size_t)row * (G * TG::ROW) + g * TG::ROW + c * 16;
                qv[g] = ok ? ld16(static_cast<const char *>(a.q) + off) : make_uint4(0u, 0u, 0u, 0u);
                gv[g] = ok ? ld16(static_cast<const char *>(a.dout) + off) : make_uint4(0u, 0u, 0u, 0u);
            }
        };
        uint4 qn[G], gn[G];
        load_qg(0, qn, gn);
#pragma unroll
        for (int pass = 0; pass < P; ++pass) issue(pass);

        for (int pass = 0; pass < npass; ++pass) {
            uint4 qc[G], gc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                qc[g] = qn[g];
                gc[g] = gn[g];
            }
            load_qg(pass + 1, qn, gn);
            cp_async_wait<P - 1>();
            const int lr = pass * RPW + rr;
            const uint32_t row = r0 + lr;
            const bool valid = row < rend;
            const char *st = stages + (pass % P) * TG::STAGE + rr * TG::RBYTES;

            float lw[S1M];
            bool act[S1M];
            ld_tile<S1M>(tile_lw + lr * S1M, lw);
#pragma unroll
            for (int jj = 0; jj < S1M; ++jj) act[jj] = valid && lw[jj] != -INFINITY;
            float2 q2[G][NP], g2[G][NP];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float f[VEC];
                // an invalid row (ragged tail) computes on zeros and stores nothing
                unpack<T>(qc[g], f);
#pragma unroll
                for (int x = 0; x < NP; ++x) q2[g][x] = make_float2(f[2 * x], f[2 * x + 1]);
                unpack<T>(gc[g], f);
#pragma unroll
                for (int x = 0; x < NP; ++x) g2[g][x] = make_float2(f[2 * x], f[2 * x + 1]);
            }
            float p[G][S1M], dz[G][S1M];
            constexpr int NV = 2 * G * S1M;  // (slot, head) pairs of q.k and dO.v per row
            if constexpr (NV <= C) {
                // Distributed softmax: the NV partial dots are reduced across the row's C lanes
                // by a transposed butterfly (each step sends half of the remaining values to the
                // partner lane), so lane L of the segment ends with value vi = L / SPREAD,
                // vi = 2 (slot * G + head) + {0: q.k, 1: dO.v}; the softmax, D and dz then take
                // one (slot, head) per lane pair, and dz (and, per record, p) are broadcast.
                constexpr int SPREAD = C / NV;
                float v[NV];
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    float kf[VEC], vf[VEC];
                    // an inactive slot's stage holds zeros: its values are masked below
                    unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RK + jj * TG::ROW + c * 16), kf);
                    unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RV + jj * TG::ROW + c * 16), vf);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        v[(jj * G + g) * 2] = chunk_dot<NP>(q2[g], kf);
                        v[(jj * G + g) * 2 + 1] = chunk_dot<NP>(g2[g], vf);
                    }
                }
#pragma unroll
                for (int cnt = NV, off = C / 2; cnt > 1; cnt >>= 1, off >>= 1) {
                    const bool up = (lane & off) != 0;
#pragma unroll
                    for (int i = 0; i < cnt / 2; ++i) {
                        const float send = up ? v[i] : v[i + cnt / 2];
                        const float keep = up ? v[i + cnt / 2] : v[i];
                        v[i] = keep + __shfl_xor_sync(FULL, send, off);
                    }
                }
                float x = v[0];
#pragma unroll
                for (int off = SPREAD / 2; off > 0; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
                const int vi = (lane & (C - 1)) / SPREAD;
                const float other = __shfl_xor_sync(FULL, x, SPREAD);
                const bool is_dp = (vi & 1) != 0;
                const float sc = is_dp ? other : x, dpv = is_dp ? x : other;
                const float mylw = tile_lw[lr * S1M + (vi >> 1) / G];
                const bool myact = valid && mylw != -INFINITY;
                const float zz = myact ? fmaf(sc, sl2, mylw) : -INFINITY;
                float m = zz;  // over the slots of this lane's head
#pragma unroll
                for (int off = 2 * G * SPREAD; off < C; off <<= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
                const float e = myact ? ex2(zz - m) : 0.0f;
                float l = e, sdp = myact ? e * dpv : 0.0f;
#pragma unroll
                for (int off = 2 * G * SPREAD; off < C; off <<= 1) {
                    l += __shfl_xor_sync(FULL, l, off);
                    sdp += __shfl_xor_sync(FULL, sdp, off);
                }
                const float inv = l > 0.0f ? rcp_fast(l) : 0.0f;  // l >= 1: its largest term is 1
                const float pj = e * inv;
                const float dzj = pj * ((myact ? dpv : 0.0f) - sdp * inv);
                const int seg = lane & ~(C - 1);
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj)
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const int src = seg + (jj * G + g) * 2 * SPREAD;
                        dz[g][jj] = __shfl_sync(FULL, dzj, src);
                        if constexpr (!GATHER) p[g][jj] = __shfl_sync(FULL, pj, src);
                    }
                if constexpr (GATHER) {
                    // a record needs p of its own slot c only
                    const int jc = c < S1M ? c : 0;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float pc = __shfl_sync(FULL, pj, seg + (jc * G + g) * 2 * SPREAD);
#pragma unroll
                        for (int jj = 0; jj < S1M; ++jj) p[g][jj] = (jj == jc) ? pc : 0.0f;
                    }
                }
            } else {
            // scores and dO.V per slot and head
            float z[G][S1M], dp[G][S1M];
#pragma unroll
            for (int jj = 0; jj < S1M; ++jj) {
                float kf[VEC], vf[VEC];
                // an inactive slot's stage holds zeros: its score and dO.V are masked below
                unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RK + jj * TG::ROW + c * 16), kf);
                unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RV + jj * TG::ROW + c * 16), vf);
#pragma unroll
                for (int g = 0; g < G; ++g) {  // q.k and dO.v reduced together (packed adds)
                    const float2 r = seg_sum2<C>(make_float2(chunk_dot<NP>(q2[g], kf), chunk_dot<NP>(g2[g], vf)));
                    z[g][jj] = act[jj] ? fmaf(r.x, sl2, lw[jj]) : -INFINITY;
                    dp[g][jj] = act[jj] ? r.y : 0.0f;
                }
            }
            // softmax, D, dz
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float m = z[g][0];
#pragma unroll
                for (int jj = 1; jj < S1M; ++jj) m = fmaxf(m, z[g][jj]);
                float l = 0.0f, sdp = 0.0f;
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    p[g][jj] = act[jj] ? ex2(z[g][jj] - m) : 0.0f;
                    l += p[g][jj];
                    sdp = fmaf(p[g][jj], dp[g][jj], sdp);
                }
                const float inv = l > 0.0f ? rcp_fast(l) : 0.0f;
                const float Dd = sdp * inv;
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    p[g][jj] *= inv;
                    dz[g][jj] = p[g][jj] * (dp[g][jj] - Dd);
                }
            }
            }
            // dq = scale sum_j dz_j k_j ; scatter dK, dV ; dlogw
            float2 dq2[G][NP];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int x = 0; x < NP; ++x) dq2[g][x] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int jj = 0; jj < S1M; ++jj) {
                // zero-filled stages: an inactive slot has dz = p = 0 and K = 0 (no branch); the
                // atomic path still skips its scatter
                if (!GATHER && !act[jj]) continue;  // per lane; no shuffles below
                float kf[VEC];
                unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RK + jj * TG::ROW + c * 16), kf);
                float2 pk[NP], pv[NP];
#pragma unroll
                for (int x = 0; x < NP; ++x) pk[x] = pv[x] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float sdz = a.scale * dz[g][jj];
                    const float2 sdz2 = make_float2(sdz, sdz), p2 = make_float2(p[g][jj], p[g][jj]);
#pragma unroll
                    for (int x = 0; x < NP; ++x) {
                        dq2[g][x] = __ffma2_rn(sdz2, make_float2(kf[2 * x], kf[2 * x + 1]), dq2[g][x]);
                        pk[x] = __ffma2_rn(sdz2, q2[g][x], pk[x]);
                        pv[x] = __ffma2_rn(p2, g2[g][x], pv[x]);
                    }
                }
                if constexpr (!GATHER) {
                    const uint32_t key = (uint32_t)tile_t[lr * S1M + jj];
                    const size_t off = (size_t)key * D + c * VEC;
#pragma unroll
                    for (int x = 0; x < NP; x += 2) {
                        red_add4(a.dk + off + 2 * x, pk[x].x, pk[x].y, pk[x + 1].x, pk[x + 1].y);
                        red_add4(a.dv + off + 2 * x, pv[x].x, pv[x].y, pv[x + 1].x, pv[x + 1].y);
                    }
                } else {
                    (void)pk;
                    (void)pv;
                }
            }
            if constexpr (GATHER) {
                // lane c < S1M files slot c's record into its target's bucket: one integer atomic
                // per pass for all slots, then one 32-byte record
                bool mine = false;
                float rc[2 * G];
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    if (c == jj) {
                        mine = act[jj];
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            rc[g] = a.scale * dz[g][jj];
                            rc[G + g] = p[g][jj];
                        }
                    }
                }
                if (c < S1M && mine) {
                    const uint32_t key = (uint32_t)tile_t[lr * S1M + c];
                    const uint32_t tp = (uint32_t)tile_pos[lr * S1M + c];
                    const uint32_t pos = tp & 0x7fffffffu;
                    // the count pass applies the same activity test, so pos stays inside the
                    // bucket; the bound only keeps a broken invariant from writing outside.
                    // The hot bit travels in bit 31 of the source row (rows < 2^31).
                    if (pos < a.rows * (uint32_t)a.s)
                        write_record<G>(a.srec, (int32_t)pos, key, row | (tp & 0x80000000u), rc);
                }
            }
            if (valid) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float *dqp = a.dq + ((size_t)row * G + g) * D + c * VEC;
#pragma unroll
                    for (int x = 0; x < NP; x += 2) {
                        float4 r = make_float4(dq2[g][x].x, dq2[g][x].y, dq2[g][x + 1].x, dq2[g][x + 1].y);
                        if (a.accumulate) {
                            const float4 o = *reinterpret_cast<const float4 *>(dqp + 2 * x);
                            r.x += o.x; r.y += o.y; r.z += o.z; r.w += o.w;
                        }
                        *reinterpret_cast<float4 *>(dqp + 2 * x) = r;
                    }
                }
                if (c < a.s) {
                    float dl = 0.0f;
#pragma unroll
                    for (int jj = 0; jj < S1M; ++jj) {
                        float sum = 0.0f;
#pragma unroll
                        for (int g = 0; g < G; ++g) sum += dz[g][jj];
                        dl = (jj == c) ? sum : dl;
                    }
                    float *pd = a.dlogw + (size_t)row * a.s + c;
                    *pd = a.accumulate ? *pd + dl : dl;
                    if constexpr (SB > 0) tile_g[lr * S1M + c] = dl;  // this call's gradient only
                }
            }
            issue(pass + P);
        }
        cp_async_wait<0>();
        __syncwarp();
        if constexpr (SB > 0) {
            // ---- phase 3: the referral backward of the tile's rows, one thread per row ------
            const uint32_t row = r0 + lane;
            if (row < rend) {
                uint32_t seq_base, h;
                a.map.split(row, seq_base, h);
                int32_t kt[S1M];
                float kw[S1M], gl[S1M];
                ld_tile<S1M>(tile_tt + lane * S1M, kt);
                ld_tile<S1M>(tile_w + lane * S1M, kw);
                ld_tile<S1M>(tile_g + lane * S1M, gl);
                ser_backward_row<SB, S1M>(a, row, seq_base, h, kt, kw, gl);
            }
            __syncwarp();  // the tile arrays are rewritten by the next tile's phase 1
        }
    }
}

}  // namespace gm
