// gm_fused_tile.cuh - fused SER -> SEA forward, tiled for small edge budgets.
//
// Same arithmetic as ser_row + sea_row (gm_ser.cuh, gm_sea.cuh); a different division of
// work that spends far fewer warp instructions per edge row when s2, s3, s1 are small
// ("Graph Machine: Towards Better Pretraining via Edges", ai.info summary, "Main Findings":
// 2 or 4 positions per KV head).
//
// A warp owns tiles of 32 consecutive edge rows (b, i, h), dealt in rounds over the whole
// grid; the rows left after the full rounds are split evenly, so the last tiles are shorter.
//  Phase 1 - referral, one thread per row. Lane L gathers its row's s2 first-leg slots and
//    the s3 second-leg slots behind each (vector loads), forms the s2*s3 candidates in
//    registers, merges duplicates in ascending candidate order (the first occurrence
//    accumulates the later ones with __fadd_rn), and selects the s1 heaviest (weight desc,
//    index asc) through a compare-exchange chain on 64-bit (weight, ~index) keys. Results: A'
//    to global memory (once, for the next layer) and to a shared-memory tile with log2
//    weights for phase 2.
//  Phase 2 - attention, C lanes (one 16-byte chunk each) per row, 32 / C rows per pass. Each
//    lane handles its chunk for all G query heads of the group, so a K/V chunk is unpacked
//    once and used G times, with packed fp32x2 FMAs. The lane stages exactly the K/V chunks
//    it will read with 16-byte cp.async, P passes ahead, so every byte in flight sits in
//    shared memory, and completion needs no spin-wait (cp.async.wait_group); an inactive
//    slot's copy reads nothing and fills zeros, so every slot is computed without a branch.
//    Its q chunks go straight to registers one pass ahead. The softmax normalises the
//    probabilities before the weighted sum of V, so the output needs no division.
// All shuffles run on all 32 lanes: slots are padded to S1M and inactive ones masked after
// the reduction, so rows at a ragged tail simply compute on zeros and store nothing.
#pragma once

#include "gm_common.cuh"
#include "gm_sea.cuh"
#include "gm_ser.cuh"

namespace gm {

template <int S> __device__ __forceinline__ void ld_vec(const int32_t *p, int32_t (&o)[S])
{
    if constexpr (S == 4) {
        const int4 v = __ldg(reinterpret_cast<const int4 *>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else if constexpr (S == 2) {
        const int2 v = __ldg(reinterpret_cast<const int2 *>(p));
        o[0] = v.x; o[1] = v.y;
    } else {
#pragma unroll
        for (int x = 0; x < S; ++x) o[x] = __ldg(p + x);
    }
}
template <int S> __device__ __forceinline__ void ld_vec(const float *p, float (&o)[S])
{
    if constexpr (S == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else if constexpr (S == 2) {
        const float2 v = __ldg(reinterpret_cast<const float2 *>(p));
        o[0] = v.x; o[1] = v.y;
    } else {
#pragma unroll
        for (int x = 0; x < S; ++x) o[x] = __ldg(p + x);
    }
}

// Target of a candidate that takes no part (zero weight): unique per candidate and negative,
// so it never equals another candidate's target.
__device__ __forceinline__ int32_t no_target(int c) { return -2 - c; }

// Duplicate merge over candidate pairs (c, c2), c < c2, in lexicographic order: when c is
// still nonzero and c2 shares its target, c absorbs c2 (one __fadd_rn) and c2 is cleared. A
// group's members are thus added to its first occurrence in ascending candidate order.
// Zero-weight candidates carry no_target(), so an equal target implies both are live (a c2
// already cleared by an earlier c' shares c's target only if c' cleared c as well).
// Unrolled (template recursion over c, an unrolled loop over c2) so the candidate arrays
// stay in registers.
template <int C0, int NC>
__device__ __forceinline__ void merge_pairs(const int32_t (&ct)[NC], float (&cu)[NC])
{
    if constexpr (C0 < NC - 1) {
        const bool live = cu[C0] != 0.0f;  // stays so while c absorbs (weights are positive)
#pragma unroll
        for (int c2 = C0 + 1; c2 < NC; ++c2) {
            const bool same = live && ct[c2] == ct[C0];
            cu[C0] = same ? __fadd_rn(cu[C0], cu[c2]) : cu[C0];
            cu[c2] = same ? 0.0f : cu[c2];
        }
        merge_pairs<C0 + 1, NC>(ct, cu);
    }
}

// One referral step of one edge row by one thread: first leg (j, w1) of S_IN slots in
// registers, second leg [rows, S3] at (leg_idx, leg_w); SF > 0 appends the row's SF refresh
// edges (a.sf == SF) after the S_IN*S3 paths. Keeps the s_keep <= S_OUT heaviest targets;
// other slots, and slots beyond the number of distinct targets, come back as (0, 0.0f).
template <int S_IN, int S3, int S_OUT, int SF = 0>
__device__ __forceinline__ void refer_thread(const SerArgs &a, uint32_t row, uint32_t seq_base,
                                             uint32_t h, const int32_t (&j)[S_IN],
                                             const float (&w1)[S_IN], const int32_t *leg_idx,
                                             const float *leg_w, int s_keep,
                                             int32_t (&to)[S_OUT], float (&wo)[S_OUT])
{
    constexpr int NP2 = S_IN * S3, NC = NP2 + SF;
    int32_t ct[NC];
    float cu[NC];
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
        if (act) {
            const size_t r2 = ((size_t)(seq_base + (uint32_t)j[x]) * a.k + h) * S3;
            ld_vec<S3>(leg_idx + r2, t2);
            ld_vec<S3>(leg_w + r2, w2);
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
    // merge: the first occurrence of a target absorbs the later ones, in ascending order
    merge_pairs<0, NC>(ct, cu);
    // top-s: each merged candidate enters a sorted list of S_OUT 64-bit keys (weight bits,
    // then the complemented target: positive fp32 weights order as their bit patterns, so
    // the larger key is the heavier target, the smaller index on equal weights; a zero
    // weight is key 0 and never enters) by a chain of compare-exchanges, no branches
    unsigned long long key[S_OUT];
#pragma unroll
    for (int r = 0; r < S_OUT; ++r) key[r] = 0ull;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        unsigned long long kc = cu[c] > 0.0f
                                    ? ((unsigned long long)__float_as_uint(cu[c]) << 32) | (uint32_t)~ct[c]
                                    : 0ull;
#pragma unroll
        for (int r = 0; r < S_OUT; ++r) {
            const unsigned long long hi = kc > key[r] ? kc : key[r];
            kc = kc > key[r] ? key[r] : kc;
            key[r] = hi;
        }
    }
#pragma unroll
    for (int r = 0; r < S_OUT; ++r) {
        const bool keep = r < s_keep && key[r] != 0ull;
        to[r] = keep ? (int32_t)~(uint32_t)key[r] : 0;
        wo[r] = keep ? __uint_as_float((uint32_t)(key[r] >> 32)) : 0.0f;
    }
}

// Referral of one edge row by one thread (exact S2, S3; s1 <= S1M), with SF refresh edges
// when SF > 0 and, when NL > 1, NL - 1 further referral steps through the chain legs (every
// intermediate of S2 = s_mid slots, the row's previous result held in registers).
template <int S2, int S3, int S1M, int SF = 0, int NL = 1>
__device__ __forceinline__ void ser_thread(const SerArgs &a, uint32_t row, int32_t (&to)[S1M],
                                           float (&wo)[S1M])
{
    uint32_t seq_base, h;
    a.map.split(row, seq_base, h);
    int32_t j[S2];
    float w1[S2];
    ld_vec<S2>(a.a1_idx + (size_t)row * S2, j);
    ld_vec<S2>(a.a1_w + (size_t)row * S2, w1);
    if constexpr (NL == 1) {
        refer_thread<S2, S3, S1M, SF>(a, row, seq_base, h, j, w1, a.a2_idx, a.a2_w, a.s1, to, wo);
    } else {
        static_assert(SF == 0, "refresh edges join single-step referrals only");
#pragma unroll
        for (int m = 0; m + 1 < NL; ++m) {
            int32_t jn[S2];
            float wn[S2];
            refer_thread<S2, S3, S2>(a, row, seq_base, h, j, w1, m == 0 ? a.a2_idx : a.chain_idx[m - 1],
                                     m == 0 ? a.a2_w : a.chain_w[m - 1], S2, jn, wn);
#pragma unroll
            for (int x = 0; x < S2; ++x) {
                j[x] = jn[x];
                w1[x] = wn[x];
            }
        }
        refer_thread<S2, S3, S1M>(a, row, seq_base, h, j, w1, a.chain_idx[NL - 2], a.chain_w[NL - 2],
                                  a.s1, to, wo);
    }
}

// The referral alone, one thread per edge row (the tiled forward's phase 1 without the
// attention): exact budgets S2, S3, s1 <= S1M, with SF refresh slots or a chain of NL steps.
// Same arithmetic and order as ser_kernel (a warp per row), so the two give the same bits.
// A' is written with 16-byte stores when s1 = S1M = 4 (16-byte aligned outputs).
template <int S2, int S3, int S1M, int SF = 0, int NL = 1>
__global__ void __launch_bounds__(128) ser_thread_kernel(SerArgs sa)
{
    const uint32_t row = blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= sa.rows) return;
    int32_t to[S1M];
    float wo[S1M];
    ser_thread<S2, S3, S1M, SF, NL>(sa, row, to, wo);
    if (sa.s1 == S1M && S1M == 4) {
        *reinterpret_cast<int4 *>(sa.out_idx + (size_t)row * 4) = make_int4(to[0], to[1], to[2], to[3]);
        *reinterpret_cast<float4 *>(sa.out_w + (size_t)row * 4) = make_float4(wo[0], wo[1], wo[2], wo[3]);
    } else {
#pragma unroll
        for (int r = 0; r < S1M; ++r) {
            if (r < sa.s1) {
                sa.out_idx[(size_t)row * sa.s1 + r] = to[r];
                sa.out_w[(size_t)row * sa.s1 + r] = wo[r];
            }
        }
    }
}

// The S entries of one row of a warp's shared-memory edge tile (16-byte aligned for S = 4,
// 8-byte for S = 2), read as one vector.
template <int S, typename V> __device__ __forceinline__ void ld_tile(const V *p, V (&o)[S])
{
    static_assert(sizeof(V) == 4, "32-bit tile entries");
    if constexpr (S == 4) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) o[x] = *reinterpret_cast<const V *>(&w[x]);
    } else if constexpr (S == 2) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        const uint32_t w[2] = {u.x, u.y};
#pragma unroll
        for (int x = 0; x < 2; ++x) o[x] = *reinterpret_cast<const V *>(&w[x]);
    } else {
#pragma unroll
        for (int x = 0; x < S; ++x) o[x] = p[x];
    }
}

// Resident one-warp blocks per SM the forward tile kernel is compiled for: caps registers at
// 65536 / (32 * WPB * MINB) without spills. With two stages in flight shared memory admits
// 24 warps; with one, registers (73 at 28 warps) are the limit.
#ifndef GM_TILE_MINB
#define GM_TILE_MINB(P) ((P) == 1 ? 28 : 24)
#endif

template <typename T, int D, int G, int S1M, int CPL = 1> struct TileGeom {
    static constexpr int VEC = Vec<T>::N;          // elements per 16-byte chunk
    static constexpr int C = D / (VEC * CPL);      // lanes per row (CPL chunks per lane)
    static constexpr int RPW = 32 / C;             // rows per warp pass
    static constexpr int NPASS = 32 / RPW;         // passes per 32-row tile
    static constexpr int ROW = D * (int)sizeof(T); // bytes per feature row
    // per row: q rows of the group, then K and V rows of the S1M slots (chunk-interleaved
    // per lane is not needed: every lane reads back only what it copied)
    // per row: the K and V rows of the S1M slots (q goes straight to registers)
    static constexpr int RK = 0, RV = S1M * ROW, RBYTES = RV + S1M * ROW;
    static constexpr int STAGE = RPW * RBYTES;
    static_assert(C >= 2 && C <= 16 && (C & (C - 1)) == 0, "two or more rows per warp pass");
};

// REFER = true: fused SER -> SEA (edges from the referral of sa's legs, plus SF refresh edges
// per row when SF > 0, or through NL legs of a multi-step referral when NL > 1);
// REFER = false: SEA alone on the edges a.idx / a.w (s = a.s <= S1M), sa unused.
template <typename T, int D, int G, bool REFER, int S2, int S3, int S1M, int P, int WPB, int CPL,
          int SF = 0, int NL = 1>
__global__ void __launch_bounds__(WPB * 32, GM_TILE_MINB(P)) sea_fwd_tile_kernel(SerArgs sa, SeaArgs a)
{
    using TG = TileGeom<T, D, G, S1M, CPL>;
    constexpr int VEC = TG::VEC, C = TG::C, RPW = TG::RPW, NP = VEC / 2;
    static_assert(VEC % 2 == 0, "packed fp32x2 math");
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    // per warp: edge tile (K/V row, log2 w) then P stages
    constexpr int TILE_BYTES = 32 * S1M * 8;
    char *wbase = smem + (size_t)wid * (TILE_BYTES + P * TG::STAGE);
    int32_t *tile_t = reinterpret_cast<int32_t *>(wbase);
    float *tile_lw = reinterpret_cast<float *>(wbase + 32 * S1M * 4);
    char *stages = wbase + TILE_BYTES;

    const uint32_t rows = a.rows;
    const uint32_t W = gridDim.x * WPB;
    const uint32_t gw = blockIdx.x * WPB + wid;
    // Rows are dealt in rounds: every warp takes a 32-row tile per round, the grid sweeping
    // the rows in order (one sequence's K/V stays in L2); the rows left after the full rounds
    // are split evenly, so every warp's last tile holds the same number of rows (at most 32)
    // and no round runs with part of the warps idle.
    const uint32_t full = rows / (W * 32);
    const uint32_t rem = rows - full * W * 32;
    const uint32_t per = (rem + W - 1) / W;
    const uint32_t nround = full + (rem > 0 ? 1u : 0u);
    const int rr = lane / C, c = lane % C;  // phase-2 row within the pass, chunk
    const float sl2 = a.scale * LOG2E;
    const T *Qg = static_cast<const T *>(a.q);
    T *O = static_cast<T *>(a.o);
    // this lane's first chunk of K/V row 0: a gathered row's chunk is one wide multiply-add away
    const char *kbase = static_cast<const char *>(a.k) + (size_t)(c * CPL) * 16;
    const char *vbase = static_cast<const char *>(a.v) + (size_t)(c * CPL) * 16;

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
        const int npass = (int)((rend - r0 + RPW - 1) / RPW);  // warp-uniform, <= NPASS

        // ---- phase 1: the tile's edges, one thread per row ------------------------------
        {
            const uint32_t row = r0 + lane;
            int32_t to[S1M];
            float wo[S1M];
#pragma unroll
            for (int r = 0; r < S1M; ++r) {
                to[r] = 0;
                wo[r] = 0.0f;
            }
            if constexpr (!REFER) {
                if (row < rend) {
#pragma unroll
                    for (int r = 0; r < S1M; ++r) {
                        if (r < a.s) {
                            const float w = __ldg(a.w + (size_t)row * a.s + r);
                            const int32_t t = __ldg(a.idx + (size_t)row * a.s + r);
                            if (w > 0.0f) {
                                if (t < 0 || t >= a.n) {
                                    raise_index_error();
                                } else {
                                    to[r] = t;
                                    wo[r] = w;
                                }
                            }
                        }
                    }
                }
            } else if (row < rend) {
                ser_thread<S2, S3, S1M, SF, NL>(sa, row, to, wo);
                if (sa.out_idx != nullptr) {
                    if (sa.s1 == S1M && S1M == 4) {
                        *reinterpret_cast<int4 *>(sa.out_idx + (size_t)row * 4) = make_int4(to[0], to[1], to[2], to[3]);
                        *reinterpret_cast<float4 *>(sa.out_w + (size_t)row * 4) = make_float4(wo[0], wo[1], wo[2], wo[3]);
                    } else {
#pragma unroll
                        for (int r = 0; r < S1M; ++r) {
                            if (r < sa.s1) {
                                sa.out_idx[(size_t)row * sa.s1 + r] = to[r];
                                sa.out_w[(size_t)row * sa.s1 + r] = wo[r];
                            }
                        }
                    }
                }
            }
            // K/V row of each slot ((b*n + t)*hkv + h), so phase 2 issues its copies without
            // decomposing the row again
            uint32_t seq_base = 0, h = 0;
            if (row < rend) a.map.split(row, seq_base, h);
#pragma unroll
            for (int r = 0; r < S1M; ++r) {
                tile_t[lane * S1M + r] = (int32_t)((seq_base + (uint32_t)to[r]) * (uint32_t)a.hkv + h);
                tile_lw[lane * S1M + r] = wo[r] > 0.0f ? lg2(wo[r]) : -INFINITY;
            }
        }
        __syncwarp();

        // ---- phase 2: attention, RPW rows per pass, P passes of copies in flight -----------
        auto issue = [&](int pass) {
            if (pass < npass) {
                const int lr = pass * RPW + rr;  // row within the tile
                const uint32_t row = r0 + lr;
                char *st = stages + (pass % P) * TG::STAGE + rr * TG::RBYTES;
                // every slot of a valid row is copied; an inactive one (or a row past the end)
                // reads nothing and gets zeros, so no branch and no stale data
                float lwv[S1M];
                int32_t tv[S1M];
                ld_tile<S1M>(tile_lw + lr * S1M, lwv);
                ld_tile<S1M>(tile_t + lr * S1M, tv);
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    const bool live = row < rend && lwv[jj] != -INFINITY;
                    const uint32_t kvrow = live ? (uint32_t)tv[jj] : 0u;
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) {
                        const size_t off = (size_t)kvrow * TG::ROW + cc * 16;
                        cp_async16_zfill(st + TG::RK + jj * TG::ROW + (c * CPL + cc) * 16, kbase + off, live);
                        cp_async16_zfill(st + TG::RV + jj * TG::ROW + (c * CPL + cc) * 16, vbase + off, live);
                    }
                }
            }
            cp_async_commit();
        };
        // q chunks of a pass, read into registers one pass ahead (a pass's compute covers the
        // load; q needs no shared memory, which leaves room for more resident warps)
        auto load_q = [&](int pass, uint4 (&qv)[G][CPL]) {
            const uint32_t row = r0 + pass * RPW + rr;
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc)
                    qv[g][cc] = (pass < npass && row < rend)
                                    ? ld16(reinterpret_cast<const char *>(Qg) + (size_t)row * (G * TG::ROW) +
                                           g * TG::ROW + (c * CPL + cc) * 16)
                                    : make_uint4(0u, 0u, 0u, 0u);
        };
        uint4 qnext[G][CPL];
        load_q(0, qnext);
#pragma unroll
        for (int pass = 0; pass < P; ++pass) issue(pass);

        for (int pass = 0; pass < npass; ++pass) {
            uint4 qcur[G][CPL];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) qcur[g][cc] = qnext[g][cc];
            load_q(pass + 1, qnext);
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
            // q chunks of the G heads as fp32 pairs
            float2 q2[G][CPL * NP];
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    float f[VEC];
                    // an invalid row (ragged tail) computes on zeros and stores nothing
                    unpack<T>(qcur[g][cc], f);
#pragma unroll
                    for (int x = 0; x < NP; ++x) q2[g][cc * NP + x] = make_float2(f[2 * x], f[2 * x + 1]);
                }
            }
            float2 acc[G][CPL * NP];
            float m[G] = {}, l[G] = {};
            constexpr int NV = G * S1M;  // (slot, head) scores per row
            if (NV > C) {  // the distributed softmax's first slot product initialises it
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int x = 0; x < CPL * NP; ++x) acc[g][x] = make_float2(0.0f, 0.0f);
            }
            if constexpr (NV <= C) {
                // Distributed softmax. The NV partial dots are reduced across the row's C lanes
                // by a transposed butterfly: each step sends half of the remaining values to
                // the partner lane and keeps the other half, so every lane adds the same pairs
                // as a full butterfly (x + partner) and the totals carry its exact bits. Lane L
                // of the segment ends with score vi = L / SPREAD (vi = slot * G + head); the
                // max, exponential and sum then take one value per lane.
                constexpr int SPREAD = C / NV;
                float v[NV];
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    float kf[CPL * VEC];
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) {
                        float f[VEC];
                        // an inactive slot's stage holds zeros: its score is masked below
                        unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RK + jj * TG::ROW + (c * CPL + cc) * 16), f);
#pragma unroll
                        for (int x = 0; x < VEC; ++x) kf[cc * VEC + x] = f[x];
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) v[jj * G + g] = chunk_dot<CPL * NP>(q2[g], kf);
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
                const float mylw = tile_lw[lr * S1M + vi / G];
                const bool myact = valid && mylw != -INFINITY;
                const float z = myact ? fmaf(x, sl2, mylw) : -INFINITY;
                float mz = z;  // max over the slots of this lane's head
#pragma unroll
                for (int off = G * SPREAD; off < C; off <<= 1) mz = fmaxf(mz, __shfl_xor_sync(FULL, mz, off));
                const float p = myact ? ex2(z - mz) : 0.0f;
                float lz = p;
#pragma unroll
                for (int off = G * SPREAD; off < C; off <<= 1) lz += __shfl_xor_sync(FULL, lz, off);
                // normalised probability (the sum is >= 1 when the head has an active slot: its
                // largest term is exp2(0)); the lane of slot 0 of each head stores its lse
                const float pn = lz > 0.0f ? p * rcp_fast(lz) : 0.0f;
                if (valid && a.lse != nullptr && vi < G && (lane & (SPREAD - 1)) == 0)
                    a.lse[(size_t)row * G + vi] = lz > 0.0f ? (mz + lg2(lz)) * LN2 : -INFINITY;
                const int seg = lane & ~(C - 1);
                float pp[S1M][G];
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj)
#pragma unroll
                    for (int g = 0; g < G; ++g) pp[jj][g] = __shfl_sync(FULL, pn, seg + (jj * G + g) * SPREAD);
#pragma unroll
                for (int jj = 0; jj < S1M; ++jj) {
                    // zero-filled stages: an inactive slot has p = 0 and V = 0, so every slot is
                    // accumulated without a branch, the first one by a multiply
                    float vf[CPL * VEC];
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) {
                        float f[VEC];
                        unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RV + jj * TG::ROW + (c * CPL + cc) * 16), f);
#pragma unroll
                        for (int x2 = 0; x2 < VEC; ++x2) vf[cc * VEC + x2] = f[x2];
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 p2 = make_float2(pp[jj][g], pp[jj][g]);
#pragma unroll
                        for (int x2 = 0; x2 < CPL * NP; ++x2) {
                            const float2 v2 = make_float2(vf[2 * x2], vf[2 * x2 + 1]);
                            if (jj == 0)
                                acc[g][x2] = __fmul2_rn(p2, v2);
                            else
                                acc[g][x2] = __ffma2_rn(p2, v2, acc[g][x2]);
                        }
                    }
                }
            } else {
            // scores (all S1M slots, masked after the reduction so shuffles stay uniform)
            float z[G][S1M];
#pragma unroll
            for (int jj = 0; jj < S1M; ++jj) {
                float kf[CPL * VEC];
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    float f[VEC];
                    // an inactive slot's stage holds zeros: its score is masked below
                    unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RK + jj * TG::ROW + (c * CPL + cc) * 16), f);
#pragma unroll
                    for (int x = 0; x < VEC; ++x) kf[cc * VEC + x] = f[x];
                }
                // the heads' partial dots are reduced two at a time (packed adds)
#pragma unroll
                for (int g = 0; g < G; g += 2) {
                    if (g + 1 < G) {
                        const float2 d2 = seg_sum2<C>(make_float2(chunk_dot<CPL * NP>(q2[g], kf),
                                                                  chunk_dot<CPL * NP>(q2[g + 1], kf)));
                        z[g][jj] = act[jj] ? fmaf(d2.x, sl2, lw[jj]) : -INFINITY;
                        z[g + 1][jj] = act[jj] ? fmaf(d2.y, sl2, lw[jj]) : -INFINITY;
                    } else {
                        const float dot = seg_sum<C>(chunk_dot<CPL * NP>(q2[g], kf));
                        z[g][jj] = act[jj] ? fmaf(dot, sl2, lw[jj]) : -INFINITY;
                    }
                }
            }
            // softmax and weighted V per head
#pragma unroll
            for (int g = 0; g < G; ++g) {
                m[g] = z[g][0];
#pragma unroll
                for (int jj = 1; jj < S1M; ++jj) m[g] = fmaxf(m[g], z[g][jj]);
                l[g] = 0.0f;
            }
#pragma unroll
            for (int jj = 0; jj < S1M; ++jj) {
                if (!act[jj]) continue;  // per lane; no shuffles below
                float vf[CPL * VEC];
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    float f[VEC];
                    unpack<T>(*reinterpret_cast<const uint4 *>(st + TG::RV + jj * TG::ROW + (c * CPL + cc) * 16), f);
#pragma unroll
                    for (int x = 0; x < VEC; ++x) vf[cc * VEC + x] = f[x];
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float p = ex2(z[g][jj] - m[g]);
                    l[g] += p;
                    const float2 p2 = make_float2(p, p);
#pragma unroll
                    for (int x = 0; x < CPL * NP; ++x)
                        acc[g][x] = __ffma2_rn(p2, make_float2(vf[2 * x], vf[2 * x + 1]), acc[g][x]);
                }
            }
            }
            if (valid) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    // the distributed softmax accumulated normalised probabilities already
                    const bool nonempty = NV <= C || l[g] > 0.0f;
                    const float inv = NV <= C ? 1.0f : (nonempty ? __frcp_rn(l[g]) : 0.0f);
#pragma unroll
                    for (int cc = 0; cc < CPL; ++cc) {
                        float of[VEC];
#pragma unroll
                        for (int x = 0; x < NP; ++x) {
                            of[2 * x] = NV <= C ? acc[g][cc * NP + x].x : acc[g][cc * NP + x].x * inv;
                            of[2 * x + 1] = NV <= C ? acc[g][cc * NP + x].y : acc[g][cc * NP + x].y * inv;
                        }
                        *reinterpret_cast<uint4 *>(O + ((size_t)row * G + g) * D + (c * CPL + cc) * VEC) = pack<T>(of);
                    }
                    if (NV > C && a.lse != nullptr && c == 0)
                        a.lse[(size_t)row * G + g] = nonempty ? (m[g] + lg2(l[g])) * LN2 : -INFINITY;
                }
            }
            issue(pass + P);
        }
        cp_async_wait<0>();
        __syncwarp();  // the tile's edge table is rewritten by the next tile's phase 1
    }
}

}  // namespace gm
