// gm_dense_refresh.cuh - refresh edges from a dense attention layer, on the tensor cores.
//
// "Graph Machine: Towards Better Pretraining via Edges", ai.info summary, "Methodology in
// Plain English", referral paragraph (refresh edges are the input edges or the top positions
// of the most recent dense attention layer) and "Main Findings", bullet on refresh and
// realignment. For every (b, i, KV head h): the sf positions t <= i with the largest attention
// mass of h - the mean over its G query heads of the causal softmax probability
// exp(scale <q[i,hq], k[t,h]> - lse[i,hq]) - ties to the smaller position; the mass is the
// edge weight; rows with fewer than sf positions are padded with (0, 0.0f).
//
// One CTA per (b, h, block of 128 query positions), the blocks with the longest causal prefix
// first. The scores S_g = Q_g K^T of the block's G query heads against each key block of the
// prefix run on the tensor cores: tcgen05.mma with bf16 operands staged by TMA in the
// 128-byte swizzle layout and fp32 accumulators in tensor memory (TMEM), two key stages and
// two accumulator sets, so the MMAs of key block j + 1 overlap the selection over block j.
// Warp roles: warps 0 .. 4 NPART - 1 select (NPART threads per query row = TMEM lane, thread
// p taking the 32-column chunks p, p + NPART, ... of a key block), warp 4 NPART loads (TMA),
// warp 4 NPART + 1 issues the MMAs. Every wait is bounded (gm_common.cuh, mbar_wait).
//
// Selection per thread, streaming over ascending t: a sorted register list of the SFM heaviest
// (mass, t) so far (SFM = sf rounded up to 2, 4 or 8; the first sf of the top SFM are the top
// sf). With x_g = scale log2(e) S_g - log2(e) lse_g the mass is mean_g 2^x_g <= 2^max_g x_g, so
// a position whose max_g x_g lies below log2 of the list's smallest mass cannot enter. The scan
// is branch-free: per column G FMAs, a max, a compare that sets a bit of a candidate mask, and
// a store of the x_g to a per-thread shared-memory slot; then each lane walks its own mask
// (computing the few candidates' masses with G exponentials and inserting those that beat the
// list), so the lanes of a warp never diverge per column. At the end the NPART threads of a
// row merge their lists.
#pragma once

#include <cuda.h>

#include "gm_common.cuh"
#include "gm_umma.cuh"

#ifndef GM_DENSE_NPART
#define GM_DENSE_NPART 4
#endif

namespace gm {

struct DenseRefreshArgs {
    const float *lse;   // [B, n, hq], natural log
    int32_t *out_idx;   // [B, n, hkv, sf]
    float *out_w;
    int n, hq, hkv, sf;
    int nblk;           // ceil(n / 128)
    int BH;             // B * hkv
    float sl2;          // scale * log2(e)
};

template <int D, int G, int BN> struct DenseGeom {
    static constexpr int BM = 128;                  // query rows per CTA (TMEM lanes)
    static constexpr int NA = D / 64;               // 128-byte swizzle atoms along d
    static constexpr int NST = 2, NACC = 2;         // key stages, accumulator sets
    static constexpr int Q_ATOM = BM * 128;         // bytes of one atom of the query tile
    static constexpr int K_ATOM = BN * 128;
    static constexpr int QBYTES = G * NA * Q_ATOM;
    static constexpr int KBYTES = NST * NA * K_ATOM;
    // selection threads per query row: one per 32-column chunk of a key block, at most
    // GM_DENSE_NPART (more threads hide more of the scan's latency)
    static constexpr int NPART = (BN / 32) < GM_DENSE_NPART ? (BN / 32) : GM_DENSE_NPART;
    static constexpr int NSEL = NPART * BM;         // selection threads
    static constexpr int THREADS = NSEL + 64;       // + the load warp and the MMA warp
    static constexpr int SUB = G == 4 ? 8 : 16;     // columns scanned per candidate mask
    static constexpr int OFF_K = QBYTES;
    static constexpr int OFF_LIST = QBYTES + KBYTES;  // x values [SUB][NSEL][G]
    static constexpr int OFF_BOUND = OFF_LIST + SUB * NSEL * G * 4;  // skip bounds [BM][NPART]
    static constexpr int OFF_BAR = OFF_BOUND + BM * NPART * 4;
    static constexpr int NBAR = 2 + 2 * NST + 2 * NACC;  // q_full, k_full/empty, acc_full/empty, mma_done
    static constexpr int TMEM_COLS = NACC * G * BN;
    // + TMEM slot and 1 KB of alignment; a CTA that takes more than half of the 512 TMEM columns
    // also takes more than half of the SM's shared memory, so no second CTA waits on the SM
    // for columns
    static constexpr int NEED = OFF_BAR + NBAR * 8 + 16 + 1024;
    static constexpr int SMEM_BYTES = TMEM_COLS > 256 && NEED < 120 * 1024 ? 120 * 1024 : NEED;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(BN == 64 || BN == 128, "key block of 64 or 128");
    static_assert((NPART - 1) * 2 * BM * 8 <= SUB * NSEL * G, "the parts' lists (SFM <= 8) fit the x slots");
    static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0,
                  "accumulators fit the 512 TMEM columns");
};

// Inserts (m, t) into the list sorted by (mass desc, position asc), dropping the last entry.
template <int SFM> __device__ __forceinline__ void list_insert(float (&kw)[SFM], int (&kt)[SFM], float m, int t)
{
#pragma unroll
    for (int r = 0; r < SFM; ++r) {
        const bool before = m > kw[r] || (m == kw[r] && t < kt[r]);
        const float w0 = kw[r];
        const int t0 = kt[r];
        kw[r] = before ? m : w0;
        kt[r] = before ? t : t0;
        m = before ? w0 : m;
        t = before ? t0 : t;
    }
}

// The same insertion for a thread's own stream of positions, which arrive in ascending t: an
// equal mass already in the list has the smaller position and stays first, so the strict
// comparison alone gives the (mass desc, position asc) order.
template <int SFM>
__device__ __forceinline__ void list_insert_ascending(float (&kw)[SFM], int (&kt)[SFM], float m, int t)
{
#pragma unroll
    for (int r = 0; r < SFM; ++r) {
        const bool before = m > kw[r];
        const float w0 = kw[r];
        const int t0 = kt[r];
        kw[r] = before ? m : w0;
        kt[r] = before ? t : t0;
        m = before ? w0 : m;
        t = before ? t0 : t;
    }
}

// Barrier over the first `count` threads of the CTA (the selection warps), id 1 (id 0 is the
// CTA-wide __syncthreads).
__device__ __forceinline__ void named_barrier_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}

// log2 of the list's smallest mass less a margin larger than lg2.approx's error (so the skip
// test never drops a position that could enter), or -inf while the list has room.
template <int SFM> __device__ __forceinline__ float skip_bound(const float (&kw)[SFM])
{
    return kw[SFM - 1] > 0.0f ? lg2(kw[SFM - 1]) - 0x1p-12f : -INFINITY;
}

template <int D, int G, int BN, int SFM>
__global__ void __launch_bounds__(DenseGeom<D, G, BN>::THREADS, 1)
dense_refresh_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     DenseRefreshArgs a)
{
    using Geo = DenseGeom<D, G, BN>;
    constexpr int NA = Geo::NA, NST = Geo::NST, NACC = Geo::NACC;
    extern __shared__ __align__(1024) uint8_t dsm[];
    // the swizzled tiles need 1024-byte aligned eight-row groups
    const uint32_t raw = smem_u32(dsm);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = dsm + (base - raw);
    const uint32_t sq = base, sk = base + Geo::OFF_K, sb = base + Geo::OFF_BAR;
    const uint32_t q_full = sb, k_full = sb + 8, k_empty = k_full + 8 * NST;
    const uint32_t acc_full = k_empty + 8 * NST, acc_empty = acc_full + 8 * NACC;
    const uint32_t mma_done = acc_empty + 8 * NACC, tslot = mma_done + 8;
    const uint32_t *tslot_p = reinterpret_cast<const uint32_t *>(sm + Geo::OFF_BAR + Geo::NBAR * 8);
    float *listx = reinterpret_cast<float *>(sm + Geo::OFF_LIST);  // [SUB][NSEL][G] x values
    // each selection thread's current skip bound, [row][part]: a position whose mass lies
    // below any part's smallest kept mass cannot enter the row's top list, so every part
    // filters by the largest of the row's bounds (they only grow; a stale read is still valid)
    volatile float *sbound = reinterpret_cast<float *>(sm + Geo::OFF_BOUND);
    if (threadIdx.x < Geo::NSEL) sbound[threadIdx.x] = -INFINITY;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ib = a.nblk - 1 - (int)(blockIdx.x / (unsigned)a.BH);  // longest prefixes first
    const int bh = (int)(blockIdx.x % (unsigned)a.BH);
    const int b = bh / a.hkv, h = bh - b * a.hkv;
    const int i0 = ib * Geo::BM;
    const int iend = min(i0 + Geo::BM, a.n);
    const int nt = (iend - 1) / BN + 1;  // key blocks that reach the block's last row
    const int row0 = b * a.n;            // first token of the sequence (B*n < 2^31)

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
#pragma unroll
        for (int s = 0; s < NST; ++s) {
            mbar_init(k_full + 8 * s, 1);
            mbar_init(k_empty + 8 * s, 1);
        }
#pragma unroll
        for (int s = 0; s < NACC; ++s) {
            mbar_init(acc_full + 8 * s, 1);
            mbar_init(acc_empty + 8 * s, Geo::NSEL);
        }
        mbar_init(mma_done, 1);
        mbar_init_fence();
    }
    if (warp == 0) umma::tmem_alloc(tslot, Geo::TMEM_COLS);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tslot_p;

    constexpr int LOAD_WARP = Geo::NSEL / 32, MMA_WARP = LOAD_WARP + 1;
    if (warp == LOAD_WARP) {
        // ---- loads: the query tile once, then the key blocks through NST stages ----------
        if (lane == 0) {
            mbar_arrive_expect(q_full, Geo::QBYTES);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int at = 0; at < NA; ++at)
                    umma::tma_load_3d(sq + (g * NA + at) * Geo::Q_ATOM, &tmq, at * 64, h * G + g, row0 + i0, q_full);
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int s = j % NST;
                if (j >= NST && !mbar_wait(k_empty + 8 * s, ((j / NST) - 1) & 1)) break;
                mbar_arrive_expect(k_full + 8 * s, NA * Geo::K_ATOM);
#pragma unroll
                for (int at = 0; at < NA; ++at)
                    umma::tma_load_3d(sk + (s * NA + at) * Geo::K_ATOM, &tmk, at * 64, h, row0 + j * BN, k_full + 8 * s);
                ++issued;
            }
            if (issued < nt) {
                // gave up: wait (bounded) for the copies still in flight before the CTA ends
                for (int j = max(0, issued - NST); j < issued; ++j) mbar_wait(k_full + 8 * (j % NST), (j / NST) & 1);
            }
        }
    } else if (warp == MMA_WARP) {
        // ---- MMAs: S_g = Q_g K^T into accumulator set j % NACC ------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = umma::idesc_bf16_f32(Geo::BM, BN);
            bool ok = mbar_wait(q_full, 0);
            for (int j = 0; ok && j < nt; ++j) {
                const int s = j % NST, as = j % NACC;
                ok = mbar_wait(k_full + 8 * s, (j / NST) & 1);
                if (ok && j >= NACC) ok = mbar_wait(acc_empty + 8 * as, ((j / NACC) - 1) & 1);
                if (!ok) break;
                umma::fence_after_sync();
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t kb = (ks % 4) * 32;  // 16 bf16 along d inside the 128-byte row
                        const uint64_t ad = umma::sdesc_sw128_kmajor(sq + (g * NA + ks / 4) * Geo::Q_ATOM + kb);
                        const uint64_t bd = umma::sdesc_sw128_kmajor(sk + (s * NA + ks / 4) * Geo::K_ATOM + kb);
                        umma::mma_bf16(tmem + (as * G + g) * BN, ad, bd, idesc, ks > 0);
                    }
                umma::commit(k_empty + 8 * s);
                umma::commit(acc_full + 8 * as);
            }
            // every MMA issued has completed before the CTA releases its tensor memory
            umma::commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else {
        // ---- selection: NPART threads per query row i = TMEM lane (warp w reads lane quarter
        // w % 4), the thread of part w / 4 scanning the chunks cc with cc % NPART == w / 4 -----
        const int quarter = warp & 3, part = warp >> 2;
        const int r = quarter * 32 + lane;
        const int tid = threadIdx.x;  // 0 .. NSEL-1
        const int i = i0 + r;
        const bool valid = i < a.n;
        float nl[G];  // -log2(e) * lse of the row's query heads
#pragma unroll
        for (int g = 0; g < G; ++g)
            nl[g] = valid ? -LOG2E * __ldg(a.lse + ((size_t)(row0 + i)) * a.hq + h * G + g) : 0.0f;
        float kw[SFM];
        int kt[SFM];
#pragma unroll
        for (int x = 0; x < SFM; ++x) {
            kw[x] = -1.0f;  // empty slot: below every mass
            kt[x] = 0;
        }
        float L = -INFINITY;
        const float sl2 = a.sl2;
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
        float *myx = listx + tid * G;  // slot c of this thread at myx[c * NSEL * G]
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const int as = j % NACC;
            ok = __all_sync(FULL, mbar_wait(acc_full + 8 * as, (j / NACC) & 1));
            if (!ok) break;
            umma::fence_after_sync();
#pragma unroll 1
            for (int cc = part; cc < BN / 32; cc += Geo::NPART) {
                uint32_t sv[G][32];
#pragma unroll
                for (int g = 0; g < G; ++g) umma::tmem_ld32(tlane + (as * G + g) * BN + cc * 32, sv[g]);
                umma::tmem_wait_ld();
#pragma unroll
                for (int sub = 0; sub < 32; sub += Geo::SUB) {
                    const int t0 = j * BN + cc * 32 + sub;
                    // columns c < SUB of this piece that are causal for the row: c <= i - t0
                    const int lim = valid ? i - t0 : -1;
                    const uint32_t causal = lim >= Geo::SUB - 1 ? (1u << Geo::SUB) - 1u
                                                                : (lim < 0 ? 0u : (2u << lim) - 1u);
                    uint32_t mask = 0;
#pragma unroll
                    for (int c = 0; c < Geo::SUB; ++c) {
                        float mx = -INFINITY;
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float x = fmaf(__uint_as_float(sv[g][sub + c]), sl2, nl[g]);
                            myx[c * Geo::NSEL * G + g] = x;
                            mx = fmaxf(mx, x);
                        }
                        mask |= (mx > L ? 1u : 0u) << c;
                    }
                    mask &= causal;
                    // each lane walks its own candidates (ascending t); the warp loops as long
                    // as its busiest lane
                    while (mask) {
                        const int c = __ffs(mask) - 1;
                        mask &= mask - 1;
                        float sum = 0.0f;
#pragma unroll
                        for (int g = 0; g < G; ++g) sum += ex2(myx[c * Geo::NSEL * G + g]);
                        const float m = sum * (1.0f / G);
                        if (m > kw[SFM - 1]) list_insert_ascending<SFM>(kw, kt, m, t0 + c);
                    }
                    L = skip_bound<SFM>(kw);
                    if constexpr (Geo::NPART > 1) {
                        sbound[r * Geo::NPART + part] = L;
#pragma unroll
                        for (int p = 0; p < Geo::NPART; ++p) L = fmaxf(L, sbound[r * Geo::NPART + p]);
                    }
                }
            }
            umma::fence_before_sync();
            mbar_arrive(acc_empty + 8 * as);
        }
        // the NPART threads of a row merge their lists: parts 1.. hand theirs over in shared
        // memory (the x-value slots, free now), part 0 inserts them and writes the row
        float *hand = listx;  // per part p >= 1: [BM][SFM] masses, then [BM][SFM] positions
        named_barrier_sync(1, Geo::NSEL);  // every scan is done with the slots
        if (part > 0) {
            float *mine = hand + (size_t)(part - 1) * 2 * Geo::BM * SFM;
#pragma unroll
            for (int x = 0; x < SFM; ++x) {
                mine[r * SFM + x] = kw[x];
                mine[Geo::BM * SFM + r * SFM + x] = __int_as_float(kt[x]);
            }
        }
        named_barrier_sync(1, Geo::NSEL);
        if (part == 0 && ok) {
#pragma unroll
            for (int p = 1; p < Geo::NPART; ++p) {
                const float *theirs = hand + (size_t)(p - 1) * 2 * Geo::BM * SFM;
#pragma unroll
                for (int x = 0; x < SFM; ++x) {
                    const float m = theirs[r * SFM + x];
                    if (m > kw[SFM - 1] || (m == kw[SFM - 1] && m >= 0.0f))
                        list_insert<SFM>(kw, kt, m, __float_as_int(theirs[Geo::BM * SFM + r * SFM + x]));
                }
            }
            if (valid) {
                const size_t o = ((size_t)(row0 + i) * a.hkv + h) * a.sf;
                for (int f = 0; f < a.sf; ++f) {
                    // f < sf <= SFM; select by unrolled compare so the list stays in registers
                    float w = 0.0f;
                    int t = 0;
#pragma unroll
                    for (int x = 0; x < SFM; ++x)
                        if (x == f) {
                            w = kw[x];
                            t = kt[x];
                        }
                    const bool kept = w >= 0.0f;
                    a.out_idx[o + f] = kept ? t : 0;
                    a.out_w[o + f] = kept ? w : 0.0f;
                }
            }
        }
    }

    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, Geo::TMEM_COLS);
    }
}

}  // namespace gm
