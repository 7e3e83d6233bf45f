// gm_bwd_gather.cuh - SEA backward without scatter atomics: dK/dV gathered per target row.
//
// The scatter dK[t_j] += scale dz_j q, dV[t_j] += p_j dO of the SEA backward (the derivative
// of the attention in "Graph Machine: Towards Better Pretraining via Edges", ai.info summary,
// "Key Contributions" item 3) is done as a gather over a reverse edge index instead of as
// fp32 read-modify-write atomics on the gradient rows:
//   1. the row pass (sea_bwd_tile_kernel with GATHER = true) stores dq and d ln w as usual and,
//      per active edge e = row * s + j, a record of 2G floats (scale dz_g, then p_g, over the
//      query heads g of the group), and counts the edges of every target row (b, t, h) with
//      an integer atomic;
//   2. an exclusive scan of the counts gives each target row its bucket [off[r], off[r+1]);
//   3. the fill pass drops every active edge id into its target's bucket;
//   4. the gather pass (one warp per run of consecutive target rows) sums scale dz_g q_g over
//      each bucket into dK and p_g dO_g into dV, and writes each row exactly once - zeros
//      where nothing points.
// The order of edges inside a bucket comes from integer atomics and varies run to run, so
// dK/dV sums vary in rounding order (not in the set of terms), as with atomics. There are no
// spin-waits: the scan is reduce -> scan of block totals -> rescan, three launches.
#pragma once

#include "gm_common.cuh"

namespace gm {

// Caller-provided scratch (sizes in elements; R = B*n*hkv target rows, E = R*s edges).
struct GatherWs {
    int32_t *cnt;     // [R]      edge count per target row (left zeroed by the fill pass)
    int32_t *off;     // [R + 1]  bucket offsets
    int32_t *list;    // [E]      edge ids grouped by target row
    float *coef;      // [E * 2G] per-edge coefficients
    int32_t *bsum;    // [nblk]   scan block totals, then their offsets
    uint32_t nblk;    // scan blocks of SCAN_TILE rows
};

constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_PER_THREAD = 4;
constexpr int SCAN_TILE = SCAN_THREADS * SCAN_PER_THREAD;

__global__ void zero_i32_kernel(int32_t *p, int64_t count)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0;
}

// Block-wide exclusive scan of one value per thread; returns the prefix, sets `total`.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t &total)
{
    __shared__ int32_t warp_tot[SCAN_THREADS / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t y = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int32_t t = lane < SCAN_THREADS / 32 ? warp_tot[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t y = __shfl_up_sync(FULL, t, off);
            if (lane >= off) t += y;
        }
        if (lane < SCAN_THREADS / 32) warp_tot[lane] = t;  // inclusive warp offsets
    }
    __syncthreads();
    total = warp_tot[SCAN_THREADS / 32 - 1];
    const int32_t before = wid > 0 ? warp_tot[wid - 1] : 0;
    __syncthreads();  // warp_tot is reused by the next call
    return before + incl - v;
}

// Scan step 1: totals of SCAN_TILE-row blocks of the counts.
__global__ void __launch_bounds__(SCAN_THREADS) scan_block_sums_kernel(const int32_t *cnt, int64_t R, int32_t *bsum)
{
    const int64_t base = (int64_t)blockIdx.x * SCAN_TILE + (int64_t)threadIdx.x * SCAN_PER_THREAD;
    int32_t s = 0;
#pragma unroll
    for (int k = 0; k < SCAN_PER_THREAD; ++k)
        if (base + k < R) s += cnt[base + k];
    int32_t total;
    block_exclusive_scan(s, total);
    if (threadIdx.x == 0) bsum[blockIdx.x] = total;
}

// Scan step 2 (one block): exclusive scan of the block totals in place; off[R] = grand total.
__global__ void __launch_bounds__(SCAN_THREADS) scan_block_offsets_kernel(int32_t *bsum, uint32_t nblk, int32_t *off_end)
{
    int32_t carry = 0;
    for (uint32_t base = 0; base < nblk; base += SCAN_THREADS) {
        const uint32_t i = base + threadIdx.x;
        const int32_t v = i < nblk ? bsum[i] : 0;
        int32_t total;
        const int32_t ex = block_exclusive_scan(v, total);
        if (i < nblk) bsum[i] = carry + ex;
        carry += total;
    }
    if (threadIdx.x == 0) *off_end = carry;
}

// Scan step 3: off[r] = block offset + exclusive prefix inside the block.
__global__ void __launch_bounds__(SCAN_THREADS) scan_apply_kernel(const int32_t *cnt, int64_t R, const int32_t *bsum, int32_t *off)
{
    const int64_t base = (int64_t)blockIdx.x * SCAN_TILE + (int64_t)threadIdx.x * SCAN_PER_THREAD;
    int32_t c[SCAN_PER_THREAD], s = 0;
#pragma unroll
    for (int k = 0; k < SCAN_PER_THREAD; ++k) {
        c[k] = base + k < R ? cnt[base + k] : 0;
        s += c[k];
    }
    int32_t total;
    int32_t run = bsum[blockIdx.x] + block_exclusive_scan(s, total);
#pragma unroll
    for (int k = 0; k < SCAN_PER_THREAD; ++k) {
        if (base + k < R) off[base + k] = run;
        run += c[k];
    }
}

// Fill: every active edge id into its target's bucket (positions from the remaining count).
__global__ void bucket_fill_kernel(const int32_t *idx, const float *w, int s, int n, RowMap map,
                                   FastDiv sdiv, int64_t E, int hkv, const int32_t *off, int32_t *cnt,
                                   int32_t *list)
{
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < E; e += (int64_t)gridDim.x * blockDim.x) {
        const float we = w[e];
        const int32_t t = idx[e];
        if (!(we > 0.0f) || t < 0 || t >= n) continue;  // inactive (range errors were reported by the row pass)
        const uint32_t row = sdiv.div((uint32_t)e);
        uint32_t seq_base, h;
        map.split(row, seq_base, h);
        const uint32_t key = (seq_base + (uint32_t)t) * (uint32_t)hkv + h;
        const int32_t rank = atomicSub(cnt + key, 1) - 1;
        list[off[key] + rank] = (int32_t)e;
    }
}

// Gather: one warp per run of TPW consecutive target rows [r0, r0 + TPW). Lanes [0, C) own
// dK chunk c, lanes [C, 2C) dV chunk c. The run's bucket offsets and up to 32 of its edge ids
// are fetched with one coalesced load each; the edges are then taken U at a time straight
// across target boundaries (every load of a group issued before any is used), and a target's
// row is written when the walk passes its end - zeros for a target nothing points at.
template <typename T, int D, int G, int WPB, int TPW, int U>
__global__ void __launch_bounds__(WPB * 32) sea_bwd_gather_kernel(const void *q, const void *dout, float *dk, float *dv,
                                                                 GatherWs ws, FastDiv sdiv, uint32_t R, int accumulate)
{
    constexpr int VEC = Vec<T>::N, C = D / VEC, NP = VEC / 2;
    static_assert(2 * C <= 32 && TPW < 32, "dK and dV halves fit one warp");
    const int lane = threadIdx.x & 31;
    const uint32_t run = blockIdx.x * WPB + (threadIdx.x >> 5);
    const uint32_t r0 = run * TPW;
    if (r0 >= R) return;  // warp-uniform
    const int nt = (int)min((uint32_t)TPW, R - r0);
    const int role = lane / C, c = lane % C;
    const bool working = role < 2;
    const T *src = static_cast<const T *>(role == 0 ? q : dout);
    float *dst_base = (role == 0 ? dk : dv) + c * VEC;

    // bucket boundaries of the run: lane L holds off[r0 + L], L <= nt
    const int32_t my_off = lane <= nt ? __ldg(ws.off + r0 + lane) : 0;
    const int beg = __shfl_sync(FULL, my_off, 0), end = __shfl_sync(FULL, my_off, nt);
    const int32_t my_e = beg + lane < end ? __ldg(ws.list + beg + lane) : 0;

    float2 acc[NP];
#pragma unroll
    for (int x = 0; x < NP; ++x) acc[x] = make_float2(0.0f, 0.0f);
    int cur = 0;                                    // target of the run being accumulated
    int cur_end = __shfl_sync(FULL, my_off, 1);     // its bucket end

    auto flush = [&]() {  // write target `cur` and move to the next one
        if (working) {
            float *dst = dst_base + (size_t)(r0 + cur) * D;
#pragma unroll
            for (int x = 0; x < NP; x += 2) {
                float4 o = make_float4(acc[x].x, acc[x].y, acc[x + 1].x, acc[x + 1].y);
                if (accumulate) {
                    const float4 old = *reinterpret_cast<const float4 *>(dst + 2 * x);
                    o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
                }
                *reinterpret_cast<float4 *>(dst + 2 * x) = o;
            }
        }
#pragma unroll
        for (int x = 0; x < NP; ++x) acc[x] = make_float2(0.0f, 0.0f);
        ++cur;
        cur_end = __shfl_sync(FULL, my_off, (cur + 1) & 31);
    };

    for (int i = beg; i < end; i += U) {
        int32_t e[U];
        uint4 raw[U][G];
        float cf[U][G];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int k = i + u - beg;
            const int32_t from_reg = __shfl_sync(FULL, my_e, k & 31);
            e[u] = i + u >= end ? -1 : (k < 32 ? from_reg : __ldg(ws.list + i + u));
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                raw[u][g] = make_uint4(0, 0, 0, 0);
                cf[u][g] = 0.0f;
            }
            if (e[u] >= 0 && working) {
                const uint32_t row = sdiv.div((uint32_t)e[u]);
                const float *rec = ws.coef + (size_t)e[u] * (2 * G) + role * G;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    cf[u][g] = __ldg(rec + g);
                    raw[u][g] = ld16(src + ((size_t)row * G + g) * D + c * VEC);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (i + u >= end) break;                 // warp-uniform
            while (i + u >= cur_end && cur < nt) flush();  // warp-uniform: targets that ended here
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float f[VEC];
                unpack<T>(raw[u][g], f);
                const float2 k2 = make_float2(cf[u][g], cf[u][g]);
#pragma unroll
                for (int x = 0; x < NP; ++x) acc[x] = __ffma2_rn(k2, make_float2(f[2 * x], f[2 * x + 1]), acc[x]);
            }
        }
    }
    while (cur < nt) flush();  // the last target, and any empty ones after it
}

}  // namespace gm
