// gm_bwd_gather.cuh - SEA backward without scatter atomics: dK/dV gathered per target row.
//
// The scatter dK[t_j] += scale dz_j q, dV[t_j] += p_j dO of the SEA backward (the derivative
// of the attention in "Graph Machine: Towards Better Pretraining via Edges", ai.info summary,
// "Key Contributions" item 3) is done as a gather over edges sorted by target instead of as
// fp32 read-modify-write atomics on the gradient rows:
//   1. a count pass counts the active edges of every target row (b, t, h) with integer
//      atomics, and keeps each edge's rank inside its target (the value its atomic returned);
//   2. an exclusive scan of the counts gives each target row its bucket [off[r], off[r+1]);
//   3. the row pass (sea_bwd_tile_kernel with GATHER = true) stores dq and d ln w as usual and
//      writes, for every active edge, a record (target row, source row, scale dz_g and p_g
//      over the group's query heads g) straight to off[target] + rank of its edge;
//   4. the gather pass walks the sorted records in chunks of 32, one warp per chunk: a warp
//      owns every target whose first record lies in its chunk (following it past the chunk
//      end if needed), sums scale dz_g q_g into dK and p_g dO_g into dV, and writes each owned
//      row once; a hot target (more than GATHER_HOT records, edges collapsed onto a few
//      positions) is instead summed by every chunk it spans, each adding its part with fp32
//      atomics into the row the scan zeroed; the target rows nothing points at (count 0) are
//      written as zeros, each warp of the grid taking an equal slice of all target rows.
// The order of records inside a bucket comes from the count pass's integer atomics and
// varies run to run, so dK/dV sums vary in rounding order (not in the set of terms). The scan
// is one launch with a decoupled look-back between its blocks; its waits are bounded.
#pragma once

#include "gm_common.cuh"

namespace gm {

// A sorted record: target row, source edge row (b*n + i)*hkv + h with the target's hot bit in
// bit 31, then scale dz_g and p_g for the G query heads (fp32 bits), padded to whole 16-byte
// words (32 bytes for G = 2), so the row pass writes and the gather pass reads it in full
// sectors.
template <int G> struct Rec {
    static constexpr int WORDS = (2 + 2 * G + 3) / 4 * 4;
};

template <int G>
__device__ __forceinline__ void write_record(int32_t *srec, int32_t pos, uint32_t key, uint32_t row,
                                             const float (&cf)[2 * G])
{
    int32_t w[Rec<G>::WORDS];
    w[0] = (int32_t)key;
    w[1] = (int32_t)row;
#pragma unroll
    for (int x = 0; x < 2 * G; ++x) w[2 + x] = __float_as_int(cf[x]);
#pragma unroll
    for (int x = 2 + 2 * G; x < Rec<G>::WORDS; ++x) w[x] = 0;
    int4 *dst = reinterpret_cast<int4 *>(srec + (size_t)pos * Rec<G>::WORDS);
#pragma unroll
    for (int x = 0; x < Rec<G>::WORDS / 4; ++x) dst[x] = make_int4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
}

template <int G>
__device__ __forceinline__ void read_record(const int32_t *srec, int64_t pos, int32_t &key, int32_t &row,
                                            float (&cf)[2 * G])
{
    int32_t w[Rec<G>::WORDS];
    const int4 *src = reinterpret_cast<const int4 *>(srec + pos * Rec<G>::WORDS);
#pragma unroll
    for (int x = 0; x < Rec<G>::WORDS / 4; ++x) {
        const int4 v = __ldg(src + x);
        w[4 * x] = v.x; w[4 * x + 1] = v.y; w[4 * x + 2] = v.z; w[4 * x + 3] = v.w;
    }
    key = w[0];
    row = w[1];
#pragma unroll
    for (int x = 0; x < 2 * G; ++x) cf[x] = __int_as_float(w[2 + x]);
}

// Caller-provided scratch (sizes in elements; R = B*n*hkv target rows, E = R*s edges). cnt,
// state and ticket are contiguous, the first zero_words int32 words, cleared at every call.
struct GatherWs {
    int32_t *cnt;               // [R]      edges per target row
    unsigned long long *state;  // [nblk]   scan tile words: status << 32 | value
    uint32_t *ticket;           //          scan tiles taken so far
    int32_t *off;               // [R + 1]  bucket offsets; off[R] = number of active edges
    int32_t *rank;              // [E]      an active edge's place inside its target's bucket
    int32_t *srec;              // [E * Rec<G>::WORDS] records sorted by target row
    uint32_t nblk;              // scan tiles of SCAN_TILE rows
    int64_t zero_words;
};

// A target row with more records than this is "hot" (edges collapsed onto a few positions):
// instead of one warp walking all of its records, every chunk sums its own part and adds it
// with fp32 atomics into the row, which the scan zeroes beforehand.
constexpr int GATHER_HOT = 256;

constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_PER_THREAD = 4;
constexpr int SCAN_TILE = SCAN_THREADS * SCAN_PER_THREAD;

__global__ void zero_i32_kernel(int32_t *p, int64_t count)
{
    pdl_trigger();
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

__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.b64 [%0], %1;\n" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.b64 %0, [%1];\n" : "=l"(v) : "l"(p) : "memory");
    return v;
}

constexpr unsigned long long SCAN_AGGREGATE = 1ull << 32, SCAN_PREFIX = 2ull << 32;

// Exclusive scan of the counts into off, in one launch (single-pass scan with decoupled
// look-back; Merrill and Garland, "Single-pass Parallel Prefix Scan with Decoupled Look-back",
// 2016). A block takes the next tile from a ticket, scans its SCAN_TILE counts, publishes the
// tile total at once and the inclusive prefix when it knows it; its prefix is the sum of the
// totals of the tiles before it back to the nearest published prefix. A tile only waits on
// tiles with earlier tickets, whose blocks are running or done, so the wait ends; it is still
// bounded (WAIT_LIMIT_NS, then ERR_WAIT_TIMEOUT and a wrong prefix instead of a hang).
__global__ void __launch_bounds__(SCAN_THREADS) scan_lookback_kernel(const int32_t *cnt, int64_t R,
                                                                     unsigned long long *state, uint32_t *ticket,
                                                                     int32_t *off, float *dk, float *dv, int D,
                                                                     int accumulate)
{
    __shared__ uint32_t s_tile;
    __shared__ int32_t s_prefix;
    pdl_wait();  // the counts
    pdl_trigger();
    if (threadIdx.x == 0) s_tile = atomicAdd(ticket, 1u);
    __syncthreads();
    const uint32_t tile = s_tile;
    const int64_t base = (int64_t)tile * SCAN_TILE + (int64_t)threadIdx.x * SCAN_PER_THREAD;
    int32_t c[SCAN_PER_THREAD], sum = 0;
#pragma unroll
    for (int k = 0; k < SCAN_PER_THREAD; ++k) {
        c[k] = base + k < R ? cnt[base + k] : 0;
        sum += c[k];
    }
    int32_t total;
    const int32_t ex = block_exclusive_scan(sum, total);
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int32_t prefix = 0;
        if (tile == 0) {
            if (lane == 0) st_release_u64(state, SCAN_PREFIX | (uint32_t)total);
        } else {
            if (lane == 0) st_release_u64(state + tile, SCAN_AGGREGATE | (uint32_t)total);
            const unsigned long long t0 = globaltimer_ns();
            bool late = false;
            for (int64_t j = (int64_t)tile - 1;; j -= 32) {
                // lane L reads tile j - L; tiles before 0 count as a zero prefix
                const int64_t mine = j - lane;
                unsigned long long st = mine >= 0 ? ld_acquire_u64(state + mine) : SCAN_PREFIX;
                while (true) {  // every exit is warp-uniform
                    const bool pending = (st >> 32) == 0;
                    if (!__any_sync(FULL, pending)) break;
                    if (__any_sync(FULL, globaltimer_ns() - t0 > WAIT_LIMIT_NS)) {
                        late = true;
                        break;
                    }
                    if (pending) st = ld_acquire_u64(state + mine);
                }
                if (late) break;
                const unsigned pre = __ballot_sync(FULL, st >= SCAN_PREFIX);
                const int stop = pre ? __ffs(pre) - 1 : 31;  // nearest published prefix
                int32_t v = lane <= stop ? (int32_t)(uint32_t)st : 0;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
                prefix += v;
                if (pre) break;
            }
            if (late && lane == 0) atomicOr(&g_error_flag, ERR_WAIT_TIMEOUT);
            if (lane == 0) st_release_u64(state + tile, SCAN_PREFIX | (uint32_t)(prefix + total));
        }
        if (lane == 0) s_prefix = prefix;
    }
    __syncthreads();
    int32_t run = s_prefix + ex;
#pragma unroll
    for (int k = 0; k < SCAN_PER_THREAD; ++k) {
        if (base + k < R) off[base + k] = run;
        run += c[k];
    }
    if (tile == gridDim.x - 1 && threadIdx.x == 0) off[R] = s_prefix + total;
    // hot rows receive atomic additions in the gather pass: start them at zero
    if (!accumulate) {
#pragma unroll
        for (int k = 0; k < SCAN_PER_THREAD; ++k) {
            if (base + k < R && c[k] > GATHER_HOT) {
                float4 *pk = reinterpret_cast<float4 *>(dk + (size_t)(base + k) * D);
                float4 *pv = reinterpret_cast<float4 *>(dv + (size_t)(base + k) * D);
                for (int x = 0; x < D / 4; ++x) {
                    pk[x] = make_float4(0.f, 0.f, 0.f, 0.f);
                    pv[x] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
    }
}

// Count: active edges per target row, and each active edge's rank among them (range errors
// are reported by the row pass, which applies the same activity test). One thread per edge
// row: its slots' atomics are independent and in flight together.
template <int S1M>
__global__ void edge_count_kernel(const int32_t *idx, const float *w, int n, RowMap map, int s, uint32_t rows,
                                 int hkv, int32_t *cnt, int32_t *rank)
{
    pdl_wait();  // the zeroed counters
    pdl_trigger();
    for (uint32_t row = blockIdx.x * blockDim.x + threadIdx.x; row < rows; row += gridDim.x * blockDim.x) {
        uint32_t seq_base, h;
        map.split(row, seq_base, h);
        int32_t t[S1M];
        float we[S1M];
#pragma unroll
        for (int r = 0; r < S1M; ++r) {
            we[r] = r < s ? __ldg(w + (size_t)row * s + r) : 0.0f;
            t[r] = r < s ? __ldg(idx + (size_t)row * s + r) : 0;
        }
#pragma unroll
        for (int r = 0; r < S1M; ++r)
            if (we[r] > 0.0f && (uint32_t)t[r] < (uint32_t)n)
                rank[(size_t)row * s + r] = atomicAdd(cnt + (seq_base + (uint32_t)t[r]) * (uint32_t)hkv + h, 1);
    }
}

// Gather: one warp per chunk of 32 sorted records. Lanes [0, C) own dK chunk c, lanes
// [C, 2C) dV chunk c (16 bytes of every feature row). Each lane stages exactly the q (or
// dO) chunks it will read with cp.async, U records per group, P groups ahead.
template <typename T, int D, int G, int WPB, int U, int P>
__global__ void __launch_bounds__(WPB * 32) sea_bwd_gather_kernel(const void *q, const void *dout, float *dk, float *dv,
                                                                 GatherWs ws, uint32_t R, int accumulate)
{
    pdl_wait();  // the records of the row pass
    constexpr int VEC = Vec<T>::N, C = D / VEC, NP = VEC / 2, ROW = D * (int)sizeof(T);
    constexpr int GROUP = U * G * 32 * 16;  // bytes of one group of records, all lanes
    static_assert(2 * C <= 32, "dK and dV halves fit one warp");
    static_assert(2 * G <= 8, "coefficients of one record fit two 16-byte loads");
    extern __shared__ __align__(16) char smem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    char *ring = smem + (size_t)wid * P * GROUP;
    const int role = lane / C, c = lane % C;
    const bool working = role < 2;
    const char *src = static_cast<const char *>(role == 0 ? q : dout);
    float *dst_base = (role == 0 ? dk : dv) + c * VEC;

    const int total = ws.off[R];
    const int64_t chunk = (int64_t)blockIdx.x * WPB + wid;
    const int64_t p0 = chunk * 32;

    float2 acc[NP];
#pragma unroll
    for (int x = 0; x < NP; ++x) acc[x] = make_float2(0.0f, 0.0f);

    // acc -> row t: stored (added to it when accumulating), or for a hot row added with fp32
    // atomics (the row was zeroed by the scan unless accumulating)
    auto write_row = [&](uint32_t t, bool hot) {
        if (!working) return;
        float *dst = dst_base + (size_t)t * D;
#pragma unroll
        for (int x = 0; x < NP; x += 2) {
            float4 o = make_float4(acc[x].x, acc[x].y, acc[x + 1].x, acc[x + 1].y);
            if (hot) {
                atomicAdd(reinterpret_cast<float4 *>(dst + 2 * x), o);
                continue;
            }
            if (accumulate) {
                const float4 old = *reinterpret_cast<const float4 *>(dst + 2 * x);
                o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
            }
            *reinterpret_cast<float4 *>(dst + 2 * x) = o;
        }
    };
    // The rows nothing points at (count 0) are zeroed by slices, every warp of the grid taking
    // an equal share of the rows whatever its chunk holds: long runs of empty targets (the late
    // positions of a sequence under uniform causal edges) never fall on one warp.
    auto zero_slice = [&]() {
        if (accumulate) return;
        const uint32_t nwarps = gridDim.x * WPB;
        const uint32_t per = (R + nwarps - 1) / nwarps;
        const uint32_t z0 = (uint32_t)chunk * per, z1 = min(z0 + per, R);
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        for (uint32_t b0 = z0; b0 < z1; b0 += 32) {
            const uint32_t t = b0 + lane;
            unsigned empty = __ballot_sync(FULL, t < z1 && __ldg(ws.cnt + t) == 0);
            while (empty) {  // warp-uniform
                const uint32_t te = b0 + (uint32_t)(__ffs(empty) - 1);
                empty &= empty - 1;
                if (working) {
                    float *dst = dst_base + (size_t)te * D;
#pragma unroll
                    for (int x = 0; x < VEC; x += 4) *reinterpret_cast<float4 *>(dst + x) = z;
                }
            }
        }
    };

    // the record walk; its early exits leave the zero slice to run after it
    auto walk = [&]() {
        if (p0 >= total) return;  // warp-uniform

        // the chunk's records (window [wbase, wbase + 32) of the sorted list, one per lane)
        int64_t wbase = p0;
        int wlen = (int)min((int64_t)32, (int64_t)total - wbase);
        int32_t mkey = -1, mrow = 0;
        bool mhot = false;
        float mcf[2 * G];
        auto load_window = [&]() {
            mkey = -1;
            mrow = 0;
    #pragma unroll
            for (int x = 0; x < 2 * G; ++x) mcf[x] = 0.0f;
            if (lane < wlen) read_record<G>(ws.srec, wbase + lane, mkey, mrow, mcf);
            mhot = mrow < 0;  // bit 31: the target is hot
            mrow &= 0x7fffffff;
        };
        load_window();
        const int32_t prev_key = p0 > 0 ? __ldg(ws.srec + (p0 - 1) * Rec<G>::WORDS) : -1;

        // a leading run that continues the previous chunk's last target belongs to that chunk,
        // unless the target is hot: then every chunk sums its own part of it
        const int start = __popc(__ballot_sync(FULL, lane < wlen && mkey == prev_key));
        const bool lead_hot = start > 0 && __shfl_sync(FULL, mhot, 0);  // warp-uniform
        const int first = lead_hot ? 0 : start;
        if (first == wlen) return;  // warp-uniform

        uint32_t cur = (uint32_t)__shfl_sync(FULL, mkey, first);
        bool cur_hot = lead_hot;  // a target starting inside the chunk is settled at its end

        // Accumulate records [lo, hi) of the current window, U per copy group, P groups in
        // flight; a change of key writes the finished target (and zeroes any empty rows between).
        auto process = [&](int lo, int hi) {
            auto issue = [&](int grp) {
    #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int k = lo + grp * U + u;
                    const int32_t row = __shfl_sync(FULL, mrow, k & 31);
                    if (k < hi && working) {
                        char *slot = ring + (grp % P) * GROUP + ((u * G) * 32 + lane) * 16;
    #pragma unroll
                        for (int g = 0; g < G; ++g)
                            cp_async16(slot + g * 32 * 16, src + ((size_t)row * G + g) * ROW + c * 16);
                    }
                }
                cp_async_commit();
            };
            const int ngroups = (hi - lo + U - 1) / U;
    #pragma unroll
            for (int grp = 0; grp < P; ++grp) issue(grp);
            for (int grp = 0; grp < ngroups; ++grp) {
                cp_async_wait<P - 1>();
    #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int k = lo + grp * U + u;
                    const uint32_t key = (uint32_t)__shfl_sync(FULL, mkey, k & 31);
                    float cf[2 * G];
    #pragma unroll
                    for (int x = 0; x < 2 * G; ++x) cf[x] = __shfl_sync(FULL, mcf[x], k & 31);
                    if (k >= hi) break;  // warp-uniform
                    if (key != cur) {    // warp-uniform: a new target starts here
                        write_row(cur, cur_hot);
                        cur_hot = false;  // it starts inside the window
    #pragma unroll
                        for (int x = 0; x < NP; ++x) acc[x] = make_float2(0.0f, 0.0f);
                        cur = key;
                    }
                    if (working) {
                        const char *slot = ring + (grp % P) * GROUP + ((u * G) * 32 + lane) * 16;
    #pragma unroll
                        for (int g = 0; g < G; ++g) {
                            float f[VEC];
                            unpack<T>(*reinterpret_cast<const uint4 *>(slot + g * 32 * 16), f);
                            const float k2 = role == 0 ? cf[g] : cf[G + g];
                            const float2 kk = make_float2(k2, k2);
    #pragma unroll
                            for (int x = 0; x < NP; ++x) acc[x] = __ffma2_rn(kk, make_float2(f[2 * x], f[2 * x + 1]), acc[x]);
                        }
                    }
                }
                issue(grp + P);
            }
            cp_async_wait<0>();
        };

        process(first, wlen);
        // the last target may continue past the chunk: a hot one is left to the chunks it
        // spans (each adds its part), any other is followed window by window with the same
        // pipeline
        int64_t pos = wbase + wlen;
        if (!cur_hot) cur_hot = __shfl_sync(FULL, mhot, wlen - 1);  // the last record is cur's
        while (!cur_hot && wlen == 32 && pos < total) {
            wbase = pos;
            wlen = (int)min((int64_t)32, (int64_t)total - wbase);
            load_window();
            const int run = __popc(__ballot_sync(FULL, lane < wlen && (uint32_t)mkey == cur));
            if (run == 0) break;  // warp-uniform
            process(0, run);
            pos = wbase + run;
            if (run < wlen) break;  // the target ended inside this window
        }
        write_row(cur, cur_hot);
    };
    walk();
    zero_slice();
}

}  // namespace gm
