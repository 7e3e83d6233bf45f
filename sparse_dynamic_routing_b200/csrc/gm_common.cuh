// gm_common.cuh - shared device helpers of the Graph Machine sparse-layer kernels.
//
// Work decomposition used by every kernel: one warp per edge row (b, i, h), i.e. per
// (token, KV head). Feature rows are moved in 16-byte chunks: a row of d elements is
// C = d * sizeof(T) / 16 chunks, and a warp covers RPI = 32 / C rows per pass ("item"),
// lane l handling chunk l % C of row l / C. The G query heads of a KV head therefore take
// NI = ceil(G / RPI) items per lane, and every per-row dot product is a shuffle reduction
// inside an aligned segment of C lanes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

// Launch shape: warps (edge rows) per block and minimum resident blocks per SM of the
// attention kernels (the latter caps registers per thread at 65536 / (32 * WPB * MINB)).
#ifndef GM_WPB_SEA
#define GM_WPB_SEA 4
#endif
#ifndef GM_WPB_BWD
#define GM_WPB_BWD 4
#endif
#ifndef GM_FWD_MINB
#define GM_FWD_MINB 8
#endif
#ifndef GM_BWD_MINB
#define GM_BWD_MINB 6
#endif

namespace gm {

constexpr unsigned FULL = 0xffffffffu;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// Device error word of this library (one per device). Bit 0: an active slot indexed
// outside [0, n). Kernels set it with atomicOr and carry on; the host reads and clears it.
// Bit 1: a bounded wait on an asynchronous copy or tensor-core operation ran out of time (the
// kernel gave up on its remaining work). Bit 2: see ERR_EDGE_INVALID.
__device__ unsigned int g_error_flag;
constexpr unsigned ERR_INDEX_RANGE = 1u;
constexpr unsigned ERR_WAIT_TIMEOUT = 2u;
// Bit 2 (checked builds only): an input edge had a negative or non-finite weight, or an
// active index beyond its row's own position.
constexpr unsigned ERR_EDGE_INVALID = 4u;

__device__ __forceinline__ void raise_index_error() { atomicOr(&g_error_flag, ERR_INDEX_RANGE); }

// ---- integer division by a launch-invariant divisor ---------------------------------------
//
// Row decomposition (row -> b, i, h) divides by n and by the head count on every warp; a
// hardware integer divide is a long instruction sequence, so the host precomputes a
// multiplier and shift (Granlund & Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994, section 4) and the device divides with one multiply-high,
// a subtract, an add and two shifts. Exact for every 32-bit unsigned dividend.
struct FastDiv {
    uint32_t d;      // divisor (>= 1)
    uint32_t mul;    // magic multiplier
    uint32_t s1, s2; // shifts

    FastDiv() = default;
    __host__ explicit FastDiv(uint32_t divisor) : d(divisor)
    {
        uint32_t l = 0;
        while (l < 32 && (uint64_t(1) << l) < divisor) ++l;  // l = ceil(log2 d)
        // mul = floor(2^32 * (2^l - d) / d) + 1
        mul = (uint32_t)(((uint64_t(1) << 32) * ((uint64_t(1) << l) - divisor)) / divisor + 1);
        s1 = l > 0 ? 1 : 0;
        s2 = l > 0 ? l - 1 : 0;
    }
    __device__ __forceinline__ uint32_t div(uint32_t x) const
    {
        const uint32_t t = __umulhi(x, mul);
        return (t + ((x - t) >> s1)) >> s2;
    }
};

// Edge row -> (sequence start b*n, head h), for row = (b*n + i)*heads + h < 2^31.
struct RowMap {
    FastDiv heads, n;
    __device__ __forceinline__ void split(uint32_t row, uint32_t &seq_base, uint32_t &h) const
    {
        const uint32_t bi = heads.div(row);
        h = row - bi * heads.d;
        seq_base = n.div(bi) * n.d;  // b * n
    }
};

// ---- 16-byte chunks of feature rows -------------------------------------------------------

// Fast base-2 exponential / logarithm (MUFU; relative error ~2^-22, subnormals kept).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x)
{
    float y;
    asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Fast reciprocal (MUFU; relative error ~2^-23). Used only on softmax sums, which are >= 1.
__device__ __forceinline__ float rcp_fast(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };

// Read-only 16-byte load through the non-coherent path (inputs never alias outputs).
__device__ __forceinline__ uint4 ld16(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// Streaming 16-byte load (data read once: evict first).
__device__ __forceinline__ uint4 ld16_stream(const void *p) { return __ldcs(reinterpret_cast<const uint4 *>(p)); }

template <typename T> __device__ __forceinline__ void unpack(const uint4 &u, float (&f)[Vec<T>::N]);

template <> __device__ __forceinline__ void unpack<float>(const uint4 &u, float (&f)[4])
{
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}

// bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 pattern.
template <> __device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4 &u, float (&f)[8])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        f[2 * x] = __uint_as_float(w[x] << 16);
        f[2 * x + 1] = __uint_as_float(w[x] & 0xffff0000u);
    }
}

template <typename T> __device__ __forceinline__ uint4 pack(const float (&f)[Vec<T>::N]);

template <> __device__ __forceinline__ uint4 pack<float>(const float (&f)[4])
{
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}

// fp32 -> bf16 rounds to nearest even.
template <> __device__ __forceinline__ uint4 pack<__nv_bfloat16>(const float (&f)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * x], f[2 * x + 1]);
        w[x] = *reinterpret_cast<uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// 16-byte asynchronous global -> shared copy (L2 only), its commit and wait (no spin loop:
// cp.async.wait_group blocks in hardware until this thread's older groups have landed).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
// The same copy with a source size of 0 or 16 bytes: 0 reads nothing and writes 16 zero bytes
// (an inactive slot's stage then holds zeros, so it can be computed on like an active one).
__device__ __forceinline__ void cp_async16_zfill(void *smem, const void *gmem, bool copy)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(copy ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream serialization
// may start while the kernel before it on the stream is still running; pdl_wait() blocks
// until that kernel has completed and its memory is visible (a no-op for a kernel launched
// the ordinary way). pdl_trigger() lets the next such kernel launch early. Both are hardware
// waits, not spin loops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---- shared-memory barriers (mbarrier) with bounded waits --------------------------------
//
// Completion of asynchronous copies (TMA) and tensor-core operations is counted on 64-bit
// shared-memory barriers. Every wait is bounded: after WAIT_LIMIT_NS without completion the
// waiting thread sets ERR_WAIT_TIMEOUT and reports failure, so a lost completion cannot hang
// the device.

constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;  // one second

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// Makes barrier initialisation visible to the asynchronous proxy (copy engine, tensor cores).
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(bar) : "memory");
}
// Announces `bytes` of incoming asynchronous copies and arrives once.
__device__ __forceinline__ void mbar_arrive_expect(uint32_t bar, uint32_t bytes)
{
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}

// Waits for the completion of the barrier phase with the given parity. Returns false, with
// ERR_WAIT_TIMEOUT set, if that takes longer than WAIT_LIMIT_NS.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            atomicOr(&g_error_flag, ERR_WAIT_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Dot product of a 16-byte chunk of q (as fp32 pairs) with a chunk of k: even and odd
// elements accumulate separately with packed fp32x2 FMAs, then the two halves are added.
// Every SEA kernel uses this same order, so all paths give identical bits.
template <int NP> __device__ __forceinline__ float chunk_dot(const float2 (&q2)[NP], const float (&kf)[2 * NP])
{
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int x = 0; x < NP; ++x) acc = __ffma2_rn(q2[x], make_float2(kf[2 * x], kf[2 * x + 1]), acc);
    return acc.x + acc.y;
}

// Sum over an aligned segment of C lanes (C a power of two <= 32); every lane of the
// segment gets the total.
template <int C> __device__ __forceinline__ float seg_sum(float x)
{
#pragma unroll
    for (int off = C / 2; off > 0; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
    return x;
}

// seg_sum of two values at once (packed fp32x2 add per step).
template <int C> __device__ __forceinline__ float2 seg_sum2(float2 x)
{
#pragma unroll
    for (int off = C / 2; off > 0; off >>= 1) {
        const float2 y = make_float2(__shfl_xor_sync(FULL, x.x, off), __shfl_xor_sync(FULL, x.y, off));
        x = __fadd2_rn(x, y);
    }
    return x;
}

// Sum across the RPI segments that share a chunk index (lanes c, c + C, c + 2C, ...).
template <int C> __device__ __forceinline__ float cross_seg_sum(float x)
{
#pragma unroll
    for (int off = C; off < 32; off <<= 1) x += __shfl_xor_sync(FULL, x, off);
    return x;
}

// Compile-time geometry of one (dtype, head_dim, group) instantiation.
template <typename T, int D, int G> struct Geom {
    static constexpr int VEC = Vec<T>::N;        // elements per 16-byte chunk
    static constexpr int C = D / VEC;            // chunks per row
    static constexpr int RPI = 32 / C;           // rows per warp pass
    static constexpr int NI = (G + RPI - 1) / RPI;  // passes per lane for G query heads
    static_assert(C >= 1 && C <= 32 && (C & (C - 1)) == 0, "row must be 1..32 chunks");
};

}  // namespace gm
