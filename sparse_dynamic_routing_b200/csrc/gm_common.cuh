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

namespace gm {

constexpr unsigned FULL = 0xffffffffu;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// Device error word of this library (one per device). Bit 0: an active slot indexed
// outside [0, n). Kernels set it with atomicOr and carry on; the host reads and clears it.
__device__ unsigned int g_error_flag;
constexpr unsigned ERR_INDEX_RANGE = 1u;

__device__ __forceinline__ void raise_index_error() { atomicOr(&g_error_flag, ERR_INDEX_RANGE); }

// ---- 16-byte chunks of feature rows -------------------------------------------------------

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

// Sum over an aligned segment of C lanes (C a power of two <= 32); every lane of the
// segment gets the total.
template <int C> __device__ __forceinline__ float seg_sum(float x)
{
#pragma unroll
    for (int off = C / 2; off > 0; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
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
