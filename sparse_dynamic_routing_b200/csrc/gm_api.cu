// gm_api.cu - host side of the C ABI declared in include/gm.h: argument checks, dispatch to
// the kernel instantiation for (dtype, head_dim, GQA group), launch on the caller's stream.
#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "../../include/gm.h"
#include "gm_bwd_gather.cuh"
#include "gm_bwd_tile.cuh"
#include "gm_common.cuh"
#include "gm_dense_refresh.cuh"
#include "gm_fused_tile.cuh"
#include "gm_leg.cuh"
#include "gm_leg_tile.cuh"
#include "gm_sea.cuh"
#include "gm_sea_bwd.cuh"
#include "gm_ser.cuh"
#include "gm_ser_bwd.cuh"
#include "gm_ser_chain.cuh"

namespace {

using gm::SeaArgs;
using gm::SeaBwdArgs;
using gm::SerArgs;

constexpr int WPB_SER = 8;   // warps (edge rows) per block
constexpr int WPB_SER_THREAD = 4;  // warps per block of the thread-per-row SER backward
constexpr int WPB_SEA = GM_WPB_SEA;
constexpr int WPB_BWD = GM_WPB_BWD;
constexpr int MAX_SLOTS = 32;
constexpr int64_t MAX_ROWS = (int64_t)1 << 31;  // edge rows B*n*heads indexed in 32 bits

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline gm_status launched()
{
    return cudaGetLastError() == cudaSuccess ? GM_OK : GM_ERR_CUDA;
}

inline unsigned blocks_for(int64_t rows, int wpb) { return (unsigned)((rows + wpb - 1) / wpb); }

inline gm::RowMap row_map(int heads, int n)
{
    return gm::RowMap{gm::FastDiv((uint32_t)heads), gm::FastDiv((uint32_t)n)};
}

gm_status check_ser(const int32_t *a1_idx, const float *a1_w, int s2, const int32_t *a2_idx,
                    const float *a2_w, int s3, int s1, int B, int n, int k)
{
    if (B < 0 || n < 0 || k < 1) return GM_ERR_INVALID_ARG;
    if (s1 < 1 || s2 < 1 || s3 < 1 || s1 > MAX_SLOTS || s2 * s3 > MAX_SLOTS) return GM_ERR_INVALID_ARG;
    if ((int64_t)B * n == 0) return GM_OK;
    if ((int64_t)B * n * k >= MAX_ROWS) return GM_ERR_UNSUPPORTED;
    if (!a1_idx || !a1_w || !a2_idx || !a2_w) return GM_ERR_INVALID_ARG;
    return GM_OK;
}

// Refresh edges of the referral: sf slots per row joining the s2*s3 path candidates.
gm_status check_refresh(const int32_t *f_idx, const float *f_w, int sf, int s2, int s3, int64_t rows)
{
    if (sf < 1 || s2 * s3 + sf > MAX_SLOTS) return GM_ERR_INVALID_ARG;
    if (rows > 0 && (!f_idx || !f_w)) return GM_ERR_INVALID_ARG;
    return GM_OK;
}

// Arguments of a multi-step referral: legs[0] is the second leg of the first step, legs[1..]
// the chain (nlegs in 1..GM_MAX_CHAIN). Fills a SerArgs for the chain kernels.
gm_status chain_args(const int32_t *a1_idx, const float *a1_w, int s2,
                     const int32_t *const *leg_idx, const float *const *leg_w, int nlegs, int s3,
                     int s_mid, int s1, int B, int n, int k, SerArgs &a)
{
    if (nlegs < 1 || nlegs > GM_MAX_CHAIN || !leg_idx || !leg_w) return GM_ERR_INVALID_ARG;
    if (s_mid < 1 || s_mid > MAX_SLOTS || s_mid * s3 > MAX_SLOTS) return GM_ERR_INVALID_ARG;
    gm_status st = check_ser(a1_idx, a1_w, s2, leg_idx[0], leg_w[0], s3, s1, B, n, k);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    for (int m = 0; m < nlegs; ++m)
        if (!leg_idx[m] || !leg_w[m]) return GM_ERR_INVALID_ARG;
    a.a1_idx = a1_idx;
    a.a1_w = a1_w;
    a.a2_idx = leg_idx[0];
    a.a2_w = leg_w[0];
    for (int m = 1; m < nlegs; ++m) {
        a.chain_idx[m - 1] = leg_idx[m];
        a.chain_w[m - 1] = leg_w[m];
    }
    a.nchain = nlegs - 1;
    a.s_mid = s_mid;
    a.s1 = s1;
    a.s2 = s2;
    a.s3 = s3;
    a.n = n;
    a.k = k;
    a.rows = (uint32_t)((int64_t)B * n * k);
    a.map = row_map(k, n);
    return GM_OK;
}

constexpr int WPB_LEG = 8;   // warps (tokens) per block of the leg kernels

gm_status check_leg(const int32_t *e_idx, const float *e_w, int s0, const float *mix1,
                    const float *mix2, int64_t mix_token_stride, int s2, int s3, int B, int n,
                    int k)
{
    if (B < 0 || n < 0 || k < 1 || s0 < 1 || s2 < 1 || s3 < 1) return GM_ERR_INVALID_ARG;
    if (k * s0 > MAX_SLOTS || s2 > MAX_SLOTS || s3 > MAX_SLOTS) return GM_ERR_INVALID_ARG;
    if (mix_token_stride != 0 && mix_token_stride != (int64_t)k * k) return GM_ERR_INVALID_ARG;
    if ((int64_t)B * n == 0) return GM_OK;
    if ((int64_t)B * n * k >= MAX_ROWS) return GM_ERR_UNSUPPORTED;
    if (!e_idx || !e_w || !mix1 || !mix2) return GM_ERR_INVALID_ARG;
    return GM_OK;
}

constexpr int WPB_LEG_TILE = 4;
constexpr int LEG_TILE_SM = 4;  // largest leg budget of the thread-per-row kernels

template <int K, int S0>
gm_status launch_leg_tile(const gm::LegArgs &a, bool backward, cudaStream_t stream)
{
    using Geo = gm::LegTileGeom<K, S0>;
    const int64_t warps = ((int64_t)a.tokens + Geo::TPW - 1) / Geo::TPW;
    const unsigned blocks = (unsigned)((warps + WPB_LEG_TILE - 1) / WPB_LEG_TILE);
    if (backward)
        gm::leg_bwd_tile_kernel<K, S0, LEG_TILE_SM, WPB_LEG_TILE><<<blocks, WPB_LEG_TILE * 32, 0, stream>>>(a);
    else
        gm::leg_fwd_tile_kernel<K, S0, LEG_TILE_SM, WPB_LEG_TILE><<<blocks, WPB_LEG_TILE * 32, 0, stream>>>(a);
    return launched();
}

// The thread-per-row kernels cover k in {4, 8, 16}, s0 in {2, 4} (k*s0 <= 32) and leg budgets
// up to LEG_TILE_SM; returns GM_ERR_UNSUPPORTED for every other shape (the caller then runs
// the warp-per-token kernel).
gm_status try_leg_tile(const gm::LegArgs &a, bool backward, cudaStream_t stream)
{
    if (a.s2 > LEG_TILE_SM || a.s3 > LEG_TILE_SM) return GM_ERR_UNSUPPORTED;
    if (a.k == 8 && a.s0 == 4) return launch_leg_tile<8, 4>(a, backward, stream);
    if (a.k == 8 && a.s0 == 2) return launch_leg_tile<8, 2>(a, backward, stream);
    if (a.k == 4 && a.s0 == 4) return launch_leg_tile<4, 4>(a, backward, stream);
    if (a.k == 4 && a.s0 == 2) return launch_leg_tile<4, 2>(a, backward, stream);
    if (a.k == 16 && a.s0 == 2) return launch_leg_tile<16, 2>(a, backward, stream);
    return GM_ERR_UNSUPPORTED;
}

// Shapes shared by SEA forward and backward. Returns GM_OK, or the error to report.
gm_status check_sea(const void *q, const void *k, const void *v, gm_dtype dtype,
                    const int32_t *idx, const float *w, int s, int B, int n, int hq, int hkv,
                    int d, float scale)
{
    if (B < 0 || n < 0 || hq < 1 || hkv < 1 || d < 1) return GM_ERR_INVALID_ARG;
    if (hq % hkv != 0 || s < 1 || s > MAX_SLOTS || !std::isfinite(scale)) return GM_ERR_INVALID_ARG;
    if (dtype != GM_F32 && dtype != GM_BF16) return GM_ERR_INVALID_ARG;
    const int G = hq / hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return GM_ERR_UNSUPPORTED;
    if (d != 32 && d != 64 && d != 128 && d != 256) return GM_ERR_UNSUPPORTED;
    if (dtype == GM_F32 && d > 128) return GM_ERR_UNSUPPORTED;
    if ((int64_t)B * n == 0) return GM_OK;
    if ((int64_t)B * n * hkv >= MAX_ROWS) return GM_ERR_UNSUPPORTED;
    if (!q || !k || !v || !idx || !w) return GM_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return GM_ERR_INVALID_ARG;
    return GM_OK;
}

// ---- checked builds ----------------------------------------------------------------------------
//
// Built with GM_CHECKED=1 (libgm_b200_checked.so), every entry point first verifies each edge
// tensor it reads: weights finite and >= 0, and every active index causal (no later than the
// position of its own row; position 0 is the padding token). A violation sets ERR_EDGE_INVALID
// in the device error word (gm_check_device_errors then returns GM_ERR_EDGE_INVALID); the call
// itself runs as in the regular build. In the regular build the check compiles to nothing.
#ifndef GM_CHECKED
#define GM_CHECKED 0
#endif

__global__ void check_edges_kernel(const int32_t *idx, const float *w, int64_t E, gm::FastDiv sdiv, gm::RowMap map)
{
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < E; e += (int64_t)gridDim.x * blockDim.x) {
        const float we = w[e];
        const int32_t t = idx[e];
        const uint32_t row = sdiv.div((uint32_t)e);
        const uint32_t bi = map.heads.div(row);
        const uint32_t pos = bi - map.n.div(bi) * map.n.d;
        const bool bad_w = !(we >= 0.0f) || isinf(we);
        const bool noncausal = we > 0.0f && t >= 0 && (uint32_t)t > pos;
        if (bad_w || noncausal) atomicOr(&gm::g_error_flag, gm::ERR_EDGE_INVALID);
    }
}

// Edge tensor [B, n, k, s] (nothing in a regular build).
void check_edges(const int32_t *idx, const float *w, int s, int64_t B, int n, int k, cudaStream_t st)
{
    if (!GM_CHECKED || idx == nullptr || w == nullptr) return;
    const int64_t E = B * n * k * s;
    if (E == 0) return;
    const int64_t want = (E + 255) / 256;
    check_edges_kernel<<<(unsigned)(want < 148 * 16 ? want : 148 * 16), 256, 0, st>>>(
        idx, w, E, gm::FastDiv((uint32_t)s), row_map(k, n));
}

// The first leg and every leg of a referral chain (arguments filled by chain_args).
void check_chain_edges(const SerArgs &a, cudaStream_t st)
{
    if (!GM_CHECKED) return;
    const int64_t B = (int64_t)a.rows / ((int64_t)a.n * a.k);
    check_edges(a.a1_idx, a.a1_w, a.s2, B, a.n, a.k, st);
    check_edges(a.a2_idx, a.a2_w, a.s3, B, a.n, a.k, st);
    for (int m = 0; m < a.nchain; ++m) check_edges(a.chain_idx[m], a.chain_w[m], a.s3, B, a.n, a.k, st);
}

// ---- dispatch over (dtype, d, G) ----------------------------------------------------------

template <template <typename, int, int> class F, typename... Args>
gm_status dispatch(gm_dtype dtype, int d, int G, Args &&...args)
{
#define GM_CASE_G(T, D)                                               \
    switch (G) {                                                      \
    case 1: return F<T, D, 1>::run(args...);                          \
    case 2: return F<T, D, 2>::run(args...);                          \
    case 4: return F<T, D, 4>::run(args...);                          \
    case 8: return F<T, D, 8>::run(args...);                          \
    default: return GM_ERR_UNSUPPORTED;                               \
    }
    if (dtype == GM_BF16) {
        switch (d) {
        case 32: GM_CASE_G(__nv_bfloat16, 32)
        case 64: GM_CASE_G(__nv_bfloat16, 64)
        case 128: GM_CASE_G(__nv_bfloat16, 128)
        case 256: GM_CASE_G(__nv_bfloat16, 256)
        default: return GM_ERR_UNSUPPORTED;
        }
    } else {
        switch (d) {
        case 32: GM_CASE_G(float, 32)
        case 64: GM_CASE_G(float, 64)
        case 128: GM_CASE_G(float, 128)
        default: return GM_ERR_UNSUPPORTED;
        }
    }
#undef GM_CASE_G
}

// Launch with programmatic stream serialization: the kernel may start while the previous one
// on the stream drains, and waits for it (pdl_wait) before touching its outputs. Used for the
// chain of kernels inside one backward call, whose first kernel is launched the ordinary way.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    (void)cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Persistent grid for a kernel with `smem` bytes of dynamic shared memory per block:
// as many blocks as fit on the device at once, but no more than the rows need.
template <typename K>
unsigned persistent_blocks(K kernel, int threads, size_t smem, int64_t rows, int rows_per_block)
{
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    const int64_t need = (rows + rows_per_block - 1) / rows_per_block;
    const int64_t fit = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    return (unsigned)(need < fit ? need : fit);
}

#ifndef GM_WPB_TILE
#define GM_WPB_TILE 1  // one-warp blocks: 96.6 -> 94.6 us for the fused forward at B = 8 against four
#endif
#ifndef GM_BWD_TILE_P
#define GM_BWD_TILE_P 2
#endif
#ifndef GM_WPB_BWD_TILE
#define GM_WPB_BWD_TILE 4
#endif
#ifndef GM_TILE_CPL
#define GM_TILE_CPL 1
#endif
// Passes of K/V copies in flight per warp in the forward tile kernel: two for budgets of 2
// (little work per pass to cover the loads), one for budgets of 4 (a pass covers them, and
// the freed shared memory admits more warps).
#ifndef GM_TILE_P4
#define GM_TILE_P4 1
#endif
template <int S1M> constexpr int tile_passes() { return S1M >= 4 ? GM_TILE_P4 : 2; }
constexpr int WPB_TILE = GM_WPB_TILE;
constexpr int TILE_CPL = GM_TILE_CPL;  // 16-byte chunks of a feature row per lane

// Shapes the tiled forward covers: 2..16 lanes per feature row, at most 16 fp32 values of
// q per lane for the whole group, head_dim 64 or 128.
template <typename T, int D, int G> struct TileOK {
    static constexpr int VEC = gm::Vec<T>::N;
    static constexpr bool value = (D == 64 || D == 128) && D / VEC >= 2 && D / VEC <= 16 && VEC * G <= 16;
};

template <typename T, int D, int G, bool REFER, int S2, int S3, int S1M, int SF = 0, int NL = 1>
gm_status launch_tile(const SerArgs &sa, const SeaArgs &a, cudaStream_t st)
{
    using TG = gm::TileGeom<T, D, G, S1M, TILE_CPL>;
    constexpr int P = tile_passes<S1M>();
    auto kern = gm::sea_fwd_tile_kernel<T, D, G, REFER, S2, S3, S1M, P, WPB_TILE, TILE_CPL, SF, NL>;
    const size_t smem = (size_t)WPB_TILE * (32 * S1M * 8 + P * TG::STAGE);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GM_ERR_CUDA;
    const int64_t tiles = ((int64_t)a.rows + 31) / 32;
    const unsigned grid = persistent_blocks(kern, WPB_TILE * 32, smem, tiles, WPB_TILE);
    kern<<<grid, WPB_TILE * 32, smem, st>>>(sa, a);
    return launched();
}

template <typename T, int D, int G> struct SerSeaFwd {
    static gm_status run(const SerArgs &sa, const SeaArgs &a, cudaStream_t st)
    {
        if (sa.nchain > 0 && !TileOK<T, D, G>::value) return GM_ERR_UNSUPPORTED;  // chains: tile only
        if constexpr (TileOK<T, D, G>::value) {
            bool aligned = aligned16(sa.a1_idx) && aligned16(sa.a1_w) && aligned16(sa.a2_idx) &&
                       aligned16(sa.a2_w) && aligned16(sa.out_idx) && aligned16(sa.out_w);
        for (int m = 0; m < sa.nchain; ++m) aligned = aligned && aligned16(sa.chain_idx[m]) && aligned16(sa.chain_w[m]);
        if (sa.nchain > 0) {
            // multi-step referral: bf16 features, s2 = s3 = s_mid in {2, 4}, s1 <= 4, 3 or 4 legs
            if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                if (aligned && sa.sf == 0 && sa.s1 <= 4 && sa.s2 == sa.s3 && sa.s_mid == sa.s2 &&
                    (sa.s2 == 2 || sa.s2 == 4) && (sa.nchain == 1 || sa.nchain == 2)) {
                    if (sa.s2 == 2)
                        return sa.nchain == 1 ? launch_tile<T, D, G, true, 2, 2, 4, 0, 2>(sa, a, st)
                                              : launch_tile<T, D, G, true, 2, 2, 4, 0, 3>(sa, a, st);
                    return sa.nchain == 1 ? launch_tile<T, D, G, true, 4, 4, 4, 0, 2>(sa, a, st)
                                          : launch_tile<T, D, G, true, 4, 4, 4, 0, 3>(sa, a, st);
                }
            }
            return GM_ERR_UNSUPPORTED;  // the caller runs the chain, then SEA
        }
            if (aligned && sa.sf == 0 && sa.s2 == 2 && sa.s3 == 2) {
                if (sa.s1 <= 2) return launch_tile<T, D, G, true, 2, 2, 2>(sa, a, st);
                if (sa.s1 <= 4) return launch_tile<T, D, G, true, 2, 2, 4>(sa, a, st);
            }
            if (aligned && sa.sf == 0 && sa.s2 == 4 && sa.s3 == 4) {
                if (sa.s1 <= 2) return launch_tile<T, D, G, true, 4, 4, 2>(sa, a, st);
                if (sa.s1 <= 4) return launch_tile<T, D, G, true, 4, 4, 4>(sa, a, st);
            }
            // refresh edges: bf16 features, budgets 2 or 4, s1 <= 4, sf in {2, 4}
            if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                if (aligned && sa.sf > 0 && aligned16(sa.f_idx) && aligned16(sa.f_w) && sa.s1 <= 4 &&
                    sa.s2 == sa.s3 && (sa.s2 == 2 || sa.s2 == 4) && (sa.sf == 2 || sa.sf == 4)) {
                    if (sa.s2 == 2)
                        return sa.sf == 2 ? launch_tile<T, D, G, true, 2, 2, 4, 2>(sa, a, st)
                                          : launch_tile<T, D, G, true, 2, 2, 4, 4>(sa, a, st);
                    return sa.sf == 2 ? launch_tile<T, D, G, true, 4, 4, 4, 2>(sa, a, st)
                                      : launch_tile<T, D, G, true, 4, 4, 4, 4>(sa, a, st);
                }
            }
        }
        gm::ser_sea_fwd_kernel<T, D, G, WPB_SEA><<<blocks_for(a.rows, WPB_SEA), WPB_SEA * 32, 0, st>>>(sa, a);
        return launched();
    }
};

template <typename T, int D, int G> struct SeaFwd {
    static gm_status run(const SeaArgs &a, cudaStream_t st)
    {
        if constexpr (TileOK<T, D, G>::value) {
            const SerArgs none{};
            if (a.s <= 2) return launch_tile<T, D, G, false, 1, 1, 2>(none, a, st);
            if (a.s <= 4) return launch_tile<T, D, G, false, 1, 1, 4>(none, a, st);
        }
        gm::sea_fwd_kernel<T, D, G, WPB_SEA><<<blocks_for(a.rows, WPB_SEA), WPB_SEA * 32, 0, st>>>(a);
        return launched();
    }
};

constexpr int BWD_TILE_P = GM_BWD_TILE_P;
constexpr int WPB_BWD_TILE = GM_WPB_BWD_TILE;

template <typename T, int D, int G, int S1M, bool GATHER, int SB = 0>
gm_status launch_bwd_tile(const SeaBwdArgs &a, cudaStream_t st, bool pdl = false)
{
    using TG = gm::BwdTileGeom<T, D, G, S1M>;
    auto kern = gm::sea_bwd_tile_kernel<T, D, G, S1M, BWD_TILE_P, WPB_BWD_TILE, GATHER, SB>;
    const size_t smem = (size_t)WPB_BWD_TILE * (gm::bwd_tile_bytes<S1M, SB, GATHER>() + BWD_TILE_P * TG::STAGE);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GM_ERR_CUDA;
    const int64_t tiles = ((int64_t)a.rows + 31) / 32;
    const unsigned grid = persistent_blocks(kern, WPB_BWD_TILE * 32, smem, tiles, WPB_BWD_TILE);
    if (pdl)
        launch_pdl(kern, grid, WPB_BWD_TILE * 32, smem, st, a);
    else
        kern<<<grid, WPB_BWD_TILE * 32, smem, st>>>(a);
    return launched();
}

template <typename T, int D, int G> struct SeaBwd {
    static gm_status run(const SeaBwdArgs &a, cudaStream_t st)
    {
        if constexpr (TileOK<T, D, G>::value) {
            if (a.s <= 2) return launch_bwd_tile<T, D, G, 2, false>(a, st);
            if (a.s <= 4) return launch_bwd_tile<T, D, G, 4, false>(a, st);
        }
        gm::sea_bwd_kernel<T, D, G, WPB_BWD><<<blocks_for(a.rows, WPB_BWD), WPB_BWD * 32, 0, st>>>(a);
        return launched();
    }
};

// ---- gather-based backward (workspace) -------------------------------------------------------

#ifndef GM_GATHER_U
#define GM_GATHER_U 4
#endif
#ifndef GM_GATHER_P
#define GM_GATHER_P 2
#endif
#ifndef GM_WPB_GATHER
#define GM_WPB_GATHER 1
#endif
// One warp per block: a block's resources are freed as soon as its one chunk is done, so
// chunks that follow a long target past their end hold back no other warp (at B = 8, n = 4096:
// 294 -> 284 us for the backward, against two warps per block).
constexpr int WPB_GATHER = GM_WPB_GATHER;
constexpr int GATHER_U = GM_GATHER_U;  // records per copy group
constexpr int GATHER_P = GM_GATHER_P;  // copy groups in flight per warp

// The gather path covers the tiled shapes with s <= 4 and fewer than 2^31 edges.
bool gather_supported(gm_dtype dtype, int d, int G, int s, int64_t E)
{
    if (s > 4 || E >= MAX_ROWS) return false;
    if (dtype == GM_BF16) return (d == 64 || d == 128) && G <= 2;
    return d == 64 && G <= 4;
}

struct WsLayout {
    size_t cnt, state, ticket, off, rank, srec, total;
    uint32_t nblk;
};

// [cnt | scan tile words | ticket] (cleared at every call) [off] [rank] [records]
WsLayout ws_layout(int64_t R, int64_t E, int G)
{
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const int words = (2 + 2 * G + 3) / 4 * 4;  // gm::Rec<G>::WORDS
    WsLayout L;
    L.nblk = (uint32_t)((R + gm::SCAN_TILE - 1) / gm::SCAN_TILE);
    L.cnt = 0;
    L.state = L.cnt + up((size_t)R * 4);
    L.ticket = L.state + (size_t)L.nblk * 8;
    L.off = L.state + up((size_t)L.nblk * 8 + 8);
    L.rank = L.off + up((size_t)(R + 1) * 4);
    L.srec = L.rank + up((size_t)E * 4);
    L.total = L.srec + up((size_t)E * words * 4);
    return L;
}

gm::GatherWs gather_ws(void *workspace, const WsLayout &L)
{
    char *base = static_cast<char *>(workspace);
    return gm::GatherWs{reinterpret_cast<int32_t *>(base + L.cnt),
                        reinterpret_cast<unsigned long long *>(base + L.state),
                        reinterpret_cast<uint32_t *>(base + L.ticket),
                        reinterpret_cast<int32_t *>(base + L.off),
                        reinterpret_cast<int32_t *>(base + L.rank),
                        reinterpret_cast<int32_t *>(base + L.srec),
                        L.nblk,
                        (int64_t)(L.off / 4)};
}

template <typename T, int D, int G> struct SeaBwdGather {
    // sb > 0: the row pass also runs the referral backward of A' = Sparsify(A1 A2) with
    // budgets s2 = s3 = sb (a.a1_idx ... a.dw2 set; the caller checked the shapes)
    static gm_status run(SeaBwdArgs a, gm::GatherWs ws, const int32_t *idx, const float *w, cudaStream_t st,
                         int sb = 0)
    {
        if constexpr (TileOK<T, D, G>::value && 2 * (D / gm::Vec<T>::N) <= 32 && 2 * G <= 8) {
            const int64_t R = a.rows, E = R * a.s;
            gm::zero_i32_kernel<<<148 * 4, 256, 0, st>>>(ws.cnt, ws.zero_words);
            const unsigned cgrid = (unsigned)((R + 255) / 256);
            if (a.s <= 2)
                launch_pdl(gm::edge_count_kernel<2>, cgrid, 256, 0, st, idx, w, a.n, a.map, a.s, a.rows, a.hkv,
                           ws.cnt, ws.rank);
            else
                launch_pdl(gm::edge_count_kernel<4>, cgrid, 256, 0, st, idx, w, a.n, a.map, a.s, a.rows, a.hkv,
                           ws.cnt, ws.rank);
            launch_pdl(gm::scan_lookback_kernel, ws.nblk, gm::SCAN_THREADS, 0, st, ws.cnt, R, ws.state, ws.ticket,
                       ws.off, a.dk, a.dv, D, a.accumulate);
            if (launched() != GM_OK) return GM_ERR_CUDA;
            a.rank = ws.rank;
            a.off = ws.off;
            a.srec = ws.srec;
            gm_status rs;
            if (sb == 2)
                rs = a.s <= 2 ? launch_bwd_tile<T, D, G, 2, true, 2>(a, st, true)
                              : launch_bwd_tile<T, D, G, 4, true, 2>(a, st, true);
            else if (sb == 4)
                rs = a.s <= 2 ? launch_bwd_tile<T, D, G, 2, true, 4>(a, st, true)
                              : launch_bwd_tile<T, D, G, 4, true, 4>(a, st, true);
            else
                rs = a.s <= 2 ? launch_bwd_tile<T, D, G, 2, true>(a, st, true)
                              : launch_bwd_tile<T, D, G, 4, true>(a, st, true);
            if (rs != GM_OK) return rs;
            auto kern = gm::sea_bwd_gather_kernel<T, D, G, WPB_GATHER, GATHER_U, GATHER_P>;
            const size_t smem = (size_t)WPB_GATHER * GATHER_P * GATHER_U * G * 32 * 16;
            if (smem > 48 * 1024 &&
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
                return GM_ERR_CUDA;
            const int64_t chunks = (E + 31) / 32;  // upper bound: the active count is on the device
            launch_pdl(kern, blocks_for(chunks, WPB_GATHER), WPB_GATHER * 32, smem, st, a.q, a.dout, a.dk, a.dv, ws,
                       (uint32_t)R, a.accumulate);
            return launched();
        } else {
            return GM_ERR_UNSUPPORTED;
        }
    }
};

// ---- refresh edges from a dense attention layer ----------------------------------------------

// cuTensorMapEncodeTiled through the runtime's driver entry point (the library does not link
// the driver library itself).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A bf16 feature tensor [rows, heads, d] as a 3-d TMA map whose boxes are 64 elements of d
// (128 bytes, the swizzle width) x 1 head x box_rows rows, in the 128-byte swizzle layout.
bool feature_tmap(CUtensorMap &m, const void *ptr, int64_t rows, int heads, int d, int box_rows)
{
    const EncodeTiledFn f = encode_tiled();
    if (f == nullptr) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return f(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G, int SFM>
gm_status launch_dense_refresh(const void *q, const void *k, int64_t tokens, const gm::DenseRefreshArgs &a,
                               cudaStream_t st)
{
    constexpr int BN = G == 4 ? 64 : 128;  // G accumulators x BN columns x 2 sets <= 512 TMEM columns
    using Geo = gm::DenseGeom<D, G, BN>;
    CUtensorMap tq, tk;
    if (!feature_tmap(tq, q, tokens, a.hq, D, Geo::BM) || !feature_tmap(tk, k, tokens, a.hkv, D, BN))
        return GM_ERR_CUDA;
    auto kern = gm::dense_refresh_kernel<D, G, BN, SFM>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::SMEM_BYTES) != cudaSuccess)
        return GM_ERR_CUDA;
    kern<<<(unsigned)((int64_t)a.BH * a.nblk), Geo::THREADS, Geo::SMEM_BYTES, st>>>(tq, tk, a);
    return launched();
}

template <int D, int G>
gm_status dense_refresh_sf(const void *q, const void *k, int64_t tokens, const gm::DenseRefreshArgs &a,
                           cudaStream_t st)
{
    if (a.sf <= 2) return launch_dense_refresh<D, G, 2>(q, k, tokens, a, st);
    if (a.sf <= 4) return launch_dense_refresh<D, G, 4>(q, k, tokens, a, st);
    return launch_dense_refresh<D, G, 8>(q, k, tokens, a, st);
}

template <int D>
gm_status dense_refresh_g(const void *q, const void *k, int64_t tokens, int G, const gm::DenseRefreshArgs &a,
                          cudaStream_t st)
{
    if (G == 1) return dense_refresh_sf<D, 1>(q, k, tokens, a, st);
    if (G == 2) return dense_refresh_sf<D, 2>(q, k, tokens, a, st);
    if (G == 4) return dense_refresh_sf<D, 4>(q, k, tokens, a, st);
    return GM_ERR_UNSUPPORTED;
}

// ---- scratch for callers that cannot allocate ------------------------------------------------
//
// gm_sea_backward_noalloc runs the gather path of gm_sea_backward on this fixed, file-scope
// device array instead of a caller workspace. Every device that loads the library holds it
// (NOALLOC_SCRATCH_BYTES) until the process exits, and every call on that device shares it.
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)32 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[NOALLOC_MAX_DEVICES] = {};

// Device address of g_noalloc_scratch on the current device. In host code the array's name
// is only a stand-in, so its address is looked up once per device (with that device
// current) and cached.
gm_status noalloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GM_ERR_CUDA;
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return GM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GM_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return GM_OK;
}

// One bounded wait that nothing completes: the thread waits on a shared-memory barrier with
// no arrivals, gives up after WAIT_LIMIT_NS, sets ERR_WAIT_TIMEOUT and returns.
__global__ void wait_timeout_selftest_kernel()
{
    __shared__ __align__(8) unsigned long long bar;
    if (threadIdx.x == 0) {
        const uint32_t b = gm::smem_u32(&bar);
        gm::mbar_init(b, 1);
        gm::mbar_init_fence();
        (void)gm::mbar_wait(b, 0);
    }
}

}  // namespace

extern "C" {

int gm_version(void) { return 100; }

gm_status gm_selftest_wait_timeout(cudaStream_t stream)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>();
    return launched();
}

int gm_checked_build(void) { return GM_CHECKED ? 1 : 0; }

const char *gm_status_string(gm_status status)
{
    switch (status) {
    case GM_OK: return "GM_OK";
    case GM_ERR_INVALID_ARG: return "GM_ERR_INVALID_ARG: invalid argument";
    case GM_ERR_UNSUPPORTED: return "GM_ERR_UNSUPPORTED: no kernel in this library for the shape";
    case GM_ERR_CUDA: return "GM_ERR_CUDA: CUDA launch or synchronisation failed";
    case GM_ERR_INDEX_RANGE: return "GM_ERR_INDEX_RANGE: an active edge index was outside [0, n)";
    case GM_ERR_SCRATCH_TOO_SMALL:
        return "GM_ERR_SCRATCH_TOO_SMALL: the problem needs more scratch than the library's fixed "
               "array holds (see gm_sea_backward_noalloc_max_scratch)";
    case GM_ERR_EDGE_INVALID:
        return "GM_ERR_EDGE_INVALID: (checked build) an input edge had a negative or non-finite "
               "weight, or an active index beyond its own row's position";
    case GM_ERR_WAIT_TIMEOUT:
        return "GM_ERR_WAIT_TIMEOUT: a kernel gave up on a bounded wait for an asynchronous copy or "
               "tensor-core operation; its outputs are incomplete";
    default: return "unknown gm_status";
    }
}

gm_status gm_ser_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                         const int32_t *a2_idx, const float *a2_w, int s3,
                         int32_t *out_idx, float *out_w, int s1,
                         int B, int n, int k, cudaStream_t stream)
{
    gm_status st = check_ser(a1_idx, a1_w, s2, a2_idx, a2_w, s3, s1, B, n, k);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!out_idx || !out_w) return GM_ERR_INVALID_ARG;
    SerArgs a{a1_idx, a1_w, a2_idx, a2_w, out_idx, out_w, s1, s2, s3, n, k,
              (uint32_t)((int64_t)B * n * k), row_map(k, n)};
    check_edges(a1_idx, a1_w, s2, B, n, k, stream);
    check_edges(a2_idx, a2_w, s3, B, n, k, stream);
    // one thread per row for budgets 2 or 4 (vector loads and stores need 16-byte alignment)
    const bool aligned = aligned16(a1_idx) && aligned16(a1_w) && aligned16(a2_idx) && aligned16(a2_w) &&
                         aligned16(out_idx) && aligned16(out_w);
    const unsigned tgrid = (unsigned)((a.rows + 127) / 128);
    if (aligned && s2 == s3 && (s2 == 2 || s2 == 4) && s1 <= 4) {
        if (s2 == 2)
            s1 <= 2 ? gm::ser_thread_kernel<2, 2, 2><<<tgrid, 128, 0, stream>>>(a)
                    : gm::ser_thread_kernel<2, 2, 4><<<tgrid, 128, 0, stream>>>(a);
        else
            s1 <= 2 ? gm::ser_thread_kernel<4, 4, 2><<<tgrid, 128, 0, stream>>>(a)
                    : gm::ser_thread_kernel<4, 4, 4><<<tgrid, 128, 0, stream>>>(a);
        return launched();
    }
    gm::ser_kernel<WPB_SER><<<blocks_for(a.rows, WPB_SER), WPB_SER * 32, 0, stream>>>(a);
    return launched();
}

gm_status gm_ser_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                          const int32_t *a2_idx, const float *a2_w, int s3,
                          const float *gout, int s1, int grad_is_log,
                          int B, int n, int k, float *dw1, float *dw2, int accumulate,
                          cudaStream_t stream)
{
    if ((grad_is_log != 0 && grad_is_log != 1) || (accumulate != 0 && accumulate != 1)) return GM_ERR_INVALID_ARG;
    gm_status st = check_ser(a1_idx, a1_w, s2, a2_idx, a2_w, s3, s1, B, n, k);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!gout || !dw1 || !dw2) return GM_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * n * k;
    check_edges(a1_idx, a1_w, s2, B, n, k, stream);
    check_edges(a2_idx, a2_w, s3, B, n, k, stream);
    if (!accumulate) {
        gm::zero_i32_kernel<<<148 * 4, 256, 0, stream>>>(reinterpret_cast<int32_t *>(dw2), rows * s3);
        if (launched() != GM_OK) return GM_ERR_CUDA;
    }
    const SerArgs f{a1_idx, a1_w, a2_idx, a2_w, nullptr, nullptr, s1, s2, s3, n, k, (uint32_t)rows, row_map(k, n)};
    const gm::SerBwdArgs b{f, gout, grad_is_log, dw1, dw2, accumulate};
    // per-thread rows for the small budgets the fused forward tiles (vector loads need
    // 16-byte aligned legs)
    const bool aligned = aligned16(a1_idx) && aligned16(a1_w) && aligned16(a2_idx) && aligned16(a2_w);
    const unsigned tblocks = blocks_for(rows, 32 * WPB_SER_THREAD);
    if (aligned && s2 == 4 && s3 == 4 && s1 <= 4) {
        launch_pdl(gm::ser_bwd_thread_kernel<4, 4, 4, WPB_SER_THREAD>, tblocks, WPB_SER_THREAD * 32, 0, stream, b);
        return launched();
    }
    if (aligned && s2 == 2 && s3 == 2 && s1 <= 4) {
        launch_pdl(gm::ser_bwd_thread_kernel<2, 2, 4, WPB_SER_THREAD>, tblocks, WPB_SER_THREAD * 32, 0, stream, b);
        return launched();
    }
    gm::ser_bwd_kernel<WPB_SER><<<blocks_for(rows, WPB_SER), WPB_SER * 32, 0, stream>>>(b);
    return launched();
}

gm_status gm_leg_sparsify(const int32_t *e_idx, const float *e_w, int s0,
                          const float *mix1, const float *mix2, int64_t mix_token_stride,
                          int32_t *a1_idx, float *a1_w, int s2,
                          int32_t *a2_idx, float *a2_w, int s3,
                          int B, int n, int k, cudaStream_t stream)
{
    gm_status st = check_leg(e_idx, e_w, s0, mix1, mix2, mix_token_stride, s2, s3, B, n, k);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!a1_idx || !a1_w || !a2_idx || !a2_w) return GM_ERR_INVALID_ARG;
    gm::LegArgs a{};
    check_edges(e_idx, e_w, s0, B, n, k, stream);
    a.e_idx = e_idx;
    a.e_w = e_w;
    a.mix1 = mix1;
    a.mix2 = mix2;
    a.mix_stride = (uint32_t)mix_token_stride;
    a.a1_idx = a1_idx;
    a.a1_w = a1_w;
    a.a2_idx = a2_idx;
    a.a2_w = a2_w;
    a.k = k;
    a.s0 = s0;
    a.s2 = s2;
    a.s3 = s3;
    a.n = n;
    a.tokens = (uint32_t)((int64_t)B * n);
    const gm_status tile = try_leg_tile(a, false, stream);
    if (tile != GM_ERR_UNSUPPORTED) return tile;
    gm::leg_fwd_kernel<WPB_LEG><<<blocks_for(a.tokens, WPB_LEG), WPB_LEG * 32, 0, stream>>>(a);
    return launched();
}

gm_status gm_leg_backward(const int32_t *e_idx, const float *e_w, int s0,
                          const float *mix1, const float *mix2, int64_t mix_token_stride,
                          const float *g1, int s2, const float *g2, int s3,
                          int B, int n, int k, float *dew, float *dmix1, float *dmix2,
                          int accumulate, cudaStream_t stream)
{
    if (accumulate != 0 && accumulate != 1) return GM_ERR_INVALID_ARG;
    gm_status st = check_leg(e_idx, e_w, s0, mix1, mix2, mix_token_stride, s2, s3, B, n, k);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!g1 || !g2 || !dew || !dmix1 || !dmix2) return GM_ERR_INVALID_ARG;
    gm::LegArgs a{};
    check_edges(e_idx, e_w, s0, B, n, k, stream);
    a.e_idx = e_idx;
    a.e_w = e_w;
    a.mix1 = mix1;
    a.mix2 = mix2;
    a.mix_stride = (uint32_t)mix_token_stride;
    a.g1 = g1;
    a.g2 = g2;
    a.dew = dew;
    a.dmix1 = dmix1;
    a.dmix2 = dmix2;
    a.accumulate = accumulate;
    a.k = k;
    a.s0 = s0;
    a.s2 = s2;
    a.s3 = s3;
    a.n = n;
    a.tokens = (uint32_t)((int64_t)B * n);
    const gm_status tile = try_leg_tile(a, true, stream);
    if (tile != GM_ERR_UNSUPPORTED) return tile;
    gm::leg_bwd_kernel<WPB_LEG><<<blocks_for(a.tokens, WPB_LEG), WPB_LEG * 32, 0, stream>>>(a);
    return launched();
}

gm_status gm_ser_refresh_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                                 const int32_t *a2_idx, const float *a2_w, int s3,
                                 const int32_t *f_idx, const float *f_w, int sf,
                                 int32_t *out_idx, float *out_w, int s1,
                                 int B, int n, int k, cudaStream_t stream)
{
    gm_status st = check_ser(a1_idx, a1_w, s2, a2_idx, a2_w, s3, s1, B, n, k);
    if (st != GM_OK) return st;
    st = check_refresh(f_idx, f_w, sf, s2, s3, (int64_t)B * n);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!out_idx || !out_w) return GM_ERR_INVALID_ARG;
    SerArgs a{a1_idx, a1_w, a2_idx, a2_w, out_idx, out_w, s1, s2, s3, n, k,
              (uint32_t)((int64_t)B * n * k), row_map(k, n), f_idx, f_w, sf};
    check_edges(a1_idx, a1_w, s2, B, n, k, stream);
    check_edges(a2_idx, a2_w, s3, B, n, k, stream);
    check_edges(f_idx, f_w, sf, B, n, k, stream);
    const bool aligned = aligned16(a1_idx) && aligned16(a1_w) && aligned16(a2_idx) && aligned16(a2_w) &&
                         aligned16(f_idx) && aligned16(f_w) && aligned16(out_idx) && aligned16(out_w);
    const unsigned tgrid = (unsigned)((a.rows + 127) / 128);
    if (aligned && s2 == s3 && (s2 == 2 || s2 == 4) && s1 <= 4 && (sf == 2 || sf == 4)) {
        if (s2 == 2)
            sf == 2 ? gm::ser_thread_kernel<2, 2, 4, 2><<<tgrid, 128, 0, stream>>>(a)
                    : gm::ser_thread_kernel<2, 2, 4, 4><<<tgrid, 128, 0, stream>>>(a);
        else
            sf == 2 ? gm::ser_thread_kernel<4, 4, 4, 2><<<tgrid, 128, 0, stream>>>(a)
                    : gm::ser_thread_kernel<4, 4, 4, 4><<<tgrid, 128, 0, stream>>>(a);
        return launched();
    }
    gm::ser_kernel<WPB_SER><<<blocks_for(a.rows, WPB_SER), WPB_SER * 32, 0, stream>>>(a);
    return launched();
}

gm_status gm_ser_refresh_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                                  const int32_t *a2_idx, const float *a2_w, int s3,
                                  const int32_t *f_idx, const float *f_w, int sf,
                                  const float *gout, int s1, int grad_is_log,
                                  int B, int n, int k, float *dw1, float *dw2, float *dfw,
                                  int accumulate, cudaStream_t stream)
{
    if ((grad_is_log != 0 && grad_is_log != 1) || (accumulate != 0 && accumulate != 1)) return GM_ERR_INVALID_ARG;
    gm_status st = check_ser(a1_idx, a1_w, s2, a2_idx, a2_w, s3, s1, B, n, k);
    if (st != GM_OK) return st;
    st = check_refresh(f_idx, f_w, sf, s2, s3, (int64_t)B * n);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!gout || !dw1 || !dw2 || !dfw) return GM_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * n * k;
    check_edges(a1_idx, a1_w, s2, B, n, k, stream);
    check_edges(a2_idx, a2_w, s3, B, n, k, stream);
    check_edges(f_idx, f_w, sf, B, n, k, stream);
    if (!accumulate) {
        gm::zero_i32_kernel<<<148 * 4, 256, 0, stream>>>(reinterpret_cast<int32_t *>(dw2), rows * s3);
        if (launched() != GM_OK) return GM_ERR_CUDA;
    }
    const SerArgs f{a1_idx, a1_w, a2_idx, a2_w, nullptr, nullptr, s1, s2, s3, n, k, (uint32_t)rows,
                    row_map(k, n), f_idx, f_w, sf};
    const gm::SerBwdArgs b{f, gout, grad_is_log, dw1, dw2, accumulate, dfw};
    // one thread per row for the small budgets (vector loads need 16-byte aligned legs)
    const bool aligned = aligned16(a1_idx) && aligned16(a1_w) && aligned16(a2_idx) && aligned16(a2_w) &&
                         aligned16(f_idx) && aligned16(f_w);
    const unsigned tblocks = blocks_for(rows, 32 * WPB_SER_THREAD);
    if (aligned && s2 == s3 && (s2 == 2 || s2 == 4) && s1 <= 4 && (sf == 2 || sf == 4)) {
        if (s2 == 4)
            sf == 4 ? launch_pdl(gm::ser_bwd_thread_kernel<4, 4, 4, WPB_SER_THREAD, 4>, tblocks, WPB_SER_THREAD * 32, 0, stream, b)
                    : launch_pdl(gm::ser_bwd_thread_kernel<4, 4, 4, WPB_SER_THREAD, 2>, tblocks, WPB_SER_THREAD * 32, 0, stream, b);
        else
            sf == 4 ? launch_pdl(gm::ser_bwd_thread_kernel<2, 2, 4, WPB_SER_THREAD, 4>, tblocks, WPB_SER_THREAD * 32, 0, stream, b)
                    : launch_pdl(gm::ser_bwd_thread_kernel<2, 2, 4, WPB_SER_THREAD, 2>, tblocks, WPB_SER_THREAD * 32, 0, stream, b);
        return launched();
    }
    gm::ser_bwd_kernel<WPB_SER><<<blocks_for(rows, WPB_SER), WPB_SER * 32, 0, stream>>>(b);
    return launched();
}

gm_status gm_ser_sea_refresh_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                                     const int32_t *a2_idx, const float *a2_w, int s3,
                                     const int32_t *f_idx, const float *f_w, int sf,
                                     int32_t *out_idx, float *out_w, int s1,
                                     const void *q, const void *k, const void *v, gm_dtype dtype,
                                     int B, int n, int hq, int hkv, int d, float scale,
                                     void *o, float *lse, cudaStream_t stream)
{
    if ((out_idx == nullptr) != (out_w == nullptr)) return GM_ERR_INVALID_ARG;
    gm_status st = check_ser(a1_idx, a1_w, s2, a2_idx, a2_w, s3, s1, B, n, hkv);
    if (st != GM_OK) return st;
    st = check_refresh(f_idx, f_w, sf, s2, s3, (int64_t)B * n);
    if (st != GM_OK) return st;
    const int32_t dummy_idx = 0;
    const float dummy_w = 0.0f;
    st = check_sea(q, k, v, dtype, &dummy_idx, &dummy_w, s1, B, n, hq, hkv, d, scale);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!o || !aligned16(o)) return GM_ERR_INVALID_ARG;
    check_edges(a1_idx, a1_w, s2, B, n, hkv, stream);
    check_edges(a2_idx, a2_w, s3, B, n, hkv, stream);
    check_edges(f_idx, f_w, sf, B, n, hkv, stream);
    const uint32_t rows = (uint32_t)((int64_t)B * n * hkv);
    SerArgs sa{a1_idx, a1_w, a2_idx, a2_w, out_idx, out_w, s1, s2, s3, n, hkv, rows, row_map(hkv, n),
               f_idx, f_w, sf};
    SeaArgs a{q, k, v, nullptr, nullptr, o, lse, s1, n, hkv, scale, rows, row_map(hkv, n)};
    return dispatch<SerSeaFwd>(dtype, d, hq / hkv, sa, a, stream);
}

gm_status gm_ser_chain_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                               const int32_t *const *leg_idx, const float *const *leg_w, int nlegs,
                               int s3, int s_mid, int32_t *out_idx, float *out_w, int s1,
                               int B, int n, int k, cudaStream_t stream)
{
    SerArgs a{};
    gm_status st = chain_args(a1_idx, a1_w, s2, leg_idx, leg_w, nlegs, s3, s_mid, s1, B, n, k, a);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!out_idx || !out_w) return GM_ERR_INVALID_ARG;
    a.out_idx = out_idx;
    check_chain_edges(a, stream);
    a.out_w = out_w;
    // one thread per row for budgets s2 = s3 = s_mid of 2 or 4 and up to 4 legs
    bool aligned = aligned16(a1_idx) && aligned16(a1_w) && aligned16(out_idx) && aligned16(out_w);
    for (int m = 0; m < nlegs; ++m) aligned = aligned && aligned16(leg_idx[m]) && aligned16(leg_w[m]);
    if (aligned && s2 == s3 && s_mid == s2 && (s2 == 2 || s2 == 4) && s1 <= 4 && nlegs >= 2 && nlegs <= 4) {
        const unsigned tgrid = (unsigned)((a.rows + 127) / 128);
        if (s2 == 2) {
            if (nlegs == 2) gm::ser_thread_kernel<2, 2, 4, 0, 2><<<tgrid, 128, 0, stream>>>(a);
            else if (nlegs == 3) gm::ser_thread_kernel<2, 2, 4, 0, 3><<<tgrid, 128, 0, stream>>>(a);
            else gm::ser_thread_kernel<2, 2, 4, 0, 4><<<tgrid, 128, 0, stream>>>(a);
        } else {
            if (nlegs == 2) gm::ser_thread_kernel<4, 4, 4, 0, 2><<<tgrid, 128, 0, stream>>>(a);
            else if (nlegs == 3) gm::ser_thread_kernel<4, 4, 4, 0, 3><<<tgrid, 128, 0, stream>>>(a);
            else gm::ser_thread_kernel<4, 4, 4, 0, 4><<<tgrid, 128, 0, stream>>>(a);
        }
        return launched();
    }
    const unsigned grid = blocks_for(a.rows, WPB_SER);
    switch (nlegs) {
    case 1: gm::ser_chain_kernel<1, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(a); break;
    case 2: gm::ser_chain_kernel<2, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(a); break;
    case 3: gm::ser_chain_kernel<3, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(a); break;
    case 4: gm::ser_chain_kernel<4, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(a); break;
    case 5: gm::ser_chain_kernel<5, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(a); break;
    case 6: gm::ser_chain_kernel<6, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(a); break;
    default: gm::ser_chain_kernel<7, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(a); break;
    }
    return launched();
}

gm_status gm_ser_chain_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                                const int32_t *const *leg_idx, const float *const *leg_w, int nlegs,
                                int s3, int s_mid, const float *gout, int s1, int grad_is_log,
                                int B, int n, int k, float *dw1, float *const *dleg, int accumulate,
                                cudaStream_t stream)
{
    if ((grad_is_log != 0 && grad_is_log != 1) || (accumulate != 0 && accumulate != 1)) return GM_ERR_INVALID_ARG;
    SerArgs a{};
    gm_status st = chain_args(a1_idx, a1_w, s2, leg_idx, leg_w, nlegs, s3, s_mid, s1, B, n, k, a);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!gout || !dw1 || !dleg) return GM_ERR_INVALID_ARG;
    gm::ChainBwdArgs b{};
    check_chain_edges(a, stream);
    b.f = a;
    b.gout = gout;
    b.grad_is_log = grad_is_log;
    b.dw1 = dw1;
    b.accumulate = accumulate;
    for (int m = 0; m < nlegs; ++m) {
        if (!dleg[m]) return GM_ERR_INVALID_ARG;
        b.dleg[m] = dleg[m];
    }
    if (!accumulate) {  // every leg gradient is scatter-added: clear them all first
        for (int m = 0; m < nlegs; ++m) {
            gm::zero_i32_kernel<<<148 * 4, 256, 0, stream>>>(reinterpret_cast<int32_t *>(dleg[m]),
                                                               (int64_t)a.rows * s3);
            if (launched() != GM_OK) return GM_ERR_CUDA;
        }
    }
    // one thread per row for budgets 2 or 4 (vector loads need 16-byte aligned legs)
    bool aligned = aligned16(a1_idx) && aligned16(a1_w);
    for (int m = 0; m < nlegs; ++m) aligned = aligned && aligned16(leg_idx[m]) && aligned16(leg_w[m]);
    if (aligned && s2 == s3 && s_mid == s2 && (s2 == 2 || s2 == 4) && s1 <= 4 && nlegs <= 4) {
        const unsigned tgrid = blocks_for(a.rows, 32 * WPB_SER_THREAD);
        constexpr int W = WPB_SER_THREAD;
        if (s2 == 2) {
            switch (nlegs) {
            case 1: gm::ser_chain_bwd_thread_kernel<2, 1, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            case 2: gm::ser_chain_bwd_thread_kernel<2, 2, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            case 3: gm::ser_chain_bwd_thread_kernel<2, 3, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            default: gm::ser_chain_bwd_thread_kernel<2, 4, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            }
        } else {
            switch (nlegs) {
            case 1: gm::ser_chain_bwd_thread_kernel<4, 1, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            case 2: gm::ser_chain_bwd_thread_kernel<4, 2, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            case 3: gm::ser_chain_bwd_thread_kernel<4, 3, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            default: gm::ser_chain_bwd_thread_kernel<4, 4, W><<<tgrid, W * 32, 0, stream>>>(b); break;
            }
        }
        return launched();
    }
    const unsigned grid = blocks_for(a.rows, WPB_SER);
    switch (nlegs) {
    case 1: gm::ser_chain_bwd_kernel<1, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(b); break;
    case 2: gm::ser_chain_bwd_kernel<2, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(b); break;
    case 3: gm::ser_chain_bwd_kernel<3, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(b); break;
    case 4: gm::ser_chain_bwd_kernel<4, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(b); break;
    case 5: gm::ser_chain_bwd_kernel<5, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(b); break;
    case 6: gm::ser_chain_bwd_kernel<6, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(b); break;
    default: gm::ser_chain_bwd_kernel<7, WPB_SER><<<grid, WPB_SER * 32, 0, stream>>>(b); break;
    }
    return launched();
}

gm_status gm_ser_sea_chain_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                                   const int32_t *const *leg_idx, const float *const *leg_w,
                                   int nlegs, int s3, int s_mid, int32_t *out_idx, float *out_w,
                                   int s1, const void *q, const void *k, const void *v,
                                   gm_dtype dtype, int B, int n, int hq, int hkv, int d,
                                   float scale, void *o, float *lse, cudaStream_t stream)
{
    if ((out_idx == nullptr) != (out_w == nullptr)) return GM_ERR_INVALID_ARG;
    SerArgs sa{};
    gm_status st = chain_args(a1_idx, a1_w, s2, leg_idx, leg_w, nlegs, s3, s_mid, s1, B, n, hkv, sa);
    if (st != GM_OK) return st;
    const int32_t dummy_idx = 0;
    const float dummy_w = 0.0f;
    st = check_sea(q, k, v, dtype, &dummy_idx, &dummy_w, s1, B, n, hq, hkv, d, scale);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!o || !aligned16(o)) return GM_ERR_INVALID_ARG;
    check_chain_edges(sa, stream);
    sa.out_idx = out_idx;
    sa.out_w = out_w;
    SeaArgs a{q, k, v, nullptr, nullptr, o, lse, s1, n, hkv, scale, sa.rows, row_map(hkv, n)};
    if (nlegs > 1) {
        st = dispatch<SerSeaFwd>(dtype, d, hq / hkv, sa, a, stream);
        if (st != GM_ERR_UNSUPPORTED) return st;
        // no fused kernel for this shape: the chain writes A', then SEA reads it
        if (!out_idx) return GM_ERR_UNSUPPORTED;
        st = gm_ser_chain_forward(a1_idx, a1_w, s2, leg_idx, leg_w, nlegs, s3, s_mid, out_idx, out_w,
                                  s1, B, n, hkv, stream);
        if (st != GM_OK) return st;
        return gm_sea_forward(q, k, v, dtype, out_idx, out_w, s1, B, n, hq, hkv, d, scale, o, lse,
                              stream);
    }
    return gm_ser_sea_forward(a1_idx, a1_w, s2, leg_idx[0], leg_w[0], s3, out_idx, out_w, s1, q, k, v,
                              dtype, B, n, hq, hkv, d, scale, o, lse, stream);
}

gm_status gm_sea_forward(const void *q, const void *k, const void *v, gm_dtype dtype,
                         const int32_t *idx, const float *w, int s,
                         int B, int n, int hq, int hkv, int d, float scale,
                         void *o, float *lse, cudaStream_t stream)
{
    gm_status st = check_sea(q, k, v, dtype, idx, w, s, B, n, hq, hkv, d, scale);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!o || !aligned16(o)) return GM_ERR_INVALID_ARG;
    check_edges(idx, w, s, B, n, hkv, stream);
    SeaArgs a{q, k, v, idx, w, o, lse, s, n, hkv, scale, (uint32_t)((int64_t)B * n * hkv),
              row_map(hkv, n)};
    return dispatch<SeaFwd>(dtype, d, hq / hkv, a, stream);
}

gm_status gm_ser_sea_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                             const int32_t *a2_idx, const float *a2_w, int s3,
                             int32_t *out_idx, float *out_w, int s1,
                             const void *q, const void *k, const void *v, gm_dtype dtype,
                             int B, int n, int hq, int hkv, int d, float scale,
                             void *o, float *lse, cudaStream_t stream)
{
    if ((out_idx == nullptr) != (out_w == nullptr)) return GM_ERR_INVALID_ARG;
    gm_status st = check_ser(a1_idx, a1_w, s2, a2_idx, a2_w, s3, s1, B, n, hkv);
    if (st != GM_OK) return st;
    // the referral output is the attention's edge set: validate SEA with a stand-in pointer
    const int32_t dummy_idx = 0;
    const float dummy_w = 0.0f;
    st = check_sea(q, k, v, dtype, &dummy_idx, &dummy_w, s1, B, n, hq, hkv, d, scale);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!o || !aligned16(o)) return GM_ERR_INVALID_ARG;
    check_edges(a1_idx, a1_w, s2, B, n, hkv, stream);
    check_edges(a2_idx, a2_w, s3, B, n, hkv, stream);
    const uint32_t rows = (uint32_t)((int64_t)B * n * hkv);
    SerArgs sa{a1_idx, a1_w, a2_idx, a2_w, out_idx, out_w, s1, s2, s3, n, hkv, rows, row_map(hkv, n)};
    SeaArgs a{q, k, v, nullptr, nullptr, o, lse, s1, n, hkv, scale, rows, row_map(hkv, n)};
    return dispatch<SerSeaFwd>(dtype, d, hq / hkv, sa, a, stream);
}

size_t gm_sea_backward_workspace_size(gm_dtype dtype, int s, int B, int n, int hq, int hkv, int d)
{
    if (B <= 0 || n <= 0 || hq < 1 || hkv < 1 || hq % hkv != 0 || s < 1) return 0;
    const int64_t R = (int64_t)B * n * hkv;
    if (R >= MAX_ROWS || !gather_supported(dtype, d, hq / hkv, s, R * s)) return 0;
    return ws_layout(R, R * s, hq / hkv).total;
}

gm_status gm_sea_backward(const void *q, const void *k, const void *v, const void *dout,
                          gm_dtype dtype, const int32_t *idx, const float *w, int s,
                          int B, int n, int hq, int hkv, int d, float scale,
                          float *dq, float *dk, float *dv, float *dlogw,
                          void *workspace, size_t workspace_bytes, int accumulate, cudaStream_t stream)
{
    if (accumulate != 0 && accumulate != 1) return GM_ERR_INVALID_ARG;
    gm_status st = check_sea(q, k, v, dtype, idx, w, s, B, n, hq, hkv, d, scale);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!dout || !dq || !dk || !dv || !dlogw) return GM_ERR_INVALID_ARG;
    if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return GM_ERR_INVALID_ARG;
    check_edges(idx, w, s, B, n, hkv, stream);
    const int64_t rows = (int64_t)B * n * hkv;
    SeaBwdArgs a{q, k, v, dout, idx, w, dq, dk, dv, dlogw, nullptr, nullptr, nullptr,
                 s, n, hkv, scale, accumulate, (uint32_t)rows, row_map(hkv, n)};

    const size_t need = gm_sea_backward_workspace_size(dtype, s, B, n, hq, hkv, d);
    if (workspace != nullptr && need > 0) {
        if (workspace_bytes < need || !aligned16(workspace)) return GM_ERR_INVALID_ARG;
        const WsLayout L = ws_layout(rows, rows * s, hq / hkv);
        const gm::GatherWs ws = gather_ws(workspace, L);
        return dispatch<SeaBwdGather>(dtype, d, hq / hkv, a, ws, idx, w, stream);
    }

    // no workspace (or a shape the gather path does not cover): fp32 scatter atomics
    if (!accumulate) {
        const int64_t count4 = rows * d / 4;
        const int64_t want = (count4 + 255) / 256;
        const unsigned grid = (unsigned)(want < 148 * 16 ? want : 148 * 16);
        gm::zero2_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<float4 *>(dk),
                                                    reinterpret_cast<float4 *>(dv), count4);
        if (launched() != GM_OK) return GM_ERR_CUDA;
    }
    return dispatch<SeaBwd>(dtype, d, hq / hkv, a, stream);
}

gm_status gm_sea_backward_noalloc(const void *q, const void *k, const void *v, const void *dout,
                                  gm_dtype dtype, const int32_t *idx, const float *w, int s,
                                  int B, int n, int hq, int hkv, int d, float scale,
                                  float *dq, float *dk, float *dv, float *dlogw,
                                  int accumulate, cudaStream_t stream)
{
    if (accumulate != 0 && accumulate != 1) return GM_ERR_INVALID_ARG;
    gm_status st = check_sea(q, k, v, dtype, idx, w, s, B, n, hq, hkv, d, scale);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    const size_t need = gm_sea_backward_workspace_size(dtype, s, B, n, hq, hkv, d);
    if (need == 0) return GM_ERR_UNSUPPORTED;
    if (need > NOALLOC_SCRATCH_BYTES) return GM_ERR_SCRATCH_TOO_SMALL;
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != GM_OK) return st;
    return gm_sea_backward(q, k, v, dout, dtype, idx, w, s, B, n, hq, hkv, d, scale, dq, dk, dv, dlogw,
                           scratch, NOALLOC_SCRATCH_BYTES, accumulate, stream);
}

size_t gm_sea_backward_noalloc_max_scratch(void) { return NOALLOC_SCRATCH_BYTES; }

gm_status gm_ser_sea_backward(const void *q, const void *k, const void *v, const void *dout, gm_dtype dtype,
                              const int32_t *a1_idx, const float *a1_w, int s2,
                              const int32_t *a2_idx, const float *a2_w, int s3,
                              const int32_t *idx, const float *w, int s1,
                              int B, int n, int hq, int hkv, int d, float scale,
                              float *dq, float *dk, float *dv, float *dlogw, float *dw1, float *dw2,
                              void *workspace, size_t workspace_bytes, int accumulate, cudaStream_t stream)
{
    if (accumulate != 0 && accumulate != 1) return GM_ERR_INVALID_ARG;
    gm_status st = check_ser(a1_idx, a1_w, s2, a2_idx, a2_w, s3, s1, B, n, hkv);
    if (st != GM_OK) return st;
    st = check_sea(q, k, v, dtype, idx, w, s1, B, n, hq, hkv, d, scale);
    if (st != GM_OK || (int64_t)B * n == 0) return st;
    if (!dout || !dq || !dk || !dv || !dlogw || !dw1 || !dw2) return GM_ERR_INVALID_ARG;
    if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return GM_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * n * hkv;
    const size_t need = gm_sea_backward_workspace_size(dtype, s1, B, n, hq, hkv, d);
    const bool legs_aligned = aligned16(a1_idx) && aligned16(a1_w) && aligned16(a2_idx) && aligned16(a2_w);
    const bool fused = workspace != nullptr && need > 0 && legs_aligned && s2 == s3 && (s2 == 2 || s2 == 4) && s1 <= 4;
    if (!fused) {
        // the unfused pair: attention backward, then the referral backward of its d ln w (which
        // needs this call's d ln w alone: no accumulation into the caller's)
        if (accumulate) return GM_ERR_UNSUPPORTED;
        st = gm_sea_backward(q, k, v, dout, dtype, idx, w, s1, B, n, hq, hkv, d, scale, dq, dk, dv, dlogw,
                             workspace, workspace_bytes, 0, stream);
        if (st != GM_OK) return st;
        return gm_ser_backward(a1_idx, a1_w, s2, a2_idx, a2_w, s3, dlogw, s1, 1, B, n, hkv, dw1, dw2, 0,
                               stream);
    }
    if (workspace_bytes < need || !aligned16(workspace)) return GM_ERR_INVALID_ARG;
    check_edges(a1_idx, a1_w, s2, B, n, hkv, stream);
    check_edges(a2_idx, a2_w, s3, B, n, hkv, stream);
    check_edges(idx, w, s1, B, n, hkv, stream);
    if (!accumulate) {
        gm::zero_i32_kernel<<<148 * 4, 256, 0, stream>>>(reinterpret_cast<int32_t *>(dw2), rows * s3);
        if (launched() != GM_OK) return GM_ERR_CUDA;
    }
    SeaBwdArgs a{q, k, v, dout, idx, w, dq, dk, dv, dlogw, nullptr, nullptr, nullptr,
                 s1, n, hkv, scale, accumulate, (uint32_t)rows, row_map(hkv, n),
                 a1_idx, a2_idx, a1_w, a2_w, dw1, dw2};
    const WsLayout L = ws_layout(rows, rows * s1, hq / hkv);
    const gm::GatherWs ws = gather_ws(workspace, L);
    return dispatch<SeaBwdGather>(dtype, d, hq / hkv, a, ws, idx, w, stream, s2);
}

gm_status gm_dense_refresh_edges(const void *q, const void *k, gm_dtype dtype, const float *lse,
                                 int B, int n, int hq, int hkv, int d, float scale, int sf,
                                 int32_t *out_idx, float *out_w, cudaStream_t stream)
{
    if (B < 0 || n < 0 || hq < 1 || hkv < 1 || d < 1 || sf < 1 || sf > 8) return GM_ERR_INVALID_ARG;
    if (hq % hkv != 0 || !std::isfinite(scale)) return GM_ERR_INVALID_ARG;
    if (dtype != GM_F32 && dtype != GM_BF16) return GM_ERR_INVALID_ARG;
    const int G = hq / hkv;
    if (dtype != GM_BF16 || (d != 64 && d != 128) || (G != 1 && G != 2 && G != 4)) return GM_ERR_UNSUPPORTED;
    if ((int64_t)B * n == 0) return GM_OK;
    if ((int64_t)B * n * hq >= MAX_ROWS) return GM_ERR_UNSUPPORTED;
    if (!q || !k || !lse || !out_idx || !out_w) return GM_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k)) return GM_ERR_INVALID_ARG;
    gm::DenseRefreshArgs a{};
    a.lse = lse;
    a.out_idx = out_idx;
    a.out_w = out_w;
    a.n = n;
    a.hq = hq;
    a.hkv = hkv;
    a.sf = sf;
    a.nblk = (n + 127) / 128;
    a.BH = B * hkv;
    a.sl2 = scale * gm::LOG2E;
    const int64_t tokens = (int64_t)B * n;
    return d == 64 ? dense_refresh_g<64>(q, k, tokens, G, a, stream) : dense_refresh_g<128>(q, k, tokens, G, a, stream);
}

gm_status gm_check_device_errors(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GM_ERR_CUDA;
    unsigned flag = 0;
    if (cudaMemcpyFromSymbol(&flag, gm::g_error_flag, sizeof(flag)) != cudaSuccess) return GM_ERR_CUDA;
    if (flag == 0) return GM_OK;
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(gm::g_error_flag, &zero, sizeof(zero)) != cudaSuccess) return GM_ERR_CUDA;
    if (flag & gm::ERR_WAIT_TIMEOUT) return GM_ERR_WAIT_TIMEOUT;
    return (flag & gm::ERR_EDGE_INVALID) ? GM_ERR_EDGE_INVALID : GM_ERR_INDEX_RANGE;
}

}  // extern "C"
