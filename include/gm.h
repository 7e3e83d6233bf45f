/*
 * gm.h - C ABI of the Graph Machine sparse-layer library for NVIDIA B200 (sm_100a).
 *
 * The library computes the data-parallel hot path of one Graph Machine sparse layer, as
 * described in "Graph Machine: Towards Better Pretraining via Edges" (arXiv 2609.02881;
 * ai.info summary, "Key Contributions" items 2-3 and "Methodology in Plain English"):
 *
 *   - sparse edge referral (SER): A' = Sparsify_s1(A1 A2), two-hop composition of each
 *     position's edges, duplicate targets merged by summation, top-s1 kept;
 *   - sparse edge attention (SEA): K/V gathered at each position's edge indices per KV head,
 *     shared by the query heads of the GQA group, score = scale * q.k + ln w, softmax over
 *     the entries, weighted sum of V;
 *   - the backward passes of both (SEA: dq, dk, dv, d ln w; SER: gradients of the kept
 *     referral weights with respect to both legs' weights);
 *   - around the referral: the legs built from the stored edges (mixed across the k edge
 *     channels and sparsified, gm_leg_sparsify) and their backward; refresh edges joining
 *     the referral's candidates (gm_ser_refresh_*); multi-step referral chains
 *     (gm_ser_chain_*), each also fused with SEA.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout. All tensors are dense, contiguous, row-major device arrays:
 *   features  q, o, dout, dq  [B, n, hq,  d]
 *             k, v, dk, dv    [B, n, hkv, d]
 *   edges     idx (int32), w (fp32), dlogw (fp32)   [B, n, k, s]   (k edge channels)
 *   lse       fp32 [B, n, hq]
 * In SEA the edge channel h drives KV head h (k = hkv), and query head hq reads KV head
 * hq / (hq_count / hkv) (contiguous GQA groups).
 *
 * Edge semantics. A slot (index, weight) is active iff weight > 0. Inactive slots are never
 * dereferenced. An active slot whose index lies outside [0, n) is treated as inactive and
 * raises the device error flag (see gm_check_device_errors); kernels never trap. Weights are
 * expected finite and >= 0; indices are expected causal (<= the row's own position); the
 * regular build does not check this, the checked build does (gm_checked_build). Position 0
 * of each sequence is the padding token: SER pads missing output slots with (index 0,
 * weight 0.0f).
 *
 * Ownership and synchrony. The caller allocates and owns every buffer. Entry points allocate
 * no device memory, enqueue their kernels on `stream` (0 = the legacy default stream) and
 * return without synchronising; only gm_check_device_errors synchronises.
 *
 * Errors. Argument checks are synchronous and happen before any launch:
 *   GM_ERR_INVALID_ARG  null pointer, negative size, hq % hkv != 0, non-finite scale,
 *                       misaligned feature pointer (16 bytes required), s out of [1, 32];
 *   GM_ERR_UNSUPPORTED  a valid shape the library has no kernel for (see each function);
 *   GM_ERR_CUDA         the launch failed (cudaGetLastError after the launch);
 *   GM_ERR_INDEX_RANGE, GM_ERR_EDGE_INVALID, GM_ERR_WAIT_TIMEOUT
 *                       returned by gm_check_device_errors only.
 * B == 0 or n == 0 is an empty problem: GM_OK, nothing launched.
 */
#ifndef GM_H
#define GM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *cudaStream_t;

typedef enum gm_status {
    GM_OK = 0,
    GM_ERR_INVALID_ARG = 1,
    GM_ERR_UNSUPPORTED = 2,
    GM_ERR_CUDA = 3,
    GM_ERR_INDEX_RANGE = 4,
    GM_ERR_SCRATCH_TOO_SMALL = 5, /* gm_sea_backward_noalloc only */
    GM_ERR_WAIT_TIMEOUT = 6,      /* from gm_check_device_errors: a kernel gave up on a wait */
    GM_ERR_EDGE_INVALID = 7       /* from gm_check_device_errors, checked builds only */
} gm_status;

/* Element type of q, k, v, o and dout. */
typedef enum gm_dtype {
    GM_F32 = 0,
    GM_BF16 = 1
} gm_dtype;

/*
 * gm_leg_sparsify - the pair of referral legs of every (token, edge channel), built from the
 * stored edges.
 * Source: ai.info summary, "Methodology in Plain English", referral paragraph (the stored
 * edges are mixed into pairs and each leg is sparsified before the composition) and "Main
 * Findings", bullet on more edges (the cross-edge mixing is full: its cost grows as k^2).
 * The pages give no formula; the reading here: leg L of channel h at token (b, i) mixes the
 * token's own stored edges across all k stored channels.
 *
 * For each (b, i, h) and leg L (coefficients M_L, budget s_L = s2 for leg 1, s3 for leg 2):
 * every stored edge (c, a), c < k, a < s0, with e_w[b,i,c,a] > 0 is a candidate with target
 * e_idx[b,i,c,a] and weight fl32(M_L[b,i,h,c] * e_w[b,i,c,a]) (one rounding, no FMA), in
 * ascending c*s0 + a. Zero products are dropped; candidates reaching the same target are
 * summed in fp32 in that order; the s_L heaviest targets are written in order of weight
 * descending, then target ascending, padded with (0, 0.0f). No renormalisation. This is
 * gm_ser_forward's sparsify applied to the mixed candidates; the outputs are its legs.
 *
 *   e_idx, e_w        device, [B, n, k, s0]   stored edges (int32 targets, fp32 weights >= 0)
 *   mix1, mix2        device fp32, coefficients >= 0 of leg 1 and leg 2: [B, n, k, k]
 *                     (mix_token_stride = k*k) or one [k, k] matrix shared by every token
 *                     (mix_token_stride = 0); element [h, c] mixes stored channel c into
 *                     leg channel h
 *   a1_idx, a1_w      device, [B, n, k, s2]   leg 1, written
 *   a2_idx, a2_w      device, [B, n, k, s3]   leg 2, written; outputs must not alias inputs
 *   limits            1 <= k*s0 <= 32, 1 <= s2, s3 <= 32
 * An active stored edge whose target lies outside [0, n) is skipped and raises the device
 * index-range flag (read by gm_check_device_errors). Deterministic, bit-identical to the
 * definition above.
 */
gm_status gm_leg_sparsify(const int32_t *e_idx, const float *e_w, int s0,
                          const float *mix1, const float *mix2, int64_t mix_token_stride,
                          int32_t *a1_idx, float *a1_w, int s2,
                          int32_t *a2_idx, float *a2_w, int s3,
                          int B, int n, int k, cudaStream_t stream);

/*
 * gm_leg_backward - gradients of gm_leg_sparsify's kept leg weights with respect to the stored
 * weights and both sets of mixing coefficients.
 * Source: as gm_leg_sparsify; and the referral paragraph's rule that only retained weights get
 * gradients (indices get none).
 *
 * The legs of every token are recomputed exactly as gm_leg_sparsify computes them. Each kept
 * weight W_r of leg L, channel h is differentiated as the sum, over the active stored edges
 * (c, a) that reach its target t_r, of M_L[h,c] * e_w[c,a]; with g_r = g_L[b,i,h,r]:
 *   dew[b,i,c,a]       += g_r * M_L[b,i,h,c]
 *   dmix_L[b,i,h,c]    += g_r * e_w[b,i,c,a]
 * summed over h, both legs and the kept slots. An active edge whose product was zero (a zero
 * coefficient) still contributes to dmix. Targets cut by the selection get nothing. fp32; each
 * output is summed by one warp in a fixed order (deterministic, no atomics).
 *
 *   e_idx, e_w, mix1, mix2, mix_token_stride, s0, k   as gm_leg_sparsify
 *   g1          device fp32 [B, n, k, s2]   gradient w.r.t. leg 1's weights (gm_ser_backward's dw1)
 *   g2          device fp32 [B, n, k, s3]   gradient w.r.t. leg 2's weights (gm_ser_backward's dw2)
 *   dew         device fp32 [B, n, k, s0]   written (added to if accumulate)
 *   dmix1/2     device fp32 [B, n, k, k]    written (added to if accumulate), per token also
 *               when the coefficients were shared (mix_token_stride = 0): the caller sums them
 *   limits      as gm_leg_sparsify
 */
gm_status gm_leg_backward(const int32_t *e_idx, const float *e_w, int s0,
                          const float *mix1, const float *mix2, int64_t mix_token_stride,
                          const float *g1, int s2, const float *g2, int s3,
                          int B, int n, int k, float *dew, float *dmix1, float *dmix2,
                          int accumulate, cudaStream_t stream);

/*
 * gm_ser_forward - sparse edge referral, A' = Sparsify_s1(A1 A2).
 * Source: ai.info summary, "Key Contributions" item 3 (A' = Sparsify_s1(A1 A2), up to s2*s3
 * candidates cut back to s1) and "Methodology in Plain English", referral paragraph (the
 * first leg's indices fetch the second leg's indices and weights; hard top-s selection).
 *
 * For each (b, i, h): candidate c = a*s3 + e (a < s2, e < s3) is the path
 * i -> j = a1_idx[b,i,h,a] -> t = a2_idx[b,j,h,e] with weight fl32(a1_w[..a] * a2_w[..e])
 * (one fp32 rounding, no FMA). Zero-weight candidates are dropped; candidates that reach the
 * same t are summed in fp32, in ascending c, each add rounded to nearest. The s1 heaviest
 * targets are written to out_idx/out_w[b,i,h,0..s1) in order of weight descending, then
 * index ascending; missing slots are (0, 0.0f). No renormalisation.
 *
 *   a1_idx, a1_w   device, [B, n, k, s2]        first leg
 *   a2_idx, a2_w   device, [B, n, k, s3]        second leg (channel h reads channel h)
 *   out_idx, out_w device, [B, n, k, s1]        written; must not alias the inputs
 *   limits         1 <= s2*s3 <= 32, 1 <= s1 <= 32, k >= 1
 * Result is deterministic and bit-identical to the plain definition above.
 */
gm_status gm_ser_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                         const int32_t *a2_idx, const float *a2_w, int s3,
                         int32_t *out_idx, float *out_w, int s1,
                         int B, int n, int k, cudaStream_t stream);

/*
 * gm_ser_backward - gradients of gm_ser_forward's kept weights with respect to both legs'
 * weights.
 * Source: ai.info summary, "Methodology in Plain English", referral paragraph (hard top-s
 * selection; only retained weights get gradients; indices get none).
 *
 * The referral of every row is recomputed exactly as gm_ser_forward computes it (same
 * candidates, merge and selection). For every candidate c = (a, e) of row (b,i,h) whose
 * target was kept in output slot r with weight W_r > 0, and g_r = gout[b,i,h,r] (divided by
 * W_r when grad_is_log = 1, i.e. when gout is the gradient with respect to ln A'.w, as
 * gm_sea_backward's dlogw is):
 *   dw1[b,i,h,a]  += g_r * a2_w[b,j,h,e]      (j = a1_idx[b,i,h,a])
 *   dw2[b,j,h,e]  += g_r * a1_w[b,i,h,a]      (summed over every row that reaches it)
 * Candidates cut by the top-s1 get nothing. fp32 throughout; dw1 is summed in a fixed order,
 * dw2 with fp32 atomics (order varies run to run).
 *
 *   a1_idx/a1_w, a2_idx/a2_w, s1   as gm_ser_forward (k edge channels)
 *   gout        device fp32 [B, n, k, s1]
 *   grad_is_log 0: gout is dL/dA'.w; 1: gout is dL/d ln A'.w
 *   dw1         device fp32 [B, n, k, s2], written (added to if accumulate)
 *   dw2         device fp32 [B, n, k, s3], zeroed by a library kernel then scatter-added
 *               (added to without zeroing if accumulate)
 *   limits      as gm_ser_forward
 */
gm_status gm_ser_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                          const int32_t *a2_idx, const float *a2_w, int s3,
                          const float *gout, int s1, int grad_is_log,
                          int B, int n, int k, float *dw1, float *dw2, int accumulate,
                          cudaStream_t stream);

/*
 * gm_ser_refresh_forward - referral with refresh edges, A' = Sparsify_s1(A1 A2 + F).
 * Source: ai.info summary, "Methodology in Plain English", referral paragraph (optional refresh
 * edges pull in the input edges or the top positions of the latest dense attention layer) and
 * "Main Findings", bullet on refresh and realignment (they help). The pages give no formula;
 * the reading here: the refresh edges are one more sparse edge set that joins the referral's
 * candidates before the cut.
 *
 * As gm_ser_forward, with sf refresh candidates after the s2*s3 two-hop paths: candidate
 * s2*s3 + f of row (b,i,h) is (f_idx[b,i,h,f], f_w[b,i,h,f]) with its own weight (weight > 0;
 * zero weights are dropped). Merge (fp32, ascending candidate order), order and cut as
 * gm_ser_forward; bit-identical to that definition.
 *
 *   f_idx, f_w  device, [B, n, k, sf]   refresh edges (int32 targets, fp32 weights >= 0)
 *   other arguments as gm_ser_forward
 *   limits      1 <= sf, s2*s3 + sf <= 32, 1 <= s1 <= 32
 * An active refresh slot whose index lies outside [0, n) is skipped and raises the device
 * index-range flag.
 */
gm_status gm_ser_refresh_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                                 const int32_t *a2_idx, const float *a2_w, int s3,
                                 const int32_t *f_idx, const float *f_w, int sf,
                                 int32_t *out_idx, float *out_w, int s1,
                                 int B, int n, int k, cudaStream_t stream);

/*
 * gm_ser_refresh_backward - gradients of gm_ser_refresh_forward's kept weights with respect to
 * both legs' weights and the refresh weights.
 * Source: as gm_ser_refresh_forward; only retained weights get gradients (referral paragraph).
 *
 * As gm_ser_backward for the path candidates; a refresh slot f whose target was kept in slot r
 * receives dfw[b,i,h,f] = g_r (the merged weight is a plain sum of it). Cut targets get nothing.
 *
 *   f_idx, f_w, sf   as gm_ser_refresh_forward
 *   dfw              device fp32 [B, n, k, sf], written (added to if accumulate)
 *   other arguments as gm_ser_backward
 */
gm_status gm_ser_refresh_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                                  const int32_t *a2_idx, const float *a2_w, int s3,
                                  const int32_t *f_idx, const float *f_w, int sf,
                                  const float *gout, int s1, int grad_is_log,
                                  int B, int n, int k, float *dw1, float *dw2, float *dfw,
                                  int accumulate, cudaStream_t stream);

/*
 * gm_ser_sea_refresh_forward - gm_ser_refresh_forward followed by gm_sea_forward on its result,
 * in one kernel (as gm_ser_sea_forward, with the refresh edges f_idx/f_w/sf of
 * gm_ser_refresh_forward). Same arguments, limits and results as the two calls in sequence.
 */
gm_status gm_ser_sea_refresh_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                                     const int32_t *a2_idx, const float *a2_w, int s3,
                                     const int32_t *f_idx, const float *f_w, int sf,
                                     int32_t *out_idx, float *out_w, int s1,
                                     const void *q, const void *k, const void *v, gm_dtype dtype,
                                     int B, int n, int hq, int hkv, int d, float scale,
                                     void *o, float *lse, cudaStream_t stream);

/*
 * gm_ser_chain_forward - multi-step referral: B_1 = A1, B_{m+1} = Sparsify(B_m A_{m+1}),
 * A' = B_l, for legs A2 .. Al.
 * Source: ai.info summary, "Key Contributions" item 2 (the soft sparse adjacency matrix is
 * raised to the l-th power and the result is sparsified) and "Main Findings", bullet on
 * referral (models with 3 and 4 legs; more steps do not always help). The pages give no
 * formula for the intermediate cuts; the reading here: every step is gm_ser_forward's
 * referral applied to the row's previous result, intermediates cut to s_mid slots, the last
 * step to s1.
 *
 *   a1_idx, a1_w     device, [B, n, k, s2]        first leg
 *   leg_idx, leg_w   HOST arrays of nlegs device pointers, each [B, n, k, s3]: the legs
 *                    A2 .. A(nlegs+1) in chain order (they may be the same tensor: A^l)
 *   nlegs            1 .. 7 (1 is gm_ser_forward)
 *   s_mid            slots of every intermediate (1 <= s_mid, s_mid*s3 <= 32)
 *   out_idx, out_w   device, [B, n, k, s1], written
 *   other limits     as gm_ser_forward
 * Deterministic and bit-identical to the steps above in sequence; no intermediate is written.
 */
gm_status gm_ser_chain_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                               const int32_t *const *leg_idx, const float *const *leg_w, int nlegs,
                               int s3, int s_mid, int32_t *out_idx, float *out_w, int s1,
                               int B, int n, int k, cudaStream_t stream);

/*
 * gm_ser_chain_backward - gradients of gm_ser_chain_forward's kept weights with respect to the
 * first leg's and every chain leg's weights.
 * Source: as gm_ser_chain_forward; only retained weights get gradients (referral paragraph).
 *
 * The chain is recomputed; the gradient runs back through the steps (each step as
 * gm_ser_backward, every intermediate's kept set held as the forward chose it).
 *
 *   gout, grad_is_log  as gm_ser_backward (grad_is_log applies to the final A')
 *   dw1                device fp32 [B, n, k, s2], written (added to if accumulate)
 *   dleg               HOST array of nlegs device pointers, fp32 [B, n, k, s3] each: the
 *                      legs' gradients, zeroed by library kernels then scatter-added (added to
 *                      without zeroing if accumulate); pointers may alias when legs do (the
 *                      contributions then add up)
 *   other arguments    as gm_ser_chain_forward
 */
gm_status gm_ser_chain_backward(const int32_t *a1_idx, const float *a1_w, int s2,
                                const int32_t *const *leg_idx, const float *const *leg_w, int nlegs,
                                int s3, int s_mid, const float *gout, int s1, int grad_is_log,
                                int B, int n, int k, float *dw1, float *const *dleg, int accumulate,
                                cudaStream_t stream);

/*
 * gm_ser_sea_chain_forward - gm_ser_chain_forward followed by gm_sea_forward on its result.
 * One fused kernel for bf16 features, s2 = s3 = s_mid in {2, 4}, s1 <= 4 and nlegs in {2, 3};
 * other shapes run the chain into out_idx/out_w and then SEA (GM_ERR_UNSUPPORTED if those are
 * NULL). Arguments as gm_ser_chain_forward and gm_ser_sea_forward (k = hkv).
 */
gm_status gm_ser_sea_chain_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                                   const int32_t *const *leg_idx, const float *const *leg_w,
                                   int nlegs, int s3, int s_mid, int32_t *out_idx, float *out_w,
                                   int s1, const void *q, const void *k, const void *v,
                                   gm_dtype dtype, int B, int n, int hq, int hkv, int d,
                                   float scale, void *o, float *lse, cudaStream_t stream);

/*
 * gm_sea_forward - sparse edge attention.
 * Source: ai.info summary, "Key Contributions" item 3 (SEA: edge indices select the K/V
 * positions; node factor = scaled q.k, edge factor = log edge weight, combined as a product
 * of experts) and "Methodology in Plain English", SEA paragraph (no RoPE inside SEA).
 *
 * For each (b, i, hq) with h = hq / (hq_count / hkv), over the active slots j of
 * idx/w[b,i,h,:]:  z_j = scale * <q[b,i,hq], k[b,t_j,h]> + ln w_j,  p = softmax(z),
 * o[b,i,hq] = sum_j p_j v[b,t_j,h],  lse[b,i,hq] = ln sum_j exp(z_j).  A row with no active
 * slot gives o = 0 and lse = -inf. Duplicate indices in a row count as separate slots.
 * Arithmetic is fp32 (bf16 inputs widened); o is rounded to `dtype` (nearest even).
 *
 *   q, k, v   device, `dtype`, 16-byte aligned, layouts above
 *   idx, w    device, [B, n, hkv, s], 1 <= s <= 32
 *   o         device, `dtype`, [B, n, hq, d], written
 *   lse       device fp32 [B, n, hq], written; may be NULL
 *   scale     any finite float (1/sqrt(d) for the standard score)
 *   limits    hq/hkv in {1, 2, 4, 8}; d in {32, 64, 128, 256} for GM_BF16 and
 *             {32, 64, 128} for GM_F32 (else GM_ERR_UNSUPPORTED)
 */
gm_status gm_sea_forward(const void *q, const void *k, const void *v, gm_dtype dtype,
                         const int32_t *idx, const float *w, int s,
                         int B, int n, int hq, int hkv, int d, float scale,
                         void *o, float *lse, cudaStream_t stream);

/*
 * gm_ser_sea_forward - SER followed by SEA on its output, in one kernel.
 * Same definitions as gm_ser_forward (with k = hkv) and gm_sea_forward (with s = s1, idx/w =
 * the referral output). The refreshed edges stay on chip between the two steps; they are
 * written to out_idx/out_w once, for the next layer, and never read back. out_idx and out_w
 * may both be NULL when the caller does not need them.
 * Results equal gm_ser_forward then gm_sea_forward bit for bit (every path computes the
 * score dot products in the same order).
 */
gm_status gm_ser_sea_forward(const int32_t *a1_idx, const float *a1_w, int s2,
                             const int32_t *a2_idx, const float *a2_w, int s3,
                             int32_t *out_idx, float *out_w, int s1,
                             const void *q, const void *k, const void *v, gm_dtype dtype,
                             int B, int n, int hq, int hkv, int d, float scale,
                             void *o, float *lse, cudaStream_t stream);

/*
 * gm_sea_backward - gradients of gm_sea_forward.
 * Source: the derivative of the SEA definition above; ai.info summary, "Methodology in
 * Plain English": indices get no gradient, the soft edge weights carry the learning signal.
 *
 * With p, z as in the forward (recomputed here from q, k, v, idx, w; no forward state is
 * needed) and dp_j = <dout, v[t_j]>, dz_j = p_j (dp_j - sum_l p_l dp_l):
 *   dq[b,i,hq]      = scale * sum_j dz_j k[b,t_j,h]
 *   dk[b,t,h]       = sum over the slots (b,i,h,j) with t_j = t of scale * dz_j q[b,i,hq]
 *   dv[b,t,h]       = sum over the same slots of p_j dout[b,i,hq]
 *   dlogw[b,i,h,j]  = sum over the group's query heads of dz_j   (gradient w.r.t. ln w_j)
 * (sums over hq in the group of h). Inactive slots get 0 in dlogw and contribute nothing.
 * All arithmetic is fp32. dk/dv are sums of many terms whose order varies run to run (the
 * set of terms does not), so their last bits may differ between calls.
 *
 * Two execution paths:
 *   - with a workspace (workspace != NULL and the shape is covered, see
 *     gm_sea_backward_workspace_size): dk/dv are gathered per target row from a reverse
 *     edge index built in the workspace; each dk/dv row is written once, without atomics,
 *     except the rows more than 256 slots point at, which are zeroed and then summed by
 *     several warps with 16-byte fp32 atomics;
 *   - without one: dk/dv are zeroed by a library kernel (unless accumulating) and
 *     scatter-added with 16-byte fp32 atomics.
 *
 *   q, k, v, dout       device, `dtype`, 16-byte aligned
 *   idx, w              device, [B, n, hkv, s]
 *   dq                  device fp32 [B, n, hq, d], 16-byte aligned
 *   dk, dv              device fp32 [B, n, hkv, d], 16-byte aligned
 *   dlogw               device fp32 [B, n, hkv, s]
 *   workspace           device scratch owned by the caller, 16-byte aligned, at least
 *                       gm_sea_backward_workspace_size(...) bytes; its contents on entry do
 *                       not matter and are garbage on return; may be NULL (atomic path);
 *                       too small (but non-NULL) is GM_ERR_INVALID_ARG
 *   accumulate          0: all four outputs are overwritten; 1: results are added to their
 *                       current contents
 *   limits              as gm_sea_forward
 */
gm_status gm_sea_backward(const void *q, const void *k, const void *v, const void *dout,
                          gm_dtype dtype, const int32_t *idx, const float *w, int s,
                          int B, int n, int hq, int hkv, int d, float scale,
                          float *dq, float *dk, float *dv, float *dlogw,
                          void *workspace, size_t workspace_bytes,
                          int accumulate, cudaStream_t stream);

/*
 * gm_sea_backward_workspace_size - bytes of workspace gm_sea_backward needs for its gather
 * path on this shape, or 0 when the gather path does not cover it (then pass NULL). Covered:
 * s <= 4, head_dim 64 or 128 with hq/hkv <= 2 for GM_BF16, head_dim 64 with hq/hkv <= 4 for
 * GM_F32. The size grows as 8*(B*n*hkv) + 36*(B*n*hkv*s) bytes (hq/hkv <= 2) plus padding.
 * Pure host function; no CUDA call.
 */
size_t gm_sea_backward_workspace_size(gm_dtype dtype, int s, int B, int n, int hq, int hkv, int d);

/*
 * gm_sea_backward_noalloc - gm_sea_backward for callers that cannot allocate device memory.
 * The paper has no counterpart to this entry point; it exists for the caller, not the method.
 *
 * Some callers may not allocate device memory at the point where they run the backward:
 * code called from inside a memory allocator's own hooks (which must not re-enter it), a
 * runtime that has given all device memory to its own pool and has no way to hand out a
 * workspace for this call, or a step loop whose policy forbids allocation because
 * cudaMalloc/cudaFree can synchronise the device and fragment memory. This entry point takes
 * exactly the arguments of gm_sea_backward minus the workspace, and runs its gather path on
 * a fixed scratch array that the library holds in device memory
 * (gm_sea_backward_noalloc_max_scratch() bytes, 32 MiB, on every device that loads the
 * library, until the process exits). It allocates nothing and calls no allocating routine.
 *
 *   - The first call on a device looks up the array's device address on that device (with it
 *     current) and caches it; make that first call before any stream capture.
 *   - All calls on a device share the array, which keeps the last call's contents (every call
 *     clears what it needs zeroed). Calls whose execution overlaps on the GPU (for instance on
 *     two streams without ordering) race on it and give wrong results: serialise them.
 *   - Shapes the gather path does not cover (see gm_sea_backward_workspace_size) return
 *     GM_ERR_UNSUPPORTED; a covered shape whose scratch need exceeds the array returns
 *     GM_ERR_SCRATCH_TOO_SMALL (about 152 bytes per edge row at s = 4, hq/hkv = 2: up to
 *     ~220k rows B*n*hkv). Both are checked before anything is launched.
 * Results: as gm_sea_backward with a workspace.
 */
gm_status gm_sea_backward_noalloc(const void *q, const void *k, const void *v, const void *dout,
                                  gm_dtype dtype, const int32_t *idx, const float *w, int s,
                                  int B, int n, int hq, int hkv, int d, float scale,
                                  float *dq, float *dk, float *dv, float *dlogw,
                                  int accumulate, cudaStream_t stream);

/* Size in bytes of the fixed scratch array gm_sea_backward_noalloc uses. Pure host function. */
size_t gm_sea_backward_noalloc_max_scratch(void);

/*
 * gm_ser_sea_backward - the backward of one sparse layer's referral and attention in one call:
 * gm_sea_backward on A' (the referral's output edges), and the referral backward of the d ln w
 * it computes, to both legs' weights. Sources: ai.info summary, "Key Contributions" item 3
 * (SEA on the referral's edges) and "Methodology in Plain English", referral paragraph (only
 * the retained referral weights receive gradient).
 *
 *   q, k, v, dout, dtype, scale, B, n, hq, hkv, d   as gm_sea_backward
 *   a1_idx/a1_w [B, n, hkv, s2], a2_idx/a2_w [B, n, hkv, s3]   the referral's legs
 *   idx/w [B, n, hkv, s1]   A' = Sparsify_s1(A1 A2), exactly as gm_ser_sea_forward returned it
 *                           (its kept set decides which paths receive gradient)
 *   dq, dk, dv, dlogw       as gm_sea_backward (dlogw is required)
 *   dw1 [B, n, hkv, s2], dw2 [B, n, hkv, s3]   gradients of the legs' weights, as
 *                           gm_ser_backward with grad_is_log = 1 and gout = dlogw
 *   workspace, workspace_bytes   as gm_sea_backward (gm_sea_backward_workspace_size(..., s1, ...))
 *   accumulate              0: overwrite every output; 1: add to them (fused shapes only)
 * With a workspace, s2 = s3 in {2, 4}, s1 <= 4, 16-byte aligned legs and a shape the gather
 * path covers, the referral backward runs inside the attention backward's row pass (the d ln w
 * of a tile stays in shared memory, A' is read once); otherwise the call runs gm_sea_backward
 * and then gm_ser_backward (accumulate must then be 0: GM_ERR_UNSUPPORTED otherwise). dw2 is
 * summed with fp32 atomics (order varies run to run); everything else is deterministic.
 * Errors: as gm_sea_backward and gm_ser_backward.
 */
gm_status gm_ser_sea_backward(const void *q, const void *k, const void *v, const void *dout, gm_dtype dtype,
                              const int32_t *a1_idx, const float *a1_w, int s2,
                              const int32_t *a2_idx, const float *a2_w, int s3,
                              const int32_t *idx, const float *w, int s1,
                              int B, int n, int hq, int hkv, int d, float scale,
                              float *dq, float *dk, float *dv, float *dlogw, float *dw1, float *dw2,
                              void *workspace, size_t workspace_bytes, int accumulate, cudaStream_t stream);

/*
 * gm_dense_refresh_edges - refresh edges from a dense attention layer: for every (b, i, KV
 * head h), the sf positions t <= i that the dense layer's attention weights most heavily.
 * Source: ai.info summary, "Methodology in Plain English", referral paragraph (refresh edges
 * are the input edges or the top positions of the most recent dense attention layer); "Main
 * Findings", bullet on refresh and realignment. Reading of the pages (they give no formula):
 * the dense layer is causal softmax attention, P_hq(i, t) = exp(scale <q[i,hq], k[t,h]> -
 * lse[i,hq]) for t <= i, h = hq / (hq_count / hkv); the attention mass of KV head h at t is
 * the mean of P_hq(i, t) over the query heads of its group; the sf positions of largest mass
 * are kept, ties to the smaller position, ordered by mass descending; the edge weight is the
 * mass. Rows with i + 1 < sf are padded with (index 0, weight 0.0f). The result [B, n, hkv, sf]
 * is an edge set for gm_ser_refresh_forward / gm_ser_sea_refresh_forward (k = hkv).
 *
 *   q         [B, n, hq, d]  bf16, the dense layer's queries
 *   k         [B, n, hkv, d] bf16, the dense layer's keys
 *   dtype     GM_BF16 (fp32 features: GM_ERR_UNSUPPORTED)
 *   lse       [B, n, hq] fp32: the dense layer's per-row normaliser (natural log), as its
 *             forward returns it
 *   scale     the dense layer's score scale (1/sqrt(d) for standard attention)
 *   sf        1..8 positions kept per (b, i, h)
 *   out_idx, out_w  [B, n, hkv, sf] int32 / fp32, written in full
 * Limits: d in {64, 128}; hq / hkv in {1, 2, 4}; q and k 16-byte aligned; B * n * hq < 2^31.
 * The scores run on the tensor cores (bf16 products, fp32 sums), the masses in fp32: a
 * position whose mass lies within fp32 rounding of the sf-th largest may be exchanged for
 * another at the same mass.
 * Errors: GM_ERR_INVALID_ARG, GM_ERR_UNSUPPORTED as above; GM_ERR_CUDA if the tensor-map
 * encoder of the driver is unavailable or the launch fails.
 */
gm_status gm_dense_refresh_edges(const void *q, const void *k, gm_dtype dtype, const float *lse,
                                 int B, int n, int hq, int hkv, int d, float scale, int sf,
                                 int32_t *out_idx, float *out_w, cudaStream_t stream);

/*
 * gm_check_device_errors - synchronise `stream`, then read and clear this device's error
 * flag. Returns GM_ERR_INDEX_RANGE if any kernel of this library on the current device met
 * an active slot whose index lay outside [0, n) since the last check, GM_ERR_EDGE_INVALID if
 * (checked build) an input edge broke the edge invariants (see gm_checked_build),
 * GM_ERR_WAIT_TIMEOUT if a kernel gave up on a bounded wait (an asynchronous copy, a
 * tensor-core operation, or the backward scan's look-back at earlier blocks; its outputs are
 * then incomplete), GM_ERR_CUDA if the synchronisation failed, else GM_OK. When several
 * occurred, the first of GM_ERR_WAIT_TIMEOUT, GM_ERR_EDGE_INVALID, GM_ERR_INDEX_RANGE.
 */
gm_status gm_check_device_errors(cudaStream_t stream);

/*
 * gm_selftest_wait_timeout - diagnostic for the bounded waits: launches one kernel whose
 * single wait (on a shared-memory barrier that nothing arrives at) runs out after about one
 * second; the kernel then sets the device error flag and returns, so the following
 * gm_check_device_errors returns GM_ERR_WAIT_TIMEOUT and the device stays usable. The
 * library's real waits (asynchronous copies and tensor-core operations of
 * gm_dense_refresh_edges, the look-back of the backward's scan) give up the same way.
 */
gm_status gm_selftest_wait_timeout(cudaStream_t stream);

/* Static, human-readable name of a status code. Never NULL. */
const char *gm_status_string(gm_status status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int gm_version(void);

/*
 * gm_checked_build - 1 for the checked build of this library (libgm_b200_checked.so), 0 for
 * the regular one. The checked build runs every entry point exactly as the regular build does,
 * after verifying each edge tensor the call reads (first and second legs, refresh edges, chain
 * legs, stored edges, SEA edges): every weight finite and >= 0, every active index (weight > 0,
 * index >= 0) no later than its own row's position i (edges are causal; position 0 is the
 * padding token). A violation is reported by gm_check_device_errors as GM_ERR_EDGE_INVALID.
 * The checks cost one extra pass over each edge tensor.
 */
int gm_checked_build(void);

#ifdef __cplusplus
}
#endif

#endif /* GM_H */
