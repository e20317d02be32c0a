/*
 * vsa.h -- C ABI of the B200 (sm_100a) library for the fine stage of Video
 * Sparse Attention (VSA): block-sparse attention over cube-major 64-token
 * tiles, the cube-mean routing that selects the tiles, and the 4x4x4
 * cube-major layout transforms.
 *
 * Conventions (shared by every entry point):
 *  - Tensor pointers are DEVICE pointers to dense, contiguous, row-major
 *    buffers, at least 16-byte aligned.  The caller owns every buffer; the
 *    library never allocates, frees, synchronises, or falls back to the CPU.
 *  - bf16 values are passed as their 16-bit patterns (vsa_bf16).
 *  - Work is enqueued on `stream`; a call returns once its kernels are
 *    launched.  A status of VSA_OK means the launch was accepted; errors
 *    raised later by the device (bad index found by a kernel, a bounded
 *    wait that ran out) are latched in a device word and read with
 *    vsa_device_status().
 *  - Every function is noexcept in effect: it returns a status and never
 *    aborts.  Arguments are checked before anything is launched; a call that
 *    returns an error has launched nothing.
 *
 * Shapes (the dataset card "wan2.2_production_values", sections "Shapes",
 * "Operator contract" and "Load"):
 *   B batch, H heads, D head dim (= 128), Nq cubes, S = 64 * Nq padded tokens,
 *   q, k, v, out : [B, S, H, D] bf16 (BSHD, cube-major)
 *   topk_idx     : [B, H, Nq, topk] int32, values in [0, Nq)
 *   vbs          : [Nq] int32, values in [0, 64], shared by batch and heads
 *   lse          : [B, H, S] fp32, natural log (optional output)
 */
#ifndef VSA_H
#define VSA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define VSA_API __attribute__((visibility("default")))
#else
#define VSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t vsa_bf16;

enum vsa_status {
    VSA_OK = 0,
    VSA_ERR_ARG = -1,       /* a size or count is out of range (see each call) */
    VSA_ERR_NULL = -2,      /* a required pointer is NULL */
    VSA_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned */
    VSA_ERR_WORKSPACE = -4, /* workspace missing or smaller than the size query says */
    VSA_ERR_ARCH = -5,      /* the current device is not sm_100 */
    VSA_ERR_LAUNCH = -6,    /* the CUDA runtime rejected a launch (cudaGetLastError) */
    VSA_ERR_DEVICE = -7     /* a kernel latched an error (see vsa_device_status) */
};

/* Human-readable name of a status code (static storage). */
VSA_API const char *vsa_status_string(int status);

/* 1 if this library has kernels for head dim D on an SM of version
 * `sm_version` (major*10+minor), else 0.  Only D = 128 on sm_100. */
VSA_API int vsa_can_implement(int D, int sm_version);

/* ------------------------------------------------------------------------
 * vsa_fwd -- fine block-sparse attention forward.
 *
 * Dataset card "wan2.2_production_values", section "Operator contract":
 * non-causal block-sparse attention in BSHD layout,
 *   out = softmax(q . k_sel^T * sm_scale) . v_sel,
 * where, for query cube i of (batch b, head h), k_sel / v_sel are the
 * tokens of the cubes listed in topk_idx[b, h, i, :], and of cube c only the
 * first vbs[c] of its 64 tokens take part.  A cube listed twice counts
 * twice; the order of a list does not matter.  Every query row (padded ones
 * included) is computed.  A row whose selected cubes hold no valid token
 * gets out = 0 and lse = -inf.  K/V slots at or beyond vbs[c] are never
 * read into the result, even if they hold NaN or Inf.
 *
 * Numerics (default mode): logits and the P.V product accumulate in fp32;
 * each softmax weight enters the P.V product rounded to bf16 and the row
 * sum adds the same rounded weights, so out is a softmax-weighted mean of
 * the selected v rows with each weight off by at most 2^-8 of itself (bf16
 * keeps 8 significant bits), then rounded to bf16; lse is the log of that
 * same row sum (within -ln(1 - 2^-8) < 4e-3 of exact, plus the fp32 logit
 * error).  VSA_FWD_PRECISE_P tightens both.
 *
 * Real (non-pad) V rows must be finite: two query cubes share a tile, and a
 * KV cube that only one of them selects enters the other's P.V product with
 * weight exactly 0, so an Inf or NaN in one of its real V rows turns into
 * NaN in that column of the other cube's rows (0 * Inf).  A non-finite
 * value in a real K row reaches only the rows whose query cube selected its
 * cube (the other rows' logits there are replaced by -inf); values in pad
 * slots never reach a product.
 *
 *   q, k, v  [B, S, H, D] bf16      in
 *   topk_idx [B, H, Nq, topk] int32 in
 *   vbs      [Nq] int32             in
 *   out      [B, S, H, D] bf16      out (may not alias inputs)
 *   lse      [B, H, S] fp32         out, natural-log log-sum-exp of the
 *            scaled logits per query row; NULL to skip.
 *   sm_scale  logit scale (1/sqrt(D) in the contract).
 *
 * Errors: VSA_ERR_ARG if S != 64*Nq, D != 128, topk < 1, B, H or Nq < 1,
 * Nq > 8192 or topk > 1024 (the kernel's shared-memory staging of the two
 * lists of a tile), or B*H*Nq, S*H*D overflow the kernel's index range;
 * VSA_ERR_NULL for a
 * NULL required pointer; VSA_ERR_ALIGN for a pointer not 16-byte aligned;
 * VSA_ERR_ARCH off sm_100; VSA_ERR_LAUNCH if a launch fails.  Out-of-range
 * topk_idx or vbs values found by the kernel set VSA_ERR_DEVICE; the
 * affected entries are skipped.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_fwd(const vsa_bf16 *q, const vsa_bf16 *k, const vsa_bf16 *v, const int32_t *topk_idx,
            const int32_t *vbs, vsa_bf16 *out, float *lse, int B, int S, int H, int D, int Nq, int topk,
            float sm_scale, cudaStream_t stream);

/* Precision options for vsa_fwd_ex. */
enum vsa_fwd_flags {
    VSA_FWD_DEFAULT = 0,
    /* Carry the softmax weights P into the P.V product as a bf16 pair
     * (P = hi + lo, within 2^-17 of P) instead of one bf16 value (within
     * 2^-8): the output is then within a small fraction of a bf16 ulp of the
     * exact result, where the default's weight rounding can move an output
     * element by up to 2^-8 * sum_u w_u |v_u - out| before its own rounding
     * (one ulp at large outputs of spread-out softmax rows).  Costs a second
     * P.V product per step (about +27 % time at Wan 832x480). */
    VSA_FWD_PRECISE_P = 1
};

/* vsa_fwd with option flags (vsa_fwd == vsa_fwd_ex with VSA_FWD_DEFAULT). */
VSA_API int vsa_fwd_ex(const vsa_bf16 *q, const vsa_bf16 *k, const vsa_bf16 *v, const int32_t *topk_idx,
               const int32_t *vbs, vsa_bf16 *out, float *lse, int B, int S, int H, int D, int Nq, int topk,
               float sm_scale, int flags, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_fwd_planned -- vsa_fwd_ex with an explicit tile plan.
 *
 * The default kernel computes two query cubes of one (b, h) per 128-row
 * tile and walks the union of their selections, loading a KV cube that
 * both select once for both.  vsa_fwd / vsa_fwd_ex pair cubes (2p, 2p+1);
 * a plan (from vsa_plan, or the caller's own) names the pairs instead:
 *
 *   plan [B*H][ceil(Nq/2)][2] int32, in: tile p of (b, h) computes query
 *        cubes plan[bh][p][0] and plan[bh][p][1]; the second may be -1 (a
 *        tile with one cube).  Every query cube of (b, h) must appear in
 *        exactly one tile of (b, h); a cube that appears in none is not
 *        written.  Entries out of range latch device error 4 and are
 *        skipped.  The plan changes only which cubes share a tile: results
 *        are those of vsa_fwd_ex up to the order of floating-point sums.
 *
 * Errors: as vsa_fwd_ex, plus VSA_ERR_NULL for a NULL plan.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_fwd_planned(const vsa_bf16 *q, const vsa_bf16 *k, const vsa_bf16 *v, const int32_t *topk_idx,
                            const int32_t *vbs, const int32_t *plan, vsa_bf16 *out, float *lse, int B, int S,
                            int H, int D, int Nq, int topk, float sm_scale, int flags, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_fwd_proxy -- proxy-compensated fine forward.
 *
 * TensorRT-LLM PR #7 (the embedded FlashInfer PR "support proxy-compensated
 * block-sparse attention") and TensorRT-Edge-LLM "Video Sparse Attention
 * Runner": the selected cubes are attended exactly, and every cube a query
 * cube did not select contributes through its mean key and summed value,
 * weighted by the number of tokens it stands for.  For query row s of cube i
 * (E its selected tokens, multiplicity kept; O the cubes j with vbs[j] > 0
 * that i did not select -- a selected cube has no proxy):
 *   out = (sum_{u in E} e^{x_u} v_u + sum_{j in O} e^{y_j} vc_j)
 *         / (sum_{u in E} e^{x_u} + sum_{j in O} vbs[j] e^{y_j}),
 *   x_u = sm_scale q_s . k_u,  y_j = sm_scale q_s . kc_j,
 * lse = the log of that denominator (natural).
 *
 *   kc, vc  [B, H, Nq, D] bf16 in: the cubes' mean keys and summed values
 *           (the bf16 cube means of k and cube sums of v; vsa_tile_qkv forms
 *           both), caller-owned
 *   plan    optional tile plan as for vsa_fwd_planned (NULL: consecutive
 *           pairs)
 *   other arguments, numerics and errors as vsa_fwd_planned / vsa_fwd_ex,
 *   plus VSA_ERR_NULL for a NULL kc or vc.  Each tile walks its selected
 *   cubes, then ceil(Nq / 128) steps of proxy keys.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_fwd_proxy(const vsa_bf16 *q, const vsa_bf16 *k, const vsa_bf16 *v, const int32_t *topk_idx,
                          const int32_t *vbs, const vsa_bf16 *kc, const vsa_bf16 *vc, const int32_t *plan,
                          vsa_bf16 *out, float *lse, int B, int S, int H, int D, int Nq, int topk, float sm_scale,
                          int flags, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_fwd_bsr / vsa_fwd_bitmask -- the fine forward with the selections in the
 * route formats of TensorRT-LLM PR #7 (the embedded FlashInfer PR "support
 * proxy-compensated block-sparse attention", "Bitmask format"): canonical BSR
 * rows, or packed UInt32 exact-block bitmaps per (batch, head, query cube),
 * either one with or without proxy compensation.  Both formats become the same
 * per-tile step list as topk_idx rows, so a BSR row, a bitmap row and a
 * topk_idx row that name the same cubes in ascending order give bit-identical
 * results.
 *
 * vsa_fwd_bsr: row r = (b*H + h)*Nq + i (query cube i of batch b, head h)
 * selects the cubes block_indices[block_indptr[r] .. block_indptr[r+1]), in
 * that order, any number from 0 to 1024 (a cube named twice counts twice).
 *   block_indptr   [B*H*Nq + 1] int32 in
 *   block_indices  [nnz] int32 in (may be NULL when nnz == 0)
 * A row outside [0, nnz] or with end < start is taken as empty and latches
 * device error 5; a row of more than 1024 entries keeps its first 1024 and
 * latches 5; an index outside [0, Nq) is dropped and latches 1.
 *
 * vsa_fwd_bitmask: bit c % 32 of word c / 32 of row (b, h, i) selects cube c.
 *   mask  [B, H, Nq, ceil(Nq / 32)] uint32 in
 * Bits at c >= Nq in a row's last word are ignored.  A row of more than 1024
 * cubes keeps its lowest 1024 and latches device error 5.
 *
 * Both: kc and vc both NULL (plain forward) or both set (proxy compensation as
 * in vsa_fwd_proxy, over the cubes a row does not select); plan as in
 * vsa_fwd_planned (NULL: consecutive pairs).  Other arguments, numerics and
 * errors as vsa_fwd_ex; VSA_ERR_NULL also for exactly one of kc, vc, and
 * VSA_ERR_ARG for nnz < 0.  Every pointer is a device pointer, 16-byte aligned.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_fwd_bsr(const vsa_bf16 *q, const vsa_bf16 *k, const vsa_bf16 *v, const int32_t *block_indptr,
                        const int32_t *block_indices, int nnz, const int32_t *vbs, const vsa_bf16 *kc,
                        const vsa_bf16 *vc, const int32_t *plan, vsa_bf16 *out, float *lse, int B, int S, int H,
                        int D, int Nq, float sm_scale, int flags, cudaStream_t stream);
/* ------------------------------------------------------------------------
 * vsa_cross_attn -- short-KV cross-attention (maxdiffusion PR #509: Wan's
 * cross-attention over the 512-token text KV, one exact softmax per query row
 * over every key, no mask):
 *   out[b, s, h, :] = softmax_u(sm_scale q[b, s, h, :] . k[b, u, h, :]) v[b, u, h, :]
 * over all u < S_kv.  The same tcgen05 kernel as the fine stage: query rows in
 * blocks of 64, two blocks to a 128-row tile, the keys in 64-key cubes (the
 * last holding the S_kv % 64 left, if any); the softmax is online over the
 * ceil(S_kv / 64) cubes, which is the exact softmax up to rounding.
 *   q, out  [B, S, H, D] bf16 (any row order, S a multiple of 64, S <= 64 * 8192)
 *   k, v    [B, S_kv, H, D] bf16, 1 <= S_kv <= 65536
 *   lse     [B, H, S] fp32 natural log-sum-exp, or NULL
 * flags: VSA_FWD_PRECISE_P as for vsa_fwd_ex.  Errors: VSA_ERR_ARG for sizes
 * out of range or D != 128, VSA_ERR_NULL, VSA_ERR_ALIGN (16 bytes),
 * VSA_ERR_ARCH, VSA_ERR_LAUNCH.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_cross_attn(const vsa_bf16 *q, const vsa_bf16 *k, const vsa_bf16 *v, vsa_bf16 *out, float *lse,
                           int B, int S, int S_kv, int H, int D, float sm_scale, int flags, cudaStream_t stream);
VSA_API int vsa_fwd_bitmask(const vsa_bf16 *q, const vsa_bf16 *k, const vsa_bf16 *v, const uint32_t *mask,
                            const int32_t *vbs, const vsa_bf16 *kc, const vsa_bf16 *vc, const int32_t *plan,
                            vsa_bf16 *out, float *lse, int B, int S, int H, int D, int Nq, float sm_scale, int flags,
                            cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_route -- cube-mean q.k routing that builds topk_idx.
 *
 * "align VisualGen VSA with block-sparse FMHA" (TensorRT-LLM PR #7), review
 * excerpts: the cube mean is the sum over the cube's valid tokens divided by
 * the valid count, cast back to the tiled dtype; the VSA predictor selects
 * KV cubes from these means ("Video Sparse Attention Runner", TensorRT-Edge
 * docs: block means of K are rounded to bf16 before routing).  The score of
 * query cube i against KV cube j is sum_d qc[i][d] * kc[j][d]; topk_idx
 * lists the topk largest scores, largest first, equal scores by lower index.
 * Arithmetic (fixed so that the result is exact and reproducible):
 *   mean = bf16_round_nearest_even(fp64_sequential_sum / vbs)  (0 if vbs = 0)
 *   score = fp64 sequential sum over d of the exact bf16 products
 *   a NaN score ranks as -inf.
 *
 *   q, k      [B, S, H, D] bf16 in
 *   vbs       [Nq] int32 in
 *   topk_idx  [B, H, Nq, topk] int32 out
 *   workspace device scratch of at least vsa_route_workspace_size(B, H, Nq, D)
 *             bytes (any 16-byte-aligned address), owned by the caller;
 *             contents on entry are ignored.
 *
 * Errors: as vsa_fwd, plus VSA_ERR_ARG for topk > Nq or Nq > 4096, and
 * VSA_ERR_WORKSPACE for a NULL or short workspace.
 * ---------------------------------------------------------------------- */
VSA_API size_t vsa_route_workspace_size(int B, int H, int Nq, int D);

VSA_API int vsa_route(const vsa_bf16 *q, const vsa_bf16 *k, const int32_t *vbs, int32_t *topk_idx, int B, int S, int H,
              int D, int Nq, int topk, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_route_noalloc -- vsa_route for callers that cannot allocate device
 * memory.  The pages have no counterpart of this call; it exists for this
 * library's users.
 *
 * Some callers cannot call cudaMalloc (or any allocator) at the point where
 * they route: code running inside a CUDA graph capture whose capture mode
 * forbids allocation, plugins and runtimes that are handed only their
 * input/output buffers by a host framework, and deployments that fix every
 * device allocation at start-up.  This entry point takes the same arguments
 * as vsa_route minus the workspace: its scratch (the bf16 cube means of q
 * and k, 2*B*H*Nq*D*2 bytes) lives in a 16 MiB array that is part of the
 * library's device code.  Every GPU that loads the library holds that array
 * until the process exits.
 *
 *  - Limit: 2*B*H*Nq*D*2 <= 16 MiB (B*H*Nq <= 32768 at D = 128); larger
 *    problems return VSA_ERR_WORKSPACE and launch nothing.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress while that device is current; make that first call
 *    before any stream capture on that device.
 *  - All calls share the one array and it keeps the last call's contents.
 *    Calls whose kernels may overlap on the GPU (different streams without
 *    ordering between them) race on it; serialise them on one stream.  The
 *    routing overwrites every scratch byte it reads, so nothing needs
 *    clearing between calls.
 *  - Otherwise as vsa_route: same arguments, checks, results and errors.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_route_noalloc(const vsa_bf16 *q, const vsa_bf16 *k, const int32_t *vbs, int32_t *topk_idx, int B,
                              int S, int H, int D, int Nq, int topk, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_plan -- pair the query cubes of every (b, h) for vsa_fwd_planned.
 *
 * The paired forward kernel computes two query cubes per tile and loads a
 * KV cube that both select once for both, so its work falls with the
 * overlap of the two selection lists.  This call pairs cubes whose lists
 * overlap most.  The pages define no such schedule; it changes only which
 * cubes share a tile, never the attention result.  Steps (integer work,
 * fixed tie rules, deterministic):
 *   1. overlap(i, j) = number of distinct cubes both lists name;
 *   2. each cube keeps its 8 best partners j != i (larger overlap first,
 *      then smaller j);
 *   3. rounds: every unpaired cube proposes to its first still-unpaired
 *      candidate; cubes that propose to each other are paired; repeated
 *      until a round pairs none;
 *   4. cubes left over are paired in index order (an odd one last, alone);
 *   5. tiles are listed by their smaller cube index: (smaller, larger) or
 *      (i, -1).
 *
 *   topk_idx  [B, H, Nq, topk] int32 in (values in [0, Nq); others are
 *             ignored and latch device error 1)
 *   plan      [B*H][ceil(Nq/2)][2] int32 out
 *   workspace device scratch of vsa_plan_workspace_size(B, H, Nq, topk)
 *             bytes, 16-byte aligned, owned by the caller.
 *
 * Errors: VSA_ERR_ARG unless 1 <= topk <= Nq <= 8192 and B, H >= 1;
 * VSA_ERR_NULL, VSA_ERR_ALIGN, VSA_ERR_WORKSPACE, VSA_ERR_ARCH,
 * VSA_ERR_LAUNCH as for the other calls.
 * ---------------------------------------------------------------------- */
VSA_API size_t vsa_plan_workspace_size(int B, int H, int Nq, int topk);

VSA_API int vsa_plan(const int32_t *topk_idx, int32_t *plan, int B, int H, int Nq, int topk, void *workspace,
                     size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Cube-major layout.  Dataset card "wan2.2_production_values", section
 * "Shapes": a T x Hh x W latent grid is cut into 4x4x4 cubes,
 * Nq = ceil(T/4) * ceil(Hh/4) * ceil(W/4), S = 64 * Nq.  Cubes are ordered
 * (ct, ch, cw) row-major; inside cube c its real tokens come first, in
 * local (t, h, w) row-major order over the cube's real extent, followed by
 * zero pads up to 64; vbs[c] is its real-token count.
 * ---------------------------------------------------------------------- */

/* Host-only: Nq and (if vbs_host != NULL) the [Nq] valid counts.
 * Errors: VSA_ERR_ARG for a non-positive extent or Nq beyond INT32. */
VSA_API int vsa_cube_counts(int T, int Hh, int W, int32_t *vbs_host, int *Nq_out);

/* x_grid [B, T*Hh*W, H, D] (raster order) -> x_tiled [B, 64*Nq, H, D]; pads
 * are written as zeros.  Requires H*D to be a multiple of 8.  Untiling by an
 * index gather is described in TensorRT-LLM PR #7 (review excerpts). */
VSA_API int vsa_tile(const vsa_bf16 *x_grid, vsa_bf16 *x_tiled, int B, int T, int Hh, int W, int H, int D,
             cudaStream_t stream);

/* Inverse of vsa_tile: x_tiled [B, 64*Nq, H, D] -> x_grid [B, T*Hh*W, H, D]. */
VSA_API int vsa_untile(const vsa_bf16 *x_tiled, vsa_bf16 *x_grid, int B, int T, int Hh, int W, int H, int D,
               cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_tile_qkv -- vsa_tile of q, k and v in one launch and, in the same
 * pass over q and k, the cube means that vsa_route scores.
 *
 * The routing's cube means (vsa_route above; TensorRT-LLM PR #7, review
 * excerpts) are sums over the first vbs[c] tokens of each cube.  Forming
 * them while the tokens pass through the tiling reads q and k from device
 * memory once instead of twice; vsa_route_means then finishes the routing.
 *
 *   q_grid, k_grid, v_grid    [B, T*Hh*W, H, D] bf16 in (raster order)
 *   q_tiled, k_tiled, v_tiled [B, 64*Nq, H, D] bf16 out, exactly as vsa_tile
 *   vbs     [Nq] int32 in: the counts the means divide by (normally those of
 *           vsa_cube_counts); may be NULL when qc and kc are NULL
 *   qc, kc  [B, H, Nq, D] bf16 out: the cube means of q and k with
 *           vsa_route's arithmetic (slots past a cube's real tokens count as
 *           zeros), bit-identical to the means vsa_route forms from the
 *           tiled tensors; both NULL to skip them
 *   vc      [B, H, Nq, D] bf16 out: the cube sums of v (sequential FP64 sum
 *           over the first vbs[c] tokens, rounded to bf16 once), the summed
 *           values of vsa_fwd_proxy; NULL to skip them
 *
 * Errors: as vsa_tile for each of the three tensors; VSA_ERR_ARG if exactly
 * one of qc, kc is NULL, or if means or sums are asked for and D != 128;
 * VSA_ERR_NULL for vbs NULL while means or sums are asked for;
 * VSA_ERR_ALIGN for qc, kc, vc or vbs not 16-byte aligned.  A vbs value
 * outside [0, 64] latches device error 2 and gives a zero mean and sum.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_tile_qkv(const vsa_bf16 *q_grid, const vsa_bf16 *k_grid, const vsa_bf16 *v_grid, vsa_bf16 *q_tiled,
                         vsa_bf16 *k_tiled, vsa_bf16 *v_tiled, const int32_t *vbs, vsa_bf16 *qc, vsa_bf16 *kc,
                         vsa_bf16 *vc, int B, int T, int Hh, int W, int H, int D, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * vsa_route_means -- the scoring and top-k steps of vsa_route, on cube means
 * already formed (by vsa_tile_qkv):
 *   qc, kc    [B, H, Nq, D] bf16 in
 *   topk_idx  [B, H, Nq, topk] int32 out
 * Same arithmetic and results as vsa_route given the tensors the means came
 * from; no workspace.  Errors: VSA_ERR_ARG unless B, H >= 1, D = 128 and
 * 1 <= topk <= Nq <= 4096; VSA_ERR_NULL, VSA_ERR_ALIGN, VSA_ERR_ARCH,
 * VSA_ERR_LAUNCH as for the other calls.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_route_means(const vsa_bf16 *qc, const vsa_bf16 *kc, int32_t *topk_idx, int B, int H, int D, int Nq,
                            int topk, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Diagnostic of the pipeline's failure handling.  Launches one warp that
 * runs the forward kernels' bounded mbarrier wait on a barrier nothing ever
 * completes: the wait gives up after ~2 s of GPU clock, latches code 3 in
 * the device error word (read it with vsa_device_status) and returns, and
 * the kernel exits normally.  `result` is a device int: bit 0 = the wait
 * reported success (never expected), bit 1 = the abort flag was raised.
 * Returns VSA_ERR_NULL or VSA_ERR_LAUNCH on failure to launch, else VSA_OK.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_stall_check(int *result, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Device error word.  Synchronises `stream`, returns VSA_OK or
 * VSA_ERR_DEVICE (and clears the word), or VSA_ERR_LAUNCH if the stream
 * reports a CUDA error.  `detail` (may be NULL) receives the latched code:
 * 1 = topk_idx value out of range, 2 = vbs value out of range,
 * 3 = a bounded pipeline wait ran out, 4 = a tile plan entry out of range,
 * 5 = a BSR row outside the index array or longer than 1024 entries, or a
 * bitmap row of more than 1024 cubes.
 * ---------------------------------------------------------------------- */
VSA_API int vsa_device_status(cudaStream_t stream, int *detail);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H */
