/*
 * tm.h -- C ABI of the B200 TokenMixer-Large forward library (libtm.so).
 *
 * The library runs the forward pass of the TokenMixer-Large block and stack on
 * one B200 (sm_100a).  Sources for what each call computes:
 *   [digest] "TokenMixer-Large: Scaling Up Large Ranking Models in Industrial
 *            Recommenders", paper digest of arXiv 2602.06563, sections 2.2-2.5;
 *   [readme] "tokenmixerlarge" README of the TensorFlow/Keras reproduction,
 *            block diagram and the list of paper-faithful choices.
 *
 * Conventions shared by every call:
 *   - Every tensor pointer is caller-owned DEVICE memory, 16-byte aligned (the
 *     element-wise utilities below ask only for one element's alignment), in
 *     row-major (C) order with the shape given beside it.  The library never
 *     allocates device memory and never frees caller memory; scratch space is
 *     the caller's `workspace`, sized by the *_workspace_bytes queries.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only
 *     enqueue work: nothing synchronises except tm_get_device_error.
 *   - Storage dtype is tm_shape.dtype (fp32 or bf16) for activations and FFN
 *     weights; router weights are always fp32; accumulation is always fp32;
 *     stores to bf16 round to nearest-even.
 *   - Weights are [out, in] ("K-major"): a hidden unit's gate row is contiguous
 *     over the input width.
 *   - Host-side validation runs before any launch.  On TM_ERR_INVALID_ARG,
 *     TM_ERR_UNSUPPORTED or TM_ERR_WORKSPACE nothing is launched and no output
 *     is touched.  A kernel that hits a bounded-wait timeout or a bounds check
 *     records it in a device error word (it never traps); read it with
 *     tm_get_device_error.
 *   - Size limits: T * D < 2^31 elements per sample and B * banks <= 2^28 rows
 *     per sub-layer (TM_ERR_UNSUPPORTED beyond them).
 *   - Results are deterministic: the same inputs give the same output bits.
 *   - Calls that share a workspace must not overlap on the GPU.
 */
#ifndef TM_H_
#define TM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TM_API __attribute__((visibility("default")))
#else
#define TM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TM_OK = 0,
    TM_ERR_INVALID_ARG = 1,     /* bad shape, null or misaligned pointer */
    TM_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. a width the kernels lack) */
    TM_ERR_WORKSPACE = 3,       /* workspace null or smaller than the query returned */
    TM_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed */
    TM_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait ran out (reported by tm_get_device_error) */
    TM_ERR_DEVICE_BOUNDS = 6    /* a kernel's bounds check fired (reported by tm_get_device_error) */
} tm_status;

typedef enum { TM_F32 = 0, TM_BF16 = 1 } tm_dtype;

/* How a sub-layer sees its input rows and writes its output.
 *   TM_LAYOUT_ROWS : x, residual and y are [B, banks, width] (for the reverting
 *                    sub-layer that is [B, T, D] with banks = T, width = D).
 *   TM_LAYOUT_MIXED: x, residual and y are token tensors [B, T, D]; the rows are
 *                    Mix(x) (banks = H, width = T*D/H, [digest] 2.3.1 Eq. 9-11)
 *                    and the output rows are written back through Revert
 *                    (Eq. 13-15), so Mix/Revert are never materialised.      */
typedef enum { TM_LAYOUT_ROWS = 0, TM_LAYOUT_MIXED = 1 } tm_layout;

/* Token tensor X in R[B, T, D] ([digest] 2.2, Eq. 4), H heads with D % H == 0,
 * RMSNorm epsilon (added inside the square root). */
typedef struct { int B, T, D, H; tm_dtype dtype; float eps; } tm_shape;

/* Per-token SwiGLU bank ([digest] 2.3.2, Eq. 17-18, no bias): one weight set per
 * bank.  w_gate, w_up: [banks, hidden, width]; w_down: [banks, width, hidden]. */
typedef struct {
    int banks, width, hidden;
    const void *w_gate, *w_up, *w_down;
} tm_swiglu_w;

/* Sparse-Pertoken MoE bank ([digest] 2.4, Eq. 19-21): per bank, an fp32 router
 * w_router [banks, E, width], E routed SwiGLU experts we_gate/we_up
 * [banks, E, hidden_e, width], we_down [banks, E, width, hidden_e], and one
 * always-on shared expert ws_gate/ws_up [banks, hidden_s, width], ws_down
 * [banks, width, hidden_s].  hidden_s == 0 (no shared expert, ws_* ignored) is accepted by
 * tm_route_topk only: the forward calls return TM_ERR_UNSUPPORTED for it (the method's MoE always
 * has the shared expert, and the combine runs as that expert's down projection).
 * Output = alpha * sum_{top-k e} softmax(router logits)_e * Expert_e + Shared. */
typedef struct {
    int banks, width, E, k, hidden_e, hidden_s;
    float alpha;
    const float *w_router;
    const void *we_gate, *we_up, *we_down;
    const void *ws_gate, *ws_up, *ws_down;
} tm_moe_w;

/* One sub-layer: RMSNorm gain [width] (NULL = all ones) and its FFN bank. */
typedef struct {
    const void *norm_gain;
    int is_moe;            /* 0: dense (uses .dense), 1: MoE (uses .moe) */
    tm_swiglu_w dense;
    tm_moe_w moe;
} tm_sublayer;

/* One block: the mixing sub-layer (banks = H, width = T*D/H) and the reverting
 * sub-layer (banks = T, width = D). */
typedef struct { tm_sublayer mix, rev; } tm_block;

/* Static string for a status code. */
TM_API const char *tm_status_string(tm_status s);

/* Library ABI version (major * 100 + minor). */
TM_API int tm_version(void);

/* Workspace bytes needed by tm_pertoken_swiglu / tm_sparse_pertoken_moe for this
 * sub-layer and layout (0 if the arguments are invalid). */
TM_API size_t tm_sublayer_workspace_bytes(const tm_shape *shape, tm_layout layout, const tm_sublayer *sub);

/* Workspace bytes needed by tm_route_topk. */
TM_API size_t tm_route_workspace_bytes(const tm_shape *shape, tm_layout layout, const tm_moe_w *w);

/* Workspace bytes needed by tm_block_forward (L = 1) or tm_stack_forward. */
TM_API size_t tm_workspace_bytes(const tm_shape *shape, const tm_block *blocks, int L, int inter_residual_gap);

/* Group-wise tokenizer stub ([digest] 2.2.1-2.2.2, Eq. 2-4), one bias-free linear
 * layer per group: X[b,0] = w_global . concat_g groups[b,g]  (the global token),
 * X[b,t] = w_group[t-1] . groups[b,t-1] for t = 1..T-1.
 * groups [B, T-1, dg]; w_group [T-1, D, dg]; w_global [D, (T-1)*dg]; X_out [B,T,D].
 * A boundary utility (plain CUDA-core kernel), not part of the timed path; pointers aligned to
 * one element suffice.  TM_ERR_INVALID_ARG for a null or misaligned pointer, dg < 1 or T < 2. */
TM_API tm_status tm_tokenize_stub(const void *groups, const void *w_group, const void *w_global, int dg,
                           const tm_shape *shape, void *X_out, void *stream);

/* Mix ([digest] 2.3.1, Eq. 9-11): Hm[b, h, t*dh + j] = X[b, t, h*dh + j],
 * X [B,T,D] -> Hm [B, H, T*D/H].  A test/API utility: the fused path never calls it.  Pointers
 * aligned to one element suffice; TM_ERR_INVALID_ARG for a null, equal or misaligned pointer. */
TM_API tm_status tm_mix(const void *X, void *Hm, const tm_shape *shape, void *stream);

/* Scoring head ([readme] block diagram: the tokens are mean-pooled, then projected to one logit;
 * bias off as the reproduction's default): logits[b] = (1/T) sum_t sum_d X[b,t,d] * w_head[d],
 * fp32 accumulation.  X [B,T,D] and w_head [D] in the shape's dtype; logits [B] fp32.
 * An HBM-bound reduction kernel (one warp per sample). */
TM_API tm_status tm_head_forward(const void *X, const tm_shape *shape, const void *w_head, float *logits,
                                 void *stream);

/* Workspace bytes needed by tm_model_forward. */
TM_API size_t tm_model_workspace_bytes(const tm_shape *shape, const tm_block *blocks, int L, int inter_residual_gap);

/* End-to-end scoring of a batch: tm_tokenize_stub -> tm_stack_forward -> tm_head_forward
 * (groups [B,T-1,dg], w_group, w_global as tm_tokenize_stub; blocks, L, gap as
 * tm_stack_forward; w_head [D]); logits [B] fp32.  The token tensors live in the workspace. */
TM_API tm_status tm_model_forward(const void *groups, const void *w_group, const void *w_global, int dg,
                                  const tm_block *blocks, int L, int inter_residual_gap, const void *w_head,
                                  const tm_shape *shape, float *logits, void *workspace, size_t workspace_bytes,
                                  void *stream);

/* Token Parallel ([digest] 2.5.3) exchange layouts.  Over P ranks, rank p holds the tokens
 * p*Tp .. (p+1)*Tp-1 (Tp = T/P) for the reverting sub-layer and the head columns p*Dp .. (p+1)*Dp-1
 * (Dp = D/P, whole heads) for the mixing sub-layer; an all-to-all buffer E [P][B][Tp][Dp] holds in
 * chunk q the part for (sending) or from (receiving) rank q.  local_layout TM_TP_TOKEN_SHARD: the
 * local tensor is the rank's token shard [B][Tp][D] = [B][Tp][P][Dp] (chunk q = the columns of rank
 * q's heads); TM_TP_HEAD_SHARD: the rank's head-column shard of every token [B][T][Dp] = [B][P][Tp][Dp]
 * (chunk q = rank q's tokens).  to_exchange != 0 copies local (src) -> E (dst), else E (src) ->
 * local (dst).  A pure permutation (bit-exact); src and dst device memory, not overlapping, aligned
 * to the element size, and to 16 bytes when Dp * element size is a multiple of 16.  TM_ERR_INVALID_ARG
 * (nothing launched) for a null, equal or misaligned pointer, a size below 1, a dtype other than f32
 * or bf16, or an unknown layout. */
#define TM_TP_TOKEN_SHARD 0
#define TM_TP_HEAD_SHARD 1
TM_API tm_status tm_tp_exchange_layout(const void *src, void *dst, int P, int B, int Tp, int Dp, tm_dtype dtype,
                                       int local_layout, int to_exchange, void *stream);

/* Revert ([digest] 2.3.1, Eq. 13-15), the inverse of Mix: Hm [B,H,T*D/H] -> X [B,T,D].  Same
 * pointer rules as tm_mix. */
TM_API tm_status tm_revert(const void *Hm, void *X, const tm_shape *shape, void *stream);

/* Router of a Sparse-Pertoken MoE sub-layer ([digest] 2.4.1 Eq. 19, 2.4.3 Eq. 21)
 * plus the expert-first bucketing that [digest] 2.5.1 calls MoEPermute.
 * For every row r = (b, bank): n = RMSNorm(row) * gain; logits = w_router[bank] . n
 * in fp32; p = softmax over all E; the k largest p (ties: lower expert index) in
 * descending order.  Outputs:
 *   topk_idx   [B, banks, k] int32  chosen experts
 *   topk_gate  [B, banks, k] fp32   alpha * p of each chosen expert (no renormalisation)
 *   logit_gap_opt [B, banks] fp32   z_(k) - z_(k+1): the k-th largest logit minus the largest
 *                                   logit left out (+inf when k == E), so a caller can tell the
 *                                   rows whose choice is a near tie (may be NULL)
 *   inv_rms    [B, banks]    fp32   1/sqrt(mean(row^2) + eps)   (may be NULL)
 *   bucket_offsets [banks*E + 1] int32  start of group g = bank*E + e in bucket_rows
 *   bucket_rows    [B*banks*k]   int32  sample index b of every routed row, grouped by
 *                                       (bank, expert), ascending b inside a group
 *   slot_of        [B, banks, k] int32  position in bucket_rows of (b, bank, j)
 * x and layout as in tm_layout. */
TM_API tm_status tm_route_topk(const void *x, tm_layout layout, const tm_shape *shape, const void *norm_gain,
                        const tm_moe_w *w, int32_t *topk_idx, float *topk_gate, float *logit_gap_opt,
                        float *inv_rms, int32_t *bucket_offsets, int32_t *bucket_rows, int32_t *slot_of,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Fixed size of the routing scratch array that tm_route_topk_noalloc keeps in the library. */
#define TM_NOALLOC_SCRATCH_BYTES (8u << 20)

/* tm_route_topk without a workspace argument, for callers that cannot allocate device memory
 * (a host framework that passes this library only its inputs and outputs and owns no allocator
 * it may call, or a serving loop that reserves all memory at start-up and allows no allocation
 * later).  The pages have no counterpart: this is a library convenience, not part of the method.
 * Same arguments, outputs and results as tm_route_topk: it calls tm_route_topk with a fixed
 * TM_NOALLOC_SCRATCH_BYTES array inside the library's device image as the workspace, held by
 * every GPU that loads the library until the process exits; problems whose
 * tm_route_workspace_bytes exceeds it return TM_ERR_WORKSPACE (message in tm_last_cuda_error)
 * before any launch.  No device memory is allocated or freed.
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress), so
 * make that first call before any stream capture; the lookup is repeated when the device's
 * context has changed (after a device reset).  All calls on a device share the array and it
 * keeps the last call's contents (none of it needs to start at zero): calls that can overlap on
 * the GPU (different streams without ordering) race on it and must not be issued. */
TM_API tm_status tm_route_topk_noalloc(const void *x, tm_layout layout, const tm_shape *shape,
                                       const void *norm_gain, const tm_moe_w *w, int32_t *topk_idx,
                                       float *topk_gate, float *logit_gap_opt, float *inv_rms,
                                       int32_t *bucket_offsets, int32_t *bucket_rows, int32_t *slot_of,
                                       void *stream);

/* Sizes the sub-layer, block and stack calls take (others return TM_ERR_UNSUPPORTED before any
 * launch): row width and hidden widths multiples of 64 (bf16) or 32 (f32); on mixed rows a head
 * width D/H that is a multiple of 8 (bf16) or 4 (f32), and of 16 for a bf16 MoE sub-layer; MoE:
 * E <= 32, k <= 8, banks * E <= 4096, a shared expert (hidden_s > 0), and the router's shared
 * memory within 220 KB: ep * (width + 4) * 4 + 16 * max(32 / ep, 4) * width * (element bytes), ep =
 * E rounded up to a power of two of at least 4 (width 768 with E = 16 takes 144 KB). */

/* Dense per-token SwiGLU sub-layer with pre-RMSNorm and residual
 * ([readme] block diagram; [digest] 2.3.2-2.3.3):
 *   y_row = SwiGLU_bank(RMSNorm(x_row) * gain) + residual_row
 * residual may be NULL (no residual) and has the layout of y.  y must not alias x. */
TM_API tm_status tm_pertoken_swiglu(const void *x, const void *residual, tm_layout layout, const tm_shape *shape,
                             const void *norm_gain, const tm_swiglu_w *w, void *y,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Sparse-Pertoken MoE sub-layer ([digest] 2.4, Eq. 19-21) with pre-RMSNorm and residual:
 *   y_row = alpha * sum_{top-k e} p_e * Expert_{bank,e}(n) + Shared_bank(n) + residual_row.
 * Routing as in tm_route_topk; the combine is a fixed-order fp32 sum (deterministic). */
TM_API tm_status tm_sparse_pertoken_moe(const void *x, const void *residual, tm_layout layout, const tm_shape *shape,
                                 const void *norm_gain, const tm_moe_w *w, void *y,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* One sub-layer of either kind (sub->is_moe: Sparse-Pertoken MoE, else per-token SwiGLU) with two
 * residual terms: y_row = FFN_bank(RMSNorm(x_row) * gain) + residual_row + extra_row, both terms
 * added in the output epilogue before y's single rounding (residual / extra NULL: none).  extra is
 * the inter-residual of [digest] 2.3.4 when a stack runs sub-layer by sub-layer, e.g. with its
 * banks sharded over GPUs (Token Parallel, [digest] 2.5.3).  x, residual, extra and y share `layout`;
 * y must not alias x or extra.  Workspace: tm_sublayer_workspace_bytes. */
TM_API tm_status tm_sublayer_forward(const void *x, const void *residual, const void *extra, tm_layout layout,
                                     const tm_shape *shape, const tm_sublayer *sub, void *y, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* One TokenMixer-Large block ([readme] block diagram; [digest] Eq. 9-16, pre-norm reading):
 *   H = Mix(X); H_next = FFN_mix(Norm(H)) + H; X_rev = Revert(H_next);
 *   Y = FFN_rev(Norm(X_rev)) + X.
 * X, Y [B,T,D]; X_revert_opt [B,T,D] receives X_rev when not NULL. */
TM_API tm_status tm_block_forward(const void *X, const tm_block *block, const tm_shape *shape, void *Y,
                           void *X_revert_opt, void *workspace, size_t workspace_bytes, void *stream);

/* One step of tm_stack_forward: Y = Block(X) + X_skip, where X_skip (NULL: none) is the skip term
 * of the inter-residual ([digest] 2.3.4), added in the block's last epilogue before Y's single
 * rounding to the storage dtype.  With X_skip NULL this is tm_block_forward.  tm_stack_forward is
 * this call repeated (X_skip = X_{l-gap} where its rule applies), so a caller that runs a stack
 * block by block -- to keep every X_l, or to interleave its own work -- gets the same bits.
 * X, X_skip, Y, X_revert_opt [B,T,D]; X_skip must not alias Y or X_revert_opt.  Workspace: as
 * tm_block_forward (tm_workspace_bytes with L = 1). */
TM_API tm_status tm_stack_step(const void *X, const void *X_skip, const tm_block *block, const tm_shape *shape,
                               void *Y, void *X_revert_opt, void *workspace, size_t workspace_bytes, void *stream);

/* L blocks with the inter-residual of [digest] 2.3.4 ([readme]: every second layer, none
 * after the final one): X_l = Block_l(X_{l-1}); X_l += X_{l-gap} when gap > 0,
 * l % gap == 0 and l < L (layers counted from 1).  Y = X_L.  Y must not alias X. */
TM_API tm_status tm_stack_forward(const void *X, const tm_block *blocks, int L, int inter_residual_gap,
                           const tm_shape *shape, void *Y, void *workspace, size_t workspace_bytes,
                           void *stream);

/* ---- FP8 E4M3 serving path of the dense per-token FFN ----------------------------------
 * [digest] 2.5.2 (FP8 quantization): serving runs on FP8 E4M3 post-training quantization of a
 * model trained in bf16.  The page names the format only; this library's reading: GEMM1 (the
 * gate and up projections, two thirds of the FFN's flops) runs on E4M3 operands on the tensor
 * cores (kind::f8f6f4) with each bank's gate/up matrix quantized with one scale and every
 * activation row quantized on its own; the SwiGLU, GEMM2 (down, bf16 weights) and the residual
 * stay as in the bf16 path (fp32 accumulation, bf16 storage).  E4M3: 1 sign bit, 4 exponent
 * bits of bias 7, 3 mantissa bits, largest finite 448; conversions round to nearest-even and
 * saturate.  bf16 activations only; row widths 128 and 256 (the fused sub-layer kernel);
 * hidden widths multiples of 128; mixed rows need a head width that is a multiple of 16.
 * Unsupported shapes return TM_ERR_UNSUPPORTED before any launch. */

/* E4M3 quantization of `groups` bf16 weight matrices w [groups, rows, cols] with one scale per
 * matrix (a bank's gate or up projection), optionally times a per-column gain [cols]
 * (multiplied and rounded to bf16 first, as the bf16 path folds the RMSNorm gain):
 * scale[g] = 2^e with e the smallest integer such that max|matrix g| * 2^-e <= 448 (1 for an
 * all-zero matrix); q [groups, rows, cols] = E4M3(w * 2^-e) (exact scaling).  rows * cols even.
 * q (1-byte codes) and scale are device memory.  E4M3 keeps a 3-bit mantissa for every value
 * inside its normal range (2^-6 .. 448 times the scale), so one scale serves all rows of a
 * projection. */
TM_API tm_status tm_quantize_fp8_weights(const void *w, const void *gain, int groups, size_t rows, int cols,
                                         uint8_t *q, float *scale, void *stream);

/* Per-row E4M3 quantization of a sub-layer's bf16 activation rows (banks, width as for the
 * sub-layer, read through `layout`): q [B*banks, width] (row b*banks + bank) = E4M3(row * 2^-e)
 * with 2^e the row's power-of-two scale (as for the weights), and rowscale [B*banks] =
 * 2^e / rms(row), rms = sqrt(mean(row^2) + eps) over the unquantized row.  bf16 rows of width
 * <= 1024 (mixed rows: head width a multiple of 8); others return TM_ERR_UNSUPPORTED. */
TM_API tm_status tm_quantize_fp8_act(const void *x, tm_layout layout, const tm_shape *shape, int banks, int width,
                                     uint8_t *q, float *rowscale, void *stream);

/* A dense bank on the FP8 path: q_gate, q_up [banks, hidden, width] E4M3 codes with s_gate,
 * s_up [banks] fp32 scales (one per bank matrix, the RMSNorm gain already folded in, as
 * tm_quantize_fp8_weights makes them); w_down bf16 [banks, width, hidden]. */
typedef struct {
    int banks, width, hidden;
    const uint8_t *q_gate, *q_up;
    const float *s_gate, *s_up;
    const void *w_down;
} tm_swiglu_w8;

/* A dense block on the FP8 path: mixing (banks = H, width = T*D/H) and reverting (banks = T,
 * width = D) sub-layers. */
typedef struct { tm_swiglu_w8 mix, rev; } tm_block_fp8;

TM_API size_t tm_pertoken_swiglu_fp8_workspace_bytes(const tm_shape *shape, tm_layout layout, const tm_swiglu_w8 *w);

/* Dense sub-layer on the FP8 path:  y_row = SwiGLU_bank(RMSNorm(x_row)) + residual_row, GEMM1 on
 * E4M3 operands: gate_n = (q_row . q_gate_n) * rowscale * s_gate, up likewise, q_row and rowscale
 * as tm_quantize_fp8_act defines them (the kernel quantizes each row tile itself from the bf16
 * rows it holds; the workspace, 256 bytes, is unused).  residual may be NULL; y must not alias x. */
TM_API tm_status tm_pertoken_swiglu_fp8(const void *x, const void *residual, tm_layout layout, const tm_shape *shape,
                                        const tm_swiglu_w8 *w, void *y, void *workspace, size_t workspace_bytes,
                                        void *stream);

TM_API size_t tm_block_fp8_workspace_bytes(const tm_shape *shape, const tm_block_fp8 *block);

/* One dense block as tm_block_forward, both sub-layers on the FP8 path (in one launch when both
 * have the same row width, T == H, as the bf16 block).  X, Y [B,T,D]; X_revert_opt [B,T,D]
 * receives X_rev when not NULL. */
TM_API tm_status tm_block_forward_fp8(const void *X, const tm_block_fp8 *block, const tm_shape *shape, void *Y,
                                      void *X_revert_opt, void *workspace, size_t workspace_bytes, void *stream);

/* A Sparse-Pertoken MoE bank on the FP8 path ([digest] 2.4, Eq. 19-21, with 2.5.2's E4M3
 * serving quantization): the fp32 router w_router [banks, E, width] and the bf16 down projections
 * we_down [banks, E, width, hidden_e], ws_down [banks, width, hidden_s] are those of tm_moe_w; the
 * gate / up projections are E4M3 codes, the routed experts' qe_gate, qe_up [banks, E, hidden_e,
 * width] with one fp32 scale per (bank, expert) matrix se_gate, se_up [banks * E], the shared
 * expert's qs_gate, qs_up [banks, hidden_s, width] with ss_gate, ss_up [banks]
 * (tm_quantize_fp8_weights makes them, the RMSNorm gain folded in; groups = banks * E, rows =
 * hidden_e for the routed experts, groups = banks, rows = hidden_s for the shared one). */
typedef struct {
    int banks, width, E, k, hidden_e, hidden_s;
    float alpha;
    const float *w_router;
    const uint8_t *qe_gate, *qe_up;
    const float *se_gate, *se_up;
    const void *we_down;
    const uint8_t *qs_gate, *qs_up;
    const float *ss_gate, *ss_up;
    const void *ws_down;
} tm_moe_w8;

/* One sub-layer on the FP8 path: a dense bank (is_moe 0, .dense) or a Sparse-Pertoken MoE bank
 * (is_moe 1, .moe).  norm_gain [width] (NULL = ones) is the RMSNorm gain that the MoE router
 * applies to the normalized row before its logits; the E4M3 weights carry it already (for a
 * dense bank it must be NULL). */
typedef struct {
    const void *norm_gain;
    int is_moe;
    tm_swiglu_w8 dense;
    tm_moe_w8 moe;
} tm_sublayer8;

/* Workspace bytes of tm_sublayer_forward_fp8 / tm_sparse_pertoken_moe_fp8 (0: arguments invalid or
 * unsupported). */
TM_API size_t tm_sublayer_fp8_workspace_bytes(const tm_shape *shape, tm_layout layout, const tm_sublayer8 *sub);

/* One sub-layer on the FP8 path with two residual terms, as tm_sublayer_forward:
 *   y_row = FFN_bank(row) + residual_row + extra_row   (residual / extra NULL: none).
 * MoE bank: the routing is the bf16 path's (fp32 logits of the normalized row, softmax, top-k,
 * gates alpha * p; tm_route_topk); each row x is quantized once, q = E4M3(x * 2^-e) with 2^e the
 * smallest power of two such that max|x| * 2^-e <= 448, and every expert that the row reaches --
 * its k routed experts and the shared one -- runs GEMM1 on E4M3 operands:
 *   gate_n = (q . q_gate_n) * 2^e / rms(x) * s_gate,  up_n likewise,  rms over the unquantized row,
 * then the bf16 SwiGLU, down projection and fixed-order combine of tm_sparse_pertoken_moe.
 * Supported: bf16, row widths multiples of 128 up to 1024 (mixed rows: head width a multiple of
 * 8), expert hidden widths multiples of 128, a shared expert (hidden_s > 0), E <= 32, k <= 8; a
 * dense bank as tm_pertoken_swiglu_fp8.  Others return TM_ERR_UNSUPPORTED before any launch.
 * y must not alias x, residual or extra. */
TM_API tm_status tm_sublayer_forward_fp8(const void *x, const void *residual, const void *extra, tm_layout layout,
                                         const tm_shape *shape, const tm_sublayer8 *sub, void *y, void *workspace,
                                         size_t workspace_bytes, void *stream);

/* The MoE sub-layer on the FP8 path with one residual: tm_sublayer_forward_fp8 with is_moe 1 and
 * extra NULL. */
TM_API tm_status tm_sparse_pertoken_moe_fp8(const void *x, const void *residual, tm_layout layout, const tm_shape *shape,
                                            const void *norm_gain, const tm_moe_w8 *w, void *y, void *workspace,
                                            size_t workspace_bytes, void *stream);

/* ---- Training: backward of the dense sub-layer and block ---------------------------------
 * The pages train the model in bf16 ([digest] 2.5.2; [readme] training flags) and print no
 * backward pass, so these calls compute the exact derivative of the forward above by the chain
 * rule, for the FFN term of a dense sub-layer (n = x / rms(x), g = n Wg^T, u = n Wu^T,
 * h = silu(g) * u, y = h Wd^T; [digest] Eq. 17-18 and 2.3.3):
 *   dWd = dy^T h;  dh = dy Wd;  dg = dh * u * s * (1 + g * (1 - s)), s = sigmoid(g);  du = dh * silu(g)
 *   dWg = dg^T n;  dWu = du^T n;  dn = dg Wg + du Wu;  dx = (dn - n * mean(dn * n)) / rms(x)
 * bf16 tensors, fp32 accumulation on the tensor cores; intermediates are stored in bf16.
 * Supported: bf16, RMSNorm gain 1 (norm_gain NULL; a gain returns TM_ERR_UNSUPPORTED), row and
 * hidden widths multiples of 128.  MoE sub-layers have no backward here (TM_ERR_UNSUPPORTED).
 * Weight gradients are written (not accumulated) in the weights' own layouts, bf16. */
typedef struct {
    void *dw_gate, *dw_up;   /* [banks, hidden, width] */
    void *dw_down;           /* [banks, width, hidden] */
} tm_swiglu_grads;

/* Weight gradients of the two sub-layers of a dense block. */
typedef struct { tm_swiglu_grads mix, rev; } tm_block_grads;

/* Workspace of tm_pertoken_swiglu_backward (0: unsupported shape or weights). */
TM_API size_t tm_pertoken_swiglu_backward_workspace_bytes(const tm_shape *shape, tm_layout layout,
                                                          const tm_swiglu_w *w);

/* Backward of the FFN term of a dense sub-layer: with y_row = SwiGLU_bank(RMSNorm(x_row)) and an
 * upstream gradient dy (the layout of x), writes dx = (dy/dx)^T dy + dx_add (dx_add NULL: none;
 * pass dy itself when the sub-layer adds its own input as the residual) and the bank weight
 * gradients into `grads`.  x, dy, dx, dx_add share `layout` (rows or the Mix view of [B,T,D]);
 * dx must not alias x or dy.  The GEMM-ready copies of the rows and the transposed operands
 * live in the workspace (about (5 W + 9 F) * 2 bytes per row and bank). */
TM_API tm_status tm_pertoken_swiglu_backward(const void *x, const void *dy, const void *dx_add, tm_layout layout,
                                             const tm_shape *shape, const void *norm_gain, const tm_swiglu_w *w,
                                             void *dx, const tm_swiglu_grads *grads, void *workspace,
                                             size_t workspace_bytes, void *stream);

/* Workspace of tm_block_backward (0: unsupported block). */
TM_API size_t tm_block_backward_workspace_bytes(const tm_shape *shape, const tm_block *block);

/* Backward of one dense block (tm_block_forward) for the gradient dY of its output:
 *   X_rev is recomputed by the mixing sub-layer's forward;
 *   dX_rev = (d FFN_rev(Norm(X_rev)) / d X_rev)^T dY;
 *   dH_next = Mix(dX_rev);  dH = (d FFN_mix(Norm(H)) / dH)^T dH_next + dH_next;
 *   dX = dY + Revert(dH)   (Mix and Revert are permutations, each the other's adjoint).
 * X, dY, dX [B,T,D] bf16; dX must not alias X or dY; grads receives both sub-layers' weight
 * gradients. */
TM_API tm_status tm_block_backward(const void *X, const void *dY, const tm_block *block, const tm_shape *shape,
                                   void *dX, const tm_block_grads *grads, void *workspace, size_t workspace_bytes,
                                   void *stream);

/* Workspace of tm_stack_backward (0: unsupported blocks). */
TM_API size_t tm_stack_backward_workspace_bytes(const tm_shape *shape, const tm_block *blocks, int L,
                                                int inter_residual_gap);

/* Backward of L dense blocks with the inter-residual of tm_stack_forward ([digest] 2.3.4), for the
 * gradient dY of the stack's output: every block input X_1 .. X_{L-1} is recomputed by the forward
 * (kept in the workspace), then, last block first, the gradient of X_{l-1} is block l's input
 * gradient (tm_block_backward) plus, when X_{l-1+gap} = Block(...) + X_{l-1}, the gradient of
 * X_{l-1+gap}.  grads[l] receives block l's weight gradients.  X, dY, dX [B,T,D] bf16; dX must not
 * alias X or dY. */
TM_API tm_status tm_stack_backward(const void *X, const void *dY, const tm_block *blocks, int L, int inter_residual_gap,
                                   const tm_shape *shape, void *dX, const tm_block_grads *grads, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* Per-kernel timing of the library's own launches (tracing). */
typedef struct {
    char name[48];       /* kernel family, e.g. "gemm_swiglu" */
    int launches;        /* launches recorded between start and stop */
    double total_ms;     /* sum of their CUDA-event durations on the launching stream */
} tm_kernel_time;

/* Start recording a CUDA event pair around every kernel the library launches from now on. */
TM_API tm_status tm_profile_start(void);

/* Stop recording, synchronise the device, and fold the recorded launches into at most
 * max_entries per-kernel totals in `out` (count written to *n_entries). */
TM_API tm_status tm_profile_stop(tm_kernel_time *out, int max_entries, int *n_entries);

/* Text of the most recent CUDA error the library saw, with the step that failed ("" if none).
 * Setting TM_DEBUG_SYNC=1 in the environment makes every launch synchronise so that a
 * failing kernel is named here (debugging only: it serialises the host and the GPU). */
TM_API const char *tm_last_cuda_error(void);

/* Number of kernels this library has launched in this process (always counted). */
TM_API unsigned long long tm_launch_count(void);

/* Synchronises `stream`, returns the first device-side error recorded since the
 * last call (TM_OK if none) and clears it. */
TM_API tm_status tm_get_device_error(void *stream);

/* Where the error that tm_get_device_error last returned was recorded (a site code of the
 * kernel's wait or bounds check, also named in tm_last_cuda_error); 0 after TM_OK. */
TM_API unsigned tm_last_device_error_site(void);

/* Failure detection.  Every device wait of the library's kernels (a pipeline barrier, a tensor-memory
 * handshake, the fused block's row-block counter) gives up after a wall-clock limit, records
 * TM_ERR_DEVICE_TIMEOUT with its site and lets the kernel return; bounds checks on indices read from
 * device data record TM_ERR_DEVICE_BOUNDS and skip the access.  No kernel traps.
 *
 * Sets that limit for the current device, in nanoseconds (1e3 .. 6e10; the default is 2 s, far
 * above any legitimate wait).  Kernels already enqueued may run with either value.  The pages have
 * no counterpart: this is a library facility, not part of the method. */
TM_API tm_status tm_set_wait_limit_ns(uint64_t ns);

/* Self-test of the bounded waits (one CTA, one thread): a wait on a barrier that nothing ever
 * completes runs out after the limit above and records TM_ERR_DEVICE_TIMEOUT at site 0x7001; a
 * second wait, made with the CTA's abort flag already raised, returns at once and records nothing.
 * result_opt (device memory, 4 x uint64, may be NULL): the first wait's duration in ns, 1 (it
 * failed), the second's duration in ns, 1 (it failed).  Read the outcome with tm_get_device_error. */
TM_API tm_status tm_selftest_wait(uint64_t *result_opt, void *stream);

/* The MoEPermute scatter of tm_route_topk run on caller-supplied tables, for tests of its bounds
 * checks: topk_idx [B, banks, k]; chunk_prefix [banks][ceil(B/128)][E], the number of rows of each
 * bank routed to each expert in the earlier 128-sample chunks; bucket_offsets [banks*E + 1];
 * bucket_rows has `capacity` entries; slot_of [B, banks, k].  A position at or past `capacity`
 * (a table that under-counts the choices) records TM_ERR_DEVICE_BOUNDS (site 0x501) and is not
 * written; nothing outside the given arrays is read or written.  E <= 64, k <= 8. */
TM_API tm_status tm_selftest_bucket_scatter(const int32_t *topk_idx, const int32_t *chunk_prefix,
                                            const int32_t *bucket_offsets, int B, int banks, int E, int k,
                                            int32_t *bucket_rows, int capacity, int32_t *slot_of, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* TM_H_ */
