/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts FFN
 * forward pass.
 *
 * The layer (one GPU, forward only):
 *
 *   z      = x W_r^T (+ bias)                      router logits, fp32
 *   p      = softmax(z); (idx, w) = top-k of z     lowest expert index wins ties
 *   w     /= sum(w)                                if renorm
 *   group (token, slot) pairs by expert, token order inside a group,
 *         dropping ranks >= C when a capacity C is set
 *   h      = act(x W1_e^T) * (x W3_e^T)            act = SiLU (SwiGLU) or erf-GELU (GeGLU)
 *   y      = h W2_e^T
 *   out_t  = sum_j w[t,j] y_{idx[t,j]}(x_t) + y_shared(x_t)
 *
 * Sources: "Sharding d'experts" (Kvasir wiki), section "Backbone x worker":
 * the router runs softmax and top-k over ``cur @ router``, the worker does the
 * three expert matmuls, the backbone adds ``combine(p, partials) +
 * shared(cur)``.  moe_stream.py (MoE-Stream), ``MoEFFN.forward``: bias-free
 * Linear gate, additive per-expert logit bias, softmax, topk, renormalised
 * gates, ``out[mask] += w * expert_out``, batch-local load-balance statistic.
 * ExpertMesh README: grouping that keeps token and top-k slot identity,
 * weighted top-k reduction, group-scaled signed INT4 experts in an [expert,
 * output, packed_input] layout behind a stable C ABI.  MoEEvolve README:
 * granular SwiGLU experts, one always-active shared expert, capacity-factor
 * static-shape dispatch.  kieve-moe: top-k GeGLU experts, load-balancing
 * auxiliary statistic.
 *
 * Conventions (every entry point):
 *  - Pointers named as device pointers must be device memory of the current
 *    device, 16-byte aligned.  All are borrowed: the caller owns them, the
 *    library keeps no reference after the call returns.
 *  - The library allocates no device memory.  Scratch comes from the caller's
 *    `workspace` (size from moe_workspace_size()).
 *  - Work is enqueued asynchronously on `stream`; no entry point synchronises
 *    the host except moe_get_status().
 *  - Errors found on the host (bad pointers, shapes, sizes) are returned
 *    before anything is enqueued.  A device-side bounded wait that gives up
 *    records MOE_DEVICE_TIMEOUT in a per-device status word read by
 *    moe_get_status(); kernels never trap.
 *  - Inputs must be finite; routing of NaN logits is undefined.
 *  - Layouts are row-major.  bf16 tensors are passed as void*.
 *  - Reentrant: every choice a call makes comes from its arguments.  The
 *    library's only mutable state is (a) the per-device status word above,
 *    (b) the wait limit of moe_set_wait_limit_ns, (c) the launch counter of
 *    moe_launch_count, (d) idempotent per-device caches filled on first use
 *    (SM count, kernel attributes, the tensor-map encoder entry point) and
 *    (e) the fixed scratch array of moe_permute_noalloc.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

enum moe_status {
  MOE_OK = 0,
  MOE_INVALID_ARGUMENT = 1,    /* NULL where a buffer is required, misaligned pointer, k > E ... */
  MOE_UNSUPPORTED_SHAPE = 2,   /* shape outside the limits below */
  MOE_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < moe_workspace_size() */
  MOE_CUDA_ERROR = 4,          /* a CUDA runtime / driver call failed */
  MOE_DEVICE_TIMEOUT = 5       /* a device-side bounded wait gave up (read via moe_get_status) */
};

enum moe_act { MOE_ACT_SWIGLU = 0, MOE_ACT_GEGLU = 1 };
enum moe_wfmt { MOE_WFMT_BF16 = 0, MOE_WFMT_INT4_G128 = 1 };

/*
 * Layer shape.
 *   T        tokens (1 .. 2^24)
 *   d        model width (multiple of 16; multiple of 128 for INT4)
 *   E        routed experts (1 .. 512)
 *   k        experts per token (1 .. min(E, 16))
 *   H        routed expert hidden width (multiple of 16; of 128 for INT4)
 *   H_s      shared expert hidden width, 0 = no shared expert (same rules as H)
 *   capacity rows per expert group C, 0 = unbounded (see moe_capacity)
 *   act      enum moe_act
 *   wfmt     enum moe_wfmt
 *   renorm   1: divide the k gates by their sum; 0: gates are the softmax probabilities
 *   flags    implementation choices, 0 = automatic; MOE_FLAG_SINGLE_CTA_GEMM runs
 *            the bf16 expert GEMMs on single-CTA 128-row tiles even where the
 *            automatic choice would pair CTAs (256-row tiles, tcgen05
 *            cta_group::2).  Both compute the same products in the same fp32
 *            order per output.  Unknown bits give MOE_INVALID_ARGUMENT.  (No
 *            counterpart on the pages.)
 */
enum moe_flags { MOE_FLAG_SINGLE_CTA_GEMM = 1 };

typedef struct moe_shape {
  int64_t T;
  int32_t d, E, k, H, H_s, capacity, act, wfmt, renorm, flags;
} moe_shape;

/*
 * Expert weight layouts ([expert, out, in], the ExpertMesh "[expert, output,
 * packed_input]" order):
 *   MOE_WFMT_BF16:      w13 [E, 2H, d] bf16, rows [0,H) = W1 (gate), rows [H,2H) = W3 (up);
 *                       w2  [E, d, H]  bf16.
 *   MOE_WFMT_INT4_G128: w13 [E, 2H, d/2] uint8, w2 [E, d, H/2] uint8: two's-complement
 *                       nibbles, input index 2i in the low nibble of byte i;
 *                       s13 [E, 2H, d/128] bf16, s2 [E, d, H/128] bf16: one scale per
 *                       128 consecutive inputs of an output row; weight = q * s.
 * The shared expert uses the same layouts with E = 1 and H = H_s.
 */

/* Number of grouped rows R: E * capacity with a capacity, else T * k. */
int64_t moe_grouped_rows(const moe_shape* s);

/*
 * C = ceil(factor * T * k / E), the per-expert capacity of the MoEEvolve
 * README's capacity-factor dispatch; factor <= 0 gives 0 (unbounded).
 * The factor is read as a decimal with at most 6 fractional digits.
 */
int moe_capacity(int64_t T, int32_t k, int32_t E, double factor, int32_t* capacity);

/* Scratch bytes moe_forward needs for this shape (an upper bound for every entry point). */
int moe_workspace_size(const moe_shape* s, size_t* bytes);

/*
 * Router (Kvasir "Backbone x worker" router line; moe_stream.py MoEFFN.forward).
 *   x        [T, d] bf16                 in
 *   w_router [E, d] fp32                 in   (a bias-free Linear(d, E))
 *   bias     [E] fp32 or NULL            in   added to the logits before softmax/top-k
 *   logits   [T, E] fp32 or NULL         out  x W_r^T + bias, the values softmax and top-k see
 *   topk_idx [T, k] int32                out  experts by decreasing logit, lowest index on ties
 *   topk_w   [T, k] fp32                 out  softmax probability of each pick (renormalised if renorm)
 *   counts   [E] int32                   out  tokens choosing each expert
 *   aux_f, aux_p [E] fp32 or NULL        out  counts/T and mean softmax probability
 *   aux      [1] fp32 or NULL            out  E * sum_e f_e P_e
 * Logit precision: fp32 FMA dot products over the inputs in order.  For large
 * T * E * d the logits are first screened on the tensor cores (two-term bf16
 * split of W_r, fp32 accumulation) and every expert that can reach the top k
 * under the screen's error bound, (2^-16 + (2d+2) 2^-23 + (d+2) 2^-24)(1 + 2^-7)
 * ||x_t|| max_e ||w_e||, is recomputed as an fp32 FMA dot product; the picks
 * and their gates then come from those values, and the other entries of
 * `logits` are the screened values (within that bound).
 * Deterministic: identical inputs give bit-identical outputs.
 */
int moe_route(const moe_shape* s, const void* x, const float* w_router, const float* bias, float* logits,
              int32_t* topk_idx, float* topk_w, int32_t* counts, float* aux_f, float* aux_p, float* aux,
              void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * The softmax / top-k / gates / statistics half of moe_route on caller
 * logits [T, E] fp32 (any bias already added).  Same outputs and rules.
 */
int moe_route_from_logits(const moe_shape* s, const float* logits, int32_t* topk_idx, float* topk_w,
                          int32_t* counts, float* aux_f, float* aux_p, float* aux, void* workspace,
                          size_t ws_bytes, moe_stream_t stream);

/*
 * Grouping by expert with (token, slot) identity kept (ExpertMesh README,
 * "Activation grouping that preserves token and top-k slot identity"; the
 * MoEEvolve capacity-factor dispatch).
 *   x         [T, d] bf16        in
 *   topk_idx  [T, k] int32       in   k distinct experts per token, each in [0, E)
 *   slot_pos  [T, k] int32       out  row of (t, j) in the grouped buffer, -1 if dropped
 *   drop_mask [T, k] uint8 / NULL out 1 where (t, j) was dropped by the capacity
 *   counts    [E] int32 / NULL   out  tokens choosing each expert (before drops)
 *   kept      [E] int32          out  rows filled in group e
 *   offsets   [E+1] int32        out  first row of group e (e*C with a capacity, else
 *                                     prefix sum of counts); offsets[E] = R
 *   row_src   [R] int32 / NULL   out  t*k + j for filled rows; unfilled rows untouched
 *   x_perm    [R, d] bf16        out  x_perm[slot_pos[t,j]] = x[t]; unfilled rows untouched
 * Rows of a group are in token order; an assignment is dropped when its rank
 * (tokens before it that chose the same expert) is >= C.  Bit-exact and
 * deterministic.
 */
int moe_permute(const moe_shape* s, const void* x, const int32_t* topk_idx, int32_t* slot_pos,
                uint8_t* drop_mask, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_src,
                void* x_perm, void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Grouped gated expert FFN (MoEEvolve SwiGLU experts; kieve-moe GeGLU; the
 * Kvasir worker's three matmuls; ExpertMesh INT4 routed-expert product).
 * Group g holds rows [group_start[g], group_start[g] + group_rows[g]) of
 * x_grouped and uses expert g's weights.  group_start / group_rows are device
 * arrays [n_groups]; both NULL means one group of all R rows.
 *   hidden        H of these experts (s->H for routed experts, s->H_s for the shared one)
 *   x_grouped     [R, d] bf16             in
 *   w13, w2       expert weights, layout per s->wfmt (n_groups experts)
 *   s13, s2       INT4 scales (NULL for bf16)
 *   h             [R, hidden] bf16        out (scratch the caller may read), or NULL for bf16 experts of
 *                                         hidden 128 or 256: then one fused kernel keeps each row tile's h
 *                                         in shared memory and h is not written (other shapes: NULL gives
 *                                         MOE_INVALID_ARGUMENT)
 *   y             [R, d] bf16             out  rows outside every group are untouched
 * Accumulation is fp32; h is rounded to bf16 once, y once (the same values with h NULL or not).
 */
int moe_expert_ffn(const moe_shape* s, int32_t n_groups, int32_t hidden, int64_t R, const void* x_grouped,
                   const int32_t* group_start, const int32_t* group_rows, const void* w13, const void* s13,
                   const void* w2, const void* s2, void* h, void* y, moe_stream_t stream);

/*
 * Weighted top-k reduction back to token order (ExpertMesh flowchart
 * "Weighted top-k reduction"; moe_stream.py ``out[mask] += w * expert_out``;
 * Kvasir ``combine(p, partials) + shared(cur)``).
 *   y_perm   [R, d] bf16       in
 *   slot_pos [T, k] int32      in   -1 = dropped, contributes nothing
 *   topk_w   [T, k] fp32       in
 *   y_shared [T, d] bf16/NULL  in   added at weight one
 *   out      [T, d] bf16       out  sum in fp32 in slot order, then shared, one rounding
 */
int moe_combine(const moe_shape* s, const void* y_perm, const int32_t* slot_pos, const float* topk_w,
                const void* y_shared, void* out, moe_stream_t stream);

/*
 * The whole layer: route -> permute -> grouped FFN -> shared expert -> combine,
 * enqueued on `stream` with no host synchronisation.
 *   x, w_router, bias          as moe_route
 *   w13, s13, w2, s2           routed experts (layout per s->wfmt; scales NULL for bf16)
 *   w13_sh, s13_sh, w2_sh, s2_sh  shared expert (E = 1, H = H_s); NULL when H_s == 0
 *   out        [T, d] bf16     out
 *   topk_idx, topk_w, counts, drop_mask, aux_f, aux_p, aux: optional outputs (NULL = not returned)
 *   workspace  >= moe_workspace_size() bytes of device memory, 256-byte aligned
 * INT4 experts: the activations are scaled per row by a power of two and rounded to f16 (exact for bf16
 * inputs from 2^-28 of the row's largest |x| up); the weights enter the MMAs as exact f16 integer codes
 * with a per-group offset that is removed in fp32, and the bf16 group scales multiply the fp32 group sums.
 *   side_stream  NULL, or a second stream of the caller's: with bf16 experts and a shared expert, the shared
 *                expert (which needs only x) runs there, forked from `stream` by an event at the start and
 *                joined back before the combine, so that it overlaps the routing, grouping and routed experts.
 *                The output is the same bit for bit.  All work is complete once `stream` passes the call's end.
 */
int moe_forward(const moe_shape* s, const void* x, const float* w_router, const float* bias, const void* w13,
                const void* s13, const void* w2, const void* s2, const void* w13_sh, const void* s13_sh,
                const void* w2_sh, const void* s2_sh, void* out, int32_t* topk_idx, float* topk_w,
                int32_t* counts, uint8_t* drop_mask, float* aux_f, float* aux_p, float* aux, void* workspace,
                size_t ws_bytes, moe_stream_t stream, moe_stream_t side_stream);

/*
 * Transposed copies of expert weights for the backward pass: wt[i][c][r] = w[i][r][c] for i < n, bf16.
 *   w   [n, rows, cols] in, wt [n, cols, rows] out (caller-owned device memory); n <= 65535.
 * For moe_backward_x: w13t = transpose of w13 ([E, d, 2H]), w2t = transpose of w2 ([E, H, d]), and the same
 * for the shared expert (n = 1).
 */
int moe_transpose_experts(const void* w, int64_t n, int32_t rows, int32_t cols, void* wt, moe_stream_t stream);

/* Scratch bytes moe_backward_x needs for this shape. */
int moe_backward_workspace_size(const moe_shape* s, size_t* bytes);

/*
 * Input gradient of the layer (training is the setting of kieve-moe Features, the MoEEvolve README and
 * MoEFFN.forward): dx = dL/dx for L = sum(dout * out) + aux_coef * aux, out as moe_forward computes it.
 * The routing decision (top-k, capacity drops) passes no gradient; the gate values, their renormalisation,
 * the softmax and the load-balance statistic aux = E sum_e f_e P_e (f_e counts, constant) do.  The forward's
 * routing, grouping and [g | u] are recomputed here; h and y are not (the gate gradient <dout, y> is taken as
 * <act(g) u, dout W2>).  bf16 experts only (MOE_UNSUPPORTED_SHAPE for INT4).
 *   x, w_router, bias, w13, w13_sh   as moe_forward (w13_sh NULL when H_s == 0)
 *   w13t, w2t, w13t_sh, w2t_sh       transposes of w13, w2, w13_sh, w2_sh (moe_transpose_experts); the down
 *                                    projections enter only through these
 *   dout      [T, d] bf16   in   dL/dout
 *   aux_coef                     weight of the statistic in L (0: none)
 *   dx        [T, d] fp32   out
 *   workspace >= moe_backward_workspace_size() bytes, 256-byte aligned
 * Precision: the expert steps run as bf16 GEMMs with fp32 accumulation (dout W2, [dg | du] and the recomputed
 * [g | u] rounded to bf16); the router's dz W_r takes bf16 operands.  dx sums its parts in fp32.
 * Errors: MOE_INVALID_ARGUMENT for a NULL or misaligned pointer, MOE_WORKSPACE_TOO_SMALL, a shape error as
 * moe_forward; nothing is enqueued then.
 */
int moe_backward_x(const moe_shape* s, const void* x, const float* w_router, const float* bias, const void* w13,
                   const void* w13t, const void* w2t, const void* w13_sh, const void* w13t_sh, const void* w2t_sh,
                   const void* dout, float aux_coef, float* dx, void* workspace, size_t ws_bytes,
                   moe_stream_t stream);

/*
 * The input gradient of moe_backward_x and the weight gradients of the same L (training: kieve-moe Features,
 * the MoEEvolve README Architecture, MoEFFN.forward), fp32, each summed over its rows:
 *   dw13      [E, 2H, d]    out  per expert, [dg | du]^T x over the expert's kept (token, slot) rows, with
 *                                dy = w_tj dout_t (dg = dh u act'(g), du = dh act(g), dh = dy W2)
 *   dw2       [E, d, H]     out  per expert, dy^T h over the same rows (h = act(g) u)
 *   dw13_sh   [1, 2H_s, d], dw2_sh [1, d, H_s]   out  the shared expert's, over all tokens with dy = dout
 *   dw_router [E, d]        out  dz^T x (dz = dL/dz of the logits, as in moe_backward_x)
 * Any weight-gradient pointer may be NULL: that gradient is not computed.  The exploration bias is a constant
 * here (its gradient would be the column sums of dz).  Other arguments, workspace and errors as
 * moe_backward_x (the same moe_backward_workspace_size covers both).
 * Precision: the weight gradients are bf16 GEMMs with fp32 accumulation over the rows of [dg | du], x,
 * dout, w h (bf16) and dz (bf16); a dense gradient (shared expert, router) sums row chunks in a fixed order.
 * Experts without kept rows get zeros.
 *   side_stream  NULL, or a second stream of the caller's: the shared expert's chain (which needs only the
 *                inputs) then runs there, forked from and joined back into `stream` by events, so that it
 *                overlaps the routed chain.  The results are the same either way.  All work the call enqueues
 *                is complete once `stream` passes the call's end.
 */
int moe_backward(const moe_shape* s, const void* x, const float* w_router, const float* bias, const void* w13,
                 const void* w13t, const void* w2t, const void* w13_sh, const void* w13t_sh, const void* w2t_sh,
                 const void* dout, float aux_coef, float* dx, float* dw13, float* dw2, float* dw13_sh,
                 float* dw2_sh, float* dw_router, void* workspace, size_t ws_bytes, moe_stream_t stream,
                 moe_stream_t side_stream);

/*
 * Hierarchical ("fractal") router (kieve-moe Features, "Fractal tiling routing": self-similar routing over a
 * branch^levels expert tree, a cheap router for very large expert pools).  Expert e is the leaf whose base-branch
 * digits d_0 .. d_{levels-1} (most significant first) choose a child per level; level l has its own router
 * W_l [branch, d] shared by all nodes of the level, q_l = softmax(x W_l^T + b_l), and the leaf probability is
 * p(e) = prod_l q_l[d_l].  Top-k of p (larger first, lower expert index first among equal values), gates
 * w_j = p(e_j), divided by their sum when s->renorm.  Cost per token: levels * branch logits, not E.
 *   s          T, d, k (<= 16, <= E), renorm; E must equal branch^levels (<= 2^20; the grouping and expert
 *              entry points take E <= 512); the other fields are not read
 *   branch     2 .. 32 children per node;  levels >= 1;  branch * levels <= 256 and a multiple of 4
 *   x          [T, d] bf16
 *   w_tree     [levels * branch, d] fp32: level l's router in rows [l * branch, (l + 1) * branch)
 *   bias_tree  [levels * branch] fp32 or NULL, added to the level logits
 *   topk_idx   [T, k] int32 out,  topk_w [T, k] fp32 out
 *   counts     [E] int32 out or NULL: selections per expert
 *   level_logits [T, levels * branch] fp32 out or NULL (then kept in the workspace)
 *   workspace  >= moe_route_tree_workspace_size() bytes, 256-byte aligned
 * Precision: the level logits are the tensor-core screen of the flat router (W split into two bf16 terms, x
 * bf16, fp32 accumulation: within about 2^-16 |x| |w| of the fp32 logits); softmax and products in fp32, each
 * leaf's product formed in level order; the top-k by a beam of the k best partial paths per level, exact for
 * those products.
 * Errors: MOE_INVALID_ARGUMENT (NULL or misaligned pointers, E != branch^levels, k > E),
 * MOE_UNSUPPORTED_SHAPE (limits above), MOE_WORKSPACE_TOO_SMALL; nothing is enqueued then.
 */
int moe_route_tree_workspace_size(const moe_shape* s, int32_t branch, int32_t levels, size_t* bytes);
int moe_route_tree(const moe_shape* s, int32_t branch, int32_t levels, const void* x, const float* w_tree,
                   const float* bias_tree, int32_t* topk_idx, float* topk_w, int32_t* counts, float* level_logits,
                   void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Group-scaled signed INT4 quantiser (ExpertMesh README: signed INT4 weights
 * with group scales).  For each row of w [rows, K] fp32 (K % 128 == 0) and
 * each group of 128 inputs: s = bf16(max|w| / 7), q = clamp(rint(w / s), -8, 7)
 * (q = 0 when s = 0), decisions in fp32.
 *   q      [rows, K/2] uint8 out   low nibble = even input index
 *   scales [rows, K/128] bf16 out
 */
int moe_quantize_int4(const float* w, int64_t rows, int32_t K, uint8_t* q, void* scales, moe_stream_t stream);

/*
 * moe_permute without a workspace argument.  No counterpart on the pages: it
 * exists for callers that cannot allocate device memory for scratch -- code
 * that runs where cudaMalloc is not allowed or not safe (inside a framework
 * that owns every device allocation, on a path that must not synchronise the
 * device, in a plug-in handed only its input and output buffers).
 *   Same arguments, outputs and rules as moe_permute, minus workspace/ws_bytes.
 *   Scratch: a fixed device array inside this library (about 1 MiB, held by
 *   every GPU that loads the library until the process exits) -- so
 *   ceil(T / 32) * E must be <= 262144, otherwise MOE_UNSUPPORTED_SHAPE is
 *   returned and nothing is enqueued.
 *   Allocates nothing: no cudaMalloc / cudaFree, no allocating library call.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and keeps it for later
 *   calls; make that first call before any stream capture.  A device reset
 *   (cudaDeviceReset) or a destroyed primary context invalidates the kept
 *   address: do not call this entry point after one.
 *   Every call shares the one array, which keeps the last call's contents:
 *   calls that overlap on the GPU (concurrent streams, or several host
 *   threads) race on it and must be serialised by the caller.
 */
int moe_permute_noalloc(const moe_shape* s, const void* x, const int32_t* topk_idx, int32_t* slot_pos,
                        uint8_t* drop_mask, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_src,
                        void* x_perm, moe_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears this device's status word.
 * *device_status receives MOE_OK or the first device-side error recorded
 * (MOE_DEVICE_TIMEOUT); *site (may be NULL) where it happened.  Returns
 * MOE_CUDA_ERROR if the synchronisation itself failed.
 */
int moe_get_status(moe_stream_t stream, int32_t* device_status, uint32_t* site);

/*
 * Upper bound, in nanoseconds, of every device-side wait (default 2e9).  The one
 * process-wide setting of the library (a debugging knob for failure tests): it
 * applies to kernels enqueued after the call, from any thread.
 */
int moe_set_wait_limit_ns(uint64_t ns);

/* Enqueue a kernel whose bounded wait on an mbarrier nobody arrives on must give
 * up after the wait limit: exercises the MOE_DEVICE_TIMEOUT path safely. */
int moe_selftest_wait_timeout(moe_stream_t stream);

/* Kernels this library has launched since load (all entry points, all threads). */
uint64_t moe_launch_count(void);

const char* moe_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
