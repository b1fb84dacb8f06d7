/*
 * moe.h - C ABI of the B200 (sm_100a) dropless sparse Mixture-of-Experts
 * feed-forward block.
 *
 * The block, for T tokens x[T,H], E routed experts of which k are used per
 * token, and S always-on shared experts:
 *
 *   logits = x Wr^T + b                      moe_route    (router linear)
 *   (idx, w) = top-k of logits, softmax      moe_route    (over the k selected)
 *   group the T*k slots by expert            moe_permute  (stable, no drops)
 *   h = SiLU(x Wg_e^T) * (x Wu_e^T)          moe_forward  (grouped GEMM 1)
 *   o = s * w * (h Wd_e^T)                   moe_forward  (grouped GEMM 2)
 *   y_t = sum_j o_(t,j) + sum_shared FFN(x_t) moe_combine (back to token order)
 *
 * Sources, by page and section:
 *  - "PhiMoE in Transformers (Phi-3.5-MoE)", section 6: the router is a
 *    bias-free nn.Linear hidden -> num_local_experts, followed (in eval mode)
 *    by greedy top-1, masking, top-2 and a softmax over the selected experts;
 *    section 2 item 3: the experts' gate and up projections are packed as
 *    gate_up_proj (E, 2*I, H) and chunked into gate then up, act(gate) * up;
 *    section 2 item 4: the block is dropless (no capacity factor, no padding).
 *  - "Mixture of Experts in Transformers", expert backends: the grouped_mm
 *    backend sorts and groups tokens by expert id and runs one grouped GEMM;
 *    the runtime must dispatch tokens to their experts, run the projections,
 *    apply the routing weights, then gather and reorder the results.
 *    WeightConverter section: w1 (gate) and w3 (up) concatenated in that
 *    order; down_proj stacked per expert (E, H, I).
 *  - Instella-MoE modeling walk-through, FarSkipMoE and "config at a glance":
 *    routed output times a scaling factor (2.5) plus always-on shared experts.
 *  - GraniteMoeSWA page, decoder layer: the shared MLP output is added to the
 *    sparse MoE output; shared experts are off when their width is 0.
 *
 * Conventions for every entry point:
 *  - Every pointer argument except `shape` is a DEVICE pointer allocated and
 *    owned by the caller; the library allocates no memory and keeps no state
 *    beyond cached driver entry points and per-device attributes.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously; nothing synchronises the host.
 *  - Arguments are validated on the host before any launch.  A failure returns
 *    a status other than MOE_OK and enqueues nothing.  A launch failure
 *    returns MOE_ERR_CUDA.  Faults that only the device can see (an expert
 *    index out of range, a pipeline wait that times out) are OR-ed into the
 *    caller's device word `err_flag` as MOE_ERR_* bit values (1 << status);
 *    the caller zeroes it beforehand and reads it after synchronising.
 *  - Layouts are row-major and dense.  moe_dtype selects float32 or bf16 for
 *    x, the expert weights, the slot outputs and y.  The router weight and
 *    bias and all routing weights are float32; indices are int32.
 *  - The bf16 path needs H and I (and I_shared) to be multiples of 8 and all
 *    device pointers 16-byte aligned; otherwise MOE_ERR_UNSUPPORTED.
 *    E <= 256, k <= min(E, 16), n_shared <= 8, T*k < 2^31.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels implement */
    MOE_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    MOE_ERR_BAD_INDEX = 5,     /* device: an expert index outside [0, E) */
    MOE_ERR_TIMEOUT = 6        /* device: a pipeline wait exceeded its limit */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef struct {
    int64_t T;            /* tokens in this call (0 allowed: nothing is launched) */
    int32_t H;            /* hidden size */
    int32_t I;            /* routed expert intermediate size */
    int32_t E;            /* routed experts */
    int32_t k;            /* experts per token */
    int32_t n_shared;     /* always-on shared experts (0 = none) */
    int32_t I_shared;     /* shared expert intermediate size (0 when n_shared == 0) */
    float routed_scale;   /* multiplies the routed sum (1.0 for plain top-k MoE) */
    int32_t dtype;        /* moe_dtype of x, expert weights, y_slots and y */
} moe_shape;

/* Human-readable name of a status. Never NULL. */
MOE_API const char* moe_status_str(moe_status status);

/* Bytes of device workspace moe_permute and moe_forward need for `shape`
 * (written to *bytes).  One buffer of this size serves both calls; its
 * contents need no initialisation and are dead after each call returns on
 * the stream. */
MOE_API moe_status moe_workspace_size(const moe_shape* shape, size_t* bytes);

/* Router and selection ("PhiMoE in Transformers", section 6).
 *   x           [T, H]  dtype
 *   w_router    [E, H]  float32 (nn.Linear layout: out x in)
 *   router_bias [E]     float32, or NULL for a bias-free router
 *   logits      [T, E]  float32 output, or NULL to skip writing it
 *   topk_idx    [T, k]  int32 output: the k largest logits of each token in
 *                       descending order; equal logits go to the lower index
 *   topk_w      [T, k]  float32 output: softmax over the k selected logits
 *   err_flag    [1]     int32 device word, or NULL (see conventions)
 * Logits accumulate in float32.  Up to 256 tokens run on the CUDA cores, a
 * cluster of 8 CTAs per 16 tokens splitting H (one CTA per token where that
 * does not fit in shared memory); more tokens with bf16 x and E <= 64 run on
 * the tensor cores, the float32 weight split into three bf16 terms (exact to
 * one float32 ulp); anything else runs on the CUDA cores. */
MOE_API moe_status moe_route(const moe_shape* shape, const void* x, const float* w_router,
                             const float* router_bias, float* logits, int32_t* topk_idx,
                             float* topk_w, int32_t* err_flag, void* stream);

/* The float32 router weight split into three bf16 terms ahead of time, for the
 * tensor-core router.  The split depends on the weight alone, so a caller does
 * it once when the weights are loaded ("Mixture of Experts in Transformers",
 * WeightConverter section: conversions belong to the weight-loading
 * pipeline), not on every call.
 *
 * moe_router_split_size writes to *bytes the size of the split weight for
 * `shape`: N * H * 2 bytes with E_PAD = 8, 16, 32 or 64 (the smallest >= E) and
 * N = 3 * E_PAD rounded up to a multiple of 16; 0 when the tensor-core router
 * does not apply (float32 x, or E > 64).
 *
 * moe_router_split fills
 *   w_split  [N, H]  bf16 output, 16-byte aligned, caller-owned: row e is
 *                    hi(W[e]), row E_PAD + e is mid(W[e]), row 2 E_PAD + e is
 *                    lo(W[e]) where hi = bf16(w), mid = bf16(w - hi),
 *                    lo = bf16(w - hi - mid) (round to nearest even), so
 *                    hi + mid + lo equals w to within 2^-24 |w|; rows of
 *                    experts >= E and rows >= 3 E_PAD are zero.
 * It returns MOE_ERR_UNSUPPORTED when the size above is 0 or a pointer is not
 * 16-byte aligned, and MOE_ERR_WORKSPACE when w_split_bytes is too small.
 *
 * moe_route_split computes what moe_route computes, with the same arguments
 * plus `w_split` (the output of moe_router_split for this shape and weight,
 * or NULL).  For more than 256 tokens with bf16 x and E <= 64 it runs the
 * tensor-core router on w_split.  When the 128-token tiles alone would leave
 * SMs idle, a cluster of up to 8 CTAs splits H between them; CTA c forms its
 * partial logit (x.hi + x.mid) + x.lo over its slice and CTA 0 adds
 * bias + p_0 + p_1 + ... in rank order.  That is a different float32
 * summation order from moe_route's, within the same error bound; the result
 * is deterministic.  Otherwise, or when w_split is NULL, it is moe_route.
 * A w_split that does not match w_router gives the routing of the weight it
 * was split from. */
MOE_API moe_status moe_router_split_size(const moe_shape* shape, size_t* bytes);
MOE_API moe_status moe_router_split(const moe_shape* shape, const float* w_router, void* w_split,
                                    size_t w_split_bytes, void* stream);
MOE_API moe_status moe_route_split(const moe_shape* shape, const void* x, const float* w_router,
                                   const void* w_split, const float* router_bias, float* logits,
                                   int32_t* topk_idx, float* topk_w, int32_t* err_flag,
                                   void* stream);

/* DeepSeek-V3 routing, "noaux_tc" (named as the top-k method of the
 * DeepSeek-V3-derived Instella-MoE, Instella-MoE walk-through, "config at a
 * glance"; the pages do not define it, and this follows the DeepSeek-V3
 * technical report, section 2.1):
 *   s_e = sigmoid(l_e)  with l = x Wr^T (no bias in the logits)
 *   c_e = s_e + score_bias[e]          the bias steers the selection only
 *   experts form n_group contiguous groups of E / n_group; a group scores the
 *   float32 sum of its two largest c_e; the topk_group best groups are kept
 *   (ties to the lower group index); the k largest c_e among the kept groups
 *   are selected in descending order (ties to the lower expert index);
 *   topk_w[t, j] = s_(idx_j) / sum_i s_(idx_i)   (sums to 1; the routed
 *   scale of the shape multiplies the routed sum later, in moe_forward).
 * Arguments as moe_route_split, plus
 *   n_group, topk_group  1 <= n_group <= 32, E % n_group == 0,
 *                        1 <= topk_group <= n_group,
 *                        k <= topk_group * E / n_group (else INVALID_ARG)
 *   score_bias [E]       float32 selection bias, or NULL
 *   logits     [T, E]    float32, REQUIRED: receives the bias-free logits,
 *                        which the selection kernel then reads.
 * Two launches: the router (moe_route_split with no bias), then one warp per
 * token for the selection. */
MOE_API moe_status moe_route_noaux_tc(const moe_shape* shape, int32_t n_group,
                                      int32_t topk_group, const void* x, const float* w_router,
                                      const void* w_split, const float* score_bias,
                                      float* logits, int32_t* topk_idx, float* topk_w,
                                      int32_t* err_flag, void* stream);

/* Dropless dispatch plan ("Mixture of Experts in Transformers", grouped_mm
 * backend: sort and group tokens by expert id).  Slot q = t*k + j.
 *   topk_idx  [T, k]  int32 input
 *   counts    [E]     int32 output: slots routed to each expert (sum = T*k)
 *   offsets   [E+1]   int32 output: exclusive prefix sum of counts
 *   perm      [T*k]   int32 output: slot id at sorted position p, ordered by
 *                     (expert ascending, slot id ascending) - deterministic
 *   inv       [T*k]   int32 output: sorted position of slot q (perm^-1)
 *   err_flag  [1]     int32, OR-ed with 1 << MOE_ERR_BAD_INDEX if an index is
 *                     outside [0, E); such slots are skipped and the outputs
 *                     are then unspecified (all writes stay in bounds)
 *   workspace         at least moe_workspace_size() bytes */
MOE_API moe_status moe_permute(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* err_flag,
                       void* workspace, size_t workspace_bytes, void* stream);

/* moe_route_split followed by moe_permute, in one call: the outputs of both,
 * equal to what the two calls write (the same logits, selection, weights and
 * plan).  Arguments as the two calls; `workspace` as moe_permute's (checked
 * in every case).  For decode batches of up to 16 tokens with the cluster
 * router (H % 4 == 0, H <= 32768, a 16-byte aligned w_router) it is ONE
 * launch: the CTA that selects the experts of all the tokens also builds the
 * plan.  Otherwise it makes the two calls. */
MOE_API moe_status moe_route_permute(const moe_shape* shape, const void* x,
                                     const float* w_router, const void* w_split,
                                     const float* router_bias, float* logits, int32_t* topk_idx,
                                     float* topk_w, int32_t* counts, int32_t* offsets,
                                     int32_t* perm, int32_t* inv, int32_t* err_flag,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* moe_permute for callers that cannot allocate device memory: for example a
 * plugin whose host framework owns every device allocation and hands it only
 * its input and output buffers, or a latency-critical path where a cudaMalloc,
 * which may synchronise the device, is not allowed.  The pages have no
 * counterpart: this is a packaging of moe_permute, not a step of the method.
 * Arguments, outputs and errors are those of moe_permute (the same shape
 * validation), without the workspace.  Its scratch (the per-block expert
 * counts) is a 1 MiB array in the library's static device memory, which every
 * GPU that loads the library holds until the process exits; shapes needing
 * more than that, ceil(T*k / 2048) * E > 262144, return MOE_ERR_UNSUPPORTED.
 * The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress) and caches it with the id of the current CUDA
 * context; a later call that finds another context current (after a device
 * reset) looks it up again.  Make the first call on a device before any
 * stream capture.  All calls share the one array, so calls that can overlap
 * on the GPU (unordered streams) race on it.  Nothing in it needs clearing
 * between calls: every entry a call reads, that call has written first.  The
 * call allocates and frees nothing. */
MOE_API moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* topk_idx,
                                       int32_t* counts, int32_t* offsets, int32_t* perm,
                                       int32_t* inv, int32_t* err_flag, void* stream);

/* The expert FFNs, grouped by expert (two grouped GEMMs with fused epilogues).
 *   x           [T, H]          dtype
 *   offsets, perm               from moe_permute
 *   topk_w      [T, k]          float32 routing weights from moe_route
 *   gate_up     [E, 2I, H]      dtype; rows [0,I) gate, [I,2I) up
 *   down        [E, H, I]       dtype
 *   sh_gate_up  [S, 2Is, H]     dtype, or NULL when n_shared == 0
 *   sh_down     [S, H, Is]      dtype, or NULL when n_shared == 0
 *   y_slots     [T*k + S*T, H]  dtype output.  Row p < T*k holds
 *               routed_scale * topk_w[perm[p]] * FFN_e(x_t) for slot perm[p]
 *               (t = perm[p] / k, e its expert), rows in sorted order; row
 *               T*k + s*T + t holds shared expert s applied to x_t (weight 1).
 *   err_flag    [1] int32 device word (see conventions)
 *   workspace   at least moe_workspace_size() bytes
 * For small T*k the call streams each active expert's weights once (decode
 * path); otherwise it runs the tensor-core grouped GEMMs. */
MOE_API moe_status moe_forward(const moe_shape* shape, const void* x, const int32_t* offsets,
                       const int32_t* perm, const float* topk_w, const void* gate_up,
                       const void* down, const void* sh_gate_up, const void* sh_down,
                       void* y_slots, int32_t* err_flag, void* workspace,
                       size_t workspace_bytes, void* stream);

/* The S always-on shared experts of `shape` rearranged, once at load time,
 * into one shared expert of intermediate size S * I_shared ("Instella-MoE
 * modeling code walk-through", FarSkipMoE and "config at a glance": two
 * shared experts whose outputs are added to every token; "Mixture of Experts
 * in Transformers", WeightConverter section: layout conversions belong to
 * weight loading).  The sum over s of down_s (SiLU(gate_s x) * up_s x) is the
 * one expert's down (SiLU(gate x) * up x) with gate, up and h stacked along
 * the intermediate dimension and down concatenated along its columns, so
 * moe_forward / moe_combine called with n_shared = 1 and
 * I_shared = S * I_shared on these arrays compute the same block with one
 * shared slot row per token instead of S (S - 1 fewer rows of H written by
 * the forward and read by the combine; one rounding of the shared sum
 * instead of S).
 *   sh_gate_up       [S, 2Is, H]  dtype input (as moe_forward)
 *   sh_down          [S, H, Is]   dtype input
 *   gate_up_merged   [2 S Is, H]  dtype output, caller-owned: rows
 *                    [s Is, (s+1) Is) are expert s's gate rows, rows
 *                    [S Is + s Is, S Is + (s+1) Is) its up rows
 *   down_merged      [H, S Is]    dtype output, caller-owned: columns
 *                    [s Is, (s+1) Is) are expert s's down columns
 * Device pointers; outputs must not overlap the inputs.  Errors:
 * MOE_ERR_INVALID_ARG for n_shared == 0 or a NULL pointer, MOE_ERR_CUDA when
 * a copy fails to launch.  The copies are enqueued on `stream`. */
MOE_API moe_status moe_shared_merge(const moe_shape* shape, const void* sh_gate_up,
                                    const void* sh_down, void* gate_up_merged,
                                    void* down_merged, void* stream);

/* moe_forward with the routed experts' weights in MXFP4, for decode batches
 * ("Mixture of Experts in Transformers", section "from dense to sparse": at
 * small batch the time is the bytes of the active experts' weights, and the
 * gpt-oss experts are stored natively in mxfp4).  MXFP4 as the OCP
 * Microscaling Formats v1.0 specification defines it: each block of 32
 * consecutive weights along the contraction shares one E8M0 scale 2^(s-127)
 * (255 = NaN); each weight is an FP4 E2M1 code (sign, 2-bit exponent with
 * bias 1, 1-bit mantissa; values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives).
 *   gate_up_q [E, 2I, H/2]  uint8, 16-byte aligned: weight 2j of a row in the
 *                           low nibble of byte j, weight 2j+1 in the high
 *                           nibble; rows [0, I) gate, [I, 2I) up
 *   gate_up_s [E, 2I, H/32] uint8 E8M0 scale of each block of 32 weights
 *   down_q    [E, H, I/2]   uint8, same packing;  down_s [E, H, I/32] uint8
 * Other arguments, outputs and workspace as moe_forward (y_slots holds the
 * T*k routed rows).  Supported: bf16 x, 1 <= T <= 64, no shared experts, H
 * and I multiples of 32, the scale arrays 4-byte aligned; otherwise
 * MOE_ERR_UNSUPPORTED.  Two kernels, chosen by shape:
 *   - H and I multiples of 128 and the code arrays 32-byte aligned (64 with
 *     moe_forward_mxfp4_prepared below): the
 *     block-scaled tensor-core MMA (E2M1 weights x E4M3 activations, E8M0
 *     scales on both).  Each bf16 activation (x, then h rounded to bf16) is
 *     split per block of 32 into two E4M3 parts under E8M0 exponents, which
 *     reproduce it exactly except for elements below about 2^-13 of their
 *     block's largest magnitude; float32 accumulation.
 *   - otherwise: f16 MMAs with float32 accumulation; each activation row is
 *     scaled by a power of two that puts its largest magnitude in
 *     [2^14, 2^15) and rounded to f16; the scaling is undone in float32.
 * Weights must stay below 2^128 in magnitude (scale codes up to 252). */
MOE_API moe_status moe_forward_mxfp4(const moe_shape* shape, const void* x,
                                     const int32_t* offsets, const int32_t* perm,
                                     const float* topk_w, const uint8_t* gate_up_q,
                                     const uint8_t* gate_up_s, const uint8_t* down_q,
                                     const uint8_t* down_s, void* y_slots, int32_t* err_flag,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* The MXFP4 weights prepared once, at load time, for the block-scaled
 * tensor-core kernel ("Mixture of Experts in Transformers", WeightConverter
 * section: such conversions belong to the weight-loading pipeline):
 *   - the E8M0 scales re-laid out per (expert, tile of 128 weight rows,
 *     K-group of 128 weights) as one 512-byte block in the order the kernel
 *     copies them into tensor memory, so that a K-group takes one bulk copy
 *     instead of 128 per-row 4-byte reads (GEMM 1 tiles: 64 gate rows and
 *     the 64 up rows of the same columns; rows past an expert's and blocks
 *     past K/32 hold 127, 2^0);
 *   - when H (gate_up) or I (down) is not a multiple of 128, a copy of those
 *     codes with each row padded by zero codes to a multiple of 128 weights
 *     (the tensor maps that unpack 4-bit codes take whole 128-weight groups).
 *
 * moe_mxfp4_prepared_size writes to *bytes the size of the prepared array for
 * `shape`, or 0 when H or I is not a multiple of 64.
 *
 * moe_mxfp4_prepare fills `prepared` (16-byte aligned, caller-owned) from the
 * raw arrays of moe_forward_mxfp4; MOE_ERR_UNSUPPORTED when the size is 0 or
 * a pointer is misaligned, MOE_ERR_WORKSPACE when prepared_bytes is too small.
 *
 * moe_forward_mxfp4_prepared is moe_forward_mxfp4 on the tensor cores with
 * the prepared array in place of the scales, for H and I multiples of 64
 * (gpt-oss: 2880) as well as 128; gate_up_q and down_q are still the raw
 * codes (read where K is a multiple of 128).  x, the codes, `prepared`,
 * y_slots and the workspace 16-byte aligned, the codes 32-byte aligned;
 * otherwise MOE_ERR_UNSUPPORTED.  Arithmetic as moe_forward_mxfp4's
 * tensor-core kernel. */
MOE_API moe_status moe_mxfp4_prepared_size(const moe_shape* shape, size_t* bytes);
MOE_API moe_status moe_mxfp4_prepare(const moe_shape* shape, const uint8_t* gate_up_q,
                                     const uint8_t* gate_up_s, const uint8_t* down_q,
                                     const uint8_t* down_s, void* prepared,
                                     size_t prepared_bytes, void* stream);
MOE_API moe_status moe_forward_mxfp4_prepared(const moe_shape* shape, const void* x,
                                              const int32_t* offsets, const int32_t* perm,
                                              const float* topk_w, const uint8_t* gate_up_q,
                                              const uint8_t* down_q, const void* prepared,
                                              void* y_slots, int32_t* err_flag, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* Combine ("Mixture of Experts in Transformers", expert backends: gather and
 * reorder the results).  y[t] = sum_j y_slots[inv[t*k+j]]
 *                               + sum_s y_slots[T*k + s*T + t],
 * summed in float32 and rounded once to dtype.
 *   y_slots [T*k + S*T, H] dtype, inv [T*k] int32, y [T, H] dtype output. */
MOE_API moe_status moe_combine(const moe_shape* shape, const void* y_slots, const int32_t* inv,
                       void* y, void* stream);

/* Expert parallelism ("Mixture of Experts in Transformers", section "expert
 * parallelism"): GroupedGemmParallel keeps E/N experts on each of N ranks, a
 * slice of dim 0 of the packed gate_up_proj and down_proj; RouterParallel maps
 * the global expert indices to the rank's local ones and masks the other
 * ranks' experts; the ranks' partial outputs are then summed by an
 * all-reduce.  Every rank routes and plans the same tokens (moe_route and
 * moe_permute over all E experts give identical results on every rank), runs
 * the FFNs of its own experts, combines the slots of its own experts into a
 * float32 partial, and the partials are summed across ranks (an all-reduce,
 * for example NCCL's, on the caller's side) before one rounding to dtype.
 *
 * moe_forward_experts: moe_forward for routed experts [e_begin, e_end) only.
 *   gate_up_local [e_end - e_begin, 2I, H], down_local [e_end - e_begin, H, I]:
 *   the weights of those experts (expert e at index e - e_begin), NULL
 *   allowed when the range is empty.  sh_gate_up / sh_down: all n_shared
 *   shared experts, or both NULL on the ranks that do not compute them.
 *   Writes the y_slots rows of the range, [offsets[e_begin], offsets[e_end]),
 *   and, with the shared experts, rows T*k ... T*k + S*T - 1; other rows are
 *   left untouched.  Other arguments, workspace and errors as moe_forward;
 *   MOE_ERR_INVALID_ARG for a range outside [0, E] or only one shared
 *   pointer.
 * moe_combine_experts: the rank's float32 partial
 *   y_partial[t] = sum over j with e_begin <= topk_idx[t*k+j] < e_end of
 *                  y_slots[inv[t*k+j]]  (j ascending)
 *                + (with_shared ? sum_s y_slots[T*k + s*T + t] : 0).
 *   y_slots [T*k + S*T, H] dtype, inv [T*k], topk_idx [T, k] int32,
 *   y_partial [T, H] float32 output (16-byte aligned for bf16).
 * moe_cast_f32: y = y32 rounded once to dtype (round to nearest even); y32
 *   [T, H] float32 (16-byte aligned), y [T, H] dtype (8-byte aligned). */
MOE_API moe_status moe_forward_experts(const moe_shape* shape, int32_t e_begin, int32_t e_end,
                                       const void* x, const int32_t* offsets,
                                       const int32_t* perm, const float* topk_w,
                                       const void* gate_up_local, const void* down_local,
                                       const void* sh_gate_up, const void* sh_down,
                                       void* y_slots, int32_t* err_flag, void* workspace,
                                       size_t workspace_bytes, void* stream);
MOE_API moe_status moe_combine_experts(const moe_shape* shape, int32_t e_begin, int32_t e_end,
                                       int32_t with_shared, const void* y_slots,
                                       const int32_t* inv, const int32_t* topk_idx,
                                       float* y_partial, void* stream);
MOE_API moe_status moe_cast_f32(const moe_shape* shape, const float* y32, void* y, void* stream);

/* Training: the backward pass of the block.
 *
 * The pages name the training side of the block without detailing it: the
 * PhiMoE page attaches a load-balancing auxiliary loss to the router
 * ("PhiMoE in Transformers", section 6: load_balancing_loss_func after Switch
 * Transformer eqs. (4)-(6), times router_aux_loss_coef) and "Mixture of
 * Experts in Transformers" mentions fast grouped-GEMM training kernels.  The
 * gradients here are the chain rule through the forward above, for top-k
 * routing with the softmax over the selected k (the selection itself carries
 * no gradient):
 *   slot (t, j), expert e, weight w:  dO = s w dy_t
 *     dh = Wd_e^T dO,  dg = dh * u * SiLU'(g),  du = dh * SiLU(g)
 *     dWd_e += dO h^T,  dWgu_e += [dg; du] x_t^T,  dx_t += Wgu_e^T [dg; du]
 *     dw = s <dy_t, FFN_e(x_t)>
 *   router: dl_tj = w_tj (dw_tj - sum_i w_ti dw_ti) on the selected experts,
 *     plus, when aux_coef != 0, the auxiliary loss
 *     coef * E * sum_e f_e P_e (f_e = tokens dispatched to e / T, P_e = mean
 *     softmax probability of e over all E logits):
 *     dl_te += coef E / T * p_te (f_e - sum_c p_tc f_c);
 *     dWr = dl^T x, d_bias = sum_t dl_t, dx_t += dl_t Wr
 *   shared experts: as a routed expert with weight 1 on every token.
 * Supported: bf16, T > 8 (the tensor-core path), H a multiple of 64, I and
 * I_shared multiples of 32; otherwise MOE_ERR_UNSUPPORTED.
 *
 * moe_train_state_size: bytes of the state moe_forward_train keeps for the
 *   backward pass (gate/up pre-activations, SwiGLU outputs and the gathered x
 *   rows, bf16).
 * moe_forward_train: moe_forward that also fills `state` (>= that size,
 *   16-byte aligned); y_slots as moe_forward.
 * moe_backward_workspace_size / moe_backward: with the forward's routing
 *   (topk_idx, topk_w, counts, offsets, perm, inv), weights, `state` and the
 *   upstream gradient dy [T, H] bf16, writes
 *     dx [T, H] bf16,
 *     d_gate_up [E, 2I, H], d_down [E, H, I], d_sh_gate_up [S, 2Is, H],
 *     d_sh_down [S, H, Is], d_w_router [E, H] float32 (overwritten, not
 *     accumulated), d_router_bias [E] float32 or NULL,
 *     d_topk_w [T, k] float32 or NULL (the routing weights' gradient),
 *     aux_loss [1] float32 or NULL (the auxiliary loss value; accumulated
 *     with atomics, so its last bits may vary run to run).
 *   logits [T, E] float32 (the router's, from moe_route) is needed only when
 *   aux_coef != 0.  Every other output is deterministic.  Workspace: at least
 *   moe_backward_workspace_size() bytes, 16-byte aligned. */
MOE_API moe_status moe_train_state_size(const moe_shape* shape, size_t* bytes);
MOE_API moe_status moe_forward_train(const moe_shape* shape, const void* x,
                                     const int32_t* offsets, const int32_t* perm,
                                     const float* topk_w, const void* gate_up, const void* down,
                                     const void* sh_gate_up, const void* sh_down, void* y_slots,
                                     void* state, size_t state_bytes, int32_t* err_flag,
                                     void* workspace, size_t workspace_bytes, void* stream);
MOE_API moe_status moe_backward_workspace_size(const moe_shape* shape, size_t* bytes);
MOE_API moe_status moe_backward(const moe_shape* shape, const void* x, const float* w_router,
                                const int32_t* topk_idx, const float* topk_w,
                                const int32_t* counts, const int32_t* offsets,
                                const int32_t* perm, const int32_t* inv, const void* gate_up,
                                const void* down, const void* sh_gate_up, const void* sh_down,
                                const void* state, const float* logits, float aux_coef,
                                const void* dy, void* dx, float* d_gate_up, float* d_down,
                                float* d_sh_gate_up, float* d_sh_down, float* d_w_router,
                                float* d_router_bias, float* d_topk_w, float* aux_loss,
                                int32_t* err_flag, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Diagnostic with no counterpart in the pages: runs the bounded pipeline wait
 * that every kernel here uses on an mbarrier nothing ever arrives on, so that
 * it expires after timeout_ns (0 < timeout_ns <= 10 s).  The kernel then ORs
 * 1 << MOE_ERR_TIMEOUT into the device word err_flag (required) and returns;
 * the context stays usable.  Lets a caller check the device-side failure
 * path without a fault. */
MOE_API moe_status moe_selftest_wait_timeout(int64_t timeout_ns, int32_t* err_flag, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
