/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) routed-experts MoE library
 * (libmoe_b200.so).
 *
 * The operation ("deepseek-ocr2-moe-experts" model card, description and
 * "Usage"):
 *
 *     out[t] = sum_{k<K} w[t,k] * down_e( SiLU(gate_e x_t) * (up_e x_t) ),
 *     e = top_k_index[t,k],
 *
 * with the argument order of the card's two ops
 * (hidden_states, gate_up_proj, down_proj, top_k_index, top_k_weights, top_k).
 * FP8 variants, the router and the quantiser follow the layer table of
 * "[Feature Request] - Supporting MegaKernel for DeepSeek Models"
 * ("Layer Tensor Details": moe_w13_fp8_layer, moe_silu_mul_layer,
 * moe_w2_fp8_layer, moe_topk_sigmoid_routing_layer, bf16_to_fp8_quantize,
 * moe_local_reduction).
 *
 * Conventions for every entry point:
 *  - Every tensor pointer is a DEVICE pointer owned by the caller; the
 *    library allocates no device memory and keeps no per-call state.  Where
 *    scratch memory is needed the caller passes a workspace of at least
 *    moe_experts_workspace_size() bytes.
 *  - Tensors are dense, row-major (last dimension contiguous), with the
 *    layouts written beside each argument.  bf16 = IEEE bfloat16,
 *    e4m3 = OCP FP8 E4M3 ("fn": no infinities, max 448), one byte per value.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *    enqueue work: they never synchronise with the host.
 *  - Arguments are validated on the host before anything is launched; a
 *    failed check returns an error code and enqueues nothing.  Launch
 *    failures return MOE_ERR_CUDA.  T == 0 is a valid no-op.
 *  - Results are deterministic: the same inputs give bitwise the same
 *    outputs on every call (no floating-point atomics; every sum has a
 *    fixed order).
 *  - Expert ids outside [0, E) contribute nothing to the output.
 *  - Calls on the same stream may reuse the same workspace; calls that may
 *    overlap (different streams) need separate workspaces.
 *  - Every workspace begins with an 8 KiB header: the int32 device status
 *    word at offset 0 (bits set by a kernel whose bounded wait expired) and
 *    the arrival counters of the fused bf16 decode kernel.  The header must
 *    be zero before a workspace's first use (allocate it zero-filled, or call
 *    moe_workspace_init once); every call that completes leaves it zero
 *    again.  After moe_workspace_status reports MOE_ERR_TIMEOUT, clear it
 *    (moe_workspace_status(..., clear = 1) does) before the next call.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

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
    MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad alignment     */
    MOE_ERR_UNSUPPORTED = 2,   /* shape or mode outside what is implemented */
    MOE_ERR_WORKSPACE = 3,     /* workspace missing or too small            */
    MOE_ERR_CUDA = 4,          /* a CUDA call or kernel launch failed       */
    MOE_ERR_TIMEOUT = 5        /* a bounded device wait of an earlier call
                                  expired (moe_workspace_status)             */
} moe_status_t;

typedef enum {
    MOE_W_BF16 = 0,            /* bf16 expert weights, bf16 activations      */
    MOE_W_FP8_E4M3 = 1,        /* e4m3 weights with fp32 per-(row,128) scales */
    MOE_W_MXFP4 = 2            /* packed E2M1 weights, E8M0 scale per (row,32),
                                  e4m3 activations (FP8 x FP4)                */
} moe_wtype_t;

/* Version of this ABI (incremented on any incompatible change). */
MOE_API int moe_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char *moe_status_string(moe_status_t status);

/*
 * Bytes of workspace needed by moe_experts_prefill (decode = 0) or
 * moe_experts_decode (decode = 1) for these sizes.  Returns 0 when the sizes
 * are invalid (the call itself then reports the error).
 */
MOE_API size_t moe_experts_workspace_size(int T, int H, int F, int E, int K, moe_wtype_t wt, int decode);

/*
 * Routed-experts forward, prefill form: a grouped GEMM over experts
 * (model card op "deepseek_ocr2_moe_experts").
 *
 *   hidden_states  [T,H]     bf16
 *   gate_up_proj   [E,2F,H]  bf16 | e4m3; rows [0,F) of each expert are the
 *                            gate projection, rows [F,2F) the up projection
 *   down_proj      [E,H,F]   bf16 | e4m3
 *   top_k_index    [T,K]     int32 expert ids
 *   top_k_weights  [T,K]     fp32 router weights
 *   top_k          K, 1 <= K <= 16
 *   T >= 0, H % 128 == 0, F % 128 == 0, 1 <= E <= 1024
 *   wt             weight dtype
 *   gate_up_scale  [E,2F,H/128] fp32 (e4m3 only; NULL for bf16): the value of
 *                  gate_up element (e,r,c) is e4m3(q) * gate_up_scale[e,r,c/128]
 *   down_scale     [E,H,F/128]  fp32 (e4m3 only; NULL for bf16)
 *   MXFP4 weights (wt = MOE_W_MXFP4; "FP8 x FP4" of the GC MoE issue and the
 *   DeepGEMM Mega MoE news page, MXFP4 of the OCP Microscaling format):
 *     gate_up_proj [E,2F,H/2] and down_proj [E,H,F/2] bytes, two E2M1 codes
 *                  per byte, the even column in the low nibble; 32-byte aligned
 *     gate_up_scale / down_scale: E8M0 bytes, one per row and 32 columns,
 *                  in the tensor cores' block layout: for each expert, one
 *                  512-byte block per (128 rows, 128 columns) in [R/128][C/128]
 *                  order, the scale of (r, c) at byte
 *                  (r%32)*16 + ((r%128)/32)*4 + (c%128)/32 of its block
 *                  (2F*H/32 and H*F/32 bytes per expert)
 *     value of element (e,r,c) = e2m1(code) * 2^(scale - 127)
 *   out            [T,H]     bf16, fully overwritten (any device-accessible
 *                            pointer, e.g. mapped pinned host memory: the
 *                            kernels store it directly)
 *   workspace      device scratch of >= moe_experts_workspace_size(..., 0)
 *                  bytes, 256-byte aligned; its 8 KiB header zero before
 *                  first use (see the conventions above), the rest needs no
 *                  initialisation
 *
 * bf16 path: h = bf16(SiLU(g) * u) is stored in bf16 between the GEMMs;
 * fp32 accumulation everywhere; the K contributions of a token are summed in
 * k order in fp32 and rounded once to bf16.
 * e4m3 path: hidden_states are quantised per 128 columns to e4m3 with a
 * power-of-two scale (the rule of quantize_fp8_block128), h is rounded to
 * bf16 and quantised the same way per 128 features, and each 128-long block
 * of every dot product is scaled by its activation and weight scales.
 * MXFP4 path: the same e4m3 activations; the tensor cores apply the weight
 * scale per 32 and the activation scale per 128 k-elements.
 * All pointers must be 16-byte aligned.
 */
MOE_API moe_status_t moe_experts_prefill(const void *hidden_states, const void *gate_up_proj,
                                 const void *down_proj, const int32_t *top_k_index,
                                 const float *top_k_weights, int top_k, int T, int H, int F,
                                 int E, moe_wtype_t wt, const void *gate_up_scale,
                                 const void *down_scale, void *out, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * Routed-experts forward, decode form for a few tokens (model card op
 * "deepseek_ocr2_moe_experts_decode", n_tokens about 1-4).  Same arguments,
 * layouts and results as moe_experts_prefill, workspace from
 * moe_experts_workspace_size(..., 1).
 *  - bf16 weights, T * K <= 16, H, F <= 2048: a fused gather-GEMV pair.
 *    The first kernel streams the gate and up rows of every touched expert
 *    once and writes h = bf16(SiLU(g) * u) for the slots routed to it; the
 *    second, a programmatic dependent of the first, streams the touched down
 *    rows once per hidden row, scales by the router weights and sums each
 *    token's K slots in k order.  The first kernel is itself launched as a
 *    programmatic dependent of the previous kernel on the stream and reads
 *    no input before that kernel has finished.
 *  - E4M3 and MXFP4 weights, and larger bf16 calls: the prefill kernels
 *    (E4M3 / MXFP4 with 16-row activation tiles at these sizes); same
 *    results within the parity tolerance.
 */
MOE_API moe_status_t moe_experts_decode(const void *hidden_states, const void *gate_up_proj,
                                const void *down_proj, const int32_t *top_k_index,
                                const float *top_k_weights, int top_k, int T, int H, int F,
                                int E, moe_wtype_t wt, const void *gate_up_scale,
                                const void *down_scale, void *out, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * The decode form as ONE kernel launch (the single-kernel fusion of the
 * DeepGEMM Mega MoE news page: the MoE steps in one kernel so that the
 * intermediate round trips between kernels go away).  Same arguments,
 * layouts and results (within the parity tolerance) as moe_experts_decode;
 * workspace from moe_experts_workspace_size(..., 1).
 *  - bf16 weights, T <= 16, T * K <= 64, H, F <= 2048: one launch does the
 *    expert dedup of the slots, the gate/up GEMV with SiLU*up, the down
 *    GEMV and the fixed-order top-K combine; the CTAs that need an expert's
 *    h wait (bounded) on a per-expert counter in the workspace header while
 *    their down-projection rows keep streaming in.  Launched as a
 *    programmatic dependent of the previous kernel on the stream.
 *  - MXFP4 weights, T <= 16, T * K <= 64: one persistent kernel after the
 *    permutation kernel (gate_up tiles, down tiles and the top-K combine;
 *    down tiles wait, bounded, for their rows' gate_up tiles).
 *  - anything else: MOE_ERR_UNSUPPORTED.
 * On B200 neither form is faster than moe_experts_decode's kernels at the
 * measured sizes, so moe_experts_decode does not use them.
 */
MOE_API moe_status_t moe_experts_decode_fused(const void *hidden_states, const void *gate_up_proj,
                                      const void *down_proj, const int32_t *top_k_index,
                                      const float *top_k_weights, int top_k, int T, int H, int F,
                                      int E, moe_wtype_t wt, const void *gate_up_scale,
                                      const void *down_scale, void *out, void *workspace,
                                      size_t workspace_bytes, void *stream);

/*
 * Bytes of workspace needed by moe_experts_with_shared for these sizes
 * (0 when the sizes are invalid).
 */
MOE_API size_t moe_experts_shared_workspace_size(int T, int H, int F, int E, int K, int S,
                                                 moe_wtype_t wt);

/*
 * Routed experts, S shared experts and a residual in one call: the expert
 * layer of a DeepSeek-style model with the two steps either side of the
 * routed op folded in ("Supporting MegaKernel for DeepSeek Models": the shared
 * expert is a SwiGLU MLP applied to every token; moe_local_reduction adds a
 * residual to the weighted sum of the expert rows):
 *
 *   out[t] = bf16( sum_{k<K} w[t,k] E_{idx[t,k]}(x_t)
 *                  + sum_{s<S} Shared_s(x_t) + residual[t] )
 *
 * summed in fp32 in that order (k ascending, then s, then the residual) and
 * rounded once.  Each shared expert has the routed experts' width F and the
 * same projections; a shared MLP of width S*F is the sum of S such experts
 * (split its rows into S blocks of F).  The shared experts run as S extra
 * expert ids of the same grouped GEMMs (every token gets them with weight
 * 1), so their rows share the routed experts' tiles, pipeline and
 * precision (e4m3: the same activation quantisation and block scales).
 *
 *   arguments shared with moe_experts_prefill: same meaning and layouts
 *   (MXFP4 routed weights return MOE_ERR_UNSUPPORTED here)
 *   shared_gate_up_proj  [S,2F,H] bf16 | e4m3 (same dtype as the routed weights)
 *   shared_down_proj     [S,H,F]  bf16 | e4m3
 *   shared_gate_up_scale [S,2F,H/128] fp32 (e4m3 only; NULL for bf16)
 *   shared_down_scale    [S,H,F/128]  fp32 (e4m3 only; NULL for bf16)
 *   S                    0 <= S, K + S <= 16, E + S <= 1024
 *                        (S = 0: routed experts plus the residual)
 *   residual             [T,H] bf16 or NULL (no residual)
 *   workspace            >= moe_experts_shared_workspace_size(T,H,F,E,K,S,wt)
 *                        bytes, 256-byte aligned
 * All pointers must be 16-byte aligned.
 */
MOE_API moe_status_t moe_experts_with_shared(
    const void *hidden_states, const void *gate_up_proj, const void *down_proj,
    const int32_t *top_k_index, const float *top_k_weights, int top_k, int T, int H, int F, int E,
    moe_wtype_t wt, const void *gate_up_scale, const void *down_scale,
    const void *shared_gate_up_proj, const void *shared_down_proj,
    const float *shared_gate_up_scale, const float *shared_down_scale, int S,
    const void *residual, void *out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode form without a workspace, for callers that cannot allocate device
 * memory where they run the layer: code recorded into a CUDA graph while
 * capture forbids allocation, serving loops and real-time hosts that fix
 * their device memory budget at start-up, plugin or embedded hosts that give
 * the code they load no allocator.  The pages have no counterpart of this
 * entry point; it exists for those callers only.
 *
 * Same arguments and layouts as moe_experts_decode, minus the workspace;
 * results equal moe_experts_decode's within the parity tolerance (relative
 * L2 error <= 5e-3), not always bit for bit: this entry always runs the
 * gather-GEMV decode kernels, which serve up to 64 slots (T*K), while
 * moe_experts_decode hands calls above 16 slots to the grouped GEMMs.  Its
 * scratch memory is a fixed 1 MiB array inside the library that every GPU
 * which loads the library holds until the process exits; 1 MiB is above the
 * largest decode scratch (64 slots x 2048 features of bf16 h).  The library
 * itself allocates nothing and calls no allocating routine.
 *  - bf16 weights only: e4m3 and MXFP4 weights return MOE_ERR_UNSUPPORTED;
 *    calls outside the decode range (T > 16, T*K > 64, H or F > 2048)
 *    return MOE_ERR_WORKSPACE.
 *  - Every call looks up the array's device address in the current context
 *    (after a cudaDeviceReset the next call finds the new one).  The first
 *    call in a context loads the library's device code there: make it before
 *    any stream capture.
 *  - All calls share the one array, which keeps the last call's contents:
 *    calls that may overlap on the GPU (other streams, or other host threads
 *    without ordering) race on it and must be serialised by the caller.
 */
MOE_API moe_status_t moe_experts_decode_static(const void *hidden_states, const void *gate_up_proj,
                                       const void *down_proj, const int32_t *top_k_index,
                                       const float *top_k_weights, int top_k, int T, int H, int F,
                                       int E, moe_wtype_t wt, const void *gate_up_scale,
                                       const void *down_scale, void *out, void *stream);

/*
 * Expert-parallel building blocks (DeepGEMM Mega MoE news page: EP dispatch
 * and combine around the expert GEMMs; "MegaMOE adaptation for SM90" PR:
 * dispatch to the ranks that own the experts, combine back to the tokens'
 * rank).  With the experts sharded over ranks, a rank runs its received
 * rows through moe_experts_rows and the tokens' rank sums the returned rows
 * with moe_combine_rows; the exchange between them is the caller's (the
 * Python package's expert-parallel layer uses NCCL all-to-all).
 *
 * moe_experts_rows: the grouped path of moe_experts_prefill without its
 * combine.  Same arguments except `out`; on return *y_offset is the byte
 * offset, inside `workspace`, of y [T*K][H] fp32: y[t*K+k] =
 * w[t,k] * down_e(SiLU(gate_e x_t) * (up_e x_t)) with e = top_k_index[t,k]
 * (rows of slots whose id is outside [0, E) are undefined).  The rows stay
 * valid until the next call that uses the workspace.
 */
MOE_API moe_status_t moe_experts_rows(const void *hidden_states, const void *gate_up_proj,
                                      const void *down_proj, const int32_t *top_k_index,
                                      const float *top_k_weights, int top_k, int T, int H, int F,
                                      int E, moe_wtype_t wt, const void *gate_up_scale,
                                      const void *down_scale, void *workspace,
                                      size_t workspace_bytes, size_t *y_offset, void *stream);

/*
 * The fixed-order top-K combine of caller rows: out[t] = bf16(sum over k
 * ascending, ids in [0, E) only, of y[t*K+k]) (the step that ends
 * moe_experts_prefill; "moe_local_reduction" of the MegaKernel layer table).
 *   y [T*K][H] fp32 (16-byte aligned), top_k_index [T][K] int32,
 *   out [T][H] bf16 (16-byte aligned), H % 128 == 0.
 */
MOE_API moe_status_t moe_combine_rows(const float *y, const int32_t *top_k_index, int top_k, int T,
                                      int H, int E, void *out, void *stream);

/*
 * Zeroes the 8 KiB header of a workspace (status word and counters),
 * asynchronously on `stream`; needed once before a workspace's first use
 * unless it was allocated zero-filled.  No allocation.
 *   workspace_bytes >= 8192; workspace 256-byte aligned.
 * Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_CUDA.
 */
MOE_API moe_status_t moe_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Device status of the calls that used `workspace`: waits for `stream`
 * (the one entry point that synchronises the host), reads the status word
 * and returns MOE_ERR_TIMEOUT when a bounded device wait of one of those
 * calls expired (that call's outputs are undefined), MOE_OK otherwise.
 * clear != 0 then zeroes the workspace header (status word and counters),
 * so that the workspace can be used again.  Grouped-GEMM (prefill-path)
 * calls restart the status word themselves; the fused decode kernel only
 * ever sets bits in it.
 * Returns MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_INVALID_ARG or MOE_ERR_CUDA.
 */
MOE_API moe_status_t moe_workspace_status(void *workspace, int clear, void *stream);

/*
 * Test-only form of moe_experts_decode for the fused bf16 decode kernel that
 * exercises its timeout path: CTA 0 never issues the weight copies of its
 * work chunk number `withhold_chunk` (0 = its first), so its bounded wait
 * for them expires (after about 2 s of SM clock cycles); the kernel then
 * sets MOE_ERR_TIMEOUT's status bit, drains its own copies and returns
 * without faulting.  The outputs of such a call are undefined.  Same
 * arguments as moe_experts_decode (bf16 weights, fused decode sizes only:
 * MOE_ERR_UNSUPPORTED otherwise).  Not part of the method (the pages have no
 * counterpart); it exists so that failure detection can be tested on a GPU
 * without a fault.
 */
MOE_API moe_status_t moe_debug_decode_withhold(const void *hidden_states, const void *gate_up_proj,
                                               const void *down_proj, const int32_t *top_k_index,
                                               const float *top_k_weights, int top_k, int T, int H,
                                               int F, int E, void *out, void *workspace,
                                               size_t workspace_bytes, int withhold_chunk,
                                               void *stream);

/*
 * Host-input staging for a step (no operation of the method: plumbing for
 * callers whose inputs arrive in host memory).  Copies `bytes` bytes from
 * `src` to the device memory `dst` with one kernel on `stream`.  `src` is
 * memory the GPU can read, typically pinned host memory allocated mapped
 * (cudaHostAllocMapped; pass its device pointer) that holds a step's hidden
 * states, top-k ids and top-k weights packed in one buffer.  Every load of
 * src bypasses the caches (ld.global.cv), so host writes made before the call
 * is enqueued are seen; the host must not modify src until the stream has
 * passed the call.  For the few KB of a decode step's inputs the kernel ends
 * sooner than a copy-engine transfer (cudaMemcpyAsync).
 *  - bytes: a multiple of 16, at most 1 GiB; src and dst 16-byte aligned and
 *    not overlapping; both buffers stay the caller's.
 *  - Returns MOE_OK (bytes == 0 is a no-op), MOE_ERR_INVALID_ARG (null or
 *    misaligned pointer, bad size) or MOE_ERR_CUDA.
 */
MOE_API moe_status_t moe_stage_inputs(const void *src, void *dst, size_t bytes, void *stream);

/*
 * Group-aware sigmoid top-k routing (layer table:
 * moe_topk_sigmoid_routing_layer, num_groups=8, topk_group=4,
 * routed_scaling_factor=2.5 for DeepSeek-V3).
 *
 *   logits [T,E] fp32, bias [E] fp32
 *   s_e = sigmoid(logit_e) evaluated in double and rounded to fp32;
 *   c_e = s_e + bias_e (fp32);
 *   group score = sum of the two largest c_e of each of num_groups equal,
 *   contiguous groups (the largest alone if a group has one expert);
 *   the topk_group best groups are kept; top_k experts with the largest c_e
 *   among the kept groups are chosen, best first;
 *   top_k_weights[t,k] = (s_k / sum_j s_j) * routed_scaling_factor in fp32,
 *   sum_j in selection order.  Equal scores rank the lower index first.
 *   top_k_index [T,K] int32, top_k_weights [T,K] fp32 (outputs);
 *   expert_offsets [E+1] int32 (optional output, may be NULL): exclusive
 *   prefix sum of the number of slots routed to each expert.
 * Limits: E % num_groups == 0, E <= 1024, num_groups <= 32,
 * topk_group <= num_groups, top_k <= 16 and top_k <= experts in kept groups.
 */
MOE_API moe_status_t moe_route_sigmoid_grouped(const float *logits, const float *bias, int T, int E,
                                       int num_groups, int topk_group, int top_k,
                                       float routed_scaling_factor, int32_t *top_k_index,
                                       float *top_k_weights, int32_t *expert_offsets,
                                       void *stream);

/*
 * Block-wise FP8 quantisation (layer table: bf16_to_fp8_quantize, block 128).
 *   x     [rows, cols] bf16, cols % 128 == 0
 *   xq    [rows, cols] e4m3 (output)
 *   scale [rows, cols/128] fp32 (output): per block of 128 values the
 *         smallest power of two s = 2^k, -127 <= k <= 127, with
 *         max|x| / s <= 448 (s = 1 for an all-zero block);
 *         xq = e4m3(x / s), round-to-nearest-even, saturating at +-448.
 */
MOE_API moe_status_t quantize_fp8_block128(const void *x, int rows, int cols, void *xq, float *scale,
                                   void *stream);

/*
 * Expert histogram and stable permutation of the T*K routing slots
 * (slot = t*K + k), exposed for exact testing of the step the prefill path
 * runs first.
 *   counts  [E]    slots routed to each expert
 *   offsets [E+1]  exclusive prefix sum of counts
 *   perm    [T*K]  slot at each permuted position; positions of one expert
 *                  hold its slots in ascending order; entries at positions
 *                  >= offsets[E] (slots with ids outside [0,E)) are -1
 *   inv     [T*K]  permuted position of each slot, -1 for ids outside [0,E)
 *   workspace      >= moe_experts_workspace_size(T, 128, 128, E, K, MOE_W_BF16, 0)
 */
MOE_API moe_status_t moe_debug_permute(const int32_t *top_k_index, int T, int K, int E, int32_t *counts,
                               int32_t *offsets, int32_t *perm, int32_t *inv, void *workspace,
                               size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
