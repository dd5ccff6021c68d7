/*
 * moe_b200.h -- C ABI of the routed sigmoid top-k MoE FFN library for one
 * NVIDIA B200 (sm_100a).
 *
 * Operations (definitions from the source pages, by page title and item):
 *
 *  - moe_route_topk     sigmoid + selection-bias top-k routing
 *                       [cortiq-engine 0.7.7, src/mimo_moe.rs: module doc
 *                       "top-8, sigmoid + selection-bias routing";
 *                       Dynamic::run, combine weight p[e] / wsum]
 *  - moe_router_topk    router projection x . W_router^T, then the routing
 *  - moe_route_weights  combine weights for ids fixed by the caller
 *                       [same page: the bank frame's "forced" picks with
 *                       "preweighted" mixes built by Dynamic::run]
 *  - moe_expert_map     per-expert counts and the expert-sorted permutation
 *                       of routed rows [mlx-native 0.13.0,
 *                       src/ops/dense_matmul_id_auto.rs: expected_dispatches,
 *                       the Grouped route's map pass; DenseMatmulIdScratch]
 *  - moe_matmul_id      y[t, j] = W[ids[t, j]] . x_row(t, j)
 *                       [same page: DenseMatmulIdShape, input layouts,
 *                       Direct and Grouped dispatch geometry]
 *  - moe_ffn_forward    y[t] = sum_j w[t, j] * down_e(silu(gate_e x) * up_e x)
 *                       [cortiq-engine src/mimo_moe.rs tests::exact_moe;
 *                       hf2q 0.1.1 eagle3/forward.rs, SwiGLU MLP "Phase
 *                       E4b.8"; hf2q qwen35/dense_ffn_arena.rs MoeFfnArena]
 *  - moe_ffn_forward_shared  the same plus a sigmoid-gated shared expert
 *                       [hf2q qwen35/dense_ffn_arena.rs: sh_logit, a_s, b_s, h_s]
 *  - moe_matmul_id_strided   moe_matmul_id over a padded expert stride
 *                       [mlx-native DenseMatmulIdShape expert_stride_bytes]
 *  - moe_ffn_slots      the FFN's per-slot rows before the weights and the
 *                       combine (for proofs of the balanced/skewed identity)
 *  - moe_matmul_id_noalloc   decode-size moe_matmul_id without a workspace
 *  - moe_ep_dispatch / moe_ep_combine   the device halves of an
 *                       expert-parallel layer step over G ranks (the
 *                       exchange between them is the caller's all-to-all)
 *
 * The library's launch sequences contain no allocation and no host
 * synchronisation, so a caller can capture moe_route_topk, moe_matmul_id and
 * moe_ffn_forward into a CUDA graph and replay it (tested).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    keeps no pointer after the call returns and never allocates, frees or
 *    synchronises the host.  Work is enqueued on `stream` (a cudaStream_t
 *    passed as void*; NULL means the legacy default stream).
 *  - Arguments are validated on the host before any launch; a failed
 *    validation returns a nonzero status with nothing enqueued and a message
 *    available from moe_last_error() (per calling thread).
 *  - Dense tensors are row-major and contiguous.  bf16 tensors are passed as
 *    moe_bf16_t (the 16-bit pattern of an IEEE bfloat16).
 *  - Routed row r = t * top_k + j names slot j of token t.
 *  - m == 0 is a valid empty call: nothing is launched and MOE_OK returned.
 *  - Errors found by kernels (an expert id outside [0, n_experts), a wait that
 *    timed out) are written to a status word inside the workspace; the kernels
 *    that follow skip their work and write nothing.  moe_check_status() reads
 *    that word (it synchronises `stream`; for tests and debugging).
 *  - Calls are deterministic: the same inputs give the same output bits, and,
 *    for a given call shape, a row's result does not depend on how many other
 *    rows chose its experts.  Each entry point picks its kernels from the
 *    shape alone (never from id values); calls of different shapes may take
 *    different paths, whose results agree to rounding.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef int moe_status_t;
typedef uint16_t moe_bf16_t;

#define MOE_OK 0
#define MOE_ERR_INVALID_ARGUMENT 1   /* null pointer, negative size, misaligned */
#define MOE_ERR_UNSUPPORTED_SHAPE 2  /* shape outside the limits listed below */
#define MOE_ERR_WORKSPACE_TOO_SMALL 3
#define MOE_ERR_CUDA 4               /* a CUDA runtime call failed */
#define MOE_ERR_DEVICE_TIMEOUT 5     /* a kernel wait exceeded its time limit */
#define MOE_ERR_DEVICE_BAD_ID 6      /* an expert id was outside [0, n_experts) */
#define MOE_ERR_DEVICE_RANGE 7       /* the grouped FFN's fp16 down projection gave a
                                        non-finite value (see moe_ffn_forward) */

/* Input layouts of mlx-native's DenseMatmulIdInputLayout. */
#define MOE_LAYOUT_SHARED_PER_TOKEN 0 /* x is [m, k]: every slot of token t reads x[t] */
#define MOE_LAYOUT_SLOTTED 1          /* x is [m, top_k, k]: slot j of token t reads x[t, j] */

/* Shape limits (others return MOE_ERR_UNSUPPORTED_SHAPE):
 *   1 <= n_experts <= 1024, 1 <= top_k <= min(n_experts, 32),
 *   m * top_k <= 2^24, every row width that is a GEMM K (k, hidden, inter)
 *   a multiple of 8 (16-byte rows for the tensor-memory copies),
 *   hidden % 4 == 0.  Pointers to bf16 and f32 tensors must be 16-byte
 *   aligned. */
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOP_K 32
#define MOE_MAX_ROUTED_ROWS (1 << 24)

/* Message describing the last failure on the calling thread ("" if none). */
MOE_API const char *moe_last_error(void);

/* Library version string. */
MOE_API const char *moe_version(void);

/*
 * Sigmoid + selection-bias top-k routing.
 *   logits  [m, n_experts] f32        router logits
 *   bias    [n_experts] f32 or NULL   selection bias (NULL = zeros)
 *   ids     [m, top_k] int32 (out)    chosen experts, slot order = key
 *                                     descending, lower expert index first
 *                                     on equal keys
 *   weights [m, top_k] f32 (out)      s[ids[t,j]] / sum_j s[ids[t,j]]
 *   scores  [m, n_experts] f32 or NULL (out)  s = sigmoid(logit)
 * with s = sigmoid(logit) computed in double and rounded once to f32,
 * key = s + bias[e] in f32 (NaN keys rank as -inf).  The bias decides the
 * choice only; the weights use s alone.  No workspace.
 */
MOE_API moe_status_t moe_route_topk(const float *logits, const float *bias, int32_t m,
                                    int32_t n_experts, int32_t top_k, int32_t *ids,
                                    float *weights, float *scores, void *stream);

/*
 * Combine weights for caller-fixed ids (forced routing):
 *   weights[t, j] = s[ids[t,j]] / sum_j s[ids[t,j]], s as in moe_route_topk.
 * An id outside [0, n_experts) makes that token's weights NaN.
 */
MOE_API moe_status_t moe_route_weights(const float *logits, const int32_t *ids, int32_t m,
                                       int32_t n_experts, int32_t top_k, float *weights,
                                       void *stream);

/*
 * Router projection followed by the routing above: the whole path from the
 * hidden state to the expert choice [cortiq-engine 0.7.7, src/mimo_moe.rs:
 * test model tensors mlp.gate.weight [NE, HS] and mlp.expert_bias [NE];
 * hf2q qwen35/dense_ffn_arena.rs: router logits buffer [seq, num_experts]].
 *   logits = x . W_router^T    x bf16 [m, hidden], W_router bf16 [E, hidden],
 *                              logits f32 [m, E] (out), f32 accumulate on the
 *                              tensor cores
 *   then ids/weights exactly as moe_route_topk computes them from `logits`.
 *   ws: moe_router_workspace() bytes, 256-byte aligned: a status word and,
 *       when the projection is split along K, its partial sums.
 * The projection runs in 256-column tiles; when few row tiles would leave
 * SMs idle, each tile's K is split into up to 8 ranges (a function of m,
 * hidden and n_experts only) whose f32 partial sums the routing kernel adds
 * in range order, so a given shape always gives the same logits bits.
 * hidden % 8 == 0; x and W_router 16-byte aligned.
 */
MOE_API size_t moe_router_workspace(int32_t m, int32_t hidden, int32_t n_experts);
MOE_API moe_status_t moe_router_topk(const moe_bf16_t *x, const moe_bf16_t *W_router,
                                     const float *bias, int32_t m, int32_t hidden,
                                     int32_t n_experts, int32_t top_k, float *logits,
                                     int32_t *ids, float *weights, void *ws, size_t ws_bytes,
                                     void *stream);

/*
 * Expert map: counting sort of the m*top_k routed rows by expert id.
 *   counts   [n_experts] int32 (out)   rows routed to each expert
 *   offsets  [n_experts+1] int32 (out) exclusive prefix sum, offsets[E] = m*top_k
 *   perm     [m*top_k] int32 (out)     routed rows of expert 0, then 1, ...;
 *                                      ascending r within an expert (stable)
 *   inv_perm [m*top_k] int32 (out)     inv_perm[perm[p]] = p
 *   ws       device workspace of at least moe_expert_map_workspace() bytes,
 *            256-byte aligned; its contents need no initialisation.
 * Ids may repeat within a token; ids out of range set MOE_ERR_DEVICE_BAD_ID in
 * the workspace status word (outputs then undefined).
 */
MOE_API size_t moe_expert_map_workspace(int32_t m, int32_t top_k, int32_t n_experts);
MOE_API moe_status_t moe_expert_map(const int32_t *ids, int32_t m, int32_t top_k,
                                    int32_t n_experts, int32_t *counts, int32_t *offsets,
                                    int32_t *perm, int32_t *inv_perm, void *ws,
                                    size_t ws_bytes, void *stream);

/*
 * Matmul by expert id:
 *   y[t, j, c] = sum_i W[ids[t,j], c, i] * x_row(t, j)[i]     (f32 accumulate)
 *   x   bf16, [m, k] (layout SHARED_PER_TOKEN) or [m, top_k, k] (SLOTTED)
 *   ids [m, top_k] int32 in [0, n_experts)
 *   W   bf16 [n_experts, n, k] (k contiguous)
 *   y   f32 [m, top_k, n] (out)
 *   ws  workspace of moe_matmul_id_workspace() bytes (256-byte aligned)
 * The path is chosen by shape only, never by id values: m*top_k <= 256 uses
 * the weight-streaming kernel (each chosen expert's rows read once with
 * 16-byte loads); larger m uses the tcgen05 grouped GEMM that gathers x rows
 * during the tensor-memory staging.
 */
MOE_API size_t moe_matmul_id_workspace(int32_t m, int32_t n, int32_t k, int32_t top_k,
                                       int32_t n_experts, int32_t layout);
MOE_API moe_status_t moe_matmul_id(const moe_bf16_t *x, const int32_t *ids, const moe_bf16_t *W,
                                   float *y, int32_t m, int32_t n, int32_t k, int32_t top_k,
                                   int32_t n_experts, int32_t layout, void *ws, size_t ws_bytes,
                                   void *stream);

/*
 * moe_matmul_id over an expert stack with a padded expert stride: expert e's
 * [n, k] matrix starts expert_stride_bytes * e bytes after W, and the bytes
 * between one expert's n*k*2 and the next expert's start are never read.
 * [mlx-native 0.13.0, src/ops/dense_matmul_id_auto.rs: DenseMatmulIdShape's
 * expert_stride_bytes, e.g. 832 for an 11 x 37 bf16 expert; the base-shape
 * keys distinguish strides]
 *   expert_stride_bytes  >= n*k*2, a multiple of 16 (TMA strides must be;
 *                        MOE_ERR_UNSUPPORTED_SHAPE otherwise), < 2^40;
 *                        0 or < n*k*2 is MOE_ERR_INVALID_ARGUMENT
 *   W    bf16, (n_experts - 1) * expert_stride_bytes + n*k*2 bytes
 * Every other argument, the workspace size (moe_matmul_id_workspace) and the
 * path choice are those of moe_matmul_id; with expert_stride_bytes = n*k*2
 * the result bits equal moe_matmul_id's.
 */
MOE_API moe_status_t moe_matmul_id_strided(const moe_bf16_t *x, const int32_t *ids,
                                           const moe_bf16_t *W, uint64_t expert_stride_bytes,
                                           float *y, int32_t m, int32_t n, int32_t k,
                                           int32_t top_k, int32_t n_experts, int32_t layout,
                                           void *ws, size_t ws_bytes, void *stream);

/*
 * Routed SwiGLU MoE FFN layer:
 *   for slot j of token t, e = ids[t, j]:
 *     a = silu(W_gate[e] . x_row) * (W_up[e] . x_row)      [inter]
 *     d = W_down[e] . a                                     [hidden]
 *   y[t] = sum_{j = 0..top_k-1} weights[t, j] * d_j         (in slot order)
 *   x       bf16 [m, hidden] or [m, top_k, hidden] (layout)
 *   ids     [m, top_k] int32; weights [m, top_k] f32 (e.g. from moe_route_topk)
 *   W_gate, W_up  bf16 [n_experts, inter, hidden]
 *   W_down        bf16 [n_experts, hidden, inter]
 *   y       f32 [m, hidden] (out)
 *   ws      workspace of moe_ffn_workspace() bytes (256-byte aligned); holds
 *           the expert map, the activation a and the per-slot weighted rows
 *           that the ordered, atomic-free combine sums.
 * The path is chosen by shape only: m*top_k <= 128 streams each chosen
 * expert's weights once (gate/up with SwiGLU, then down; a stays f32); larger
 * m runs the tcgen05 grouped GEMMs, whose down projection multiplies in fp16:
 * a is stored as fp16(a * 2^-4) (11 significant bits, the relative precision
 * of a bf16 value with 3 more bits), each W_down tile is rewritten in shared
 * memory as fp16(w) (exact for every bf16 w with 2^-17 <= |w| <= 65280;
 * smaller ones round with an absolute error of at most 2^-25), and the f32
 * accumulator is multiplied by 2^4, so every product and partial sum is the
 * unscaled one.  An |a| above 65504 * 2^4, a W_down entry of magnitude 65536
 * or more, or on this path a NaN or infinite input, makes the result
 * non-finite: the call then sets MOE_ERR_DEVICE_RANGE in the ws status word
 * (moe_check_status) and leaves y unwritten.
 */
MOE_API size_t moe_ffn_workspace(int32_t m, int32_t hidden, int32_t inter, int32_t top_k,
                                 int32_t n_experts, int32_t layout);
MOE_API moe_status_t moe_ffn_forward(const moe_bf16_t *x, const int32_t *ids,
                                     const float *weights, const moe_bf16_t *W_gate,
                                     const moe_bf16_t *W_up, const moe_bf16_t *W_down, float *y,
                                     int32_t m, int32_t hidden, int32_t inter, int32_t top_k,
                                     int32_t n_experts, int32_t layout, void *ws,
                                     size_t ws_bytes, void *stream);

/*
 * Proof/debug export of the routed layer's per-slot rows before the combine:
 *   d_slots[t, j, :] = W_down[e] . (silu(W_gate[e] . x_row) * (W_up[e] . x_row)),
 *   e = ids[t, j], unweighted, f32 [m, top_k, hidden] (out).
 * [mlx-native 0.13.0 dense_matmul_id_auto.rs: the balanced and maximally
 * skewed routing profiles must give identical per-row results; this export
 * lets a test compare every (token, expert) pair the two profiles share.]
 * Same kernels, path choice, arguments and workspace (moe_ffn_workspace) as
 * moe_ffn_forward, without the weights and the combine; moe_ffn_forward's
 * y[t] equals the slot-order f32 sum of weights[t, j] * d_slots[t, j] bit for
 * bit.
 */
MOE_API moe_status_t moe_ffn_slots(const moe_bf16_t *x, const int32_t *ids,
                                   const moe_bf16_t *W_gate, const moe_bf16_t *W_up,
                                   const moe_bf16_t *W_down, float *d_slots, int32_t m,
                                   int32_t hidden, int32_t inter, int32_t top_k,
                                   int32_t n_experts, int32_t layout, void *ws, size_t ws_bytes,
                                   void *stream);

/*
 * The routed layer plus a shared expert that every token takes
 * [hf2q qwen35/dense_ffn_arena.rs MoeFfnArena: sh_logit [seq, 1] (the shared
 * expert's gate input logit), a_s / b_s [seq, m_sh] (its gate and up
 * outputs), h_s [seq, m_sh] (their silu_mul)].  The page fixes the buffers,
 * not the formula; this library's reading is
 *     y[t] = moe_ffn_forward's y[t]
 *            + sigmoid(w_sh . x[t]) * W_sh_down (silu(W_sh_gate x[t]) * W_sh_up x[t])
 * with the shared term added after the last routed slot.
 *   x          bf16 [m, hidden] (one row per token: the shared-per-token layout)
 *   ids, weights, W_gate, W_up, W_down   as in moe_ffn_forward
 *   w_sh       bf16 [hidden]            (the shared expert's gate row)
 *   W_sh_gate, W_sh_up  bf16 [inter_sh, hidden]
 *   W_sh_down  bf16 [hidden, inter_sh]
 *   y          f32 [m, hidden] (out)
 *   ws         workspace of moe_ffn_shared_workspace() bytes (256-byte aligned)
 * inter_sh follows the hidden/inter rules (a multiple of 8).  The routed part
 * picks its kernels as moe_ffn_forward does (by m*top_k); the shared part
 * streams its weights for m <= 128 and runs the grouped GEMMs above, with the
 * gate logit from the tcgen05 dense projection.  Errors as moe_ffn_forward
 * (the grouped GEMMs' fp16 down projection and its range included).
 */
MOE_API size_t moe_ffn_shared_workspace(int32_t m, int32_t hidden, int32_t inter,
                                        int32_t inter_sh, int32_t top_k, int32_t n_experts);
MOE_API moe_status_t moe_ffn_forward_shared(
    const moe_bf16_t *x, const int32_t *ids, const float *weights, const moe_bf16_t *W_gate,
    const moe_bf16_t *W_up, const moe_bf16_t *W_down, const moe_bf16_t *w_sh,
    const moe_bf16_t *W_sh_gate, const moe_bf16_t *W_sh_up, const moe_bf16_t *W_sh_down, float *y,
    int32_t m, int32_t hidden, int32_t inter, int32_t inter_sh, int32_t top_k, int32_t n_experts,
    void *ws, size_t ws_bytes, void *stream);

/*
 * Matmul by expert id without a workspace, for callers that cannot allocate
 * device memory (a plugin whose host runtime owns every allocation, a decode
 * loop that must never enter the driver's allocator).  The source pages have
 * no counterpart of this entry point.
 *
 * Same arguments and result as moe_matmul_id, minus the workspace: the
 * expert-map scratch lives in a static device array of
 * MOE_NOALLOC_SCRATCH_BYTES that every GPU loading the library reserves until
 * the process exits.  Limits: m*top_k <= MOE_NOALLOC_MAX_ROUTED_ROWS (the
 * weight-streaming path); larger shapes return MOE_ERR_UNSUPPORTED_SHAPE.
 * The first call on a device looks up the array's address; make that first
 * call before any stream capture.  Destroying the device's primary context
 * after that first call (cudaDeviceReset) is not supported: the address stays
 * cached for the life of the process.  All calls on a device share the array and
 * leave the last call's contents in it: calls that overlap on the GPU (other
 * streams or threads without ordering) race and give wrong results.  Nothing
 * is allocated or freed.
 *
 * Device-side errors: an expert id outside [0, n_experts) leaves y unwritten
 * and sets the status word held in the static array (each call clears it
 * first).  moe_matmul_id_noalloc_status(stream) synchronises `stream` and
 * returns that word of the latest call on the current device: MOE_OK,
 * MOE_ERR_DEVICE_BAD_ID or MOE_ERR_DEVICE_TIMEOUT (for tests and debugging,
 * as moe_check_status is for the workspace entry points).
 */
#define MOE_NOALLOC_SCRATCH_BYTES (64 * 1024)
#define MOE_NOALLOC_MAX_ROUTED_ROWS 256
MOE_API moe_status_t moe_matmul_id_noalloc(const moe_bf16_t *x, const int32_t *ids,
                                           const moe_bf16_t *W, float *y, int32_t m, int32_t n,
                                           int32_t k, int32_t top_k, int32_t n_experts,
                                           int32_t layout, void *stream);
MOE_API moe_status_t moe_matmul_id_noalloc_status(void *stream);

/*
 * Expert parallelism over G ranks (one process per GPU; rank g owns experts
 * [g*E/G, (g+1)*E/G)).  The pages run every expert on one device and have no
 * counterpart of this split; the arithmetic is the routed FFN's own
 * [cortiq-engine 0.7.7, src/mimo_moe.rs tests::exact_moe; hf2q
 * qwen35/dense_ffn_arena.rs MoeFfnArena: per-slot rows y_all, then the
 * weighted reduce over the top-k slots].  One layer step on rank g:
 *
 *   1. moe_ep_dispatch: owner rank of routed row r = ids[r] / (E/G); the
 *      routed rows sorted by (owner, r) (stable) give the send order; their
 *      input rows are packed into send_x and their local expert ids
 *      (ids[r] - owner * E/G) into send_expert; send_counts[g'] = rows for
 *      rank g'.
 *   2. the caller exchanges send_x / send_expert by all-to-all (counts first)
 *      and runs moe_ffn_slots on what it received (layout SLOTTED, top_k 1,
 *      its E/G experts' weights), giving the unweighted per-slot rows d;
 *   3. the caller returns d by the reverse all-to-all, into d_back in this
 *      rank's send order;
 *   4. moe_ep_combine: y[t] = sum_j fl(weights[t,j] * d_back[pos(t,j)]), added
 *      in slot order in f32 (the same arithmetic as moe_ffn_forward's
 *      weighted epilogue and ordered combine).
 * With G = 1, or whenever each owner runs the kernels moe_ffn_forward would
 * run on those rows (m*top_k > 128 on both sides: the grouped GEMMs), y has
 * the bits of moe_ffn_forward's.
 *
 * moe_ep_dispatch:
 *   x            bf16 [m, hidden] (SHARED_PER_TOKEN) or [m, top_k, hidden] (SLOTTED)
 *   ids          int32 [m, top_k] in [0, n_experts)
 *   send_x       bf16 [m*top_k, hidden] (out), send order
 *   send_expert  int32 [m*top_k] (out), local expert id of each sent row
 *   send_counts  int32 [n_ranks] (out, device), rows for each rank (the
 *                rows for rank g' start at sum_{g'' < g'} send_counts[g''])
 *   ws           moe_ep_dispatch_workspace() bytes, 256-byte aligned; it holds
 *                the send order that moe_ep_combine reads, so keep it
 *                unchanged until the combine of the same step
 * n_experts % n_ranks == 0, 1 <= n_ranks <= n_experts; hidden % 8 == 0.
 * An id out of range sets MOE_ERR_DEVICE_BAD_ID in the ws status word
 * (moe_check_status); send_x, send_expert and the combine then stay unwritten.
 *
 * moe_ep_combine:
 *   d_back   f32 [m*top_k, hidden], row p = the owner's d for send position p
 *   weights  f32 [m, top_k];  y  f32 [m, hidden] (out)
 *   ws       the workspace of this step's moe_ep_dispatch (same m, top_k, n_ranks)
 */
MOE_API size_t moe_ep_dispatch_workspace(int32_t m, int32_t top_k, int32_t n_ranks);
MOE_API moe_status_t moe_ep_dispatch(const moe_bf16_t *x, const int32_t *ids, int32_t m,
                                     int32_t hidden, int32_t top_k, int32_t n_experts,
                                     int32_t n_ranks, int32_t layout, moe_bf16_t *send_x,
                                     int32_t *send_expert, int32_t *send_counts, void *ws,
                                     size_t ws_bytes, void *stream);
MOE_API moe_status_t moe_ep_combine(const float *d_back, const float *weights, float *y, int32_t m,
                                    int32_t hidden, int32_t top_k, int32_t n_ranks,
                                    const void *ws, size_t ws_bytes, void *stream);

/*
 * Stage timing hook (per calling thread).  When `events` is not NULL,
 * moe_ffn_forward records events[0..4] (cudaEvent_t values passed as void*)
 * on its stream: before the expert map, before gate/up, before down, before
 * the combine, and after the combine; moe_matmul_id records events[0..2]:
 * before the map, before the matmul, after it.  The caller owns the events;
 * pass NULL to stop recording.  n_events must be >= 5 (or 0 with NULL).
 */
MOE_API moe_status_t moe_set_stage_events(void *const *events, int32_t n_events);

/*
 * Reads the device status word of a workspace used by moe_expert_map,
 * moe_matmul_id or moe_ffn_forward (synchronises `stream`).  Returns MOE_OK,
 * MOE_ERR_DEVICE_BAD_ID or MOE_ERR_DEVICE_TIMEOUT.
 */
MOE_API moe_status_t moe_check_status(const void *ws, void *stream);

/*
 * Clock probe (measurement helper; the pages have no counterpart): launches
 * n_blocks blocks (1..4096) whose first thread each writes three uint64 to
 * out[3*b ..]: the SM id it ran on, that SM's cycle counter and the global
 * nanosecond timer.  Two probes enqueued around a timed region give the
 * average SM clock over it: (cycles_end - cycles_start) / (ns_end - ns_start)
 * for an SM present in both.  out: device memory of 3 * n_blocks uint64.
 */
MOE_API moe_status_t moe_clock_probe(uint64_t *out, int32_t n_blocks, void *stream);

/*
 * Self-test of the bounded wait that every kernel barrier uses: launches one
 * block that waits on a barrier nothing will complete, with the given limit
 * in nanoseconds (1..10^9).  The wait gives up, the kernel records
 * MOE_ERR_DEVICE_TIMEOUT in status_word (one int32 of device memory, which
 * the call first clears) and returns; the context stays usable.
 */
MOE_API moe_status_t moe_selftest_wait_timeout(int32_t *status_word, int64_t limit_ns,
                                               void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
