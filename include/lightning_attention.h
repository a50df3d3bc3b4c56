/*
 * lightning_attention.h - C ABI of the B200 (sm_100a) Lightning Attention library.
 *
 * Causal linear attention with no decay, no feature map and no normaliser:
 *
 *     O_t = q_t . S0 + sum_{s in seq(t), s <= t} (q_t . k_s) v_s
 *
 * computed the Lightning way (page "MiniMax-01 Lightning Attention", section
 * "Lightning Attention 设计"; page "首个线性注意力架构的大模型来了…", section
 * "4.1 创新的线性注意力"): tokens are cut into blocks of B; inside a block the
 * left product (Q_b K_b^T masked causally) V_b, across blocks the right product
 * Q_b . KV with the d x d prefix state KV = S0 + sum_{c<b} K_c^T V_c. The
 * decode step is the recurrent form S <- S + k^T v, o = q S, O(d^2) per token
 * (same page, same section, and section "与标准 Softmax Attention 的区别").
 *
 * Beside the method itself: its final states in the same pass
 * (la_prefill_with_state), its gradients (la_prefill_backward), the prefix of
 * LASP+ sequence parallelism (la_state_exclusive_prefix), a variant with a
 * decay rate per head on the state (la_prefill_decay, la_state_decay,
 * la_decode_step_decay, la_state_exclusive_prefix_decay; not on the pages),
 * and the feature map of one page as a separate pre-pass (la_feature_map).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    allocates no memory and performs no host synchronisation, except
 *    la_get_device_status, which synchronises the given stream.
 *  - q, k, v, o are packed token-major [total_tokens][heads][d], d fastest,
 *    element type given by `dtype` (bf16 or fp32). Sequences of a varlen pack
 *    are concatenated; cu_seqlens (device, int32 [num_seqs + 1]) holds their
 *    offsets: cu_seqlens[0] = 0, non-decreasing, cu_seqlens[num_seqs] =
 *    total_tokens. cu_seqlens = NULL means one sequence (num_seqs must be 1).
 *    No state crosses a sequence boundary.
 *  - States are fp32 [num_seqs or batch][heads][d][d], row-major, with
 *    element [i][j] = sum_t k_t[i] * v_t[j] (row index from k, column from v).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every launch is enqueued on it; nothing else is touched.
 *  - Arithmetic: fp32 accumulation throughout. For bf16 inputs the intra-block
 *    scores are rounded to bf16 (RNE) before the P.V product and the prefix
 *    state is rounded to bf16 (RNE) before the Q.KV product; O is rounded to
 *    bf16 (RNE) once at the end. fp32 inputs are computed in fp32 end to end.
 *
 * Errors
 * ------
 *  Host-checkable argument errors are returned before anything is enqueued.
 *  Launch errors return LA_ERR_CUDA. Conditions only visible on the device
 *  (cu_seqlens inconsistent with total_tokens, a bounded wait that ran out, a
 *  decay rate outside [0, 1]) set a per-device status word that
 *  la_get_device_status reports; the affected launch then writes no output
 *  rows (the decay entry points state what they leave unwritten).
 */
#ifndef LIGHTNING_ATTENTION_H
#define LIGHTNING_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARGUMENT = 1,    /* null pointer, negative size, aliasing, bad num_seqs   */
    LA_ERR_UNSUPPORTED = 2,         /* shape or dtype outside the supported set               */
    LA_ERR_MISALIGNED = 3,          /* a tensor pointer is not 16-byte aligned                */
    LA_ERR_WORKSPACE_TOO_SMALL = 4, /* workspace_bytes below the *_workspace_size() result     */
    LA_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed                   */
    LA_ERR_TIMEOUT = 6,             /* device: a bounded wait ran out (reported by status)    */
    LA_ERR_BAD_SEQLENS = 7,         /* device: cu_seqlens not 0..total_tokens non-decreasing  */
    LA_ERR_BAD_DECAY = 8            /* device: a decay rate outside [0, 1] (or NaN)            */
} la_status;

typedef enum { LA_BF16 = 0, LA_FP32 = 1 } la_dtype;

/*
 * Supported shapes: heads >= 1, d a multiple of 16 with 16 <= d <= 128,
 * B in {64, 128, 256}, total_tokens >= 0, num_seqs >= 1.
 * bf16 with d = 128 and B in {128, 256} runs on a tcgen05 tensor-core kernel:
 * the on-chip-state kernel (one CTA per sequence, head and half of the value
 * columns, the running state kept in tensor memory) when num_seqs * heads * 2
 * >= 64, else the block-parallel kernel (block prefixes by a single-pass
 * decoupled look-back scan; its CTAs take (block, head) tiles by atomic
 * ticket, so a tile only ever waits on tiles drawn earlier by CTAs already
 * running, and the launch finishes even while another kernel holds SMs);
 * la_debug_set_path overrides the choice. Every other supported combination
 * runs on the CUDA-core (SIMT) path.
 */

/* Bytes of device workspace la_prefill needs for these sizes (0 if unsupported). */
size_t la_prefill_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                 la_dtype dtype);

/*
 * Block-tiled causal linear attention prefill.
 *   q, k, v     in   [total_tokens][heads][d] (dtype)
 *   o           out  [total_tokens][heads][d] (dtype); must not overlap q, k or v
 *   cu_seqlens  in   device int32 [num_seqs + 1] or NULL (one sequence)
 *   init_state  in   device fp32 [num_seqs][heads][d][d] carried-in state S0, or NULL (zero)
 *   workspace   scratch, >= la_prefill_workspace_size(...) bytes, 256-byte aligned;
 *               its contents on entry do not matter and are undefined on exit
 * The result does not depend on B except through rounding.
 */
la_status la_prefill(const void* q, const void* k, const void* v, void* o,
                     const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens,
                     int heads, int d, int B, la_dtype dtype,
                     const float* init_state, void* workspace, size_t workspace_bytes,
                     void* stream);

/*
 * la_prefill without a workspace argument (no counterpart on the pages), for
 * callers that cannot allocate device memory: allocator-free runtimes, fixed
 * memory budgets, hooks that run inside another library's memory manager. Its
 * scratch is one static device array of LA_NOALLOC_SCRATCH_BYTES that every
 * GPU loading the library holds until the process exits. Arguments and
 * results are those of la_prefill. Problems whose la_prefill_workspace_size
 * exceeds LA_NOALLOC_SCRATCH_BYTES are rejected with
 * LA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued. It allocates
 * nothing: the first call on each device (with that device current) looks up
 * the array's device address once, so make that first call before any stream
 * capture. All calls on a device share the array; calls that overlap on the
 * GPU race and give undefined results. The scratch used is the copy of the
 * device current on the calling thread, so `stream` must belong to that
 * device. The looked-up address is kept for the life of the process: after a
 * cudaDeviceReset of a device, this entry point may not be called on it again.
 */
#define LA_NOALLOC_SCRATCH_BYTES (64u << 20)
la_status la_prefill_noalloc(const void* q, const void* k, const void* v, void* o,
                             const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens,
                             int heads, int d, int B, la_dtype dtype,
                             const float* init_state, void* stream);

/* Bytes of device workspace la_state_from_prefill needs (0 if unsupported). */
size_t la_state_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, la_dtype dtype);

/*
 * Final recurrent state of each sequence after its prefill:
 *   state_out[s][h] = S0[s][h] + sum_{t in seq s} k_t^T v_t    (fp32, [num_seqs][heads][d][d])
 * This is the state the decode step continues from (the d x d KV state the
 * right product carries, page "MiniMax-01 Lightning Attention", section
 * "Lightning Attention 设计"). init_state may be NULL (zero) or equal to
 * state_out (in-place accumulate); it must not partially overlap it.
 */
la_status la_state_from_prefill(const void* k, const void* v, const int32_t* cu_seqlens,
                                int num_seqs, int64_t total_tokens, int heads, int d,
                                la_dtype dtype, const float* init_state, float* state_out,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * la_prefill that also returns each sequence's final state, the state a decode
 * (or the next chunk of a chunked prefill) continues from:
 *   o          as la_prefill
 *   state_out  fp32 [num_seqs][heads][d][d] = init_state + sum_{t in seq} k_t^T v_t
 * On the on-chip-state path (bf16, d = 128, B in {128, 256}, at least 64
 * (sequence, head, value-half) work items) this is one pass: the prefill
 * kernel's accumulator already holds the running state, and the kernel writes
 * it out after each sequence's last block. Sequences of one token (a serving
 * batch's continuations) are not work items there: at the end of the same
 * launch they are run as decode steps, S = S0 + k^T v, o = q S0 + (q . k) v,
 * at close to the HBM rate of their states (page "MiniMax-01 Lightning
 * Attention", section "计算优化": prefill and decode kept apart, fused into one
 * batched launch). Elsewhere it is la_prefill followed by
 * la_state_from_prefill. state_out may be init_state itself (in-place
 * update); it must not overlap q, k, v, o or the workspace otherwise. The
 * workspace is la_prefill_with_state_workspace_size bytes. Errors as
 * la_prefill, plus LA_ERR_INVALID_ARGUMENT for a NULL state_out.
 */
size_t la_prefill_with_state_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                            la_dtype dtype);
la_status la_prefill_with_state(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                                int num_seqs, int64_t total_tokens, int heads, int d, int B, la_dtype dtype,
                                const float* init_state, float* state_out, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * Backward pass of la_prefill (the training pass; the pages give the forward
 * only, so this is the calculus of its definition). With
 * S_t = S0 + sum_{s <= t, same sequence} k_s^T v_s, O_t = q_t S_t and
 * L = sum_t dout_t . O_t:
 *   dq_t = dout_t S_t^T
 *   dk_s = v_s R_s^T,  dv_s = k_s R_s,  R_s = sum_{t >= s, same sequence} q_t^T dout_t
 *   dinit_state = R at each sequence's first token (= sum_t q_t^T dout_t)
 * Computed with the forward kernels: dq is a prefill of (dout, v, k) from
 * init_state^T; dv and dk are anti-causal prefills (keys at or after each
 * query) of (k, q, dout) and (v, dout, q): on the on-chip-state path by that
 * kernel's anti-causal instance, which walks each sequence's blocks from the
 * last, elsewhere by causal prefills over every sequence reversed, reversed
 * back; dinit_state is la_state_from_prefill of (q, dout). Rounding is that of
 * those prefills (bf16 operands, fp32 accumulation; bf16 outputs for bf16
 * inputs).
 *   q, k, v, dout     in   [total_tokens][heads][d], dtype (device)
 *   init_state        in   fp32 [num_seqs][heads][d][d] or NULL (the forward's S0)
 *   dq, dk, dv        out  [total_tokens][heads][d], dtype; no overlap with the
 *                          inputs, each other or the workspace
 *   dinit_state       out  fp32 [num_seqs][heads][d][d], or NULL (not computed)
 * Shapes, dtypes and errors as la_prefill; the workspace is
 * la_prefill_backward_workspace_size bytes (on the reversal path five
 * [T][H][d] tensors, plus the prefill's and the state pass's workspaces),
 * 256-byte aligned, caller-owned.
 * Asynchronous on `stream`; allocates nothing.
 */
size_t la_prefill_backward_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                          la_dtype dtype);
la_status la_prefill_backward(const void* q, const void* k, const void* v, const void* dout,
                              const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, int heads, int d, int B,
                              la_dtype dtype, const float* init_state, void* dq, void* dk, void* dv,
                              float* dinit_state, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sequence parallelism (LASP+): each of `world` ranks holds a contiguous
 * segment of the same sequences, computes its segments' states from a zero
 * state (la_state_from_prefill with init_state = NULL), exchanges them with
 * one all-gather, and takes a local prefix sum as the init_state of its own
 * la_prefill (page "MiniMax-01 Lightning Attention", section "计算优化",
 * item 3: AllGather + local prefix sum instead of serial send/receive; page
 * "首个线性注意力架构的大模型来了…", section "4.2 计算优化"). This call is
 * that local prefix sum:
 *   out[i] = init[i] + sum_{r < rank} gathered[r][i]     (fp32, rank order)
 *   gathered  in   fp32 [world][n][d][d], n = num_seqs * heads, the gathered
 *                  segment states (device)
 *   init      in   fp32 [n][d][d], the state before the first segment, or NULL
 *                  (zero); may equal out, must not partially overlap it
 *   out       out  fp32 [n][d][d] (device); must not overlap gathered
 * rank = world gives the state after the last segment (the decode state).
 * Errors: LA_ERR_INVALID_ARGUMENT (world < 1, rank outside [0, world], n < 0,
 * null pointers, overlaps), LA_ERR_UNSUPPORTED (d), LA_ERR_MISALIGNED (any
 * pointer not 16-byte aligned). Asynchronous on `stream`; allocates nothing.
 */
la_status la_state_exclusive_prefix(const float* gathered, int world, int rank, int64_t n, int d,
                                    const float* init, float* out, void* stream);

/*
 * One recurrent decode step for `batch` independent sequences:
 *   S <- S + k^T v ;  o = q S      (o sees the updated state: s <= t)
 *   q, k, v  in      [batch][heads][d] (dtype)
 *   state    in/out  fp32 [batch][heads][d][d], updated in place
 *   o        out     [batch][heads][d] (dtype); must not overlap q, k, v or state
 * O(d^2) work per (sequence, head), independent of how many tokens came before
 * (page "MiniMax-01 Lightning Attention", section "与标准 Softmax Attention 的区别").
 */
la_status la_decode_step(const void* q, const void* k, const void* v, float* state, void* o,
                         int batch, int heads, int d, la_dtype dtype, void* stream);

/* ------------------------------------------------------------------ decay variant
 * Not on the pages: Lightning Attention with a decay rate per head on the
 * state, the Lightning Attention-2 form of the same method taken in its
 * plainest reading (a rate of 1 is the method without decay):
 *
 *     S_t = lambda_h S_{t-1} + k_t^T v_t,   S_{start-1} = S0,   o_t = q_t S_t
 *     O_t = lambda^(t-start+1) q_t . S0 + sum_{s in seq(t), s <= t} lambda^(t-s) (q_t . k_s) v_s
 *
 * `decay` is fp32 [heads] in device memory, 4-byte aligned, read only, each
 * rate in [0, 1]; lambda^0 = 1 also for lambda = 0. A rate outside [0, 1] or
 * NaN is a device-side condition: la_get_device_status reports
 * LA_ERR_BAD_DECAY; la_prefill_decay and la_state_decay then write nothing at
 * all, la_decode_step_decay nothing for that head.
 * la_prefill_decay runs on the on-chip-state tensor-core kernel where
 * la_prefill would (bf16, d = 128, B in {128, 256}, at least 64 work items of
 * (sequence, head, value half)); there the state's increments read
 * lambda^(n-1-c) v_c rounded to bf16. Every other shape, and la_state_decay,
 * runs on CUDA cores in fp32.
 */

/*
 * The exclusive prefix of LASP+ sequence parallelism with decay: rank `rank`'s
 * starting state when every rank holds one contiguous segment of the same
 * sequences, ranks in sequence order.
 *   P_0 = S0 (init, or zero),  P_r = lambda_h^(n_{r-1}) P_{r-1} + S_{r-1}
 *   gathered  in   fp32 [world][num_seqs][heads][d][d]: rank r's segment states
 *                  from a zero start (la_state_decay of its segments)
 *   seg_lens  in   int32 [world][num_seqs]: length of rank r's segment of each
 *                  sequence (>= 0); may be NULL when rank == 0
 *   decay     in   fp32 [heads], rates in [0, 1]
 *   init      in   fp32 [num_seqs][heads][d][d] or NULL; may be `out` itself
 *   out       out  fp32 [num_seqs][heads][d][d]; rank == world gives the state
 *                  after the last segment
 * All device pointers; gathered, init and out 16-byte aligned, seg_lens and
 * decay 4-byte aligned. Errors as la_state_exclusive_prefix; on the device a bad
 * rate (LA_ERR_BAD_DECAY) or a negative length (LA_ERR_BAD_SEQLENS) leaves the
 * affected states unwritten.
 */
la_status la_state_exclusive_prefix_decay(const float* gathered, const int32_t* seg_lens, int world, int rank,
                                          int num_seqs, int heads, int d, const float* decay, const float* init,
                                          float* out, void* stream);

/* Workspace for la_prefill_decay; 0 for an unsupported shape. */
size_t la_prefill_decay_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                       la_dtype dtype);

/*
 * Prefill with decay. Arguments, layouts and errors as la_prefill, plus:
 *   decay      in   fp32 [heads] (see above); may not overlap o, state_out or the workspace
 *   state_out  out  fp32 [num_seqs][heads][d][d], each sequence's final state
 *                   lambda^n S0 + sum_t lambda^(end-1-t) k_t^T v_t, or NULL for none. It may
 *                   be init_state itself (updated in place); it may not overlap any other
 *                   argument. Empty sequences get S0 (or zero).
 * Block decomposition (block of n tokens from b0, KV the state before b0, r = t - b0):
 *   O_t = sum_{u=b0..t} lambda^(t-u) (q_t . k_u) v_u + lambda^(r+1) q_t KV,
 *   KV' = lambda^n KV + sum_u lambda^(b0+n-1-u) k_u^T v_u;
 * the result does not depend on B beyond rounding. Launches: tensor-core path:
 * sequence table, rate check, (empty-sequence states,) prefill; CUDA cores:
 * block table (2), rate check, block states, scan, prefill.
 */
la_status la_prefill_decay(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                           int num_seqs, int64_t total_tokens, int heads, int d, int B, la_dtype dtype,
                           const float* init_state, const float* decay, float* state_out, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Workspace for la_prefill_backward_decay; 0 for an unsupported shape. */
size_t la_prefill_backward_decay_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                                la_dtype dtype);

/*
 * Gradients of L = sum_t dout_t . O_t for O = la_prefill_decay(...): arguments, layouts and errors
 * as la_prefill_backward, plus `decay` as above. With R_s = sum_{t >= s} lambda^(t-s) q_t^T dO_t:
 *   dq_t = dO_t S_t^T   (the decay prefill of (dO, V, K) from S0^T),
 *   dk_s = R_s v_s, dv_s = R_s^T k_s   (decay prefills over the reversed sequences, reversed back),
 *   dS0  = lambda R_start   (the decayed state of the reversed (Q, dO), times lambda).
 * The rates are constants of this pass: no gradient with respect to lambda is
 * computed or returned. `decay` may not overlap the workspace or dinit_state
 * (LA_ERR_INVALID_ARGUMENT).
 */
la_status la_prefill_backward_decay(const void* q, const void* k, const void* v, const void* dout,
                                    const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, int heads, int d,
                                    int B, la_dtype dtype, const float* init_state, const float* decay, void* dq,
                                    void* dk, void* dv, float* dinit_state, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Workspace for la_state_decay; 0 for an unsupported shape. */
size_t la_state_decay_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, la_dtype dtype);

/*
 * Final state with decay of each sequence, without the output:
 *   state_out[s][h] = lambda_h^n S0 + sum_t lambda_h^(end-1-t) k_t^T v_t  (n tokens).
 * Arguments and errors as la_state_from_prefill, plus `decay` as above.
 */
la_status la_state_decay(const void* k, const void* v, const int32_t* cu_seqlens, int num_seqs,
                         int64_t total_tokens, int heads, int d, la_dtype dtype, const float* init_state,
                         const float* decay, float* state_out, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * One decode step with decay: S <- lambda_h S + k^T v ; o = q S.
 * Arguments and errors as la_decode_step, plus `decay` as above (it may not
 * overlap state or o). Same bandwidth as la_decode_step: one read and one
 * write of the fp32 state.
 */
la_status la_decode_step_decay(const void* q, const void* k, const void* v, float* state, void* o, int batch,
                               int heads, int d, la_dtype dtype, const float* decay, void* stream);

/*
 * Feature map phi(x) = ELU(x) + alpha x, elementwise over n values (page
 * "MiniMax-M2.5语言模型：Linear Attention架构解析与实践", section "2.2 Linear
 * Attention的数学原理", which takes alpha = 0.3; ELU(x) = x for x > 0,
 * e^x - 1 otherwise). A pre-pass for q and k before a prefill or decode step,
 * for callers that want the feature map; the prefill itself uses q and k as
 * given.
 *   x  in   n values of `dtype`, 16-byte aligned
 *   y  out  n values of `dtype`, 16-byte aligned; may be x itself (in place),
 *           may not overlap x otherwise
 * Computed in fp32, rounded to nearest even for bf16. Errors:
 * LA_ERR_INVALID_ARGUMENT (n < 0, null pointer, partial overlap, alpha not
 * finite), LA_ERR_UNSUPPORTED (dtype), LA_ERR_MISALIGNED.
 */
la_status la_feature_map(const void* x, void* y, int64_t n, la_dtype dtype, float alpha, void* stream);

/*
 * Synchronises `stream`, then returns and clears the status word of the
 * current device: LA_OK, LA_ERR_BAD_SEQLENS, LA_ERR_TIMEOUT or
 * LA_ERR_BAD_DECAY (the first condition recorded since the last call), or
 * LA_ERR_CUDA if the synchronisation itself failed.
 */
la_status la_get_device_status(void* stream);

/*
 * Instrumentation (no counterpart on the pages). Arms a one-shot timer for the
 * calling host thread: the next la_prefill or la_decode_step call made by this
 * thread records `start_event` on its stream immediately before enqueuing its
 * main kernel (the fused intra/inter-block kernel, or the decode kernel) and
 * `stop_event` immediately after, then disarms. Both are cudaEvent_t passed as
 * void*, owned by the caller; NULL, NULL disarms. Lets a caller time the
 * dominant kernel alone with cudaEventElapsedTime.
 */
la_status la_set_kernel_timer(void* start_event, void* stop_event);

/*
 * Test hook (no counterpart on the pages). For the following la_prefill calls
 * made by this host thread on the tensor-core path, every device-side wait
 * gives up after `wait_ns` nanoseconds (0 = the default of 4 s), and
 * `suppress_tile` (-1 = none) names a unit of work that withholds one hand-off:
 *  - block-parallel kernel: tile block * heads + head (over the blocks of all
 *    sequences) publishes no state, so its successors' look-backs wait;
 *  - on-chip-state kernel: work item w (2 * (rank * heads + head) + half, rank
 *    = position of the sequence in longest-first order) never hands the prefix
 *    of its second block to the tensor cores.
 * The bounded waits then expire: the launch ends by itself,
 * la_get_device_status reports LA_ERR_TIMEOUT and the CUDA context stays
 * usable. Call with (-1, 0) to reset.
 */
la_status la_debug_set_fault(long long suppress_tile, uint64_t wait_ns);

/*
 * Tracing (no counterpart on the pages). While a buffer is set, every
 * la_prefill call made by this host thread on a tensor-core path records
 * phase stamps into `device_buffer`; unused slots are left as they were.
 *  - Block-parallel kernel: for each tile (block * heads + head over the
 *    blocks of all sequences), 48 uint64 globaltimer stamps (ns): [0] first Q
 *    tile ready, [1] chunk MMAs issued, [2] prefix available, [3]/[4]
 *    look-back start/end, [5] prefix written, [6] inclusive state published,
 *    [7] output stored, [8] aggregate published, [9] last P written, [10..47]
 *    finer steps of the worker roles. The buffer must hold max_tiles * 384
 *    bytes, max_tiles = (ceil(total_tokens / B) + num_seqs) * heads, or the
 *    call records nothing.
 *  - On-chip-state kernel, in builds compiled with -DLA_CHAIN_TRACE only (the
 *    stamps cost instruction-cache space in every role, so a default build
 *    records nothing): for each CTA and each block it processes (in
 *    order), 16 uint64 SM-clock stamps (clock64) of its roles: [0] Q load,
 *    [1]/[2] first/last K/V load, [3] first score MMA, [4] first PV MMA,
 *    [5]/[7] inter-block MMAs, [6] last state MMA, [8]/[9] first/last P,
 *    [10] state ready, [11] prefix handed over, [12]/[13] output accumulators
 *    complete, [14] last output store, [15] last PV MMA. The buffer holds
 *    grid * blocks_per_cta * 128 bytes for as many blocks per CTA as fit
 *    (grid = min(2 * num_seqs * heads, SM count)).
 * NULL, 0 stops tracing.
 */
la_status la_debug_set_trace(void* device_buffer, size_t bytes);

/*
 * Test hook (no counterpart on the pages). Chooses, for the following calls
 * made by this host thread, which tensor-core prefill kernel la_prefill,
 * la_prefill_noalloc and la_prefill_workspace_size use for bf16, d = 128,
 * B in {128, 256}: 0 = automatic (the default), 1 = the on-chip-state kernel
 * (one CTA per sequence, head and half of the value columns, blocks walked in
 * order), 2 = the block-parallel kernel (one CTA per SM over (block, head)
 * tiles, block prefixes by a single-pass decoupled look-back scan). Automatic
 * picks the on-chip-state kernel when num_seqs * heads * 2 >= 64. Results are
 * the same up to rounding. Returns LA_ERR_INVALID_ARGUMENT for any other value.
 */
la_status la_debug_set_path(int path);

/*
 * Number of kernels this library has launched, from every host thread, since
 * the process loaded it (no counterpart on the pages). Read it before and
 * after a sequence of calls to count the launches they made. Never fails.
 */
uint64_t la_launch_count(void);

/* Static, human-readable name of a status code. */
const char* la_status_string(la_status s);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_ATTENTION_H */
