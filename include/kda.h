/*
 * kda.h -- C ABI of libkda, the B200 (sm_100a) Kimi Delta Attention forward.
 *
 * KDA keeps, per head, a fixed-size state S and updates it once per token t:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t
 *
 * i.e. decay each key channel of the state by alpha_t, predict the value the
 * decayed state holds for k_t, write beta_t times the prediction error along
 * k_t, and read the updated state with the query scaled by 1/sqrt(d_k).
 * Source: "Kimi Delta Attention: The Linear Attention Behind Kimi K2 and
 * Qwen3", §TL;DR (per-channel decay Diag(alpha_t), delta rule scaled by
 * beta_t) and §How Kimi Delta Attention works step by step (the order of the
 * operations, in prose); "KDA Technical Deep Dive", §From attention to
 * recurrent state (delta rule, forgetting form) and §How the Kimi gate
 * changes memory (gate).
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor arguments are DEVICE pointers to dense, contiguous, row-major
 *   arrays on the current CUDA device.  The caller owns and allocates every
 *   buffer.  The library's own device memory is the workspace pool of
 *   kda_forward and kda_gdn_forward (see kda_forward) and the fixed scratch of
 *   kda_forward_noalloc; every other call uses only what it is given.
 * - The state is stored as [dk, dv] per head (key channels are rows, the value
 *   axis is contiguous).  The pages write the same matrix as (d_v, d_k); this
 *   is its transpose, so the per-channel decay scales rows.
 * - The gate is passed as log_alpha = log(alpha), fp32, alpha in (0, 1).
 *   beta is fp32; any finite value is accepted (the pages use (0, 1)).
 * - Keys (and queries) are expected L2-normalised by the caller, as the pages
 *   require for stability; the library does not renormalise.
 * - `scale` multiplies the query on the read.  Pass 0.0f for the pages'
 *   default 1/sqrt(dk).  A non-finite scale is KDA_ERR_INVALID_ARG.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *   asynchronous: a KDA_OK return means the work was validated and enqueued.
 *   Launch failures are reported as KDA_ERR_CUDA; a device-side wait that ran
 *   out of its iteration limit is reported by kda_check_status().
 * - Every argument is validated on the host before anything is enqueued; on
 *   any error status nothing is launched and no output is touched.
 * - Calls never throw and never abort; they are safe to call from several
 *   host threads on different streams.
 * - Outputs are fp32 for both input dtypes (bf16 output would already exceed
 *   the 2e-3 relative error the bf16 path is held to).
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kda_status {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null required pointer, bad size, non-finite scale, bad dtype */
    KDA_ERR_UNSUPPORTED = 2,   /* head dimensions this build has no kernel for */
    KDA_ERR_MISALIGNED = 3,    /* a tensor pointer is not 16-byte aligned */
    KDA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed (see kda_last_cuda_error) */
    KDA_ERR_TIMEOUT = 5        /* a device-side wait gave up after its iteration limit */
} kda_status;

typedef enum kda_dtype {
    KDA_BF16 = 0,              /* q, k, v are bfloat16 */
    KDA_F32 = 1                /* q, k, v are float32 */
} kda_dtype;

/*
 * kda_forward -- chunked prefill over a whole sequence batch.
 *
 * Computes o_t for every token and, optionally, the state after the last
 * token, processing the sequence in chunks of 64 tokens whose boundary state
 * is the initial condition of the next chunk ("KDA Technical Deep Dive",
 * §Systems and implementation tradeoffs, Training; the chunkwise mode noted
 * under §How Kimi Delta Attention works step by step of the other page).
 *
 *   q, k          [B, T, H, dk]  dtype            (16-byte aligned)
 *   v             [B, T, H, dv]  dtype            (16-byte aligned)
 *   log_alpha     [B, T, H, dk]  float32          (16-byte aligned)
 *   beta          [B, T, H]      float32          (4-byte aligned)
 *   initial_state [B, H, dk, dv] float32 or NULL  (NULL = zero state)
 *   out           [B, T, H, dv]  float32          (16-byte aligned)
 *   final_state   [B, H, dk, dv] float32 or NULL  (NULL = not written)
 *
 * final_state may be the same pointer as initial_state (in-place carry); any
 * other overlap between inputs and outputs is undefined.  B, H >= 1, T >= 0.
 * Supported head dimensions: dk, dv in {64, 128} for both dtypes.  T = 0
 * writes no output and sets final_state to initial_state (or zeros).
 * q, k, v, log_alpha, beta and out may be NULL only when T = 0.
 *
 * Schedule: with bf16 inputs and dk = dv = 128 the call is kda_forward_ws on a
 * workspace the library takes from its own stream-ordered memory pool (one
 * per device, created on first use) and gives back on `stream` once the
 * call's kernels are enqueued, so results are bit-identical to kda_forward_ws.
 * The workspace is kda_forward_workspace_bytes() capped at 1 GiB (never below
 * kda_forward_workspace_min_bytes()); the pool keeps up to 1 GiB between
 * calls (kda_workspace_pool_bytes, kda_workspace_pool_trim).  If the pool
 * cannot supply it, and for other dtypes or head dimensions, the call runs the
 * one-kernel prefill, which needs no device memory beyond its arguments (what
 * kda_forward_ws does with no workspace).
 */
kda_status kda_forward(const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta,
                       const float *initial_state, float *out, float *final_state,
                       int B, int T, int H, int dk, int dv,
                       kda_dtype dtype, float scale, void *stream);

/*
 * kda_forward_ws -- kda_forward with a caller-provided device workspace.
 *
 * Same computation, arguments and results as kda_forward.  With bf16 inputs and
 * dk = dv = 128 and a workspace of at least kda_forward_workspace_min_bytes(),
 * the prefill runs as two kernels per block of chunks: one computes every
 * chunk's chunk-local quantities in parallel (the in-chunk decay sums, A and
 * its UT inverse, and the products that do not involve the state), writing one
 * record per chunk into the workspace; the other walks the chunks of each
 * (b, h) in order, carrying the state through them ("KDA Technical Deep
 * Dive", §Systems and implementation tradeoffs, Training: chunk-local work in
 * parallel, the boundary state seeding the next chunk).  Blocks of chunks
 * carry the state between them in the workspace:
 *   - few heads, long sequence (2 B H at most the SM count, at least 128 chunks),
 *     and room for two blocks of 8 or more chunks: pipelined.  The chain of
 *     block i (one CTA per (b, h)) runs beside the chunk-local kernel of block
 *     i + 1 on the other SMs, their records in alternating halves of the
 *     workspace.  All launches go to `stream`; the chunk-local launch of block
 *     i + 1 is programmatically dependent on the chain of block i (it starts
 *     once the chain's CTAs are resident and does not wait for it to finish).
 *   - otherwise: the chunk-local kernel, then the chain, per block of as many
 *     chunks as fit (the whole sequence with its full record size).
 * Which chain kernel runs depends only on B, T and H, so every workspace size
 * gives bit-identical results.
 *
 *   workspace        device memory, 256-byte aligned, owned by the caller; its
 *                    contents on entry do not matter and on return are
 *                    unspecified.  It must not be used by another call that
 *                    may run at the same time.
 *   workspace_bytes  its size in bytes.
 *
 * With a NULL or too small workspace, or for other dtypes and head dimensions,
 * the call runs the one-kernel prefill: each (b, h) walks its chunks in one CTA
 * that computes the chunk-local quantities and carries the state, using no
 * device memory beyond the call's arguments.  A workspace not 256-byte aligned
 * is KDA_ERR_MISALIGNED.
 */
kda_status kda_forward_ws(const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta,
                          const float *initial_state, float *out, float *final_state,
                          int B, int T, int H, int dk, int dv,
                          kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes,
                          void *stream);

/*
 * Workspace sizes for kda_forward_ws: the size the fastest schedule uses, and the
 * smallest size that still takes the two-kernel path (one chunk per block plus the
 * carried state).  Both are 0 when the two-kernel path does not apply (dtype, head
 * dimensions, T = 0 or bad sizes).  The records take about 145 KB per chunk of 64
 * tokens per (b, h).  For few heads (2 B H at most the SM count) and sequences of
 * at least 128 chunks, the fastest schedule is pipelined: blocks of up to 64 chunks
 * (the first and the last of 32) whose records alternate between two slots while the
 * chain of one block runs beside the chunk-local kernel of the next, so the size is
 * two 64-chunk blocks' records plus the carried state (0.61 GB for B1 H32 T65536);
 * otherwise it is the whole sequence's records.
 */
size_t kda_forward_workspace_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype);
size_t kda_forward_workspace_min_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype);

/*
 * Workspace size for kda_segment_local / kda_segment_correct: every chunk record of
 * the segment (they must all stay for the correction).  0 where the two-kernel path
 * does not apply.
 */
size_t kda_segment_workspace_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype);

/* Steps before the path that kda_forward_raw can fuse into the prefill. */
enum {
    KDA_PREP_LOGSIGMOID_GATE = 1,  /* gate holds pre-activations x; log alpha = log(sigmoid(x)) */
    KDA_PREP_L2NORM_QK = 2         /* q and k rows are L2-normalised (a zero row stays zero) */
};

/*
 * kda_forward_raw -- kda_forward_ws on raw layer activations.
 *
 * The step before the path is fused into the prefill's first kernel: with
 * KDA_PREP_LOGSIGMOID_GATE, `gate` [B, T, H, dk] fp32 holds the gate
 * pre-activations x and the decay is alpha = sigmoid(x) (the sigmoid-like
 * retention gate of "KDA Technical Deep Dive", §How the Kimi gate changes
 * memory); with KDA_PREP_L2NORM_QK, q and k are divided by the L2 norm of
 * their dk channels per (b, t, h) (the normalised keys and queries that "Kimi
 * Delta Attention: The Linear Attention Behind Kimi K2 and Qwen3" expects the
 * path to receive).  Both run in fp32 on the bf16 inputs before the chunk
 * algebra; nothing is written back.
 *
 *   prep       an OR of KDA_PREP_* flags (other bits: KDA_ERR_INVALID_ARG).
 *              prep = 0 is exactly kda_forward_ws.
 *   gate       [B, T, H, dk] fp32, 16-byte aligned: log alpha, or x with
 *              KDA_PREP_LOGSIGMOID_GATE.
 *   workspace, workspace_bytes  as for kda_forward_ws.
 *
 * With prep != 0 the call needs the two-kernel path: bf16 inputs, dk = dv = 128
 * and a workspace of at least kda_forward_workspace_min_bytes(); otherwise it
 * returns KDA_ERR_UNSUPPORTED before anything is enqueued.
 */
kda_status kda_forward_raw(const void *q, const void *k, const void *v,
                           const float *gate, const float *beta,
                           const float *initial_state, float *out, float *final_state,
                           int B, int T, int H, int dk, int dv,
                           kda_dtype dtype, float scale, unsigned int prep,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Time-axis split of one long sequence (context parallelism).
 *
 * The chunk-boundary state seeds the next chunk ("KDA Technical Deep Dive",
 * §Systems and implementation tradeoffs, Training), and the chunked recurrence
 * is linear in (values, starting state).  So a segment of the sequence run
 * from a zero state gives its outputs and final state up to the contribution
 * of the true starting state S_in, which enters as
 *     final = local_final + P S_in,    out += (outputs of S_in propagated alone),
 * with P [dk, dk] the segment's transfer (its state map with zero values).  The
 * associative combination of these affine transfers across segments is the
 * "associative scan" the deep dive mentions (same section).  With segments
 * 0..R-1 in time order (on one device or one per rank): run
 * kda_segment_local on each (segment 0 with the sequence's initial state),
 * exchange the (transfer, local_final) pairs, then for each segment r >= 1
 * compute its start with kda_segment_start_state over segments 0..r-1 and
 * finish it with kda_segment_correct.  bf16 inputs, dk = dv = 128.
 *
 * kda_segment_local -- outputs `out` and `local_final` of the segment from
 *   `initial_state` (NULL = zero), and its `transfer` [B, H, dk, dk] fp32
 *   (16-byte aligned).  Other arguments as kda_forward_ws; the workspace must
 *   hold the whole segment (kda_segment_workspace_bytes) and must be passed
 *   unchanged to kda_segment_correct.  T >= 1.
 */
kda_status kda_segment_local(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             const float *initial_state, float *out, float *local_final, float *transfer,
                             int B, int T, int H, int dk, int dv,
                             kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes, void *stream);

/*
 * kda_segment_start_state -- the state entering segment R of a sequence from the
 * R earlier segments: start = F_0, then start = F_j + P_j start for j = 1..R-1,
 * where transfers = P [R][B, H, dk, dk] and local_finals = F [R][B, H, dk, dv]
 * (segment 0's F already includes the sequence's initial state; P_0 is not
 * read).  fp32; all pointers 16-byte aligned device memory.  R >= 1.
 */
kda_status kda_segment_start_state(const float *transfers, const float *local_finals, int R,
                                   float *start, int B, int H, int dk, int dv, void *stream);

/*
 * kda_segment_correct -- finish a segment given its true start state: adds the
 * outputs of `start` propagated through the segment to `out` (the segment's
 * local outputs) and writes final_state = local_final + the propagated start
 * (NULL = not written).  Reads the chunk records kda_segment_local left in
 * `workspace` (same B, T, H); q, k, v are not needed again.
 */
kda_status kda_segment_correct(const float *start, const float *local_final, float *out, float *final_state,
                               int B, int T, int H, int dk, int dv,
                               const void *workspace, size_t workspace_bytes, void *stream);

/*
 * kda_forward_noalloc -- kda_forward on the two-kernel prefill with scratch that
 * belongs to the library, so that the call allocates nothing and needs no
 * workspace from the caller.
 *
 * The pages have no counterpart to this call: they describe no memory
 * management.  It computes exactly what kda_forward computes, with the same
 * arguments, layouts, statuses and aliasing rules.  The scratch is a fixed
 * 128 MiB array in the library's device image (kda_forward_noalloc_scratch_bytes),
 * so the sequence runs in blocks of as many 64-token chunks as fit it (results
 * are bit-identical to kda_forward_ws with a workspace of that size).  When a
 * single chunk of every (b, h) plus the carried state does not fit, and for
 * other dtypes or head dimensions, the call runs the one-kernel prefill
 * (kda_forward_ws with no workspace).  Calls that use the
 * scratch on one device are ordered by the library (an event per device), on
 * any streams; they run one after another.
 */
kda_status kda_forward_noalloc(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               const float *initial_state, float *out, float *final_state,
                               int B, int T, int H, int dk, int dv,
                               kda_dtype dtype, float scale, void *stream);

/* Size in bytes of the scratch kda_forward_noalloc uses on each device. */
size_t kda_forward_noalloc_scratch_bytes(void);

/*
 * The workspace pool of kda_forward and kda_gdn_forward on the current device.
 *
 * kda_workspace_pool_bytes -- device memory the pool holds now (in use by
 *   calls in flight or kept for the next ones); 0 before the first call.
 * kda_workspace_pool_trim -- waits for the work enqueued on `stream`, then
 *   returns to the device every byte of the pool that no call still uses
 *   (workspaces of calls in flight on other streams stay).  A later call
 *   takes memory again.  KDA_OK when there is no pool yet.
 */
size_t kda_workspace_pool_bytes(void);
kda_status kda_workspace_pool_trim(void *stream);

/*
 * kda_decode_step -- one token per sequence, state updated in place.
 *
 * The per-token update and query-state product of the decode path, whose cost
 * does not depend on how many tokens came before ("KDA Technical Deep Dive",
 * §Systems and implementation tradeoffs, Decoding; the state is updated in
 * place, §How the Kimi gate changes memory).
 *
 *   q, k          [B, H, dk]     dtype     (16-byte aligned)
 *   v             [B, H, dv]     dtype     (16-byte aligned)
 *   log_alpha     [B, H, dk]     float32   (16-byte aligned)
 *   beta          [B, H]         float32
 *   state_inout   [B, H, dk, dv] float32   (16-byte aligned), read and overwritten
 *   out           [B, H, dv]     float32   (16-byte aligned)
 *
 * Equivalent to kda_forward with T = 1 and final_state == initial_state.
 * Supported head dimensions: dk, dv in {64, 128}.  All pointers are required.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           float *state_inout, float *out,
                           int B, int H, int dk, int dv,
                           kda_dtype dtype, float scale, void *stream);

/*
 * kda_gdn_forward -- chunked prefill of the scalar-gate members of the family:
 * Gated DeltaNet (one decay per token and head) and DeltaNet (no decay).
 *
 * The token step is KDA's with Diag(alpha_t) replaced by a scalar alpha_t that
 * decays every key channel alike ("Kimi Delta Attention: The Linear Attention
 * Behind Kimi K2 and Qwen3", §DeltaNet, Gated DeltaNet, and KDA, comparison
 * table, and the FAQ entry on how Gated DeltaNet and KDA differ), or with no
 * decay at all (the delta rule of "KDA Technical Deep Dive", §From attention
 * to recurrent state (delta rule)).  KDA with every channel of log_alpha equal
 * to the scalar gives the same result.
 *
 *   q, k          [B, T, H, dk]  dtype            (16-byte aligned)
 *   v             [B, T, H, dv]  dtype            (16-byte aligned)
 *   log_alpha     [B, T, H]      float32 or NULL  (4-byte aligned; NULL = DeltaNet, alpha = 1)
 *   beta          [B, T, H]      float32          (4-byte aligned)
 *   initial_state, out, final_state: as for kda_forward.
 *
 * log_alpha must be finite and <= 0 (alpha in (0, 1]).  Everything else --
 * sizes, head dimensions, aliasing, T = 0, statuses, the pooled workspace and
 * the one-kernel fallback -- is as for kda_forward.
 */
kda_status kda_gdn_forward(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *initial_state, float *out, float *final_state,
                           int B, int T, int H, int dk, int dv,
                           kda_dtype dtype, float scale, void *stream);

/*
 * kda_gdn_forward_ws -- kda_gdn_forward with a caller-provided device workspace,
 * as kda_forward_ws is to kda_forward: bf16 with dk = dv = 128 and a workspace of
 * at least kda_forward_workspace_min_bytes(B, T, H, dk, dv, dtype) bytes (256-byte
 * aligned) take the two-kernel prefill: chunk records from a chunk-local kernel of
 * the scalar gate's own, in which the per-token decay factors out of every
 * product, and the per-head chain's scalar-gate form; anything else runs the
 * one-kernel scalar-gate prefill, which needs no device memory beyond its
 * arguments.  Same arguments, statuses and results as kda_gdn_forward.
 */
kda_status kda_gdn_forward_ws(const void *q, const void *k, const void *v,
                              const float *log_alpha, const float *beta,
                              const float *initial_state, float *out, float *final_state,
                              int B, int T, int H, int dk, int dv,
                              kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * kda_gdn_decode_step -- one token per sequence of the scalar-gate variants,
 * state updated in place.
 *
 *   log_alpha     [B, H]  float32 or NULL  (4-byte aligned; NULL = DeltaNet)
 *   every other argument as for kda_decode_step.
 *
 * Equivalent to kda_gdn_forward with T = 1 and final_state == initial_state.
 */
kda_status kda_gdn_decode_step(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               float *state_inout, float *out,
                               int B, int H, int dk, int dv,
                               kda_dtype dtype, float scale, void *stream);

/*
 * kda_forward_host -- kda_forward with every tensor argument in HOST memory.
 *
 * For a prefill whose activations live on the host (no counterpart on the
 * pages): the sequence is cut into blocks of block_tokens tokens (a multiple of
 * 64; 0 = 8192) that carry the state, and the library overlaps the host-to-device
 * copy of block i + 1, the kernels of block i and the device-to-host copy of
 * block i - 1, with two internal copy streams.  The chunk boundaries are those of
 * the whole sequence, so the results equal kda_forward_ws's bit for bit.
 *
 *   q, k, v, log_alpha, beta, initial_state (NULL = zero), out, final_state (NULL
 *                 = not wanted): host buffers in kda_forward's layouts (page-locked
 *                 memory lets the copies run asynchronously)
 *   workspace     device buffer of kda_forward_host_workspace_bytes(...) bytes
 *                 (256-byte aligned, caller-owned): two input slots and two output
 *                 slots of one block, the carried state, one block's chunk records
 *
 * The kernels run on `stream`, which also waits for the last copy: synchronise it
 * before reading out / final_state or reusing the host inputs.  Supported shapes,
 * statuses and dispatch as for kda_forward_ws (per-channel gate).  T = 0 copies
 * (or zeroes) the final state on the host and returns.
 */
kda_status kda_forward_host(const void *q, const void *k, const void *v,
                            const float *log_alpha, const float *beta,
                            const float *initial_state, float *out, float *final_state,
                            int B, int T, int H, int dk, int dv,
                            kda_dtype dtype, float scale, int block_tokens,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes kda_forward_host needs for these sizes and block length (0 for
 * invalid arguments). */
size_t kda_forward_host_workspace_bytes(int B, int T, int H, int dk, int dv, kda_dtype dtype, int block_tokens);

/*
 * kda_backward -- gradients of kda_forward with respect to every input.
 *
 * The pages give the forward's token step ("Kimi Delta Attention: The Linear
 * Attention Behind Kimi K2 and Qwen3", §How Kimi Delta Attention works step by
 * step) and name chunkwise training ("KDA Technical Deep Dive", §Systems and
 * implementation tradeoffs, Training) but print no gradient; this call returns
 * the exact derivative of that step (no counterpart on the pages).  With the
 * loss L = sum(out * grad_out) + sum(final_state * grad_final_state):
 *
 *   q, k          [B, T, H, dk]  dtype    (16-byte aligned)   forward inputs, as for kda_forward
 *   v             [B, T, H, dv]  dtype    (16-byte aligned)
 *   log_alpha     [B, T, H, dk]  float32  (16-byte aligned)
 *   beta          [B, T, H]      float32  (4-byte aligned)
 *   initial_state [B, H, dk, dv] float32  (16-byte aligned) or NULL (zero state)
 *   grad_out      [B, T, H, dv]  float32  (16-byte aligned)   dL/d out
 *   grad_final_state [B, H, dk, dv] float32 or NULL (zero)    dL/d final_state
 *   grad_q, grad_k [B, T, H, dk], grad_v [B, T, H, dv], grad_log_alpha [B, T, H, dk]:
 *                  float32 outputs (16-byte aligned), overwritten
 *   grad_beta     [B, T, H]      float32 output (4-byte aligned), overwritten
 *   grad_initial_state [B, H, dk, dv] float32 output or NULL (not wanted)
 *   workspace     device buffer of kda_backward_workspace_bytes(B, T, H, dk, dv)
 *                 bytes (256-byte aligned), caller-owned; holds the forward state
 *                 before every 8th token and the adjoint at the end of every
 *                 chunk of 64 tokens
 *
 * Supported: dk = dv in {64, 128}, bf16 or fp32 inputs; fp32 arithmetic on CUDA
 * cores (KDA_ERR_UNSUPPORTED otherwise).  Every buffer is caller-owned device
 * memory; nothing is allocated.  The outputs may not alias the inputs.  T = 0
 * writes grad_initial_state = grad_final_state (or zeros) and nothing else.
 * Bad pointers, sizes, dtype or scale -> KDA_ERR_INVALID_ARG; misaligned ->
 * KDA_ERR_MISALIGNED; a workspace below the size -> KDA_ERR_INVALID_ARG; launch
 * failures -> KDA_ERR_CUDA.  Asynchronous on `stream`; deterministic.
 */
kda_status kda_backward(const void *q, const void *k, const void *v,
                        const float *log_alpha, const float *beta, const float *initial_state,
                        const float *grad_out, const float *grad_final_state,
                        float *grad_q, float *grad_k, float *grad_v, float *grad_log_alpha,
                        float *grad_beta, float *grad_initial_state,
                        int B, int T, int H, int dk, int dv,
                        kda_dtype dtype, float scale, void *workspace, size_t workspace_bytes,
                        void *stream);

/* Workspace bytes kda_backward needs: (ceil(T / 8) + ceil(T / 64)) * B * H *
 * dk * dv * 4 (0 for unsupported shapes). */
size_t kda_backward_workspace_bytes(int B, int T, int H, int dk, int dv);

/* Static, human-readable name of a status code (never NULL). */
const char *kda_status_string(kda_status status);

/*
 * kda_check_status -- synchronise `stream`, then report (and clear) any
 * device-side failure the library's kernels recorded on the current device:
 * KDA_ERR_TIMEOUT if a bounded wait gave up, KDA_ERR_CUDA if the stream
 * reports an error, else KDA_OK.
 */
kda_status kda_check_status(void *stream);

/*
 * kda_selftest_timeout -- exercise the failure detection without a fault.
 *
 * Enqueues one small kernel whose bounded wait on a barrier that nothing
 * completes gives up after about wait_ms milliseconds (1..10000; else
 * KDA_ERR_INVALID_ARG) and records the device-side status that the prefill
 * kernels record when one of their waits gives up; the next kda_check_status
 * then returns KDA_ERR_TIMEOUT and clears it.  The device context stays usable.
 * The pages have no counterpart; this exists to test the failure path.
 */
kda_status kda_selftest_timeout(unsigned int wait_ms, void *stream);

/* Text of the last CUDA error seen by a kda_* call on this host thread
 * ("" if none).  The pointer stays valid until the next kda_* call on the
 * same thread. */
const char *kda_last_cuda_error(void);

/* Number of kernels this process has enqueued through libkda so far (all
 * devices, all threads).  Meant for accounting: a caller reads it before and
 * after a region to count the library's launches inside it. */
unsigned long long kda_launch_count(void);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
