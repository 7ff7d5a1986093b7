/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention forward library.
 *
 * The chunkwise forward (prefill) pass of Kimi Delta Attention, i.e. for every
 * sequence and head the recurrence of the Kimi Linear feature page (chapter 4,
 * "innovation 2", state-update equation)
 *
 *     S_t = (Diag(alpha_t) - beta_t k_t (k_t (.) alpha_t)^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t,          alpha_t = exp(g_t) per key channel,
 *
 * with a 128 x 128 state per head (rows: key channels, columns: value
 * channels), evaluated in chunks of 64 tokens. The library interface follows
 * the FlashKDA README summary (GitHub trending page, "kernel API and
 * constraints"): query, key, value, gate, beta tensors, head dims K = V = 128
 * only, variable-length packing through cu_seqlens with batch 1, and optional
 * bf16 or fp32 initial / final states whose dtypes must match when both are
 * given. A single-token step of the same recurrence for a batch of requests
 * (decode) is kda_decode.
 *
 * Conventions for every entry point below:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device, owned
 *    by the caller; the library keeps no reference after the call returns.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *    stream) and runs asynchronously: no host synchronisation happens inside.
 *  - Argument errors are detected before anything is enqueued and returned as
 *    a kda_status; nothing is written then. Launch failures return
 *    KDA_ERR_CUDA (the CUDA error is left for cudaGetLastError()).
 *  - kda_fwd allocates, on its first call on each device, one 123 MiB scratch
 *    pool (the operand-set rings of its kernel, 256 x 492 KiB) and holds it for
 *    the life of the process; later calls allocate nothing. kda_fwd_noalloc
 *    never allocates (see there).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kda_stream_t; /* same type as cudaStream_t */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_NULL_PTR = 1,          /* a required pointer is NULL                         */
    KDA_ERR_BAD_SHAPE = 2,         /* head dims != 128, negative sizes, H < 1, ...       */
    KDA_ERR_VARLEN_BATCH = 3,      /* cu_seqlens given with batch != 1                   */
    KDA_ERR_STATE_DTYPE = 4,       /* state dtype not bf16/fp32, or initial != final     */
    KDA_ERR_CUDA = 5,              /* a CUDA call failed (launch, attribute, device query) */
    KDA_ERR_UNSUPPORTED_DEVICE = 6,/* the current device is not sm_100 (B200 class)      */
    KDA_ERR_BAD_ALIGNMENT = 7,     /* a tensor pointer is not 16-byte aligned            */
    KDA_ERR_TOO_LARGE = 8,         /* sizes exceed what the library indexes              */
    KDA_ERR_TIMEOUT = 9,           /* a kernel gave up on a bounded wait (see kda_device_error) */
    KDA_ERR_NOALLOC_LIMIT = 10,    /* kda_fwd_noalloc: more (sequence, head) pairs than its scratch holds */
    KDA_ERR_STATE_OVERLAP = 11,    /* kda_decode: distinct state_in and state_out buffers overlap */
    KDA_ERR_BAD_CU_SEQLENS = 12,   /* (kda_device_error) cu_seqlens was not 0, ..., seq_len non-decreasing */
    KDA_ERR_INTERNAL = 13,         /* (kda_device_error) a kernel ran where its scratch has no slot for it */
    KDA_ERR_BAD_OPTION = 14,       /* kda_fwd_ex: unknown gate kind or flag bit */
    KDA_ERR_WORKSPACE = 15         /* kda_fwd_segmented: workspace smaller than it needs */
} kda_status;

typedef enum { KDA_DTYPE_NONE = 0, KDA_DTYPE_BF16 = 1, KDA_DTYPE_FP32 = 2 } kda_dtype;

/*
 * kda_fwd -- chunkwise KDA forward over a batch of independent sequences.
 *
 * Layouts (row-major, innermost last, all contiguous):
 *   q, k, v  : bf16  [batch, seq_len, num_heads, 128]
 *   g        : fp32  [batch, seq_len, num_heads, 128]  log alpha, raw per token
 *              (not cumulative); the kernel applies no activation to it
 *   beta     : fp32  [batch, seq_len, num_heads]
 *   out      : bf16  [batch, seq_len, num_heads, 128]  (written)
 *   initial_state, final_state : [num_seqs_eff, num_heads, 128 (key), 128 (value)],
 *              value index fastest, dtype initial_dtype / final_dtype.
 * q and k are used as given (the kernel does not normalise them).
 *
 * Sequences:
 *   cu_seqlens == NULL : num_seqs_eff = batch, sequence b is row b (seq_len tokens).
 *   cu_seqlens != NULL : batch must be 1; cu_seqlens is a DEVICE int32 array of
 *                        num_seqs + 1 offsets into the seq_len packed tokens,
 *                        cu_seqlens[0] = 0, non-decreasing, last = seq_len;
 *                        num_seqs_eff = num_seqs. The table lives on the
 *                        device, so it is checked there: a malformed table
 *                        raises KDA_ERR_BAD_CU_SEQLENS in the device error word
 *                        (read by kda_device_error). Its entries are clamped
 *                        into [0, seq_len] and a decreasing pair is read as an
 *                        empty sequence, so the kernel still accesses no memory
 *                        out of bounds; the results are then unspecified.
 *                        Zero-length sequences are allowed: their final state
 *                        equals their initial state.
 *
 * State:
 *   initial_state == NULL (initial_dtype ignored) means zero initial states.
 *   final_state   == NULL (final_dtype ignored) means the final states are not
 *   written. A given state must be KDA_DTYPE_BF16 or KDA_DTYPE_FP32 and, when
 *   both are given, the two dtypes must be equal. The state is carried in fp32
 *   inside the kernel; a bf16 final state is rounded to nearest even.
 *
 * scale multiplies the output (o_t = scale * S_t^T q_t); callers normally
 * pass 1/sqrt(128).
 *
 * Gate range: g may be any value <= 0, including -inf (alpha = 0). A chunk in
 * which some channel decays by more than 2^-50 over a 16-token quarter takes a
 * slower path with one decay anchor per 16 tokens instead of one per chunk, and
 * on that path per-token log-decays below -10 count as -10 (alpha >= e^-10 =
 * 4.5e-5): a channel that keeps less than that of its state per token has
 * forgotten it to below the precision of its bf16 operands either way, and the
 * change in any state entry is at most e^-10 of the entry it decays.
 *
 * head_dim_k and head_dim_v must both be 128. All tensor pointers must be
 * 16-byte aligned (cu_seqlens 4-byte). Returns KDA_OK once the work is
 * enqueued.
 */
kda_status kda_fwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, float scale, const int32_t *cu_seqlens,
                   int32_t num_seqs, int32_t batch, int64_t seq_len, int32_t num_heads,
                   int32_t head_dim_k, int32_t head_dim_v, const void *initial_state,
                   kda_dtype initial_dtype, void *final_state, kda_dtype final_dtype,
                   void *out, kda_stream_t stream);

/*
 * kda_fwd_ex -- kda_fwd with the input variants of the same operator.
 *
 * The Kimi Linear feature page (chapter 4, "innovation 1") defines the forget
 * gate per channel and sets it against Gated DeltaNet's single decay per token
 * (the Kimi Delta Attention review page, "Kimi Delta Attention" section, makes
 * the same contrast). The workloads give q and k L2-normalised and g as a
 * log-sigmoid; these variants take those steps, or cheaper inputs, into the
 * kernel instead of a separate pass over HBM:
 *
 *   gate_kind  KDA_GATE_FP32        g fp32 [batch, seq_len, num_heads, 128] (kda_fwd)
 *              KDA_GATE_BF16        g bf16 [batch, seq_len, num_heads, 128]: 256 fewer
 *                                   bytes to read per token and head (1284 instead of 1540)
 *              KDA_GATE_SCALAR_FP32 g fp32 [batch, seq_len, num_heads]: one decay per token
 *                                   and head, the same on every channel (Gated DeltaNet);
 *                                   4-byte alignment suffices
 *   flags      KDA_FLAG_L2NORM_QK        q and k are divided by their L2 norm over the 128
 *                                        channels of each token and head (a zero vector
 *                                        stays zero) before use
 *              KDA_FLAG_GATE_LOGSIGMOID  g holds the gate's pre-activation x, and
 *                                        log alpha = logsigmoid(x) = -log(1 + e^-x)
 *
 * Everything else, and every status, is as for kda_fwd; an unknown gate_kind or
 * flag bit returns KDA_ERR_BAD_OPTION.
 */
#define KDA_GATE_FP32 0
#define KDA_GATE_BF16 1
#define KDA_GATE_SCALAR_FP32 2
#define KDA_FLAG_L2NORM_QK 1u
#define KDA_FLAG_GATE_LOGSIGMOID 2u
kda_status kda_fwd_ex(const void *q, const void *k, const void *v, const void *g, int32_t gate_kind,
                      const float *beta, float scale, const int32_t *cu_seqlens, int32_t num_seqs,
                      int32_t batch, int64_t seq_len, int32_t num_heads, int32_t head_dim_k,
                      int32_t head_dim_v, const void *initial_state, kda_dtype initial_dtype,
                      void *final_state, kda_dtype final_dtype, void *out, uint32_t flags,
                      kda_stream_t stream);

/*
 * kda_fwd_segmented -- kda_fwd over long sequences split into pieces that run at
 * once, for batches with few (sequence, head) pairs.
 *
 * The Kimi Linear feature page (chapter 8) keeps the state at a fixed 128 x 128
 * per head however long the context (1M tokens on the release page). kda_fwd runs
 * each (sequence, head) pair's chunks in order on one set of SMs, so a batch of few
 * pairs leaves most of the GPU idle. The recurrence is affine in the state: a piece
 * of a sequence maps its entering state S to M S + B. This entry point splits every
 * row into pieces of segment_len tokens and makes three launches on `stream`:
 *   1. every piece twice, with no output: from a zero state (giving B) and from the
 *      identity with v = 0 (giving M); all pieces of all rows at once;
 *   2. the scan S_0 = initial state, S_(j+1) = M_j S_j + B_j, per row and head;
 *   3. every piece again from its S_j, writing the outputs and, for the last piece,
 *      the row's final state.
 * That is about three times kda_fwd's work, done in parallel over the pieces: it
 * pays when batch * num_heads is small next to the number of SMs.
 *
 * Arguments and layouts are kda_fwd's for fixed-length rows (no cu_seqlens), plus:
 *   segment_len     tokens per piece, a positive multiple of 64; a row that fits in
 *                   one piece runs as in kda_fwd;
 *   workspace       caller-owned device memory, 256-byte aligned, of at least
 *                   kda_fwd_segmented_workspace(batch, seq_len, num_heads,
 *                   segment_len) bytes (three fp32 states per piece and head); its
 *                   contents on entry do not matter. KDA_ERR_WORKSPACE if smaller.
 * Results agree with kda_fwd's to the rounding of the bf16 state copies the
 * products use; the pieces' states are carried in fp32. A bad segment_len returns
 * KDA_ERR_BAD_SHAPE, and kda_fwd_segmented_workspace returns 0 for one.
 */
size_t kda_fwd_segmented_workspace(int32_t batch, int64_t seq_len, int32_t num_heads, int64_t segment_len);
kda_status kda_fwd_segmented(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, float scale, int32_t batch, int64_t seq_len,
                             int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v,
                             const void *initial_state, kda_dtype initial_dtype, void *final_state,
                             kda_dtype final_dtype, void *out, int64_t segment_len, void *workspace,
                             size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_bwd -- gradients of the chunkwise forward: of L = sum(dout . out) +
 * sum(dfinal_state . final_state) with respect to q, k, v, g, beta and the initial
 * state.
 *
 * The FlashKDA release page describes the library as forward and backward kernels
 * for KDA; this is the backward of kda_fwd's operator (the state-update equation of
 * the Kimi Linear feature page, chapter 4), for training. It runs the chunk form of
 * the recurrence backwards, last chunk first, in chunks of 16 tokens, in fp32: a
 * forward sweep stores the state entering every 64 tokens in `workspace`, and the
 * reverse sweep recomputes each chunk from its stored state.
 *
 * Inputs are kda_fwd's (q, k, v bf16, g fp32 log alpha per channel, beta fp32,
 * cu_seqlens, initial_state bf16/fp32/NULL, same layouts and rules) plus:
 *   dout           bf16 [batch, seq_len, num_heads, 128]: dL/d out
 *   dfinal_state   fp32 [num_seqs_eff, num_heads, 128, 128] or NULL (zero): dL/d final state
 * Outputs (fp32, written; every pointer 16-byte aligned, dbeta 4-byte):
 *   dq, dk, dv, dg [batch, seq_len, num_heads, 128];  dbeta [batch, seq_len, num_heads]
 *   dinitial_state [num_seqs_eff, num_heads, 128, 128], or NULL (not written)
 *   workspace      caller-owned device memory, 256-byte aligned, at least
 *                  kda_bwd_workspace(total_tokens, num_seqs_eff, num_heads) bytes
 *                  (64 KiB per 64 tokens per head, plus one state per sequence
 *                  and head); contents on entry do not matter.
 * total_tokens is batch * seq_len (seq_len with cu_seqlens). The gates are taken
 * as in kda_fwd's sub-block path: a per-token log-decay below -10 counts as -10,
 * and its gradient is 0. dq, dk, dg and dbeta gather four partial sums by fp32
 * atomic adds, so they can differ from run to run in the last bits.
 * KDA_ERR_WORKSPACE if the workspace is smaller than needed.
 */
size_t kda_bwd_workspace(int64_t total_tokens, int32_t num_seqs, int32_t num_heads);
kda_status kda_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta, float scale,
                   const int32_t *cu_seqlens, int32_t num_seqs, int32_t batch, int64_t seq_len, int32_t num_heads,
                   int32_t head_dim_k, int32_t head_dim_v, const void *initial_state, kda_dtype initial_dtype,
                   const void *dout, const float *dfinal_state, float *dq, float *dk, float *dv, float *dg,
                   float *dbeta, float *dinitial_state, void *workspace, size_t workspace_bytes,
                   kda_stream_t stream);

/*
 * kda_fwd_noalloc -- kda_fwd for callers that cannot allocate device memory.
 *
 * The method's pages define no such call; it exists for the library's own
 * callers. Some cannot let a library allocate: a process whose device memory is
 * handed out entirely by its own pool or by a framework's caching allocator, a
 * caller that must keep its memory footprint fixed once it has started serving,
 * or code that enqueues work where an allocation would stall or be refused.
 * kda_fwd's scratch pool is allocated on its first call on a device; this entry
 * point uses instead a scratch array that is part of the library's device image
 * (KDA_NOALLOC_MAX_UNITS operand-set rings, 15.4 MiB, present once the library's
 * kernels are loaded on the device), and calls no allocating routine at all.
 *
 * Arguments, layouts, results and status codes are those of kda_fwd, plus:
 *  - num_seqs_eff * num_heads must not exceed KDA_NOALLOC_MAX_UNITS (32): one
 *    ring of the scratch per (sequence, head) pair. A larger call returns
 *    KDA_ERR_NOALLOC_LIMIT before anything is enqueued; split it, or use kda_fwd.
 *  - The first call on each device looks up the scratch's device address (the
 *    device must be current; a failed lookup returns KDA_ERR_CUDA) and may load
 *    the library's kernels onto the device. Make that first call before any
 *    stream capture begins.
 *  - The scratch is shared by every call on a device: two kda_fwd_noalloc calls
 *    whose work overlaps in time (on different streams, or from different host
 *    threads without ordering) race on it and give wrong results. Order them on
 *    one stream, or use kda_fwd, whose kernels never share a ring.
 *  - Nothing in the scratch needs to start at zero, and the call clears nothing:
 *    every ring slot is written by the kernel before the kernel reads it.
 */
#define KDA_NOALLOC_MAX_UNITS 32
kda_status kda_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, float scale, const int32_t *cu_seqlens,
                           int32_t num_seqs, int32_t batch, int64_t seq_len, int32_t num_heads,
                           int32_t head_dim_k, int32_t head_dim_v, const void *initial_state,
                           kda_dtype initial_dtype, void *final_state, kda_dtype final_dtype,
                           void *out, kda_stream_t stream);

/*
 * kda_decode -- one recurrent step (a single new token) for a batch of
 * independent requests, each with its own state per head.
 *
 * For every request b and head h this is the state-update equation above for
 * one token, with the output read from the updated state (as in kda_fwd):
 *     S <- (Diag(alpha) - beta k (k (.) alpha)^T) S + beta k v^T,   o = scale * S^T q,
 * alpha = exp(g) per key channel. kda_fwd over a sequence of length 1 with an
 * initial and a final state computes the same thing; this entry point exists
 * because a decode step is bound by reading and writing the 128 x 128 state,
 * which it does once, with no chunk machinery. The pages describe the step (the
 * decode-speed claims of the Kimi Linear feature page) but define no such call.
 *
 * Layouts (row-major, innermost last, all contiguous):
 *   q, k, v  : bf16 [batch, num_heads, 128]
 *   g        : fp32 [batch, num_heads, 128]  log alpha (raw, no activation)
 *   beta     : fp32 [batch, num_heads]
 *   out      : bf16 [batch, num_heads, 128]  (written)
 *   state_in, state_out : [batch, num_heads, 128 (key), 128 (value)], value
 *              index fastest, dtype state_dtype (KDA_DTYPE_BF16 or _FP32).
 *   state_in  == NULL means zero states; state_out == NULL means the updated
 *   states are not written. state_out may be the same pointer as state_in (the
 *   step then updates the states in place); distinct buffers that overlap are
 *   refused with KDA_ERR_STATE_OVERLAP.
 * The state is carried in fp32 inside the step; a bf16 state is rounded to
 * nearest even when written. head_dim_k and head_dim_v must both be 128; all
 * tensor pointers must be 16-byte aligned (beta 4-byte). batch == 0 is a no-op.
 * Nothing is allocated. Returns KDA_OK once the work is enqueued.
 */
kda_status kda_decode(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float scale, int32_t batch, int32_t num_heads,
                      int32_t head_dim_k, int32_t head_dim_v, const void *state_in,
                      void *state_out, kda_dtype state_dtype, void *out, kda_stream_t stream);

/*
 * kda_device_error -- synchronise the current device, then read and clear the
 * library's device-side error word, which the kernels raise instead of
 * faulting or hanging. Since the previous call on this device, if any kernel:
 *  - found cu_seqlens malformed (see kda_fwd): KDA_ERR_BAD_CU_SEQLENS;
 *  - gave up on a bounded wait (every wait is bounded, a few seconds) and
 *    returned early, leaving its outputs unspecified: KDA_ERR_TIMEOUT;
 *  - ran a chain CTA on an SM id beyond the scratch pool's rings (none exists
 *    on a B200) and returned at once: KDA_ERR_INTERNAL;
 * the first of these in this order is returned, else KDA_OK; KDA_ERR_CUDA if
 * the device could not be synchronised or read.
 */
kda_status kda_device_error(void);

/* Human-readable name of a status code (static storage, never NULL). */
const char *kda_status_string(kda_status status);

/* Library ABI version, (major << 16) | minor. */
int32_t kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
