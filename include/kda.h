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
    KDA_ERR_STATE_OVERLAP = 11     /* kda_decode: distinct state_in and state_out buffers overlap */
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
 *                        num_seqs_eff = num_seqs. Entries are clamped into
 *                        [0, seq_len] and a decreasing pair is read as an empty
 *                        sequence, so a malformed table cannot make the kernel
 *                        access memory out of bounds (its results are then
 *                        unspecified). Zero-length sequences are allowed: their
 *                        final state equals their initial state.
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
 * library's device-side error word. Every wait inside the kernels is bounded
 * (a few seconds); a kernel that gives up raises this word and returns early
 * instead of hanging, leaving its outputs unspecified. Returns KDA_ERR_TIMEOUT
 * if that happened on this device since the previous call, KDA_OK otherwise,
 * KDA_ERR_CUDA if the device could not be synchronised or read.
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
