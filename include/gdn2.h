/*
 * gdn2.h -- C ABI of libgdn2, the sm_100a (B200) implementation of the Gated DeltaNet-2
 * state recurrence.
 *
 * The operation (per sequence n and value head h; tokens t in order):
 *   S'_t = Diag(alpha_t) S_{t-1},  alpha_t = exp(log_alpha_t)     channel-wise decay, key axis
 *   r_t  = S'_t^T k_t                                              key read of the old state
 *   S_t  = S'_t - (b_t (.) k_t) r_t^T + k_t (w_t (.) v_t)^T        erase (key axis), write (value axis)
 *   o_t  = S_t^T q_t                                               query read of the updated state
 * Sources: the tilnote.io note on Gated DeltaNet-2, section "Gated DeltaNet-2 design
 * point" (a channel-wise erase gate b_t on the key axis, a channel-wise write gate w_t on
 * the value axis, the KDA channel-wise decay; decay, then remove the key-side component,
 * then add the value-side component); the ai-systems-engineering.com post "Delta rule:
 * correcting the state's associations toward the new Value", sections "Why read with the
 * Key, why with the Query" and "Recording the difference between the read value and the
 * new Value" (key read before the edit, query read after it, r^T = k^T S, rows of S are
 * key channels and columns value channels); the Gated DeltaNet wiki page
 * (aiki.softdaddy-o.com), section "How it works" (query/key heads shared by groups of
 * value heads). No scale is applied to q.
 *
 * Layouts (row-major, innermost index last, every tensor contiguous):
 *   q, k        [T_total, h_qk, dk]   dtype
 *   v, w        [T_total, h_v,  dv]   dtype
 *   o           [T_total, h_v,  dv]   o_dtype
 *   log_alpha   [T_total, h_v,  dk]   float32
 *   b           [T_total, h_v,  dk]   dtype
 *   S0, S_T, S  [n_seq, h_v, dk, dv]  float32 (dv contiguous)
 *   cu_seqlens  [n_seq + 1] int32     packed sequence offsets (0, ..., T_total)
 * dtype GDN2_BF16 means bfloat16, GDN2_F32 float32. o_dtype is chosen separately: a bf16
 * output carries a rounding error of up to 2^-8 |o| per element, which for these
 * recurrences (max|o| / rms(o) of 10 to 15) alone exceeds 2e-2 of rms(o); GDN2_F32 output
 * keeps the result within the kernels' arithmetic error.
 * Value head h reads query/key head h / (h_v / h_qk).
 *
 * Ownership: every tensor pointer is a device pointer owned by the caller and must stay
 * valid until the work queued on `stream` has finished. The library allocates no device
 * memory. Calls are asynchronous on `stream` (0 = the legacy default stream); nothing is
 * synchronised.
 *
 * Errors: arguments are checked on the host before anything is queued. A rejected call
 * queues nothing and returns GDN2_ERR_INVALID_ARG (bad pointer, size, alignment,
 * layout) or GDN2_ERR_UNSUPPORTED (a valid shape these kernels do not handle); a
 * failed launch returns GDN2_ERR_CUDA. gdn2_last_error_string() describes the last
 * failure of the calling thread. Nothing is thrown or aborted across the ABI.
 *
 * Supported: dk, dv in {64, 128}; h_v a multiple of h_qk; 1 <= n_seq <= 65535,
 * h_v <= 65535 and n_seq * h_v <= 2^31 - 1; every pointer 16-byte aligned.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN2_API __attribute__((visibility("default")))
#else
#define GDN2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gdn2_stream_t; /* a cudaStream_t */

typedef enum { GDN2_F32 = 0, GDN2_BF16 = 1 } gdn2_dtype;

typedef enum {
    GDN2_OK = 0,
    GDN2_ERR_INVALID_ARG = 1,
    GDN2_ERR_UNSUPPORTED = 2,
    GDN2_ERR_CUDA = 3
} gdn2_status;

typedef struct {
    int n_seq;        /* sequences in the batch (>= 1) */
    int T_total;      /* packed tokens over all sequences (>= 0) */
    int h_qk;         /* query/key heads */
    int h_v;          /* value heads (a multiple of h_qk) */
    int dk;           /* key channels per head: 64 or 128 */
    int dv;           /* value channels per head: 64 or 128 */
    gdn2_dtype dtype;   /* element type of q, k, v, b, w */
    gdn2_dtype o_dtype; /* element type of o */
} gdn2_shape;

/*
 * Bytes of device workspace gdn2_chunk_fwd needs for this shape and cu_seqlens choice
 * (varlen = 1 when a cu_seqlens pointer will be passed). 0 means no workspace.
 */
GDN2_API size_t gdn2_chunk_fwd_workspace_size(const gdn2_shape* shape, int varlen);

/*
 * Prefill over whole sequences (chunkwise-parallel; the recurrence above for every
 * token). Sequences are packed by cu_seqlens; with cu_seqlens == NULL, T_total must be a
 * multiple of n_seq and sequence n is tokens [n*T, (n+1)*T), T = T_total / n_seq.
 * S0 == NULL starts every sequence from a zero state. S_T == NULL skips the final state.
 * S_T may be S0 itself (the states are then updated in place); no other output may overlap
 * an input. A zero-length sequence writes S_T = S0 (or 0) and no output.
 * workspace: device memory of at least gdn2_chunk_fwd_workspace_size() bytes, 256-byte
 * aligned, owned by the caller, reused freely after the call's work completes; may be
 * NULL when that size is 0.
 */
GDN2_API gdn2_status gdn2_chunk_fwd(const gdn2_shape* shape,
                           const void* q, const void* k, const void* v,
                           const float* log_alpha, const void* b, const void* w,
                           const float* S0, const int32_t* cu_seqlens,
                           void* o, float* S_T,
                           void* workspace, size_t workspace_bytes,
                           gdn2_stream_t stream);

/*
 * One decode step: one new token for each of the n_seq sequences (shape->T_total must
 * equal shape->n_seq; token n belongs to sequence n). The state S [n_seq, h_v, dk, dv] is
 * read and updated in place; o receives the query read of the updated state.
 */
GDN2_API gdn2_status gdn2_decode_step(const gdn2_shape* shape,
                             const void* q, const void* k, const void* v,
                             const float* log_alpha, const void* b, const void* w,
                             float* S, void* o, gdn2_stream_t stream);

/*
 * Serving-style decode: n_tok (1..GDN2_DECODE_MAX_TOKENS) new tokens for each of the n_seq
 * sequences, whose states live in a pool. The same recurrence as gdn2_decode_step, token
 * after token; the pages describe single-token decode only, and the slot pool and the
 * multi-token step are interface choices for continuous batching and for verifying
 * drafted tokens.
 *   shape->T_total must equal n_seq * n_tok; token t of sequence n is row n * n_tok + t of
 *   q, k, v, log_alpha, b, w and o (layouts as above).
 *   S_pool [n_slots, h_v, dk, dv] float32: sequence n reads and updates, in place, the state
 *   in slot slots[n] (slots: device int32 [n_seq]; NULL means slot n, and then n_slots must
 *   be at least n_seq). A sequence whose slot is negative or >= n_slots is skipped: its
 *   rows of o are not written and no state is touched. Two active sequences must not share
 *   a slot (they would race).
 *   S_steps (nullable) [n_seq, n_tok, h_v, dk, dv] float32 receives the state after each
 *   token, so that a caller that accepts only the first j drafted tokens can put back the
 *   state after token j - 1 (S_pool itself always ends after all n_tok tokens).
 * Errors as for the other calls; slot values are only checked on the device (skipped).
 * GDN2_ERR_UNSUPPORTED if n_slots * h_v * dk exceeds 2^31 - 1 (the pool's state rows are
 * addressed as 32-bit coordinates). With n_tok > 1 (or S_steps given) each state is
 * loaded by TMA and its wait is bounded like the prefill's (GDN2_DEVICE_WAIT_TIMEOUT).
 */
#define GDN2_DECODE_MAX_TOKENS 8
GDN2_API gdn2_status gdn2_decode_multi(const gdn2_shape* shape, int n_tok, const int32_t* slots,
                              const void* q, const void* k, const void* v,
                              const float* log_alpha, const void* b, const void* w,
                              float* S_pool, int n_slots, void* o, float* S_steps,
                              gdn2_stream_t stream);

/*
 * gdn2_decode_multi with the pre-processing of gdn2_chunk_fwd_prologue fused in (raw q, k,
 * b, w; a_raw in dtype in place of log_alpha). Any dk, dv of the decode kernel.
 */
GDN2_API gdn2_status gdn2_decode_multi_prologue(const gdn2_shape* shape, int n_tok, const int32_t* slots,
                                       const void* q_raw, const void* k_raw, const void* v,
                                       const void* a_raw, const void* b_raw, const void* w_raw,
                                       float* S_pool, int n_slots, void* o, float* S_steps,
                                       gdn2_stream_t stream);

/*
 * Prefill with the pre-processing fused in: the inputs are raw projections, and the kernel
 * applies, in fp32, per token and head,
 *   q = q_raw / max(|q_raw|_2, 1e-12), k = k_raw / max(|k_raw|_2, 1e-12)   (over dk)
 *   log_alpha = -softplus(a_raw) = -log(1 + e^a_raw)                        (per key channel)
 *   b = sigmoid(b_raw), w = sigmoid(w_raw)
 * before the recurrence above. Unit-length keys are what the delta-rule post
 * (ai-systems-engineering.com, section on the correction strength beta) needs for the
 * correction to land exactly, and gates computed from the input are what it describes; the
 * activation functions themselves are not on the pages (softplus and sigmoid are the
 * reading adopted). a_raw has dtype (not float32) and log_alpha's layout [T_total, h_v, dk];
 * q_raw, k_raw, b_raw, w_raw replace q, k, b, w with the same layouts. Otherwise as
 * gdn2_chunk_fwd (same workspace). Supported for bf16 inputs with dk = dv = 128 (else
 * GDN2_ERR_UNSUPPORTED).
 */
GDN2_API gdn2_status gdn2_chunk_fwd_prologue(const gdn2_shape* shape,
                                    const void* q_raw, const void* k_raw, const void* v,
                                    const void* a_raw, const void* b_raw, const void* w_raw,
                                    const float* S0, const int32_t* cu_seqlens,
                                    void* o, float* S_T,
                                    void* workspace, size_t workspace_bytes,
                                    gdn2_stream_t stream);

/*
 * Gradients of the recurrence for the loss L = sum(o * dO) + sum(S_T * dS_T): given the
 * forward's inputs (as for gdn2_chunk_fwd) and dO [T_total, h_v, dv] float32 (dS_T nullable,
 * [n_seq, h_v, dk, dv] float32), writes, all float32 and in the inputs' layouts,
 *   dq, dk [T_total, h_qk, dk]  (a query/key head sums over the value heads that read it)
 *   dv, dw [T_total, h_v, dv];  dlog_alpha, db [T_total, h_v, dk]
 *   dS0 (nullable) [n_seq, h_v, dk, dv].
 * The pages describe the forward recurrence only (they state the model was trained, which
 * needs these); the derivation is the chain rule through the per-token update, in fp32.
 * One CTA runs per (sequence, value head), each warp owning 8 value columns of the state
 * in registers: a forward pass stores the state at every 8th token, then, from the end, each
 * 8-token sub-chunk's states are recomputed into a scratch area and its tokens walked
 * backwards.
 * workspace: device memory of gdn2_chunk_bwd_workspace_size(shape) bytes, 256-byte
 * aligned (required). With h_v > h_qk, dq and dk are zeroed on the stream and accumulated
 * with atomics (the order of those additions varies from run to run).
 * Any dtype and dk, dv in {64, 128}.
 */
GDN2_API size_t gdn2_chunk_bwd_workspace_size(const gdn2_shape* shape);
GDN2_API gdn2_status gdn2_chunk_bwd(const gdn2_shape* shape,
                           const void* q, const void* k, const void* v,
                           const float* log_alpha, const void* b, const void* w,
                           const float* S0, const int32_t* cu_seqlens,
                           const float* dO, const float* dS_T,
                           float* dq, float* dk, float* dv,
                           float* dlog_alpha, float* db, float* dw, float* dS0,
                           void* workspace, size_t workspace_bytes,
                           gdn2_stream_t stream);

/*
 * Prefill for callers that cannot allocate device memory. The pages have no counterpart:
 * this is an interface choice. It computes exactly what gdn2_chunk_fwd computes (same
 * kernels, same arguments, no workspace), for callers that have no way to give the
 * library scratch memory: code that owns no device allocator (a plug-in living inside
 * another runtime's memory pool), code that must not allocate after start-up (a serving
 * loop with a fixed memory budget), or code where a cudaMalloc would synchronise the
 * device at the wrong moment. The scratch that packed batches need (the longest-first
 * order of the sequences) lives in a 64 KB array inside the library image instead, held
 * by every GPU that loads the library until the process exits.
 * Limits: with cu_seqlens, at most 16384 sequences per call (more: GDN2_ERR_INVALID_ARG,
 * nothing queued). All calls on a device share that array; each call writes every entry
 * it reads, but calls whose work overlaps on the GPU (concurrent streams) race on it: such
 * an overlap can give wrong or missing results (a work item that meets an out-of-range
 * sequence index is skipped and flags GDN2_DEVICE_BAD_ORDER), but never writes outside
 * the caller's buffers. The
 * first call on each device looks the array up with that device current: make it before
 * any stream capture. Nothing is allocated by this call.
 */
GDN2_API gdn2_status gdn2_chunk_fwd_noalloc(const gdn2_shape* shape,
                                    const void* q, const void* k, const void* v,
                                    const float* log_alpha, const void* b, const void* w,
                                    const float* S0, const int32_t* cu_seqlens,
                                    void* o, float* S_T, gdn2_stream_t stream);

/*
 * Device-side status. The pages describe no interface, so this is an interface choice: some
 * errors can only be seen once the kernels run, after the call that queued them has
 * returned GDN2_OK. The kernels record them in a status word per device (bits below), and
 * gdn2_device_status waits for the work queued so far on `stream`, returns the bits set
 * since the previous gdn2_device_status on this device in *flags, and clears them. It
 * synchronises `stream` (0 = the legacy default stream); work queued on other streams is
 * covered once it has completed.
 *   GDN2_DEVICE_WAIT_TIMEOUT  a bounded wait inside the tensor-core prefill or the
 *                             multi-token decode ran out (4 s): that CTA released its
 *                             tensor memory (prefill) and returned without writing its rows
 *                             of o and its states, so the outputs of that call are
 *                             incomplete.
 *   GDN2_DEVICE_BAD_SEQLENS   cu_seqlens was not 0 = c_0 <= c_1 <= ... <= c_n = T_total.
 *                             Kernels clamp every sequence to [0, T_total], so nothing is
 *                             accessed out of bounds, but the results follow the clamped
 *                             ranges, not the caller's intent.
 *   GDN2_DEVICE_BAD_ORDER     a work item met a sequence index outside [0, n_seq) in the
 *                             packed-batch order (only possible when gdn2_chunk_fwd_noalloc
 *                             calls overlap on the GPU): that item was skipped, its outputs
 *                             are missing, and nothing was written out of bounds.
 *   GDN2_DEVICE_DECAY_RANGE   in the tensor-core prefill, some key channel's cumulative
 *                             log-decay varied by more than ~166 nats (e^(2 x 83)) within one
 *                             64-token chunk. The kernel scales each chunk's operands by
 *                             e^(+-(G - Gref)) around the chunk's mid-point, and beyond that
 *                             span the factors leave fp32's range; the CTA of that (sequence,
 *                             head) then recomputes its o and S_T token by token in fp32
 *                             within the same launch, from S0 (which it has not overwritten),
 *                             so the results are valid. The bit says that this slower route
 *                             ran (~1.1 us per token of the longest such pair, measured on
 *                             B200: 5.0 ms for 4096 tokens against 0.57 ms). A mean log_alpha of
 *                             -2.6 per token over a chunk reaches it.
 * Returns GDN2_ERR_CUDA if the stream or the copies fail.
 */
#define GDN2_DEVICE_WAIT_TIMEOUT 0x1u
#define GDN2_DEVICE_BAD_SEQLENS 0x2u
#define GDN2_DEVICE_BAD_ORDER 0x4u
#define GDN2_DEVICE_DECAY_RANGE 0x8u
GDN2_API gdn2_status gdn2_device_status(unsigned int* flags, gdn2_stream_t stream);

/*
 * Testing only: the limit of the bounded waits of the tensor-core prefill and of the
 * multi-token decode for later calls from any thread (wait_ns = 0 restores the default of
 * 4 s), and, when withhold_first_load is non-zero, a prefill whose producer never issues its
 * first loads and a multi-token decode that never issues its first state load. With a short
 * limit the waits then run out, the kernel records GDN2_DEVICE_WAIT_TIMEOUT and returns,
 * which lets a test check that path without any fault: nothing asynchronous is in flight
 * when the waits give up. Not for production use.
 */
GDN2_API void gdn2_testing_set_wait_limit(unsigned long long wait_ns, int withhold_first_load);

/* Description of the calling thread's last failure ("" if none). Never NULL. */
GDN2_API const char* gdn2_last_error_string(void);

/* Library version as major * 10000 + minor * 100 + patch. */
GDN2_API int gdn2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
