/*
 * infini_attn.h -- C ABI of the B200 (sm_100a) Infini-attention forward library.
 *
 * What is computed (AI Wiki "Infini-Attention", "What happens inside the Infini-attention
 * block?" and "How does the compressive memory work?"; the Hugging Face reproduction
 * analysis, "Infini-Attention Mechanism", steps 1-6):
 *
 *   The length-L sequence of every (batch b, query head h) is cut into segments of N
 *   tokens, processed in order; when N does not divide L the last segment is shorter
 *   (L mod N tokens) and is processed the same way, its update included.  For segment s
 *   and query row q_t:
 *     A_dot = causal softmax(q_t K_s^T / sqrt(d)) V_s     keys of segment s only, j <= t
 *     A_mem = sigma(q_t) M_{s-1} / (sigma(q_t) . z_{s-1}) sigma(x) = ELU(x) + 1; 0 while the
 *                                                          denominator is exactly 0
 *     out_t = g_h A_mem + (1 - g_h) A_dot                  g_h = 1 / (1 + exp(-beta[h]))
 *   After the segment the memory of its key/value head advances:
 *     linear: M_s = M_{s-1} + sigma(K_s)^T V_s
 *     delta : M_s = M_{s-1} + sigma(K_s)^T (V_s - sigma(K_s) M_{s-1} / (sigma(K_s) z_{s-1}))
 *             (one batch update per segment; a row whose denominator is 0 predicts 0)
 *     both  : z_s = z_{s-1} + sum_t sigma(K_{s,t})
 *   Query head h reads key/value head h / (H / Hkv) (grouped-query attention).
 *
 * Layouts: row-major, contiguous, on the device:
 *   q, out  [B, H,   L, d]        k, v  [B, Hkv, L, d]        beta [H] float
 *   M0, M_out [B, Hkv, d, d] float (row = key feature, column = value feature)
 *   z0, z_out [B, Hkv, d]    float
 *
 * Conventions shared by every entry point:
 *   - All pointers are DEVICE pointers owned by the caller; the library keeps none of them
 *     after the call returns.  Every pointer must be 16-byte aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 *     runs asynchronously: results are valid once that stream has synchronised.
 *   - M0 / z0 may be NULL (an empty memory: zeros).  M_out / z_out may alias M0 / z0
 *     exactly (in-place state update); a partial overlap is INFINI_ERR_INVALID_ARG.  out
 *     must not overlap any input.
 *   - Preconditions not checked: z0 >= 0 elementwise (sigma > 0 then makes a zero
 *     denominator mean an empty memory); inputs finite.
 *   - On an argument error nothing is launched and nothing is written.  Nothing aborts,
 *     throws or traps; every failure is an int status below.
 *   - Scratch: the call allocates its workspace (per-segment memory snapshots; the size
 *     is infini_attn_workspace_bytes) stream-ordered on `stream` from a memory pool the
 *     library owns on each device, and frees it on the same stream.  The pool keeps freed
 *     memory for the next call (up to the largest workspace used so far).
 */
#ifndef INFINI_ATTN_H
#define INFINI_ATTN_H

#include <stdint.h>

#if defined(__GNUC__)
#define INFINI_API __attribute__((visibility("default")))
#else
#define INFINI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *infini_stream_t;

enum {
    INFINI_UPDATE_LINEAR = 0, /* M += sigma(K)^T V                      */
    INFINI_UPDATE_DELTA = 1   /* M += sigma(K)^T (V - sigma(K) M / den) */
};

enum {
    INFINI_OK = 0,
    INFINI_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or position, bad rule,
                                   partial overlap of a state output with its input        */
    INFINI_ERR_UNSUPPORTED = 2, /* valid but not built: d not in {32, 64, 128}, N % 64 != 0 */
    INFINI_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed                      */
    INFINI_ERR_OOM = 4,         /* the workspace allocation failed                           */
    INFINI_ERR_TIMEOUT = 5      /* a bounded device wait gave up (infini_attn_device_status) */
};

/*
 * Infini-attention forward, bf16 activations (q, k, v, out are __nv_bfloat16; arithmetic
 * in fp32, memory M / z in fp32, out rounded to nearest-even).
 *
 *   B, H, Hkv : batch, query heads, key/value heads (H % Hkv == 0)
 *   L, N, d   : sequence length, segment length, head dimension (L need not be a
 *               multiple of N: the final L mod N tokens form a shorter last segment)
 *   update_rule : INFINI_UPDATE_LINEAR or INFINI_UPDATE_DELTA
 * Returns INFINI_OK or an error status.
 */
INFINI_API int infini_attn_fwd(const void *q, const void *k, const void *v, const float *beta,
                    const float *M0, const float *z0, void *out, float *M_out, float *z_out,
                    int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N, int64_t d,
                    int update_rule, infini_stream_t stream);

/* The same operation with fp32 activations (q, k, v, out are float); identical parameters. */
INFINI_API int infini_attn_fwd_f32(const void *q, const void *k, const void *v, const float *beta,
                        const float *M0, const float *z0, void *out, float *M_out,
                        float *z_out, int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N,
                        int64_t d, int update_rule, infini_stream_t stream);

/*
 * Backward pass: the gradients of  <dout, out> + <dM, M_out> + <dz, z_out>  of the forward
 * above (same q, k, v, beta, M0, z0, N, update rule) with respect to every input, through
 * the local attention, the retrieval, the gate and the memory recurrence of every segment
 * (AI Wiki "Infini-Attention", "How is an Infini-attention model trained?": gradients flow
 * through the memory from segment to segment).  A quotient whose denominator is 0 (an
 * empty memory) is 0 and passes no gradient.
 *
 *   dout [B, H, L, d] (activation dtype): gradient of out;  dM [B, Hkv, d, d], dz [B, Hkv, d]
 *     fp32: gradients of M_out, z_out (NULL = zero)
 *   dq [B, H, L, d], dk / dv [B, Hkv, L, d] (activation dtype), dbeta [H], dM0 [B, Hkv, d, d],
 *     dz0 [B, Hkv, d] fp32: written; dbeta, dM0 and dz0 may be NULL (not written)
 *
 * infini_attn_bwd takes bf16 activations, infini_attn_bwd_f32 fp32 ones; all arithmetic is
 * fp32.  Outputs must not overlap any input or each other.  The call recomputes the
 * forward's memory and softmax statistics itself and allocates its workspace (fp32, about
 * 4 x (q + 3 k) bytes plus 3 memory snapshots per segment) like the forward.  Shapes,
 * alignment, streams and errors as for infini_attn_fwd.
 */
INFINI_API int infini_attn_bwd(const void *q, const void *k, const void *v, const float *beta,
                               const float *M0, const float *z0, const void *dout,
                               const float *dM, const float *dz, void *dq, void *dk, void *dv,
                               float *dbeta, float *dM0, float *dz0, int64_t B, int64_t H,
                               int64_t Hkv, int64_t L, int64_t N, int64_t d, int update_rule,
                               infini_stream_t stream);
INFINI_API int infini_attn_bwd_f32(const void *q, const void *k, const void *v,
                                   const float *beta, const float *M0, const float *z0,
                                   const void *dout, const float *dM, const float *dz, void *dq,
                                   void *dk, void *dv, float *dbeta, float *dM0, float *dz0,
                                   int64_t B, int64_t H, int64_t Hkv, int64_t L, int64_t N,
                                   int64_t d, int update_rule, infini_stream_t stream);

/*
 * The memory after the whole sequence, without the outputs (bf16 keys / values; the _f32
 * variant takes fp32 ones): M_out / z_out exactly as infini_attn_fwd would leave them, from
 * the forward's memory kernels alone.  With M0 = z0 = NULL this is the increment of a
 * sequence chunk under the additive rule, the quantity ranks exchange when one sequence is
 * cut across devices (the memory before a chunk is M0 plus the increments of the chunks
 * before it).  Arguments, layouts, aliasing and errors as for infini_attn_fwd, without q,
 * beta and out.
 */
INFINI_API int infini_attn_state(const void *k, const void *v, const float *M0, const float *z0,
                                 float *M_out, float *z_out, int64_t B, int64_t Hkv, int64_t L,
                                 int64_t N, int64_t d, int update_rule, infini_stream_t stream);
INFINI_API int infini_attn_state_f32(const void *k, const void *v, const float *M0,
                                     const float *z0, float *M_out, float *z_out, int64_t B,
                                     int64_t Hkv, int64_t L, int64_t N, int64_t d,
                                     int update_rule, infini_stream_t stream);

/*
 * Token-by-token decode (bf16 activations; the _f32 variant takes fp32 ones).  One call
 * processes one new token of every (batch, head) at offset `pos` of its current segment
 * and gives the output the forward would give that token:
 *   - local attention over the current segment's keys at offsets 0..pos: rows 0..pos-1 of
 *     the cache, then this token's own key and value, which the call writes into row pos;
 *   - retrieval from (M, z), the memory from before the current segment;
 *   - the gate, as in the forward.
 * When pos == N - 1 the segment is complete: after the output, the call folds all N cached
 * rows into (M, z) in place (the linear or delta update of the forward), and the next
 * token starts a new segment at pos = 0.  At the end of a stream whose last segment is
 * shorter, infini_attn_fold folds the rows cached so far; feeding a whole sequence this way
 * then leaves the forward's M_out / z_out in (M, z).
 *
 *   q [B, H, d], k / v [B, Hkv, d]: this token;  out [B, H, d]
 *   k_cache / v_cache [B, Hkv, N, d]: the current segment's keys and values (caller-owned;
 *     rows >= pos are not read)
 *   M [B, Hkv, d, d], z [B, Hkv, d] fp32: read, and updated in place when pos == N - 1
 *     (start a stream with zeros, or with a forward's M_out / z_out)
 *   0 <= pos < N; N any positive length; d in {32, 64, 128}
 * Everything runs on `stream`, and neither call allocates memory (both may be captured in
 * a CUDA graph).  out must not overlap any other buffer; caches, M and z must not overlap
 * one another.
 */
INFINI_API int infini_attn_decode_step(const void *q, const void *k, const void *v,
                                       const float *beta, void *k_cache, void *v_cache,
                                       int64_t pos, float *M, float *z, void *out, int64_t B,
                                       int64_t H, int64_t Hkv, int64_t N, int64_t d,
                                       int update_rule, infini_stream_t stream);
INFINI_API int infini_attn_decode_step_f32(const void *q, const void *k, const void *v,
                                           const float *beta, void *k_cache, void *v_cache,
                                           int64_t pos, float *M, float *z, void *out,
                                           int64_t B, int64_t H, int64_t Hkv, int64_t N,
                                           int64_t d, int update_rule, infini_stream_t stream);

/*
 * Fold the first n rows (0 <= n <= N; 0 does nothing) of every chain's cache into (M, z),
 * in place, with the update rule of the forward: the end of a stream whose last segment is
 * shorter than N.  Layouts as for infini_attn_decode_step; no allocation.
 */
INFINI_API int infini_attn_fold(const void *k_cache, const void *v_cache, int64_t n, float *M,
                                float *z, int64_t B, int64_t Hkv, int64_t N, int64_t d,
                                int update_rule, infini_stream_t stream);
INFINI_API int infini_attn_fold_f32(const void *k_cache, const void *v_cache, int64_t n,
                                    float *M, float *z, int64_t B, int64_t Hkv, int64_t N,
                                    int64_t d, int update_rule, infini_stream_t stream);

/*
 * Allocation-free variant of infini_attn_fwd (bf16 activations); same parameters, same
 * results.  The pages have no counterpart to this entry point: it exists for callers that
 * may not allocate device memory while they run, for example a serving loop whose device
 * memory is planned and handed out by its own allocator up front (a stream-ordered
 * allocation there could fail when that allocator holds nearly all of HBM, or stall the
 * loop while the driver's pool grows), or a host program that gives plugins buffers but
 * no allocation rights.  This call makes no cudaMalloc / cudaFree / cudaMallocAsync /
 * cudaFreeAsync call and calls no allocating library routine.
 *
 *   - Its workspace is a fixed device array of INFINI_NOALLOC_SCRATCH_BYTES inside the
 *     library; every GPU that loads the library holds that array until the process exits.
 *     A problem whose workspace exceeds it is rejected with INFINI_ERR_UNSUPPORTED, before
 *     anything is launched.  The size that counts is what the kernels chosen for the
 *     problem need: infini_attn_workspace_bytes is an upper bound over all of them, and the
 *     fused 64-token paths need much less.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before any
 *     stream capture begins.
 *   - All calls on a device share that device's one array, which keeps the last call's
 *     contents.  Calls on the same device that overlap on the GPU (issued on different
 *     streams or from different host threads without ordering between them) race and
 *     corrupt each other's results: order them on one stream or with events.  Calls on
 *     different devices do not interfere.  Nothing in the array has to start at zero: each
 *     call writes every workspace byte it reads before reading it.
 */
#define INFINI_NOALLOC_SCRATCH_BYTES (16ull << 20)
INFINI_API int infini_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                       const float *beta, const float *M0, const float *z0,
                                       void *out, float *M_out, float *z_out, int64_t B,
                                       int64_t H, int64_t Hkv, int64_t L, int64_t N, int64_t d,
                                       int update_rule, infini_stream_t stream);

/* Bytes of workspace one call allocates for these sizes (an upper bound over the kernels
 * the call may choose; 0 on invalid sizes). */
INFINI_API int64_t infini_attn_workspace_bytes(int64_t B, int64_t Hkv, int64_t L, int64_t N, int64_t d);

/*
 * Synchronises `stream`, then reports whether a bounded wait inside a kernel of this
 * library gave up since the last check: INFINI_ERR_TIMEOUT (and the record is cleared),
 * INFINI_OK, or INFINI_ERR_CUDA if the synchronisation itself failed.  A kernel whose wait
 * gave up stops early and leaves part of its outputs unwritten.  The record is sticky:
 * until it is read here, later launches of the waiting kernels return without work.
 */
INFINI_API int infini_attn_device_status(infini_stream_t stream);

/* Static, NUL-terminated description of a status code. */
INFINI_API const char *infini_attn_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
INFINI_API int infini_attn_version(void);

/*
 * Launch tracing (off by default).  While enabled, every kernel this library enqueues is
 * bracketed by two CUDA events recorded on the call's stream.  infini_attn_trace_enable(1)
 * starts a new trace (clearing the previous one); it returns the previous setting.
 * infini_attn_trace_report synchronises on the recorded events, adds them to a per-kernel
 * table and writes it as JSON, {"<kernel>": {"launches": n, "ms": total}, ...}
 * (NUL-terminated, truncated to len - 1 bytes; buf may be NULL), and returns the size
 * the full report needs.  Reporting does not clear the table.
 */
INFINI_API int infini_attn_trace_enable(int on);
INFINI_API int64_t infini_attn_trace_report(char *buf, int64_t len);

/*
 * Test hooks: they let the library's failure paths be exercised without a real failure.
 * None of them is needed for normal use, and all are off by default.
 *
 * infini_attn_test_fail_allocations(n): the next n workspace allocations of this process
 *   fail as an exhausted device would make them fail: the calls return INFINI_ERR_OOM before
 *   anything is launched or written.  n = 0 turns the hook off.  INFINI_ERR_INVALID_ARG if
 *   n < 0.
 * infini_attn_test_wait_limit(cycles): the bound every device wait of the current device
 *   applies, in SM clock cycles (default about 0.5 s at the top clock; cycles <= 0 restores
 *   it).  A wait that reaches it gives up as described for infini_attn_device_status.
 * infini_attn_test_withhold_publish(on): on the current device, the first unit of every head
 *   in the fused 64-token kernel (additive rule, d = 64, N = 64, at most 64 units of 128
 *   tokens per head) skips publishing its memory aggregate, so the later units'
 *   waits for it run out: the call's outputs are then incomplete and
 *   infini_attn_device_status reports INFINI_ERR_TIMEOUT.  Nothing traps or hangs.
 * The last two copy to device variables synchronously (INFINI_ERR_CUDA if that fails); use
 * them while no call of this library is running on the device.
 */
INFINI_API int infini_attn_test_fail_allocations(int n);
INFINI_API int infini_attn_test_wait_limit(int64_t cycles);
INFINI_API int infini_attn_test_withhold_publish(int on);

#ifdef __cplusplus
}
#endif

#endif /* INFINI_ATTN_H */
