/*
 * la.h -- C ABI of the B200 (sm_100a) causal kernelized linear attention library.
 *
 * The library computes, per (batch b, head h) chain of N tokens,
 *
 *   kernelized modes (LA_PLAIN, LA_DECAY)
 *     S_t = gamma_h S_{t-1} + phi(k_t) v_t^T          S: d x dv, fp32
 *     z_t = gamma_h z_{t-1} + phi(k_t)                z: d,      fp32
 *     o_t = phi(q_t)^T S_t / (phi(q_t)^T z_t + eps)   (write, then read)
 *     phi(x) = elu(x) + 1 = (x > 0 ? x + 1 : exp(x)),  gamma_h = 1 in LA_PLAIN
 *   ("What Is Linear Attention?" §4 and §5.1; "Efficient attention variants"
 *    §4, §5 and §7.1; eps in the denominator: "Transformers Are RNNs" notes)
 *
 *   gated delta mode (LA_GATED_DELTA)
 *     S_t = alpha_t S_{t-1} + g_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T
 *     o_t = S_t^T q_t            (no feature map, no normaliser)
 *   ("Efficient attention variants" §7.4; "What Is Linear Attention?" §5.2-5.3)
 *
 * Prefill runs chunkwise: parallel inside a chunk, state carried between
 * chunks ("Efficient attention variants" §8).  Decode applies the recurrence
 * to one token per (sequence, head) against a resident state.
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Layouts are row-major and contiguous:
 *     q, k  [B,H,N,d]     v, out  [B,H,N,dv]      (prefill)
 *     q, k  [B,H,d]       v, out  [B,H,dv]        (decode)
 *     S     [B,H,d,dv] fp32, rows = key feature, columns = value
 *     z     [B,H,d]    fp32
 *     gamma [H] fp32;  alpha, g [B,H,N] fp32 (prefill) or [B,H] (decode)
 * - q, k, v and out share the element type cfg->dtype (fp32 or bf16).  All
 *   arithmetic accumulates in fp32; states are always fp32.
 * - Every pointer is a DEVICE pointer owned by the caller; the library keeps
 *   no pointer after a call returns and allocates no device memory.
 * - Every pointer must be 16-byte aligned (LA_ERR_ALIGN otherwise).
 * - Calls are asynchronous on cfg->stream (a cudaStream_t; NULL = the legacy
 *   default stream).  Argument errors are detected before anything is
 *   launched and returned synchronously; launch failures are reported as
 *   LA_ERR_CUDA.  Outputs must not alias inputs unless stated.
 * - Supported head sizes: d, dv in {64, 128}; anything else returns
 *   LA_ERR_UNSUPPORTED.  B, H, N >= 0 (zero sizes are valid and launch only
 *   what is needed to write the final state).
 */
#ifndef LA_H
#define LA_H

#include <stddef.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID = 1,      /* null pointer where one is required, negative size, bad enum */
    LA_ERR_UNSUPPORTED = 2,  /* head size or dtype/mode combination not implemented */
    LA_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned */
    LA_ERR_CUDA = 4,         /* a CUDA runtime/driver call or kernel launch failed */
    LA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (reported by la_prefill_check) */
    LA_ERR_WORKSPACE = 6     /* workspace missing or smaller than la_prefill_workspace_bytes() */
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

typedef enum { LA_PLAIN = 0, LA_DECAY = 1, LA_GATED_DELTA = 2, LA_GLA = 3 } la_mode;

typedef struct {
    la_dtype dtype;          /* element type of q, k, v, out */
    la_mode mode;            /* which recurrence */
    float eps;               /* denominator epsilon (kernelized modes); 1e-6 is the usual value */
    void* stream;            /* cudaStream_t the work is enqueued on */
    const float* S0;         /* prefill start state [B,H,d,dv] or NULL (zero state) */
    const float* z0;         /* prefill start normaliser [B,H,d] or NULL (zero); ignored in LA_GATED_DELTA */
    void* workspace;         /* device scratch for prefill; may be NULL when la_prefill_workspace_bytes() == 0 */
    size_t workspace_bytes;  /* size of workspace in bytes */
} la_config;

/*
 * la_prefill -- causal prefill of B*H chains of N tokens.
 *
 * Defined by the recurrences above ("What Is Linear Attention?" §4, §5.1;
 * "Efficient attention variants" §5, §7.1, §7.4), evaluated chunkwise
 * ("Efficient attention variants" §8).
 *
 *   q, k, v          inputs, layouts above, element type cfg->dtype.
 *   gamma_or_alpha   LA_PLAIN: must be NULL.  LA_DECAY: gamma [H], each in (0,1]
 *                    (bf16 inputs: each >= 0.1, the range of the tensor-core
 *                    path's scaled frame; a smaller gamma is reported as
 *                    LA_ERR_UNSUPPORTED by la_prefill_check).
 *                    LA_GATED_DELTA: alpha [B,H,N], each in (0,1].
 *                    LA_GLA: alpha [B,H,N,d], each in (0,1]: the per-key-channel
 *                    gate ("Efficient attention variants" §7.2),
 *                    S_t = diag(alpha_t) S_{t-1} + k_t v_t^T, o_t = S_t^T q_t.
 *   g                LA_GATED_DELTA: write strength g [B,H,N]; otherwise NULL.
 *   out              o [B,H,N,dv], element type cfg->dtype.
 *   S_out            final state S_N [B,H,d,dv] fp32 (required).
 *   z_out            final normaliser z_N [B,H,d] fp32 (kernelized modes, required);
 *                    must be NULL in LA_GATED_DELTA and LA_GLA.
 *   cfg              dtype, mode, eps, stream, optional start state and workspace.
 *
 * In LA_GATED_DELTA no feature map is applied; k is expected to be
 * L2-normalised by the caller (the rule is stable for ||k|| = 1, 0 < g <= 1).
 * LA_GLA applies no feature map and no normaliser either (eps is unused); it
 * runs a token-serial SIMT kernel (one thread per state column) for both
 * dtypes.
 * S_out and z_out must not share a byte with cfg->S0 or cfg->z0 (blocks of
 * one call read the start state while others write the final state);
 * continue a sequence by alternating two state buffers.  LA_ERR_INVALID if
 * any of these ranges overlap, in whole or in part.
 * Returns LA_OK once the work is enqueued.
 */
LA_API la_status la_prefill(const void* q, const void* k, const void* v,
                     const float* gamma_or_alpha, const float* g,
                     void* out, float* S_out, float* z_out,
                     int B, int H, int N, int d, int dv, const la_config* cfg);

/*
 * la_prefill_noalloc -- la_prefill for callers that cannot allocate device
 * memory on their launch path: a server that plans all device memory before
 * it starts, a plugin host that offers no workspace, or code that must avoid
 * the device synchronisation an allocation may cause.  The pages have no
 * counterpart; this is a service of this library.
 *
 * Arguments, layouts and results are those of la_prefill; cfg->workspace is
 * ignored.  The bf16 tensor-core prefill of the kernelized modes (LA_PLAIN,
 * LA_DECAY) keeps its segment summaries in a fixed 16 MiB array of device
 * memory inside the library instead of a caller workspace; every GPU that
 * loads the library holds that array until the process exits.  The
 * summaries of one call must fit in it: (B*H) * ceil(N / L) * (d*dv + d) * 4
 * bytes for a segment length L the call picks (a multiple of 64, at least
 * 128; the call lengthens segments until the summaries fit).  A problem that
 * does not fit even with one segment per chain, i.e. B*H*(d*dv + d)*4 >
 * 16 MiB, is rejected with LA_ERR_WORKSPACE before anything is launched.
 * Configurations whose la_prefill needs no workspace (fp32 inputs in every
 * mode, LA_GLA) run exactly as la_prefill does.  bf16 LA_GATED_DELTA, whose
 * workspace grows with N, returns LA_ERR_UNSUPPORTED.
 *
 * All calls in one process share the array and it keeps the last call's
 * contents: calls whose work can overlap on the GPU (enqueued on different
 * streams, or from different host threads) race on it and must be
 * serialised by the caller.  Separate processes each have their own copy.
 * The first call on each device looks up the array's device address with
 * that device current; make that first call before any stream capture on
 * that device.
 */
LA_API la_status la_prefill_noalloc(const void* q, const void* k, const void* v,
                                    const float* gamma_or_alpha, const float* g,
                                    void* out, float* S_out, float* z_out,
                                    int B, int H, int N, int d, int dv, const la_config* cfg);

/*
 * la_prefill_workspace_bytes -- device scratch la_prefill needs for these
 * sizes and this cfg (dtype, mode).  0 means no workspace is needed.  The
 * workspace carries data between the kernels of one call: per-segment state
 * summaries for bf16 LA_PLAIN / LA_DECAY, and for bf16 LA_GATED_DELTA the
 * per-chunk operands of each part of the sequence (-W, T' and the masked
 * score block, bf16, d + 128 values per token, and the per-token decay
 * factors, two fp32 values per token) plus, for more than one part, two
 * fp32 states that carry the chain between parts.  Its content need not be
 * initialised and
 * is dead after the call's work completes.  Two calls in flight at once need
 * two workspaces.
 */
LA_API size_t la_prefill_workspace_bytes(int B, int H, int N, int d, int dv, const la_config* cfg);

/*
 * la_prefill_kernel_count -- how many kernels one la_prefill call with these
 * sizes and this cfg (dtype, mode) launches, i.e. how many events
 * la_set_stage_events records for it: 3 for bf16 LA_PLAIN / LA_DECAY (segment
 * summaries, scan, chunk loop); 2 P for bf16 LA_GATED_DELTA, whose sequence
 * runs as P <= 8 parts (each a chunk prep pass and a chain pass; the prep
 * pass of part i + 1 overlaps the chain pass of part i); 2 for fp32
 * LA_PLAIN / LA_DECAY with N <= 1024 (the parallel form: outputs, then the
 * final state); 1 otherwise; 0 when
 * the call launches no kernel (N = 0, nothing to do, or unsupported sizes).
 * Host-only.  Not from the pages: a service for profiling.
 */
LA_API int la_prefill_kernel_count(int B, int H, int N, int d, int dv, const la_config* cfg);

/*
 * la_prefill_varlen -- la_prefill over a right-padded batch of sequences of
 * different lengths: sequence b holds seq_lens[b] tokens in rows
 * 0 .. seq_lens[b]-1 of its [H, N, .] block.  Real batches carry padding and
 * chunk boundaries that the pages' single-sequence examples leave out
 * ("Efficient attention variants" §10, closing remarks); with a start state
 * per sequence this is chunked-prefill continuation of a mixed batch.
 *
 *   q, k, v, out, gamma_or_alpha, g, S_out, z_out, cfg
 *                    as in la_prefill, laid out for the padded length N:
 *                    q, k [B,H,N,d]; v, out [B,H,N,dv]; alpha [B,H,N]
 *                    (LA_GATED_DELTA) or [B,H,N,d] (LA_GLA); g [B,H,N];
 *                    S_out, cfg->S0 [B,H,d,dv]; z_out, cfg->z0 [B,H,d].
 *   seq_lens         HOST array of B lengths, each 0 <= seq_lens[b] <= N
 *                    (LA_ERR_INVALID otherwise, or if NULL while B*H > 0).
 *
 * Sequence b's results equal those of la_prefill on that sequence alone
 * (B = 1, N = seq_lens[b]) from its start state: out[b, :, t] for
 * t < seq_lens[b], and S_out[b], z_out[b] after its last token (its start
 * state when seq_lens[b] == 0), up to rounding: the bf16 LA_PLAIN / LA_DECAY
 * path may cut a sequence into segments at other points than the solo call
 * does.  Padding rows of out are never written.  Padding rows of q, k, v,
 * alpha, g never affect a result, whatever they hold (NaN and inf included).
 *
 * bf16 LA_PLAIN / LA_DECAY with B <= 64: the whole batch runs as one set of
 * three kernels (segment summaries, scan, chunk loop) whose segments are the
 * (sequence, head, segment) triples of all sequences, with one segment length
 * chosen so that they fill one wave of the GPU; these kernels may read
 * padding rows of q, k, v inside a sequence's last 64-token chunk and discard
 * them.  Otherwise the sequences run one after another on cfg->stream, each
 * through the kernels la_prefill uses, and padding rows are not read; each
 * has a slice of cfg->workspace, so a sequence's first kernel may start while
 * the previous sequence's last kernel drains.  cfg->workspace must hold
 * la_prefill_varlen_workspace_bytes() bytes.  Returns LA_OK once all the work
 * is enqueued; on an error from sequence b of the one-by-one form, sequences
 * before b are enqueued and the rest are not.
 */
LA_API la_status la_prefill_varlen(const void* q, const void* k, const void* v,
                                   const float* gamma_or_alpha, const float* g,
                                   void* out, float* S_out, float* z_out, const int* seq_lens,
                                   int B, int H, int N, int d, int dv, const la_config* cfg);

/*
 * la_prefill_varlen_workspace_bytes -- the workspace la_prefill_varlen needs
 * (seq_lens: host array of B lengths).  For the one-launch-set form (bf16
 * LA_PLAIN / LA_DECAY, B <= 64) one fp32 summary of d*dv + d values per
 * segment of the batch; otherwise the sum over the batch of
 * la_prefill_workspace_bytes(1, H, seq_lens[b], d, dv, cfg), each rounded up
 * to a multiple of 256 bytes.  0 means none is needed.
 */
LA_API size_t la_prefill_varlen_workspace_bytes(const int* seq_lens, int B, int H, int d, int dv,
                                                const la_config* cfg);

/*
 * la_decode_step -- one decode step for B sequences x H heads, kernelized
 * recurrence with gamma = 1 (the state cache of "What Is Linear Attention?"
 * §6; update order of §4: write, then read):
 *     S += phi(k) v^T;  z += phi(k);  out = phi(q)^T S / (phi(q)^T z + eps)
 *
 *   q, k   [B,H,d], v [B,H,dv], element type cfg->dtype.
 *   S      [B,H,d,dv] fp32, read and updated in place.
 *   z      [B,H,d] fp32, read and updated in place.
 *   out    [B,H,dv], element type cfg->dtype.
 *   cfg    dtype, eps, stream; mode must be LA_PLAIN; S0/z0/workspace unused.
 */
LA_API la_status la_decode_step(const void* q, const void* k, const void* v,
                         float* S, float* z, void* out,
                         int B, int H, int d, int dv, const la_config* cfg);

/*
 * la_gated_delta_decode_step -- one decode step of the gated delta rule for
 * B sequences x H heads ("Efficient attention variants" §7.4):
 *     S = alpha S + g k (v - alpha S^T k)^T;  out = S^T q
 *
 *   q, k   [B,H,d], v [B,H,dv], element type cfg->dtype (k L2-normalised).
 *   alpha, g  [B,H] fp32.
 *   S      [B,H,d,dv] fp32, read and updated in place.
 *   out    [B,H,dv], element type cfg->dtype.
 *   cfg    dtype, stream; mode must be LA_GATED_DELTA.
 */
LA_API la_status la_gated_delta_decode_step(const void* q, const void* k, const void* v,
                                     const float* alpha, const float* g,
                                     float* S, void* out,
                                     int B, int H, int d, int dv, const la_config* cfg);

/*
 * la_causal_conv -- short causal convolution over the token axis with a conv
 * cache ("What Is Linear Attention?" §5.4: a short convolution over the last
 * w tokens beside the linear state; inference keeps the recent window as a
 * conv cache).  One filter per (head, channel), no activation:
 *
 *   xh = [cache; x]  (the chain's previous w-1 inputs, then its N new ones)
 *   out_t[c] = sum_{i=0}^{w-1} weight[h][c][i] * xh[t + i][c]
 *
 * i.e. weight i multiplies the input w-1-i tokens back (the last weight the
 * current token); cache_out = the last w-1 rows of xh.
 *
 *   x          [B,H,N,d] input, element type cfg->dtype (bf16 or fp32).
 *   weight     [H,d,w] fp32 filters.
 *   cache      [B,H,w-1,d] (cfg->dtype) previous inputs, or NULL for zero history.
 *   out        [B,H,N,d] (cfg->dtype); fp32 arithmetic, rounded once.
 *   cache_out  [B,H,w-1,d] (cfg->dtype) or NULL; must not overlap cache or x
 *              (continue a stream by alternating two cache buffers).
 *   w          1..8.  d in {64, 128}.  N >= 0 (N = 0 only moves the cache).
 *   cfg        dtype and stream are used; mode, eps, S0, z0, workspace ignored.
 *
 * Decoding is the N = 1 call.  Returns LA_OK once the work is enqueued;
 * LA_ERR_INVALID for bad sizes, NULL x/weight/out (when N > 0) or an
 * overlapping cache_out; LA_ERR_UNSUPPORTED for d or w out of range;
 * LA_ERR_ALIGN for a pointer not 16-byte aligned.  Not part of the pages'
 * attention method itself: the adjacent local operator the same layer runs.
 */
LA_API la_status la_causal_conv(const void* x, const float* weight, const void* cache,
                                void* out, void* cache_out,
                                int B, int H, int N, int d, int w, const la_config* cfg);

/*
 * la_set_stage_events -- profiling hook, off by default.  With n > 0, every
 * later la_prefill / la_decode_step / la_gated_delta_decode_step /
 * la_causal_conv records
 * events[i] on its cfg->stream right after launching its i-th kernel
 * (i < n; a call launches 1 to 16 kernels, la_prefill_kernel_count gives the
 * number for a prefill: bf16 LA_PLAIN/LA_DECAY prefill = segment summaries,
 * scan, chunk loop; bf16 LA_GATED_DELTA prefill = chunk prep and chain per
 * part; every other path, la_causal_conv included, one kernel).  events are cudaEvent_t handles
 * owned by the caller, who must keep them alive while the hook is set; n = 0
 * turns it off.  The setting is process-wide and not thread-safe: set it
 * only while no other thread launches through this library.  Returns
 * LA_ERR_INVALID for n outside 0..16 or a NULL handle.  Not from the pages: a
 * service for timing each kernel of a call with CUDA events.
 */
LA_API la_status la_set_stage_events(void* const* events, int n);

/*
 * la_prefill_check -- wait for the work enqueued on `stream` and report any
 * device-side error recorded in `workspace` by the last la_prefill that used
 * it (LA_ERR_TIMEOUT if a bounded wait between cooperating blocks gave up).
 * Synchronises the stream.  A NULL workspace only synchronises.
 */
LA_API la_status la_prefill_check(const void* workspace, void* stream);

/*
 * la_selftest_wait_timeout -- exercise the failure path of the bounded
 * device-side waits.  Enqueues on `stream` one kernel of 32 threads whose
 * single mbarrier wait has nothing to wait for: the wait gives up after its
 * bound (about a second), records the timeout in the device error word and
 * returns, leaving the context usable.  The next la_prefill_check on that
 * stream returns LA_ERR_TIMEOUT and clears the word.  For tests of error
 * reporting; it issues no copy and no MMA.  Returns LA_OK once enqueued.
 */
LA_API la_status la_selftest_wait_timeout(void* stream);

/* Human-readable name of a status code (static storage). */
LA_API const char* la_status_string(la_status s);

/* Library version as "major.minor.patch" (static storage). */
LA_API const char* la_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LA_H */
