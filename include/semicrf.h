/*
 * semicrf.h -- C ABI of the B200 (sm_100a) streaming semi-CRF library.
 *
 * The library computes, on one GPU, the hot path of the semi-Markov CRF
 * described by "Streaming Structured Inference with Flash-SemiCRF"
 * (abstract; explainer sections 1-2):
 *
 *   1. prefix sums of zero-centred emissions        semicrf_prefix_center
 *   2. a streaming log-semiring forward pass with a
 *      K-slot ring, normalised and checkpointed      semicrf_forward
 *   3. a checkpointed backward pass giving exact
 *      marginals and gradients                       semicrf_backward
 *   4. max-semiring (Viterbi) decoding               semicrf_viterbi
 *   and the score of a given segmentation with its
 *   gradient, for the training loss                  semicrf_path_score
 *   with boundary projections                        semicrf_*_proj
 *
 * Model.  A sequence b has length L_b (0 <= L_b <= T).  A segmentation
 * splits its positions 0..L_b-1 into consecutive segments [s, t) of duration
 * k = t - s in 1..K, each with a label c in 0..C-1.  Its score is the sum over
 * segments of  content(s,t,c) + dur[k-1, c]  plus  trans[c', c]  between
 * consecutive segments (labels c' then c); the first segment has no
 * transition term and there is no end term.  content(s,t,c) is the sum of the
 * centred emissions e~[u, c] = em[b, u, c] - nu[b, c] over u = s..t-1, with
 * nu[b, c] the mean of em[b, :L_b, c] (explainer section 2, "Emission
 * Baseline Centering"; centering can be switched off).  log Z_b is the
 * log-sum-exp of the scores of all segmentations.
 *
 * Conventions shared by every entry point.
 *  - All array arguments are DEVICE pointers to contiguous row-major memory
 *    owned by the caller.  The library never allocates, frees or keeps a
 *    pointer after the call returns.
 *  - em       [B, T, C] float32 raw emissions; rows u >= L_b are never read.
 *  - lengths  [B] int32, device memory.  A length outside [0, T] is reported
 *             through the workspace status word (SEMICRF_ERR_BAD_LENGTH); that
 *             sequence's outputs are zeroed and its log Z is NaN.
 *  - trans    [C, C] float32, trans[c', c] scores the transition c' -> c.
 *  - dur      [K, C] float32, dur[k-1, c] scores a label-c segment of length k.
 *  - stream   a cudaStream_t (NULL = legacy default stream).  All work is
 *             asynchronous on that stream; a return value of SEMICRF_OK means
 *             the launches were enqueued.
 *  - Every call returns a status code.  Argument errors are detected on the
 *    host before anything is launched.  Device-side conditions (bad lengths,
 *    a bounded wait that gave up) are recorded in the workspace status word,
 *    read with semicrf_get_status.
 *  - Limits of the library: 1 <= C <= 128, T <= 2^26, B <= 2^20, and
 *    K <= 8192 (C <= 8), K <= 512 (C <= 16), K <= 256 (C <= 32),
 *    K <= 128 (C <= 64), K <= 64 (C <= 128).  Larger values return
 *    SEMICRF_ERR_UNSUPPORTED.  (Durations of K = 2000-8000 on sequences of
 *    10^6 positions are the pages' genomic regime, explainer section 4 and
 *    the Chinese explainer's section 4.)  Long durations, 2048 < K <= 8192,
 *    run on the exponential-domain rings and the pipelined decoder only:
 *    a sequence whose scores leave those rings' exponent range (see
 *    SEMICRF_FLAG_LOG_DOMAIN) is reported through the status word as
 *    SEMICRF_ERR_UNSUPPORTED with log Z = NaN and zero posteriors, and
 *    SEMICRF_FLAG_LOG_DOMAIN itself returns SEMICRF_ERR_UNSUPPORTED.
 *  - Numbers are computed in float32 in base-2 log units with exactly
 *    representable integer frames and float64 normalisers; results are
 *    deterministic (no floating-point atomics).
 */
#ifndef SEMICRF_H
#define SEMICRF_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SEMICRF_API __attribute__((visibility("default")))
#else
#define SEMICRF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *semicrf_stream_t;

enum semicrf_status {
    SEMICRF_OK = 0,
    SEMICRF_ERR_INVALID_ARG = 1,         /* null pointer, negative size, unknown flag */
    SEMICRF_ERR_UNSUPPORTED = 2,         /* C, K, K*C, T or B above the limits above */
    SEMICRF_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < semicrf_workspace_bytes(...) */
    SEMICRF_ERR_CUDA = 4,                /* a CUDA launch or copy failed */
    SEMICRF_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device wait gave up */
    SEMICRF_ERR_BAD_LENGTH = 6,          /* some lengths[b] outside [0, T] */
    SEMICRF_ERR_BOUNDS = 7               /* bounds-checking build only: an index check
                                            failed; (status >> 8) names the check site */
};

/* flags */
#define SEMICRF_FLAG_NO_CENTER 0x1u    /* use raw emissions (nu = 0) */
#define SEMICRF_FLAG_FORWARD_ONLY 0x2u /* forward skips the backward ring (inference);
                                          a backward given the same flag runs it itself */
#define SEMICRF_FLAG_LOG_DOMAIN 0x4u   /* run the rings in the log domain for every
                                          sequence (by default a sequence whose scores
                                          keep every step within float32's exponent
                                          range runs in the faster exponential domain;
                                          results agree to rounding) */
#define SEMICRF_FLAG_NEGATE_GRAD 0x8u  /* semicrf_path_score subtracts its gradient
                                          (w_b = -grad_score[b]); the other calls
                                          ignore it */

/*
 * Bytes of device workspace needed by forward/backward/viterbi for these
 * sizes and flags.  The workspace holds the status word, the prefix-sum array
 * (stored as an exact integer part plus a float32 fraction, 8 bytes per
 * entry), the ring checkpoints taken every Delta = ceil(sqrt(T*K)) positions
 * (explainer section 2, "Streaming Forward-Backward with Ring Buffers",
 * checkpointing), the per-segment recompute buffers and the partial sums of
 * the backward pass.  Host-only; launches nothing.
 */
SEMICRF_API int semicrf_workspace_bytes(int B, int T, int C, int K, unsigned flags, size_t *bytes);

/*
 * Where the workspace bytes go (host-only, launches nothing; no counterpart
 * on the pages: it itemises the memory the pages' "Memory Complexity
 * Breakthrough" discussion counts, explainer section 3).  Writes
 * bytes[i] for i < n, the size of workspace group i below (0 for
 * i >= SEMICRF_WS_GROUPS); the groups add up to semicrf_workspace_bytes.
 * Returns the same codes as semicrf_workspace_bytes.
 */
enum semicrf_ws_group {
    SEMICRF_WS_OTHER = 0,        /* status word, log Z, per-sequence flags and bounds */
    SEMICRF_WS_PREFIX = 1,       /* split prefix sums [B][T+1][C] x 8 bytes, chunk sums */
    SEMICRF_WS_CHECKPOINTS = 2,  /* ring checkpoints every Delta positions, both directions */
    SEMICRF_WS_RECOMPUTE = 3,    /* per-segment recompute store and count partials */
    SEMICRF_WS_VITERBI = 4,      /* decoder rows: chosen durations, V, backpointer words */
    SEMICRF_WS_KEPT_ROWS = 5,    /* exponential-domain ring values kept per boundary */
    SEMICRF_WS_PATH = 6,         /* path-score counts and partial sums */
    SEMICRF_WS_PROJ = 7,         /* boundary-projection start terms */
    SEMICRF_WS_GROUPS = 8
};
SEMICRF_API int semicrf_workspace_itemize(int B, int T, int C, int K, unsigned flags, size_t *bytes,
                                          int n);

/*
 * Launch geometry the library picks for these sizes (host-only diagnostic,
 * launches nothing; no counterpart on the pages).  Writes shape[i] for
 * i < n (0 past the fields): CTAs per ring of the exponential-domain rings
 * and pipelined decoder (0: those kernels do not serve these sizes; 1: one
 * CTA per ring; more: a thread-block cluster), labels per CTA, combine lanes
 * per label, weights per combine lane, helper lanes per label, durations per
 * helper lane, threads per CTA, checkpoint spacing Delta, checkpoint
 * segments per sequence, posterior tile rows, the log-domain kernels'
 * durations per lane, lanes per label, labels per lane and threads per CTA
 * (0: no log-domain kernel for these sizes), the segment-end rows the
 * posterior pass stages at once, and the cut-normaliser grid spacing.
 * Returns the same codes as semicrf_workspace_bytes.
 */
#define SEMICRF_SHAPE_FIELDS 16
SEMICRF_API int semicrf_launch_shape(int B, int T, int C, int K, int32_t *shape, int n);

/*
 * Step 1 (explainer section 2, "On-the-Fly Edge Computation via Prefix Sums"
 * and "Emission Baseline Centering"): nu[b, c] = mean of em[b, :L_b, c]
 * (0 with SEMICRF_FLAG_NO_CENTER) and the float64 prefix sums
 * S[b, t, c] = sum_{u < t} (em[b, u, c] - nu[b, c]) for t = 0..L_b; rows
 * t > L_b are zero.  S is [B, T+1, C] float64, nu is [B, C] float32.
 * ws must hold semicrf_workspace_bytes(B, T, C, 1, flags) bytes (per-chunk
 * partial sums and the status word live there).
 */
SEMICRF_API int semicrf_prefix_center(const float *em, const int32_t *lengths, int B, int T, int C,
                          unsigned flags, void *ws, size_t ws_bytes, double *S, float *nu,
                          semicrf_stream_t stream);

/*
 * Steps 1-2 (explainer section 2, "Streaming Forward-Backward with Ring
 * Buffers"; abstract): writes logZ[b] (float64) for every sequence.  The
 * forward recursion
 *   alpha[t, c] = LSE_{k <= min(K,t)} LSE_{c'} alpha[t-k, c'] + trans[c', c]
 *                 + S[t, c] - S[t-k, c] + dur[k-1, c]
 * (no c' term when t-k = 0) keeps a K-slot ring per sequence in shared memory,
 * never materialises an edge, and saves the ring plus its normaliser every
 * Delta positions into the workspace.  Unless SEMICRF_FLAG_FORWARD_ONLY is
 * given, the backward ring runs in the same launch on other SMs and is
 * checkpointed the same way, so a following semicrf_backward needs only the
 * workspace.  The workspace must be 256-byte aligned (cudaMalloc is).
 */
SEMICRF_API int semicrf_forward(const float *em, const int32_t *lengths, const float *trans, const float *dur,
                    int B, int T, int C, int K, unsigned flags, void *ws, size_t ws_bytes,
                    double *logZ, semicrf_stream_t stream);

/*
 * Step 3 (explainer section 2, checkpointing; section 4 "Correctness"):
 * consumes the workspace of the immediately preceding semicrf_forward with
 * the same arguments (the workspace must not be reused in between).  Each
 * checkpoint segment restores its ring checkpoints, recomputes alpha and beta
 * locally and accumulates the exact posteriors.  Outputs:
 *   grad_em    [B, T, C]  g_b * d logZ_b / d em[b, u, c]  (through centering)
 *   grad_trans [C, C]     sum_b g_b * E[#transitions c' -> c]
 *   grad_dur   [K, C]     sum_b g_b * E[#label-c segments of length k]
 *   pos_marg   [B, T, C]  P(position u lies in a label-c segment)   (nullable)
 *   start_marg [B, T+1, C] P(a label-c segment starts at boundary s) (nullable)
 *   end_marg   [B, T+1, C] P(a label-c segment ends at boundary t)   (nullable)
 * g_b = grad_logZ[b] (device float64 [B]; NULL means all ones).  Marginals
 * are not scaled by g_b.  Entries past L_b are zero.
 */
SEMICRF_API int semicrf_backward(const int32_t *lengths, const float *trans, const float *dur,
                     int B, int T, int C, int K, unsigned flags, void *ws, size_t ws_bytes,
                     const double *grad_logZ, float *grad_em, float *grad_trans, float *grad_dur,
                     float *pos_marg, float *start_marg, float *end_marg,
                     semicrf_stream_t stream);

/*
 * Step 3 with the segment marginals (explainer section 4, "Correctness --
 * Self-Consistency": the boundary and segment probabilities are valid
 * distributions): everything semicrf_backward computes, plus
 *   seg_marg [B, T, K, C]  P(a label-c segment covers exactly [s, s+k)) at
 *                          [b, s, k-1, c]; zero where s >= L_b or s + k > L_b
 * (float32, not scaled by g_b).  Summed over k it is start_marg, over s (and
 * times g) grad_dur.  The array is O(T K C): meant for moderate sizes (the
 * speech-scale batch needs 150 MB).  seg_marg must not be NULL when B, T > 0
 * (SEMICRF_ERR_INVALID_ARG); the other arguments and errors are those of
 * semicrf_backward.  Not for a workspace filled by semicrf_forward_proj.
 */
SEMICRF_API int semicrf_backward_segments(const int32_t *lengths, const float *trans,
                                          const float *dur, int B, int T, int C, int K,
                                          unsigned flags, void *ws, size_t ws_bytes,
                                          const double *grad_logZ, float *grad_em,
                                          float *grad_trans, float *grad_dur, float *pos_marg,
                                          float *start_marg, float *end_marg, float *seg_marg,
                                          semicrf_stream_t stream);

/*
 * Step 4: max-semiring decoding with the same recursion (max in place of
 * log-sum-exp).  Ties go to the smallest duration k, then the smallest
 * previous label c', and at the end to the smallest final label.  Writes
 * score[b] (float64), labels[b, u] (int32, -1 for u >= L_b) and
 * seg_start[b, u] (1 where a segment starts, else 0).  Uses the workspace for
 * the prefix sums and the backpointers.
 */
SEMICRF_API int semicrf_viterbi(const float *em, const int32_t *lengths, const float *trans, const float *dur,
                    int B, int T, int C, int K, unsigned flags, void *ws, size_t ws_bytes,
                    double *score, int32_t *labels, uint8_t *seg_start, semicrf_stream_t stream);

/*
 * Score of given segmentations, for the training loss (explainer section 4,
 * "Results and Benchmarks", Correctness: the model is trained to the CRF loss,
 * the negative log-likelihood log Z - score(gold)).  The path of sequence b is
 * labels[b, u] (int32) and seg_start[b, u] (uint8, nonzero where a segment
 * starts), u < L_b, the form semicrf_viterbi writes; entries u >= L_b are
 * never read.  Writes score[b] (float64, nullable): the model score of that
 * segmentation, the same sum as in the model above (centred unless
 * SEMICRF_FLAG_NO_CENTER).  A malformed path -- no start at u = 0, a label
 * outside [0, C), a label that changes inside a segment, a segment longer
 * than K -- gets score NaN and no gradient; L_b = 0 scores 0.
 *
 * Gradients are ACCUMULATED: for each non-null output,
 *   grad_em    [B, T, C] += w_b * d score_b / d em[b, u, c]
 *                           = w_b * ([labels[b,u] = c] - n_bc / L_b)  (u < L_b;
 *                             n_bc positions labelled c, the second term
 *                             through the centring mean)
 *   grad_trans [C, C]    += sum_b w_b * (#c' -> c transitions on path b)
 *   grad_dur   [K, C]    += sum_b w_b * (#label-c segments of length k)
 * with w_b = grad_score[b] (device float64 [B]; NULL means all ones), negated
 * under SEMICRF_FLAG_NEGATE_GRAD.  For the NLL log Z - score, run
 * semicrf_backward with grad_logZ = g (gradients of log Z) and then this call
 * with grad_score = g and SEMICRF_FLAG_NEGATE_GRAD on the same output buffers.  The path-score part of the
 * workspace is its own, so the call may sit between semicrf_forward and
 * semicrf_backward.  (B, T, C, K) and the workspace are as for
 * semicrf_forward; a length outside [0, T] sets SEMICRF_ERR_BAD_LENGTH.
 * Deterministic: counts use integer atomics, every float sum a fixed order.
 */
SEMICRF_API int semicrf_path_score(const float *em, const int32_t *lengths, const float *trans,
                                   const float *dur, const int32_t *labels,
                                   const uint8_t *seg_start, int B, int T, int C, int K,
                                   unsigned flags, void *ws, size_t ws_bytes,
                                   const double *grad_score, double *score, float *grad_em,
                                   float *grad_trans, float *grad_dur, semicrf_stream_t stream);

/*
 * Boundary projections ("Streaming Structured Inference with Flash-SemiCRF",
 * explainer section 2, "Boundary Projections": separately computed start and
 * end features added to the edge potentials).  p_start and p_end are
 * [B, T, C] float32 device arrays (either may be NULL): a segment [s, t) with
 * label c scores p_start[b, s, c] + p_end[b, t-1, c] on top of the model
 * above.  Entries u >= L_b are never read.
 *
 * semicrf_forward_proj: as semicrf_forward.  The rings run in the log domain
 *   (the exponential-domain kernels have no projection term); the workspace
 *   records that projections are on for the backward that consumes it.
 * semicrf_backward_proj: as semicrf_backward, after semicrf_forward_proj on
 *   the same workspace (a workspace filled by semicrf_forward_proj must be
 *   consumed by semicrf_backward_proj: under SEMICRF_FLAG_FORWARD_ONLY the
 *   plain semicrf_backward would run the backward ring without the
 *   projection terms); additionally writes (each nullable)
 *     grad_p_start [B, T, C] = g_b * start_marg[b, u, c]
 *     grad_p_end   [B, T, C] = g_b * end_marg[b, u + 1, c]   (0 for u >= L_b),
 *   the gradients of g_b * log Z_b.  The marginal outputs stay optional.
 * semicrf_viterbi_proj: as semicrf_viterbi with the projection terms.
 * semicrf_path_score_proj: as semicrf_path_score with the projection terms;
 *   also ADDS w_b to grad_p_start[b, s, c] at the first position s and to
 *   grad_p_end[b, u, c] at the last position u of each label-c segment
 *   (each nullable).
 * A plain call (semicrf_forward, semicrf_viterbi) clears the record.
 */
SEMICRF_API int semicrf_forward_proj(const float *em, const int32_t *lengths, const float *trans,
                                     const float *dur, const float *p_start, const float *p_end,
                                     int B, int T, int C, int K, unsigned flags, void *ws,
                                     size_t ws_bytes, double *logZ, semicrf_stream_t stream);
SEMICRF_API int semicrf_backward_proj(const int32_t *lengths, const float *trans, const float *dur,
                                      int B, int T, int C, int K, unsigned flags, void *ws,
                                      size_t ws_bytes, const double *grad_logZ, float *grad_em,
                                      float *grad_trans, float *grad_dur, float *grad_p_start,
                                      float *grad_p_end, float *pos_marg, float *start_marg,
                                      float *end_marg, semicrf_stream_t stream);
SEMICRF_API int semicrf_viterbi_proj(const float *em, const int32_t *lengths, const float *trans,
                                     const float *dur, const float *p_start, const float *p_end,
                                     int B, int T, int C, int K, unsigned flags, void *ws,
                                     size_t ws_bytes, double *score, int32_t *labels,
                                     uint8_t *seg_start, semicrf_stream_t stream);
SEMICRF_API int semicrf_path_score_proj(const float *em, const int32_t *lengths,
                                        const float *trans, const float *dur,
                                        const float *p_start, const float *p_end,
                                        const int32_t *labels, const uint8_t *seg_start, int B,
                                        int T, int C, int K, unsigned flags, void *ws,
                                        size_t ws_bytes, const double *grad_score, double *score,
                                        float *grad_em, float *grad_trans, float *grad_dur,
                                        float *grad_p_start, float *grad_p_end,
                                        semicrf_stream_t stream);

/*
 * Synchronises `stream`, then reads the device status word of workspace
 * `ws` into *status (a semicrf_status value; the first device error wins).
 * Forward and viterbi reset the word when they start.
 */
SEMICRF_API int semicrf_get_status(const void *ws, semicrf_stream_t stream, int *status);

/*
 * Which arithmetic ran each ring of the last forward (or forward-only
 * backward) on this workspace: synchronises `stream` and copies 2*B host ints
 * into `domains` -- [0, B) the forward rings, [B, 2B) the backward rings --
 * each 1 (exponential domain), 2 (log domain) or 0 (not run).  (B, T, C, K,
 * flags) must be those of that call.  Diagnostic; nothing else depends on it.
 */
SEMICRF_API int semicrf_ring_domains(const void *ws, size_t ws_bytes, int B, int T, int C, int K,
                                     unsigned flags, semicrf_stream_t stream, int32_t *domains);

/* Human-readable name of a status code (static string, never NULL). */
SEMICRF_API const char *semicrf_strerror(int code);

/*
 * The sha256 (64 hex digits) of the kernel sources this library was built
 * from (csrc/*.cu and *.cuh: name, NUL, contents, in name order), or
 * "unknown" when the build did not define it.  Static string, never NULL.
 * Lets a caller check that the library it loaded matches the sources.
 */
SEMICRF_API const char *semicrf_source_digest(void);

/*
 * Diagnostic: runs the library's bounded shared-memory-barrier wait on a
 * barrier nothing will ever complete, with a limit of `spins` polls, and
 * records the outcome in the workspace status word (SEMICRF_ERR_DEVICE_TIMEOUT
 * when the limit is hit).  Lets a test check that a wait that never
 * completes ends with an error status instead of hanging.  No counterpart on
 * the pages.
 */
SEMICRF_API int semicrf_selftest_bounded_wait(void *ws, size_t ws_bytes, int spins, semicrf_stream_t stream);

/*
 * Self-test of the bounds-checking debug build (libsemicrf_b200_check.so,
 * compiled with -DSEMICRF_BOUNDS_CHECK; no counterpart on the pages): clears
 * the status word of `ws` and launches one CTA whose only guarded store uses
 * an index one past its 32-entry shared array; the check records
 * SEMICRF_ERR_BOUNDS | site << 8 and skips the store, so nothing is written
 * out of bounds.  Read the result with semicrf_get_status.  The release
 * build returns SEMICRF_ERR_UNSUPPORTED and launches nothing.
 */
SEMICRF_API int semicrf_selftest_bounds(void *ws, size_t ws_bytes, semicrf_stream_t stream);

/*
 * Diagnostic timing (no counterpart on the pages).  semicrf_profile_enable(1)
 * clears the record and starts bracketing every kernel this library launches
 * with two CUDA events on the launch stream; semicrf_profile_enable(0) stops.
 * semicrf_profile_read(name, &ms, &n) waits for the recorded events of kernel
 * `name` (e.g. "chain_kernel", "segment_kernel", "viterbi_kernel") and returns
 * their summed device time in milliseconds and the number of launches.
 * Host-side bookkeeping only; not thread-safe across concurrent enables.
 */
SEMICRF_API int semicrf_profile_enable(int on);
SEMICRF_API int semicrf_profile_read(const char *kernel, double *total_ms, int *launches);

/*
 * log Z without a workspace and without allocating (no counterpart on the
 * pages).  For callers that cannot allocate device memory when they run --
 * a plugin whose execution hook may not allocate because its memory was
 * planned ahead, or code where a cudaMalloc would stall the device -- this
 * runs the same prefix-sum and forward-ring kernels as semicrf_forward with
 * SEMICRF_FLAG_FORWARD_ONLY, keeping their scratch in one fixed array inside
 * the library's device image (SEMICRF_NOALLOC_SCRATCH_BYTES; every GPU that
 * loads the library holds it until the process exits).  The caller still
 * passes the inputs and logZ [B] (float64), all device memory.
 *  - Sizes whose forward working set exceeds the array (prefix sums, chunk
 *    sums and ring checkpoints: about 8*B*(T+1)*C bytes plus the
 *    checkpoints) return SEMICRF_ERR_UNSUPPORTED before anything runs.
 *  - The first call on each device looks up the array's device address with
 *    that device current; make that first call before any stream capture.
 *    The address is kept for the life of the process: after a device reset
 *    (which unloads the library's device image) restart the process before
 *    calling this again.
 *  - No cudaMalloc, cudaFree or allocating library call is made.
 *  - Every call on a device shares the array and leaves its contents behind;
 *    only the status word is cleared per call.  Calls that overlap on the GPU
 *    (two streams or two host threads at once) race on it: serialise them.
 *  - A length outside [0, T] gives logZ[b] = NaN (no status word to read).
 */
#define SEMICRF_NOALLOC_SCRATCH_BYTES (32u << 20)
SEMICRF_API int semicrf_forward_noalloc(const float *em, const int32_t *lengths, const float *trans,
                                        const float *dur, int B, int T, int C, int K,
                                        unsigned flags, double *logZ, semicrf_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SEMICRF_H */
