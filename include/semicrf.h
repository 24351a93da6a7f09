/*
 * semicrf.h -- C ABI of libsemicrf.so: exact semi-CRF streaming forward-backward
 * on NVIDIA B200 (sm_100a).
 *
 * The operation is the semi-Markov CRF of "Streaming Structured Inference with
 * Flash-SemiCRF" (abstract; technical summary sections 1-2): segments [s, s+d)
 * with label c score S[s+d,c] - S[s,c] + D[d-1,c], consecutive segments add
 * A[c',c], S is the prefix sum of zero-centred emissions (section 2.A, 2.C), and
 * the library returns log Z, its exact gradients (section 2.C: checkpointed
 * streaming forward-backward with local recompute) and the Viterbi segmentation.
 *
 * Shapes (all row-major, contiguous, last index fastest):
 *   x          float32 [B, T, C]    emissions; positions t >= L_b are never read
 *   lengths    int32   [B]          L_b in [1, T]  (checked on the device)
 *   S          float64 [B, T+1, C]  prefix sums of centred emissions
 *   nu         float64 [B, C]       centring baseline (mean over t < L_b)
 *   A          float32 [C, C]       transition score, A[from, to]
 *   D          float32 [K, C]       duration bias, row d-1 for duration d
 *   logZ       float64 [B]
 *   grad_logZ  float64 [B]          upstream weights g_b, or NULL for all ones
 *   dX         float32 [B, T, C]    g_b * dlogZ_b/dx (through S and nu); 0 for t >= L_b
 *   dA         float64 [C, C]       sum_b g_b dlogZ_b/dA
 *   dD         float64 [K, C]       sum_b g_b dlogZ_b/dD
 *   score      float64 [B]          Viterbi score (or a gold segmentation's score)
 *   labels     int32   [B, T]       label per position (Viterbi output, or a gold
 *                                   segmentation's input); -1 for t >= L_b in outputs
 *   seg_start  uint8   [B, T]       1 where a segment begins, else 0
 *   mu         float32 [B, T, C]    posterior coverage P(position lies in a segment of label c)
 *   pstart     float32 [B, T]       posterior probability that a segment begins at t
 *
 * Ownership and execution: every data pointer is caller-owned DEVICE memory
 * (except where a function says otherwise).  The library allocates nothing and
 * frees nothing.  Every call is asynchronous on the caller's CUDA stream, passed
 * as an opaque pointer (a cudaStream_t; NULL is the legacy default stream), and
 * returns after launching.  Only semicrf_get_device_status synchronises.
 *
 * Workspace: the caller provides `ws` of at least semicrf_workspace_bytes(dims,
 * what) bytes, 256-byte aligned.  The same workspace must be passed unchanged
 * from semicrf_forward to semicrf_backward (it holds the checkpoints and the
 * log-normaliser).  semicrf_prefix_scan also uses it (scratch for chunk sums).
 *
 * Errors: argument checks happen on the host before any launch and return a
 * status; nothing is launched then.  Device-side findings (a length outside
 * [1, T], a non-finite log Z) are recorded in the workspace's status word and
 * read back by semicrf_get_device_status.  Outputs of a call that found an
 * error are unspecified.
 */
#ifndef SEMICRF_H
#define SEMICRF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SEMICRF_OK = 0,
    SEMICRF_ERR_INVALID_ARG = 1,        /* null pointer, non-positive size, bad flag   */
    SEMICRF_ERR_UNSUPPORTED_SHAPE = 2,  /* K or C beyond the compiled limits           */
    SEMICRF_ERR_WORKSPACE_TOO_SMALL = 3,
    SEMICRF_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed        */
    SEMICRF_ERR_DEVICE_TIMEOUT = 5,     /* a bounded device-side wait expired          */
    SEMICRF_ERR_DEVICE_RANGE = 6,       /* device saw a non-finite normaliser          */
    SEMICRF_ERR_INVALID_LENGTH = 7,     /* device saw a length outside [1, T]          */
    SEMICRF_ERR_INVALID_SEGMENTATION = 8 /* device saw a malformed gold segmentation   */
} semicrf_status;

/* Problem dimensions.  ckpt_interval is the checkpoint spacing Delta in positions
 * (0 selects ceil(sqrt(T))); results do not depend on it. */
typedef struct {
    int32_t B, T, K, C;
    int32_t ckpt_interval;
} semicrf_dims;

/* what: which calls the workspace serves (a TRAIN or VITERBI workspace also
 * serves prefix_scan) */
#define SEMICRF_WS_TRAIN 0   /* prefix_scan + forward + backward */
#define SEMICRF_WS_VITERBI 1 /* prefix_scan + viterbi            */
#define SEMICRF_WS_SCAN 2    /* prefix_scan only                 */

/* Compiled limits (SEMICRF_ERR_UNSUPPORTED_SHAPE beyond them). */
#define SEMICRF_MAX_C 256
#define SEMICRF_MAX_K 4096

/*
 * Bytes of device workspace needed for `what` at these dims; 0 if the dims are
 * invalid or unsupported (semicrf_check_dims says which).
 */
size_t semicrf_workspace_bytes(const semicrf_dims *dims, int32_t what);

/* Host check of dims alone (no CUDA calls). */
semicrf_status semicrf_check_dims(const semicrf_dims *dims);

/*
 * Centring and prefix scan (technical summary 2.A and 2.C):
 *   nu[b,c]    = (1/L_b) sum_{t<L_b} x[b,t,c]
 *   S[b,0,c]   = 0,  S[b,t+1,c] = S[b,t,c] + x[b,t,c] - nu[b,c]  (t < L_b)
 *   S[b,t,c]   = S[b,L_b,c] for t > L_b
 * Accumulates in float64; x rows t >= L_b are not read.
 */
semicrf_status semicrf_prefix_scan(const semicrf_dims *dims, const float *x,
                                   const int32_t *lengths, double *S, double *nu,
                                   void *ws, size_t ws_bytes, void *stream);

/*
 * The same centring and prefix scan without a workspace, for callers that are
 * given only their input and output buffers (a plugin or custom-op interface
 * with no workspace hook) or that cannot call cudaMalloc under a fixed memory
 * budget.  The pages have no counterpart to this entry point.
 * Scratch: a library-owned static device array of 1 MiB (+256 bytes), held by
 * every GPU that loads the library until exit; requires B*C <= 131072
 * (SEMICRF_ERR_UNSUPPORTED_SHAPE otherwise).  Allocates nothing.  The first call
 * on a device looks up the array's device address (make it before any stream
 * capture) and keeps it for the life of the process, so after cudaDeviceReset
 * on a device this entry point must not be called on that device again.  All
 * calls share the array: calls issued in order on one stream are safe; calls
 * that can overlap on the GPU (different streams, or host threads without an
 * ordering between their streams) race and must be serialised by the caller.
 * Device-side length errors are not reported by this entry point (such
 * sequences are skipped).
 */
semicrf_status semicrf_prefix_scan_noalloc(const semicrf_dims *dims, const float *x,
                                           const int32_t *lengths, double *S, double *nu,
                                           void *stream);

/*
 * Streaming forward (abstract: prefix-sum lookup instead of an edge tensor;
 * technical summary 2.B-2.C: O(K*C) ring of forward messages, normalised
 * checkpoints every ckpt_interval positions).  Writes logZ[b] and keeps the
 * checkpoints and log-normaliser in ws for semicrf_backward.
 */
semicrf_status semicrf_forward(const semicrf_dims *dims, const double *S, const float *A,
                               const float *D, const int32_t *lengths, double *logZ,
                               void *ws, size_t ws_bytes, void *stream);

/*
 * Backward (technical summary 2.C: recompute the forward messages inside each
 * checkpoint segment, stream the backward messages through a K*C ring, form the
 * segment and transition marginals).  Overwrites dX, dA, dD with the exact
 * gradients of sum_b g_b logZ_b, where g = grad_logZ (NULL: ones).  ws must be the
 * workspace the matching semicrf_forward call used.
 */
semicrf_status semicrf_backward(const semicrf_dims *dims, const double *S, const float *A,
                                const float *D, const int32_t *lengths,
                                const double *grad_logZ, void *ws, size_t ws_bytes,
                                float *dX, double *dA, double *dD, void *stream);

/*
 * Forward and backward in one call: log Z and the gradients of semicrf_backward
 * (weights grad_logZ, NULL: ones), without checkpoints.  The forward chain and
 * the backward (beta) chain run side by side -- the backward chain needs only
 * S, A, D and the lengths -- and each stores its per-position rows; the
 * marginals, coverage and parameter gradients are then parallel passes over
 * them (technical summary 2.C computes the same quantities by checkpointed
 * recompute, which semicrf_forward / semicrf_backward keep for callers that
 * split the two).  Same workspace kind and outputs as the pair; the result
 * equals theirs up to rounding order.
 */
semicrf_status semicrf_forward_backward(const semicrf_dims *dims, const double *S, const float *A,
                                       const float *D, const int32_t *lengths, const double *grad_logZ,
                                       void *ws, size_t ws_bytes, double *logZ, float *dX, double *dA,
                                       double *dD, void *stream);

/*
 * One forward/backward step from host memory, for callers whose inputs and
 * results live on the host: copies x, A, D, lengths (and grad_logZ unless
 * NULL) to the device, runs semicrf_prefix_scan and semicrf_forward_backward,
 * and copies logZ, dA, dD (and dX unless dX is NULL) back, all on `stream`
 * with one cudaMemcpyAsync per array.  Asynchronous: the host outputs hold the
 * results once the stream has synchronised.  The host buffers should be pinned
 * (cudaHostAlloc / cudaHostRegister) for the copies to run asynchronously;
 * pageable buffers work, but then the copies block the calling thread.
 * stage: caller-owned device memory of semicrf_host_stage_bytes(dims) bytes,
 * 256-byte aligned, for the device copies, S and the device outputs (its
 * regions: x, A, D, lengths, grad, S, nu, logZ, dX, dA, dD, each 256-byte
 * aligned, so the results also stay readable there).  ws as for
 * semicrf_forward_backward.  Errors: those of the two calls, plus
 * SEMICRF_ERR_WORKSPACE_TOO_SMALL for a short stage and SEMICRF_ERR_CUDA for a
 * failed copy.  semicrf_last_launch_count reports the kernels of both calls.
 */
size_t semicrf_host_stage_bytes(const semicrf_dims *dims);
semicrf_status semicrf_forward_backward_host(const semicrf_dims *dims, const float *x, const float *A,
                                            const float *D, const int32_t *lengths, const double *grad_logZ,
                                            double *logZ, float *dX, double *dA, double *dD, void *stage,
                                            size_t stage_bytes, void *ws, size_t ws_bytes, void *stream);

/*
 * Viterbi: the forward recursion in (max, +), float64.  Ties pick the smallest
 * duration, then the smallest previous label; the final label is the smallest
 * reaching the maximum.  (The pages do not describe decoding; this follows the
 * same segment score.)
 */
semicrf_status semicrf_viterbi(const semicrf_dims *dims, const double *S, const float *A,
                               const float *D, const int32_t *lengths, double *score,
                               int32_t *labels, uint8_t *seg_start, void *ws,
                               size_t ws_bytes, void *stream);

/*
 * Posterior marginals (abstract: uncertainty estimates at segment boundaries;
 * technical summary 2.C: the marginals the backward pass forms):
 *   mu[b,u,c]   = P(position u lies in a segment labelled c)    (u < L_b; 0 beyond)
 *   pstart[b,t] = P(a segment begins at t) = sum_c P(a segment of label c begins at t)
 *                 (t < L_b; 0 beyond; pstart[b,0] = 1)
 * Either output may be NULL.  Runs the recompute and backward passes of
 * semicrf_backward on the forward's workspace (pass ws unchanged from the
 * matching semicrf_forward) and forms no parameter gradients.
 */
semicrf_status semicrf_posteriors(const semicrf_dims *dims, const double *S, const float *A,
                                  const float *D, const int32_t *lengths, void *ws,
                                  size_t ws_bytes, float *mu, float *pstart, void *stream);

/*
 * Score of given ("gold") segmentations, the term the training loss subtracts
 * from log Z (technical summary section 3: negative log-likelihood
 * log Z - score(y*)).  Segment i of sequence b starts at a position s with
 * seg_start[b,s] = 1 (seg_start[b,0] must be 1), ends at the next start or at
 * L_b, has length at most K and label c = labels[b,s], which every position of
 * the segment must carry (0 <= c < C).  Then
 *   score[b] = sum_i (S[b,e_i,c_i] - S[b,s_i,c_i] + D[e_i-s_i-1,c_i]) + sum_{i>=2} A[c_{i-1},c_i].
 * A malformed segmentation records SEMICRF_ERR_INVALID_SEGMENTATION in the
 * workspace status (its score is then unspecified).  ws: a SEMICRF_WS_TRAIN
 * workspace (its status word and count buffers are used).
 */
semicrf_status semicrf_gold_score(const semicrf_dims *dims, const double *S, const float *A,
                                  const float *D, const int32_t *lengths, const int32_t *labels,
                                  const uint8_t *seg_start, double *score, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Gradient of sum_b g_b score[b] (g = grad_score, NULL: ones) for the same
 * segmentations, ADDED to dX, dA, dD (so that after semicrf_backward with
 * weights g and this call with weights -g they hold the gradient of the
 * negative log-likelihood):
 *   dX[b,u,c] += g_b (1[u lies in a segment labelled c] - n_{b,c} / L_b)   (u < L_b)
 *   dA[c',c]  += sum_b g_b * (number of c' -> c transitions in b)
 *   dD[d-1,c] += sum_b g_b * (number of segments of length d and label c in b)
 * where n_{b,c} counts the positions labelled c (the path through nu).  Checks
 * the segmentations as semicrf_gold_score does.
 */
semicrf_status semicrf_gold_backward(const semicrf_dims *dims, const int32_t *lengths,
                                     const int32_t *labels, const uint8_t *seg_start,
                                     const double *grad_score, float *dX, double *dA, double *dD,
                                     void *ws, size_t ws_bytes, void *stream);

/*
 * Training objective (technical summary section 3: training by negative
 * log-likelihood): nll[b] = log Z_b - score_b(y*) for the gold segmentations
 * given as for semicrf_gold_score.  Runs semicrf_forward (log Z into logZ, the
 * checkpoints into ws) and the gold score (into score), and forms nll on the
 * device.  Errors and device findings as for those two calls.
 */
semicrf_status semicrf_nll(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                           const int32_t *lengths, const int32_t *labels, const uint8_t *seg_start,
                           double *logZ, double *score, double *nll, void *ws, size_t ws_bytes, void *stream);

/*
 * Gradient of sum_b g_b nll[b] (g = grad_nll, NULL: ones) with respect to the
 * emissions (through S and nu), A and D, OVERWRITING dX, dA, dD: semicrf_backward
 * with weights g, then the gold-segmentation counts with weights -g.  ws must be
 * the workspace of the matching semicrf_nll call.
 */
semicrf_status semicrf_nll_backward(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                                    const int32_t *lengths, const int32_t *labels, const uint8_t *seg_start,
                                    const double *grad_nll, void *ws, size_t ws_bytes, float *dX, double *dA,
                                    double *dD, void *stream);

/* Zero the device status word in ws (asynchronous on stream). */
semicrf_status semicrf_clear_device_status(void *ws, void *stream);

/*
 * Synchronise `stream`, read the device status word from ws and return it
 * (SEMICRF_OK when no device-side error was recorded).
 */
semicrf_status semicrf_get_device_status(const void *ws, void *stream);

/* Static, human-readable name of a status. */
const char *semicrf_status_string(semicrf_status s);

/*
 * Launch geometry of the sequential chains for these dims, for tuning and
 * diagnostics (no counterpart on the pages).  path: 0 the forward_backward
 * step (forward and backward chains in one launch), 1 semicrf_forward,
 * 2 semicrf_backward.  The geometry is the one the launch uses: the cheapest by
 * the library's cost model among those of which the current device holds all
 * of the launch's clusters at once (the cheapest overall if none does).
 * Fills info[0..8] (n >= 9):
 *   info[0]  kernel family: 0 = one CTA per sequence (C <= 32 and K <= 32),
 *            1 = one thread-block cluster per chain
 *   info[1]  CTAs per cluster G      info[2] threads per CTA
 *   info[3]  labels per CTA          info[4] transition lanes per label
 *   info[5]  window lanes per label  info[6] dynamic shared memory per CTA (bytes)
 *   info[7]  clusters of this shape the current device can hold at once
 *            (-1 when not queried or when the CUDA query fails)
 *   info[8]  clusters the launch needs (2B for path 0, else B)
 * Family 0 fills info[0], info[1] = 1, info[7] = -1 and info[8] only.  Host
 * only, except the occupancy query (a CUDA runtime call, no launch).
 */
semicrf_status semicrf_chain_plan(const semicrf_dims *dims, int32_t path, int32_t *info, int32_t n);

/* Kernel launches issued by the most recent successful call on this thread. */
int32_t semicrf_last_launch_count(void);

/*
 * Per-kernel timing for profilers and benchmarks.  `events` points to n
 * caller-created cudaEvent_t handles (host array; the library keeps the pointer,
 * so it must stay valid while set).  While set, each API call on this thread
 * records events[2i] just before and events[2i+1] just after its i-th kernel
 * launch (i < n/2), on the call's stream.  Pass NULL, 0 to stop.
 */
semicrf_status semicrf_set_profile_events(void *const *events, int32_t n);

#ifdef __cplusplus
}
#endif

#endif /* SEMICRF_H */
