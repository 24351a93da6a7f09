// semicrf_internal.h -- host-side launch plan, workspace layout and launcher
// declarations shared by the translation units of libsemicrf.so.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "semicrf.h"

namespace semicrf {

// Ring columns are rebased (scaled by an exact power of two) when the weighted
// column sum leaves [2^-kRebaseBits, 2^kRebaseBits].  Within one step a column's
// newest entry moves by a bounded factor (transition, duration and one emission
// term), so with 512 bits every product formed in a step stays far inside the
// float64 range (2^+-1022).
constexpr int kRebaseBits = 512;
constexpr int kMaxThreads = 512;
constexpr size_t kSmemBudget = 220 * 1024;

// Per-sequence log-normaliser of the forward pass: log Z = ln2 * k + logn.
struct LogZState {
    double logn;
    int32_t k;
    int32_t pad;
};

// How one sequence is spread over a thread-block cluster.  CTA g of the cluster
// owns labels [g*Cg, min(C, (g+1)*Cg)).  Inside a CTA thread tid works on label
// column lc = tid % Cg and lane j = tid / Cg (j < JL); lane j handles durations
// d = 1 + j + m*JL (m < DPT) and previous/next labels j + m*JL (m < CPT).
struct Plan {
    int G = 0, NT = 0, Cg = 0, JL = 0, DPT = 0, CPT = 0;
    size_t smem_fwd = 0, smem_bwd = 0, smem_vit = 0;
    bool ok() const { return G > 0; }
};

// Byte offsets of every region inside the caller's workspace.
struct Layout {
    int delta = 0;   // checkpoint interval
    int J = 0;       // checkpoints per sequence (ceil(T / delta))
    int NCH = 0;     // prefix-scan chunks per sequence
    size_t status = 0;      // int32[4]
    size_t scan = 0;        // double [B][NCH][C]
    size_t logz = 0;        // LogZState [B]
    size_t ckpt = 0;        // [B][J] records of ckpt_stride bytes
    size_t ckpt_stride = 0; // ring double[K*C], r int32[C], two normaliser exponents int32
    // Recomputed forward quantities per position t and label c, as mantissa and
    // power-of-two exponent relative to Z:
    //   exp(at[t,c] - S[t,c] - log Z) = cU * 2^eU,   exp(al[t,c] - log Z) = cA * 2^eA
    // exp(S[t,c]) split as es * 2^m with |log es| <= ln2/2 (es, 1/es, m per position)
    size_t tES = 0;         // double [B][T+1][C]  exp(s)
    size_t tIES = 0;        // double [B][T+1][C]  exp(-s)
    size_t tM = 0;          // int32  [B][T+1][C]  m
    size_t cU = 0;          // double [B][T+1][C]
    size_t cA = 0;          // double [B][T+1][C]
    size_t eU = 0;          // int32  [B][T+1][C]
    size_t eA = 0;          // int32  [B][T+1]
    size_t accD = 0;        // double [B][K][C]
    size_t accA = 0;        // double [B][C][C]
    // Cluster-kernel backward rows, consumed by the parameter-gradient kernels:
    //   V[t,c] = exp(ga[t,c] + S[t,c] - ln2 rb[t,c]) at the reference rb it was written at,
    //   bp[s,c] = exp(be[s,c] - ln2 kb[s]) (normalised beta), kb[s] the backward normaliser.
    size_t Vst = 0;         // double [B][T+1][C]
    size_t rbst = 0;        // int32  [B][T+1][C]
    size_t bpst = 0;        // double [B][T+1][C]
    size_t kbst = 0;        // int32  [B][T+1]
    int nsD = 0, nsA = 0;   // partial-sum splits of the dD and dA contractions
    int npost = 0;          // CTAs of the C, K <= 32 post pass (team_post.cu), 0 otherwise
    size_t partD = 0;       // double [max(nsD, npost)][K][C]
    size_t partA = 0;       // double [max(nsA, npost)][C][C]
    size_t stst = 0;        // double [B][T+1][C]  P(segment of label c starts at s) (posteriors)
    size_t gcA = 0;         // int32  [B][C][C]    gold transition counts
    size_t gcD = 0;         // int32  [B][K][C]    gold duration counts
    size_t gcN = 0;         // int32  [B][C]       gold positions per label
    size_t covd = 0;        // double [B][ceil(T/cov_chunk(T))][C]  coverage chunk totals
    size_t covm = 0;        // double [B][ceil(T/32)][C]  coverage chunk sums over positions
    size_t musum = 0;       // double [B][C]
    size_t mures = 0;       // double [B][C]
    size_t logzb = 0;       // double [B]
    size_t bd = 0;          // uint16 [B][T+1][C]  Viterbi best duration
    size_t bc = 0;          // uint16 [B][T+1][C]  Viterbi best previous label
    size_t vfin = 0;        // int32 [B]           Viterbi final label
    size_t total = 0;
};

// Streaming multiprocessors of the current device (cached per device; 148, the
// B200 count, when no device can be queried, e.g. on a host without a GPU).
int device_sm_count();

// Optional per-launch event recording (semicrf_set_profile_events).
void prof_before(cudaStream_t st);
void prof_after(cudaStream_t st);
void prof_reset();
// Sets what semicrf_last_launch_count reports for this thread.
void record_launches(int n);

Plan make_plan(int K, int C);
bool make_layout(const semicrf_dims &d, int what, const Plan &p, Layout *out);
int default_delta(int T);

// Launchers: return cudaSuccess or the launch error.
struct ScanArgs {
    int B, T, C, NCH;
    const float *x;
    const int32_t *lengths;
    double *S, *nu, *part;
    int32_t *status;
};
cudaError_t launch_prefix_scan(const ScanArgs &a, cudaStream_t st, int *launches);

struct FbArgs {
    int B, T, K, C, delta, J;
    const double *S;
    const float *A, *D;
    const int32_t *lengths;
    const double *grad;
    double *logZ;
    LogZState *lz;
    unsigned char *ckpt;
    size_t ckpt_stride;
    double *cU, *cA;
    int32_t *eU, *eA;
    double *tES, *tIES;
    int32_t *tM;
    double *accD, *accA, *musum, *mures, *logzb;
    double *Vst, *bpst, *partD, *partA;
    int32_t *rbst, *kbst;
    int nsD, nsA, npost;
    double *stst;   // when set, the backward stores the start marginals (posteriors)
    double *covd, *covm;
    int covch;
    float *dX;
    double *dA, *dD;
    int32_t *status;
};
// Cluster kernels (fb_cluster.cu): G CTAs per sequence, Cg labels per CTA.  In a
// CTA the first NWO warps are owner warps (one lane per label runs its chain),
// the next NWT warps transition warps (LPL lanes per label, CPL terms per lane),
// the next NWW warps window warps (LPW lanes per label; PW partial sums per label
// when LPW > 32).
// RS is the shared-memory row stride (doubles) of the ring, duration-weight and
// duration-accumulator arrays, chosen so that the 16 lanes of a half-warp's
// window loads (16/LPW labels x LPW consecutive rows) fall in distinct banks.
// GP is the pitch of the exchanged values: G blocks of Cg labels each padded to
// an even count (16-byte units for the owners' bulk copies), zeros in the
// padding and past the last block, at least the positions the transition lanes
// read, so they read without bounds tests.
// NRB: rows per window lane read with the weights in registers (8, 16 or 32;
// 0: the weights stay in shared memory); PAD: zero ring rows before and after
// the ring for the rows a window lane reads past the window.  TS (clusters): 1 =
// the transition lanes form each position's value as soon as their sum is done
// and store it into every CTA with st.async, and all window lanes share the
// rescale of rebased labels (plans with at least four transition warps: many
// labels per CTA, a long sum); 0 = the owners form the value and bulk-copy it,
// and each label's window lanes rescale its rows.
struct ClGeom {
    int G = 0, Cg = 0, LPL = 0, CPL = 0, LPW = 0, PW = 0, NWO = 0, NWT = 0, NWW = 0, NT = 0, RS = 0, GP = 0;
    int NRB = 0, PAD = 0, TS = 0;
};
bool cl_plan(int K, int C, bool bwd, ClGeom *out);
cudaError_t launch_cl_forward(const FbArgs &a, cudaStream_t st, bool recompute);
cudaError_t launch_cl_backward(const FbArgs &a, cudaStream_t st);
// Forward storing its rows and the beta chain in one launch (2B clusters).
cudaError_t launch_cl_fused(const FbArgs &a, cudaStream_t st);
// Planner's choice for path 0 (fused), 1 (forward) or 2 (backward) and how many
// such clusters the GPU holds at once (see semicrf_chain_plan).
bool cl_plan_info(int K, int C, int B, int path, int32_t *info);
// dD and dA from the cluster backward's stored rows (cl_grads.cu): two contraction
// kernels writing split partial sums, one kernel reducing them (3 launches).
constexpr int kGradChunk = 64;   // start positions per staged chunk
void cl_grad_splits(int B, int T, int K, int C, int *nsD, int *nsA);
cudaError_t launch_cl_param_grads(const FbArgs &a, cudaStream_t st);
// After the forward stored its rows unscaled (fused path): the recompute's scaling.
cudaError_t launch_rows_rescale(const FbArgs &a, cudaStream_t st);
// Coverage mu (raw, into dX) and its per-label sum (musum) from the stored rows (4 launches),
// in chunks of cov_chunk(T) positions.
inline int cov_chunk(int T)
{
    int ch = 32;
    while ((long long)ch * 1024 < T) ch *= 2;
    return ch;
}
cudaError_t launch_coverage(const FbArgs &a, cudaStream_t st);
// C, K <= 32: dD, dA, the coverage and dX from the stored rows in two launches
// (team_post.cu): npost CTAs over (sequence, 32-position) items, then the finalise.
int team_post_splits(int B, int T);
int team_post_chunks(int T);
cudaError_t launch_team_post(const FbArgs &a, cudaStream_t st);
// Forward and backward chains side by side, then the parallel passes (fused path).
cudaError_t launch_forward_backward(const FbArgs &a, cudaStream_t st, int *launches);

// Warp-per-sequence kernels for C <= 32, K <= 32 (kind 0 forward, 1 recompute, 2 backward,
// 3 forward storing its rows beside the beta chain).
bool small_path_ok(int K, int C);
cudaError_t launch_small(const FbArgs &a, cudaStream_t st, int kind);

// exp tables of S (tES, tIES, tM) for every position; fully parallel, HBM-bound.
cudaError_t launch_exp_tables(const FbArgs &a, cudaStream_t st);

cudaError_t launch_forward(const Plan &p, const FbArgs &a, cudaStream_t st, int *launches);
cudaError_t launch_backward(const Plan &p, const FbArgs &a, cudaStream_t st, int *launches);

struct VitArgs {
    int B, T, K, C;
    const double *S;
    const float *A, *D;
    const int32_t *lengths;
    double *score;
    int32_t *labels;
    uint8_t *seg_start;
    uint16_t *bd, *bc;
    int32_t *vfin;
    int32_t *status;
};
cudaError_t launch_viterbi(const Plan &p, const VitArgs &a, cudaStream_t st, int *launches);

// Posterior marginals: the recompute and backward chains with a.dX = mu (raw
// coverage, or NULL) and a.stst set, then one kernel for pstart and the padding.
cudaError_t launch_posteriors(const FbArgs &a, float *mu, float *pstart, cudaStream_t st, int *launches);

// Gold segmentations (gold.cu).
struct GoldArgs {
    int B, T, K, C;
    const double *S;
    const float *A, *D;
    const int32_t *lengths, *labels;
    const uint8_t *seg_start;
    const double *grad;   // backward weights, NULL: ones
    double wsign;         // the weights are wsign * grad[b] (wsign * 1 when grad is NULL)
    double *score;
    const double *logZ;   // when set with nll: nll[b] = logZ[b] - score[b]
    double *nll;
    float *dX;
    double *dA, *dD;
    int32_t *cntA, *cntD, *cntN;
    int32_t *status;
};
cudaError_t launch_gold_score(const GoldArgs &a, cudaStream_t st, int *launches);
cudaError_t launch_gold_backward(const GoldArgs &a, cudaStream_t st, int *launches);

}  // namespace semicrf
