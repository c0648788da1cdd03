// gdn_internal.h -- kernel launchers shared by the C-ABI host code (gdn_api.cu).
// Not part of the public interface; see include/gdn.h for the operation and layouts.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

namespace gdn {

// Floor applied to log_alpha inside the chunkwise forward: exp(-40) < 5e-18,
// below float32 resolution of a state next to O(1) terms, and chunk-local
// log-decay sums stay small enough for float32 differences g_t - g_s.
constexpr float kLogAlphaFloor = -40.0f;

// Segment transfers of long sequences (the chunk-level parallelism of the
// forward) use a bound on how much a state entering a span of chunks can still
// matter at its end.  Over one token the state is multiplied on the right by
// alpha_t (I - beta_t k_t k_t^T), whose spectral norm is
// alpha_t max(1, |1 - beta_t |k_t|^2|) (the matrix is symmetric, with
// eigenvalue 1 - beta_t |k_t|^2 along k_t and 1 across it).  The product of
// these factors over a chunk, rho_C = gamma_C prod_t max(1, |1 - beta_t |k_t|^2|),
// bounds the chunk's transfer, and the product of rho_C over a span bounds the
// span's.  When that product is at most kNegligibleTransfer (e^-40), a state
// entering the span contributes at most e^-40 of its own norm (bounded by the
// paper's App. A.2 estimate) at the span's end: far below float32 resolution
// of the result.  Such spans need no exact transfer matrix.
constexpr float kNegligibleTransfer = 4.248354e-18f;  // e^-40

// Brackets one kernel launch with CUDA events on its stream while
// gdn_timing_start() recording is on (gdn_timing.cu); a no-op otherwise.
// Construct it right before the launch, in a scope that ends right after it.
class TimedLaunch {
  public:
    TimedLaunch(int kind, cudaStream_t stream);
    ~TimedLaunch();
    TimedLaunch(const TimedLaunch &) = delete;
    TimedLaunch &operator=(const TimedLaunch &) = delete;

  private:
    int kind_;
    cudaStream_t stream_;
    cudaEvent_t begin_ = nullptr, end_ = nullptr;
};

struct FwdProblem {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    void *out;
    float *S_final;
    int64_t B, T, H, dk, dv, chunk;
    int dtype;  // gdn_dtype
    // 1: q, k are not yet L2-normalised and log_alpha, beta hold the gate logits x_alpha,
    // x_beta (log alpha = -softplus(x_alpha), beta = sigmoid(x_beta)); only the two-kernel
    // forward takes this form, the others get the output of launch_input_stage()
    int raw_inputs = 0;
    // CUDA-core and two-kernel forwards: when set, the state entering every chunk is written
    // here, [B*H][chunks][dv][dk] float32 (the backward's checkpoints); the CUDA-core forward
    // then also accepts out == nullptr
    float *ckpt = nullptr;
    // grouped heads: H query heads share the memories of H / group key-value heads (k, v and the
    // gates have H / group heads; S0 / S_final stay per query head, expanded by the caller).
    // The two-kernel and the CUDA-core forwards take it.
    int group = 1;
    // two-kernel forward, for the tensor-core backward's recompute: checkpoints in bf16 instead of
    // float32, and T = (I + A)^{-1} of every chunk into t_out (bf16 [B*H*chunks][64][64], lower
    // triangle written; the caller zeroes the rest), or nullptr
    int ckpt_bf16 = 0;
    void *t_out = nullptr;
    // two-kernel forward with grouped heads: lead = group runs one memory per key-value head (the
    // transfers, prefix and chain of query heads hk * group only, with S0 / S_final, the segment
    // scratch and the checkpoints per key-value head) and writes U^T of every chunk into u_out
    // (bf16 [B * H / group][chunks][128][64]); the other query heads' outputs come from
    // launch_grouped_outputs.  1: every head runs its own chain.
    int lead = 1;
    void *u_out = nullptr;
};

struct DecodeProblem {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    float *S;
    void *out;
    int64_t B, H, dk, dv;
    int dtype;
    int raw_inputs = 0;  // as FwdProblem::raw_inputs
    int group = 1;       // grouped heads: H query heads, H / group key-value heads (and states)
};

// Input stage epsilon: x / sqrt(sum x^2 + kNormEps), so that a zero vector stays zero.
constexpr float kNormEps = 1e-12f;

// decode.cu
cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream);

// Device error words: set by a kernel whose bounded wait gave up (the kernel then aborts and
// returns); take_* reads and clears one.  status.cu holds the self-test's word and the wait.
bool take_split_timeout();
bool take_tc_timeout();
bool take_selftest_timeout();
cudaError_t launch_selftest_timeout(cudaStream_t stream);

// grouped.cu -- per-key-value-head states <-> per-query-head copies (grouped heads):
// dst[b, h] = src[b, h / group] for h < H, and dst[b, hk] = src[b, hk * group].
cudaError_t launch_expand_states(const float *src, float *dst, int64_t B, int64_t H, int group, int64_t n,
                                 cudaStream_t stream);
cudaError_t launch_pick_states(const float *src, float *dst, int64_t B, int64_t H, int group, int64_t n,
                               cudaStream_t stream);

// causal_conv.cu -- depthwise causal convolution over [B, T, C] (dtype), weights [C, W] float32,
// carried states [B, W - 1, C] float32 (either may be nullptr); W in 1..4.  state_out must not
// alias state_in when T > 128 (the host copies first).
cudaError_t launch_causal_conv(const void *x, const float *w, const float *state_in, void *y, float *state_out,
                               int64_t B, int64_t T, int64_t C, int W, int dtype, cudaStream_t stream);
// Up to three convolutions over the same (B, T) in one launch (the state is not written): tensor i is
// x[i] [B, T, C[i]] with weights w[i] [C[i], W] and carried inputs state_in[i] [B, W - 1, C[i]] (or
// nullptr), into y[i].  One launch when every tensor allows 16-byte words, else one per tensor.
cudaError_t launch_causal_conv3(const void *const x[3], const float *const w[3], const float *const state_in[3],
                                void *const y[3], const int64_t C[3], int njobs, int64_t B, int64_t T, int W, int dtype,
                                cudaStream_t stream);
// The carried state of the short convolution after a call of T tokens (the last W - 1 inputs, oldest
// first); state_out may equal state_in.
cudaError_t launch_conv_state_update(const void *x, const float *state_in, float *state_out, int64_t B, int64_t T,
                                     int64_t C, int W, int dtype, cudaStream_t stream);

// input_stage.cu -- the input stage as a pass of its own, for the forwards that do not fuse
// it: L2-normalised q, k (dtype of the problem) and log alpha, beta from the gate logits, for
// `rows` (token, head) rows of dk elements; outputs may not alias inputs.
cudaError_t launch_input_stage(const void *q, const void *k, const float *x_alpha, const float *x_beta, void *qn,
                               void *kn, float *log_alpha, float *beta, int64_t rows, int64_t dk, int dtype,
                               cudaStream_t stream);

// fwd_simt.cu -- float32 SIMT chunkwise forward, any supported (dk, dv, chunk).
cudaError_t launch_fwd_simt(const FwdProblem &p, int sm_count, cudaStream_t stream);

// bwd_simt.cu -- reverse mode of the forward (float32 CUDA cores, any supported shape).
struct BwdProblem {
    FwdProblem f;             // inputs and sizes (f.out, f.S_final unused)
    const void *d_out;        // [B, T, H, dv] dtype
    const float *dS_final;    // [B, H, dv, dk] or nullptr (zero)
    void *dq, *dk, *dv;       // [B, T, H, dk|dv] dtype
    float *dlog_alpha, *dbeta;  // [B, T, H]
    float *dS0;               // [B, H, dv, dk] or nullptr (not written)
};
size_t bwd_simt_workspace_bytes(const BwdProblem &p, int sm_count);
cudaError_t launch_bwd_simt(const BwdProblem &p, int sm_count, void *workspace, cudaStream_t stream);
// bwd_tc.cu -- the same reverse mode on the tensor cores (bf16, dk = dv = 128, chunk = 64, one head
// per memory): a forward recompute, a reverse chain over the chunks of each (b, h) and a
// chunk-parallel gradient pass.
bool bwd_tc_supported(const BwdProblem &p);
size_t bwd_tc_workspace_bytes(const BwdProblem &p, int sm_count);
cudaError_t launch_bwd_tc(const BwdProblem &p, int sm_count, void *workspace, cudaStream_t stream);
bool take_bwd_timeout();

// fwd_tc.cu -- tcgen05 chunkwise forward: bf16, dk = dv = 128, chunk = 64.
// Long sequences with few (b, h) are cut into segments: a transfer pass, a
// float32 prefix over segments and an output pass, with
// fwd_tc_workspace_bytes() of scratch (device memory, caller-provided).
bool fwd_tc_supported(const FwdProblem &p);
int fwd_tc_segments(const FwdProblem &p, int sm_count, bool paired_transfers);
size_t fwd_tc_workspace_bytes(const FwdProblem &p, int nseg);
cudaError_t launch_fwd_tc(const FwdProblem &p, int nseg, void *workspace, cudaStream_t stream);
// Entry states of segments 1..nseg-1 from the segment transfers, in float32.  Mflag (or nullptr)
// marks the transfer matrices that are negligible and were not written.  Without a table, heads
// (b, h) of nseg segments each; with one (device memory), `heads` rows {S0 index, first slot,
// steps, unused}.
cudaError_t launch_seg_prefix(const float *S0, const float *Bw, const float *Mw, const int *Mflag, float *S_entry,
                              int64_t heads, int nseg, cudaStream_t stream, const int4 *tab = nullptr);

// fwd_split.cu -- the same forward as two kernels: a chunk-parallel prep
// kernel writes P, T diag(beta), W^T and the gates of every chunk to the
// workspace, and a chain kernel runs the state recurrence and the outputs
// from them.  The workspace (fwd_split_workspace_bytes) holds 32.5 KB
// per chunk plus the segment scratch of fwd_tc_workspace_bytes.
bool fwd_split_supported(const FwdProblem &p);
size_t fwd_split_workspace_bytes(const FwdProblem &p, int nseg);
// The P and T diag(beta) tiles (bf16 [items][64][64] each) inside a two-kernel workspace.
void fwd_split_ws_tiles(void *workspace, int64_t items, void **p_tiles, void **tb_tiles);
// The gate records (float32 [items][132]) inside a two-kernel workspace.
const float *fwd_split_ws_gates(const void *workspace, int64_t items);
// grouped_out.cu -- outputs of the query heads hk * group + r (r = 1 .. group - 1) from the memory
// of key-value head hk that a lead = group two-kernel forward left behind: its bf16 checkpoints
// (ckpt, [B * Hkv][chunks][128][128]) and U^T (u, [B * Hkv][chunks][128][64]), with each query
// head's P tiles and gate records from that forward's workspace (p_tiles, gates):
// O^T = S (diag(gamma) Q)^T + U^T P^T.
cudaError_t launch_grouped_outputs(const FwdProblem &p, const void *ckpt, const void *u, const void *p_tiles,
                                   const float *gates, int sm_count, cudaStream_t stream);
bool take_grouped_timeout();
cudaError_t launch_fwd_split(const FwdProblem &p, int nseg, int sm_count, void *workspace, cudaStream_t stream);
// Packed variable-length sequences (p.B = 1, p.T = total tokens; cu_seqlens on the host, N + 1
// entries).  plan_packed builds the host tables: the chunk table over the packed tokens and the
// per-CTA work.  A sequence longer than the plan's segment length runs as segments, with segment
// transfers and a prefix as for fixed-length problems, so that one long sequence among short ones
// still spreads over the SMs.  GDN_SEGMENTS=k cuts the longest sequence into k segments (1: none).
struct PackedPlan {
    int64_t H = 0, chunks = 0;  // heads, packed chunks over all sequences
    int sm_count = 148;
    int seg_len = 0;            // chunks per segment (0: no sequence is cut)
    int64_t slots = 0;          // segment boundaries over all (sequence, head)
    int64_t n_chain = 0, n_transfer = 0, n_prefix = 0;  // CTAs of the three passes
    std::vector<uint8_t> tables;  // chunk table | chain | chain segments | transfers | prefix rows
    size_t off_chain = 0, off_seg = 0, off_transfer = 0, off_prefix = 0;
};
bool plan_packed(const int64_t *cu_seqlens, int64_t N, int64_t H, int sm_count, PackedPlan *plan);
size_t packed_workspace_bytes(const PackedPlan &plan);
cudaError_t launch_fwd_split_packed(const FwdProblem &p, const PackedPlan &plan, void *workspace,
                                    cudaStream_t stream);

}  // namespace gdn
