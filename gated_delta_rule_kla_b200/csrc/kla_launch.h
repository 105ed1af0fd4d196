// kla_launch.h -- internal launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace kla {

constexpr int kChunkLen = 64;  // the only chunk length the library accepts

struct DecodeArgs {
    const void *q, *k, *v;
    const float *eta, *g;
    float eps;
    float* S;
    void* o;
    int B, H, Dk, Dv;
    bool bf16;      // q, k, v are bf16 (else fp32)
    bool out_bf16;  // o is bf16 (else fp32)
    bool inject_timeout;  // failure injection: every CTA's first wait expires (nothing is stored)
    bool diag = false;    // g is [B, H, Dk]: one log-decay per key channel (diagonal gating)
};

struct FwdArgs {
    const void *q, *k, *v;
    const float *eta, *g;
    float eps;
    const float* S0;  // may be null (zero state)
    void* o;          // may be null
    float* S_T;       // may be null; may alias S0
    float* S_chunks;  // may be null
    int B, T, H, Dk, Dv;
    bool bf16;      // q, k, v are bf16 (else fp32)
    bool out_bf16;  // o is bf16 (else fp32)
    // Segmented long-sequence mode (split state pass only).  nseg > 1 splits each sequence
    // into nseg runs of seg_chunks chunks processed by separate CTAs; S0 and S_T then index
    // [B*H, nseg, Dk, Dv] (S_T: [kinds, B*H, nseg, Dk, Dv]) and a second grid row (kind 1)
    // runs each segment from the identity state with zero values (the segment's transition).
    int nseg, seg_chunks, kinds;
    // Extra outputs of the split path for the tensor-core backward (all may be null), per chunk
    // and head as bf16 hi then lo tile images in the 128-byte swizzle:
    //   T_tiles  16 KB  T = (I + L)^{-1}: [64 rows of T][64]                   (preparation kernel)
    //   S_tiles  64 KB  the chunk's incoming state: [dk half][128 dv rows][64 dk]     (state pass)
    //   U_tiles  32 KB  U = T (Diag(c) V - Diag(b gamma) Khat S): [128 dv rows][64 tokens]
    void* T_tiles;
    void* S_tiles;
    void* U_tiles;
    // First chunk of a non-segmented state-pass run of seg_chunks chunks (0 for a whole
    // sequence): the host splits a sequence into slabs handled by consecutive runs.
    int chunk0;
    // Diagonal-gated split forward: also store what the backward needs in each record (the Gram
    // A, the inverse T and the per-channel log-decay prefix G of every 16-token chunk).
    bool rec_extras = false;
    // Tensor-core split forward with diagonal gating: g is [B, T, H, Dk] (one log-decay per key
    // channel) and each chunk's record also holds Q o Gam and the next chunk's per-channel
    // decay (the split path's entry points choose it; the CUDA-core kernels do not read it).
    bool diag = false;
};

struct BwdArgs {
    const void *q, *k, *v;
    const float *eta, *g;
    float eps;
    const float* S_chunks;  // [B,H,NC,Dk,Dv], required here
    const void* dO;
    const float* dS_T;  // may be null
    void *dq, *dk, *dv;
    float *deta, *dg, *dS0;
    // fp32 accumulators (zeroed by the launcher): [B,T,H,Dk] x2, [B,T,H] x3
    float *acc_dq, *acc_dkh, *acc_db, *acc_dc, *acc_dG;
    int B, T, H, Dk, Dv;
    bool bf16;      // q, k, v, dO are bf16 (else fp32)
    bool out_bf16;  // dq, dk, dv are bf16 (else fp32)
};

// Tensor-core backward (bf16 inputs, Dk == Dv == 128).
struct BwdTcArgs {
    const void *q, *k, *v;
    const float *eta, *g;
    float eps;
    const float* S0;        // may be null (zero state)
    const void* dO;         // bf16, [B,T,H,Dv]
    const float* dS_T;      // may be null
    const float* S_chunks;  // may be null (then recomputed into the workspace)
    void *dq, *dk, *dv;
    float *deta, *dg, *dS0;
    int B, T, H;
    bool out_bf16;
};
// Workspace bytes of the tensor-core backward: the split forward's records and, per chunk and
// head, T (16 KB), U (32 KB), lambda (64 KB), dR (32 KB) and, without S_chunks, S (64 KB).
size_t chunk_bwd_tc_workspace(int B, int T, int H, bool have_S_chunks);
cudaError_t launch_chunk_bwd_tc(const BwdTcArgs& a, void* ws, size_t ws_bytes, cudaStream_t st);
// The two halves of launch_chunk_bwd_tc for a training step: the forward (o and S_T as `f` asks,
// plus the backward's records and tiles in ws), then the backward from that ws.
cudaError_t launch_chunk_fwd_train_tc(const FwdArgs& f, void* ws, size_t ws_bytes, cudaStream_t st);
cudaError_t launch_chunk_bwd_tc_reverse(const BwdTcArgs& a, void* ws, size_t ws_bytes, cudaStream_t st);
cudaError_t bwd_tc_take_error(cudaStream_t st, unsigned int* flag);

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

// Gate prologue: eta = sigmoid(z[:, :H]), g = -softplus(z[:, H:]) with z = x W^T + bias, and
// (when q is given) qhat = q / ||q|| per (token, head).  x [N, D], W [2H, D], q/qhat [N, H, Dk]
// in the input type; bias [2H], eta, g [N, H] fp32.
struct GateArgs {
    const void *x, *W;
    const float* bias;
    const void* q;  // may be null (then qhat is not written)
    float *eta, *g;
    void* qhat;
    int N, D, H, Dk;
    bool bf16;
};
// Backward of the prologue from its outputs eta, g and the upstream gradients; writes
// dx [N, D], dW [2H, D], dbias [2H], and dq [N, H, Dk] when q is given (all fp32).
struct GateBwdArgs {
    const void *x, *W;
    const float *eta, *g, *deta, *dg;
    const void* q;
    const float* dqhat;
    float *dx, *dW, *db, *dq;
    int N, D, H, Dk;
    bool bf16;
};
cudaError_t launch_gate_prologue(const GateArgs& a, cudaStream_t st);
size_t gate_bwd_workspace(int N, int D, int H);
cudaError_t launch_gate_prologue_bwd(const GateBwdArgs& a, void* ws, cudaStream_t st);
cudaError_t gates_take_error(cudaStream_t st, unsigned int* flag);
// Diagonal (per-key-channel) gating on CUDA cores: g is [B, T, H, Dk].  The kernels work in
// chunks of diag_chunk_len() tokens; S_chunks of the forward (optional) and of the backward
// (required: the workspace region the backward launcher fills first) are per such chunk.  The
// backward's acc_dG is [B, T, H, Dk]; every accumulator must be zeroed before the launch.
// With at least diag_fwd_workspace() bytes in ws the forward runs split: a chunk-parallel
// preparation kernel writes fp32 records there, then a sequential state pass reads them;
// otherwise one kernel per (head, 64 value columns) does everything.
int diag_chunk_len();
size_t diag_fwd_workspace(int B, int T, int H, int Dk, int Dv);
cudaError_t launch_chunk_fwd_diag(const FwdArgs& a, void* ws, size_t ws_bytes, cudaStream_t st);
cudaError_t launch_chunk_bwd_diag(const BwdArgs& a, const float* S0, void* rec_ws, size_t rec_bytes,
                                  cudaStream_t st);
cudaError_t diag_take_error(cudaStream_t st, unsigned int* flag);
cudaError_t launch_chunk_fwd_simt(const FwdArgs& a, cudaStream_t st);
cudaError_t launch_chunk_bwd_simt(const BwdArgs& a, cudaStream_t st);
// Tensor-core (tcgen05) forward for bf16 inputs with Dk == Dv == 128.
bool chunk_fwd_tc_supported(const FwdArgs& a);
cudaError_t launch_chunk_fwd_tc(const FwdArgs& a, cudaStream_t st);
// Sequential fp32 scan over segments: S_{s+1} = M_s S_s + N_s per head, recording each
// segment's start in Sstart [BH, nseg, Dk, Dv] (MN: [2, BH, nseg, Dk, Dv], N first) and the
// final state in S_T (may be null).
cudaError_t launch_seg_scan(const float* S0, const float* MN, float* Sstart, float* S_T, int BH, int nseg,
                            cudaStream_t st);
// Split tensor-core forward: a chunk-parallel preparation kernel writes every chunk's
// state-independent operands to the workspace, then a sequential state pass (segmented for
// long sequences over few heads).  Workspace bytes for these sizes (0: shapes not supported).
size_t chunk_fwd_split_workspace(const FwdArgs& a);
// Diagonal gating on the split tensor-core path (bf16, Dk = Dv = 128): a.diag must be set.
bool chunk_fwd_diag_tc_supported(const FwdArgs& a);
cudaError_t launch_chunk_fwd_split(const FwdArgs& a, void* ws, cudaStream_t st);
// Kernels one launch_chunk_fwd_split call launches (preparation and state passes).
int chunk_fwd_split_launches(const FwdArgs& a);
// The two stages of the split path: the chunk-parallel preparation (writes the per-chunk
// records into ws) and the state pass that reads them.  stage 0 runs the whole state pass;
// with parallel segments 1, 2 and 3 run its transition pass, segment scan and output pass
// alone (in that order they equal stage 0); with one run per head 3 runs it and 1, 2 do nothing.
cudaError_t launch_chunk_fwd_split_prep(const FwdArgs& a, void* ws, cudaStream_t st);
cudaError_t launch_chunk_fwd_split_state(const FwdArgs& a, void* ws, cudaStream_t st, int stage = 0);
// Parallel segments of the split path's state pass per head (1: one run per head).
int chunk_fwd_split_segments(const FwdArgs& a);
cudaError_t split_take_error(cudaStream_t st, unsigned int* flag);
// The side stream of the split path's two-slab schedules (one per device, created once).
cudaError_t split_side_stream(cudaStream_t* out);
// Newest chunks in the first of the backward reverse pass's two slabs (0: one run per head).
int bwd_slab_newest(int BH, int NC);
// Segments of the backward's reverse state pass for BH heads of NC chunks (1: one run per head);
// the forward state pass's cost model, which the reverse pass shares.
int reverse_nseg(int BH, int NC);
// Synchronise `st`, then read and clear the device error word of the tensor-core kernels
// (non-zero when a bounded wait expired).
cudaError_t tc_take_error(cudaStream_t st, unsigned int* flag);
cudaError_t decode_take_error(cudaStream_t st, unsigned int* flag);
// Record `msg` as the calling thread's last error (see kla_last_error) and return `status`.
int set_last_error(int status, const char* msg);

}  // namespace kla
