// gdr2_launch.h -- host-side launchers behind the C ABI (internal).
// Each returns cudaSuccess or the launch error; argument checks happen in
// gdr2_api.cu before any of these is called.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace gdr2 {

struct FwdArgs {
    int B, T, H, dk, dv;
    bool bf16;
    const void *q, *k, *v;
    const float *log_alpha;
    const void *b, *w;
    const float *S0;
    void *o;
    float *S_T;
    float *saved_states;
    void *workspace;   // chunk intermediates of the tensor-core path
    size_t workspace_bytes;
    unsigned *status;  // device status word
    const int *cu_seqlens;  // packed sequences: B = their number, T = total tokens (null = dense)
    int gates;              // kGate* bits: b and/or w one value per token-head
    // block epilogue on o (tensor-core path only): o / rms(o) * norm_weight (.) silu(out_gate)
    const void *out_gate;      // bf16, the layout of o, or null
    const float *norm_weight;  // [dv], or null for no norm
    float norm_eps;
    // backward's use of the tensor-core forward (dense, vector gates): the chunk kernel also
    // writes T and W of every task here; chunks_only leaves out the scan kernel
    unsigned char *bwd_ext = nullptr;
    bool chunks_only = false;
    // the fused forward's queue counter and task flags (fused_sync_bytes_for(tasks) bytes), when
    // the workspace has no room for them behind the slots; null: behind the slots, if it fits
    unsigned char *fused_sync = nullptr;
};

struct DecodeArgs {
    int N, H, dk, dv;
    bool bf16;
    const void *q, *k, *v;
    const float *log_alpha;
    const void *b, *w;
    float *S;
    void *o;
    unsigned *status;
    int gates;  // kGate* bits
};

struct BwdArgs {
    int B, T, H, dk, dv;
    bool bf16;
    const void *q, *k, *v;
    const float *log_alpha;
    const void *b, *w;
    const float *S0;
    const void *dO;
    const float *dS_T;
    const float *saved_states;
    void *gq, *gk, *gv;  // gradient outputs dq, dk, dv
    float *glog_alpha;
    void *gb, *gw;
    float *gS0;
    void *workspace;
    size_t workspace_bytes;
    unsigned *status;
    int gates = 0;  // kGate* bits: b (and db) and/or w (and dw) one value per token-head
};

// Block prologue (csrc/prologue.cu).
struct ConvArgs {
    int N, T, H, d, width;  // sequences (batches when dense), tokens, heads, channels per head, taps
    bool bf16, l2norm;
    float eps;
    const int *cu_seqlens;  // packed sequences, or null (dense [N, T, H, d])
    const void *x;
    const float *weight;    // [H * d][width]
    const void *state_in;   // [N][width - 1][H][d] or null
    void *state_out;        // same layout, or null
    void *y;
    unsigned *status;       // device status word
};

struct ActArgs {
    bool bf16;
    long long n_alpha, n_b, n_w;
    const void *a, *b_pre, *w_pre;
    float *log_alpha;
    void *b, *w;
};

// States entering the segments of split sequences (csrc/segments.cu).
struct SegArgs {
    int B, G, H, dk, dv;   // batch, segments, heads, state rows and columns
    const float *A;        // [B][G][H][dk][dk] segment transitions
    const float *Bst;      // [B][G][H][dk][dv] segment offsets (final states from zero)
    const float *S0;       // [B][H][dk][dv] or null (zeros)
    float *S_starts;       // [B][G][H][dk][dv] out: the state entering each segment
    float *S_T;            // [B][H][dk][dv] or null: the state after the last segment
};

cudaError_t launch_segment_states(const SegArgs &a, cudaStream_t s);

// The backward's first two steps as one cooperative launch (fwd_tc.cu): the forward's chunk
// tasks (backward instance, T and W to fa.bwd_ext; chunk-major from the last chunk) and the
// reverse scans of the state gradient. Runs only for dense sequences with saved chunk states
// (fa.chunks_only) where B H leaves 32 SMs to the chunk tasks; *launched says whether it ran.
struct BwdFrontArgs {
    const void *dO;       // [B][T][H][dv] bf16
    const float *dS_T;    // [B][H][dk][dv] or null
    float *gS0;           // [B][H][dk][dv] or null
    unsigned char *dsc;   // the dS'^T images, one per task
    unsigned char *sync;  // fused_sync_bytes_for(tasks) bytes: the queue counter and task flags
};
cudaError_t launch_backward_front_fused(const FwdArgs &fa, const BwdFrontArgs &r, cudaStream_t s, bool *launched);
size_t fused_sync_bytes_for(size_t ntasks);
int debug_giveup_flag();  // gdr2_debug_force_timeout's setting
int debug_unfused_flag();  // gdr2_debug_forward_unfused's setting
cudaError_t launch_recip_eval(const float *x, float *y, long long n, cudaStream_t s);
cudaError_t launch_short_conv(const ConvArgs &a, cudaStream_t s);
cudaError_t launch_gate_activations(const ActArgs &a, cudaStream_t s);
cudaError_t launch_forward_simt(const FwdArgs &a, cudaStream_t s);
cudaError_t launch_forward_tc(const FwdArgs &a, cudaStream_t s);
bool forward_tc_supported(const FwdArgs &a);
size_t forward_tc_workspace_bytes(int B, int T, int H);
size_t forward_tc_varlen_workspace_bytes(int N, int T, int H);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv, bool bf16);
cudaError_t launch_backward(const BwdArgs &a, cudaStream_t s);
size_t backward_noalloc_scratch_needed(int B, int T, int H, int dk, int dv, bool have_saved_states);
cudaError_t launch_backward_noalloc(const BwdArgs &a, cudaStream_t s);
bool backward_tc_supported(const BwdArgs &a);
size_t backward_tc_workspace_bytes(int B, int T, int H);
cudaError_t launch_backward_tc(const BwdArgs &a, cudaStream_t s);

}  // namespace gdr2
