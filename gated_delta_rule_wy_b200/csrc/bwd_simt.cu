// bwd_simt.cu -- gate-aware GDR-2 backward on CUDA cores (fp32 arithmetic).
//
// Reverse-mode gradient of the recurrence of the Gated DeltaNet-2 note
// (sec. 3: the backward passes through the asymmetric factor (I - k_t e_t^T);
// the gate gradients follow the gated key e = b (.) k and the gated value
// z = w (.) v). With Sb = Diag(a) S_{t-1}, delta = z - Sb^T e,
// S_t = Sb + k delta^T and o_t = S_t^T q, one reverse token is
//   dS  += q dO^T            dq = S_t dO
//   dk   = dS delta          ddelta = dS^T k
//   dw   = ddelta (.) v      dv = ddelta (.) w
//   de   = -Sb ddelta        db = de (.) k,   dk += de (.) b
//   dSb  = dS - e ddelta^T   dlog_alpha = rowsum(dSb (.) Sb)
//   dS   = Diag(a) dSb
//
// Schedule: the columns of S (and of dS) evolve independently, so one CTA
// owns (batch, head, block of JB = 32 value columns). The states entering each
// chunk of 64 tokens come from the forward (saved_states) or from a forward
// sweep here. For each chunk, last to first, the CTA replays the chunk forward
// from its entry state, keeping every token's state block and delta in the
// workspace, then walks the chunk backwards. Thread (c, half) owns the 16
// columns half*16 .. +15 of row c of the block in registers. Column
// reductions (over key channels) finish inside the CTA (a shuffle
// transpose-reduce in each warp, then shared memory across warps); the
// per-key-channel gradients dq, dk, de = dk's erase part and dlog_alpha are
// partial sums over the block's columns, added into fp32 accumulators with
// atomics; a finishing kernel forms dk = dk' + de (.) b, db = de (.) k and
// converts to the output types.

#include <mutex>

#include "../../include/gdr2.h"
#include "gdr2_common.cuh"
#include "gdr2_launch.h"

namespace gdr2 {
namespace {

constexpr int C = 64;

__host__ __device__ constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int JB = 32;  // value columns per CTA

struct BwdLayout {
    size_t cs_off, ts_off, dl_off, acc_off, total;
};

// cs: chunk-entry states [BH][NC][dk][dv] (only without saved_states);
// ts: per-CTA token states of one chunk [BH * NJ][C + 1][dk][JB];
// dl: per-CTA deltas of one chunk [BH * NJ][C][JB];
// acc: fp32 accumulators dq, dk', de, dlog_alpha, each [B][T][H][dk].
__host__ __device__ inline BwdLayout bwd_layout(int B, int T, int H, int dk, int dv, bool need_cs)
{
    const size_t BH = (size_t)B * H;
    const size_t NC = (size_t)(T + C - 1) / C;
    BwdLayout L;
    size_t off = 0;
    L.cs_off = off;
    if (need_cs) off += align256(BH * NC * dk * dv * sizeof(float));
    L.ts_off = off;
    off += align256(BH * (C + 1) * dk * dv * sizeof(float));
    L.dl_off = off;
    off += align256(BH * C * dv * sizeof(float));
    L.acc_off = off;
    off += align256(4 * (size_t)B * T * H * dk * sizeof(float));
    L.total = off;
    return L;
}

// Sum `vals` over the 16 lanes that share bit 4 of the lane id. On return
// lane L (L = lane & 15) holds, in vals[0 .. N/16), the sums of the N/16
// consecutive entries starting at (N/16) * L.
template <int N>
__device__ __forceinline__ void transpose_reduce16(float (&vals)[N], int lane)
{
#pragma unroll
    for (int o = 8, n = N; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? vals[i] : vals[i + n / 2];
            const float keep = upper ? vals[i + n / 2] : vals[i];
            vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
}

template <int DK>
struct BwdSmem {
    float red[2 * DK / 32][JB];  // per-warp column partials
    float vec[JB];               // reduced column vector (delta or ddelta)
    float z[JB], dO[JB], v[JB], w[JB];
};

template <typename TIn, int DK>
__device__ __forceinline__ void load_row_gates(const BwdArgs &a, size_t ok, int c, float &kc, float &bc,
                                               float &al)
{
    kc = to_f32(static_cast<const TIn *>(a.k)[ok + c]);
    bc = to_f32(static_cast<const TIn *>(a.b)[ok + c]);
    al = expf(clamp_log_alpha(a.log_alpha[ok + c]));
}

// One forward token on this thread's 16 columns of row c (columns j0 + jb ..).
// Leaves delta (the block's JB columns) in sm.vec and writes it to dl when not null.
template <typename TIn, int DK, int DV>
__device__ __forceinline__ void fwd_token(const BwdArgs &a, BwdSmem<DK> &sm, float (&S)[JB / 2], int t, int bb,
                                          int h, int j0, int c, int jb, int lane, int warp, int tid, float *dl)
{
    constexpr int HJ = JB / 2;
    const size_t ok = (((size_t)bb * a.T + t) * a.H + h) * DK;
    const size_t ov = (((size_t)bb * a.T + t) * a.H + h) * DV + j0;
    if (tid < JB)
        sm.z[tid] = to_f32(static_cast<const TIn *>(a.w)[ov + tid]) * to_f32(static_cast<const TIn *>(a.v)[ov + tid]);
    float kc, bc, al;
    load_row_gates<TIn, DK>(a, ok, c, kc, bc, al);
    const float ae = al * bc * kc;
    float part[HJ];
#pragma unroll
    for (int j = 0; j < HJ; ++j) part[j] = ae * S[j];
    transpose_reduce16<HJ>(part, lane);
    sm.red[warp][jb + (lane & 15)] = part[0];
    __syncthreads();
    if (tid < JB) {
        float r = 0.f;
#pragma unroll
        for (int wv = 0; wv < 2 * DK / 32; ++wv) r += sm.red[wv][tid];
        const float d = sm.z[tid] - r;
        sm.vec[tid] = d;
        if (dl) dl[tid] = d;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < HJ; ++j) S[j] = fmaf(al, S[j], kc * sm.vec[jb + j]);
}

template <typename TIn, int DK, int DV>
__global__ void __launch_bounds__(2 * DK, 1) bwd_kernel(BwdArgs a, float *CS, float *TS, float *DL, float *ACC)
{
    constexpr int HJ = JB / 2;
    constexpr int NJ = DV / JB;
    static_assert(HJ == 16, "one transpose-reduce step per column");
    __shared__ BwdSmem<DK> sm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = warp * 16 + (lane & 15);
    const int half = lane >> 4;
    const int jb = half * HJ;            // this thread's first column within the block
    const int bh = blockIdx.x / NJ;
    const int j0 = (blockIdx.x % NJ) * JB;  // the block's first value column
    const int bb = bh / a.H, h = bh % a.H;
    const int T = a.T, H = a.H;
    const int NC = (T + C - 1) / C;
    const size_t SS = (size_t)DK * DV;        // one full state
    const size_t BS = (size_t)DK * JB;        // one state block
    const size_t nacc = (size_t)a.B * T * H * DK;
    float *ts = TS + (size_t)blockIdx.x * (C + 1) * BS;
    float *dl = DL + (size_t)blockIdx.x * C * JB;
    float *acc_dq = ACC, *acc_dk = ACC + nacc, *acc_de = ACC + 2 * nacc, *acc_dla = ACC + 3 * nacc;
    const size_t srow = (size_t)c * DV + j0 + jb;  // this thread's columns in a full state

    float S[HJ];
    // ---- states entering each chunk ----
    const float *chunk_states;
    if (a.saved_states) {
        chunk_states = a.saved_states + (size_t)bh * NC * SS;
    } else {
        float *cs = CS + (size_t)bh * NC * SS;
#pragma unroll
        for (int j = 0; j < HJ; ++j) S[j] = a.S0 ? a.S0[(size_t)bh * SS + srow + j] : 0.f;
        for (int t = 0; t < T; ++t) {
            if (t % C == 0) {
#pragma unroll
                for (int j = 0; j < HJ; ++j) cs[(size_t)(t / C) * SS + srow + j] = S[j];
            }
            fwd_token<TIn, DK, DV>(a, sm, S, t, bb, h, j0, c, jb, lane, warp, tid, nullptr);
        }
        chunk_states = cs;
    }

    float dS[HJ];
#pragma unroll
    for (int j = 0; j < HJ; ++j) dS[j] = a.dS_T ? a.dS_T[(size_t)bh * SS + srow + j] : 0.f;

    for (int n = NC - 1; n >= 0; --n) {
        const int t0 = n * C;
        const int Cn = min(C, T - t0);
        // ---- replay the chunk forward, keeping every state block and delta ----
#pragma unroll
        for (int j = 0; j < HJ; ++j) {
            S[j] = chunk_states[(size_t)n * SS + srow + j];
            ts[(size_t)c * JB + jb + j] = S[j];
        }
        for (int t = 0; t < Cn; ++t) {
            fwd_token<TIn, DK, DV>(a, sm, S, t0 + t, bb, h, j0, c, jb, lane, warp, tid, dl + (size_t)t * JB);
#pragma unroll
            for (int j = 0; j < HJ; ++j) ts[(size_t)(t + 1) * BS + (size_t)c * JB + jb + j] = S[j];
        }
        // Each thread reads back only the rows and deltas it wrote itself.
        __syncthreads();
        // ---- reverse tokens ----
        for (int t = Cn - 1; t >= 0; --t) {
            const int tg = t0 + t;
            const size_t ok = (((size_t)bb * T + tg) * H + h) * DK;
            const size_t ov = (((size_t)bb * T + tg) * H + h) * DV + j0;
            if (tid < JB) {
                sm.dO[tid] = to_f32(static_cast<const TIn *>(a.dO)[ov + tid]);
                sm.v[tid] = to_f32(static_cast<const TIn *>(a.v)[ov + tid]);
                sm.w[tid] = to_f32(static_cast<const TIn *>(a.w)[ov + tid]);
                sm.vec[tid] = dl[(size_t)t * JB + tid];  // delta_t
            }
            const float qc = to_f32(static_cast<const TIn *>(a.q)[ok + c]);
            float kc, bc, al;
            load_row_gates<TIn, DK>(a, ok, c, kc, bc, al);
            const float ec = bc * kc;
            __syncthreads();
            const float *St = ts + (size_t)(t + 1) * BS + (size_t)c * JB + jb;
            const float *Sp = ts + (size_t)t * BS + (size_t)c * JB + jb;
            float dq = 0.f, dk = 0.f;
            float part[HJ];
#pragma unroll
            for (int j = 0; j < HJ; ++j) {
                const float dOj = sm.dO[jb + j];
                dq = fmaf(St[j], dOj, dq);
                dS[j] = fmaf(qc, dOj, dS[j]);
                dk = fmaf(dS[j], sm.vec[jb + j], dk);
                part[j] = dS[j] * kc;
            }
            transpose_reduce16<HJ>(part, lane);
            sm.red[warp][jb + (lane & 15)] = part[0];
            __syncthreads();
            if (tid < JB) {
                float dd = 0.f;
#pragma unroll
                for (int wv = 0; wv < 2 * DK / 32; ++wv) dd += sm.red[wv][tid];
                sm.vec[tid] = dd;  // ddelta_t
                static_cast<TIn *>(a.gw)[ov + tid] = from_f32<TIn>(dd * sm.v[tid]);
                static_cast<TIn *>(a.gv)[ov + tid] = from_f32<TIn>(dd * sm.w[tid]);
            }
            __syncthreads();
            float de = 0.f, dla = 0.f;
#pragma unroll
            for (int j = 0; j < HJ; ++j) {
                const float dd = sm.vec[jb + j];
                const float sb = al * Sp[j];
                de = fmaf(-sb, dd, de);
                const float g = fmaf(-ec, dd, dS[j]);
                dla = fmaf(g, sb, dla);
                dS[j] = al * g;
            }
            dq += __shfl_xor_sync(0xffffffffu, dq, 16);
            dk += __shfl_xor_sync(0xffffffffu, dk, 16);
            de += __shfl_xor_sync(0xffffffffu, de, 16);
            dla += __shfl_xor_sync(0xffffffffu, dla, 16);
            if (half == 0) {
                atomicAdd(acc_dq + ok + c, dq);
                atomicAdd(acc_dk + ok + c, dk);
                atomicAdd(acc_de + ok + c, de);
                atomicAdd(acc_dla + ok + c, dla);
            }
            __syncthreads();
        }
    }
    if (a.gS0) {
#pragma unroll
        for (int j = 0; j < HJ; ++j) a.gS0[(size_t)bh * SS + srow + j] = dS[j];
    }
}

// dq = sum of the blocks' dq; dk = dk' + de (.) b; db = de (.) k; dlog_alpha, all per key channel.
template <typename TIn>
__global__ void bwd_finish_kernel(BwdArgs a, const float *ACC, size_t n)
{
    const float *acc_dq = ACC, *acc_dk = ACC + n, *acc_de = ACC + 2 * n, *acc_dla = ACC + 3 * n;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const float kc = to_f32(static_cast<const TIn *>(a.k)[i]);
        const float bc = to_f32(static_cast<const TIn *>(a.b)[i]);
        const float de = acc_de[i];
        static_cast<TIn *>(a.gq)[i] = from_f32<TIn>(acc_dq[i]);
        static_cast<TIn *>(a.gk)[i] = from_f32<TIn>(fmaf(de, bc, acc_dk[i]));
        static_cast<TIn *>(a.gb)[i] = from_f32<TIn>(de * kc);
        a.glog_alpha[i] = acc_dla[i];
    }
}

template <typename TIn, int DK, int DV>
cudaError_t launch_t(const BwdArgs &a, cudaStream_t s)
{
    const BwdLayout L = bwd_layout(a.B, a.T, a.H, a.dk, a.dv, a.saved_states == nullptr);
    char *ws = static_cast<char *>(a.workspace);
    float *acc = reinterpret_cast<float *>(ws + L.acc_off);
    const size_t n = (size_t)a.B * a.T * a.H * DK;
    cudaError_t e = cudaMemsetAsync(acc, 0, 4 * n * sizeof(float), s);
    if (e != cudaSuccess) return e;
    bwd_kernel<TIn, DK, DV><<<a.B * a.H * (DV / JB), 2 * DK, 0, s>>>(
        a, reinterpret_cast<float *>(ws + L.cs_off), reinterpret_cast<float *>(ws + L.ts_off),
        reinterpret_cast<float *>(ws + L.dl_off), acc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (n == 0) return cudaSuccess;
    const size_t blocks = (n + 255) / 256;
    bwd_finish_kernel<TIn><<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(a, acc, n);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_dt(const BwdArgs &a, cudaStream_t s)
{
    if (a.dk == 128 && a.dv == 128) return launch_t<TIn, 128, 128>(a, s);
    if (a.dk == 128 && a.dv == 64) return launch_t<TIn, 128, 64>(a, s);
    if (a.dk == 64 && a.dv == 128) return launch_t<TIn, 64, 128>(a, s);
    return launch_t<TIn, 64, 64>(a, s);
}

}  // namespace

// The token-level path (any supported dk, dv and dtype).
static cudaError_t launch_backward_simt(const BwdArgs &a, cudaStream_t s)
{
    if (a.B * a.H == 0) return cudaSuccess;
    return a.bf16 ? launch_dt<__nv_bfloat16>(a, s) : launch_dt<float>(a, s);
}

// bf16 at dk = dv = 128 takes the chunkwise tensor-core path (bwd_tc.cu); its workspace is
// the larger, so the size covers either path.
size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv, bool bf16)
{
    const size_t simt = bwd_layout(B, T, H, dk, dv, true).total;
    if (bf16 && dk == 128 && dv == 128 && T > 0) {
        const size_t tcb = backward_tc_workspace_bytes(B, T, H);
        return tcb > simt ? tcb : simt;
    }
    return simt;
}

cudaError_t launch_backward(const BwdArgs &a, cudaStream_t s)
{
    if (a.B * a.H == 0) return cudaSuccess;
    if (backward_tc_supported(a)) return launch_backward_tc(a, s);
    return launch_backward_simt(a, s);
}

}  // namespace gdr2

// ---------------------------------------------------------------------------
// Variant for callers that may not allocate device memory: the workspace is a
// file-scope device array of GDR2_NOALLOC_SCRATCH_BYTES, used by the token-level
// kernels (whose scratch the array is sized for). Host code must not use the
// array's name as a device address (it is a host-side stand-in): the address is
// looked up per device with cudaGetSymbolAddress, with that device current, and
// passed to the kernel. Only a successful lookup is kept; after a failure the
// next call looks again. The kernel writes every scratch word before reading
// it, so stale contents from the previous call do no harm; concurrent calls on
// one device share the array and race.
namespace gdr2 {
namespace {

static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[GDR2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxNoAllocDevices = 64;
void *g_noalloc_ptr[kMaxNoAllocDevices];  // null until a lookup on that device succeeds
std::mutex g_noalloc_mu;

}  // namespace

size_t backward_noalloc_scratch_needed(int B, int T, int H, int dk, int dv, bool have_saved_states)
{
    return bwd_layout(B, T, H, dk, dv, !have_saved_states).total;
}

cudaError_t launch_backward_noalloc(const BwdArgs &a_in, cudaStream_t s)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxNoAllocDevices) return cudaErrorInvalidDevice;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        scratch = g_noalloc_ptr[dev];
        if (!scratch) {
            e = cudaGetSymbolAddress(&scratch, g_bwd_noalloc_scratch);
            if (e != cudaSuccess) return e;
            g_noalloc_ptr[dev] = scratch;
        }
    }
    BwdArgs a = a_in;
    a.workspace = scratch;
    a.workspace_bytes = GDR2_NOALLOC_SCRATCH_BYTES;
    return launch_backward_simt(a, s);
}

}  // namespace gdr2
