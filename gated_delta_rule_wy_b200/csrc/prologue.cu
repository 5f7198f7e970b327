// prologue.cu -- the Gated DeltaNet-2 block prologue in front of the mixer ("Gated
// DeltaNet-2: Decoupling Erase and Write in Linear Attention", sec. 3, block data-flow
// paragraph): query and key go through a short convolution, SiLU and an L2 norm, the
// value through the convolution and SiLU, and three separate branches give the decay and
// the erase and write gates.
//
// Readings (the note names the steps only): the convolution is causal and depthwise over
// time with the tap layout of a depthwise Conv1d weight [C, 1, W] left-padded by W - 1
// (tap i multiplies the input W - 1 - i tokens back); a state holds the W - 1 inputs
// before a sequence's first token; the L2 norm is x / sqrt(sum_head x^2 + eps);
// log alpha = -softplus(a), b = sigmoid(b'), w = sigmoid(w').
//
// Both kernels are HBM streams (one read and one write per element). The convolution
// stages each 32-token run's rows, and the rows before it that the taps reach (mostly
// L2 hits), in shared memory by bulk asynchronous copies, all in flight at once.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr2_common.cuh"
#include "gdr2_launch.h"
#include "sm100_ptx.cuh"

namespace gdr2 {
namespace {

using namespace sm100;

constexpr int kMaxWidth = 4;    // taps; the window keeps the kMaxWidth - 1 previous rows
constexpr int kRun = 32;        // tokens per warp task
constexpr int kConvWarps = 8;
constexpr uint64_t kConvWaitNs = 2000000000ull;  // bounded wait for a run's rows (2 s)

template <typename TIn> struct Vec;
template <> struct Vec<float> {
    template <int V> __device__ static void load(const float *p, float (&v)[V])
    {
        if constexpr (V == 4) {
            const float4 a = *reinterpret_cast<const float4 *>(p);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        } else {
            const float2 a = *reinterpret_cast<const float2 *>(p);
            v[0] = a.x; v[1] = a.y;
        }
    }
    template <int V> __device__ static void store(float *p, const float (&v)[V])
    {
        if constexpr (V == 4) *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
        else *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    }
};
template <> struct Vec<__nv_bfloat16> {
    template <int V> __device__ static void load(const __nv_bfloat16 *p, float (&v)[V])
    {
        if constexpr (V == 4) {
            const uint2 a = *reinterpret_cast<const uint2 *>(p);
            const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&a.x));
            const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&a.y));
            v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
        } else {
            const uint32_t a = *reinterpret_cast<const uint32_t *>(p);
            const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&a));
            v[0] = f0.x; v[1] = f0.y;
        }
    }
    template <int V> __device__ static void store(__nv_bfloat16 *p, const float (&v)[V])
    {
        const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
        if constexpr (V == 4) {
            const __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
            uint2 a;
            a.x = *reinterpret_cast<const uint32_t *>(&h0);
            a.y = *reinterpret_cast<const uint32_t *>(&h1);
            *reinterpret_cast<uint2 *>(p) = a;
        } else {
            *reinterpret_cast<uint32_t *>(p) = *reinterpret_cast<const uint32_t *>(&h0);
        }
    }
};

struct ConvParams {
    int N, T, H, W;          // sequences (batches when dense), tokens, heads, taps
    int Bm;                  // token streams: N dense, 1 packed
    int runs;                // ceil(T / kRun) warp tasks per (stream, head)
    const int *cu_seqlens;   // packed: sequence s is tokens cu[s] .. cu[s+1] - 1 of the stream
    const void *x;           // [Bm, T, H, D]
    const float *weight;     // [H * D][W]
    const void *state_in;    // [N][W - 1][H][D] or null (zeros)
    void *state_out;         // [N][W - 1][H][D] or null
    void *y;                 // [Bm, T, H, D]
    float eps;
    unsigned *status;        // device status word (a wait given up)
};

// silu(v) = v / (1 + e^-v); below v = -87 the denominator overflows and the quotient is 0
__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.f + __expf(-v)); }

// The sequence that token t of a packed stream belongs to: the s with cu[s] <= t < cu[s+1].
__device__ __forceinline__ int find_sequence(const int *cu, int N, int t)
{
    int lo = 0, hi = N - 1;  // the last s with cu[s] <= t (empty sequences share cu[s] with the next)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu + mid) <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Shared memory of one warp's task: its mbarrier, then the run's rows from kMaxWidth - 1
// tokens before it (kRun + kMaxWidth - 1 rows of D values).
template <typename TIn, int D>
constexpr uint32_t conv_rows_bytes() { return (uint32_t)((kRun + kMaxWidth - 1) * D * sizeof(TIn)); }
template <typename TIn, int D>
constexpr uint32_t conv_smem_bytes() { return kConvWarps * (128 + conv_rows_bytes<TIn, D>()); }

template <typename TIn, int D, bool L2>
__global__ void __launch_bounds__(kConvWarps * 32) short_conv_kernel(ConvParams p)
{
    constexpr int V = D / 32;  // channels per lane
    constexpr uint32_t kRowBytes = D * sizeof(TIn);
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char *wsm = smem_raw + warp * (128 + conv_rows_bytes<TIn, D>());
    uint64_t *bar = reinterpret_cast<uint64_t *>(wsm);
    const TIn *rows = reinterpret_cast<const TIn *>(wsm + 128);  // row r = token t0 - (kMaxWidth - 1) + r

    const long long task = (long long)blockIdx.x * kConvWarps + warp;
    const long long ntasks = (long long)p.Bm * p.H * p.runs;
    if (task >= ntasks) return;
    // heads fastest: the warps of a block read and write neighbouring slices of the same rows
    const int h = (int)(task % p.H);
    const int run = (int)((task / p.H) % p.runs);
    const int bs = (int)(task / ((long long)p.runs * p.H));  // token stream
    const int t0 = run * kRun, t1 = min(p.T, t0 + kRun);
    const int c0 = lane * V;
    const TIn *x = static_cast<const TIn *>(p.x);
    TIn *y = static_cast<TIn *>(p.y);
    const TIn *sin = static_cast<const TIn *>(p.state_in);
    TIn *sout = static_cast<TIn *>(p.state_out);
    const size_t HD = (size_t)p.H * D;
    auto grow = [&](int t) -> size_t { return ((size_t)bs * p.T + t) * HD + (size_t)h * D; };

    // the run's rows (and the halo before it) into shared memory, all copies in flight at
    // once; rows before the stream's start are never read
    const int r_lo = max(0, (kMaxWidth - 1) - t0), r_hi = t1 - t0 + (kMaxWidth - 1);
    if (lane == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar, (uint32_t)(r_hi - r_lo) * kRowBytes);
    }
    __syncwarp();
    for (int r = r_lo + lane; r < r_hi; r += 32)
        bulk_load(wsm + 128 + r * kRowBytes, x + grow(t0 - (kMaxWidth - 1) + r), kRowBytes, bar);

    // taps, right-aligned in kMaxWidth: wt[i] multiplies the input kMaxWidth - 1 - i back
    float wt[kMaxWidth][V];
#pragma unroll
    for (int i = 0; i < kMaxWidth; ++i)
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int j = i - (kMaxWidth - p.W);
            wt[i][v] = j >= 0 ? __ldg(p.weight + ((size_t)h * D + c0 + v) * p.W + j) : 0.f;
        }
    // the sequence of t0, its first token and one past its last
    int s = bs, sbeg = 0, send = p.T;
    if (p.cu_seqlens) {
        s = find_sequence(p.cu_seqlens, p.N, t0);
        sbeg = __ldg(p.cu_seqlens + s);
        send = __ldg(p.cu_seqlens + s + 1);
    }
    if (!mbar_wait_bounded(bar, 0, kConvWaitNs)) {
        if (lane == 0) atomicOr(p.status, kStatusTimeout);
        mbar_wait_bounded(bar, 0, kConvWaitNs);  // let the copies land before the block's memory goes
        return;
    }
    // input tau of this lane's channels: the sequence's own token, its state, or zero
    auto input = [&](int tau, float (&v)[V]) {
        if (tau >= sbeg) {
            Vec<TIn>::template load<V>(rows + (tau - t0 + (kMaxWidth - 1)) * D + c0, v);
        } else {
            const int js = (p.W - 1) - (sbeg - tau);  // state row (oldest first), if it has one
            if (sin && js >= 0)
                Vec<TIn>::template load<V>(sin + (((size_t)s * (p.W - 1) + js) * p.H + h) * D + c0, v);
            else
#pragma unroll
                for (int k = 0; k < V; ++k) v[k] = 0.f;
        }
    };
    // window: win[i] = input t - (kMaxWidth - 1) + i for the next token t, refilled through
    // the general path only where a sequence starts; each token then reads one row
    float win[kMaxWidth - 1][V];
    auto refill = [&](int t) {
#pragma unroll
        for (int i = 0; i < kMaxWidth - 1; ++i) input(t - (kMaxWidth - 1) + i, win[i]);
    };
    refill(t0);
    const TIn *xr = rows + (kMaxWidth - 1) * D + c0;  // token t's row in shared memory
    TIn *yr = y + grow(t0) + c0;                      // token t's output row
#pragma unroll 4
    for (int t = t0; t < t1; ++t, xr += D, yr += HD) {
        if (t >= send) {  // the next non-empty sequence starts here
            while (s + 1 < p.N && __ldg(p.cu_seqlens + s + 1) <= t) ++s;  // stays in [0, N) for any array
            sbeg = __ldg(p.cu_seqlens + s);
            send = __ldg(p.cu_seqlens + s + 1);
            refill(t);
        }
        float xt[V], o[V];
        Vec<TIn>::template load<V>(xr, xt);
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float a = wt[kMaxWidth - 1][v] * xt[v];
#pragma unroll
            for (int i = 0; i < kMaxWidth - 1; ++i) a = fmaf(wt[i][v], win[i][v], a);
            o[v] = silu(a);
        }
        if constexpr (L2) {
            float ss = 0.f;
#pragma unroll
            for (int v = 0; v < V; ++v) ss = fmaf(o[v], o[v], ss);
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            const float inv = rsqrtf(ss + p.eps);
#pragma unroll
            for (int v = 0; v < V; ++v) o[v] *= inv;
        }
        Vec<TIn>::template store<V>(yr, o);
#pragma unroll
        for (int v = 0; v < V; ++v) {
#pragma unroll
            for (int i = 0; i < kMaxWidth - 2; ++i) win[i][v] = win[i + 1][v];
            win[kMaxWidth - 2][v] = xt[v];
        }
        if (sout && t == send - 1) {
            // the sequence's last token: its state is the last W - 1 inputs, oldest first;
            // after the shift win[i] is input t - (kMaxWidth - 2) + i, so state row
            // j = i - (kMaxWidth - W), 0 <= j <= W - 2; every read of the old state above
            // precedes these writes in this lane
#pragma unroll
            for (int i = 0; i < kMaxWidth - 1; ++i) {
                const int j = i - (kMaxWidth - p.W);
                if (j >= 0)
                    Vec<TIn>::template store<V>(sout + (((size_t)s * (p.W - 1) + j) * p.H + h) * D + c0, win[i]);
            }
        }
    }
}

// Packed sequences without tokens keep their state (or get zeros): one block per sequence.
template <typename TIn>
__global__ void empty_state_kernel(ConvParams p, int D)
{
    const int s = blockIdx.x;
    if (__ldg(p.cu_seqlens + s) != __ldg(p.cu_seqlens + s + 1)) return;
    const size_t n = (size_t)(p.W - 1) * p.H * D;
    const TIn *sin = static_cast<const TIn *>(p.state_in);
    TIn *sout = static_cast<TIn *>(p.state_out);
    for (size_t i = threadIdx.x; i < n; i += blockDim.x)
        sout[(size_t)s * n + i] = sin ? sin[(size_t)s * n + i] : TIn(0.f);
}

template <typename TIn, int D>
cudaError_t launch_conv(const ConvParams &p, bool l2, cudaStream_t st)
{
    const long long ntasks = (long long)p.Bm * p.H * p.runs;
    const unsigned blocks = (unsigned)((ntasks + kConvWarps - 1) / kConvWarps);
    if (blocks > 0) {
        auto kern = l2 ? short_conv_kernel<TIn, D, true> : short_conv_kernel<TIn, D, false>;
        constexpr uint32_t smem = conv_smem_bytes<TIn, D>();
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<blocks, kConvWarps * 32, smem, st>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.cu_seqlens && p.state_out && p.W > 1 && p.N > 0) {
        empty_state_kernel<TIn><<<p.N, 256, 0, st>>>(p, D);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

// ---------------------------------------------------------------- activations
// -softplus(a) = -(max(a, 0) + log(1 + e)) with e = exp(-|a|) in (0, 1]: log(1 + e) by its
// Taylor series e - e^2/2 + e^3/3 below e = 1/32 (truncation below e^4/4, 7e-6 of the value),
// else from the logarithm intrinsic (absolute error below 4e-7 on [1, 2], 1.2e-5 of the value)
__device__ __forceinline__ float neg_softplus(float a)
{
    const float e = __expf(-fabsf(a));
    const float l = e < 0.03125f ? e * fmaf(e, fmaf(e, 1.f / 3.f, -0.5f), 1.f) : __logf(1.f + e);
    return -(fmaxf(a, 0.f) + l);
}
// 1 / (1 + e^-a); below a = -87 the denominator overflows and the quotient is 0
__device__ __forceinline__ float sigmoid(float a) { return __fdividef(1.f, 1.f + __expf(-a)); }

template <typename TIn>
__device__ __forceinline__ float ld1(const TIn *p, long long i)
{
    if constexpr (sizeof(TIn) == 2) return __bfloat162float(p[i]);
    else return p[i];
}

// Eight consecutive elements i * 8 .. i * 8 + 7 of a 16-byte aligned array, as fp32.
template <typename TIn>
__device__ __forceinline__ void load8(const TIn *in, long long i, float (&v)[8])
{
    if constexpr (sizeof(TIn) == 2) {
        const uint4 a = *reinterpret_cast<const uint4 *>(in + 8 * i);
        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u[k]));
            v[2 * k] = f.x;
            v[2 * k + 1] = f.y;
        }
    } else {
        const float4 a = *reinterpret_cast<const float4 *>(in + 8 * i);
        const float4 b = *reinterpret_cast<const float4 *>(in + 8 * i + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// kind 0: log_alpha = -softplus(v) to fp32; kinds 1, 2: sigmoid(v) in the input dtype.
template <typename TIn>
__device__ __forceinline__ void act8(float (&v)[8], void *out, long long i, int kind)
{
    if (kind == 0) {
        float *o = static_cast<float *>(out) + 8 * i;
        *reinterpret_cast<float4 *>(o) =
            make_float4(neg_softplus(v[0]), neg_softplus(v[1]), neg_softplus(v[2]), neg_softplus(v[3]));
        *reinterpret_cast<float4 *>(o + 4) =
            make_float4(neg_softplus(v[4]), neg_softplus(v[5]), neg_softplus(v[6]), neg_softplus(v[7]));
        return;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = sigmoid(v[k]);
    TIn *o = static_cast<TIn *>(out) + 8 * i;
    if constexpr (sizeof(TIn) == 2) {
        uint32_t u[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
            u[k] = *reinterpret_cast<const uint32_t *>(&hv);
        }
        *reinterpret_cast<uint4 *>(o) = make_uint4(u[0], u[1], u[2], u[3]);
    } else {
        *reinterpret_cast<float4 *>(o) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4 *>(o + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// One activation over a flat array: 8-element vectors, two per thread per step (both
// loads in flight), then the ragged tail element by element.
template <typename TIn>
__global__ void __launch_bounds__(256) gate_act_kernel(long long n, const TIn *in, void *out, int kind)
{
    const long long nv = n / 8;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long half = (nv + 1) / 2;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < half; i += stride) {
        const long long j = i + half;
        float va[8], vb[8];
        load8(in, i, va);
        if (j < nv) load8(in, j, vb);
        act8<TIn>(va, out, i, kind);
        if (j < nv) act8<TIn>(vb, out, j, kind);
    }
    for (long long i = 8 * nv + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float a = ld1(in, i);
        if (kind == 0) static_cast<float *>(out)[i] = neg_softplus(a);
        else if constexpr (sizeof(TIn) == 2) static_cast<__nv_bfloat16 *>(out)[i] = __float2bfloat16_rn(sigmoid(a));
        else static_cast<float *>(out)[i] = sigmoid(a);
    }
}

template <typename TIn>
cudaError_t launch_act(long long n, const void *in, void *out, int kind, int nsm, cudaStream_t st)
{
    if (n <= 0) return cudaSuccess;
    const long long want = (n / 16 + 255) / 256 + 1;
    const int blocks = (int)(want < 8LL * nsm ? want : 8LL * nsm);
    gate_act_kernel<TIn><<<blocks, 256, 0, st>>>(n, static_cast<const TIn *>(in), out, kind);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_short_conv(const ConvArgs &a, cudaStream_t st)
{
    ConvParams p;
    p.N = a.N;
    p.T = a.T;
    p.H = a.H;
    p.W = a.width;
    p.Bm = a.cu_seqlens ? 1 : a.N;
    p.runs = (a.T + kRun - 1) / kRun;
    p.cu_seqlens = a.cu_seqlens;
    p.x = a.x;
    p.weight = a.weight;
    p.state_in = a.state_in;
    p.state_out = a.state_out;
    p.y = a.y;
    p.eps = a.eps;
    p.status = a.status;
    if (a.bf16)
        return a.d == 128 ? launch_conv<__nv_bfloat16, 128>(p, a.l2norm, st) : launch_conv<__nv_bfloat16, 64>(p, a.l2norm, st);
    return a.d == 128 ? launch_conv<float, 128>(p, a.l2norm, st) : launch_conv<float, 64>(p, a.l2norm, st);
}

cudaError_t launch_gate_activations(const ActArgs &a, cudaStream_t st)
{
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const void *in[3] = {a.a, a.b_pre, a.w_pre};
    void *out[3] = {a.log_alpha, a.b, a.w};
    const long long n[3] = {a.n_alpha, a.n_b, a.n_w};
    for (int k = 0; k < 3; ++k) {
        if (!in[k] || n[k] <= 0) continue;
        const cudaError_t e = a.bf16 ? launch_act<__nv_bfloat16>(n[k], in[k], out[k], k, nsm, st)
                                     : launch_act<float>(n[k], in[k], out[k], k, nsm, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdr2
