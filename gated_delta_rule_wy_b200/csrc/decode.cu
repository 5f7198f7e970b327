// decode.cu -- one recurrent GDR-2 token for N*H resident fp32 states.
//
// Constant-memory decoding (Gated DeltaNet-2 note, sec. 1) with the per-token
// steps of sec. 3. Reading the old state S once gives both column reductions
//   r = S^T (a (.) e)      s = S^T (a (.) q)          (a = alpha, e = b (.) k)
// because S_t^T q = (Diag(a) S)^T q + (z - r)(k . q). One write stores
//   S <- Diag(a) S + k (z - r)^T.
// So the kernel moves exactly 2 * dk * dv * 4 bytes of state per (sequence,
// head), which is the whole cost: the step is HBM-bound (about 2 flops per
// byte).
//
// One CTA per (sequence, head); 256 threads. Each thread keeps its slice of
// S in registers between the read and the write: a lane owns four adjacent
// value columns (one 16-byte vector) and a warp covers whole rows, so every
// load and store is a fully coalesced 512-byte (dv = 128) row segment. State
// traffic bypasses L1 and is marked evict-first (the state is far larger
// than L2 and is touched once per step).

#include "gdr2_common.cuh"
#include "gdr2_launch.h"

namespace gdr2 {
namespace {

constexpr int NT = 256;
constexpr int NW = NT / 32;

// GATED: a scalar gate may be in use (the other instantiation has vector gates only).
template <typename TIn, int DK, int DV, bool GATED>
__global__ void __launch_bounds__(NT) decode_kernel(DecodeArgs a)
{
    constexpr int LPR = DV / 4;        // lanes per state row
    constexpr int RPW = 32 / LPR;      // rows per warp per pass
    constexpr int RSTRIDE = NW * RPW;  // row stride between a thread's rows
    constexpr int NR = DK / RSTRIDE;   // rows per thread
    __shared__ float s_ae[DK], s_aq[DK], s_al[DK], s_k[DK];
    __shared__ float s_z[DV], s_d[DV];
    __shared__ float s_red[2][NW][DV];
    __shared__ float s_kq[NW];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nh = blockIdx.x;
    const int col4 = lane % LPR;
    const int row0 = warp * RPW + lane / LPR;
    float4 *S4 = reinterpret_cast<float4 *>(a.S + (size_t)nh * DK * DV);

    // Issue every state load first: they do not depend on the token.
    float4 st[NR];
#pragma unroll
    for (int m = 0; m < NR; ++m) st[m] = __ldcs(&S4[(size_t)(row0 + m * RSTRIDE) * LPR + col4]);

    const TIn *q = static_cast<const TIn *>(a.q) + (size_t)nh * DK;
    const TIn *k = static_cast<const TIn *>(a.k) + (size_t)nh * DK;
    const bool bsc = GATED && (a.gates & kGateScalarB) != 0, wsc = GATED && (a.gates & kGateScalarW) != 0;
    const TIn *bg = static_cast<const TIn *>(a.b) + (size_t)nh * (bsc ? 1 : DK);
    const float *la = a.log_alpha + (size_t)nh * DK;
    const TIn *v = static_cast<const TIn *>(a.v) + (size_t)nh * DV;
    const TIn *wg = static_cast<const TIn *>(a.w) + (size_t)nh * (wsc ? 1 : DV);

    float kq = 0.f;
    if (tid < DK) {
        const float kv = to_f32(k[tid]), qv = to_f32(q[tid]);
        const float al = expf(clamp_log_alpha(la[tid]));
        s_ae[tid] = al * to_f32(bg[bsc ? 0 : tid]) * kv;
        s_aq[tid] = al * qv;
        s_al[tid] = al;
        s_k[tid] = kv;
        kq = kv * qv;
    }
    if (tid < DV) s_z[tid] = to_f32(wg[wsc ? 0 : tid]) * to_f32(v[tid]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    if (lane == 0) s_kq[warp] = kq;
    __syncthreads();

    // Partial column reductions over this thread's rows.
    float r[4] = {0.f, 0.f, 0.f, 0.f}, sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < NR; ++m) {
        const int c = row0 + m * RSTRIDE;
        const float ae = s_ae[c], aq = s_aq[c];
        r[0] = fmaf(ae, st[m].x, r[0]); sq[0] = fmaf(aq, st[m].x, sq[0]);
        r[1] = fmaf(ae, st[m].y, r[1]); sq[1] = fmaf(aq, st[m].y, sq[1]);
        r[2] = fmaf(ae, st[m].z, r[2]); sq[2] = fmaf(aq, st[m].z, sq[2]);
        r[3] = fmaf(ae, st[m].w, r[3]); sq[3] = fmaf(aq, st[m].w, sq[3]);
    }
    // Lanes of a warp that share a column set sit LPR apart.
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            r[x] += __shfl_xor_sync(0xffffffffu, r[x], off);
            sq[x] += __shfl_xor_sync(0xffffffffu, sq[x], off);
        }
    }
    if (lane < LPR) {
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            s_red[0][warp][4 * col4 + x] = r[x];
            s_red[1][warp][4 * col4 + x] = sq[x];
        }
    }
    __syncthreads();
    if (tid < DV) {
        float rs = 0.f, ss = 0.f, kqs = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            rs += s_red[0][w][tid];
            ss += s_red[1][w][tid];
        }
#pragma unroll
        for (int w = 0; w < NW; ++w) kqs += s_kq[w];
        const float d = s_z[tid] - rs;
        s_d[tid] = d;
        TIn *o = static_cast<TIn *>(a.o) + (size_t)nh * DV;
        o[tid] = from_f32<TIn>(fmaf(d, kqs, ss));
    }
    __syncthreads();
    const float d0 = s_d[4 * col4], d1 = s_d[4 * col4 + 1], d2 = s_d[4 * col4 + 2], d3 = s_d[4 * col4 + 3];
#pragma unroll
    for (int m = 0; m < NR; ++m) {
        const int c = row0 + m * RSTRIDE;
        const float al = s_al[c], kc = s_k[c];
        float4 y;
        y.x = fmaf(al, st[m].x, kc * d0);
        y.y = fmaf(al, st[m].y, kc * d1);
        y.z = fmaf(al, st[m].z, kc * d2);
        y.w = fmaf(al, st[m].w, kc * d3);
        __stcs(&S4[(size_t)c * LPR + col4], y);
    }
}

template <typename TIn>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s)
{
    const int grid = a.N * a.H;
    if (a.gates) {
        if (a.dk == 128 && a.dv == 128) decode_kernel<TIn, 128, 128, true><<<grid, NT, 0, s>>>(a);
        else if (a.dk == 128 && a.dv == 64) decode_kernel<TIn, 128, 64, true><<<grid, NT, 0, s>>>(a);
        else if (a.dk == 64 && a.dv == 128) decode_kernel<TIn, 64, 128, true><<<grid, NT, 0, s>>>(a);
        else decode_kernel<TIn, 64, 64, true><<<grid, NT, 0, s>>>(a);
    } else {
        if (a.dk == 128 && a.dv == 128) decode_kernel<TIn, 128, 128, false><<<grid, NT, 0, s>>>(a);
        else if (a.dk == 128 && a.dv == 64) decode_kernel<TIn, 128, 64, false><<<grid, NT, 0, s>>>(a);
        else if (a.dk == 64 && a.dv == 128) decode_kernel<TIn, 64, 128, false><<<grid, NT, 0, s>>>(a);
        else decode_kernel<TIn, 64, 64, false><<<grid, NT, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s)
{
    if (a.N * a.H == 0) return cudaSuccess;
    return a.bf16 ? launch_t<__nv_bfloat16>(a, s) : launch_t<float>(a, s);
}

}  // namespace gdr2
