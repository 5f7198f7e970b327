// fwd_simt.cu -- chunkwise GDR-2 forward on CUDA cores, fp32 arithmetic.
//
// This is the fp32-input path (parity at 1e-4 needs fp32 products, which a
// bf16 or tf32 tensor-core operand cannot give). It implements the chunkwise
// algorithm of the Gated DeltaNet-2 note, sec. 3 (chunkwise training
// paragraph): within a chunk of C = 64 tokens and with the decay-normalised
// state S_r = Diag(gamma_r) S^_r, the recurrence becomes a pure asymmetric
// delta rule whose products collapse into a triangular solve and matmuls.
//
// Per chunk (local tokens t, i in [0, C), entry state S, G_t = sum_{s<=t} log alpha_s):
//   A_ti = sum_c e_t[c] k_i[c] exp(G_t[c] - G_i[c])      i <  t   (strictly lower)
//   P_ti = sum_c q_t[c] k_i[c] exp(G_t[c] - G_i[c])      i <= t
//   T    = (I + A)^{-1}                                   (UT form)
//   W    = T (E (.) exp G),   U~ = T Z,   U = U~ - W S
//   O    = (Q (.) exp G) S + P U
//   S   <- Diag(exp G_C) S + (K (.) exp(G_C - G))^T U
// Every exponent is a difference G_t - G_i with i <= t (or G_C - G_t), so it
// is <= 0: nothing overflows whatever the decay. The pairwise exponentials
// are computed directly (exactness over speed); the tensor-core kernel for
// bf16 inputs factorises them instead.
//
// One CTA handles one (batch, head) and a tile of DVT value columns; state
// columns evolve independently, so tiles need no communication. Rows of a
// partial last chunk are zero-padded, which makes them inert (zero keys,
// gated keys, queries and values; zero log-decay).

#include "gdr2_common.cuh"
#include "gdr2_launch.h"

namespace gdr2 {
namespace {

constexpr int C = 64;    // chunk length
constexpr int DVT = 32;  // value columns per CTA
constexpr int NT = 256;  // threads per CTA

template <int DK>
struct SimtSmem {
    float S[DK][DVT];      // state tile (persistent across chunks)
    float Q[C][DK + 1];    // q, then q (.) exp G
    float K[C][DK + 1];    // k, then k (.) exp(G_C - G)
    float E[C][DK + 1];    // e = b (.) k, then e (.) exp G
    float G[C][DK + 1];    // cumulative log decay, then W
    float A[C][C + 1];
    float P[C][C + 1];
    float Tm[C][C + 1];    // (I + A)^{-1}
    float Z[C][DVT];       // z = w (.) v, then U
    float gC[DK];          // exp(G_C)
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(NT, 1) fwd_simt_kernel(FwdArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem<DK> &sm = *reinterpret_cast<SimtSmem<DK> *>(smem_raw);
    const int tid = threadIdx.x;
    const int bh = blockIdx.y;
    const int bb = bh / a.H, h = bh % a.H;
    const int T = a.T, H = a.H, dv = a.dv;
    const int j0 = blockIdx.x * DVT;
    const TIn *q = static_cast<const TIn *>(a.q);
    const TIn *k = static_cast<const TIn *>(a.k);
    const TIn *v = static_cast<const TIn *>(a.v);
    const TIn *bg = static_cast<const TIn *>(a.b);
    const TIn *wg = static_cast<const TIn *>(a.w);
    TIn *o = static_cast<TIn *>(a.o);
    const size_t state_off = (size_t)bh * DK * dv;

    for (int idx = tid; idx < DK * DVT; idx += NT) {
        const int c = idx / DVT, j = idx % DVT;
        sm.S[c][j] = a.S0 ? a.S0[state_off + (size_t)c * dv + j0 + j] : 0.f;
    }

    const int NC = (T + C - 1) / C;
    for (int n = 0; n < NC; ++n) {
        const int t0 = n * C;
        const int Cn = min(C, T - t0);
        __syncthreads();  // S tile complete; previous chunk done with every buffer
        if (a.saved_states) {
            float *dst = a.saved_states + ((size_t)bh * NC + n) * DK * dv;
            for (int idx = tid; idx < DK * DVT; idx += NT) {
                const int c = idx / DVT, j = idx % DVT;
                dst[(size_t)c * dv + j0 + j] = sm.S[c][j];
            }
        }
        // ---- gates: e = b (.) k, z = w (.) v; zero-padded tail ----
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int t = idx / DK, c = idx % DK;
            float qv = 0.f, kv = 0.f, bv = 0.f, la = 0.f;
            if (t < Cn) {
                const size_t row = ((size_t)bb * T + t0 + t) * H + h;
                const size_t off = row * DK + c;
                qv = to_f32(q[off]);
                kv = to_f32(k[off]);
                bv = to_f32(bg[(a.gates & kGateScalarB) ? row : off]);
                la = clamp_log_alpha(a.log_alpha[off]);
            }
            sm.Q[t][c] = qv;
            sm.K[t][c] = kv;
            sm.E[t][c] = bv * kv;
            sm.G[t][c] = la;
        }
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int t = idx / DVT, j = idx % DVT;
            float z = 0.f;
            if (t < Cn) {
                const size_t row = ((size_t)bb * T + t0 + t) * H + h;
                const size_t off = row * dv + j0 + j;
                z = to_f32(wg[(a.gates & kGateScalarW) ? row : off]) * to_f32(v[off]);
            }
            sm.Z[t][j] = z;
        }
        __syncthreads();
        // ---- cumulative log decay G (per key channel) ----
        if (tid < DK) {
            float g = 0.f;
            for (int t = 0; t < C; ++t) {
                g += sm.G[t][tid];
                sm.G[t][tid] = g;
            }
            sm.gC[tid] = expf(g);
        }
        __syncthreads();
        // ---- A (strictly lower) and P (lower), exact pairwise decay ----
        {
            const int t = tid >> 2;
            const int i0 = (tid & 3) * 16;
            float accA[16], accP[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) accA[m] = accP[m] = 0.f;
            if (i0 <= t) {
                for (int c = 0; c < DK; ++c) {
                    const float gt = sm.G[t][c], et = sm.E[t][c], qt = sm.Q[t][c];
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const int i = i0 + m;
                        if (i <= t) {
                            const float f = sm.K[i][c] * expf(gt - sm.G[i][c]);
                            accA[m] = fmaf(et, f, accA[m]);
                            accP[m] = fmaf(qt, f, accP[m]);
                        }
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int i = i0 + m;
                sm.A[t][i] = (i < t) ? accA[m] : 0.f;
                sm.P[t][i] = (i <= t) ? accP[m] : 0.f;
            }
        }
        __syncthreads();
        // ---- UT solve: column s of T = (I + A)^{-1} by forward substitution ----
        if (tid < C) {
            const int s = tid;
            float col[C];
#pragma unroll
            for (int t = 0; t < C; ++t) {
                float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
                for (int i = 0; i + 3 < t; i += 4) {
                    acc0 = fmaf(sm.A[t][i], col[i], acc0);
                    acc1 = fmaf(sm.A[t][i + 1], col[i + 1], acc1);
                    acc2 = fmaf(sm.A[t][i + 2], col[i + 2], acc2);
                    acc3 = fmaf(sm.A[t][i + 3], col[i + 3], acc3);
                }
#pragma unroll
                for (int i = (t / 4) * 4; i < t; ++i) acc0 = fmaf(sm.A[t][i], col[i], acc0);
                const float acc = (acc0 + acc1) + (acc2 + acc3);
                col[t] = (t < s) ? 0.f : (t == s ? 1.f : -acc);
            }
#pragma unroll
            for (int t = 0; t < C; ++t) sm.Tm[t][s] = col[t];
        }
        // ---- decay-weighted operands, in place (reads G, not written here) ----
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int t = idx / DK, c = idx % DK;
            const float g = sm.G[t][c];
            const float eg = expf(g);
            sm.Q[t][c] *= eg;
            sm.E[t][c] *= eg;
            sm.K[t][c] *= expf(sm.G[C - 1][c] - g);
        }
        __syncthreads();
        // ---- W = T (E (.) exp G), stored over G ----
        {
            constexpr int RSTEP = NT / DK;
            constexpr int NR = C / RSTEP;
            const int c = tid % DK, r0 = tid / DK;
            float acc[NR];
#pragma unroll
            for (int m = 0; m < NR; ++m) acc[m] = 0.f;
            for (int s = 0; s < C; ++s) {
                const float ev = sm.E[s][c];
#pragma unroll
                for (int m = 0; m < NR; ++m) acc[m] = fmaf(sm.Tm[r0 + m * RSTEP][s], ev, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < NR; ++m) sm.G[r0 + m * RSTEP][c] = acc[m];
        }
        __syncthreads();
        // ---- U = T Z - W S, stored over Z ----
        const int j = tid & 31, r0 = tid >> 5;
        {
            float u[C / 8];
#pragma unroll
            for (int m = 0; m < C / 8; ++m) u[m] = 0.f;
            for (int s = 0; s < C; ++s) {
                const float zv = sm.Z[s][j];
#pragma unroll
                for (int m = 0; m < C / 8; ++m) u[m] = fmaf(sm.Tm[r0 + 8 * m][s], zv, u[m]);
            }
            for (int c = 0; c < DK; ++c) {
                const float sv = sm.S[c][j];
#pragma unroll
                for (int m = 0; m < C / 8; ++m) u[m] = fmaf(-sm.G[r0 + 8 * m][c], sv, u[m]);
            }
            __syncthreads();
#pragma unroll
            for (int m = 0; m < C / 8; ++m) sm.Z[r0 + 8 * m][j] = u[m];
        }
        __syncthreads();
        // ---- O = (Q (.) exp G) S + P U ----
        {
            float acc[C / 8];
#pragma unroll
            for (int m = 0; m < C / 8; ++m) acc[m] = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float sv = sm.S[c][j];
#pragma unroll
                for (int m = 0; m < C / 8; ++m) acc[m] = fmaf(sm.Q[r0 + 8 * m][c], sv, acc[m]);
            }
            for (int i = 0; i < C; ++i) {
                const float uv = sm.Z[i][j];
#pragma unroll
                for (int m = 0; m < C / 8; ++m) acc[m] = fmaf(sm.P[r0 + 8 * m][i], uv, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < C / 8; ++m) {
                const int t = r0 + 8 * m;
                if (t < Cn) o[(((size_t)bb * T + t0 + t) * H + h) * dv + j0 + j] = from_f32<TIn>(acc[m]);
            }
        }
        // ---- S <- Diag(exp G_C) S + (K (.) exp(G_C - G))^T U ----
        {
            constexpr int NR = DK / 8;
            float acc[NR];
#pragma unroll
            for (int m = 0; m < NR; ++m) {
                const int c = r0 + 8 * m;
                acc[m] = sm.gC[c] * sm.S[c][j];
            }
            for (int t = 0; t < C; ++t) {
                const float uv = sm.Z[t][j];
#pragma unroll
                for (int m = 0; m < NR; ++m) acc[m] = fmaf(sm.K[t][r0 + 8 * m], uv, acc[m]);
            }
            __syncthreads();  // every thread is done reading S
#pragma unroll
            for (int m = 0; m < NR; ++m) sm.S[r0 + 8 * m][j] = acc[m];
        }
    }
    __syncthreads();
    if (a.S_T) {
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            a.S_T[state_off + (size_t)c * dv + j0 + j] = sm.S[c][j];
        }
    }
}

template <typename TIn, int DK>
cudaError_t launch_one(const FwdArgs &a, cudaStream_t s)
{
    const size_t smem = sizeof(SimtSmem<DK>);
    cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<TIn, DK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.dv / DVT, a.B * a.H);
    fwd_simt_kernel<TIn, DK><<<grid, NT, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward_simt(const FwdArgs &a, cudaStream_t s)
{
    if (a.B * a.H == 0) return cudaSuccess;
    if (a.bf16) return a.dk == 64 ? launch_one<__nv_bfloat16, 64>(a, s) : launch_one<__nv_bfloat16, 128>(a, s);
    return a.dk == 64 ? launch_one<float, 64>(a, s) : launch_one<float, 128>(a, s);
}

}  // namespace gdr2
