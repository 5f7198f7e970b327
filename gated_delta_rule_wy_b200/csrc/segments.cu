// segments.cu -- the states entering the segments of a sequence split for parallel work.
//
// Across a segment the recurrence of the Gated DeltaNet-2 note (sec. 3, forward-pass
// paragraph: S_t = (I - k_t e_t^T) Diag(alpha_t) S_{t-1} + k_t z_t^T) is affine in the
// entering state: S_out = A_g S_in + B_g, with A_g the product of the segment's
// (I - k e^T) Diag(alpha) factors (the segment's final state from S_in = I with the write
// gate off) and B_g its final state from S_in = 0. The states entering the segments then
// follow from one short scan: S_0 = S0, S_{g+1} = A_g S_g + B_g.
//
// One CTA per (batch, head, 32-column block of the state); the chain over segments is
// sequential, each step a d_k x d_k by d_k x 32 product in fp32 (A_g streamed from global
// memory, the column block kept in shared memory).

#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr2_launch.h"

namespace gdr2 {
namespace {

constexpr int kCols = 32;      // state columns per CTA
constexpr int kThreads = 256;  // 8 warps

template <int DK>
__global__ void __launch_bounds__(kThreads) segment_states_kernel(SegArgs a)
{
    __shared__ float S[DK][kCols + 1];  // the column block of the running state (+1: no bank conflicts)
    const int ncb = a.dv / kCols;
    const int cb = blockIdx.x % ncb;
    const int bh = blockIdx.x / ncb;
    const int b = bh / a.H, h = bh % a.H;
    const int tid = threadIdx.x;
    const int c = tid % kCols;                 // this thread's column
    const int r0 = tid / kCols;                // rows r0, r0 + 8, ...
    constexpr int kRowsPer = DK / (kThreads / kCols);
    const size_t sd = (size_t)DK * a.dv;       // one state
    auto sidx = [&](int g) -> size_t { return ((size_t)b * a.G + g) * a.H + h; };  // [B][G][H] order

    for (int i = 0; i < kRowsPer; ++i) {
        const int r = r0 + i * (kThreads / kCols);
        S[r][c] = a.S0 ? a.S0[((size_t)bh * DK + r) * a.dv + cb * kCols + c] : 0.f;
    }
    __syncthreads();
    for (int g = 0; g < a.G; ++g) {
        // the state entering segment g
        for (int i = 0; i < kRowsPer; ++i) {
            const int r = r0 + i * (kThreads / kCols);
            a.S_starts[sidx(g) * sd + (size_t)r * a.dv + cb * kCols + c] = S[r][c];
        }
        // S <- A_g S + B_g (each thread its rows of column c; all reads of S before the barrier)
        const float *Ag = a.A + sidx(g) * (size_t)DK * DK;
        float acc[kRowsPer];
        for (int i = 0; i < kRowsPer; ++i) {
            const int r = r0 + i * (kThreads / kCols);
            acc[i] = a.Bst[sidx(g) * sd + (size_t)r * a.dv + cb * kCols + c];
        }
        for (int k = 0; k < DK; ++k) {
            const float s = S[k][c];
#pragma unroll
            for (int i = 0; i < kRowsPer; ++i) acc[i] = fmaf(__ldg(Ag + (size_t)(r0 + i * (kThreads / kCols)) * DK + k), s, acc[i]);
        }
        __syncthreads();
        for (int i = 0; i < kRowsPer; ++i) S[r0 + i * (kThreads / kCols)][c] = acc[i];
        __syncthreads();
    }
    if (a.S_T)
        for (int i = 0; i < kRowsPer; ++i) {
            const int r = r0 + i * (kThreads / kCols);
            a.S_T[((size_t)bh * DK + r) * a.dv + cb * kCols + c] = S[r][c];
        }
}

}  // namespace

cudaError_t launch_segment_states(const SegArgs &a, cudaStream_t st)
{
    const unsigned blocks = (unsigned)((size_t)a.B * a.H * (a.dv / kCols));
    if (blocks == 0) return cudaSuccess;
    if (a.dk == 128) segment_states_kernel<128><<<blocks, kThreads, 0, st>>>(a);
    else segment_states_kernel<64><<<blocks, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace gdr2
