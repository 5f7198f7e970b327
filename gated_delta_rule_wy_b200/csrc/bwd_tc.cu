// bwd_tc.cu -- chunkwise gate-aware GDR-2 backward on the sm_100a tensor cores
// (bf16 inputs and gradients, fp32 state and state gradient), dk = dv = 128.
//
// The gate-aware backward of the Gated DeltaNet-2 note (sec. 3: the gradient
// flows back through the asymmetric factor (I - k_t e_t^T), with e = b (.) k
// and z = w (.) v) taken chunk by chunk, in the chunkwise form of the same
// section. The forward's chunk step, regrouped (fwd_tc.cu), is
//   S' = (Diag(gamma) + M) S + K~^T U~,      O = Q' S + P U~,
// and with U = U~ - W S = T (Z - E^ S) its reverse per chunk (entry state S,
// state gradient dS' at the chunk's end, output gradient dO) is
//   dS  = (Diag(gamma) + M)^T dS' + Q'^T dO                 (reverse scan)
//   dU~ = P^T dO + K~ dS'           dz = T^T dU~            dw = dz (.) v, dv = dz (.) w
//   dP  = dO U^T   (lower)          dA = -dz U^T  (strictly lower)
//   dq  = (dO S^T) (.) e^G + [dP K^] (.) e^G              (K^ = K (.) e^-G)
//   de  = -(dz S^T) (.) e^G + [dA K^] (.) e^G
//   dk  = [dA^T E^ + dP^T Q^] (.) e^-G + (U dS'^T) (.) e^{G_C - G} + de (.) b,  db = de (.) k
//   dG  = de (.) e - dk_AP (.) k + dq (.) q;  dlog_alpha[t] = sum_{t' >= t} dG[t']
//         + sum_j dS' (.) S e^{G_C} + sum_{t' < t} dk_t (.) k (.) e^{G_C - G}  (within the chunk).
// The diagonal of dP stays out of the two decay products: it adds dP_tt k_t to dq and
// dP_tt q_t to dk in fp32, and its two contributions to dG cancel exactly.
//
// Launches (one stream):
//   1. the forward's chunk tasks (backward instance): the workspace slots ([Q'; M], K~,
//      U~, P, gamma) plus T and W; and, without saved states, the forward's scans for the
//      chunk-entry states. Where B H leaves 32 SMs to the chunk tasks, both run as one
//      cooperative launch: with saved states steps 1 and 2 (bwd_front_kernel, fwd_tc.cu:
//      the chunk tasks from the last chunk back, then the reverse scans on B H of the CTAs),
//      without them the chunk tasks and the forward's scans (fwd_fused_kernel);
//   2. reverse scan (one CTA per (batch, head), chunks last to first): dS^T in TMEM in
//      fp32; per chunk a bf16 image of dS' for the chunk kernels, then
//      dS^T = dS'^T Diag(gamma) + dS'^T M + dO^T Q' as 12 MMAs;
//   3. value kernel (persistent, every chunk in parallel): U, dU~, dz -> dv, dw; dP, dA;
//      dO S^T, dz S^T and U dS'^T, passed on in bf16 with dP's diagonal and sum_j dS' S;
//   4. key kernel (persistent): the decay-weighted operands of the forward (half-chunk
//      references), the four decay products and the per-channel epilogue -> dq, dk, db,
//      dlog_alpha. A chunk whose decay range trips the forward's 70-neper guard forms the
//      decay products with one exponential per token pair instead.
// Every mbarrier wait is bounded; a CTA that gives up records kStatusTimeout, waits for
// its copies, frees its TMEM and exits.

#include <cuda.h>
#include <cstddef>

#include "gdr2_common.cuh"
#include "gdr2_launch.h"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"
#include "bwd_rscan.cuh"

namespace gdr2 {
namespace {

using namespace sm100;
using namespace tc;

constexpr uint32_t DPA_IMG = 16384;  // [dA_0; dP_0; dA_1; dP_1] rows t (32 each) x 64 i, bf16
constexpr uint32_t X_ARR = 16384;    // one [64 t][128 c] bf16 array of the value kernel's record
constexpr uint32_t XREC_BYTES = 3 * X_ARR + 64 * 4 + 128 * 4;  // 3 arrays, dP_tt [64], sum_j dS' S [128]

__host__ __device__ constexpr size_t al1k(size_t x) { return (x + 1023) & ~size_t(1023); }

// ============================================================ reverse scan
// (definitions and the fused kernel's eight-warp version in bwd_rscan.cuh)
__global__ void __launch_bounds__(RS_NT, 1) bwd_scan_kernel(const __grid_constant__ CUtensorMap tm_do, RsParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    RsMisc &ms = *reinterpret_cast<RsMisc *>(sm + RS_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, colhalf = (warp >> 2) & 1;
    const int bh = blockIdx.x, bb = bh / p.H, h = bh % p.H;
    const int NC = p.NC;
    const size_t base = (size_t)bh * NC;
    const int c0 = colhalf * 64;
    const int j = quarter * 32 + lane;

    if (tid == 0) {
        mbar_init(&ms.bar_full[0], 1);
        mbar_init(&ms.bar_full[1], 1);
        mbar_init(&ms.bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&ms.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tm = ms.tmem_base;
    const uint32_t tm_lane = tm + ((uint32_t)(quarter * 32) << 16);

    unsigned pend = 0;  // thread 0: bit b set while buffer b's loads are issued and not yet waited for
    auto issue = [&](int n, int sl) {
        const size_t task = base + n;
        unsigned char *buf = sm + sl * RS_BUF;
        mbar_arrive_expect_tx(&ms.bar_full[sl], 2 * B1_ROWS * 128 + GAMMA_BYTES + C * DV * 2);
        bulk_load(buf, p.ws + task * SLOT_BYTES + SLOT_B1, 2 * B1_ROWS * 128, &ms.bar_full[sl]);
        pend |= 1u << sl;
        bulk_load(ms.gam[sl], p.ws + (size_t)p.ntasks * SLOT_BYTES + task * GAMMA_BYTES, GAMMA_BYTES,
                  &ms.bar_full[sl]);
        tma_load_4d(buf + RS_DO, &tm_do, &ms.bar_full[sl], 0, h, n * C, bb);
        tma_load_4d(buf + RS_DO + 8192, &tm_do, &ms.bar_full[sl], 64, h, n * C, bb);
    };
    if (tid == 0) {
        if (NC > 0) issue(NC - 1, 0);
        if (NC > 1) issue(NC - 2, 1);
    }
    // dS_T^T into region 1, the region "before" iteration 0
    if (warp < 8) {
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = p.dS_T ? p.dS_T[((size_t)bh * DK + c0 + q2 * 32 + i) * DV + j] : 0.f;
            tmem_st32(tm_lane + 128 + c0 + q2 * 32, v);
        }
    }
    tc_fence_before_sync();
    __syncthreads();

    unsigned phf = 0;  // bit b: the parity of buffer b's next load phase
    uint32_t ph_mma = 0;
    bool timed_out = false;
    if (NC > 0) {
        const bool ok = mbar_wait_bounded(&ms.bar_full[0], 0, kWaitLimitNs);
        if (ok) phf ^= 1u, pend &= ~1u;
        if (__syncthreads_or(!ok)) timed_out = true;
    }
    for (int k = 0; k < NC && !timed_out; ++k) {
        const int n = NC - 1 - k, sl = k & 1;
        const uint32_t rg = 128u * sl, rgp = 128u * (sl ^ 1);
        unsigned char *ds_img = sm + RS_DS + sl * DS_IMG;
        tc_fence_after_sync();
        // ---- dS'^T (previous region) -> bf16 operand in TMEM and the chunk's dS' image;
        //      gamma-scaled dS'^T -> this region ----
        if (warp < 8) {
            float s0[32], s1[32];
            tmem_ld32x2(tm_lane + rgp + c0, tm_lane + rgp + c0 + 32, s0, s1);
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __nv_bfloat162 h0 = __floats2bfloat162_rn(s0[2 * i], s0[2 * i + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(s1[2 * i], s1[2 * i + 1]);
                pk[i] = *reinterpret_cast<uint32_t *>(&h0);
                pk[16 + i] = *reinterpret_cast<uint32_t *>(&h1);
            }
            tmem_st32u_nw(tm_lane + RS_SA + (uint32_t)(c0 >> 1), pk);
#pragma unroll
            for (int k8 = 0; k8 < 8; ++k8)
                *reinterpret_cast<uint4 *>(ds_img + sw_chunk(j, colhalf * 8 + k8, 128)) =
                    make_uint4(pk[4 * k8], pk[4 * k8 + 1], pk[4 * k8 + 2], pk[4 * k8 + 3]);
            const float4 *g4 = reinterpret_cast<const float4 *>(&ms.gam[sl][c0]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 ga = g4[i], gb = g4[8 + i];
                s0[4 * i] *= ga.x; s0[4 * i + 1] *= ga.y; s0[4 * i + 2] *= ga.z; s0[4 * i + 3] *= ga.w;
                s1[4 * i] *= gb.x; s1[4 * i + 1] *= gb.y; s1[4 * i + 2] *= gb.z; s1[4 * i + 3] *= gb.w;
            }
            tmem_st32_nw(tm_lane + rg + c0, s0);
            tmem_st32_nw(tm_lane + rg + c0 + 32, s1);
            tmem_wait_st();
            fence_proxy_async_smem();  // the dS' image -> the bulk store below
        }
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        // ---- dS^T += dS'^T M (A from TMEM) ;  dS^T += dO^T Q' ----
        if (warp == 8 && lane == 0) {
            const uint32_t buf = sbase + sl * RS_BUF;
            const uint32_t idM = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t bm = sdesc_sw128(buf + 64 * 128 + ks * 2048, B1_ROWS * 128, 1024);
                mma_bf16_ts(tm + rg, tm + RS_SA + ks * 8, bm, idM, 1);
            }
            const uint32_t idQ = idesc_bf16(128, 128, true, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc_sw128(buf + RS_DO + ks * 2048, 8192, 1024);
                const uint64_t bq = sdesc_sw128(buf + ks * 2048, B1_ROWS * 128, 1024);
                mma_bf16(tm + rg, ad, bq, idQ, 1);
            }
            mma_commit(&ms.bar_mma);
        }
        if (tid == 0) {
            bulk_store(p.dsc + (base + n) * DS_IMG, ds_img, DS_IMG);
            bulk_commit_group();
            bulk_wait_group_read1();  // the other image (iteration k - 1) is free for iteration k + 1
        }
        {
            bool ok = true;
            if (k + 1 < NC) {
                const unsigned nb = (unsigned)(sl ^ 1);
                ok = mbar_wait_bounded(&ms.bar_full[nb], (phf >> nb) & 1u, kWaitLimitNs);
                if (ok) phf ^= 1u << nb, pend &= ~(1u << nb);
            }
            ok = mbar_wait_bounded(&ms.bar_mma, ph_mma, kWaitLimitNs) && ok;
            ph_mma ^= 1u;
            tc_fence_before_sync();
            if (__syncthreads_or(!ok)) { timed_out = true; break; }
        }
        if (tid == 0 && k + 2 < NC) issue(n - 2, sl);  // this buffer's MMAs are done
    }
    tc_fence_after_sync();
    if (!timed_out && p.gS0 && warp < 8) {
        const uint32_t rl = NC > 0 ? 128u * ((NC - 1) & 1) : 128u;
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            float v[32];
            tmem_ld32(tm_lane + rl + c0 + q2 * 32, v);
            float *dst = p.gS0 + ((size_t)bh * DK + c0 + q2 * 32) * DV + j;
#pragma unroll
            for (int i = 0; i < 32; ++i) dst[(size_t)i * DV] = v[i];
        }
    }
    if (tid == 0) bulk_wait_group0();
    if (timed_out && tid == 0) {
        // loads still in flight (issued, never waited for) land before shared memory goes
        for (int b2 = 0; b2 < 2; ++b2)
            if (pend & (1u << b2)) mbar_wait_bounded(&ms.bar_full[b2], (phf >> b2) & 1u, kWaitLimitNs);
        atomicOr(p.status, kStatusTimeout);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ============================================================ value kernel
// shared memory (1024-aligned offsets); images are bf16, 128-byte swizzled
constexpr uint32_t VA_DO = 0;        // dO      [t 64][j: 2 blocks]  (TMA)
constexpr uint32_t VA_S0 = 16384;    // S^T     [j 128][c: 2 blocks] (from the fp32 saved state)
constexpr uint32_t VA_DS = 49152;    // dS'^T   [j 128][c: 2 blocks] (reverse scan)
constexpr uint32_t VA_T = 81920;     // T       [t 64][s]
constexpr uint32_t VA_P = 90112;     // P       [t 64][i]
constexpr uint32_t VA_W = 98304;     // W       [c 128][t]          then dU~^T [j 128][i]
constexpr uint32_t VA_UT = 114688;   // U~^T    [j 128][t]          then dz^T  [j 128][t]
constexpr uint32_t VA_KT = 131072;   // K~      [i 64][c: 2 blocks] then [dA_0; dP_0; dA_1; dP_1]
constexpr uint32_t VA_U = 147456;    // U^T     [j 128][i]
constexpr uint32_t VA_X = 163840;    // record staging: 3 x [64 t][128 c] bf16, plain rows
constexpr uint32_t VA_MISC = VA_X + 3 * X_ARR;
constexpr uint32_t VA_DU = VA_W, VA_DZ = VA_UT, VA_DPA = VA_KT;
constexpr uint32_t VA_GV = VA_DU;  // dv tile [64 t][128 j] bf16, once dU~^T's product is done
constexpr uint32_t VA_GW = VA_T;   // dw tile over T and P (16 KB), once their products are done
static_assert(VA_P == VA_T + 8192, "T and P are one 16 KB region");
constexpr uint32_t VA_TX = 16384 + 32768 + 8192 + 8192 + 16384 + 16384 + 16384;

struct VaMisc {
    uint64_t bar_ld, bar_a, bar_b, bar_c, bar_d;
    uint32_t tmem_base;
    int pad;
    float red[8][64];             // per-warp partial sums of dS' (.) S over 32 value channels
    alignas(16) float dpd[64];    // dP_tt (record tail, with rowsum)
    float rowsum[DK];             // sum_j dS'[c][j] S[c][j]
};
constexpr uint32_t VA_SMEM = VA_MISC + sizeof(VaMisc) + 1024;
static_assert(offsetof(VaMisc, dpd) % 16 == 0 && offsetof(VaMisc, rowsum) == offsetof(VaMisc, dpd) + 256,
              "dP_tt and the row sums are one bulk-copy source");

// TMEM columns of the value kernel
constexpr uint32_t VT_U = 0, VT_DU = 64, VT_DZ = 128, VT_DP = 192, VT_DA = 256, VT_XQ = 320, VT_XE = 384,
                   VT_XK = 448;

struct VaParams {
    int B, T, H, NC, ntasks;
    const unsigned char *ws;    // slots
    const unsigned char *ext;   // T and W per task
    const unsigned char *dsc;   // dS'^T images per task
    const float *states;        // chunk-entry states [B][H][NC][DK][DV] fp32
    const __nv_bfloat16 *v, *w;
    __nv_bfloat16 *gv, *gw;
    unsigned char *dpa;         // [ntasks][DPA_IMG]
    unsigned char *xrec;        // [ntasks][XREC_BYTES]
    unsigned *status;
    int wsc;                    // w (and dw) one value per token-head: [B][T][H]
};

__global__ void __launch_bounds__(256, 1) bwd_value_kernel(const __grid_constant__ CUtensorMap tm_do,
                                                          const __grid_constant__ CUtensorMap tm_gv,
                                                          const __grid_constant__ CUtensorMap tm_gw, VaParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    VaMisc &ms = *reinterpret_cast<VaMisc *>(sm + VA_MISC);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, colhalf = warp >> 2;
    const int row = quarter * 32 + lane;  // this thread's TMEM lane (j or c)

    if (tid == 0) {
        mbar_init(&ms.bar_ld, 1);
        mbar_init(&ms.bar_a, 1);
        mbar_init(&ms.bar_b, 1);
        mbar_init(&ms.bar_c, 1);
        mbar_init(&ms.bar_d, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&ms.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tm = ms.tmem_base;
    const uint32_t tm_lane = tm + ((uint32_t)(quarter * 32) << 16);

    // A task's copies, in three groups: dO, dS'^T and U~^T land where no store reads; T, P and
    // W where the dv and dw tiles were staged; K~ where the dA/dP image was (thread 0 waits
    // for those stores to have read their source before the later groups).
    auto issue_loads = [&](int task, bool first) {
        const int bhh = task / p.NC, n = task % p.NC;
        const int bb = bhh / p.H, hh = bhh % p.H;
        const unsigned char *slot = p.ws + (size_t)task * SLOT_BYTES;
        const unsigned char *ext = p.ext + (size_t)task * EXT_BYTES;
        mbar_arrive_expect_tx(&ms.bar_ld, VA_TX);
        tma_load_4d(sm + VA_DO, &tm_do, &ms.bar_ld, 0, hh, n * C, bb);
        tma_load_4d(sm + VA_DO + 8192, &tm_do, &ms.bar_ld, 64, hh, n * C, bb);
        bulk_load(sm + VA_DS, p.dsc + (size_t)task * DS_IMG, DS_IMG, &ms.bar_ld);
        bulk_load(sm + VA_UT, slot + SLOT_U, 16384, &ms.bar_ld);
        if (!first) bulk_wait_group_read1();  // the dv and dw tiles have left W, T and P
        bulk_load(sm + VA_T, ext + EXT_T, 8192, &ms.bar_ld);
        bulk_load(sm + VA_P, slot + SLOT_P, 8192, &ms.bar_ld);
        bulk_load(sm + VA_W, ext + EXT_W, 16384, &ms.bar_ld);
        if (!first) bulk_wait_group_read0();  // the dA/dP image has left K~
        bulk_load(sm + VA_KT, slot + SLOT_KT, 16384, &ms.bar_ld);
    };
    const int ntasks = p.ntasks;
    if (tid == 0 && (int)blockIdx.x < ntasks) issue_loads(blockIdx.x, true);

    uint32_t ph_ld = 0, ph_a = 0, ph_b = 0, ph_c = 0, ph_d = 0;
    bool timed_out = false, loads_pending = (int)blockIdx.x < ntasks;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) -> bool {
        const bool ok = mbar_wait_bounded(bar, ph, kWaitLimitNs);
        ph ^= 1u;
        return __syncthreads_or(!ok) == 0;
    };
    auto mma_sync_point = [&]() {
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    };

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int bhh = task / p.NC, n = task % p.NC;
        const int bb = bhh / p.H, hh = bhh % p.H;
        const int t0 = n * C, Cn = min(C, p.T - t0);
        // the chunk-entry state, S[c][j] for this thread's value channel j and 64 key channels
        const int sj = tid & 127, sch = tid >> 7;
        float sv[64];
        {
            const float *S = p.states + (size_t)task * DK * DV + (size_t)(64 * sch) * DV + sj;
#pragma unroll
            for (int i = 0; i < 64; ++i) sv[i] = S[(size_t)i * DV];
        }
        {
            const bool ok = mbar_wait_bounded(&ms.bar_ld, ph_ld, kWaitLimitNs);
            if (__syncthreads_or(!ok)) { timed_out = true; break; }
            ph_ld ^= 1u;
        }
        loads_pending = false;
        // ---- S^T image and sum_j dS'[c][j] S[c][j] ----
        {
            float part[64];
#pragma unroll
            for (int k8 = 0; k8 < 8; ++k8) {
                float d8[8], f8[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + VA_DS + sw_chunk(sj, sch * 8 + k8, 128)), d8);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    f8[x] = sv[8 * k8 + x];
                    part[8 * k8 + x] = f8[x] * d8[x];
                }
                *reinterpret_cast<uint4 *>(sm + VA_S0 + sw_chunk(sj, sch * 8 + k8, 128)) = pack8(f8);
            }
            transpose_reduce32<64>(part, lane);  // lane L: key channels 64 sch + 2L, +1 over this warp's 32 j
            ms.red[warp][2 * lane] = part[0];
            ms.red[warp][2 * lane + 1] = part[1];
        }
        mma_sync_point();
        if (tid < DK) {
            const int g = tid >> 6, c = tid & 63;
            ms.rowsum[tid] = ms.red[4 * g][c] + ms.red[4 * g + 1][c] + ms.red[4 * g + 2][c] + ms.red[4 * g + 3][c];
        }
        // ---- U^T' = S^T W^T ;  dU~^T = dO^T P + dS'^T K~^T ;  X_q = S dO^T ----
        if (tid == 0) {
            const uint32_t id1 = idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sb + VA_S0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(sb + VA_W + ks * 2048, 8192, 1024);
                mma_bf16(tm + VT_U, a, b, id1, ks > 0);
            }
            mma_commit(&ms.bar_a);
            const uint32_t id2a = idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t a = sdesc_sw128(sb + VA_DO + ks * 2048, 8192, 1024);
                const uint64_t b = sdesc_sw128(sb + VA_P + ks * 2048, 8192, 1024);
                mma_bf16(tm + VT_DU, a, b, id2a, ks > 0);
            }
            const uint32_t id2b = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sb + VA_DS + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(sb + VA_KT + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                mma_bf16(tm + VT_DU, a, b, id2b, 1);
            }
            mma_commit(&ms.bar_b);
            const uint32_t idq = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sb + VA_S0 + ks * 2048, 16384, 1024);
                const uint64_t b = sdesc_sw128(sb + VA_DO + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                mma_bf16(tm + VT_XQ, a, b, idq, ks > 0);
            }
        }
        // ---- U^T = U~^T - U^T' -> bf16 image ----
        if (!wait_bar(&ms.bar_a, ph_a)) { timed_out = true; break; }
        tc_fence_after_sync();
        {
            float du[32];
            tmem_ld32(tm_lane + VT_U + 32 * colhalf, du);
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                const uint32_t off = sw_chunk(row, colhalf * 4 + k8, 128);
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + VA_UT + off), f);
#pragma unroll
                for (int x = 0; x < 8; ++x) f[x] -= du[8 * k8 + x];
                *reinterpret_cast<uint4 *>(sm + VA_U + off) = pack8(f);
            }
        }
        mma_sync_point();
        // ---- dP = dO U^T (M = 64) ;  X_k = dS' U^T ----
        if (tid == 0) {
            const uint32_t idp = idesc_bf16(64, 64, false, true);
            const uint32_t idk = idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t bu = sdesc_sw128(sb + VA_U + ks * 2048, 8192, 1024);
                const uint64_t ad = sdesc_sw128(sb + VA_DO + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                mma_bf16(tm + VT_DP, ad, bu, idp, ks > 0);
                const uint64_t as = sdesc_sw128(sb + VA_DS + ks * 2048, 16384, 1024);
                mma_bf16(tm + VT_XK, as, bu, idk, ks > 0);
            }
        }
        // ---- dU~^T -> bf16 image (over W: its product is done) ----
        if (!wait_bar(&ms.bar_b, ph_b)) { timed_out = true; break; }
        tc_fence_after_sync();
        {
            float d[32];
            tmem_ld32(tm_lane + VT_DU + 32 * colhalf, d);
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                float f[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) f[x] = d[8 * k8 + x];
                *reinterpret_cast<uint4 *>(sm + VA_DU + sw_chunk(row, colhalf * 4 + k8, 128)) = pack8(f);
            }
        }
        mma_sync_point();
        // ---- dz^T = dU~^T T ----
        if (tid == 0) {
            const uint32_t id3 = idesc_bf16(128, 64, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t a = sdesc_sw128(sb + VA_DU + ks * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(sb + VA_T + ks * 2048, 8192, 1024);
                mma_bf16(tm + VT_DZ, a, b, id3, ks > 0);
            }
            mma_commit(&ms.bar_c);
        }
        // v and w of this thread's value channel while the product runs
        __nv_bfloat16 vv[32], wv[32];
#pragma unroll
        for (int s = 0; s < 32; ++s) {
            const int t = 32 * colhalf + s;
            const size_t th = ((size_t)bb * p.T + t0 + t) * p.H + hh;
            vv[s] = t < Cn ? p.v[th * DV + row] : __float2bfloat16_rn(0.f);
            wv[s] = t < Cn ? p.w[p.wsc ? th : th * DV + row] : __float2bfloat16_rn(0.f);
        }
        if (!wait_bar(&ms.bar_c, ph_c)) { timed_out = true; break; }
        tc_fence_after_sync();
        {
            // dv = dz (.) w and dw = dz (.) v as [t][j] tiles over dU~^T and T, P (their products
            // are done), stored by TMA below (rows past T clipped)
            float dz[32];
            tmem_ld32(tm_lane + VT_DZ + 32 * colhalf, dz);
            __nv_bfloat16 *tv = reinterpret_cast<__nv_bfloat16 *>(sm + VA_GV);
            __nv_bfloat16 *tw = reinterpret_cast<__nv_bfloat16 *>(sm + VA_GW);
#pragma unroll
            for (int s = 0; s < 32; ++s) {
                const int t = 32 * colhalf + s;
                tv[t * DV + row] = __float2bfloat16_rn(dz[s] * __bfloat162float(wv[s]));
                if (!p.wsc) tw[t * DV + row] = __float2bfloat16_rn(dz[s] * __bfloat162float(vv[s]));
            }
            if (p.wsc) {
                // a scalar write gate: dw_t = sum_j dz[t][j] v[t][j], this warp's 32 channels first
                // (lane L ends with token 32 colhalf + L), then the four warp quarters below
                float dw[32];
#pragma unroll
                for (int s = 0; s < 32; ++s) dw[s] = dz[s] * __bfloat162float(vv[s]);
                transpose_reduce32<32>(dw, lane);
                ms.red[warp][lane] = dw[0];
            }
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                float f[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) f[x] = dz[8 * k8 + x];
                *reinterpret_cast<uint4 *>(sm + VA_DZ + sw_chunk(row, colhalf * 4 + k8, 128)) = pack8(f);
            }
        }
        mma_sync_point();
        if (tid == 0) {
            tma_store_4d(&tm_gv, sm + VA_GV, 0, hh, t0, bb);
            if (!p.wsc) tma_store_4d(&tm_gw, sm + VA_GW, 0, hh, t0, bb);
            bulk_commit_group();
        }
        if (p.wsc && tid < C && tid < Cn) {
            const int g = tid >> 5, l = tid & 31;
            const float dw = ms.red[4 * g][l] + ms.red[4 * g + 1][l] + ms.red[4 * g + 2][l] + ms.red[4 * g + 3][l];
            p.gw[((size_t)bb * p.T + t0 + tid) * p.H + hh] = __float2bfloat16_rn(dw);
        }
        // ---- dA' = dz U^T (M = 64) ;  X_e = S dz^T ----
        if (tid == 0) {
            const uint32_t ida = idesc_bf16(64, 64, true, true);
            const uint32_t ide = idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t bz = sdesc_sw128(sb + VA_DZ + ks * 2048, 8192, 1024);
                const uint64_t bu = sdesc_sw128(sb + VA_U + ks * 2048, 8192, 1024);
                mma_bf16(tm + VT_DA, bz, bu, ida, ks > 0);
                const uint64_t as = sdesc_sw128(sb + VA_S0 + ks * 2048, 16384, 1024);
                mma_bf16(tm + VT_XE, as, bz, ide, ks > 0);
            }
            mma_commit(&ms.bar_d);
        }
        if (!wait_bar(&ms.bar_d, ph_d)) { timed_out = true; break; }
        tc_fence_after_sync();
        // ---- [dA_0; dP_0; dA_1; dP_1] image (over K~) and dP_tt: rows t of the M = 64
        //      accumulators sit in lanes t % 16 of warp quarter t / 16 ----
        {
            float dp[32], da[32];
            tmem_ld32x2(tm_lane + VT_DP + 32 * colhalf, tm_lane + VT_DA + 32 * colhalf, dp, da);
            if (lane < 16) {
                const int t = quarter * 16 + lane, i0 = 32 * colhalf;
                const int rowA = 64 * (t >> 5) + (t & 31), rowP = rowA + 32;
#pragma unroll
                for (int k8 = 0; k8 < 4; ++k8) {
                    float fp[8], fa[8];
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const bool low = i0 + 8 * k8 + x < t;
                        fp[x] = low ? dp[8 * k8 + x] : 0.f;
                        fa[x] = low ? -da[8 * k8 + x] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(sm + VA_DPA + sw_chunk(rowP, colhalf * 4 + k8, 128)) = pack8(fp);
                    *reinterpret_cast<uint4 *>(sm + VA_DPA + sw_chunk(rowA, colhalf * 4 + k8, 128)) = pack8(fa);
                }
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    if (i0 + x == t) ms.dpd[t] = dp[x];
            }
        }
        // ---- record: X_q = S dO^T, X_e = S dz^T, X_k = dS' U^T as [t][c] bf16 ----
        {
            __nv_bfloat16 *X = reinterpret_cast<__nv_bfloat16 *>(sm + VA_X);
            float x0[32], x1[32];
            tmem_ld32x2(tm_lane + VT_XQ + 32 * colhalf, tm_lane + VT_XE + 32 * colhalf, x0, x1);
#pragma unroll
            for (int s = 0; s < 32; ++s) {
                const int t = 32 * colhalf + s;
                X[t * DK + row] = __float2bfloat16_rn(x0[s]);
                X[(64 + t) * DK + row] = __float2bfloat16_rn(x1[s]);
            }
            tmem_ld32(tm_lane + VT_XK + 32 * colhalf, x0);
#pragma unroll
            for (int s = 0; s < 32; ++s) X[(128 + 32 * colhalf + s) * DK + row] = __float2bfloat16_rn(x0[s]);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            bulk_store(p.dpa + (size_t)task * DPA_IMG, sm + VA_DPA, DPA_IMG);
            bulk_store(p.xrec + (size_t)task * XREC_BYTES, sm + VA_X, 3 * X_ARR);
            bulk_store(p.xrec + (size_t)task * XREC_BYTES + 3 * X_ARR, ms.dpd, 64 * 4 + 128 * 4);
            bulk_commit_group();
            if (task + (int)gridDim.x < ntasks) {
                issue_loads(task + gridDim.x, false);
                loads_pending = true;
            }
        }
    }
    if (tid == 0) {
        bulk_wait_group0();
        if (timed_out) {
            if (loads_pending) mbar_wait_bounded(&ms.bar_ld, ph_ld, kWaitLimitNs);
            atomicOr(p.status, kStatusTimeout);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ============================================================ key kernel
constexpr uint32_t KB_Q = 0;          // q        [64 t][128 c] bf16 (TMA, plain rows)
constexpr uint32_t KB_K = 16384;      // k
constexpr uint32_t KB_B = 32768;      // b
constexpr uint32_t KB_LA = 49152;     // log_alpha [64][128] fp32; then G; then dlog_alpha
constexpr uint32_t KB_STACK = 81920;  // [L^e_0; L^q_0; L^e_1; L^q_1] 128 x 128; then dq, dk (plain rows)
constexpr uint32_t KB_R = 114688;     // [R_0; R_1] 96 x 128; then db (plain rows)
constexpr uint32_t KB_DPA = 139264;   // [dA_0; dP_0; dA_1; dP_1]
constexpr uint32_t KB_X = 155648;     // the value kernel's record
constexpr uint32_t KB_SCAN = KB_X + al1k(XREC_BYTES);  // prefix-scan scratch [16][128] fp32
constexpr uint32_t KB_MISC = KB_SCAN + 8192;
constexpr uint32_t KB_TX = 3 * 16384 + 32768 + DPA_IMG;  // q, k, b, log_alpha and the dA/dP image
constexpr int R_ROWS = 96;

struct KbMisc {
    uint64_t bar_ld, bar_mma, bar_x;  // bar_x: the value kernel's record
    uint32_t tmem_base;
    int pad;
    alignas(16) float g0[DK];       // G at tokens 15 and 47 (half-chunk references; float4 reads)
    alignas(16) float g1[DK];
    float gC[DK];                   // G at the chunk's end
    float hsum[2][DK];              // sum of dG over each half-chunk
    float kts[2][DK];               // sum of dk_t (.) k over each half-chunk
    float red[4][C];                // a scalar erase gate: per-warp-quarter sums of de (.) k per token
};
constexpr uint32_t KB_SMEM = KB_MISC + sizeof(KbMisc) + 1024;
static_assert(offsetof(KbMisc, g0) % 16 == 0 && offsetof(KbMisc, g1) % 16 == 0, "float4 reads of the references");
static_assert(KB_MISC % 16 == 0 && KB_SCAN % 16 == 0 && KB_X % 16 == 0, "16-byte aligned regions");
static_assert(KB_STACK + 2 * 16384 <= KB_R && KB_R + 16384 <= KB_DPA, "output staging fits STACK and R");

// TMEM columns of the key kernel: D_0, D_1 ([c][dA_I rows | dP_I rows]), E_0, E_1 ([c][i])
constexpr uint32_t KT_D0 = 0, KT_D1 = 64, KT_E0 = 128, KT_E1 = 192;

struct KbParams {
    int B, T, H, NC, ntasks;
    const unsigned char *dpa;
    const unsigned char *xrec;
    unsigned *status;
    const __nv_bfloat16 *bsc;  // b one value per token-head [B][T][H] (its tile map unused), or null
    __nv_bfloat16 *gbsc;       // db for such a b, [B][T][H]
};

// element (row, col) of a 128-row, 64-column bf16 image
__device__ __forceinline__ float img64(const unsigned char *img, int r, int c)
{
    return __bfloat162float(
        *reinterpret_cast<const __nv_bfloat16 *>(img + r * 128 + (((c >> 3) ^ (r & 7)) << 4) + (c & 7) * 2));
}

__global__ void __launch_bounds__(256, 1)
bwd_key_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_la,
               const __grid_constant__ CUtensorMap tm_gq, const __grid_constant__ CUtensorMap tm_gk,
               const __grid_constant__ CUtensorMap tm_gb, const __grid_constant__ CUtensorMap tm_gla, KbParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    KbMisc &ms = *reinterpret_cast<KbMisc *>(sm + KB_MISC);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, hf = warp >> 2;

    if (tid == 0) {
        mbar_init(&ms.bar_ld, 1);
        mbar_init(&ms.bar_mma, 1);
        mbar_init(&ms.bar_x, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&ms.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tm = ms.tmem_base;
    const uint32_t tm_lane = tm + ((uint32_t)(quarter * 32) << 16);

    const bool bsc = p.bsc != nullptr;
    auto issue_loads = [&](int task) {
        const int bhh = task / p.NC, n = task % p.NC;
        const int bb = bhh / p.H, hh = bhh % p.H;
        mbar_arrive_expect_tx(&ms.bar_ld, KB_TX - (bsc ? 16384u : 0u));
        tma_load_4d(sm + KB_Q, &tm_q, &ms.bar_ld, 0, hh, n * C, bb);
        tma_load_4d(sm + KB_K, &tm_k, &ms.bar_ld, 0, hh, n * C, bb);
        if (!bsc) tma_load_4d(sm + KB_B, &tm_b, &ms.bar_ld, 0, hh, n * C, bb);
        tma_load_4d(sm + KB_LA, &tm_la, &ms.bar_ld, 0, hh, n * C, bb);
        bulk_load(sm + KB_DPA, p.dpa + (size_t)task * DPA_IMG, DPA_IMG, &ms.bar_ld);
    };
    // the record lands over the previous task's dlog_alpha tile: issued once that has left
    auto issue_record = [&](int task) {
        mbar_arrive_expect_tx(&ms.bar_x, XREC_BYTES);
        bulk_load(sm + KB_X, p.xrec + (size_t)task * XREC_BYTES, XREC_BYTES, &ms.bar_x);
    };
    const int ntasks = p.ntasks;
    if (tid == 0 && (int)blockIdx.x < ntasks) {
        issue_loads(blockIdx.x);
        issue_record(blockIdx.x);
    }

    uint32_t ph_ld = 0, ph_mma = 0, ph_x = 0;
    bool timed_out = false, loads_pending = (int)blockIdx.x < ntasks, x_pending = loads_pending;
    const int o8 = tid & 15, tg = tid >> 4, HI = tg >> 3;  // prep: channels 8 o8.., tokens 4 tg..
    const __nv_bfloat16 *qs = reinterpret_cast<const __nv_bfloat16 *>(sm + KB_Q);
    const __nv_bfloat16 *ks_ = reinterpret_cast<const __nv_bfloat16 *>(sm + KB_K);
    const __nv_bfloat16 *bs = reinterpret_cast<const __nv_bfloat16 *>(sm + KB_B);
    float *Gs = reinterpret_cast<float *>(sm + KB_LA);
    float *scan = reinterpret_cast<float *>(sm + KB_SCAN);

    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int bhh = task / p.NC, n = task % p.NC;
        const int bb = bhh / p.H, hh = bhh % p.H;
        const int t0 = n * C, Cn = min(C, p.T - t0);
        // a scalar erase gate: this thread's four rows (t = tid / 16 + 16 k), read while the copies land
        __nv_bfloat16 gb4[4];
        if (bsc) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = (tid >> 4) + 16 * k;
                gb4[k] = t < Cn ? p.bsc[((size_t)bb * p.T + t0 + t) * p.H + hh] : __float2bfloat16_rn(0.f);
            }
        }
        {
            const bool ok = mbar_wait_bounded(&ms.bar_ld, ph_ld, kWaitLimitNs);
            if (__syncthreads_or(!ok)) { timed_out = true; break; }
            ph_ld ^= 1u;
        }
        loads_pending = false;
        if (bsc) {
            // its rows of the b tile hold that value in every channel (first read after the
            // barrier that ends the decay scan below)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = (tid >> 4) + 16 * k;
                const __nv_bfloat162 g2 = __halves2bfloat162(gb4[k], gb4[k]);
                uint4 u;
                u.x = u.y = u.z = u.w = *reinterpret_cast<const uint32_t *>(&g2);
                *reinterpret_cast<uint4 *>(sm + KB_B + t * 256 + (tid & 15) * 16) = u;
            }
        }
        // ================= prep: cumulative decay, references, decay-weighted operands =================
        float G[4][8];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float la[8];
            load8f(Gs + (tg * 4 + m) * DK + o8 * 8, la);
#pragma unroll
            for (int x = 0; x < 8; ++x) G[m][x] = (m == 0 ? 0.f : G[m - 1][x]) + clamp_log_alpha(la[x]);
        }
        store8f(scan + tg * DK + o8 * 8, G[3]);
        __syncthreads();
        if (tid < DK) {
            float run = 0.f, g0 = 0.f, g1 = 0.f;
#pragma unroll
            for (int g = 0; g < 16; ++g) {
                if (g == 4) g0 = run;
                if (g == 12) g1 = run;
                const float v = scan[g * DK + tid];
                scan[g * DK + tid] = run;
                run += v;
            }
            ms.g0[tid] = g0;
            ms.g1[tid] = g1;
            ms.gC[tid] = run;
        }
        if (tid == 0 && task != (int)blockIdx.x) {
            bulk_wait_group_read0();  // the previous task's gradient tiles have left STACK, R and X
            issue_record(task);
            x_pending = true;
        }
        __syncthreads();
        bool risky = false;
        {
            float ex[8], g0[8], g1[8];
            load8f(scan + tg * DK + o8 * 8, ex);
            load8f(ms.g0 + o8 * 8, g0);
            load8f(ms.g1 + o8 * 8, g1);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
                for (int x = 0; x < 8; ++x) G[m][x] += ex[x];
                store8f(Gs + (tg * 4 + m) * DK + o8 * 8, G[m]);  // over this thread's own log_alpha
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int t = tg * 4 + m;
                float qv[8], kv[8], bv[8], le[8], lq[8], r[8];
                unpack8(*reinterpret_cast<const uint4 *>(qs + t * DK + o8 * 8), qv);
                unpack8(*reinterpret_cast<const uint4 *>(ks_ + t * DK + o8 * 8), kv);
                unpack8(*reinterpret_cast<const uint4 *>(bs + t * DK + o8 * 8), bv);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float d = G[m][x] - (HI ? g1[x] : g0[x]);
                    risky |= fabsf(d) > kFactorLimit;
                    const float xl = __expf(d), yr = recip_newton2(xl);
                    le[x] = bv[x] * kv[x] * xl;
                    lq[x] = qv[x] * xl;
                    r[x] = kv[x] * yr;
                }
                const int tl = t - 32 * HI;
                *reinterpret_cast<uint4 *>(sm + KB_STACK + sw_chunk(64 * HI + tl, o8, 128)) = pack8(le);
                *reinterpret_cast<uint4 *>(sm + KB_STACK + sw_chunk(64 * HI + 32 + tl, o8, 128)) = pack8(lq);
                if (HI == 0) {
                    *reinterpret_cast<uint4 *>(sm + KB_R + sw_chunk(t, o8, R_ROWS)) = pack8(r);
                    float r1[8];
#pragma unroll
                    for (int x = 0; x < 8; ++x) r1[x] = kv[x] * __expf(g1[x] - G[m][x]);
                    *reinterpret_cast<uint4 *>(sm + KB_R + sw_chunk(32 + t, o8, R_ROWS)) = pack8(r1);
                } else {
                    *reinterpret_cast<uint4 *>(sm + KB_R + sw_chunk(32 + t, o8, R_ROWS)) = pack8(r);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        const bool exact = __syncthreads_or(risky) != 0;
        tc_fence_after_sync();
        if (!exact) {
            // D_I[c][r] = sum_i R_I[i][c] DPA[64 I + r][i];  E_I[c][i] = sum_r STACK[64 I + r][c] DPA[64 I + r][i]
            if (tid == 0) {
                const uint32_t idD = idesc_bf16(128, 64, true, false);
                const uint32_t idE = idesc_bf16(128, 64, true, true);
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2)
                    mma_bf16(tm + KT_D0, sdesc_sw128(sb + KB_R + k2 * 2048, R_ROWS * 128, 1024),
                             sdesc_sw128(sb + KB_DPA + k2 * 32, 16, 1024), idD, k2 > 0);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    mma_bf16(tm + KT_D1, sdesc_sw128(sb + KB_R + 4096 + k4 * 2048, R_ROWS * 128, 1024),
                             sdesc_sw128(sb + KB_DPA + 8192 + k4 * 32, 16, 1024), idD, k4 > 0);
                    mma_bf16(tm + KT_E0, sdesc_sw128(sb + KB_STACK + k4 * 2048, 16384, 1024),
                             sdesc_sw128(sb + KB_DPA + k4 * 2048, 8192, 1024), idE, k4 > 0);
                    mma_bf16(tm + KT_E1, sdesc_sw128(sb + KB_STACK + 8192 + k4 * 2048, 16384, 1024),
                             sdesc_sw128(sb + KB_DPA + 8192 + k4 * 2048, 8192, 1024), idE, k4 > 0);
                }
                mma_commit(&ms.bar_mma);
            }
            const bool ok = mbar_wait_bounded(&ms.bar_mma, ph_mma, kWaitLimitNs);
            ph_mma ^= 1u;
            if (__syncthreads_or(!ok)) { timed_out = true; break; }
            tc_fence_after_sync();
        }
        {
            const bool ok = mbar_wait_bounded(&ms.bar_x, ph_x, kWaitLimitNs);
            if (__syncthreads_or(!ok)) { timed_out = true; break; }
            ph_x ^= 1u;
            x_pending = false;
        }
        // ================= per channel: thread (c, half hf) walks tokens 32 hf .. 32 hf + 31 =================
        const int c = quarter * 32 + lane;
        const float g0c = ms.g0[c], g1c = ms.g1[c], gCc = ms.gC[c];
        const float ghc = hf ? g1c : g0c;
        const __nv_bfloat16 *X = reinterpret_cast<const __nv_bfloat16 *>(sm + KB_X);
        const float *dpd = reinterpret_cast<const float *>(sm + KB_X + 3 * X_ARR);
        const float rowsum = dpd[64 + c];
        __nv_bfloat16 *oq = reinterpret_cast<__nv_bfloat16 *>(sm + KB_STACK);
        __nv_bfloat16 *ok_ = reinterpret_cast<__nv_bfloat16 *>(sm + KB_STACK + 16384);
        __nv_bfloat16 *ob = reinterpret_cast<__nv_bfloat16 *>(sm + KB_R);
        const unsigned char *dpa = sm + KB_DPA;
        if (exact) {
            // A chunk past the decay guard: the four decay products with one exponential per token
            // pair (exponents never positive), written where the tensor-core path leaves D and E,
            // with every decay factor 1 below. Kept out of the unrolled loop: it is rare, and its
            // code there would be repeated for every token.
            for (int blk = 0; blk < 2; ++blk) {
                uint32_t pq[16], pe[16], pk[16], zz[16];
                for (int u = 0; u < 16; ++u) {
                    const int t = 32 * hf + 16 * blk + u;
                    const float Gt = Gs[t * DK + c];
                    float dqP = 0.f, deA = 0.f, dkAP = 0.f;
                    const int rA = 64 * (t >> 5) + (t & 31);
                    for (int i = 0; i < t; ++i) {
                        const float f = __bfloat162float(ks_[i * DK + c]) * __expf(Gt - Gs[i * DK + c]);
                        dqP = fmaf(img64(dpa, rA + 32, i), f, dqP);
                        deA = fmaf(img64(dpa, rA, i), f, deA);
                    }
                    for (int s2 = t + 1; s2 < C; ++s2) {
                        const int rs = 64 * (s2 >> 5) + (s2 & 31);
                        const float ksv = __bfloat162float(ks_[s2 * DK + c]);
                        const float x = img64(dpa, rs, t) * __bfloat162float(bs[s2 * DK + c]) * ksv +
                                        img64(dpa, rs + 32, t) * __bfloat162float(qs[s2 * DK + c]);
                        dkAP = fmaf(x, __expf(Gs[s2 * DK + c] - Gt), dkAP);
                    }
                    pq[u] = __float_as_uint(dqP);
                    pe[u] = __float_as_uint(deA);
                    pk[u] = __float_as_uint(dkAP);
                    zz[u] = 0u;
                }
                tmem_st16u(tm_lane + (hf ? KT_D1 : KT_D0) + 16 * blk, pe);
                tmem_st16u(tm_lane + (hf ? KT_D1 : KT_D0) + 32 + 16 * blk, pq);
                tmem_st16u(tm_lane + KT_E1 + 32 * hf + 16 * blk, pk);
                tmem_st16u(tm_lane + KT_E0 + 32 * hf + 16 * blk, zz);
            }
        }
        float dG[32];
        float hs = 0.f, kts = 0.f;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            float De[16], Dq[16], E1[16], E0[16];
            tmem_ld16(tm_lane + (hf ? KT_D1 : KT_D0) + 16 * blk, De);
            tmem_ld16(tm_lane + (hf ? KT_D1 : KT_D0) + 32 + 16 * blk, Dq);
            tmem_ld16(tm_lane + KT_E1 + 32 * hf + 16 * blk, E1);
            tmem_ld16(tm_lane + KT_E0 + 32 * hf + 16 * blk, E0);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int tl = 16 * blk + u, t = 32 * hf + tl;
                const float Gt = Gs[t * DK + c];
                const float qf = __bfloat162float(qs[t * DK + c]);
                const float kf = __bfloat162float(ks_[t * DK + c]);
                const float bf_ = __bfloat162float(bs[t * DK + c]);
                const float xq = __bfloat162float(X[t * DK + c]);
                const float xe = __bfloat162float(X[(64 + t) * DK + c]);
                const float xk = __bfloat162float(X[(128 + t) * DK + c]);
                const float eG = __expf(Gt), kcf = __expf(gCc - Gt);
                // the decay factors of the products' half-chunk references (1 on the exact path)
                const float Lf = exact ? 1.f : __expf(Gt - ghc);
                const float dqP = Dq[u] * Lf;
                const float deA = De[u] * Lf;
                float dkAP = E1[u] * (exact ? 1.f : __expf(g1c - Gt));
                if (hf == 0 && !exact) dkAP = fmaf(E0[u], __expf(g0c - Gt), dkAP);
                const float dq = fmaf(xq, eG, dqP);
                const float de = fmaf(-xe, eG, deA);
                const float dkt = xk * kcf;
                // dG without its dk~ term: that term enters dlog_alpha as a prefix sum below
                const float g = de * bf_ * kf - dkAP * kf + dq * qf;
                dG[tl] = g;
                hs += g;
                kts = fmaf(dkt, kf, kts);
                const float dpt = dpd[t];
                oq[t * DK + c] = __float2bfloat16_rn(fmaf(dpt, kf, dq));
                ok_[t * DK + c] = __float2bfloat16_rn(dkAP + dpt * qf + dkt + de * bf_);
                if (!bsc) {
                    ob[t * DK + c] = __float2bfloat16_rn(de * kf);
                } else {
                    // db_t = sum_c de[t][c] k[t][c]: this warp's 32 channels here, the quarters below
                    float x = de * kf;
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                    if (lane == 0) ms.red[quarter][t] = x;
                }
            }
        }
        ms.hsum[hf][c] = hs;
        ms.kts[hf][c] = kts;
        __syncthreads();  // every read of G (the exact path reads the other half's) is done
        if (bsc && tid < Cn)
            p.gbsc[((size_t)bb * p.T + t0 + tid) * p.H + hh] =
                __float2bfloat16_rn(ms.red[0][tid] + ms.red[1][tid] + ms.red[2][tid] + ms.red[3][tid]);
        // dlog_alpha[t] = sum_{t' >= t} dG[t'] + sum_j dS' (.) S e^{G_C} + sum_{t' < t} dk~ (.) k~:
        // the last sum as a prefix (as total minus suffix it cancels: the last token's term is
        // O(1) while under strong decay every other term, and the result, are near e^-32)
        // (staged as a [64 t][128 c] fp32 tile over X_q and X_e, whose reads ended at the barrier)
        {
            float *Dl = reinterpret_cast<float *>(sm + KB_X);
            static_assert(2 * X_ARR == C * DK * 4, "the dlog_alpha tile fits X_q and X_e");
            float pre = hf ? ms.kts[0][c] : 0.f;
#pragma unroll 4
            for (int tl = 0; tl < 32; ++tl) {
                const int t = 32 * hf + tl;
                const float Gt = Gs[t * DK + c];
                const float ktk = __bfloat162float(X[(128 + t) * DK + c]) * __expf(gCc - Gt) *
                                  __bfloat162float(ks_[t * DK + c]);
                Dl[t * DK + c] = pre;
                pre += ktk;
            }
            float run = rowsum * __expf(gCc) + (hf == 0 ? ms.hsum[1][c] : 0.f);
#pragma unroll
            for (int tl = 31; tl >= 0; --tl) {
                run += dG[tl];
                Dl[(32 * hf + tl) * DK + c] += run;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_gq, sm + KB_STACK, 0, hh, n * C, bb);
            tma_store_4d(&tm_gk, sm + KB_STACK + 16384, 0, hh, n * C, bb);
            if (!bsc) tma_store_4d(&tm_gb, sm + KB_R, 0, hh, n * C, bb);
            tma_store_4d(&tm_gla, sm + KB_X, 0, hh, n * C, bb);
            bulk_commit_group();
            // q, k, b, log_alpha and the dA/dP image are no store's source: the next task's
            // copies go out now, under the stores (its record follows once they have left)
            if (task + (int)gridDim.x < ntasks) {
                issue_loads(task + gridDim.x);
                loads_pending = true;
            }
        }
    }
    if (tid == 0) {
        bulk_wait_group0();
        if (timed_out) {
            if (loads_pending) mbar_wait_bounded(&ms.bar_ld, ph_ld, kWaitLimitNs);
            if (x_pending) mbar_wait_bounded(&ms.bar_x, ph_x, kWaitLimitNs);
            atomicOr(p.status, kStatusTimeout);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

struct BwdTcLayout {
    size_t ntasks, ext, dsc, dpa, xrec, states, o, sync, total;
};

BwdTcLayout bwd_tc_layout(int B, int T, int H)
{
    BwdTcLayout L;
    const size_t NC = (size_t)(T + C - 1) / C;
    L.ntasks = (size_t)B * H * NC;
    size_t off = al1k(L.ntasks * (SLOT_BYTES + GAMMA_BYTES));  // the forward's slots and gammas
    L.ext = off;
    off += al1k(L.ntasks * EXT_BYTES);
    L.dsc = off;
    off += al1k(L.ntasks * DS_IMG);
    L.dpa = off;
    off += al1k(L.ntasks * DPA_IMG);
    L.xrec = off;
    off += al1k(L.ntasks * XREC_BYTES);
    L.states = off;  // chunk-entry states when the caller has none
    off += al1k(L.ntasks * DK * DV * sizeof(float));
    L.o = off;       // the forward's output, unused
    off += al1k((size_t)B * T * H * DV * 2);
    L.sync = off;    // the fused front's queue counter and task flags
    off += al1k(fused_sync_bytes_for(L.ntasks));
    L.total = off;
    return L;
}

}  // namespace

bool backward_tc_supported(const BwdArgs &a)
{
    return a.bf16 && a.dk == DK && a.dv == DV && a.T > 0 && encode_fn() != nullptr;
}

size_t backward_tc_workspace_bytes(int B, int T, int H) { return bwd_tc_layout(B, T, H).total; }

cudaError_t launch_backward_tc(const BwdArgs &a, cudaStream_t s)
{
    const BwdTcLayout L = bwd_tc_layout(a.B, a.T, a.H);
    unsigned char *ws = static_cast<unsigned char *>(a.workspace);
    const int NC = (a.T + C - 1) / C;
    const int ntasks = (int)L.ntasks;
    float *states = a.saved_states ? const_cast<float *>(a.saved_states) : reinterpret_cast<float *>(ws + L.states);

    // 1. the forward's chunk tasks (and, without saved states, its scans for the states)
    FwdArgs fa{};
    fa.B = a.B; fa.T = a.T; fa.H = a.H; fa.dk = DK; fa.dv = DV; fa.bf16 = true;
    fa.q = a.q; fa.k = a.k; fa.v = a.v; fa.log_alpha = a.log_alpha; fa.b = a.b; fa.w = a.w; fa.S0 = a.S0;
    fa.o = ws + L.o;
    fa.S_T = nullptr;
    fa.saved_states = a.saved_states ? nullptr : states;
    fa.workspace = ws;
    fa.workspace_bytes = L.ext;
    fa.status = a.status;
    fa.cu_seqlens = nullptr;
    fa.gates = a.gates;
    fa.out_gate = nullptr;
    fa.norm_weight = nullptr;
    fa.norm_eps = 0.f;
    fa.bwd_ext = ws + L.ext;
    fa.chunks_only = a.saved_states != nullptr;
    fa.fused_sync = ws + L.sync;  // without saved states: the forward's fused launch keeps T and W
    // with saved states, the chunk tasks and the reverse scans (step 2) as one launch where it fits
    bool front_fused = false;
    cudaError_t e = cudaSuccess;
    if (a.saved_states) {
        const BwdFrontArgs r{a.dO, a.dS_T, a.gS0, ws + L.dsc, ws + L.sync};
        e = launch_backward_front_fused(fa, r, s, &front_fused);
        if (e != cudaSuccess) return e;
    }
    if (!front_fused) {
        e = launch_forward_tc(fa, s);
        if (e != cudaSuccess) return e;
    }

    const bool bsc = (a.gates & kGateScalarB) != 0, wsc = (a.gates & kGateScalarW) != 0;
    CUtensorMap mdo, mq, mk, mb, mla, mgq, mgk, mgb, mgla;
    if (!make_map(&mdo, a.dO, false, a.B, a.T, a.H, DV, 64, true) ||
        !make_map(&mq, a.q, false, a.B, a.T, a.H, DK) || !make_map(&mk, a.k, false, a.B, a.T, a.H, DK) ||
        !make_map(&mla, a.log_alpha, true, a.B, a.T, a.H, DK) || !make_map(&mgq, a.gq, false, a.B, a.T, a.H, DK) ||
        !make_map(&mgk, a.gk, false, a.B, a.T, a.H, DK) || !make_map(&mgla, a.glog_alpha, true, a.B, a.T, a.H, DK))
        return cudaErrorInvalidValue;
    // a scalar erase gate has no tiles to copy: the q and dq maps stand in, unused
    if (bsc) {
        mb = mq;
        mgb = mgq;
    } else if (!make_map(&mb, a.b, false, a.B, a.T, a.H, DK) || !make_map(&mgb, a.gb, false, a.B, a.T, a.H, DK)) {
        return cudaErrorInvalidValue;
    }
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int grid = ntasks < nsm ? ntasks : nsm;

    // 2. reverse scan
    if (!front_fused) {
        e = cudaFuncSetAttribute(bwd_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RS_SMEM);
        if (e != cudaSuccess) return e;
        RsParams rp{a.B, a.T, a.H, NC, ntasks, ws, a.dS_T, a.gS0, ws + L.dsc, a.status};
        bwd_scan_kernel<<<a.B * a.H, RS_NT, RS_SMEM, s>>>(mdo, rp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }

    // 3. value side
    e = cudaFuncSetAttribute(bwd_value_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)VA_SMEM);
    if (e != cudaSuccess) return e;
    CUtensorMap mgv, mgw;
    if (!make_map(&mgv, a.gv, false, a.B, a.T, a.H, DV)) return cudaErrorInvalidValue;
    if (wsc) mgw = mgv;  // a scalar write gate's dw is reduced in the kernel: no tile
    else if (!make_map(&mgw, a.gw, false, a.B, a.T, a.H, DV)) return cudaErrorInvalidValue;
    VaParams vp{a.B, a.T, a.H, NC, ntasks, ws, ws + L.ext, ws + L.dsc, states,
                static_cast<const __nv_bfloat16 *>(a.v), static_cast<const __nv_bfloat16 *>(a.w),
                static_cast<__nv_bfloat16 *>(a.gv), static_cast<__nv_bfloat16 *>(a.gw), ws + L.dpa, ws + L.xrec,
                a.status, wsc ? 1 : 0};
    bwd_value_kernel<<<grid, 256, VA_SMEM, s>>>(mdo, mgv, mgw, vp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // 4. key side
    e = cudaFuncSetAttribute(bwd_key_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KB_SMEM);
    if (e != cudaSuccess) return e;
    KbParams kp{a.B,      a.T,         a.H,      NC,
                ntasks,   ws + L.dpa,  ws + L.xrec, a.status,
                bsc ? static_cast<const __nv_bfloat16 *>(a.b) : nullptr,
                bsc ? static_cast<__nv_bfloat16 *>(a.gb) : nullptr};
    bwd_key_kernel<<<grid, 256, KB_SMEM, s>>>(mq, mk, mb, mla, mgq, mgk, mgb, mgla, kp);
    return cudaGetLastError();
}

}  // namespace gdr2
