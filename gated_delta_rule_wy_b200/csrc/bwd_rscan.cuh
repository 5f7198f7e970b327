// bwd_rscan.cuh -- the backward's reverse scan of the state gradient: definitions shared by
// bwd_scan_kernel (bwd_tc.cu, nine warps) and the eight-warp role that the fused backward
// front kernel (fwd_tc.cu) runs after its chunk tasks.
//
// Per (batch, head), chunks last to first: dS^T lives in TMEM in fp32 in one of two
// regions that alternate per chunk; a pass writes the previous region's dS'^T as a bf16
// operand in TMEM and as the chunk's bf16 image for the chunk-parallel kernels, and the
// gamma-scaled dS'^T into this region; then dS^T += dS'^T M (A from TMEM) + dO^T Q' as 12
// MMAs.
#pragma once
#include <cstddef>

#include "gdr2_common.cuh"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"

namespace gdr2 {
namespace {

using namespace sm100;
using namespace tc;

constexpr uint32_t DS_IMG = 32768;               // dS'^T in bf16, [j rows 128][c: 2 blocks of 64]
constexpr int RS_NT = 288;                        // bwd_scan_kernel: 8 TMEM warps + the MMA warp
constexpr uint32_t RS_BUF = 65536;                // one chunk: [Q'; M] (49152) then the dO image
constexpr uint32_t RS_DO = 49152;
constexpr uint32_t RS_DS = 2 * RS_BUF;            // two dS'^T images
constexpr uint32_t RS_MISC = RS_DS + 2 * DS_IMG;  // 196608
constexpr uint32_t RS_SA = 256;                   // TMEM: regions at 0 and 128, bf16 copy at 256

struct RsMisc {
    uint64_t bar_full[2];
    uint64_t bar_mma;
    uint32_t tmem_base;
    int pad;
    alignas(16) float gam[2][DK];
};
constexpr uint32_t RS_SMEM = RS_MISC + sizeof(RsMisc) + 1024;
static_assert(offsetof(RsMisc, gam) % 16 == 0, "gamma rows are bulk-copy destinations");

struct RsParams {
    int B, T, H, NC, ntasks;
    const unsigned char *ws;  // slots, then gammas
    const float *dS_T;        // [B][H][DK][DV] or null (zero)
    float *gS0;               // [B][H][DK][DV] or null
    unsigned char *dsc;       // [ntasks][DS_IMG]: dS'^T of every chunk, bf16 images
    unsigned *status;
};

// The reverse scan of (batch, head) bh on eight warps of a CTA whose TMEM allocation (512
// columns at tm) and shared memory it takes over; thread 0 issues the MMAs and the copies,
// and copies a chunk's slot only once flags[task] is set. Records a timeout in the status
// word and in timed_out.
__device__ __forceinline__ void rscan_role(const CUtensorMap &tm_do, const RsParams &p, const unsigned *flags,
                                           unsigned char *sm, uint32_t tm, int bh, bool &timed_out)
{
    RsMisc &ms = *reinterpret_cast<RsMisc *>(sm + RS_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, colhalf = warp >> 2;
    const int bb = bh / p.H, h = bh % p.H;
    const int NC = p.NC;
    const size_t base = (size_t)bh * NC;
    const int c0 = colhalf * 64;
    const int j = quarter * 32 + lane;
    const uint32_t tm_lane = tm + ((uint32_t)(quarter * 32) << 16);

    if (tid == 0) {
        mbar_init(&ms.bar_full[0], 1);
        mbar_init(&ms.bar_full[1], 1);
        mbar_init(&ms.bar_mma, 1);
        fence_mbar_init();
    }
    __syncthreads();
    unsigned pend = 0;  // thread 0: bit b set while buffer b's loads are issued and not yet waited for
    auto issue = [&](int n, int sl) {
        const size_t task = base + n;
        if (!flag_wait_bounded(flags + task, kWaitLimitNs)) return;  // never issued: the wait below gives up
        fence_proxy_async_global();
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
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = p.dS_T ? p.dS_T[((size_t)bh * DK + c0 + q2 * 32 + i) * DV + j] : 0.f;
        tmem_st32(tm_lane + 128 + c0 + q2 * 32, v);
    }
    tc_fence_before_sync();
    __syncthreads();

    unsigned phf = 0;  // bit b: the parity of buffer b's next load phase
    uint32_t ph_mma = 0;
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
        {
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
        if (tid == 0) {
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
    if (!timed_out && p.gS0) {
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
}

}  // namespace
}  // namespace gdr2
