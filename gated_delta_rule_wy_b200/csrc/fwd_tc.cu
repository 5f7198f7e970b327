// fwd_tc.cu -- chunkwise GDR-2 forward on the sm_100a tensor cores (bf16
// inputs, fp32 state), dk = dv = 128.
//
// Algorithm: the chunkwise WY form of the Gated DeltaNet-2 note, sec. 3
// (chunkwise training paragraph): within a chunk of C = 64 tokens the decay
// is absorbed into the gated keys (decay-normalised state S_r =
// Diag(gamma_r) S^_r), which leaves an asymmetric delta recurrence whose
// token products collapse into a unit-lower-triangular solve (UT form) and a
// chain of matmuls; the state crosses chunk boundaries in fp32.
//
//   A_ti = sum_c e_t[c] k_i[c] exp(G_t[c] - G_i[c])   i < t      (e = b (.) k)
//   P_ti = sum_c q_t[c] k_i[c] exp(G_t[c] - G_i[c])   i <= t
//   T = (I + A)^{-1};  W = T (E (.) exp G);  U~ = T Z              (z = w (.) v)
//   U = U~ - W S;  O = (Q (.) exp G) S + P U;  S' = Diag(gamma) S + K~^T U
//
// Regrouped so that the state enters one batch of products per chunk:
//   S' = Diag(gamma) S + M S + K~^T U~,   M  = -K~^T W
//   O  = Q' S + P U~,                     Q' = Q (.) exp G - P W
// Everything except those two lines is independent of S, so the path is two
// kernels:
//   1. chunk kernel (persistent, every (batch, head, chunk) task in parallel
//      on all SMs): decay, gated keys, [A;P], the UT solve, W, U~, M, Q';
//      writes [Q'; M], K~, U~, P (bf16, already in the tensor-core operand
//      layouts of kernel 2) and gamma = exp(G_C) to the workspace;
//   2. scan kernel (one CTA per (batch, head), chunks in order): S^T stays in
//      TMEM as fp32; per chunk one pass copies it to a bf16 TMEM operand and
//      scales it by gamma, then one batch of MMAs produces S'^T and O^T.
// A scan's chunks are a serial chain (about 2.3 K cycles each) on one SM, so run
// after the chunk kernel the scans leave most SMs idle. Where B H leaves at least
// 32 SMs free, both run as one cooperative launch instead (fwd_fused_kernel):
// every CTA takes chunk tasks from a queue in chunk-major order, and CTA b < B H
// leaves the queue near its end for the scan of (batch, head) b, which copies a
// chunk's workspace slot only once that task's flag says it is written. The scans
// then overlap the last quarter or so of the chunk tasks. The same launch serves a
// forward that saves its chunk-entry states and the backward's recomputation of them
// (T and W kept); the backward's front (bwd_front_kernel) is fused alike, its queue
// running from the last chunk back for the reverse scans of the state gradient.
//
// Decay range. exp(G_t - G_i) is formed as a product of two factors around a
// per-channel reference g_I, the cumulative decay at the midpoint of the
// 32-token half-chunk I that holds t:
//   L_t = x_t exp(G_t - g_I),   R_i = k_i exp(g_I - G_i).
// The guard requires |G_t - g_I| <= 70 for every token against its own
// half's reference. Keys of the first half also meet second-half rows, through
// R1_i = k_i exp(g_1 - G_i), formed with one exponential: if it underflows
// (g_1 - G_i < -87), every product it enters has G_t - G_i = (G_t - g_1) +
// (g_1 - G_i) < 70 - 87, so only terms below exp(-17) are lost; the same bound
// covers the other factors that can underflow (exp(g_I), exp(G_C - g_I)).
// When the guard trips (alpha near 0 over much of a chunk, e.g. a reset) the
// chunk takes an exact path: A and P with one exponential per (t, i, c), and
// the decay-weighted operands from exp(G) directly.
//
// Tensor-core mapping (M = 128 everywhere; t, i, s tokens, c key channel,
// j value channel; accumulators fp32 in TMEM, operands bf16 in
// 128-byte-swizzled shared memory written by the threads, inputs staged by
// TMA without multicast; one thread issues every MMA):
//   chunk kernel: [A;P] = [L^e_0; L^q_0; L^e_1; L^q_1] [R_0; R_1]^T (K = c)
//                 W^T_I = (L^e_I)^T T[:, I]^T, W = sum_I exp(g_I) W_I
//                 U~^T = Z^T T^T;  Q' - Q^ = -P W (M = 64);  M = -K~^T W
//   scan kernel:  [O^T | S^T] += S_bf16^T [Q'; M]^T   (A from TMEM, N = 192)
//                 S^T += U~^T K~;  O^T += U~^T P^T
// Every mbarrier wait is bounded; a CTA that gives up records kStatusTimeout,
// frees its TMEM and exits.

#include <cuda.h>
#include <cstddef>
#include <mutex>

#include "gdr2_common.cuh"
#include "gdr2_launch.h"
#include "sm100_ptx.cuh"
#include "tc_common.cuh"
#include "bwd_rscan.cuh"

namespace gdr2 {
namespace {

using namespace sm100;
using namespace tc;

constexpr int NT = 256;                           // 8 warps; warps w and w+4 share TMEM lanes 32*(w%4)..

// ---- shared-memory map (bytes from a 1024-aligned base) ----
constexpr uint32_t OFF_STG_Q = 0;       // q  [64][128] bf16
constexpr uint32_t OFF_STG_K = 16384;   // k
constexpr uint32_t OFF_STG_B = 32768;   // b
constexpr uint32_t OFF_STG_V = 49152;   // v; exact path: A (fp32 [64][68]) over V and W
constexpr uint32_t OFF_STG_W = 65536;   // w
constexpr uint32_t OFF_STG_LA = 81920;  // log_alpha [64][128] fp32; then G
constexpr uint32_t OFF_STACK = 114688;  // [L^e_0; L^q_0; L^e_1; L^q_1] 128 x 128; later W as [c][64 t]
constexpr uint32_t OFF_R0 = 147456;     // [R_0; R_1] (32 + 64 rows) x 128 as one B operand (24 KB); then
                                        // A and T (fp32 [64][68]) with the block-product scratch, then
                                        // T (bf16 [64][64]); last, the tail of [Q'; M] (staged from STACK on)

constexpr uint32_t OFF_Z = 172032;      // Z 64 x 128 (value side); later U~^T as [j][64 t] for the slot
constexpr uint32_t OFF_QH = 188416;     // Q^ = Q (.) exp G, [t rows][128 c] (K-major chunks)
constexpr uint32_t OFF_KT = 204800;     // K (.) exp(G_C - G), 64 x 128
constexpr uint32_t OFF_P = 221184;      // per-channel references during prep; then P 64 x 64
constexpr uint32_t OFF_MISC = 229376;   // barriers, per-channel vectors
constexpr uint32_t MISC_BYTES = 1664;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
constexpr int F_LD = 68;                // fp32 row stride of the A / T scratch
constexpr uint32_t OFF_A32 = OFF_R0;     // A, solved in place into T
constexpr uint32_t OFF_Y = OFF_R0 + 64 * F_LD * 4;  // block-product scratch, 32 x 36 fp32
constexpr int Y_LD = 36;
constexpr uint32_t OFF_TB = OFF_R0;      // T in bf16, K-major [t][64 s]
constexpr uint32_t TX_BYTES = 5 * 16384 + 32768;
constexpr int R_ROWS = 96;               // rows of the stacked [R_0; R_1] operand
static_assert(OFF_STACK + 2 * 192 * 128 <= OFF_Z, "[Q'; M] (48 KB) is staged over STACK and R, clear of Z");

constexpr uint32_t TM_COLS = 512;  // TMEM columns of the chunk kernel
// Fused kernel: at least this many CTAs stay on the chunk queue while B H of them scan, and the
// ratio of a scan's time per chunk to a chunk task's time that places the switch.
constexpr int kFusedMinQueueCtas = 32;
constexpr double kScanToTaskTime = 0.25;
constexpr double kLongScanToTaskTime = 0.22;    // from 256 chunks per sequence (measured better there)
constexpr double kSavingScanToTaskTime = 0.35;  // the same when the scans also write the chunk states
constexpr double kRevScanToTaskTime = 0.25;  // the same for the backward's front (reverse scans)

struct Misc {
    uint64_t bar_tma;
    uint64_t bar_mma;
    uint32_t tmem_base;
    int q_next;      // fused kernel: the queue index this CTA takes next
    int pad[2];
    int loc_next[4];  // packed sequences: where the next task's chunk lives (h, t0, bb, Cn)
    float gC[DK];    // exp(G_C)
    float eg0[DK];   // W combine factor of half-chunk 0: exp(g_0)
    float eg1[DK];   // ... of half-chunk 1: exp(g_1)
};
static_assert(sizeof(Misc) <= MISC_BYTES, "misc region");
static_assert(offsetof(Misc, gC) % 16 == 0, "per-channel vectors are 16-byte aligned");

struct ChunkParams {
    int B, T, H, NC;
    int ntasks;            // slot capacity: B * H * NC (dense), task = bh * NC + n
    unsigned char *ws;     // workspace: ntasks slots, then ntasks gamma vectors
    unsigned *status;
    // packed sequences (null when dense): B sequences of cu_seqlens[s+1] - cu_seqlens[s]
    // tokens in one [1, T, H, D] tensor; sequence s owns the H * nc_s tasks from
    // H * cu_chunks[s] on (head-major, then chunk), nc_s = cu_chunks[s+1] - cu_chunks[s]
    const int *cu_seqlens;
    const int *cu_chunks;
    const int *ntasks_dev;  // H * cu_chunks[B], written by the prefix kernel
    int gates;              // kGate* bits: a scalar gate is read here, not by the copy engine
    const __nv_bfloat16 *bg, *wg;
    unsigned char *ext;     // backward: T and W of every task (EXT_BYTES each), else null
    int debug_giveup;       // test hook: give up a 1 us wait before the first copy
    // fused kernel (dense, vector gates): a task queue in chunk-major order and one ready flag
    // per task (both zero at launch); CTA b < BH leaves the queue for the scan of (sequence,
    // head) b once the queue index it holds reaches switch_at
    int *queue = nullptr;
    unsigned *flags = nullptr;
    int BH = 0, switch_at = 0;
};

// Where a task's chunk lives: tensor-map coordinates (token t0, sequence bb), head h, and the
// number of real tokens Cn in it.
struct ChunkLoc {
    int h, t0, bb, Cn;
};

template <bool GENERAL>
__device__ __forceinline__ ChunkLoc locate_chunk(const ChunkParams &p, int task)
{
    ChunkLoc L;
    if (!GENERAL || !p.cu_seqlens) {
        const int bh = task / p.NC, n = task % p.NC;
        L.bb = bh / p.H;
        L.h = bh % p.H;
        L.t0 = n * C;
        L.Cn = min(C, p.T - n * C);
        return L;
    }
    // the sequence s with H cu_chunks[s] <= task < H cu_chunks[s + 1] (binary search)
    int lo = 0, hi = p.B;  // invariant: H cu_chunks[lo] <= task < H cu_chunks[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.H * p.cu_chunks[mid] <= task) lo = mid; else hi = mid;
    }
    const int nc = p.cu_chunks[lo + 1] - p.cu_chunks[lo];
    const int rem = task - p.H * p.cu_chunks[lo];
    const int n = rem % nc;
    L.h = rem / nc;
    L.bb = 0;
    L.t0 = p.cu_seqlens[lo] + n * C;
    L.Cn = min(C, p.cu_seqlens[lo + 1] - L.t0);
    return L;
}

// Packed sequences: chunk offsets per sequence and the task count, after checking that
// cu_seqlens runs from 0 to T without decreasing. If it does not, no task runs (the count
// is 0 and every offset 0) and the status word records it. Also the order in which the scan
// kernel takes the sequences: longest first (a scan's time is its chunk count, so the long
// ones must not start last), ties by index; up to kOrderMax sequences, by a bitonic sort in
// shared memory, else the given order. One block.
constexpr int kOrderMax = 2048;

__global__ void __launch_bounds__(1024) varlen_prefix_kernel(const int *cu, int N, int T, int H, int *cu_chunks,
                                                             int *ntasks, int *order, unsigned *status)
{
    __shared__ int part[1024];
    __shared__ int key[kOrderMax], idx[kOrderMax];
    const int tid = threadIdx.x;
    const int per = (N + 1023) / 1024;
    const int i0 = tid * per, i1 = min(N, i0 + per);
    int sum = 0;
    bool bad = false;
    for (int i = i0; i < i1; ++i) {
        const int len = cu[i + 1] - cu[i];
        bad |= len < 0;
        sum += (max(len, 0) + C - 1) / C;
    }
    if (tid == 0) bad |= cu[0] != 0 || cu[N] != T;
    bad = __syncthreads_or(bad) != 0;
    part[tid] = sum;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive scan of the per-thread sums
        const int v = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    int run = part[tid] - sum;  // exclusive
    for (int i = i0; i < i1; ++i) {
        cu_chunks[i] = bad ? 0 : run;
        run += (max(cu[i + 1] - cu[i], 0) + C - 1) / C;
    }
    if (tid == 1023) {
        cu_chunks[N] = bad ? 0 : part[1023];
        *ntasks = bad ? 0 : H * part[1023];
        if (bad) atomicOr(status, kStatusBadSeqlens);
    }
    if (N > kOrderMax || bad) {
        for (int i = tid; i < N; i += 1024) order[i] = i;
        return;
    }
    int P = 1;
    while (P < N) P <<= 1;
    for (int i = tid; i < P; i += 1024) {
        key[i] = i < N ? (max(cu[i + 1] - cu[i], 0) + C - 1) / C : -1;  // padding sorts last
        idx[i] = i;
    }
    __syncthreads();
    // "a before b": more chunks, or as many and a smaller index
    auto before = [&](int a, int b) { return key[a] > key[b] || (key[a] == key[b] && idx[a] < idx[b]); };
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += 1024) {
                const int l = i ^ j;
                if (l > i && (((i & k) == 0) ? before(l, i) : before(i, l))) {
                    const int tk = key[i], ti = idx[i];
                    key[i] = key[l]; idx[i] = idx[l];
                    key[l] = tk; idx[l] = ti;
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < N; i += 1024) order[i] = idx[i];
}

// TMEM columns of the chunk kernel
constexpr uint32_t CK_M = 0, CK_U = 128, CK_W0 = 256, CK_W1 = 320, CK_AP0 = 384, CK_AP1 = 416;
constexpr uint32_t CK_Q = CK_W0;  // Q' - Q^ (M = 64 layout, 128 columns) over W_0, W_1 once those are read

// The chunk kernel's work. GENERAL: packed sequences and/or scalar gates may be in use; the
// other instantiation is the dense, vector-gate kernel with those branches compiled away. BWD
// (dense sequences): T and W of each task also go to p.ext for the backward. FUSED (dense
// sequences): the first role of the fused forward or backward-front kernel -- tasks come from a queue in chunk-major
// order, each finished task is published by its flag, and the TMEM allocation is kept for the
// scan role (tm_out). Returns whether a bounded wait gave up (the same on every thread).
template <bool GENERAL, bool BWD, bool FUSED, bool REV = false>
__device__ __forceinline__ bool chunk_body(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_b,
                                           const CUtensorMap &tm_v, const CUtensorMap &tm_w, const CUtensorMap &tm_la,
                                           const ChunkParams &p, unsigned char *sm, uint32_t &tm_out)
{
    Misc &ms = *reinterpret_cast<Misc *>(sm + OFF_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, colhalf = warp >> 2;

    if (tid == 0) {
        mbar_init(&ms.bar_tma, 1);
        mbar_init(&ms.bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&ms.tmem_base, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tm = ms.tmem_base;
    const uint32_t tm_lane = tm + ((uint32_t)(quarter * 32) << 16);  // this warp's TMEM lanes
    const int row = quarter * 32 + lane;                              // this thread's TMEM lane

    const int ntasks = (GENERAL && p.cu_seqlens) ? *p.ntasks_dev : p.ntasks;
    const bool bsc = GENERAL && (p.gates & kGateScalarB) != 0, wsc = GENERAL && (p.gates & kGateScalarW) != 0;
    const uint32_t tx_bytes = TX_BYTES - (bsc ? 16384u : 0u) - (wsc ? 16384u : 0u);
    // Packed sequences: a task's location takes a binary search over cu_chunks (dependent global
    // loads), so the thread that issues its copies also leaves it in shared memory for the rest.
    const bool varlen = GENERAL && p.cu_seqlens;
    auto issue_loads = [&](int task) {
        const ChunkLoc L = locate_chunk<GENERAL>(p, task);
        if (varlen) {
            ms.loc_next[0] = L.h;
            ms.loc_next[1] = L.t0;
            ms.loc_next[2] = L.bb;
            ms.loc_next[3] = L.Cn;
        }
        mbar_arrive_expect_tx(&ms.bar_tma, tx_bytes);
        tma_load_4d(sm + OFF_STG_Q, &tm_q, &ms.bar_tma, 0, L.h, L.t0, L.bb);
        tma_load_4d(sm + OFF_STG_K, &tm_k, &ms.bar_tma, 0, L.h, L.t0, L.bb);
        if (!bsc) tma_load_4d(sm + OFF_STG_B, &tm_b, &ms.bar_tma, 0, L.h, L.t0, L.bb);
        tma_load_4d(sm + OFF_STG_V, &tm_v, &ms.bar_tma, 0, L.h, L.t0, L.bb);
        if (!wsc) tma_load_4d(sm + OFF_STG_W, &tm_w, &ms.bar_tma, 0, L.h, L.t0, L.bb);
        tma_load_4d(sm + OFF_STG_LA, &tm_la, &ms.bar_tma, 0, L.h, L.t0, L.bb);
    };
    bool timed_out = false;
    if (p.debug_giveup) {
        // test hook: nothing has been issued yet and nothing arrives on bar_mma, so this
        // bounded wait runs out and the CTA takes its give-up path below
        const bool ok = mbar_wait_bounded(&ms.bar_mma, 0, 1000);
        timed_out = __syncthreads_or(!ok) != 0;
    }
    // queue index -> task (slot): FUSED takes chunk n of every (sequence, head) before chunk n + 1;
    // REV (for the backward's reverse scans) from the last chunk back
    auto task_of = [&](int qi) -> int {
        if (!FUSED) return qi;
        const int n = qi / p.BH;
        return (qi % p.BH) * p.NC + (REV ? p.NC - 1 - n : n);
    };
    int q0 = blockIdx.x;
    if (FUSED) {
        if (tid == 0) ms.q_next = atomicAdd(p.queue, 1);
        __syncthreads();
        q0 = ms.q_next;
    }
    if (!timed_out && tid == 0 && q0 < ntasks) issue_loads(task_of(q0));
    if (varlen) __syncthreads();  // the first task's location
    // the scan kernel may be scheduled now: its CTAs take an SM only once this (persistent) CTA
    // has left it, and they read the workspace only after this whole grid has completed
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    uint32_t ph_tma = 0, ph_mma = 0;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) -> bool {
        const bool ok = mbar_wait_bounded(bar, ph, kWaitLimitNs);
        ph ^= 1u;
        return __syncthreads_or(!ok) == 0;
    };
    auto mma_sync_point = [&]() {  // operands written by threads -> visible to the tensor core
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    };

    // prep mapping: channel octet o8 (channels 8*o8 .. +7), token group tg (tokens 4*tg .. +3)
    const int o8 = tid & 15;
    const int tg = tid >> 4;
    const int HI = tg >> 3;  // half-chunk of this thread's tokens
    float *A32 = reinterpret_cast<float *>(sm + OFF_A32);
    float *Ys = reinterpret_cast<float *>(sm + OFF_Y);

    int prev_task = -1;  // FUSED: the task finished last, whose flag is still to be set
    for (int qi = q0; qi < ntasks && !timed_out;) {
        const int task = task_of(qi);
        ChunkLoc loc;
        if (varlen) {  // left by the thread that issued this task's copies (barriers since)
            loc.h = ms.loc_next[0];
            loc.t0 = ms.loc_next[1];
            loc.bb = ms.loc_next[2];
            loc.Cn = ms.loc_next[3];
        } else {
            loc = locate_chunk<GENERAL>(p, task);
        }
        const int Cn = loc.Cn;
        // a scalar gate: this thread's four rows (t = tid / 16 + 16 k), read while the copies land
        static_assert(C * 16 == 4 * NT, "four 16-byte pieces of a staging row set per thread");
        __nv_bfloat16 gb4[4], gw4[4];
        if (bsc || wsc) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = (tid >> 4) + 16 * k;
                const size_t row = ((size_t)loc.bb * p.T + loc.t0 + t) * p.H + loc.h;
                gb4[k] = (bsc && t < Cn) ? p.bg[row] : __float2bfloat16_rn(0.f);
                gw4[k] = (wsc && t < Cn) ? p.wg[row] : __float2bfloat16_rn(0.f);
            }
        }
        // this task's workspace slot: each section is staged in shared memory and bulk-copied
        unsigned char *slot = p.ws + (size_t)task * SLOT_BYTES;
        if (tid == 64) {
            // K~, P and U~ of the previous task have left shared memory (FUSED: and reached
            // global memory, for its flag)
            if (FUSED) {
                bulk_wait_group0();
                fence_proxy_async_global();
            } else {
                bulk_wait_group_read0();
            }
        }
        if (!wait_bar(&ms.bar_tma, ph_tma)) { timed_out = true; break; }
        if (GENERAL && Cn < C) {
            // a packed sequence's partial chunk: the rows past its end hold the next sequence's
            // tokens (dense chunks get zeros from the copy engine's fill past T); zero them,
            // which makes those rows inert in every product
            for (int i = tid; i < (C - Cn) * 16; i += NT) {
                const int t = Cn + (i >> 4), o = i & 15;
                const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(sm + OFF_STG_Q + t * 256 + o * 16) = z4;
                *reinterpret_cast<uint4 *>(sm + OFF_STG_K + t * 256 + o * 16) = z4;
                *reinterpret_cast<uint4 *>(sm + OFF_STG_B + t * 256 + o * 16) = z4;
                *reinterpret_cast<uint4 *>(sm + OFF_STG_V + t * 256 + o * 16) = z4;
                *reinterpret_cast<uint4 *>(sm + OFF_STG_W + t * 256 + o * 16) = z4;
                *reinterpret_cast<uint4 *>(sm + OFF_STG_LA + t * 512 + o * 32) = z4;
                *reinterpret_cast<uint4 *>(sm + OFF_STG_LA + t * 512 + o * 32 + 16) = z4;
            }
            __syncthreads();
        }
        if (bsc || wsc) {
            // a gate given as one value per token-head: its rows of the staging buffer hold
            // that value in every channel (zero past the chunk's tokens), so that everything
            // below treats it as the vector gate it stands for (first read after the barrier
            // that ends the decay scan)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = (tid >> 4) + 16 * k, o = tid & 15;
                if (bsc) {
                    const __nv_bfloat162 g2 = __halves2bfloat162(gb4[k], gb4[k]);
                    uint4 u;
                    u.x = u.y = u.z = u.w = *reinterpret_cast<const uint32_t *>(&g2);
                    *reinterpret_cast<uint4 *>(sm + OFF_STG_B + t * 256 + o * 16) = u;
                }
                if (wsc) {
                    const __nv_bfloat162 g2 = __halves2bfloat162(gw4[k], gw4[k]);
                    uint4 u;
                    u.x = u.y = u.z = u.w = *reinterpret_cast<const uint32_t *>(&g2);
                    *reinterpret_cast<uint4 *>(sm + OFF_STG_W + t * 256 + o * 16) = u;
                }
            }
        }

        // ================= prep: cumulative decay and decay-weighted operands =================
        // Rows beyond T are zero-filled by TMA (per-sequence extent): padded tokens are inert.
        // Thread (key channel c, half-chunk hc) sums its channel over its 32 tokens in
        // registers; the second half adds the first half's total. G replaces log_alpha in
        // shared memory (each thread overwrites only what it read).
        float *Gs = reinterpret_cast<float *>(sm + OFF_STG_LA);
        float *refs = reinterpret_cast<float *>(sm + OFF_P);  // g0, g1, G_C, first-half totals (until P)
        {
            const int c = tid & (DK - 1), hc = tid >> 7;
            float g[32];
            float run = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                run += clamp_log_alpha(Gs[(32 * hc + i) * DK + c]);
                g[i] = run;
            }
            if (hc == 0) refs[3 * DK + c] = run;  // G at token 31
            __syncthreads();
            const float off = hc ? refs[3 * DK + c] : 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) Gs[(32 * hc + i) * DK + c] = g[i] + off;
            if (hc == 0) {
                refs[c] = g[15];  // G at token 15: reference of half-chunk 0
                ms.eg0[c] = __expf(g[15]);
            } else {
                refs[DK + c] = g[15] + off;       // G at token 47: reference of half-chunk 1
                refs[2 * DK + c] = g[31] + off;   // G_C
                ms.eg1[c] = __expf(g[15] + off);
                ms.gC[c] = __expf(g[31] + off);
            }
        }
        if (tid == 0) {  // ... and [Q'; M] too, before the operands are rebuilt
            if (FUSED) {
                bulk_wait_group0();
                fence_proxy_async_global();
            } else {
                bulk_wait_group_read0();
            }
        }
        __syncthreads();
        if (FUSED && tid == 0 && prev_task >= 0) {
            // every section of the previous task's slot and its gamma are in global memory
            __threadfence();
            st_release_gpu(p.flags + prev_task, 1u);
        }
        bool risky = false;
        float G[4][8];
        float g0[8], g1[8], gC[8];
        load8f(refs + o8 * 8, g0);
        load8f(refs + DK + o8 * 8, g1);
        load8f(refs + 2 * DK + o8 * 8, gC);
#pragma unroll
        for (int m = 0; m < 4; ++m) load8f(Gs + (tg * 4 + m) * DK + o8 * 8, G[m]);
        {
            const __nv_bfloat16 *qs = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_Q);
            const __nv_bfloat16 *ks = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_K);
            const __nv_bfloat16 *bs = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_B);
            const __nv_bfloat16 *vs = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_V);
            const __nv_bfloat16 *ws = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_W);
            float egI[8], kcf[8], gr[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                gr[x] = HI ? g1[x] : g0[x];
                egI[x] = __expf(gr[x]);          // exp(g_I)
                kcf[x] = __expf(gC[x] - gr[x]);  // exp(G_C - g_I)
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int t = tg * 4 + m;
                float qv[8], kv[8], bv[8];
                unpack8(*reinterpret_cast<const uint4 *>(qs + t * DK + o8 * 8), qv);
                unpack8(*reinterpret_cast<const uint4 *>(ks + t * DK + o8 * 8), kv);
                unpack8(*reinterpret_cast<const uint4 *>(bs + t * DK + o8 * 8), bv);
                // z = w (.) v in bf16 pairs: the product of two bf16 values is exact in fp32,
                // so one rounding to bf16 gives the same value as the fp32 route
                uint4 z;
                {
                    const uint4 vr = *reinterpret_cast<const uint4 *>(vs + t * DV + o8 * 8);
                    const uint4 wr = *reinterpret_cast<const uint4 *>(ws + t * DV + o8 * 8);
                    const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vr);
                    const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&wr);
                    __nv_bfloat162 *z2 = reinterpret_cast<__nv_bfloat162 *>(&z);
#pragma unroll
                    for (int x = 0; x < 4; ++x) z2[x] = __hmul2(w2[x], v2[x]);
                }
                float le[8], lq[8], r[8], kt[8], qh[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float d = G[m][x] - gr[x];
                    risky |= fabsf(d) > kFactorLimit;
                    // |d| <= 70 here (or the exact path replaces these): exp(-d) as the
                    // reciprocal of exp(d), off the special-function unit
                    const float xl = __expf(d), yr = recip_newton2(xl);
                    le[x] = bv[x] * kv[x] * xl;
                    lq[x] = qv[x] * xl;
                    r[x] = kv[x] * yr;
                    kt[x] = r[x] * kcf[x];
                    qh[x] = lq[x] * egI[x];
                }
                const int tl = t - 32 * HI;  // token within its half-chunk
                *reinterpret_cast<uint4 *>(sm + OFF_STACK + sw_chunk(64 * HI + tl, o8, 128)) = pack8(le);
                *reinterpret_cast<uint4 *>(sm + OFF_STACK + sw_chunk(64 * HI + 32 + tl, o8, 128)) = pack8(lq);
                if (HI == 0) {
                    *reinterpret_cast<uint4 *>(sm + OFF_R0 + sw_chunk(t, o8, R_ROWS)) = pack8(r);
                    // R_1 row of a first-half key: one exponential, exp(g_1 - G_i), so that no
                    // intermediate factor (such as exp(g_1 - g_0) alone) can underflow
                    float r1[8];
#pragma unroll
                    for (int x = 0; x < 8; ++x) r1[x] = kv[x] * __expf(g1[x] - G[m][x]);
                    *reinterpret_cast<uint4 *>(sm + OFF_R0 + sw_chunk(32 + t, o8, R_ROWS)) = pack8(r1);
                } else {
                    *reinterpret_cast<uint4 *>(sm + OFF_R0 + sw_chunk(32 + t, o8, R_ROWS)) = pack8(r);
                }
                *reinterpret_cast<uint4 *>(sm + OFF_KT + sw_chunk(t, o8, 64)) = pack8(kt);
                *reinterpret_cast<uint4 *>(sm + OFF_Z + sw_chunk(t, o8, 64)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_QH + sw_chunk(t, o8, 64)) = pack8(qh);
            }
        }
        const bool exact = __syncthreads_or(risky) != 0;
        if (exact) {
            // ---- exact path: pairwise exponentials (G is in shared memory already) ----
            const __nv_bfloat16 *qs = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_Q);
            const __nv_bfloat16 *ks = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_K);
            const __nv_bfloat16 *bs = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG_B);
            // operands with one exponential of a non-positive argument each
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int t = tg * 4 + m;
                float qv[8], kv[8], bv[8], le[8], kt[8], qh[8];
                unpack8(*reinterpret_cast<const uint4 *>(qs + t * DK + o8 * 8), qv);
                unpack8(*reinterpret_cast<const uint4 *>(ks + t * DK + o8 * 8), kv);
                unpack8(*reinterpret_cast<const uint4 *>(bs + t * DK + o8 * 8), bv);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float eg = __expf(G[m][x]);
                    le[x] = bv[x] * kv[x] * eg;
                    qh[x] = qv[x] * eg;
                    kt[x] = kv[x] * __expf(gC[x] - G[m][x]);
                }
                const int tl = t - 32 * HI;
                *reinterpret_cast<uint4 *>(sm + OFF_STACK + sw_chunk(64 * HI + tl, o8, 128)) = pack8(le);
                *reinterpret_cast<uint4 *>(sm + OFF_KT + sw_chunk(t, o8, 64)) = pack8(kt);
                *reinterpret_cast<uint4 *>(sm + OFF_QH + sw_chunk(t, o8, 64)) = pack8(qh);
            }
            if (tid < DK) ms.eg0[tid] = ms.eg1[tid] = 1.f;
            // A and P rows: thread -> row t = tid / 4, columns 16*(tid % 4) .. +15
            {
                const int t = tid >> 2, i0 = (tid & 3) * 16;
                float accA[16], accP[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) accA[u] = accP[u] = 0.f;
                if (i0 <= t && t < Cn) {
                    for (int c = 0; c < DK; ++c) {
                        const float gt = Gs[t * DK + c];
                        const float kt_ = __bfloat162float(ks[t * DK + c]);
                        const float et = __bfloat162float(bs[t * DK + c]) * kt_;
                        const float qt = __bfloat162float(qs[t * DK + c]);
#pragma unroll
                        for (int u = 0; u < 16; ++u) {
                            const int i = i0 + u;
                            if (i <= t) {
                                const float f = __bfloat162float(ks[i * DK + c]) * __expf(gt - Gs[i * DK + c]);
                                accA[u] = fmaf(et, f, accA[u]);
                                accP[u] = fmaf(qt, f, accP[u]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = i0 + u;
                    A32[t * F_LD + i] = (i < t) ? accA[u] : 0.f;
                }
#pragma unroll
                for (int k8 = 0; k8 < 2; ++k8) {
                    float pr[8];
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const int i = i0 + k8 * 8 + x;
                        pr[x] = (i <= t) ? accP[k8 * 8 + x] : 0.f;
                    }
                    {
                        const uint4 v = pack8(pr);
                        *reinterpret_cast<uint4 *>(sm + OFF_P + sw_chunk(t, (i0 >> 3) + k8, 64)) = v;
                    }
                }
            }
            fence_proxy_async_smem();  // P and K~ -> the bulk stores below
            __syncthreads();
        } else {
            // ---- tensor-core path: [A;P] = STACK R_I^T ----
            mma_sync_point();
            if (tid == 0) {
                // one N = 96 product: columns [0, 32) against R_0, [32, 96) against R_1
                static_assert(CK_AP1 == CK_AP0 + 32, "AP0 and AP1 are one accumulator");
                const uint32_t idR = idesc_bf16(128, R_ROWS, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks & 3) * 32;
                    const uint64_t ad = sdesc_sw128(sbase + OFF_STACK + (ks >> 2) * 16384 + koff, 16, 1024);
                    const uint64_t br = sdesc_sw128(sbase + OFF_R0 + (ks >> 2) * (R_ROWS * 128) + koff, 16, 1024);
                    mma_bf16(tm + CK_AP0, ad, br, idR, ks > 0);
                }
                mma_commit(&ms.bar_mma);
            }
            if (!wait_bar(&ms.bar_mma, ph_mma)) { timed_out = true; break; }
            tc_fence_after_sync();
            // quarter 0: A rows 0..31, 1: P rows 0..31 (32 columns of AP0),
            // quarter 2: A rows 32..63, 3: P rows 32..63 (64 columns of AP1); colhalf splits columns
            const bool isP = (quarter & 1) != 0;
            const int t = (quarter >= 2 ? 32 : 0) + lane;
            if (quarter < 2) {
                if (colhalf == 0) {
                    float v[32];
                    tmem_ld32(tm_lane + CK_AP0, v);
                    if (!isP) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4 *>(A32 + t * F_LD + i) =
                                make_float4(i < t ? v[i] : 0.f, i + 1 < t ? v[i + 1] : 0.f,
                                            i + 2 < t ? v[i + 2] : 0.f, i + 3 < t ? v[i + 3] : 0.f);
                    } else {
#pragma unroll
                        for (int k8 = 0; k8 < 4; ++k8) {
                            float pr[8];
#pragma unroll
                            for (int x = 0; x < 8; ++x) pr[x] = (k8 * 8 + x <= t) ? v[k8 * 8 + x] : 0.f;
                            {
                                const uint4 v = pack8(pr);
                                *reinterpret_cast<uint4 *>(sm + OFF_P + sw_chunk(t, k8, 64)) = v;
                            }
                        }
                    }
                } else {
                    // columns 32..63 of rows 0..31 are zero
                    if (!isP) {
#pragma unroll
                        for (int i = 32; i < 64; i += 4)
                            *reinterpret_cast<float4 *>(A32 + t * F_LD + i) = make_float4(0.f, 0.f, 0.f, 0.f);
                    } else {
                        const float zz[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int k8 = 4; k8 < 8; ++k8)
                            {
                                const uint4 v = pack8(zz);
                                *reinterpret_cast<uint4 *>(sm + OFF_P + sw_chunk(t, k8, 64)) = v;
                            }
                    }
                }
            } else {
                float v[32];
                tmem_ld32(tm_lane + CK_AP1 + colhalf * 32, v);
                const int ib = colhalf * 32;
                if (!isP) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(A32 + t * F_LD + ib + i) =
                            make_float4(ib + i < t ? v[i] : 0.f, ib + i + 1 < t ? v[i + 1] : 0.f,
                                        ib + i + 2 < t ? v[i + 2] : 0.f, ib + i + 3 < t ? v[i + 3] : 0.f);
                } else {
#pragma unroll
                    for (int k8 = 0; k8 < 4; ++k8) {
                        float pr[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x) pr[x] = (ib + k8 * 8 + x <= t) ? v[k8 * 8 + x] : 0.f;
                        {
                            const uint4 v = pack8(pr);
                            *reinterpret_cast<uint4 *>(sm + OFF_P + sw_chunk(t, colhalf * 4 + k8, 64)) = v;
                        }
                    }
                }
            }
            fence_proxy_async_smem();  // P -> the bulk store below
            tc_fence_before_sync();
            __syncthreads();
        }
        // The staging buffers are free: prefetch the next task. K~ and P are final: copy them to
        // the slot in the background. Both are issued from warp 2, idle in the first solve levels.
        if (tid == 64) {
            int qn = qi + (int)gridDim.x;
            if (FUSED) {
                // a CTA that will run a scan leaves the queue once its index reaches switch_at
                qn = ((int)blockIdx.x < p.BH && qi >= p.switch_at) ? ntasks : atomicAdd(p.queue, 1);
                ms.q_next = qn;  // read by every thread after the barriers below
            }
            if (qn < ntasks) issue_loads(task_of(qn));
            bulk_store(slot + SLOT_KT, sm + OFF_KT, 16384);
            bulk_store(slot + SLOT_P, sm + OFF_P, 8192);
            bulk_commit_group();
        }

        // ================= UT solve: T = (I + A)^{-1} =================
        // Doubling from the sixteen 4 x 4 diagonal blocks: a unit lower-triangular block
        // [[X, 0], [Y, Z]] has the inverse [[X^-1, 0], [-Z^-1 (Y X^-1), Z^-1]], so each level
        // forms its lower-left blocks as two small products with the inverses of the level
        // below. A holds zeros on and above the diagonal; levels 4..32 overwrite it in place
        // (warps 0-1), level 64 (warps 0-3) writes T straight into its bf16 K-major copy
        // while warps 4-7 convert the parts of T that are already final.
        {
            // level 4: one thread per diagonal block, by substitution
            if (tid < 16) {
                float *B0 = A32 + (4 * tid) * F_LD + 4 * tid;
                const float4 r1 = *reinterpret_cast<const float4 *>(B0 + F_LD);
                const float4 r2 = *reinterpret_cast<const float4 *>(B0 + 2 * F_LD);
                const float4 r3 = *reinterpret_cast<const float4 *>(B0 + 3 * F_LD);
                const float t10 = -r1.x;
                const float t21 = -r2.y, t20 = -fmaf(r2.y, t10, r2.x);
                const float t32 = -r3.z, t31 = -fmaf(r3.z, t21, r3.y);
                const float t30 = -fmaf(r3.z, t20, fmaf(r3.y, t10, r3.x));
                *reinterpret_cast<float4 *>(B0) = make_float4(1.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4 *>(B0 + F_LD) = make_float4(t10, 1.f, 0.f, 0.f);
                *reinterpret_cast<float4 *>(B0 + 2 * F_LD) = make_float4(t20, t21, 1.f, 0.f);
                *reinterpret_cast<float4 *>(B0 + 3 * F_LD) = make_float4(t30, t31, t32, 1.f);
            }
            __syncwarp();
            // level 8: warp 0, lane = (block h, row r of the lower half); Y rows through shuffles
            if (tid < 32) {
                const int h = tid >> 2, r = tid & 3;
                float *Ar = A32 + (8 * h + 4 + r) * F_LD + 8 * h;  // A_10 row r, then T_1 row r at +4
                const float *T0 = A32 + (8 * h) * F_LD + 8 * h;
                const float4 a = *reinterpret_cast<const float4 *>(Ar);
                const float av[4] = {a.x, a.y, a.z, a.w};
                float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 tv = *reinterpret_cast<const float4 *>(T0 + k * F_LD);
                    y[0] = fmaf(av[k], tv.x, y[0]); y[1] = fmaf(av[k], tv.y, y[1]);
                    y[2] = fmaf(av[k], tv.z, y[2]); y[3] = fmaf(av[k], tv.w, y[3]);
                }
                const float4 t1 = *reinterpret_cast<const float4 *>(Ar + 4);
                const float tv1[4] = {t1.x, t1.y, t1.z, t1.w};
                float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int c = 0; c < 4; ++c) o[c] = fmaf(tv1[u], __shfl_sync(0xffffffffu, y[c], (tid & ~3) | u), o[c]);
                *reinterpret_cast<float4 *>(Ar) = make_float4(-o[0], -o[1], -o[2], -o[3]);
            }
            if (tid < 64) {
                named_barrier(1, 64);  // level 8 (warp 0) -> warp 1
                // level 16: block I = tid / 16, row r of the lower half, column half ch
                {
                    const int I = tid >> 4, r = (tid >> 1) & 7, ch = tid & 1, base = 16 * I;
                    float *Ar = A32 + (base + 8 + r) * F_LD + base;  // A_10 row r (8 wide), T_1 row r at +8
                    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const float4 a = *reinterpret_cast<const float4 *>(Ar + 4 * kk);
                        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float4 tv =
                                *reinterpret_cast<const float4 *>(A32 + (base + 4 * kk + k) * F_LD + base + 4 * ch);
                            y[0] = fmaf(av[k], tv.x, y[0]); y[1] = fmaf(av[k], tv.y, y[1]);
                            y[2] = fmaf(av[k], tv.z, y[2]); y[3] = fmaf(av[k], tv.w, y[3]);
                        }
                    }
                    *reinterpret_cast<float4 *>(Ys + (8 * I + r) * Y_LD + 4 * ch) = make_float4(y[0], y[1], y[2], y[3]);
                    __syncwarp();
                    float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int uu = 0; uu < 2; ++uu) {
                        const float4 t = *reinterpret_cast<const float4 *>(Ar + 8 + 4 * uu);
                        const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float4 yv = *reinterpret_cast<const float4 *>(Ys + (8 * I + 4 * uu + u) * Y_LD + 4 * ch);
                            o[0] = fmaf(tv[u], yv.x, o[0]); o[1] = fmaf(tv[u], yv.y, o[1]);
                            o[2] = fmaf(tv[u], yv.z, o[2]); o[3] = fmaf(tv[u], yv.w, o[3]);
                        }
                    }
                    *reinterpret_cast<float4 *>(Ar + 4 * ch) = make_float4(-o[0], -o[1], -o[2], -o[3]);
                }
                __syncwarp();
                // level 32: block b = warp (its two 16-blocks came from this warp), two rows x four columns
                {
                    const int b = tid >> 5, rp = lane >> 2, cg = lane & 3, base = 32 * b;
                    float *A0 = A32 + (base + 16 + 2 * rp) * F_LD + base;  // A_10 rows 2rp, 2rp+1; T_1 at +16
                    float *A1 = A0 + F_LD;
                    float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const float4 a0 = *reinterpret_cast<const float4 *>(A0 + 4 * kk);
                        const float4 a1 = *reinterpret_cast<const float4 *>(A1 + 4 * kk);
                        const float av0[4] = {a0.x, a0.y, a0.z, a0.w}, av1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float4 tv =
                                *reinterpret_cast<const float4 *>(A32 + (base + 4 * kk + k) * F_LD + base + 4 * cg);
                            y0[0] = fmaf(av0[k], tv.x, y0[0]); y0[1] = fmaf(av0[k], tv.y, y0[1]);
                            y0[2] = fmaf(av0[k], tv.z, y0[2]); y0[3] = fmaf(av0[k], tv.w, y0[3]);
                            y1[0] = fmaf(av1[k], tv.x, y1[0]); y1[1] = fmaf(av1[k], tv.y, y1[1]);
                            y1[2] = fmaf(av1[k], tv.z, y1[2]); y1[3] = fmaf(av1[k], tv.w, y1[3]);
                        }
                    }
                    float *Yb = Ys + (16 * b) * Y_LD;
                    *reinterpret_cast<float4 *>(Yb + (2 * rp) * Y_LD + 4 * cg) = make_float4(y0[0], y0[1], y0[2], y0[3]);
                    *reinterpret_cast<float4 *>(Yb + (2 * rp + 1) * Y_LD + 4 * cg) =
                        make_float4(y1[0], y1[1], y1[2], y1[3]);
                    __syncwarp();
                    float o0[4] = {0.f, 0.f, 0.f, 0.f}, o1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int uu = 0; uu < 4; ++uu) {
                        const float4 t0 = *reinterpret_cast<const float4 *>(A0 + 16 + 4 * uu);
                        const float4 t1 = *reinterpret_cast<const float4 *>(A1 + 16 + 4 * uu);
                        const float tv0[4] = {t0.x, t0.y, t0.z, t0.w}, tv1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float4 yv = *reinterpret_cast<const float4 *>(Yb + (4 * uu + u) * Y_LD + 4 * cg);
                            o0[0] = fmaf(tv0[u], yv.x, o0[0]); o0[1] = fmaf(tv0[u], yv.y, o0[1]);
                            o0[2] = fmaf(tv0[u], yv.z, o0[2]); o0[3] = fmaf(tv0[u], yv.w, o0[3]);
                            o1[0] = fmaf(tv1[u], yv.x, o1[0]); o1[1] = fmaf(tv1[u], yv.y, o1[1]);
                            o1[2] = fmaf(tv1[u], yv.z, o1[2]); o1[3] = fmaf(tv1[u], yv.w, o1[3]);
                        }
                    }
                    *reinterpret_cast<float4 *>(A0 + 4 * cg) = make_float4(-o0[0], -o0[1], -o0[2], -o0[3]);
                    *reinterpret_cast<float4 *>(A1 + 4 * cg) = make_float4(-o1[0], -o1[1], -o1[2], -o1[3]);
                }
            }
            __syncthreads();
            // level 64: rows 32 + 2rp, +1 and columns 4cg .. 4cg+3 of T_10 = -T_1 (A_10 T_0)
            const int rp = tid >> 3, cg = tid & 7;
            const float *A0 = A32 + (32 + 2 * rp) * F_LD;  // A_10 row (32 wide), T_1 row at +32
            const float *A1 = A0 + F_LD;
            if (tid < 128) {
                float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
                for (int kk = 0; kk < 8; ++kk) {
                    const float4 a0 = *reinterpret_cast<const float4 *>(A0 + 4 * kk);
                    const float4 a1 = *reinterpret_cast<const float4 *>(A1 + 4 * kk);
                    const float av0[4] = {a0.x, a0.y, a0.z, a0.w}, av1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float4 tv = *reinterpret_cast<const float4 *>(A32 + (4 * kk + k) * F_LD + 4 * cg);
                        y0[0] = fmaf(av0[k], tv.x, y0[0]); y0[1] = fmaf(av0[k], tv.y, y0[1]);
                        y0[2] = fmaf(av0[k], tv.z, y0[2]); y0[3] = fmaf(av0[k], tv.w, y0[3]);
                        y1[0] = fmaf(av1[k], tv.x, y1[0]); y1[1] = fmaf(av1[k], tv.y, y1[1]);
                        y1[2] = fmaf(av1[k], tv.z, y1[2]); y1[3] = fmaf(av1[k], tv.w, y1[3]);
                    }
                }
                *reinterpret_cast<float4 *>(Ys + (2 * rp) * Y_LD + 4 * cg) = make_float4(y0[0], y0[1], y0[2], y0[3]);
                *reinterpret_cast<float4 *>(Ys + (2 * rp + 1) * Y_LD + 4 * cg) = make_float4(y1[0], y1[1], y1[2], y1[3]);
            }
            __syncthreads();
            // T in bf16, K-major [t][64 s] over the front of the fp32 array: every read of
            // the array below precedes the barrier, every write follows it
            float o0[4] = {0.f, 0.f, 0.f, 0.f}, o1[4] = {0.f, 0.f, 0.f, 0.f};
            float lo[8], hi[8];
            const int ct = (tid - 128) >> 2, c8 = tid & 3;  // converter: row, 8-column chunk
            if (tid < 128) {
#pragma unroll 2
                for (int uu = 0; uu < 8; ++uu) {
                    const float4 t0 = *reinterpret_cast<const float4 *>(A0 + 32 + 4 * uu);
                    const float4 t1 = *reinterpret_cast<const float4 *>(A1 + 32 + 4 * uu);
                    const float tv0[4] = {t0.x, t0.y, t0.z, t0.w}, tv1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4 yv = *reinterpret_cast<const float4 *>(Ys + (4 * uu + u) * Y_LD + 4 * cg);
                        o0[0] = fmaf(tv0[u], yv.x, o0[0]); o0[1] = fmaf(tv0[u], yv.y, o0[1]);
                        o0[2] = fmaf(tv0[u], yv.z, o0[2]); o0[3] = fmaf(tv0[u], yv.w, o0[3]);
                        o1[0] = fmaf(tv1[u], yv.x, o1[0]); o1[1] = fmaf(tv1[u], yv.y, o1[1]);
                        o1[2] = fmaf(tv1[u], yv.z, o1[2]); o1[3] = fmaf(tv1[u], yv.w, o1[3]);
                    }
                }
            } else {
                // T rows 0..31 (columns 0..31; 32..63 are zero) and T_1 (rows and columns 32..63)
                load8f(A32 + ct * F_LD + 8 * c8, lo);
                load8f(A32 + (32 + ct) * F_LD + 32 + 8 * c8, hi);
            }
            __syncthreads();
            if (tid < 128) {
                __nv_bfloat162 h0 = __floats2bfloat162_rn(-o0[0], -o0[1]), h1 = __floats2bfloat162_rn(-o0[2], -o0[3]);
                uint2 u0;
                u0.x = *reinterpret_cast<uint32_t *>(&h0);
                u0.y = *reinterpret_cast<uint32_t *>(&h1);
                h0 = __floats2bfloat162_rn(-o1[0], -o1[1]);
                h1 = __floats2bfloat162_rn(-o1[2], -o1[3]);
                uint2 u1;
                u1.x = *reinterpret_cast<uint32_t *>(&h0);
                u1.y = *reinterpret_cast<uint32_t *>(&h1);
                *reinterpret_cast<uint2 *>(sm + OFF_TB + sw_chunk(32 + 2 * rp, cg >> 1, 64) + (cg & 1) * 8) = u0;
                *reinterpret_cast<uint2 *>(sm + OFF_TB + sw_chunk(32 + 2 * rp + 1, cg >> 1, 64) + (cg & 1) * 8) = u1;
            } else {
                const float zz[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                *reinterpret_cast<uint4 *>(sm + OFF_TB + sw_chunk(ct, c8, 64)) = pack8(lo);
                *reinterpret_cast<uint4 *>(sm + OFF_TB + sw_chunk(ct, 4 + c8, 64)) = pack8(zz);
                *reinterpret_cast<uint4 *>(sm + OFF_TB + sw_chunk(32 + ct, 4 + c8, 64)) = pack8(hi);
            }
        }
        mma_sync_point();
        // ================= W^T_I = (L^e_I)^T T[:,I]^T ;  U~^T = Z^T T^T =================
        if (tid == 0) {
            const uint32_t idW = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int I = 0; I < 2; ++I)
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const uint64_t ad = sdesc_sw128(sbase + OFF_STACK + (64 * I + 16 * ks) * 128, 16384, 1024);
                    const uint64_t bd = sdesc_sw128(sbase + OFF_TB + (32 * I + 16 * ks) * 2, 16, 1024);
                    mma_bf16(tm + (I ? CK_W1 : CK_W0), ad, bd, idW, ks > 0);
                }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc_sw128(sbase + OFF_Z + ks * 2048, 8192, 1024);
                const uint64_t bd = sdesc_sw128(sbase + OFF_TB + ks * 32, 16, 1024);
                mma_bf16(tm + CK_U, ad, bd, idW, ks > 0);
            }
            mma_commit(&ms.bar_mma);
        }
        if (!wait_bar(&ms.bar_mma, ph_mma)) { timed_out = true; break; }
        tc_fence_after_sync();

        // ================= W -> [c][64 t] over STACK;  U~^T -> [j][64 t] over Z (for the slot) =================
        {
            const float e0 = ms.eg0[row], e1 = ms.eg1[row];
            float w0[32], w1[32];
            tmem_ld32x2(tm_lane + CK_W0 + colhalf * 32, tm_lane + CK_W1 + colhalf * 32, w0, w1);
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                float f[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) f[x] = e0 * w0[k8 * 8 + x] + e1 * w1[k8 * 8 + x];
                *reinterpret_cast<uint4 *>(sm + OFF_STACK + sw_chunk(row, colhalf * 4 + k8, 128)) = pack8(f);
            }
            float u[32];
            tmem_ld32(tm_lane + CK_U + colhalf * 32, u);
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                float f[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) f[x] = u[k8 * 8 + x];
                *reinterpret_cast<uint4 *>(sm + OFF_Z + sw_chunk(row, colhalf * 4 + k8, 128)) = pack8(f);
            }
        }
        mma_sync_point();
        // U~^T is staged: to the slot in the background (from warp 2, which has nothing to issue)
        if (tid == 64) {
            bulk_store(slot + SLOT_U, sm + OFF_Z, 16384);
            if (BWD) {
                unsigned char *ext = p.ext + (size_t)task * EXT_BYTES;
                bulk_store(ext + EXT_T, sm + OFF_TB, 8192);
                bulk_store(ext + EXT_W, sm + OFF_STACK, 16384);
            }
            bulk_commit_group();
        }
        // ================= Q' - Q^ = -P W (M = 64) ;  M = -K~^T W =================
        if (tid == 0) {
            const uint32_t idQ = idesc_bf16(64, 128, false, false, true);
            const uint32_t idM = idesc_bf16(128, 128, true, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t aw = sdesc_sw128(sbase + OFF_STACK + ks * 32, 16, 1024);  // W as [c][64 s]
                const uint64_t ap = sdesc_sw128(sbase + OFF_P + ks * 32, 16, 1024);      // P as [t][64 s]
                mma_bf16(tm + CK_Q, ap, aw, idQ, ks > 0);
                const uint64_t ak = sdesc_sw128(sbase + OFF_KT + ks * 2048, 8192, 1024);
                mma_bf16(tm + CK_M, ak, aw, idM, ks > 0);
            }
            mma_commit(&ms.bar_mma);
        }
        if (BWD && tid == 64) bulk_wait_group_read0();  // T and W have left STACK and R
        if (!wait_bar(&ms.bar_mma, ph_mma)) { timed_out = true; break; }
        tc_fence_after_sync();
        // ================= [Q'; M] -> [c' block][192 rows][64 c'] over STACK and R (for the slot) =================
        {
            // M: lane c, columns c' of this thread's half -> rows 64 + c
            float m0[32], m1[32];
            tmem_ld32x2(tm_lane + CK_M + colhalf * 64, tm_lane + CK_M + colhalf * 64 + 32, m0, m1);
#pragma unroll
            for (int k8 = 0; k8 < 8; ++k8) {
                float f[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) f[x] = k8 < 4 ? m0[k8 * 8 + x] : m1[(k8 - 4) * 8 + x];
                *reinterpret_cast<uint4 *>(sm + OFF_STACK + sw_chunk(64 + row, colhalf * 8 + k8, B1_ROWS)) = pack8(f);
            }
            // Q': the M = 64 accumulator holds row t in lane t % 16 of warp quarter t / 16
            float d0[32], d1[32];
            tmem_ld32x2(tm_lane + CK_Q + colhalf * 64, tm_lane + CK_Q + colhalf * 64 + 32, d0, d1);
            if (lane < 16) {
                const int t = quarter * 16 + lane;
#pragma unroll
                for (int k8 = 0; k8 < 8; ++k8) {
                    float f[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_QH + sw_chunk(t, colhalf * 8 + k8, 64)), f);
#pragma unroll
                    for (int x = 0; x < 8; ++x) f[x] += k8 < 4 ? d0[k8 * 8 + x] : d1[(k8 - 4) * 8 + x];
                    *reinterpret_cast<uint4 *>(sm + OFF_STACK + sw_chunk(t, colhalf * 8 + k8, B1_ROWS)) = pack8(f);
                }
            }
        }
        if (tid < DK) reinterpret_cast<float *>(p.ws + (size_t)p.ntasks * SLOT_BYTES + (size_t)task * GAMMA_BYTES)[tid] =
            ms.gC[tid];
        fence_proxy_async_smem();  // [Q'; M] -> the bulk store below
        tc_fence_before_sync();
        __syncthreads();  // every TMEM read of this task is done before the next task's MMAs
        if (tid == 0) {
            bulk_store(slot + SLOT_B1, sm + OFF_STACK, 2 * B1_ROWS * 128);
            bulk_commit_group();
        }
        prev_task = task;
        qi = FUSED ? ms.q_next : qi + (int)gridDim.x;
    }
    if (tid == 0 || tid == 64) {
        bulk_wait_group0();  // each waits for the bulk groups it committed
        if (FUSED) fence_proxy_async_global();
    }
    if (FUSED) {
        __syncthreads();
        if (!timed_out && tid == 0 && prev_task >= 0) {
            __threadfence();
            st_release_gpu(p.flags + prev_task, 1u);
        }
    }
    if (timed_out && tid == 0) atomicOr(p.status, kStatusTimeout);
    tc_fence_before_sync();
    __syncthreads();
    if (!FUSED && warp == 0) tmem_dealloc(tm, TM_COLS);
    tm_out = tm;
    return timed_out;
}

template <bool GENERAL, bool BWD = false>
__global__ void __launch_bounds__(NT, 1)
fwd_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_la,
                 ChunkParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t tm;
    chunk_body<GENERAL, BWD, false>(tm_q, tm_k, tm_b, tm_v, tm_w, tm_la, p, sm, tm);
}

// ---- scan kernel ----
// One CTA per (b, h). TMEM holds S^T (lane j, column c) in fp32 in one of two
// regions that alternate per chunk, each laid out [O^T (64 t) | S^T (128 c)] so
// that one N = 192 product writes a chunk's output and state together; the
// bf16 copy of S^T that those products read as their A operand sits in TMEM
// too. O^T of chunk n is stored while chunk n + 1 runs in the other region.
constexpr uint32_t SC_SLOT0 = 0;
constexpr uint32_t SC_SLOT1 = SLOT_BYTES;          // 90112, 1024-aligned
constexpr uint32_t SC_O = 2 * SLOT_BYTES;          // O tile [64 t][128 j] bf16
constexpr uint32_t SC_MISC = SC_O + 16384;
constexpr int SC_NT = NT + 32;  // 8 warps on the TMEM lanes + warp 8, which issues the MMAs
constexpr uint32_t SC_REG = 256;                    // region r at columns 256 r: O^T then S^T
constexpr uint32_t SC_OT = 0, SC_ST = 64;           // offsets within a region
constexpr uint32_t SC_SA = 448;                     // S^T in bf16, two values per column (64 columns)
constexpr uint32_t SC_COLS = 512;

struct ScanMisc {
    uint64_t bar_full[2];
    uint64_t bar_mma;
    uint32_t tmem_base;
    alignas(16) float gam[2][DK];  // bulk-copy destination and float4 reads: 16-byte aligned
};
static_assert(sizeof(ScanMisc) <= 1280, "scan misc region");
static_assert(offsetof(ScanMisc, gam) % 16 == 0, "gamma rows are 16-byte aligned");

struct ScanParams {
    int B, T, H, NC, ntasks;
    const unsigned char *ws;
    const float *S0;
    float *S_T;
    float *saved_states;
    unsigned *status;
    const int *cu_seqlens;  // packed sequences (null when dense), as in ChunkParams
    const int *cu_chunks;
    __nv_bfloat16 *o;       // for the row-by-row store of a packed sequence's last, partial tile
    const int *seq_order = nullptr;  // packed: CTA group g (H CTAs) scans sequence seq_order[g]
};

constexpr uint32_t SC_SMEM = SC_MISC + 1280 + 1024;  // + alignment slack

__global__ void __launch_bounds__(SC_NT, 1)  // 168 registers: allocation rounds 9 warps up to 12
fwd_scan_kernel(const __grid_constant__ CUtensorMap tm_o, ScanParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    ScanMisc &ms = *reinterpret_cast<ScanMisc *>(sm + SC_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, colhalf = warp >> 2;
    int bh = blockIdx.x;  // (sequence, head)
    int bb = bh / p.H;
    const int h = bh % p.H;
    const int c0 = colhalf * 64;  // this thread's 64 state columns c (S^T columns)
    // this (sequence, head)'s chunks: count, first task, first token and length, map batch
    int NC = p.NC, tstart = 0, len = p.T, tb = bb;
    size_t base = (size_t)bh * p.NC;

    if (tid == 0) {
        mbar_init(&ms.bar_full[0], 1);
        mbar_init(&ms.bar_full[1], 1);
        mbar_init(&ms.bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&ms.tmem_base, SC_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tm = ms.tmem_base;
    const uint32_t tm_lane = tm + ((uint32_t)(quarter * 32) << 16);
    const int j = quarter * 32 + lane;  // this thread's TMEM lane = value channel

    // Launched as a programmatic dependent of the chunk kernel: everything above overlaps its
    // tail; the workspace is read only after that grid has completed and flushed its memory.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (p.cu_seqlens) {
        bb = p.seq_order[bb];  // the longest sequences first
        bh = bb * p.H + h;
        NC = p.cu_chunks[bb + 1] - p.cu_chunks[bb];
        base = (size_t)p.H * p.cu_chunks[bb] + (size_t)h * NC;
        tstart = p.cu_seqlens[bb];
        len = p.cu_seqlens[bb + 1] - tstart;
        tb = 0;
    }

    auto issue_slot = [&](int n) {
        const int sl = n & 1;
        const size_t task = base + n;
        mbar_arrive_expect_tx(&ms.bar_full[sl], SLOT_BYTES + GAMMA_BYTES);
        bulk_load(sm + (sl ? SC_SLOT1 : SC_SLOT0), p.ws + task * SLOT_BYTES, SLOT_BYTES, &ms.bar_full[sl]);
        bulk_load(ms.gam[sl], p.ws + (size_t)p.ntasks * SLOT_BYTES + task * GAMMA_BYTES, GAMMA_BYTES,
                  &ms.bar_full[sl]);
    };
    if (tid == 0) {
        if (NC > 0) issue_slot(0);
        if (NC > 1) issue_slot(1);
    }
    // initial state S^T[j][c] = S0[c][j] into region 1 (chunk 0 reads the region of "chunk -1")
    if (warp < 8) {
        float v[32];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[i] = p.S0 ? p.S0[((size_t)bh * DK + c0 + q2 * 32 + i) * DV + j] : 0.f;
            tmem_st32(tm_lane + SC_REG + SC_ST + c0 + q2 * 32, v);
        }
        float zz[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) zz[i] = 0.f;
        tmem_st32(tm_lane + SC_OT + colhalf * 32, zz);  // chunk 0's O^T starts at zero
    }
    tc_fence_before_sync();
    __syncthreads();

    uint32_t ph_full[2] = {0, 0}, ph_mma = 0;
    bool timed_out = false;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) -> bool {
        const bool ok = mbar_wait_bounded(bar, ph, kWaitLimitNs);
        ph ^= 1u;
        return __syncthreads_or(!ok) == 0;
    };

    // O^T of chunk m -> bf16 tile [t][j] -> one TMA store (rows past T are
    // clipped). Warps 0-7 under named barrier 1, while warp 8 keeps the tensor core busy with
    // the next chunk: warp quarter q reads TMEM lanes (value channels) j = 32 q + lane, warp
    // group colhalf the tokens t = 32 colhalf .. 32 colhalf + 31.
    auto store_o = [&](int m) {
        if (tid == 0) bulk_wait_group_read0();  // the previous tile has left shared memory
        named_barrier(1, 256);
        const int t0 = colhalf * 32;
        float o0[32];
        tmem_ld32(tm_lane + SC_REG * (m & 1) + SC_OT + t0, o0);
        __nv_bfloat16 *ot = reinterpret_cast<__nv_bfloat16 *>(sm + SC_O);
#pragma unroll
        for (int i = 0; i < 32; ++i) ot[(t0 + i) * DV + j] = __float2bfloat16_rn(o0[i]);
        fence_proxy_async_smem();
        tc_fence_before_sync();
        named_barrier(1, 256);
        const int rows = min(C, len - m * C);
        if (p.cu_seqlens && rows < C) {
            // a packed sequence's partial last tile: its rows only (a tile store would write
            // into the next sequence)
            for (int i = tid; i < rows * 16; i += 256) {
                const int r = i >> 4, c16 = i & 15;
                *reinterpret_cast<uint4 *>(p.o + ((size_t)(tstart + m * C + r) * p.H + h) * DV + c16 * 8) =
                    *reinterpret_cast<const uint4 *>(ot + r * DV + c16 * 8);
            }
        } else if (tid == 0) {
            tma_store_4d(&tm_o, sm + SC_O, 0, h, tstart + m * C, tb);
            bulk_commit_group();
        }
    };

    if (NC > 0 && !wait_bar(&ms.bar_full[0], ph_full[0])) timed_out = true;
    for (int n = 0; n < NC && !timed_out; ++n) {
        const int sl = n & 1;
        const uint32_t slot = sbase + (sl ? SC_SLOT1 : SC_SLOT0);
        const uint32_t rg = SC_REG * (uint32_t)sl, rg_prev = SC_REG * (uint32_t)(sl ^ 1);
        // ---- S^T (previous region) -> bf16 operand; gamma-scaled S^T -> this region ----
        if (warp < 8) {
            float s0[32], s1[32];
            tmem_ld32x2(tm_lane + rg_prev + SC_ST + c0, tm_lane + rg_prev + SC_ST + c0 + 32, s0, s1);
            if (p.saved_states) {
                float *dst = p.saved_states + ((base + n) * DK + c0) * DV + j;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    dst[(size_t)i * DV] = s0[i];
                    dst[(size_t)(32 + i) * DV] = s1[i];
                }
            }
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __nv_bfloat162 h0 = __floats2bfloat162_rn(s0[2 * i], s0[2 * i + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(s1[2 * i], s1[2 * i + 1]);
                pk[i] = *reinterpret_cast<uint32_t *>(&h0);
                pk[16 + i] = *reinterpret_cast<uint32_t *>(&h1);
            }
            tmem_st32u_nw(tm_lane + SC_SA + (uint32_t)(c0 >> 1), pk);
            const float4 *g4 = reinterpret_cast<const float4 *>(&ms.gam[sl][c0]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 ga = g4[i], gb = g4[8 + i];
                s0[4 * i] *= ga.x; s0[4 * i + 1] *= ga.y; s0[4 * i + 2] *= ga.z; s0[4 * i + 3] *= ga.w;
                s1[4 * i] *= gb.x; s1[4 * i + 1] *= gb.y; s1[4 * i + 2] *= gb.z; s1[4 * i + 3] *= gb.w;
            }
            tmem_st32_nw(tm_lane + rg + SC_ST + c0, s0);
            tmem_st32_nw(tm_lane + rg + SC_ST + c0 + 32, s1);
            tmem_wait_st();
        }
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        // ---- [O^T | S^T] += S_bf16^T [Q'; M]^T ;  S^T += U~^T K~ ;  O^T += U~^T P^T ----
        if (warp == 8 && lane == 0) {
            const uint32_t id1 = idesc_bf16(128, B1_ROWS, false, false);
            const uint32_t idS = idesc_bf16(128, 128, false, true);
            const uint32_t idO = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t b1 =
                    sdesc_sw128(slot + SLOT_B1 + (ks >> 2) * (B1_ROWS * 128) + (ks & 3) * 32, 16, 1024);
                mma_bf16_ts(tm + rg + SC_OT, tm + SC_SA + ks * 8, b1, id1, 1);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t au = sdesc_sw128(slot + SLOT_U + ks * 32, 16, 1024);
                const uint64_t bk = sdesc_sw128(slot + SLOT_KT + ks * 2048, 8192, 1024);
                mma_bf16(tm + rg + SC_ST, au, bk, idS, 1);
                const uint64_t bp = sdesc_sw128(slot + SLOT_P + ks * 32, 16, 1024);
                mma_bf16(tm + rg + SC_OT, au, bp, idO, 1);
            }
            mma_commit(&ms.bar_mma);
        }
        if (warp < 8) {
            // overlaps this chunk's MMAs (the other region), then clears that region's O^T
            // for chunk n + 1 (each thread rewrites only the lane and columns it has just read)
            if (n > 0) store_o(n - 1);
            float zz[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) zz[i] = 0.f;
            tmem_st32_nw(tm_lane + rg_prev + SC_OT + colhalf * 32, zz);
            tmem_wait_st();
        }
        // the next slot (issued two chunks ago) and this chunk's MMAs, one barrier for both
        {
            bool ok = true;
            if (n + 1 < NC) {
                ok = mbar_wait_bounded(&ms.bar_full[sl ^ 1], ph_full[sl ^ 1], kWaitLimitNs);
                ph_full[sl ^ 1] ^= 1u;
            }
            ok = mbar_wait_bounded(&ms.bar_mma, ph_mma, kWaitLimitNs) && ok;
            ph_mma ^= 1u;
            tc_fence_before_sync();
            if (__syncthreads_or(!ok)) { timed_out = true; break; }
            tc_fence_after_sync();
        }
        if (tid == 0 && n + 2 < NC) issue_slot(n + 2);  // this slot's MMAs are done
    }
    if (!timed_out && NC > 0 && warp < 8) store_o(NC - 1);
    if (!timed_out && p.S_T && warp < 8) {
        const uint32_t rg_last = SC_REG * (uint32_t)((NC + 1) & 1);  // region of chunk NC - 1 (region 1 if NC = 0)
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            const int cb = c0 + q2 * 32;
            float sv[32];
            tmem_ld32(tm_lane + rg_last + SC_ST + cb, sv);
            float *dst = p.S_T + ((size_t)bh * DK + cb) * DV + j;
#pragma unroll
            for (int i = 0; i < 32; ++i) dst[(size_t)i * DV] = sv[i];
        }
    }
    if (tid == 0) bulk_wait_group0();
    if (timed_out && tid == 0) atomicOr(p.status, kStatusTimeout);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, SC_COLS);
}

// ---- fused kernel: chunk tasks, then (CTA b < B H) the scan of (sequence, head) b ----
// One cooperative launch of one CTA per SM, so every CTA is resident and a scan that waits for
// a chunk task only waits for CTAs that are running and never wait themselves. All CTAs first
// take chunk tasks from a queue in chunk-major order; CTA b < B H leaves the queue near its
// end (switch_at) and runs the scan of (sequence, head) b, whose first chunks are long done,
// while the other CTAs finish the queue. The scan copies a slot only after its task's flag is
// set. The scan's steps are those of fwd_scan_kernel, on eight warps: thread 0 issues the
// products and the slot copies.
__device__ __forceinline__ void fused_scan(const CUtensorMap &tm_o, const ScanParams &p, const unsigned *flags,
                                           unsigned char *sm, uint32_t tm, int bh, bool &timed_out)
{
    ScanMisc &ms = *reinterpret_cast<ScanMisc *>(sm + SC_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, colhalf = warp >> 2;
    const int bb = bh / p.H, h = bh % p.H;
    const int c0 = colhalf * 64;  // this thread's 64 state columns c (S^T columns)
    const int NC = p.NC;
    const size_t base = (size_t)bh * p.NC;
    const uint32_t tm_lane = tm + ((uint32_t)(quarter * 32) << 16);
    const int j = quarter * 32 + lane;  // this thread's TMEM lane = value channel

    if (tid == 0) {
        mbar_init(&ms.bar_full[0], 1);
        mbar_init(&ms.bar_full[1], 1);
        mbar_init(&ms.bar_mma, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // thread 0: a task's slot is copied once its flag is set; if a flag never comes, the copy is
    // not issued and the wait for it below gives up as well
    auto issue_slot = [&](int n) {
        const int sl = n & 1;
        const size_t task = base + n;
        if (!flag_wait_bounded(flags + task, kWaitLimitNs)) return;
        fence_proxy_async_global();
        mbar_arrive_expect_tx(&ms.bar_full[sl], SLOT_BYTES + GAMMA_BYTES);
        bulk_load(sm + (sl ? SC_SLOT1 : SC_SLOT0), p.ws + task * SLOT_BYTES, SLOT_BYTES, &ms.bar_full[sl]);
        bulk_load(ms.gam[sl], p.ws + (size_t)p.ntasks * SLOT_BYTES + task * GAMMA_BYTES, GAMMA_BYTES,
                  &ms.bar_full[sl]);
    };
    if (tid == 0) {
        if (NC > 0) issue_slot(0);
        if (NC > 1) issue_slot(1);
    }
    // initial state S^T[j][c] = S0[c][j] into region 1 (chunk 0 reads the region of "chunk -1")
    {
        float v[32];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[i] = p.S0 ? p.S0[((size_t)bh * DK + c0 + q2 * 32 + i) * DV + j] : 0.f;
            tmem_st32(tm_lane + SC_REG + SC_ST + c0 + q2 * 32, v);
        }
        float zz[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) zz[i] = 0.f;
        tmem_st32(tm_lane + SC_OT + colhalf * 32, zz);  // chunk 0's O^T starts at zero
    }
    tc_fence_before_sync();
    __syncthreads();

    uint32_t ph_full = 0, ph_mma = 0;  // bit s: phase of bar_full[s]
    auto store_o = [&](int m) {  // as in fwd_scan_kernel: O^T of chunk m -> bf16 tile -> TMA store
        if (tid == 0) bulk_wait_group_read0();
        named_barrier(1, NT);
        const int t0 = colhalf * 32;
        float o0[32];
        tmem_ld32(tm_lane + SC_REG * (m & 1) + SC_OT + t0, o0);
        __nv_bfloat16 *ot = reinterpret_cast<__nv_bfloat16 *>(sm + SC_O);
#pragma unroll
        for (int i = 0; i < 32; ++i) ot[(t0 + i) * DV + j] = __float2bfloat16_rn(o0[i]);
        fence_proxy_async_smem();
        tc_fence_before_sync();
        named_barrier(1, NT);
        if (tid == 0) {
            tma_store_4d(&tm_o, sm + SC_O, 0, h, m * C, bb);
            bulk_commit_group();
        }
    };

    if (NC > 0) {
        const bool ok = mbar_wait_bounded(&ms.bar_full[0], 0, kWaitLimitNs);
        ph_full ^= 1u;
        if (__syncthreads_or(!ok)) timed_out = true;
    }
    for (int n = 0; n < NC && !timed_out; ++n) {
        const int sl = n & 1;
        const uint32_t slot = sbase + (sl ? SC_SLOT1 : SC_SLOT0);
        const uint32_t rg = SC_REG * (uint32_t)sl, rg_prev = SC_REG * (uint32_t)(sl ^ 1);
        // ---- S^T (previous region) -> bf16 operand; gamma-scaled S^T -> this region ----
        {
            float s0[32], s1[32];
            tmem_ld32x2(tm_lane + rg_prev + SC_ST + c0, tm_lane + rg_prev + SC_ST + c0 + 32, s0, s1);
            if (p.saved_states) {  // the state entering chunk n, for the backward
                float *dst = p.saved_states + ((base + n) * DK + c0) * DV + j;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    dst[(size_t)i * DV] = s0[i];
                    dst[(size_t)(32 + i) * DV] = s1[i];
                }
            }
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __nv_bfloat162 h0 = __floats2bfloat162_rn(s0[2 * i], s0[2 * i + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(s1[2 * i], s1[2 * i + 1]);
                pk[i] = *reinterpret_cast<uint32_t *>(&h0);
                pk[16 + i] = *reinterpret_cast<uint32_t *>(&h1);
            }
            tmem_st32u_nw(tm_lane + SC_SA + (uint32_t)(c0 >> 1), pk);
            const float4 *g4 = reinterpret_cast<const float4 *>(&ms.gam[sl][c0]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 ga = g4[i], gb = g4[8 + i];
                s0[4 * i] *= ga.x; s0[4 * i + 1] *= ga.y; s0[4 * i + 2] *= ga.z; s0[4 * i + 3] *= ga.w;
                s1[4 * i] *= gb.x; s1[4 * i + 1] *= gb.y; s1[4 * i + 2] *= gb.z; s1[4 * i + 3] *= gb.w;
            }
            tmem_st32_nw(tm_lane + rg + SC_ST + c0, s0);
            tmem_st32_nw(tm_lane + rg + SC_ST + c0 + 32, s1);
            tmem_wait_st();
        }
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
        // ---- [O^T | S^T] += S_bf16^T [Q'; M]^T ;  S^T += U~^T K~ ;  O^T += U~^T P^T ----
        if (tid == 0) {
            const uint32_t id1 = idesc_bf16(128, B1_ROWS, false, false);
            const uint32_t idS = idesc_bf16(128, 128, false, true);
            const uint32_t idO = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t b1 =
                    sdesc_sw128(slot + SLOT_B1 + (ks >> 2) * (B1_ROWS * 128) + (ks & 3) * 32, 16, 1024);
                mma_bf16_ts(tm + rg + SC_OT, tm + SC_SA + ks * 8, b1, id1, 1);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t au = sdesc_sw128(slot + SLOT_U + ks * 32, 16, 1024);
                const uint64_t bk = sdesc_sw128(slot + SLOT_KT + ks * 2048, 8192, 1024);
                mma_bf16(tm + rg + SC_ST, au, bk, idS, 1);
                const uint64_t bp = sdesc_sw128(slot + SLOT_P + ks * 32, 16, 1024);
                mma_bf16(tm + rg + SC_OT, au, bp, idO, 1);
            }
            mma_commit(&ms.bar_mma);
        }
        // overlaps this chunk's MMAs (the other region), then clears that region's O^T for
        // chunk n + 1 (each thread rewrites only the lane and columns it has just read)
        if (n > 0) store_o(n - 1);
        {
            float zz[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) zz[i] = 0.f;
            tmem_st32_nw(tm_lane + rg_prev + SC_OT + colhalf * 32, zz);
            tmem_wait_st();
        }
        // the next slot and this chunk's MMAs, one barrier for both
        {
            bool ok = true;
            if (n + 1 < NC) {
                ok = mbar_wait_bounded(&ms.bar_full[sl ^ 1], (ph_full >> (sl ^ 1)) & 1u, kWaitLimitNs);
                ph_full ^= 1u << (sl ^ 1);
            }
            ok = mbar_wait_bounded(&ms.bar_mma, ph_mma, kWaitLimitNs) && ok;
            ph_mma ^= 1u;
            tc_fence_before_sync();
            if (__syncthreads_or(!ok)) { timed_out = true; break; }
            tc_fence_after_sync();
        }
        if (tid == 0 && n + 2 < NC) issue_slot(n + 2);  // this slot's MMAs are done
    }
    if (!timed_out && NC > 0) store_o(NC - 1);
    if (!timed_out && p.S_T) {
        const uint32_t rg_last = SC_REG * (uint32_t)((NC + 1) & 1);  // region of chunk NC - 1 (region 1 if NC = 0)
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            const int cb = c0 + q2 * 32;
            float sv[32];
            tmem_ld32(tm_lane + rg_last + SC_ST + cb, sv);
            float *dst = p.S_T + ((size_t)bh * DK + cb) * DV + j;
#pragma unroll
            for (int i = 0; i < 32; ++i) dst[(size_t)i * DV] = sv[i];
        }
    }
    if (tid == 0) bulk_wait_group0();
    if (timed_out && tid == 0) atomicOr(p.status, kStatusTimeout);
}

template <bool GENERAL, bool BWD>
__global__ void __launch_bounds__(NT, 1)
fwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_la,
                 const __grid_constant__ CUtensorMap tm_o, ChunkParams cp, ScanParams sp)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t tm = 0;
    bool timed_out = chunk_body<GENERAL, BWD, true>(tm_q, tm_k, tm_b, tm_v, tm_w, tm_la, cp, sm, tm);
    if (!timed_out && (int)blockIdx.x < cp.BH) fused_scan(tm_o, sp, cp.flags, sm, tm, blockIdx.x, timed_out);
    tc_fence_before_sync();
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(tm, TM_COLS);
}

// ---- the backward's front as one launch: the forward's chunk tasks (backward instance) from
// the last chunk back, then (CTA b < B H) the reverse scan of (sequence, head) b, each chunk's
// slot copied once its flag is set. The same residency argument as fwd_fused_kernel.
template <bool GENERAL>
__global__ void __launch_bounds__(NT, 1)
bwd_front_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_la,
                 const __grid_constant__ CUtensorMap tm_do, ChunkParams cp, RsParams rp)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t tm = 0;
    bool timed_out = chunk_body<GENERAL, true, true, true>(tm_q, tm_k, tm_b, tm_v, tm_w, tm_la, cp, sm, tm);
    if (!timed_out && (int)blockIdx.x < cp.BH) rscan_role(tm_do, rp, cp.flags, sm, tm, blockIdx.x, timed_out);
    tc_fence_before_sync();
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(tm, TM_COLS);
}

// ---------------------------------------------------------------- host side
}  // namespace

namespace {
// Block output epilogue as its own pass over o (bf16 [rows][DV], one row per token-head):
// y = o / sqrt(mean_j o_j^2 + eps) * weight (.) silu(g), each factor optional, in place.
// A half-warp per row, eight channels per lane (16-byte loads), each thread with two rows in
// flight. Run inside the scan kernel's per-chunk chain, the same arithmetic lengthened that
// serial chain by more than this extra pass over o and g costs in HBM time.
__device__ __forceinline__ void epilogue_row(uint4 &ov, uint4 gv, const float (&w)[8], bool norm, bool gate,
                                             float eps)
{
    float o[8], gg[8];
    unpack8(ov, o);
    if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(o[i], o[i], ss);
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);  // within the half-warp
        const float rinv = rsqrtf(ss * (1.f / DV) + eps);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] *= rinv * w[i];
    }
    if (gate) {
        unpack8(gv, gg);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            // silu(g) = g / (1 + exp(-g)), exp argument kept below 80 so 1 + exp stays finite
            // (for g < -80, silu(g) is below 2e-33 in magnitude either way)
            o[i] *= gg[i] * recip_newton2(1.f + __expf(-fmaxf(gg[i], -80.f)));
    }
    ov = pack8(o);
}

__global__ void __launch_bounds__(256) output_epilogue_kernel(__nv_bfloat16 *y, const __nv_bfloat16 *g,
                                                              const float *weight, float eps, long long nrows)
{
    static_assert(DV == 128, "eight channels per lane of a half-warp");
    const int lane = threadIdx.x & 31, hl = lane & 15, half = lane >> 4;
    const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    float w[8];  // weight is only 4-byte aligned: scalar loads
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = weight ? weight[8 * hl + i] : 1.f;
    const bool norm = weight != nullptr, gate = g != nullptr;
    // each warp takes four rows per step (base is the same for all its lanes, so every lane
    // runs the half-warp shuffles): this half-warp's rows base + half and base + 2 + half
    for (long long base = 4 * wid; base < nrows; base += 4 * nw) {
        const long long r0 = base + half, r1 = base + 2 + half;
        const bool v0 = r0 < nrows, v1 = r1 < nrows;
        uint4 o0 = make_uint4(0u, 0u, 0u, 0u), o1 = o0, g0 = o0, g1 = o0;
        if (v0) o0 = reinterpret_cast<const uint4 *>(y + r0 * DV)[hl];
        if (v1) o1 = reinterpret_cast<const uint4 *>(y + r1 * DV)[hl];
        if (gate && v0) g0 = reinterpret_cast<const uint4 *>(g + r0 * DV)[hl];
        if (gate && v1) g1 = reinterpret_cast<const uint4 *>(g + r1 * DV)[hl];
        epilogue_row(o0, g0, w, norm, gate, eps);
        epilogue_row(o1, g1, w, norm, gate, eps);
        if (v0) reinterpret_cast<uint4 *>(y + r0 * DV)[hl] = o0;
        if (v1) reinterpret_cast<uint4 *>(y + r1 * DV)[hl] = o1;
    }
}

__global__ void recip_eval_kernel(const float *x, float *y, long long n)
{
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        y[i] = recip_newton2(x[i]);
}
}  // namespace

cudaError_t launch_recip_eval(const float *x, float *y, long long n, cudaStream_t s)
{
    const long long blocks = (n + 255) / 256;
    recip_eval_kernel<<<(unsigned)(blocks < 1024 ? blocks : 1024), 256, 0, s>>>(x, y, n);
    return cudaGetLastError();
}

bool forward_tc_supported(const FwdArgs &a)
{
    return a.bf16 && a.dk == DK && a.dv == DV && a.T > 0 && encode_fn() != nullptr;
}

// Dense: the slots, the gammas, then the fused kernel's queue counter (16 bytes) and task flags.
static size_t fused_sync_bytes(size_t ntasks) { return (16 + ntasks * 4 + 255) / 256 * 256; }

size_t forward_tc_workspace_bytes(int B, int T, int H)
{
    const size_t ntasks = (size_t)B * H * ((T + C - 1) / C);
    return ntasks * (SLOT_BYTES + GAMMA_BYTES) + fused_sync_bytes(ntasks);
}

// Packed sequences: at most H (ceil(T / 64) + N) tasks (each sequence adds at most one
// partial chunk), then the chunk offsets (N + 1 ints) and the task count.
static size_t varlen_task_capacity(int N, int T, int H) { return (size_t)H * ((T + C - 1) / C + N); }

size_t forward_tc_varlen_workspace_bytes(int N, int T, int H)
{
    // then cu_chunks (N + 1 ints), the task count and the scan order (N ints)
    return varlen_task_capacity(N, T, H) * (SLOT_BYTES + GAMMA_BYTES) +
           ((2 * (size_t)N + 2) * sizeof(int) + 255) / 256 * 256;
}

// The block's output epilogue, a pass over o after the forward's kernels (when asked for).
static cudaError_t launch_output_epilogue(const FwdArgs &a, int nsm, cudaStream_t s)
{
    if (!a.out_gate && !a.norm_weight) return cudaSuccess;
    const long long nrows = (long long)(a.cu_seqlens ? 1 : a.B) * a.T * a.H;
    if (nrows == 0) return cudaSuccess;
    const long long blocks = (nrows + 31) / 32;  // 8 warps of four rows per block
    const int eg = (int)(blocks < (long long)nsm * 16 ? blocks : (long long)nsm * 16);
    output_epilogue_kernel<<<eg, 256, 0, s>>>(static_cast<__nv_bfloat16 *>(a.o),
                                              static_cast<const __nv_bfloat16 *>(a.out_gate), a.norm_weight,
                                              a.norm_eps, nrows);
    return cudaGetLastError();
}

cudaError_t launch_forward_tc(const FwdArgs &a, cudaStream_t s)
{
    const bool varlen = a.cu_seqlens != nullptr;
    const int Bm = varlen ? 1 : a.B;  // tensor-map batch extent: packed sequences share one
    const bool bsc = (a.gates & kGateScalarB) != 0, wsc = (a.gates & kGateScalarW) != 0;
    CUtensorMap mq, mk, mb, mv, mw, mla, mo;
    if (!make_map(&mq, a.q, false, Bm, a.T, a.H, DK) || !make_map(&mk, a.k, false, Bm, a.T, a.H, DK) ||
        !make_map(&mv, a.v, false, Bm, a.T, a.H, DV) || !make_map(&mla, a.log_alpha, true, Bm, a.T, a.H, DK) ||
        !make_map(&mo, a.o, false, Bm, a.T, a.H, DV))
        return cudaErrorInvalidValue;
    // a scalar gate has no tile to copy: its map slot is never used (the q map stands in)
    if (bsc) mb = mq; else if (!make_map(&mb, a.b, false, Bm, a.T, a.H, DK)) return cudaErrorInvalidValue;
    if (wsc) mw = mq; else if (!make_map(&mw, a.w, false, Bm, a.T, a.H, DV)) return cudaErrorInvalidValue;
    const bool general = varlen || bsc || wsc;
    const bool bwd = a.bwd_ext != nullptr;
    if (bwd && varlen) return cudaErrorInvalidValue;
    void (*chunk)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                  const CUtensorMap, ChunkParams) =
        general ? (bwd ? fwd_chunk_kernel<true, true> : fwd_chunk_kernel<true>)
                : (bwd ? fwd_chunk_kernel<false, true> : fwd_chunk_kernel<false>);
    cudaError_t e = cudaFuncSetAttribute(chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fwd_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SC_SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int NC = (a.T + C - 1) / C;
    const int ntasks = varlen ? (int)varlen_task_capacity(a.B, a.T, a.H) : a.B * a.H * NC;
    unsigned char *ws = static_cast<unsigned char *>(a.workspace);
    int *cu_chunks = nullptr, *ntasks_dev = nullptr, *seq_order = nullptr;
    if (varlen) {
        cu_chunks = reinterpret_cast<int *>(ws + (size_t)ntasks * (SLOT_BYTES + GAMMA_BYTES));
        ntasks_dev = cu_chunks + a.B + 1;
        seq_order = ntasks_dev + 1;
        varlen_prefix_kernel<<<1, 1024, 0, s>>>(a.cu_seqlens, a.B, a.T, a.H, cu_chunks, ntasks_dev, seq_order,
                                                 a.status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    ChunkParams cp{a.B,         a.T,       a.H,        NC,
                   ntasks,      ws,        a.status,   a.cu_seqlens,
                   cu_chunks,   ntasks_dev, a.gates,   static_cast<const __nv_bfloat16 *>(a.b),
                   static_cast<const __nv_bfloat16 *>(a.w), a.bwd_ext, debug_giveup_flag()};
    // The fused kernel (chunk tasks, then the scans on B H of the CTAs) when the scans leave
    // enough SMs to the queue's tail: dense sequences and room for the queue and flags. With
    // the backward's extras it also keeps T and W (bwd_ext) and the chunk-entry states; a
    // call for the chunk tasks alone (chunks_only) takes the chunk kernel.
    const int BH = a.B * a.H;
    int coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    // the queue and flags: behind the slots in a forward's workspace, or where the caller says
    unsigned char *sync = a.fused_sync ? a.fused_sync
                          : (a.workspace_bytes >= forward_tc_workspace_bytes(a.B, a.T, a.H)
                                 ? ws + (size_t)ntasks * (SLOT_BYTES + GAMMA_BYTES) : nullptr);
    const bool fused = !varlen && !a.chunks_only && sync != nullptr && coop != 0 && !debug_unfused_flag() &&
                       BH + kFusedMinQueueCtas <= nsm;
    if (fused) {
        void (*fk)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                   const CUtensorMap, const CUtensorMap, ChunkParams, ScanParams) =
            general ? (bwd ? fwd_fused_kernel<true, true> : fwd_fused_kernel<true, false>)
                    : (bwd ? fwd_fused_kernel<false, true> : fwd_fused_kernel<false, false>);
        e = cudaFuncSetAttribute(fk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fk, NT, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        e = cudaMemsetAsync(sync, 0, fused_sync_bytes(ntasks), s);
        if (e != cudaSuccess) return e;
        cp.queue = reinterpret_cast<int *>(sync);
        cp.flags = reinterpret_cast<unsigned *>(sync + 16);
        cp.BH = BH;
        // The scans start once (nsm - BH) CTAs can finish the rest of the queue in about the
        // time of one scan: rest ~ (nsm - BH) * NC * (scan time per chunk / chunk task time).
        const double ratio = a.saved_states ? kSavingScanToTaskTime : (NC >= 256 ? kLongScanToTaskTime : kScanToTaskTime);
        const double rest = (double)(nsm - BH) * NC * ratio;
        cp.switch_at = rest >= ntasks ? 0 : ntasks - (int)rest;
        ScanParams sp{a.B, a.T, a.H, NC, ntasks, ws, a.S0, a.S_T, a.saved_states, a.status, nullptr, nullptr,
                      static_cast<__nv_bfloat16 *>(a.o)};
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(nsm);
        cfg.blockDim = dim3(NT);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the scans wait on the others
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, fk, mq, mk, mb, mv, mw, mla, mo, cp, sp);
        if (e == cudaSuccess) return launch_output_epilogue(a, nsm, s);
        // the device could not hold every CTA at once (another context holds SMs): the two
        // kernels below do the same work without that requirement
        if (e != cudaErrorCooperativeLaunchTooLarge) return e;
        (void)cudaGetLastError();
        cp.queue = nullptr;
        cp.flags = nullptr;
        cp.BH = cp.switch_at = 0;
    }
    const int grid = ntasks < nsm ? ntasks : nsm;
    chunk<<<grid, NT, SMEM_BYTES, s>>>(mq, mk, mb, mv, mw, mla, cp);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.chunks_only) return e;
    ScanParams sp{a.B,          a.T,          a.H,    NC,       ntasks,    ws,
                  a.S0,         a.S_T,        a.saved_states, a.status, a.cu_seqlens, cu_chunks,
                  static_cast<__nv_bfloat16 *>(a.o)};
    sp.seq_order = seq_order;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.H);
    cfg.blockDim = dim3(SC_NT);
    cfg.dynamicSmemBytes = SC_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, fwd_scan_kernel, mo, sp);
    if (e != cudaSuccess) return e;
    return launch_output_epilogue(a, nsm, s);
}

size_t fused_sync_bytes_for(size_t ntasks) { return fused_sync_bytes(ntasks); }

cudaError_t launch_backward_front_fused(const FwdArgs &a, const BwdFrontArgs &r, cudaStream_t s, bool *launched)
{
    *launched = false;
    if (a.cu_seqlens || !a.bwd_ext || !a.chunks_only || debug_unfused_flag()) return cudaSuccess;
    int dev = 0, nsm = 148, coop = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    const int BH = a.B * a.H;
    if (!coop || BH + kFusedMinQueueCtas > nsm) return cudaSuccess;
    const bool bsc = (a.gates & kGateScalarB) != 0, wsc = (a.gates & kGateScalarW) != 0;
    CUtensorMap mq, mk, mb, mv, mw, mla, mdo;
    if (!make_map(&mq, a.q, false, a.B, a.T, a.H, DK) || !make_map(&mk, a.k, false, a.B, a.T, a.H, DK) ||
        !make_map(&mv, a.v, false, a.B, a.T, a.H, DV) || !make_map(&mla, a.log_alpha, true, a.B, a.T, a.H, DK) ||
        !make_map(&mdo, r.dO, false, a.B, a.T, a.H, DV, 64, true))
        return cudaErrorInvalidValue;
    if (bsc) mb = mq; else if (!make_map(&mb, a.b, false, a.B, a.T, a.H, DK)) return cudaErrorInvalidValue;
    if (wsc) mw = mq; else if (!make_map(&mw, a.w, false, a.B, a.T, a.H, DV)) return cudaErrorInvalidValue;
    const bool general = bsc || wsc;
    void (*fk)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
               const CUtensorMap, const CUtensorMap, ChunkParams, RsParams) =
        general ? bwd_front_kernel<true> : bwd_front_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(fk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fk, NT, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaSuccess;
    const int NC = (a.T + C - 1) / C;
    const int ntasks = BH * NC;
    e = cudaMemsetAsync(r.sync, 0, fused_sync_bytes(ntasks), s);
    if (e != cudaSuccess) return e;
    ChunkParams cp{a.B,     a.T,     a.H,      NC,
                   ntasks,  static_cast<unsigned char *>(a.workspace), a.status, nullptr,
                   nullptr, nullptr, a.gates,  static_cast<const __nv_bfloat16 *>(a.b),
                   static_cast<const __nv_bfloat16 *>(a.w), a.bwd_ext, debug_giveup_flag()};
    cp.queue = reinterpret_cast<int *>(r.sync);
    cp.flags = reinterpret_cast<unsigned *>(r.sync + 16);
    cp.BH = BH;
    const double rest = (double)(nsm - BH) * NC * kRevScanToTaskTime;
    cp.switch_at = rest >= ntasks ? 0 : ntasks - (int)rest;
    RsParams rp{a.B, a.T, a.H, NC, ntasks, static_cast<const unsigned char *>(a.workspace), r.dS_T, r.gS0, r.dsc,
                a.status};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nsm);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the scans wait on the others
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, fk, mq, mk, mb, mv, mw, mla, mdo, cp, rp);
    if (e == cudaSuccess) *launched = true;
    if (e == cudaErrorCooperativeLaunchTooLarge) {  // not every CTA fits at once: the caller's two launches
        (void)cudaGetLastError();
        return cudaSuccess;
    }
    return e;
}

}  // namespace gdr2
