// tc_common.cuh -- pieces shared by the tensor-core forward (fwd_tc.cu) and
// backward (bwd_tc.cu) at dk = dv = 128, chunk C = 64: the 128-byte-swizzled
// operand addressing, bf16 packing, the workspace slot that the forward's
// chunk kernel writes, and the TMA tensor maps of token-major [B, T, H, D]
// tensors.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace gdr2 {
namespace tc {

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per bounded wait
constexpr float kFactorLimit = 70.f;              // |exponent| of one decay factor

// Offset of the 16-byte chunk holding columns [8*o8, 8*o8 + 8) of `row` in an
// operand image of `rows` rows whose columns come in blocks of 64 bf16 (128 B),
// each block rows x 128 B, 128-byte swizzled (chunk index XOR row % 8). Such an
// image is K-major for (M or N = rows, K = columns) and MN-major for (K = rows,
// M or N = columns).
__device__ __forceinline__ uint32_t sw_chunk(int row, int o8, int rows)
{
    const int blk = o8 >> 3, ch = o8 & 7;
    return (uint32_t)(blk * rows * 128 + row * 128 + ((ch ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8])
{
    uint4 u;
    __nv_bfloat162 h;
    h = __floats2bfloat162_rn(f[0], f[1]); u.x = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[2], f[3]); u.y = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[4], f[5]); u.z = *reinterpret_cast<uint32_t *>(&h);
    h = __floats2bfloat162_rn(f[6], f[7]); u.w = *reinterpret_cast<uint32_t *>(&h);
    return u;
}

__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8])
{
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ void load8f(const float *p, float (&f)[8])
{
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ void store8f(float *p, const float (&f)[8])
{
    *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// 1 / d for normal 2^-126 <= d < 2^125, relative error at most 6.6e-6. The method: the
// bit pattern of a positive float is close to 2^23 (log2 d + 127), so subtracting it from
// a constant negates log2 d and one integer operation gives a seed for 1 / d (the
// integer-arithmetic approximations of J. Blinn, "Floating-point tricks", IEEE Computer
// Graphics and Applications 17(4), 1997). The constant 0x7EF311C2 makes the seed's relative
// error equioscillate at +-5.051% over a binade, hence in every binade. Two Newton-Raphson
// steps r <- r + r (1 - d r), each squaring the relative error, leave 6.6e-6. (At d >= 2^125
// the seed is subnormal and the bound fails; the callers stay below e^80 < 2^116.) All of it
// on the FMA and integer pipes: the special-function unit is the scarce one.
__device__ __forceinline__ float recip_newton2(float d)
{
    float r = __int_as_float(0x7EF311C2 - __float_as_int(d));
    r = fmaf(r, fmaf(-d, r, 1.f), r);
    return fmaf(r, fmaf(-d, r, 1.f), r);
}

// Sum vals over the 32 lanes of a warp for each of its N entries; on return lane L holds, in
// vals[0 .. N/32), the sums of the N/32 entries from (N/32) L on.
template <int N>
__device__ __forceinline__ void transpose_reduce32(float (&vals)[N], int lane)
{
#pragma unroll
    for (int o = 16, n = N; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? vals[i] : vals[i + n / 2];
            const float keep = upper ? vals[i + n / 2] : vals[i];
            vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
}

// ---- workspace slot written by the forward's chunk kernel (one per (batch, head, chunk)
// task), in the operand layouts of the kernels that read it ----
constexpr uint32_t SLOT_B1 = 0;       // [Q'; M]  [c' block][64 t + 128 c rows][64 c']
constexpr uint32_t SLOT_KT = 49152;   // K~       [c block][t rows][64 c]
constexpr uint32_t SLOT_U = 65536;    // U~^T     [j rows][64 t]
constexpr uint32_t SLOT_P = 81920;    // P        [t rows][64 i]
constexpr uint32_t SLOT_BYTES = 90112;
constexpr int B1_ROWS = 192;          // rows of [Q'; M]: t first, then c
constexpr uint32_t GAMMA_BYTES = DK * 4;  // exp(G_C) per task, stored after all slots
// What the backward also needs from the chunk kernel, in a region of its own (one per task):
constexpr uint32_t EXT_T = 0;         // T = (I + A)^-1 in bf16, [t rows][64 s]
constexpr uint32_t EXT_W = 8192;      // W in bf16, [c rows][64 t]
constexpr uint32_t EXT_BYTES = 24576;

// ---- host side: TMA tensor maps ----
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [B, T, H, D] token-major tensor as a 4-D map {D, H, T, B}. Box: `box_d` channels x 1 head x
// 64 tokens x 1 sequence, unswizzled rows of box_d elements, or 128-byte swizzled (box_d x
// element size = 128 B) to land as an operand image. The per-sequence extent T makes loads
// past the end of a sequence read zeros and stores past it drop.
inline bool make_map(CUtensorMap *m, const void *base, bool f32, int B, int T, int H, int D, int box_d = 0,
                     bool sw128 = false)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t esz = f32 ? 4 : 2;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * esz, (cuuint64_t)H * D * esz, (cuuint64_t)T * H * D * esz};
    cuuint32_t box[4] = {(cuuint32_t)(box_d > 0 ? box_d : D), 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace gdr2
