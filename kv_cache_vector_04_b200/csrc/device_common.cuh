// Device-side helpers shared by the TurboQuant kernels (sm_100a).
#pragma once
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "tq.h"

namespace tq {

constexpr unsigned kFull = 0xffffffffu;

// Bit positions inside a lane string of the packed tile format (B_K, B_V, qjl)
// at head dim D (include/tq.h): for pair slot p (k-step p / 4, fragment
// register p % 4) and element e in {0, 1},
//   key cell:    kbit(p, e), B_K bits;   QJL sign: sbit(p, e), 1 bit;
//   value cell:  vbit(p, e), B_V bits.
// Generic layout: key pairs packed at 2 B_K bits a pair, then the sign words
// (pair p at bits p % 16 and 16 + p % 16 of sign word p / 16), then the value
// pairs. With 3-bit keys and QJL ((3, 4, 1)) a key pair and its two signs fill
// one byte each: key pair p in the low 6 bits of byte p, the sign pairs of
// word w at bits a and a + 16 for a = 6, 7, 14, 15 (pairs 4w .. 4w + 3), so
// the decoder finds a key pair's table row with one byte permute and a sign
// pair with one shift. With 2-bit keys, 3-bit values and QJL ((2, 3, 1)) a
// value pair and two signs fill one byte each the same way, in the region
// after the key codes. With 4-bit cells the generic layout is byte-aligned
// already.
template <int D, int KB, int VB, int QJ>
struct TileLayout {
    static constexpr bool KS_BYTES = QJ == 1 && KB == 3;
    static constexpr bool VS_BYTES = QJ == 1 && KB == 2 && VB == 3;
    static constexpr int SB0 = KB * D / 2;                   // first sign bit (generic)
    static constexpr int VB0 = VS_BYTES ? KB * D / 2 : (KB + QJ) * D / 2;   // first value bit
    __host__ __device__ static constexpr int kbit(int p, int e)
    {
        return (KS_BYTES ? 8 : 2 * KB) * p + e * KB;
    }
    __host__ __device__ static constexpr int sbit(int p, int e)
    {
        return KS_BYTES   ? 32 * (p >> 2) + 16 * e + 6 + (p & 1) + 8 * ((p >> 1) & 1)
               : VS_BYTES ? VB0 + 32 * (p >> 2) + 16 * e + 6 + (p & 1) + 8 * ((p >> 1) & 1)
                          : SB0 + 32 * (p >> 4) + 16 * e + (p & 15);
    }
    __host__ __device__ static constexpr int vbit(int p, int e)
    {
        return VS_BYTES ? VB0 + 8 * p + 3 * e : VB0 + 2 * VB * p + e * VB;
    }
};

// Device copies of one context's tables (all pointers into one allocation).
struct DevTables {
    const float* centroids_k;   // [2^BK] fp32
    const double* bounds_k;     // [2^BK - 1] fp64 copies of the fp32 bounds
    const double* centroids_kd; // [2^BK] fp64 copies of the fp32 centroids
    const double* bounds_v;     // [2^BV - 1]
    const float* signs;         // D as fp32 +-1, [d]
    const uint2* s_frag;        // S^T as m16n8k16 B fragments: [d/16][m/8][32 lanes] (fp16 pairs)
    const float* s_t;           // S^T fp32 [d][m]
    const uint32_t* lut_k;      // [4^BK] fp16x2: alpha_k sqrt(d) (cK[f & (2^BK-1)], cK[f >> BK])
    const uint32_t* lut_v;      // [4^BV] fp16x2, the same for the value codebook
    unsigned* status;           // sticky TQ_STATUS_* bits
    float alpha_k;              // lut_k holds alpha_k * sqrt(d) * cK (see choose_decode_scale)
};

// D = A(16x16, row) * B(16x8, col) + D with fp16 inputs and fp32 accumulation.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same product with a zero accumulator (the first k-step of a chain).
__device__ __forceinline__ void mma_16816_first(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// D = A(16x32, row, u8) * B(32x8, col, s8 or u8) + D with int32 accumulation
// (exact). BS8 selects a signed B.
template <bool BS8>
__device__ __forceinline__ void imma_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1)
{
    if constexpr (BS8)
        asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
            : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
            : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same product with a zero accumulator (the first k-step of a chain).
template <bool BS8>
__device__ __forceinline__ void imma_16832_first(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                 uint32_t a3, uint32_t b0, uint32_t b1)
{
    if constexpr (BS8)
        asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
            : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
    else
        asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
            : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// 2^x with the SFU's approximate exponential (relative error ~2^-22;
// subnormal results flush to 0, which only touches weights below 2^-126).
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// Transpose an 8x8 matrix of 16-bit values held in the m8n8 fragment layout
// (lane 4g+t holds row g, columns 2t and 2t+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b)
{
    return __half2float(__ushort_as_half(b));
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v)
{
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(kFull, v, s);
    return v;
}

// In-lane Walsh–Hadamard butterflies over the V consecutive coordinates a lane
// holds (coordinate = lane * V + k), then the cross-lane stages by shuffles.
// Sylvester (natural) order, unnormalised.
template <int V>
__device__ __forceinline__ void wht_warp(double (&x)[V], int lane)
{
#pragma unroll
    for (int s = 1; s < V; s <<= 1) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            if (!(i & s)) {
                const double a = x[i], b = x[i + s];
                x[i] = a + b;
                x[i + s] = a - b;
            }
        }
    }
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const double o = __shfl_xor_sync(kFull, x[i], s);
            x[i] = upper ? (o - x[i]) : (x[i] + o);
        }
    }
}

// Cell index = number of boundaries strictly below y (binary search over the
// 2^B - 1 sorted boundaries).
template <int B>
__device__ __forceinline__ int encode_cell(double y, const double* bounds)
{
    int idx = 0;
#pragma unroll
    for (int s = (1 << B) / 2; s >= 1; s >>= 1)
        if (y > bounds[idx + s - 1]) idx += s;
    return idx;
}

// fp16 storage of a norm: round to nearest even, saturating at 65504.
__device__ __forceinline__ uint16_t norm_to_half_bits(double v, unsigned& sat)
{
    if (v > 65504.0) {
        sat = 1u;
        return 0x7bffu;
    }
    return __half_as_ushort(__double2half(v));
}

}  // namespace tq
