// qmm_common.cuh -- the per-lane arithmetic every qmm kernel shares, so that
// all of them reduce a row in the same order (see qmm_gemv.cu for the order).
#pragma once

#include "tf_common.cuh"
#include "tf_kernels.h"

namespace tf {

constexpr int kChunk = 1024;             // k per warp-wide 16-byte load of packed codes

// Whole-matrix row of output column `col` (NONE), or of member `which`
// (0 = gate, 1 = up) of column `col` (GLU).
__device__ __forceinline__ int seg_row(const SegTable &t, int col, int glu, int which) {
    if (glu) return t.row0[which] + col;
    int r = -1;
#pragma unroll
    for (int s = 0; s < TF_MAX_SEGS; ++s)
        if (s < t.nseg && col >= t.col0[s] && col < t.col0[s] + t.nrows[s]) r = t.row0[s] + (col - t.col0[s]);
    return r;
}

// 8 codes of one 32-bit word -> fp32, exactly.  Each nibble is masked in place
// and OR-ed with the exponent that makes its bit position worth 1, so the
// float holds 2^E + q; subtracting 2^E leaves q.  Positions 0..4 are read
// from w, positions 5..7 from w >> 12.
struct Codes8 {
    float f[8];
};
__device__ __forceinline__ Codes8 decode8(uint32_t w) {
    const uint32_t h = w >> 12;
    Codes8 c;
    c.f[0] = __uint_as_float((w & 0x0000000Fu) | 0x4B000000u) - 8388608.0f;  // 2^23
    c.f[1] = __uint_as_float((w & 0x000000F0u) | 0x49000000u) - 524288.0f;   // 2^19
    c.f[2] = __uint_as_float((w & 0x00000F00u) | 0x47000000u) - 32768.0f;    // 2^15
    c.f[3] = __uint_as_float((w & 0x0000F000u) | 0x45000000u) - 2048.0f;     // 2^11
    c.f[4] = __uint_as_float((w & 0x000F0000u) | 0x43000000u) - 128.0f;      // 2^7
    c.f[5] = __uint_as_float((h & 0x00000F00u) | 0x47000000u) - 32768.0f;
    c.f[6] = __uint_as_float((h & 0x0000F000u) | 0x45000000u) - 2048.0f;
    c.f[7] = __uint_as_float((h & 0x000F0000u) | 0x43000000u) - 128.0f;
    return c;
}

// P = sum_{i<32} q_i x_i for one lane-chunk, two accumulators (even/odd i).
// xv[j] holds x for the lane's elements 4j..4j+3.
__device__ __forceinline__ float lane_chunk_dot(const uint4 &q, const float4 *xv) {
    float pe = 0.0f, po = 0.0f;
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        Codes8 c = decode8(words[w]);
        const float4 a = xv[2 * w], b = xv[2 * w + 1];
        pe = fmaf(c.f[0], a.x, pe);
        po = fmaf(c.f[1], a.y, po);
        pe = fmaf(c.f[2], a.z, pe);
        po = fmaf(c.f[3], a.w, po);
        pe = fmaf(c.f[4], b.x, pe);
        po = fmaf(c.f[5], b.y, po);
        pe = fmaf(c.f[6], b.z, pe);
        po = fmaf(c.f[7], b.w, po);
    }
    return pe + po;
}

// X = ascending fp32 sum of the lane's 32 x values.
__device__ __forceinline__ float lane_chunk_xsum(const float4 *xv) {
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        s += xv[j].x;
        s += xv[j].y;
        s += xv[j].z;
        s += xv[j].w;
    }
    return s;
}

__device__ __forceinline__ float warp_sum_to_lane0(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, o);
    return v;
}

// The same P from bf16 x: x8[j] holds the lane's elements 8j..8j+7 as bf16
// pairs.  Codes become bf16 (128 + q) two at a time (nibbles i and i+4 of a
// word, one lop3 each), 128 is taken off exactly in bf16x2, and each product
// q*x is added to the fp32 accumulators with one mixed-precision FMA.  q*x is
// exact (4 x 8 significant bits) and the additions happen in the same order,
// so the result is bit-identical to lane_chunk_dot.
__device__ __forceinline__ uint32_t bf16x2_sub128(uint32_t t) {
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(t), "r"(0x43004300u));
    return r;
}
#define TF_MFMA(SEL_A, SEL_B)                                                                                   \
    __device__ __forceinline__ float mfma_##SEL_A##_##SEL_B(uint32_t a, uint32_t b, float c) {                 \
        asm("{ .reg .b16 a0, a1, b0, b1;\n mov.b32 {a0, a1}, %1;\n mov.b32 {b0, b1}, %2;\n"                  \
            " fma.rn.f32.bf16 %0, a" #SEL_A ", b" #SEL_B ", %0;\n}"                                           \
            : "+f"(c)                                                                                         \
            : "r"(a), "r"(b));                                                                                \
        return c;                                                                                              \
    }
TF_MFMA(0, 0)
TF_MFMA(0, 1)
TF_MFMA(1, 0)
TF_MFMA(1, 1)
#undef TF_MFMA

__device__ __forceinline__ float lane_chunk_dot_bf16(const uint4 &q, const uint4 *x8) {
    float pe = 0.0f, po = 0.0f;
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t v = words[w];
        const uint32_t t0 = bf16x2_sub128((v & 0x000F000Fu) | 0x43004300u);          // (q0, q4)
        const uint32_t t1 = bf16x2_sub128(((v >> 4) & 0x000F000Fu) | 0x43004300u);   // (q1, q5)
        const uint32_t t2 = bf16x2_sub128(((v >> 8) & 0x000F000Fu) | 0x43004300u);   // (q2, q6)
        const uint32_t t3 = bf16x2_sub128(((v >> 12) & 0x000F000Fu) | 0x43004300u);  // (q3, q7)
        const uint4 xx = x8[w];   // (x0,x1) (x2,x3) (x4,x5) (x6,x7)
        pe = mfma_0_0(t0, xx.x, pe);
        po = mfma_0_1(t1, xx.x, po);
        pe = mfma_0_0(t2, xx.y, pe);
        po = mfma_0_1(t3, xx.y, po);
        pe = mfma_1_0(t0, xx.z, pe);
        po = mfma_1_1(t1, xx.z, po);
        pe = mfma_1_0(t2, xx.w, pe);
        po = mfma_1_1(t3, xx.w, po);
    }
    return pe + po;
}

// X from bf16 x: the same ascending fp32 sum as lane_chunk_xsum.
__device__ __forceinline__ float lane_chunk_xsum_bf16(const uint4 *x8) {
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w[4] = {x8[j].x, x8[j].y, x8[j].z, x8[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            s += __uint_as_float(w[e] << 16);
            s += __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
    return s;
}

}  // namespace tf
