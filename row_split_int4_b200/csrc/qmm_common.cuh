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

// sum_{i<32} x_i w_i for one lane-chunk with w_i = s q_i + b formed in fp32 per
// element, two accumulators (even / odd i, ascending), added at the end.  Each
// product is of x and the weight itself, so a large x whose weight is zero adds
// exactly nothing, whatever the other x are.  xv[j] holds x for the lane's
// elements 4j..4j+3.
__device__ __forceinline__ float lane_chunk_wdot(const uint4 &q, const float4 *xv, float s, float b) {
    float pe = 0.0f, po = 0.0f;
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        Codes8 c = decode8(words[w]);
        const float4 u = xv[2 * w], v = xv[2 * w + 1];
        pe = fmaf(fmaf(s, c.f[0], b), u.x, pe);
        po = fmaf(fmaf(s, c.f[1], b), u.y, po);
        pe = fmaf(fmaf(s, c.f[2], b), u.z, pe);
        po = fmaf(fmaf(s, c.f[3], b), u.w, po);
        pe = fmaf(fmaf(s, c.f[4], b), v.x, pe);
        po = fmaf(fmaf(s, c.f[5], b), v.y, po);
        pe = fmaf(fmaf(s, c.f[6], b), v.z, pe);
        po = fmaf(fmaf(s, c.f[7], b), v.w, po);
    }
    return pe + po;
}

__device__ __forceinline__ float warp_sum_to_lane0(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, o);
    return v;
}

}  // namespace tf
