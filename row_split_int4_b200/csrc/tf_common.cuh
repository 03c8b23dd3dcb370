// tf_common.cuh -- small device helpers shared by the kernels of libtf.so.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tf.h"

namespace tf {

constexpr int kGroup = TF_GROUP;
constexpr int kNumSMs = 148;   // B200: 2 dies x 74 SMs; grids are sized in multiples of it

// bf16 bit pattern -> fp32 (exact: a bf16 is the top half of an fp32).
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// fp32 -> bf16 bits, round to nearest even; NaN becomes 0x7FC0 (the NaN the
// pages use for a broken link), overflow rounds to +-Inf.  The rounding adds
// 0x7FFF plus the lowest kept bit, the usual carry-propagation form of RNE.
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)TF_NAN_BF16;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// g * SiLU(u) in fp32, SiLU(u) = u / (1 + exp(-u)).  For u < 0 the same
// quantity is written u*e/(1+e) with e = exp(u), which stays finite where
// exp(-u) would overflow.
__device__ __forceinline__ float glu_f32(float g, float u) {
    float s;
    if (u >= 0.0f) {
        s = u / (1.0f + expf(-u));
    } else {
        float e = expf(u);
        s = (u * e) / (1.0f + e);
    }
    return g * s;
}

__host__ __forceinline__ bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

}  // namespace tf
