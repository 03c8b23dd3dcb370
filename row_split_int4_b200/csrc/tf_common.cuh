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

// A candidate is one 64-bit key whose unsigned order is the selection order:
//   bit 63      non-finite flag (flagged beats every finite value)
//   bits 62..31 16-bit order-preserving image of the bf16 value (finite only;
//               -0 is mapped to +0 so that the two tie)
//   bits 30..0  0x7FFFFFFF - id (the lower id wins among equals)
// max() over keys is associative and commutative, so the block and grid
// reduction trees cannot change the result.  0 is below every real key.
__device__ __forceinline__ uint64_t cand_key(uint32_t h, uint32_t id) {
    const uint64_t idpart = (uint64_t)(0x7FFFFFFFu - id);
    if ((h & 0x7F80u) == 0x7F80u) return (1ull << 63) | idpart;   // NaN or +-Inf
    if (h == 0x8000u) h = 0u;
    const uint32_t mono = (h & 0x8000u) ? (~h & 0xFFFFu) : (h | 0x8000u);
    return ((uint64_t)mono << 31) | idpart;
}

__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t umin64(uint64_t a, uint64_t b) { return a < b ? a : b; }

__device__ __forceinline__ uint64_t warp_max64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = umax64(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// The word of a row from its best key: the id, and the winning value read back
// from the logits so that a winning -0 keeps its sign; a flagged key gives the
// flag and the first non-finite id.
__device__ __forceinline__ uint64_t word_of_key(uint64_t best, const uint16_t *row, uint32_t id_base) {
    const uint32_t id = 0x7FFFFFFFu - (uint32_t)(best & 0x7FFFFFFFull);
    if (best == 0) {
        // unreachable for n >= 1 (every element yields a nonzero key); kept so that
        // no input can make the read below leave the row
        return ((uint64_t)(TF_PAIR_FLAG | id_base) << 32) | 0x7FC00000ull;
    }
    if (best >> 63) return ((uint64_t)(TF_PAIR_FLAG | id) << 32) | 0x7FC00000ull;
    const uint32_t h = row[id - id_base];
    return ((uint64_t)id << 32) | ((uint64_t)h << 16);
}

__host__ __forceinline__ bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// ------------------------------------------------ programmatic dependent launch
// Every kernel of the library is launched with programmatic stream
// serialization: it may be scheduled while the kernel before it on the stream is
// still running, once every block of that kernel has called pdl_trigger() (or
// exited).  pdl_wait() blocks the calling thread until the kernels before it
// have finished and their writes are visible.  Each kernel calls pdl_wait()
// before it reads any array it was given or writes any output, with one
// exception: a qmm kernel may read weights first (into L2 or shared memory).
// No kernel of the library writes weights, and a kernel from elsewhere never
// calls launch_dependents, so the kernel after it starts only once it has
// ended and the weights it wrote are in place.  Each
// qmm kernel calls pdl_trigger() once its own pdl_wait() has returned, so that
// the next one queues behind it but no further; the short kernels between them
// (gather, argmax, pick, ...) call it first thing, so that the qmm after them
// can take each SM as soon as the qmm before them leaves it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// false when the environment sets TF_PDL=0: launches then keep the plain stream
// order (the kernels' pdl_wait/pdl_trigger do nothing)
bool pdl_enabled();

// kernel<<<grid, block, smem, stream>>>(args...) with programmatic stream serialization
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace tf
