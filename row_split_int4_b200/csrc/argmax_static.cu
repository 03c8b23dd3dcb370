// argmax_static.cu -- tf_argmax_rows_static: the argmax with its partial-result
// scratch in a device array of this library instead of a caller buffer, for
// callers that cannot allocate device memory (see include/tf.h).
#include <atomic>
#include <cstring>

#include "tf_common.cuh"
#include "tf_kernels.h"

namespace tf {

// Per-block candidate keys of tf_argmax_rows, TF_STATIC_SCRATCH_BYTES bytes on
// every device that loads the library.  Host code must not use this name as an
// address: it only identifies the symbol for cudaGetSymbolAddress.
static __device__ __align__(256) uint64_t g_argmax_static_scratch[TF_STATIC_SCRATCH_BYTES / sizeof(uint64_t)];

// Its device address, looked up once per device (with that device current).
static std::atomic<void *> g_static_scratch_addr[64];

static cudaError_t static_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    void *p = g_static_scratch_addr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        e = cudaGetSymbolAddress(&p, g_argmax_static_scratch);
        if (e != cudaSuccess) return e;
        g_static_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace tf

using namespace tf;

extern "C" tf_status tf_argmax_rows_static(const void *logits, int M, int n, int ld, uint32_t id_base, uint64_t *words,
                                           tf_stream stream) {
    if (M < 0 || M > 65535 || n < 1 || ld < n) return TF_E_ARG;
    if ((unsigned long long)id_base + (unsigned long long)n > 0x80000000ull) return TF_E_RANGE;
    if (M == 0) return TF_OK;
    if (!logits || !words) return TF_E_ARG;
    if (tf_argmax_scratch_bytes(M, n) > TF_STATIC_SCRATCH_BYTES) return TF_E_ARG;
    if (!aligned(logits, 2) || !aligned(words, 8)) return TF_E_ALIGN;
    void *scratch = nullptr;
    if (cuda_status(static_scratch(&scratch)) != TF_OK) return TF_E_CUDA;
    ArgmaxArgs a;
    std::memset(&a, 0, sizeof a);
    a.logits = static_cast<const uint16_t *>(logits);
    a.ld = ld;
    a.n = n;
    a.id_base = id_base;
    a.M = M;
    a.partial = static_cast<uint64_t *>(scratch);
    a.words = words;
    a.vec = aligned(logits, 16) && (ld % 8 == 0);
    return cuda_status(launch_argmax(a, reinterpret_cast<cudaStream_t>(stream)));
}
