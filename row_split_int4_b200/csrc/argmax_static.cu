// argmax_static.cu -- tf_argmax_rows_static: the argmax with its partial-result
// scratch in a device array of this library instead of a caller buffer, for
// callers that cannot allocate device memory (see include/tf.h).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "tf_common.cuh"
#include "tf_kernels.h"

namespace tf {

// Per-block candidate keys of tf_argmax_rows, TF_STATIC_SCRATCH_BYTES bytes on
// every device that loads the library.  Host code must not use this name as an
// address: it only identifies the symbol for cudaGetSymbolAddress.
static __device__ __align__(256) uint64_t g_argmax_static_scratch[TF_STATIC_SCRATCH_BYTES / sizeof(uint64_t)];

// Its device address on each device, with the id of the context it was looked
// up in.  The address belongs to the module as loaded in that context: after a
// cudaDeviceReset (or any teardown of the primary context) the library's module
// is loaded again in a new context, possibly elsewhere, so an address is reused
// only while the current context is the one it came from.  Context ids are
// unique for the life of the process (cuCtxGetId), unlike context handles.
static std::mutex g_static_mu;
static void *g_static_addr[64];
static unsigned long long g_static_ctx[64];   // 0: no usable id, look up again next call

static bool current_context_id(unsigned long long *id) {
    static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
    });
    if (!get_cur || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

static cudaError_t static_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (have_id && g_static_addr[dev] != nullptr && g_static_ctx[dev] == id) {
        *out = g_static_addr[dev];
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_argmax_static_scratch);   // with the device current
    if (e != cudaSuccess) return e;
    unsigned long long id2 = 0;   // the lookup may have made the context current
    g_static_addr[dev] = p;
    g_static_ctx[dev] = current_context_id(&id2) ? id2 : 0ull;
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
