// seam.cu -- the kernels that join row slices and decide the head's token:
// gather (a pure copy of whole bf16 rows), the per-slice argmax and the pick
// (TensorFold PR #1433, step-1 body: pair_gather, pair_argmax, pair_pick
// move bf16 frames and compare values only).
#include "tf_common.cuh"
#include "tf_kernels.h"

namespace tf {

// ---------------------------------------------------------------- gather --
// One thread per 8 bf16 (16 bytes) of the output; every part's width and
// offset and the row pitches are multiples of 8, the pointers 16-byte aligned.
__global__ void gather_vec_kernel(GatherArgs a) {
    pdl_trigger();
    pdl_wait();
    const int total = a.off[a.nparts];
    const int per_row = total / 8;
    const long long n = (long long)a.M * per_row;
    const uint4 nan8 = make_uint4(TF_NAN_BF16 * 0x10001u, TF_NAN_BF16 * 0x10001u, TF_NAN_BF16 * 0x10001u,
                                  TF_NAN_BF16 * 0x10001u);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i / per_row);
        const int col = (int)(i % per_row) * 8;
        int h = 0;
#pragma unroll
        for (int p = 1; p < TF_MAX_PARTS; ++p)
            if (p < a.nparts && col >= a.off[p]) h = p;
        const int j = col - a.off[h];
        uint4 v = nan8;
        if (a.part[h]) v = *reinterpret_cast<const uint4 *>(a.part[h] + (long long)m * a.width[h] + j);
        *reinterpret_cast<uint4 *>(a.dst + (long long)m * a.ld_dst + col) = v;
    }
}

// Element-wise form for pitches or widths that are not multiples of 8.
__global__ void gather_scalar_kernel(GatherArgs a) {
    pdl_trigger();
    pdl_wait();
    const int total = a.off[a.nparts];
    const long long n = (long long)a.M * total;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i / total);
        const int col = (int)(i % total);
        int h = 0;
#pragma unroll
        for (int p = 1; p < TF_MAX_PARTS; ++p)
            if (p < a.nparts && col >= a.off[p]) h = p;
        const int j = col - a.off[h];
        a.dst[(long long)m * a.ld_dst + col] =
            a.part[h] ? a.part[h][(long long)m * a.width[h] + j] : (uint16_t)TF_NAN_BF16;
    }
}

cudaError_t launch_gather(const GatherArgs &a, bool vec, cudaStream_t stream) {
    const long long total = (long long)a.M * a.off[a.nparts] / (vec ? 8 : 1);
    if (total == 0) return cudaSuccess;
    long long blocks = (total + 255) / 256;
    if (blocks > kNumSMs * 16) blocks = kNumSMs * 16;
    if (vec) return launch_pdl(gather_vec_kernel, dim3((int)blocks), dim3(256), 0, stream, a);
    return launch_pdl(gather_scalar_kernel, dim3((int)blocks), dim3(256), 0, stream, a);
}

// ---------------------------------------------------------------- argmax --
constexpr int kArgmaxThreads = 256;

__global__ void __launch_bounds__(kArgmaxThreads) argmax_partial_kernel(ArgmaxArgs a) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.y;
    const int b = blockIdx.x;
    const uint16_t *row = a.logits + (long long)m * a.ld;
    const int j0 = b * a.span;
    const int j1 = min(a.n, j0 + a.span);
    uint64_t best = 0;
    if (a.vec) {
        const int jv_end = j0 + ((j1 - j0) / 8) * 8;
        for (int j = j0 + threadIdx.x * 8; j < jv_end; j += kArgmaxThreads * 8) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + j);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                best = umax64(best, cand_key(w[e] & 0xFFFFu, a.id_base + j + 2 * e));
                best = umax64(best, cand_key(w[e] >> 16, a.id_base + j + 2 * e + 1));
            }
        }
        for (int j = jv_end + threadIdx.x; j < j1; j += kArgmaxThreads) best = umax64(best, cand_key(row[j], a.id_base + j));
    } else {
        for (int j = j0 + threadIdx.x; j < j1; j += kArgmaxThreads) best = umax64(best, cand_key(row[j], a.id_base + j));
    }
    best = warp_max64(best);
    __shared__ uint64_t red[kArgmaxThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = best;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint64_t v = threadIdx.x < kArgmaxThreads / 32 ? red[threadIdx.x] : 0ull;
        v = warp_max64(v);
        if (threadIdx.x == 0) a.partial[(long long)m * a.blocks_per_row + b] = v;
    }
}

// One warp per row: max over the row's partial keys, then the word.
__global__ void argmax_final_kernel(ArgmaxArgs a) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (m >= a.M) return;
    const int lane = threadIdx.x & 31;
    uint64_t best = 0;
    for (int b = lane; b < a.blocks_per_row; b += 32) best = umax64(best, a.partial[(long long)m * a.blocks_per_row + b]);
    best = warp_max64(best);
    if (lane == 0) a.words[m] = word_of_key(best, a.logits + (long long)m * a.ld, a.id_base);
}

// Blocks per row: enough CTAs to cover the GPU a few times over for small M,
// at least 2048 elements per block.  The scratch size is derived from it.
int argmax_blocks_per_row(int M, int n) {
    const int by_size = (n + 2047) / 2048;
    int by_grid = (4 * kNumSMs + (M > 0 ? M : 1) - 1) / (M > 0 ? M : 1);
    if (by_grid < 1) by_grid = 1;
    int b = by_size < by_grid ? by_size : by_grid;
    if (b < 1) b = 1;
    if (b > 1024) b = 1024;
    return b;
}

cudaError_t launch_argmax(ArgmaxArgs a, cudaStream_t stream) {
    a.blocks_per_row = argmax_blocks_per_row(a.M, a.n);
    int span = (a.n + a.blocks_per_row - 1) / a.blocks_per_row;
    span = (span + 7) / 8 * 8;
    a.span = span;
    dim3 grid(a.blocks_per_row, a.M);
    const cudaError_t e = launch_pdl(argmax_partial_kernel, grid, dim3(kArgmaxThreads), 0, stream, a);
    if (e != cudaSuccess) return e;
    return launch_pdl(argmax_final_kernel, dim3((a.M + 7) / 8), dim3(256), 0, stream, a);
}

// ------------------------------------------------------------- top two --
// The merged top two of the head (TensorFold PR #1433, step-1 and step-2
// bodies: the session keeps the merged top two for its cross-block tie test).
// Keys are the argmax's (flag, order-preserving value, inverted id), unique per
// element, so a pair (k1 > k2) of the two largest keys is the top two; 0 is an
// empty place.  Two pairs merge into max(a1, b1), max(min(a1, b1), a2, b2).
__device__ __forceinline__ void top2_insert(uint64_t &k1, uint64_t &k2, uint64_t k) {
    if (k > k1) {
        k2 = k1;
        k1 = k;
    } else if (k > k2) {
        k2 = k;
    }
}
__device__ __forceinline__ void top2_merge_pair(uint64_t &k1, uint64_t &k2, uint64_t b1, uint64_t b2) {
    const uint64_t lo = umin64(k1, b1);
    k1 = umax64(k1, b1);
    k2 = umax64(lo, umax64(k2, b2));
}
__device__ __forceinline__ void warp_top2(uint64_t &k1, uint64_t &k2) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t b1 = __shfl_xor_sync(0xFFFFFFFFu, k1, o);
        const uint64_t b2 = __shfl_xor_sync(0xFFFFFFFFu, k2, o);
        top2_merge_pair(k1, k2, b1, b2);
    }
}

__global__ void __launch_bounds__(kArgmaxThreads) top2_partial_kernel(ArgmaxArgs a) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.y;
    const int b = blockIdx.x;
    const uint16_t *row = a.logits + (long long)m * a.ld;
    const int j0 = b * a.span;
    const int j1 = min(a.n, j0 + a.span);
    uint64_t k1 = 0, k2 = 0;
    if (a.vec) {
        const int jv_end = j0 + ((j1 - j0) / 8) * 8;
        for (int j = j0 + threadIdx.x * 8; j < jv_end; j += kArgmaxThreads * 8) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + j);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                top2_insert(k1, k2, cand_key(w[e] & 0xFFFFu, a.id_base + j + 2 * e));
                top2_insert(k1, k2, cand_key(w[e] >> 16, a.id_base + j + 2 * e + 1));
            }
        }
        for (int j = jv_end + threadIdx.x; j < j1; j += kArgmaxThreads) top2_insert(k1, k2, cand_key(row[j], a.id_base + j));
    } else {
        for (int j = j0 + threadIdx.x; j < j1; j += kArgmaxThreads) top2_insert(k1, k2, cand_key(row[j], a.id_base + j));
    }
    warp_top2(k1, k2);
    __shared__ uint64_t red[kArgmaxThreads / 32][2];
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5][0] = k1;
        red[threadIdx.x >> 5][1] = k2;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        k1 = threadIdx.x < kArgmaxThreads / 32 ? red[threadIdx.x][0] : 0ull;
        k2 = threadIdx.x < kArgmaxThreads / 32 ? red[threadIdx.x][1] : 0ull;
        warp_top2(k1, k2);
        if (threadIdx.x == 0) {
            uint64_t *dst = a.partial + ((long long)m * a.blocks_per_row + b) * 2;
            dst[0] = k1;
            dst[1] = k2;
        }
    }
}

// One warp per row: the top two of the row's partial pairs, then the two words.
// A flagged row gives its flagged word twice; an empty second place gives
// TF_TOP2_NONE.
__global__ void top2_final_kernel(ArgmaxArgs a) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (m >= a.M) return;
    const int lane = threadIdx.x & 31;
    uint64_t k1 = 0, k2 = 0;
    for (int b = lane; b < a.blocks_per_row; b += 32) {
        const uint64_t *p = a.partial + ((long long)m * a.blocks_per_row + b) * 2;
        top2_merge_pair(k1, k2, p[0], p[1]);
    }
    warp_top2(k1, k2);
    if (lane == 0) {
        const uint16_t *row = a.logits + (long long)m * a.ld;
        const uint64_t w1 = word_of_key(k1, row, a.id_base);
        uint64_t w2;
        if (k1 >> 63)
            w2 = w1;
        else
            w2 = k2 == 0 ? TF_TOP2_NONE : word_of_key(k2, row, a.id_base);
        a.words[2 * (long long)m] = w1;
        a.words[2 * (long long)m + 1] = w2;
    }
}

cudaError_t launch_top2(ArgmaxArgs a, cudaStream_t stream) {
    a.blocks_per_row = argmax_blocks_per_row(a.M, a.n);
    int span = (a.n + a.blocks_per_row - 1) / a.blocks_per_row;
    span = (span + 7) / 8 * 8;
    a.span = span;
    dim3 grid(a.blocks_per_row, a.M);
    const cudaError_t e = launch_pdl(top2_partial_kernel, grid, dim3(kArgmaxThreads), 0, stream, a);
    if (e != cudaSuccess) return e;
    return launch_pdl(top2_final_kernel, dim3((a.M + 7) / 8), dim3(256), 0, stream, a);
}

// One thread per row: the lowest part whose winner is flagged gives its flagged
// word twice; otherwise the two highest of all the parts' words, compared by
// their argmax keys (the words themselves are carried, so a winning -0 keeps
// its sign).
__device__ __forceinline__ uint64_t key_of_word(uint64_t w) {
    if (w == TF_TOP2_NONE) return 0ull;
    return cand_key((uint32_t)(w & 0xFFFFFFFFull) >> 16, (uint32_t)(w >> 32));
}
__global__ void top2_merge_kernel(const uint64_t *words2, int nparts, int M, uint64_t *out2) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M) return;
    for (int p = 0; p < nparts; ++p) {
        const uint64_t w = words2[((long long)p * M + m) * 2];
        if ((uint32_t)(w >> 32) & TF_PAIR_FLAG) {
            out2[2 * (long long)m] = w;
            out2[2 * (long long)m + 1] = w;
            return;
        }
    }
    uint64_t k1 = 0, k2 = 0, w1 = TF_TOP2_NONE, w2 = TF_TOP2_NONE;
    for (int p = 0; p < nparts; ++p)
        for (int i = 0; i < 2; ++i) {
            const uint64_t w = words2[((long long)p * M + m) * 2 + i];
            const uint64_t k = key_of_word(w);
            if (k > k1) {
                k2 = k1;
                w2 = w1;
                k1 = k;
                w1 = w;
            } else if (k > k2) {
                k2 = k;
                w2 = w;
            }
        }
    out2[2 * (long long)m] = w1;
    out2[2 * (long long)m + 1] = w2;
}

cudaError_t launch_top2_merge(const uint64_t *words2, int nparts, int M, uint64_t *out2, cudaStream_t stream) {
    return launch_pdl(top2_merge_kernel, dim3((M + 127) / 128), dim3(128), 0, stream, words2, nparts, M, out2);

}

// ------------------------------------------------------------------ pick --
// One thread per row: any flagged id word -> the sentinel; otherwise the larger
// value, the lower id on equal values (fp32 compare: +0 == -0).
__global__ void pick_kernel(const uint64_t *words, int nparts, int M, uint32_t *ids) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M) return;
    bool flagged = false;
    uint32_t best_id = 0;
    float best_v = 0.0f;
    for (int p = 0; p < nparts; ++p) {
        const uint64_t w = words[(long long)p * M + m];
        const uint32_t id = (uint32_t)(w >> 32);
        const float v = __uint_as_float((uint32_t)w);
        if (id & TF_PAIR_FLAG) flagged = true;
        if (p == 0 || v > best_v || (v == best_v && id < best_id)) {
            best_id = id;
            best_v = v;
        }
    }
    ids[m] = flagged ? TF_PICK_FAILED : best_id;
}

cudaError_t launch_pick(const uint64_t *words, int nparts, int M, uint32_t *ids, cudaStream_t stream) {
    return launch_pdl(pick_kernel, dim3((M + 127) / 128), dim3(128), 0, stream, words, nparts, M, ids);

}

}  // namespace tf
