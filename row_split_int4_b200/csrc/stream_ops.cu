// stream_ops.cu -- the steps on either side of the seam: the fp32 residual add of
// a gathered bf16 row, and the whole-table embedding gather.
//
// Both are pure HBM streams (no reuse): 10 bytes per element for the add (read
// the fp32 stream and the bf16 row, write the stream) and 4 bytes per element
// for the embedding rows (read the table row, write the output row), moved in
// 16-byte vectors when the pointers and leading dimensions allow, with grids
// sized in multiples of the SM count.
#include "tf_common.cuh"
#include "tf_kernels.h"

namespace tf {

// h[m][j] = fp32(h[m][j] + y[m][j]): one rounding, the IEEE fp32 addition.
// Vector path: eight elements a thread (two float4 of h, one uint4 of y).
__global__ void residual_add_vec_kernel(float *h, long long ld_h, const uint16_t *y, long long ld_y, int M, int n) {
    pdl_trigger();
    pdl_wait();
    const int n8 = n / 8;
    const long long total = (long long)M * n8;
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < total; v += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(v / n8), j = (int)(v % n8) * 8;
        float4 *hp = reinterpret_cast<float4 *>(h + m * ld_h + j);
        const uint4 yv = *reinterpret_cast<const uint4 *>(y + m * ld_y + j);
        float4 a = hp[0], b = hp[1];
        a.x = __fadd_rn(a.x, __uint_as_float(yv.x << 16));
        a.y = __fadd_rn(a.y, __uint_as_float(yv.x & 0xFFFF0000u));
        a.z = __fadd_rn(a.z, __uint_as_float(yv.y << 16));
        a.w = __fadd_rn(a.w, __uint_as_float(yv.y & 0xFFFF0000u));
        b.x = __fadd_rn(b.x, __uint_as_float(yv.z << 16));
        b.y = __fadd_rn(b.y, __uint_as_float(yv.z & 0xFFFF0000u));
        b.z = __fadd_rn(b.z, __uint_as_float(yv.w << 16));
        b.w = __fadd_rn(b.w, __uint_as_float(yv.w & 0xFFFF0000u));
        hp[0] = a;
        hp[1] = b;
    }
    // the ragged tail of each row (n % 8 elements), one element a thread
    const int tail = n - n8 * 8;
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < (long long)M * tail;
         v += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(v / tail), j = n8 * 8 + (int)(v % tail);
        h[m * ld_h + j] = __fadd_rn(h[m * ld_h + j], bf16_bits_to_f32(y[m * ld_y + j]));
    }
}

__global__ void residual_add_scalar_kernel(float *h, long long ld_h, const uint16_t *y, long long ld_y, int M, int n) {
    pdl_trigger();
    pdl_wait();
    const long long total = (long long)M * n;
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < total; v += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(v / n), j = (int)(v % n);
        h[m * ld_h + j] = __fadd_rn(h[m * ld_h + j], bf16_bits_to_f32(y[m * ld_y + j]));
    }
}

cudaError_t launch_residual_add(float *h, long long ld_h, const uint16_t *y, long long ld_y, int M, int n, bool vec,
                                cudaStream_t stream) {
    const long long work = vec ? (long long)M * (n / 8 + n % 8) : (long long)M * n;
    long long blocks = (work + 255) / 256;
    const long long cap = (long long)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (vec) return launch_pdl(residual_add_vec_kernel, dim3((int)blocks), dim3(256), 0, stream, h, ld_h, y, ld_y, M, n);
    return launch_pdl(residual_add_scalar_kernel, dim3((int)blocks), dim3(256), 0, stream, h, ld_h, y, ld_y, M, n);
}

// out[m][:H] = table[ids[m]][:H] for ids below the bound, else the bf16 NaN.
// One CTA per output row (grid-strided), 16-byte vectors when aligned.
__global__ void embed_rows_kernel(const uint16_t *table, long long ld_table, uint32_t bound, int H, const uint32_t *ids,
                                  int M, uint16_t *out, long long ld_out, int vec) {
    pdl_trigger();
    pdl_wait();
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const uint32_t id = ids[m];
        uint16_t *dst = out + m * ld_out;
        if (id >= bound) {
            for (int j = threadIdx.x; j < H; j += blockDim.x) dst[j] = (uint16_t)TF_NAN_BF16;
            continue;
        }
        const uint16_t *src = table + (long long)id * ld_table;
        if (vec) {
            const int h8 = H / 8;
            for (int j = threadIdx.x; j < h8; j += blockDim.x)
                reinterpret_cast<uint4 *>(dst)[j] = reinterpret_cast<const uint4 *>(src)[j];
            for (int j = h8 * 8 + threadIdx.x; j < H; j += blockDim.x) dst[j] = src[j];
        } else {
            for (int j = threadIdx.x; j < H; j += blockDim.x) dst[j] = src[j];
        }
    }
}

cudaError_t launch_embed_rows(const uint16_t *table, long long ld_table, uint32_t bound, int H, const uint32_t *ids,
                              int M, uint16_t *out, long long ld_out, bool vec, cudaStream_t stream) {
    int blocks = M < num_sms() * 8 ? M : num_sms() * 8;
    if (blocks < 1) blocks = 1;
    return launch_pdl(embed_rows_kernel, dim3(blocks), dim3(256), 0, stream, table, ld_table, bound, H, ids, M, out, ld_out, vec ? 1 : 0);
}

}  // namespace tf
