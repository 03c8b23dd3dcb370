// qmm_gemv.cu -- 4-bit affine (group 64) quantized GEMV over a slice of rows.
//
// y[m, c] = bf16_RNE( sum_k x[m,k] * (s[n,k/64] q[n,k] + b[n,k/64]) ), fp32
// accumulation, for the whole-matrix rows n the segments list (TensorFold
// PR #1433 step-1 body: each rank reduces its own output rows over the full
// K; PR #1437 Receipt: 4-bit affine, group 64).
//
// Reduction order (fixed by K alone, so a slice reproduces the whole matrix's
// bits -- PR #1433 review, "a different sk is a different fp32 order"):
//   * K is cut into chunks of 1024; in chunk c lane l owns the 32 consecutive
//     k in [1024c + 32l, +32), which lie inside group 16c + l/2.
//   * The lane forms sum of x_k w_k over its 32 k, w_k = s q_k + b in fp32,
//     with two fp32 accumulators (even / odd k, ascending) added at the end,
//     and adds that to its running sum.  (The streaming M = 1 kernels of
//     qmm_stream.cu take the same lane-chunks, lanes and tree with exact
//     integer dot products instead.)
//   * The lane's running sum goes over the chunks in ascending c; the 32 lane
//     sums are then added by a shfl_down tree (16, 8, 4, 2, 1) and lane 0's
//     total is rounded to bf16.
// Nothing in that order depends on which rows a launch covers, where a row sits
// in a segment, or on the grid, so split == whole holds bit for bit.
#include "tf_common.cuh"
#include "tf_kernels.h"
#include "qmm_common.cuh"

namespace tf {

constexpr int kWarps = 8;                // warps per CTA
constexpr int kSlots = 4;                // weight rows a warp carries at once

// Read-once weight stream: bypass L1.
__device__ __forceinline__ uint4 ld_stream_u4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_stream_u16(const uint16_t *p) {
    unsigned short r;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// ---------------------------------------------------------------------------
// M = 1.  x is staged once per CTA into shared memory as fp32, permuted so that
// the float4 holding elements 4j..4j+3 of lane l's 32 in chunk c sits at
// float4 index (c*8 + j)*32 + l: a warp's 128-bit reads are conflict-free.
// Positions past K are zero.
// Each warp walks its own contiguous range of row groups (kSlots rows each);
// the (group, chunk) pairs form one sequence and the codes of step t+1 are
// loaded while step t computes.
// ---------------------------------------------------------------------------
struct StepLoad {
    uint4 q[kSlots];
    uint32_t s[kSlots], b[kSlots];
};

__global__ void __launch_bounds__(kWarps * 32, 2) qmm_m1_kernel(QmmArgs a, int units) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) float smem[];
    const int K = a.K;
    const int nch = (K + kChunk - 1) / kChunk;
    float4 *xs = reinterpret_cast<float4 *>(smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // stage x (row 0) into the permuted fp32 layout
    for (int k = tid; k < nch * kChunk; k += blockDim.x) {
        float v = 0.0f;
        if (k < K) v = bf16_bits_to_f32(a.x[k]);
        const int c = k / kChunk, r = k % kChunk, l = r / 32, e = r % 32;
        smem[(((c * 8 + e / 4) * 32 + l) << 2) + (e & 3)] = v;
    }
    __syncthreads();

    // contiguous, balanced ranges: every warp gets floor or ceil(units / warps)
    const long long gw = (long long)blockIdx.x * kWarps + warp;
    const long long nw = (long long)gridDim.x * kWarps;
    const int u_begin = (int)(gw * units / nw);
    const int u_end = (int)((gw + 1) * units / nw);
    if (u_begin >= u_end) return;

    const int rowbytes = K / 2;
    const int G = K / kGroup;
    const int per_unit = a.glu ? kSlots / 2 : kSlots;   // output columns per unit

    // whole-matrix rows of the four slots of unit u (-1 = unused slot)
    auto slot_rows = [&](int u, int *rows) {
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
            const int col = u * per_unit + (a.glu ? s / 2 : s);
            rows[s] = (col < a.seg.ncols) ? seg_row(a.seg, col, a.glu, a.glu ? (s & 1) : 0) : -1;
        }
    };
    auto load_step = [&](const int *rows, int c, StepLoad &L) {
        const int kk = c * kChunk + lane * 32;
        const bool live = kk < K;
        const int g = kk / kGroup;
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
            if (live && rows[s] >= 0) {
                const size_t r = (size_t)rows[s];
                L.q[s] = ld_stream_u4(a.wq + r * rowbytes + (size_t)(c * (kChunk / 2) + lane * 16));
                L.s[s] = ld_stream_u16(a.scales + r * G + g);
                L.b[s] = ld_stream_u16(a.biases + r * G + g);
            } else {
                L.q[s] = make_uint4(0u, 0u, 0u, 0u);
                L.s[s] = 0u;
                L.b[s] = 0u;
            }
        }
    };

    int u = u_begin, c = 0;
    int rows[kSlots];
    slot_rows(u, rows);
    StepLoad cur, nxt;
    load_step(rows, 0, cur);
    float acc[kSlots];
#pragma unroll
    for (int s = 0; s < kSlots; ++s) acc[s] = 0.0f;

    while (true) {
        // next step's (unit, chunk) and its loads
        int nu = u, ncn = c + 1;
        if (ncn == nch) {
            ncn = 0;
            nu = u + 1;
        }
        int nrows_[kSlots];
        const bool more = nu < u_end;
        if (more) {
            if (nu != u) slot_rows(nu, nrows_);
            else {
#pragma unroll
                for (int s = 0; s < kSlots; ++s) nrows_[s] = rows[s];
            }
            load_step(nrows_, ncn, nxt);
        }

        // compute step (u, c)
        float4 xv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) xv[j] = xs[(c * 8 + j) * 32 + lane];
#pragma unroll
        for (int s = 0; s < kSlots; ++s)
            acc[s] += lane_chunk_wdot(cur.q[s], xv, bf16_bits_to_f32(cur.s[s]), bf16_bits_to_f32(cur.b[s]));

        if (c == nch - 1) {
            // unit u complete: reduce and store
            float tot[kSlots];
#pragma unroll
            for (int s = 0; s < kSlots; ++s) {
                tot[s] = warp_sum_to_lane0(acc[s]);
                acc[s] = 0.0f;
            }
            if (lane == 0) {
                if (a.glu) {
#pragma unroll
                    for (int p = 0; p < kSlots / 2; ++p) {
                        const int col = u * per_unit + p;
                        if (col < a.seg.ncols) {
                            const float g = bf16_bits_to_f32(f32_to_bf16_rne(tot[2 * p]));
                            const float uu = bf16_bits_to_f32(f32_to_bf16_rne(tot[2 * p + 1]));
                            a.y[col] = f32_to_bf16_rne(glu_f32(g, uu));
                        }
                    }
                } else {
#pragma unroll
                    for (int s = 0; s < kSlots; ++s) {
                        const int col = u * per_unit + s;
                        if (col < a.seg.ncols) a.y[col] = f32_to_bf16_rne(tot[s]);
                    }
                }
            }
        }
        if (!more) break;
        u = nu;
        c = ncn;
#pragma unroll
        for (int s = 0; s < kSlots; ++s) rows[s] = nrows_[s];
        cur = nxt;
    }
}

// ---------------------------------------------------------------------------
// Any M (1..128) and any K: the same per-row order, x read straight from
// global memory.  One warp per output column, activation rows in tiles of
// kMT.  Correct everywhere; the fast paths are the M = 1 kernel above and the
// tensor-core kernel for prompt chunks.
// ---------------------------------------------------------------------------
constexpr int kMT = 4;

__device__ __forceinline__ void load_x_lane(const uint16_t *xrow, int k0, int K, float4 *xv) {
    // 32 bf16 at x[k0 .. k0+32) -> 8 float4 (zeros past K)
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        uint4 raw = make_uint4(0u, 0u, 0u, 0u);
        if (k0 + 8 * h < K) raw = *reinterpret_cast<const uint4 *>(xrow + k0 + 8 * h);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        xv[2 * h] = make_float4(__uint_as_float(w[0] << 16), __uint_as_float(w[0] & 0xFFFF0000u),
                                __uint_as_float(w[1] << 16), __uint_as_float(w[1] & 0xFFFF0000u));
        xv[2 * h + 1] = make_float4(__uint_as_float(w[2] << 16), __uint_as_float(w[2] & 0xFFFF0000u),
                                    __uint_as_float(w[3] << 16), __uint_as_float(w[3] & 0xFFFF0000u));
    }
}

__global__ void __launch_bounds__(kWarps * 32) qmm_generic_kernel(QmmArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int nw = gridDim.x * kWarps;
    const int K = a.K, nch = (K + kChunk - 1) / kChunk, rowbytes = K / 2, G = K / kGroup;
    const int nmem = a.glu ? 2 : 1;
    for (int col = gw; col < a.seg.ncols; col += nw) {
        int rows[2];
        rows[0] = seg_row(a.seg, col, a.glu, 0);
        rows[1] = a.glu ? seg_row(a.seg, col, a.glu, 1) : -1;
        for (int m0 = 0; m0 < a.M; m0 += kMT) {
            float acc[2][kMT];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int i = 0; i < kMT; ++i) acc[r][i] = 0.0f;
            for (int c = 0; c < nch; ++c) {
                const int kk = c * kChunk + lane * 32;
                if (kk >= K) continue;
                const int g = kk / kGroup;
                float4 xv[kMT][8];
#pragma unroll
                for (int i = 0; i < kMT; ++i) {
                    if (m0 + i < a.M) load_x_lane(a.x + (size_t)(m0 + i) * a.ldx, kk, K, xv[i]);
                    else
#pragma unroll
                        for (int j = 0; j < 8; ++j) xv[i][j] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    if (r >= nmem) break;
                    const size_t n = (size_t)rows[r];
                    const uint4 q = *reinterpret_cast<const uint4 *>(a.wq + n * rowbytes + (size_t)(c * (kChunk / 2) + lane * 16));
                    const float s = bf16_bits_to_f32(a.scales[n * G + g]);
                    const float b = bf16_bits_to_f32(a.biases[n * G + g]);
#pragma unroll
                    for (int i = 0; i < kMT; ++i) acc[r][i] += lane_chunk_wdot(q, xv[i], s, b);
                }
            }
#pragma unroll
            for (int i = 0; i < kMT; ++i) {
                const float t0 = warp_sum_to_lane0(acc[0][i]);
                const float t1 = warp_sum_to_lane0(acc[1][i]);
                if (lane == 0 && m0 + i < a.M) {
                    uint16_t out;
                    if (a.glu) {
                        const float g = bf16_bits_to_f32(f32_to_bf16_rne(t0));
                        const float uu = bf16_bits_to_f32(f32_to_bf16_rne(t1));
                        out = f32_to_bf16_rne(glu_f32(g, uu));
                    } else {
                        out = f32_to_bf16_rne(t0);
                    }
                    a.y[(size_t)(m0 + i) * a.ldy + col] = out;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
static int g_num_sms[64];
static size_t g_m1_smem_set[64];

static int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    return dev;
}

int num_sms() {
    const int dev = current_device();
    if (g_num_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            g_num_sms[dev] = n;
        else
            g_num_sms[dev] = kNumSMs;
    }
    return g_num_sms[dev];
}

size_t qmm_m1_smem_bytes(int K) {
    const int nch = (K + kChunk - 1) / kChunk;
    return (size_t)nch * kChunk * sizeof(float);
}

constexpr size_t kM1SmemMax = 200 * 1024;

cudaError_t launch_qmm(const QmmArgs &a, cudaStream_t stream) {
    const int ncols = a.seg.ncols;
    if (qmm_m1_stream_eligible(a)) return launch_qmm_m1_stream(a, stream);
    if (qmm_tc_eligible(a)) return launch_qmm_tc(a, stream);
    if (a.M == 1 && qmm_m1_smem_bytes(a.K) <= kM1SmemMax) {
        const size_t smem = qmm_m1_smem_bytes(a.K);
        const int dev = current_device();
        if (smem > 48 * 1024 && g_m1_smem_set[dev] < kM1SmemMax) {
            cudaError_t e = cudaFuncSetAttribute(qmm_m1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kM1SmemMax);
            if (e != cudaSuccess) return e;
            g_m1_smem_set[dev] = kM1SmemMax;
        }
        const int per_unit = a.glu ? kSlots / 2 : kSlots;
        const int units = (ncols + per_unit - 1) / per_unit;
        const int blocks_per_sm = (smem * 2 <= 220 * 1024) ? 2 : 1;
        int blocks = num_sms() * blocks_per_sm;
        const int need = (units + kWarps - 1) / kWarps;
        if (need < blocks) blocks = need;
        return launch_pdl(qmm_m1_kernel, dim3(blocks), dim3(kWarps * 32), smem, stream, a, units);
    }
    int blocks = (ncols + kWarps - 1) / kWarps;
    blocks = min(blocks, num_sms() * 8);
    return launch_pdl(qmm_generic_kernel, dim3(blocks), dim3(kWarps * 32), 0, stream, a);
}

}  // namespace tf
