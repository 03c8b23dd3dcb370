// qmm8.cu -- the int8 head: y = bf16(s[n] * sum_k x[k] q8[n][k]) with int8 codes
// [N][K] and one bf16 scale per row (the b70 lab's runtime INT8 target lm_head
// with a bf16 scale).  At one byte a weight it is a pure HBM stream like the
// 4-bit path, so it uses the same design:
//   * M = 1: each warp owns a ring of shared-memory slots (kRU rows x 1,024 K)
//     refilled by cp.async.bulk, one 1 KB copy per row and step; the codes are
//     bytes already, so dp4a takes them as they are: per 32-code lane-chunk,
//     x in fixed point with the lane-chunk's own exponent (three byte limbs,
//     exact for every x within 2^15 of the lane-chunk's largest), three dp4a
//     per four codes, the integer sum scaled by the exact power of two; lanes
//     add their lane-chunks in K order, a fixed shuffle tree joins the lanes,
//     and the row scale multiplies the total.  A lane-chunk with a nonzero x
//     more than 2^15 below its largest keeps its raw x and is taken by the
//     whole warp in fp32 (lane j forms x_j q_j, exact, a fixed butterfly adds
//     them), so small x are never rounded to the largest one's precision.  The
//     order of every operation depends on K alone, so split == whole bit for bit.
//   * M > 1, or K / pointers the streaming kernel does not take: one warp per
//     output row and activation row, fp32 products of the bf16 x and the code,
//     a per-lane sum over K in order and the same shuffle tree.
#include "qmm_common.cuh"
#include "stream_common.cuh"

namespace tf {

constexpr int k8KS = 1024;                  // K (bytes of a row) per step
constexpr int k8LaneVecs = 6;               // uint4 of limb words per 32-x lane-chunk
constexpr int k8MaxWarps = 20;
constexpr int stages8(int ru) { return ru >= 4 ? 2 : 6; }
constexpr long long k8SpinLimit = 1ll << 22;

__host__ __device__ inline size_t r128(size_t v) { return (v + 127) / 128 * 128; }

struct Stream8Layout {
    int nch;
    size_t limb_off, scale_off, bar_off, ring_off, total;
};

__host__ __device__ inline Stream8Layout stream8_layout(int K, int warps, int ru) {
    Stream8Layout L;
    L.nch = (K + k8KS - 1) / k8KS;
    L.limb_off = 0;
    L.scale_off = r128(L.limb_off + (size_t)L.nch * 32 * k8LaneVecs * 16);
    L.bar_off = r128(L.scale_off + (size_t)L.nch * 32 * 4);
    L.ring_off = r128(L.bar_off + (size_t)warps * stages8(ru) * 8);
    L.total = L.ring_off + (size_t)warps * stages8(ru) * ru * k8KS;
    return L;
}

// 2^(E-23) * sum over the lane's 32 codes of q_k * F_k.  limb vector
// (limb * 2 + (w >> 2)), component w & 3, holds the limb bytes of x[4w .. 4w+3]
// (code word w holds codes 4w .. 4w+3, byte j = code 4w + j).
__device__ __forceinline__ float lane_chunk_idot8(const uint4 &q0, const uint4 &q1, const uint4 *lm, float scale) {
    int a0 = 0, a1 = 0, a2 = 0;
    const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const uint32_t *L = reinterpret_cast<const uint32_t *>(lm);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const int h = w >> 2, c = w & 3;
        asm("dp4a.s32.u32 %0, %1, %2, %0;" : "+r"(a0) : "r"(words[w]), "r"(L[(0 * 2 + h) * 4 + c]));
        asm("dp4a.s32.u32 %0, %1, %2, %0;" : "+r"(a1) : "r"(words[w]), "r"(L[(1 * 2 + h) * 4 + c]));
        asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(a2) : "r"(words[w]), "r"(L[(2 * 2 + h) * 4 + c]));
    }
    return fmaf((float)a2, 65536.0f, fmaf((float)a1, 256.0f, (float)a0)) * scale;   // exact power-of-two scaling
}

template <int kRU>
__global__ void __launch_bounds__(k8MaxWarps * 32, 1) qmm8_m1_stream_kernel(Qmm8Args a, int units) {
    constexpr int kStages = stages8(kRU);
    constexpr int kSlotBytes = kRU * k8KS;
    extern __shared__ __align__(128) uint8_t smem[];
    const int W = blockDim.x >> 5;
    const Stream8Layout L = stream8_layout(a.K, W, kRU);
    const int K = a.K, nch = L.nch;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_trigger();
    uint8_t *limbs = smem + L.limb_off;
    float *Ss = reinterpret_cast<float *>(smem + L.scale_off);
    uint8_t *ring = smem + L.ring_off + (size_t)warp * kStages * kSlotBytes;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar0 = smem_addr(smem + L.bar_off) + (uint32_t)(warp * kStages * 8);

    const long long gw = (long long)blockIdx.x * W + warp;
    const long long nw = (long long)gridDim.x * W;
    const int u0 = (int)(gw * units / nw);
    const int u1 = (int)((gw + 1) * units / nw);
    const int steps = (u1 - u0) * nch;

    // lane r < kRU copies row r of the unit
    auto unit_row = [&](int u, int r) {   // whole-matrix row of unit row r, -1 past the end
        const int col = u * kRU + r;
        return col < a.seg.ncols ? seg_row(a.seg, col, 0, 0) : -1;
    };
    int iu = u0, ij = 0, it_ = 0;
    int my_row = lane < kRU && u0 < u1 ? unit_row(u0, lane) : -1;
    int live = u0 < u1 ? min(kRU, a.seg.ncols - u0 * kRU) : 0;
    auto issue_next = [&]() {
        const int slot = it_ % kStages;
        const int k0 = ij * k8KS, len = min(k8KS, K - k0);
        const uint32_t bar = bar0 + 8 * slot;
        if (lane == 0) mbar_expect_tx(bar, (uint32_t)(live * len));
        __syncwarp();
        if (my_row >= 0)
            bulk_g2s(ring_s + slot * kSlotBytes + lane * k8KS, a.q8 + (size_t)my_row * K + k0, (uint32_t)len, bar);
        if (++ij == nch) {
            ij = 0;
            if (++iu < u1) {
                my_row = lane < kRU ? unit_row(iu, lane) : -1;
                live = min(kRU, a.seg.ncols - iu * kRU);
            }
        }
        ++it_;
    };

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    for (int t = 0; t < kStages && t < steps; ++t) issue_next();

    // fixed-point limbs of x, one warp per lane-chunk, one lane per value, from the
    // bf16 fields: x = sign * M * 2^(e-134) (M = 128 + mantissa, or the mantissa with
    // e read as 1 for subnormals); with emax the lane-chunk's largest e,
    // F = x * 2^(23-E), E = emax - 126, is sign * M * 2^(e - emax + 15), a left shift
    // when e >= emax - 15 (exact), else a right shift rounded to nearest even.
    // (loads go out eight lane-chunks at a time: one L2 round trip covers all eight)
    constexpr int kPrep = 8;
    for (int lc0 = warp; lc0 < nch * 32; lc0 += W * kPrep) {
      uint32_t hb[kPrep];
#pragma unroll
      for (int i = 0; i < kPrep; ++i) {
          const int lc = lc0 + i * W;
          const int k = (lc >> 5) * k8KS + (lc & 31) * 32 + lane;
          hb[i] = (lc < nch * 32 && k < K) ? (uint32_t)a.x[k] : 0u;
      }
#pragma unroll
      for (int i = 0; i < kPrep; ++i) {
        const int lc = lc0 + i * W;
        if (lc >= nch * 32) break;
        const int c = lc >> 5, l = lc & 31;
        const uint32_t h = hb[i];
        const uint32_t ef = (h >> 7) & 0xFFu;
        const bool bad = __any_sync(0xFFFFFFFFu, ef == 0xFFu);
        const int e = ef == 0 ? 1 : (int)ef;
        const int M = ef == 0 ? (int)(h & 0x7Fu) : (int)(0x80u | (h & 0x7Fu));
        const int emax = __reduce_max_sync(0xFFFFFFFFu, M != 0 ? e : 0);
        const int sh = e - emax + 15;
        // wide: a nonzero x more than 2^15 below the largest, which fixed point would
        // round; such a lane-chunk keeps its raw x and is taken in fp32 below
        const bool wide = !bad && __any_sync(0xFFFFFFFFu, sh < 0 && M != 0);
        int F = sh >= 0 ? M << sh : 0;
        if (h & 0x8000u) F = -F;
        if (bad) F = 0;
        const int w = lane >> 2, byte = lane & 3;   // element `lane` of the lane-chunk: word w, byte j
        uint8_t *lcb = limbs + ((size_t)(c * k8LaneVecs) * 32 + l) * 16;
        if (wide) {
            // value j in 16-byte vector j / 8 of the lane-chunk
            reinterpret_cast<uint16_t *>(lcb + (size_t)(lane >> 3) * 32 * 16)[lane & 7] = (uint16_t)h;
        } else {
            uint8_t *base = lcb + (w & 3) * 4 + byte;
#pragma unroll
            for (int lb = 0; lb < 3; ++lb) base[(size_t)(lb * 2 + (w >> 2)) * 32 * 16] = (uint8_t)((F >> (8 * lb)) & 0xFF);
        }
        if (lane == 0)
            Ss[lc] = bad ? __int_as_float(0x7FC00000)
                         : (wide ? __int_as_float(0x80000000)
                                 : (emax >= 23 ? __int_as_float((emax - 22) << 23) : ldexpf(1.0f, emax - 149)));
      }
    }
    __syncthreads();

    float acc[kRU];
#pragma unroll
    for (int r = 0; r < kRU; ++r) acc[r] = 0.0f;
    int u = u0, j = 0, slot = 0;
    uint32_t par = 0;
    bool failed = false;
    const uint4 *limb_l = reinterpret_cast<const uint4 *>(limbs) + lane;
    for (int t = 0; t < steps; ++t) {
        const bool ok = __all_sync(0xFFFFFFFFu, wait_slot(bar0 + 8 * slot, par, failed ? 64 : k8SpinLimit));
        failed = failed || !ok;
        const uint8_t *sl = ring + slot * kSlotBytes;
        // lanes past the end of a short last step idle; a wide lane-chunk (scale -0)
        // adds nothing here and is taken element by element below
        const bool live = j * k8KS + lane * 32 < K;
        const float scale = live ? Ss[j * 32 + lane] : 0.0f;
        const uint32_t wm = __ballot_sync(0xFFFFFFFFu, live && __float_as_uint(scale) == 0x80000000u);
        if (live) {
            uint4 lm[k8LaneVecs];
#pragma unroll
            for (int q = 0; q < k8LaneVecs; ++q) lm[q] = limb_l[(j * k8LaneVecs + q) * 32];
#pragma unroll
            for (int r = 0; r < kRU; ++r) {
                const uint4 *qp = reinterpret_cast<const uint4 *>(sl + r * k8KS) + 2 * lane;
                acc[r] += lane_chunk_idot8(qp[0], qp[1], lm, scale);
            }
        }
        for (uint32_t m = wm; m != 0; m &= m - 1) {   // wide lane-chunks, warp-uniform
            const int l = __ffs(m) - 1;
            const uint16_t *xv = reinterpret_cast<const uint16_t *>(
                limbs + ((size_t)(j * k8LaneVecs + (lane >> 3)) * 32 + l) * 16);
            const float xj = bf16_bits_to_f32(xv[lane & 7]);
#pragma unroll
            for (int r = 0; r < kRU; ++r) {
                // lane t takes code t of the lane-chunk: x q in fp32 (exact), then a
                // butterfly adds the 32 products in a fixed order
                float p = xj * (float)reinterpret_cast<const int8_t *>(sl + r * k8KS)[l * 32 + lane];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xFFFFFFFFu, p, o);
                if (lane == l) acc[r] += p;
            }
        }
        if (++j == nch) {
            float tot[kRU];
#pragma unroll
            for (int r = 0; r < kRU; ++r) {
                tot[r] = warp_sum_to_lane0(acc[r]);
                acc[r] = 0.0f;
            }
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < kRU; ++r) {
                    const int col = u * kRU + r;
                    if (col < a.seg.ncols) {
                        const float s = bf16_bits_to_f32(__ldg(a.scales + seg_row(a.seg, col, 0, 0)));
                        a.y[col] = failed ? (uint16_t)TF_NAN_BF16 : f32_to_bf16_rne(s * tot[r]);
                    }
                }
            }
            j = 0;
            ++u;
        }
        if (++slot == kStages) {
            slot = 0;
            par ^= 1u;
        }
        __syncwarp();
        if (it_ < steps && !failed) issue_next();
    }
    if (failed)
        for (int s2 = 0; s2 < kStages; ++s2) wait_slot(bar0 + 8 * s2, 0, 1024);
}

// M > 1 (or a layout the streaming kernel does not take): one warp per output
// column and activation row; lanes take every 32nd k, add in K order, the same
// shuffle tree joins them, the row scale multiplies the total.
__global__ void qmm8_generic_kernel(Qmm8Args a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const long long task = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long ntask = (long long)a.M * a.seg.ncols;
    for (long long tk = task; tk < ntask; tk += (long long)gridDim.x * (blockDim.x >> 5)) {
        const int m = (int)(tk / a.seg.ncols), col = (int)(tk % a.seg.ncols);
        const int row = seg_row(a.seg, col, 0, 0);
        const int8_t *q = a.q8 + (size_t)row * a.K;
        const uint16_t *x = a.x + (size_t)m * a.ldx;
        float acc = 0.0f;
        for (int k = lane; k < a.K; k += 32) acc = fmaf(bf16_bits_to_f32(x[k]), (float)q[k], acc);
        acc = warp_sum_to_lane0(acc);
        if (lane == 0) a.y[(size_t)m * a.ldy + col] = f32_to_bf16_rne(bf16_bits_to_f32(a.scales[row]) * acc);
    }
}

static int stream8_warps(int K, int ru) {
    for (int w = k8MaxWarps; w >= 4; --w)
        if (stream8_layout(K, w, ru).total <= 227 * 1024) return w;
    return 0;
}

static bool g_q8_smem_set[64][2];

template <int RU>
static cudaError_t launch_q8(const Qmm8Args &a, int ri, cudaStream_t stream) {
    const int W = stream8_warps(a.K, RU);
    const Stream8Layout L = stream8_layout(a.K, W, RU);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!g_q8_smem_set[dev][ri]) {
        const cudaError_t e = cudaFuncSetAttribute(qmm8_m1_stream_kernel<RU>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        g_q8_smem_set[dev][ri] = true;
    }
    const int units = (a.seg.ncols + RU - 1) / RU;
    int blocks = num_sms();
    const int need = (units + W - 1) / W;
    if (need < blocks) blocks = need;
    return launch_pdl(qmm8_m1_stream_kernel<RU>, dim3(blocks), dim3(W * 32), L.total, stream, a, units);
}

cudaError_t launch_qmm8(const Qmm8Args &a, cudaStream_t stream) {
    // the streaming kernel needs 16-byte rows and a 16-byte aligned code array for its
    // copies, whole 32-code lane-chunks, and its layout in shared memory
    const bool stream_ok = a.M == 1 && a.K % 32 == 0 && aligned(a.q8, 16) && stream8_warps(a.K, 4) > 0 &&
                           stream8_warps(a.K, 1) > 0;
    if (stream_ok) {
        // rows per unit only change how often a lane reuses its limbs, never a row's arithmetic
        const long long warps = (long long)num_sms() * stream8_warps(a.K, 4);
        if (a.seg.ncols >= 8 * warps) return launch_q8<4>(a, 0, stream);
        return launch_q8<1>(a, 1, stream);
    }
    long long blocks = ((long long)a.M * a.seg.ncols + 7) / 8;
    if (blocks > num_sms() * 16) blocks = num_sms() * 16;
    if (blocks < 1) blocks = 1;
    return launch_pdl(qmm8_generic_kernel, dim3((int)blocks), dim3(256), 0, stream, a);
}

}  // namespace tf
