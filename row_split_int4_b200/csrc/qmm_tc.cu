// qmm_tc.cu -- prompt-chunk qmm (M = 2..128 activation rows) on the 5th-generation
// tensor cores: tcgen05.mma with the weights dequantised into tensor memory (the
// A operand), the activations in shared memory (the B operand) and the fp32
// accumulator in tensor memory.
//
// A tile is 128 weight rows (the MMA's M) against all M activation rows of the
// call (the MMA's N, rounded up to a multiple of 16; the extra rows are zero).
// A tile never straddles two segments of the call; with TF_EPI_GLU its rows
// 0-63 are gate rows and 64-127 the up rows of the same outputs.
//
// The K loop runs in stages of 64 values (one scale group):
//   * warp 0, one thread: per stage one TMA copy of the activation tile [N x 64]
//     (128-byte swizzle) and two of the tile's packed codes [2 x 64 rows x 32 B]
//     into a four-deep ring in shared memory.  No multicast.
//   * warps 2-5, one thread per weight row (= tensor-memory lane): take the
//     row's 64 codes from the ring and its scale and bias (loaded eight groups
//     at a time, one period ahead), form w = s*q + b in fp32, split it into two
//     bf16, hi = RN(w) and lo = RN(w - hi), and store both into one of two
//     A stages in tensor memory (tcgen05.st).  hi + lo carries w's 16
//     significant bits, so the contraction sees the weights of the 4-bit format,
//     not a rounded copy of them.
//   * warp 1, one thread: tcgen05.mma kind::f16 with A in tensor memory, four
//     K=16 steps per stage, each on hi and then on lo, into one accumulator;
//     tcgen05.commit releases the ring slot and the A stage.
//
// Split K.  The stages are cut into `ks` slices, given to the `ks` CTAs of one
// thread-block cluster; ks and the cut are functions of K and of the whole
// matrix's row count only (never of M, of the segments, or of the device), so a
// row's result does not depend on which call or which half computes it.  Each
// CTA moves its accumulator to shared memory; after a cluster barrier CTA r
// reads the partial sums of all CTAs of the cluster through distributed shared
// memory for its share of the activation rows, adds them in rank order in fp32,
// rounds to bf16 (and applies gate*SiLU(up) with TF_EPI_GLU), and writes y.
//
// Every wait on an mbarrier is bounded; a wait that gives up marks the CTA
// failed, and every output the cluster writes becomes NaN.  All threads still
// reach both cluster barriers, and tensor memory is released before exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "qmm_common.cuh"

namespace tf {

constexpr int kTcRows = 128;       // weight rows per tile (MMA M)
constexpr int kTcK = 64;           // K per stage
constexpr int kTcRing = 4;         // activation + code ring depth
constexpr int kTcAStages = 2;      // A stages in tensor memory
constexpr int kTcThreads = 192;    // 6 warps
constexpr int kTcMaxN = 128;       // activation rows per call
constexpr int kTcMaxSplit = 8;     // CTAs per cluster
constexpr int kTcXBytes = kTcMaxN * kTcK * 2;       // 16 KB
constexpr int kTcCBytes = kTcRows * kTcK / 2;       // 4 KB of codes
constexpr int kTcSlot = kTcXBytes + kTcCBytes;      // 20 KB, a multiple of 1 KB
constexpr int kTcRingBytes = kTcRing * kTcSlot;     // 80 KB; later the partial sums
constexpr int kTcSmem = kTcRingBytes + 256 /* barriers, flag */ + 1024 /* alignment */;
constexpr uint32_t kTcTmemCols = 256;              // accumulator 128 + 2 x (hi 32 + lo 32)
constexpr long long kTcSpin = 1ll << 24;
static_assert(kTcMaxN * kTcRows * 4 <= kTcRingBytes, "partial sums must fit in the ring");

// Plan of one launch, computed on the host.
struct TcPlan {
    int ks;                        // CTAs per cluster (K slices)
    int periods;                   // K / 512: eight stages each
    int n_mma;                     // MMA N
    int ntiles;
    int tstart[TF_MAX_SEGS + 1];   // first tile of each segment (TF_EPI_NONE)
};

// ------------------------------------------------------------ PTX helpers --
__device__ __forceinline__ uint32_t tc_smem(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void tc_mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void tc_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Bounded wait for the phase `parity` of `bar` to complete; gives up after
// `limit` polls, or early once another thread of the CTA has marked it failed.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int *fail, long long limit = kTcSpin) {
    for (long long it = 0; it < limit; ++it) {
        uint32_t ok;
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
                     : "=r"(ok)
                     : "r"(bar), "r"(parity)
                     : "memory");
        if (ok) return true;
        if ((it & 1023) == 1023 && *fail) return false;
    }
    return false;
}
__device__ __forceinline__ void tc_tma_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t tc_cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t tc_mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ float tc_ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ int tc_ld_cluster_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row core groups
// 1,024 bytes apart (SBO), version 1, no base offset.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                          // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset
    d |= (uint64_t)1u << 46;                          // descriptor version
    d |= (uint64_t)2u << 61;                          // 128-byte swizzle
    return d;
}
// Instruction descriptor: bf16 A and B, fp32 D, both K-major, M = 128, N = n.
__host__ __device__ __forceinline__ uint32_t tc_idesc(int n) {
    uint32_t d = 0;
    d |= 1u << 4;                          // D format f32
    d |= 1u << 7;                          // A format bf16
    d |= 1u << 10;                         // B format bf16
    d |= (uint32_t)(n >> 3) << 17;         // N / 8
    d |= (uint32_t)(kTcRows >> 4) << 24;   // M / 16
    return d;
}
// D[tmem] (+)= A[tmem] * B[smem]^T
__device__ __forceinline__ void tc_mma_ts(uint32_t dtm, uint32_t atm, uint64_t b, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(dtm),
        "r"(atm), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t *r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Two fp32 -> packed bf16x2 (first argument in the low half), round to nearest even.
__device__ __forceinline__ uint32_t tc_pack_bf16(float lo_half, float hi_half) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi_half), "f"(lo_half));
    return r;
}

// 8 codes of a word -> the hi and lo bf16 pairs of w = s*q + b (element 2p in
// the low half of pair p).  hi = RN(w); w - hi is exact in fp32 and lo = RN(w - hi).
__device__ __forceinline__ void tc_dequant8(uint32_t word, float s, float b, uint32_t *hi, uint32_t *lo) {
    const Codes8 c = decode8(word);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float w0 = fmaf(s, c.f[2 * p], b), w1 = fmaf(s, c.f[2 * p + 1], b);
        hi[p] = tc_pack_bf16(w0, w1);
        lo[p] = tc_pack_bf16(w0 - __uint_as_float(hi[p] << 16), w1 - __uint_as_float(hi[p] & 0xFFFF0000u));
    }
}

// bf16 number j (0..7) of a 16-byte vector, compile-time j.
template <int j>
__device__ __forceinline__ float tc_pick_bf16(const uint4 &v) {
    const uint32_t w = (j >> 1) == 0 ? v.x : (j >> 1) == 1 ? v.y : (j >> 1) == 2 ? v.z : v.w;
    return __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// Dequantise one stage (group g) of this thread's row into A stage `acol` of its lane.
template <int j>
__device__ __forceinline__ void tc_stage_dequant(const uint4 &q0, const uint4 &q1, const uint4 &s8, const uint4 &b8,
                                                 uint32_t taddr) {
    const float sf = tc_pick_bf16<j>(s8), bf = tc_pick_bf16<j>(b8);
    uint32_t hi[32], lo[32];
    const uint32_t words[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) tc_dequant8(words[c], sf, bf, hi + 4 * c, lo + 4 * c);
    tc_st32(taddr, hi);
    tc_st32(taddr + 32, lo);
}

__global__ void __launch_bounds__(kTcThreads, 2)
    qmm_tc_kernel(QmmArgs a, const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap, TcPlan plan) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *ring = smem;                                            // [slot][x | codes], later partial sums
    float *part = reinterpret_cast<float *>(smem);                   // [n_mma][128] fp32
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kTcRingBytes);
    // bars: full[R], xfree[R], cfree[R], afull[A], aempty[A], acc_full; then the TMEM address and the flag
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * kTcRing + 2 * kTcAStages + 1);
    volatile int *fail = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ks = plan.ks;
    const int rank = (int)tc_cluster_rank();
    const int tile = blockIdx.x / ks;
    const int p0 = rank * plan.periods / ks, p1 = (rank + 1) * plan.periods / ks;
    const int i0 = 8 * p0, nst = 8 * (p1 - p0);          // this CTA's stages [i0, i0 + nst)
    const uint32_t bar_s = tc_smem(bars);
    auto full = [=](int s) { return bar_s + 8u * s; };
    auto xfree = [=](int s) { return bar_s + 8u * (kTcRing + s); };
    auto cfree = [=](int s) { return bar_s + 8u * (2 * kTcRing + s); };
    auto afull = [=](int s) { return bar_s + 8u * (3 * kTcRing + s); };
    auto aempty = [=](int s) { return bar_s + 8u * (3 * kTcRing + kTcAStages + s); };
    const uint32_t acc_full = bar_s + 8u * (3 * kTcRing + 2 * kTcAStages);

    // The tile's rows: box A (tile rows 0-63) and box B (64-127) of the whole
    // matrix, how many of each box are valid, and the output column of tile row 0.
    int rowA, rowB, validA, validB, col_base;
    if (a.glu) {
        rowA = a.seg.row0[0] + 64 * tile;
        rowB = a.seg.row0[1] + 64 * tile;
        validA = validB = min(64, a.seg.ncols - 64 * tile);
        col_base = 64 * tile;
    } else {
        // the segment holding this tile (unrolled, so the parameter arrays are not indexed at run time)
        int tfirst = 0, nr = 0, r0 = 0, c0 = 0;
#pragma unroll
        for (int j = 0; j < TF_MAX_SEGS; ++j)
            if (j < a.seg.nseg && tile >= plan.tstart[j]) {
                tfirst = plan.tstart[j];
                nr = a.seg.nrows[j];
                r0 = a.seg.row0[j];
                c0 = a.seg.col0[j];
            }
        const int local = tile - tfirst;
        const int nv = min(kTcRows, nr - kTcRows * local);
        rowA = r0 + kTcRows * local;
        rowB = rowA + 64;
        validA = min(64, nv);
        validB = nv - validA;
        col_base = c0 + kTcRows * local;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcRing; ++s) {
            tc_mbar_init(full(s), 1);
            tc_mbar_init(xfree(s), 1);
            tc_mbar_init(cfree(s), 4);
        }
        for (int s = 0; s < kTcAStages; ++s) {
            tc_mbar_init(afull(s), 4);
            tc_mbar_init(aempty(s), 1);
        }
        tc_mbar_init(acc_full, 1);
        *fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(tmem_slot)),
                     "r"(kTcTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_mma = plan.n_mma;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0) {
            const uint32_t bytes = (uint32_t)n_mma * kTcK * 2 + kTcCBytes;
            int issued = 0;
            for (int li = 0; li < nst; ++li) {
                const int s = li % kTcRing;
                if (li >= kTcRing) {
                    const uint32_t par = ((li / kTcRing) - 1) & 1;
                    if (!tc_wait(xfree(s), par, fail) || !tc_wait(cfree(s), par, fail)) { *fail = 1; break; }
                }
                if (*fail) break;
                const int i = i0 + li;
                const uint32_t slot = tc_smem(ring + s * kTcSlot);
                tc_expect_tx(full(s), bytes);
                tc_tma_2d(slot, &xmap, i * kTcK, 0, full(s));
                tc_tma_2d(slot + kTcXBytes, &cmap, i * (kTcK / 2), rowA, full(s));
                tc_tma_2d(slot + kTcXBytes + kTcCBytes / 2, &cmap, i * (kTcK / 2), rowB, full(s));
                issued = li + 1;
            }
            // every copy issued must land before the ring is reused or the CTA exits
            for (int li = issued - kTcRing; li < issued; ++li)
                if (li >= 0) tc_wait(full(li % kTcRing), (li / kTcRing) & 1, fail, 1 << 16);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t idesc = tc_idesc(n_mma);
            for (int li = 0; li < nst; ++li) {
                const int s = li % kTcRing, sa = li % kTcAStages;
                if (!tc_wait(full(s), (li / kTcRing) & 1, fail) || !tc_wait(afull(sa), (li / kTcAStages) & 1, fail)) {
                    *fail = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t xb = tc_smem(ring + s * kTcSlot);
                const uint32_t ahi = tmem + 128u + 64u * sa, alo = ahi + 32u;
#pragma unroll
                for (int kk = 0; kk < kTcK / 16; ++kk) {
                    const uint64_t db = tc_desc(xb + kk * 32);
                    tc_mma_ts(tmem, ahi + 8 * kk, db, idesc, (li > 0 || kk > 0) ? 1u : 0u);
                    tc_mma_ts(tmem, alo + 8 * kk, db, idesc, 1u);
                }
                tc_commit(xfree(s));
                tc_commit(aempty(sa));
            }
            tc_commit(acc_full);
        }
    } else {
        // ---------------------------------------------------------------- dequant
        const int q = warp & 3;                        // TMEM lane quarter of this warp
        const int t = 32 * q + lane;                   // tile row == TMEM lane
        const int G = a.K / kGroup;
        const bool valid = t < 64 ? t < validA : (t - 64) < validB;
        const int row = t < 64 ? rowA + t : rowB + (t - 64);
        const uint16_t *srow = valid ? a.scales + (size_t)row * G : nullptr;
        const uint16_t *brow = valid ? a.biases + (size_t)row * G : nullptr;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + 128u;
        uint4 s8 = make_uint4(0, 0, 0, 0), b8 = s8, sn = s8, bn = s8;
        if (srow) {
            s8 = __ldg(reinterpret_cast<const uint4 *>(srow + 8 * p0));
            b8 = __ldg(reinterpret_cast<const uint4 *>(brow + 8 * p0));
        }
        int li = 0;
        for (int p = p0; p < p1 && !*fail; ++p) {
            if (srow && p + 1 < p1) {   // next period's eight scales and biases
                sn = __ldg(reinterpret_cast<const uint4 *>(srow + 8 * (p + 1)));
                bn = __ldg(reinterpret_cast<const uint4 *>(brow + 8 * (p + 1)));
            }
#define TC_STAGE(J)                                                                                                  \
    {                                                                                                                \
        const int s = li % kTcRing, sa = li % kTcAStages;                                                            \
        bool ok = tc_wait(full(s), (li / kTcRing) & 1, fail);                                                        \
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;                                                                  \
        if (ok) {                                                                                                    \
            const uint4 *src = reinterpret_cast<const uint4 *>(ring + s * kTcSlot + kTcXBytes + 32 * t);             \
            q0 = src[0];                                                                                             \
            q1 = src[1];                                                                                             \
        }                                                                                                            \
        __syncwarp();                                                                                                \
        if (lane == 0) tc_arrive(cfree(s));                                                                          \
        if (ok && li >= kTcAStages) ok = tc_wait(aempty(sa), ((li / kTcAStages) - 1) & 1, fail);                     \
        if (!ok) *fail = 1;                                                                                          \
        if (__any_sync(0xFFFFFFFFu, !ok)) break;                                                                     \
        tc_fence_after();                                                                                            \
        tc_stage_dequant<J>(q0, q1, s8, b8, lane_base + 64u * sa);                                                     \
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");                                                \
        tc_fence_before();                                                                                           \
        __syncwarp();                                                                                                \
        if (lane == 0) tc_arrive(afull(sa));                                                                         \
        ++li;                                                                                                        \
    }
            do {
                TC_STAGE(0) TC_STAGE(1) TC_STAGE(2) TC_STAGE(3) TC_STAGE(4) TC_STAGE(5) TC_STAGE(6) TC_STAGE(7)
            } while (0);
#undef TC_STAGE
            s8 = sn;
            b8 = bn;
        }
        // ---- accumulator -> shared memory, as part[m][t]
        bool ok = !*fail && tc_wait(acc_full, 0, fail);
        if (!ok) *fail = 1;
        ok = __all_sync(0xFFFFFFFFu, ok);
        tc_fence_after();
        if (ok) {
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16);
            for (int c0 = 0; c0 < n_mma; c0 += 16) {
                uint32_t r[16];
                tc_ld16(taddr + c0, r);
#pragma unroll
                for (int j = 0; j < 16; ++j) part[(c0 + j) * kTcRows + t] = __uint_as_float(r[j]);
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    tc_cluster_sync();   // every partial sum and failure flag of the cluster is in place

    if (warp >= 2) {
        const int t = 32 * (warp & 3) + lane;
        int bad = 0;
        for (int j = 0; j < ks; ++j) bad |= tc_ld_cluster_s32(tc_mapa(tc_smem((const void *)fail), j));
        const int mper = (a.M + ks - 1) / ks;
        const int m0 = rank * mper, m1 = min(a.M, m0 + mper);
        const uint32_t pbase = tc_smem(part);
        auto total = [=](int m, int r) {   // partial sums of tile row r, activation row m, in rank order
            const uint32_t off = pbase + (uint32_t)(m * kTcRows + r) * 4u;
            float acc = tc_ld_cluster_f32(tc_mapa(off, 0));
            for (int j = 1; j < ks; ++j) acc += tc_ld_cluster_f32(tc_mapa(off, j));
            return acc;
        };
        if (a.glu) {
            const int pr = t & 63;
            if (pr < validA) {
                for (int m = m0 + (t >> 6); m < m1; m += 2) {
                    uint16_t out = (uint16_t)TF_NAN_BF16;
                    if (!bad) {
                        const float g = bf16_bits_to_f32(f32_to_bf16_rne(total(m, pr)));
                        const float u = bf16_bits_to_f32(f32_to_bf16_rne(total(m, pr + 64)));
                        out = f32_to_bf16_rne(glu_f32(g, u));
                    }
                    a.y[(size_t)m * a.ldy + col_base + pr] = out;
                }
            }
        } else if (t < validA + validB) {
            for (int m = m0; m < m1; ++m)
                a.y[(size_t)m * a.ldy + col_base + t] = bad ? (uint16_t)TF_NAN_BF16 : f32_to_bf16_rne(total(m, t));
        }
    }
    __syncwarp();
    tc_cluster_sync();   // no CTA leaves while another still reads its shared memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
    }
}

// ------------------------------------------------------------------ host --
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

static cudaError_t get_encode() {
    if (g_encode) return cudaSuccess;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return e != cudaSuccess ? e : cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return cudaSuccess;
}

// K slices per tile: from K and the whole matrix's row count alone.  The whole
// matrix should give about 512 CTAs; a slice keeps at least four periods of
// eight stages unless the periods divide evenly.
int qmm_tc_split(int K, int n_whole) {
    const int periods = K / 512;
    const int tiles = (n_whole + kTcRows - 1) / kTcRows;
    int want = (512 + tiles - 1) / tiles;
    want = want < 1 ? 1 : (want > kTcMaxSplit ? kTcMaxSplit : want);
    if (want > periods) want = periods;
    for (int k = want; k > 1; --k)
        if (periods % k == 0 || periods / k >= 4) return k;
    return 1;
}

// The codes and group constants are read by 16-byte rows and TMA boxes: K must be
// a multiple of 512 (eight scales per 16 bytes) and the three weight arrays
// 16-byte aligned.  The activation rows are 16-byte aligned with a leading
// dimension that is a multiple of 8, which the ABI already requires.
bool qmm_tc_eligible(const QmmArgs &a) {
    return a.M >= 2 && a.M <= kTcMaxN && a.K % 512 == 0 && aligned(a.wq, 16) && aligned(a.scales, 16) &&
           aligned(a.biases, 16);
}

static bool g_tc_smem_set[64];

cudaError_t launch_qmm_tc(const QmmArgs &a, cudaStream_t stream) {
    cudaError_t e = get_encode();
    if (e != cudaSuccess) return e;
    TcPlan plan;
    std::memset(&plan, 0, sizeof plan);
    plan.ks = qmm_tc_split(a.K, a.n_whole);
    plan.periods = a.K / 512;
    plan.n_mma = ((a.M + 15) / 16) * 16;
    if (a.glu) {
        plan.ntiles = (a.seg.ncols + 63) / 64;
    } else {
        int n = 0;
        for (int s = 0; s < a.seg.nseg; ++s) {
            plan.tstart[s] = n;
            n += (a.seg.nrows[s] + kTcRows - 1) / kTcRows;
        }
        for (int s = a.seg.nseg; s <= TF_MAX_SEGS; ++s) plan.tstart[s] = n;
        plan.ntiles = n;
    }
    if (plan.ntiles == 0) return cudaSuccess;

    CUtensorMap xmap, cmap;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
        const cuuint64_t strides[1] = {(cuuint64_t)a.ldx * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kTcK, (cuuint32_t)plan.n_mma};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(a.x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(a.K / 2), (cuuint64_t)a.n_whole};
        const cuuint64_t strides[1] = {(cuuint64_t)(a.K / 2)};
        const cuuint32_t box[2] = {(cuuint32_t)(kTcK / 2), 64u};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a.wq), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!g_tc_smem_set[dev]) {
        e = cudaFuncSetAttribute(qmm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
        if (e != cudaSuccess) return e;
        g_tc_smem_set[dev] = true;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)(plan.ntiles * plan.ks));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = kTcSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)plan.ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, qmm_tc_kernel, a, xmap, cmap, plan);
}

}  // namespace tf
