// qmm_tc.cu -- prompt-chunk qmm (M = 2..128 activation rows) on the 5th-generation
// tensor cores.
//
// The weights enter the tensor core as their 4-bit codes taken about their
// middle, q - 8 (-8..7, exact in bf16), so one group of 64 values gives
// D_g = sum_{k in g} (q_k - 8) x_k per weight row and activation row, with the
// fp32 sums in tensor memory.  The group's scale and bias are applied on the CUDA
// cores:
//     y += s_g * D_g + (b_g + 8 s_g) * X_g,        X_g = sum_{k in g} x_k,
// which is sum_{k in g} x_k (s_g q_k + b_g) -- the affine format's dot product,
// with no rounded copy of the weights anywhere.  With the usual bias b ~ -8 s
// both terms stay near the size of their sum, and a large x whose weight is
// zero (q = 8, b = -8 s) adds exactly nothing to either.
// Per output the fp32 sum runs over the groups in ascending order, an order fixed
// by K alone.
//
// A tile is 128 weight rows (the MMA's M) against the call's M activation rows
// (the MMA's N: 16, 32, 64 or 128, the rows past M zero).  A tile never
// straddles two segments; with TF_EPI_GLU its rows 0-63 are gate rows and
// 64-127 the up rows of the same outputs.  Two CTAs per SM for N <= 32 (each
// with half of tensor memory), one CTA per SM above; 10 to 22 warps:
//   * warp 0, three threads: per four groups one TMA copy of the activation
//     tiles [4 x N x 64] and two of the tile's packed codes [2 x 64 rows x
//     128 B] (both with the 128-byte swizzle) into a ring of 2 to 4 slots in
//     shared memory, each copy from a lane of its own.  No multicast.
//   * 4 or 8 decoder warps, one thread per weight row (= tensor-memory lane):
//     the row's codes -> bf16 pairs, stored into an A stage in tensor memory
//     (tcgen05.st), software-pipelined so that a store drains while the next
//     group is decoded; four of them, one thread per activation row, also form
//     X_g from the activation tile, except where a table holds it (below).
//   * warp 1, one thread: tcgen05.mma kind::f16, A from tensor memory, B (the
//     activations) from shared memory, four K=16 steps per group into one of
//     several D buffers; tcgen05.commit releases the ring slot and the A stage and
//     publishes the D buffer.
//   * scale warps, per tensor-memory lane quarter one per 32 activation rows
//     (4 to 16 warps): read D_g (tcgen05.ld), fold it and X_g into fp32
//     accumulators held in registers, release the D buffer.
//
// Persistent CTAs.  When one slice covers K (and no GLU), one CTA per resident
// slot walks every gridDim.x-th tile, its ring, stages and barrier phases
// running on across tiles, and writes each tile's outputs itself.  X_g depends on
// x alone, so where it fits a shared-memory table holds the X_g of all the CTA's
// groups: at N = 16 the scale warps fill it from x in global memory at the start
// (no decoder forms X_g), at N = 32 and 64 a persistent CTA forms X_g on its
// first tile and folds the later ones from the table.  Same sums, same bits.
//
// Split K.  The groups are cut into `ks` slices, one per CTA of a thread-block
// cluster of `ks` CTAs; ks and the cut depend on K and the whole matrix's row
// count only (never on M, the segments or the device), so a row's result does
// not depend on which call or which half computes it.  Each CTA puts its
// accumulators in shared memory; after a cluster barrier CTA r reads the partial
// sums of the whole cluster through distributed shared memory for its share of
// the activation rows, adds them in rank order in fp32, rounds to bf16 (and
// forms gate*SiLU(up) with TF_EPI_GLU) and writes y.
//
// Every wait on an mbarrier is bounded; a wait that gives up marks the CTA
// failed and every output the cluster writes becomes NaN.  All threads still
// reach both cluster barriers, and tensor memory is released before exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "qmm_common.cuh"
#include "tmap.h"

namespace tf {

constexpr int kTcRows = 128;                    // weight rows per tile (MMA M)
constexpr int kTcK = 64;                        // K per group / pipeline stage
constexpr int kTcXbSlots = 8;                   // X_g slots in shared memory
constexpr int kTcGps = 4;                       // groups per ring slot
// Per MMA N: CTAs per SM (two for N <= 32, each with half of tensor memory),
// decoder and scale warps, and pipeline depths.  Ring slot: four groups, the
// activation tiles [4][N][128 B] and the codes [128 rows][128 B], both with the
// 128-byte swizzle.  The roles hand work on in steps of tc_bg(N) groups (one
// barrier wait and one release per step: for small N a barrier round costs
// about as much as a group's work).  Tensor memory: tc_dbufs(N) D stages of
// tc_bg(N) x N columns from column 0, tc_astages(N) A stages of tc_bg(N) x 32
// columns at the top.
__host__ __device__ constexpr int tc_ctas_per_sm(int n) { return n <= 32 ? 2 : 1; }
__host__ __device__ constexpr uint32_t tc_tmem_cols(int n) { return n <= 32 ? 256u : 512u; }
__host__ __device__ constexpr int tc_dec_warps(int n) { return n == 64 ? 8 : 4; }
// Scale warps: per tensor-memory lane quarter one warp per 32 activation rows.
__host__ __device__ constexpr int tc_scale_warps(int n) { return 4 * (n < 32 ? 1 : n / 32); }
__host__ __device__ constexpr int tc_threads(int n) { return 32 * (2 + tc_dec_warps(n) + tc_scale_warps(n)); }
__host__ __device__ constexpr int tc_slot_bytes(int n) { return kTcGps * (n * kTcK * 2 + kTcRows * kTcK / 2); }
__host__ __device__ constexpr int tc_ring(int n) { return n == 16 ? 4 : (n == 32 ? 3 : (n == 64 ? 4 : 2)); }
__host__ __device__ constexpr int tc_bg(int) { return 2; }
__host__ __device__ constexpr int tc_astages(int n) { return n <= 32 ? 2 : (n == 64 ? 3 : 4); }
__host__ __device__ constexpr int tc_dfit(int n) {
    return (int)(tc_tmem_cols(n) - 32 * tc_bg(n) * tc_astages(n)) / (tc_bg(n) * n);
}
__host__ __device__ constexpr int tc_dbufs(int n) { return tc_dfit(n) < 8 ? tc_dfit(n) : 8; }
constexpr int kTcMaxN = 128;                    // activation rows per call
constexpr int kTcMaxSplit = 8;                  // CTAs per cluster
constexpr int kTcXbBytes = kTcXbSlots * kTcMaxN * 4;
constexpr int kTcBarBytes = 1024;               // mbarriers, TMEM address, failure flag
constexpr int kTcSmemMax = 227 * 1024;          // dynamic shared memory of one CTA
constexpr int kTcSmemSM = 228 * 1024;           // shared memory of an SM (1 KB of it reserved per CTA)
// X_g table of a CTA: its groups of K, fp32 per activation row of the MMA
__host__ __device__ constexpr int tc_xtab_bytes(int n, int groups) { return groups * n * 4; }
__host__ __device__ constexpr int tc_num_bars(int n) {
    return 3 * tc_ring(n) + 2 * tc_astages(n) + 2 * tc_dbufs(n) + 2 * kTcXbSlots;
}
// Shared memory per CTA.  A CTA that takes all 512 tensor-memory columns asks for
// more than half of the SM's shared memory, so that a second CTA is never placed
// beside it only to wait in tcgen05.alloc; with two CTAs per SM each fits in half.
__host__ __device__ constexpr int tc_smem_need(int n) { return tc_ring(n) * tc_slot_bytes(n) + kTcXbBytes + kTcBarBytes + 1024; }
__host__ __device__ constexpr int tc_smem_bytes(int n) {
    return tc_ctas_per_sm(n) == 2 ? tc_smem_need(n) : (tc_smem_need(n) > 120 * 1024 ? tc_smem_need(n) : 120 * 1024);
}
constexpr long long kTcSpin = 1ll << 24;
template <int N>
struct TcChecks {
    static_assert(tc_slot_bytes(N) % 1024 == 0, "ring slots keep the 1 KB alignment of the swizzled tile");
    static_assert(N * kTcRows * 4 <= tc_ring(N) * tc_slot_bytes(N), "partial sums must fit in the ring");
    static_assert(tc_num_bars(N) * 8 + 8 <= kTcBarBytes, "barrier area");
    static_assert(tc_dbufs(N) >= 1 && tc_bg(N) * (tc_dbufs(N) * N + 32 * tc_astages(N)) <= (int)tc_tmem_cols(N),
                  "tensor memory map");
    static_assert(kTcGps % tc_bg(N) == 0 && kTcXbSlots % tc_bg(N) == 0 && 8 % tc_bg(N) == 0, "steps of whole groups");
    static_assert(tc_smem_bytes(N) <= 227 * 1024, "shared memory");
    static_assert(tc_ctas_per_sm(N) == 1 || (tc_smem_bytes(N) + 1024) * 3 > 228 * 1024, "at most two CTAs per SM");
    static_assert(tc_ctas_per_sm(N) == 2 || (tc_smem_bytes(N) + 1024) * 2 > 228 * 1024, "one CTA per SM");
};

// Plan of one launch, computed on the host.
struct TcPlan {
    int ks;                        // CTAs per cluster (K slices)
    int persist;                   // 1: each CTA walks tiles blockIdx.x, + gridDim.x, ... (ks == 1, no GLU)
    int xtab;                      // 1: the X_g of the CTA's groups in a shared-memory table (see the kernel)
    int xgroups;                   // groups of K a CTA covers at most (its table's rows)
    int periods;                   // K / 512: eight groups each
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
__device__ __forceinline__ void tc_tma_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
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

template <int X>
__device__ __forceinline__ void tc_ld(uint32_t taddr, uint32_t *r);
template <>
__device__ __forceinline__ void tc_ld<8>(uint32_t taddr, uint32_t *r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tc_ld<16>(uint32_t taddr, uint32_t *r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tc_ld<32>(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
        "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// X consecutive 32-bit columns of this thread's lane.
template <int X>
__device__ __forceinline__ void tc_st(uint32_t taddr, const uint32_t *v);
template <>
__device__ __forceinline__ void tc_st<16>(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
template <>
__device__ __forceinline__ void tc_st<32>(uint32_t taddr, const uint32_t *v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Codes 2j and 2j+1 of a packed word as the bf16 pair (q_2j - 8, q_2j+1 - 8),
// exactly (code 2j in the low half).  w holds code i at bits 4i, ws = w >> 4.
// Byte j of w has code 2j in its low nibble, byte j of ws has code 2j+1 there;
// prmt puts them at bits 0 and 16, the mask keeps the nibbles and ORs in the
// bf16 exponent of 128, which makes each half 128 + q; one bf16x2 subtraction of
// 136 leaves q - 8 (exact: every value involved is an integer below 2^8).
template <int j>
__device__ __forceinline__ uint32_t tc_code_pair(uint32_t w, uint32_t ws) {
    constexpr uint32_t sel = j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12);
    uint32_t p, r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(p) : "r"(w), "r"(ws), "n"(sel));
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"((p & 0x000F000Fu) | 0x43004300u), "r"(0x43084308u));
    return r;
}

// Two outputs' fold, a_i = fma(b, X_i, fma(s, D_i, a_i)), as two packed fp32x2
// FMAs: each half is the IEEE fma of its own operands, so the bits are those of
// four scalar fmaf in the same order, at half the instructions.
__device__ __forceinline__ void tc_fold2(float &a0, float &a1, float s, float d0, float d1, float b, float x0, float x1) {
    asm("{\n .reg .b64 A, S, D, B, X;\n mov.b64 A, {%0, %1};\n mov.b64 S, {%2, %2};\n mov.b64 D, {%3, %4};\n"
        " mov.b64 B, {%5, %5};\n mov.b64 X, {%6, %7};\n fma.rn.f32x2 A, S, D, A;\n fma.rn.f32x2 A, B, X, A;\n"
        " mov.b64 {%0, %1}, A;\n}"
        : "+f"(a0), "+f"(a1)
        : "f"(s), "f"(d0), "f"(d1), "f"(b), "f"(x0), "f"(x1));
}

// acc + lo(w) + hi(w) for a bf16 pair w, each add fp32 += bf16 (Blackwell's
// mixed-precision add: the bf16 operand is widened exactly, one rounding per add).
__device__ __forceinline__ float tc_add_bf16x2(float acc, uint32_t w) {
    float r;
    asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n add.rn.f32.bf16 %0, l, %2;\n add.rn.f32.bf16 %0, h, %0;\n}"
        : "=f"(r)
        : "r"(w), "f"(acc));
    return r;
}

// bf16 number j (0..7) of a 16-byte vector, compile-time j.
template <int j>
__device__ __forceinline__ float tc_pick_bf16(const uint4 &v) {
    const uint32_t w = (j >> 1) == 0 ? v.x : (j >> 1) == 1 ? v.y : (j >> 1) == 2 ? v.z : v.w;
    return __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

template <int N, bool kPersist>
__global__ void __launch_bounds__(tc_threads(N), tc_ctas_per_sm(N))
    qmm_tc_kernel(QmmArgs a, const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap, TcPlan plan) {
    constexpr int SW = tc_scale_warps(N);     // scale warps
    constexpr int NT = N / (SW / 4);          // activation rows per scale thread (16 or 32)
    // columns per tcgen05.ld: the persistent walk at N = 128 keeps the tile's
    // state in registers beside its 32 sums, so its loads take 8 columns at a time;
    // one tile per CTA at N = 64 has the room to load its 32 in one go (one wait)
    constexpr int CH = kPersist ? (N == 128 ? 8 : 16) : (N == 64 ? 32 : 16);
    constexpr int R = tc_ring(N), NA = tc_astages(N), ND = tc_dbufs(N);
    constexpr int SLOT = tc_slot_bytes(N), XG = N * kTcK * 2, XBYTES = kTcGps * XG, RING = R * SLOT;
    constexpr uint32_t TCOLS = tc_tmem_cols(N);
    constexpr int BG = tc_bg(N), XS = kTcXbSlots / BG;   // groups per step; X_g slots of a step's size
    constexpr uint32_t ACOL = TCOLS - 32 * BG * NA;   // first A-stage column
    constexpr int DW = tc_dec_warps(N);               // decoder warps
    constexpr int VW = 32 * 4 / DW;                   // bf16 pairs per decoder thread and group: 32 or 16
    (void)sizeof(TcChecks<N>);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *ring = smem;                                               // [slot][x: 4 groups | codes]
    float *part = reinterpret_cast<float *>(smem);                      // at the end: [N][128] fp32
    float *xbar = reinterpret_cast<float *>(smem + RING);       // [slot][128] fp32
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + RING + kTcXbBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + tc_num_bars(N));
    volatile int *fail = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // X_g depends on the activations alone, the same for every tile, so where it
    // fits it goes into a table [group][activation row] in shared memory.  At
    // N = 16 the scale warps fill it from x in global memory while the first copies,
    // decodes and MMAs run, and no decoder forms X_g.  At N = 32 and 64 (filling it
    // would take the scale warps too long) a persistent CTA forms X_g through the
    // ring on its first tile only, writing the table too, and folds its later
    // tiles from it.  Not at N = 128: the table's registers would spill the fold's
    // sums.
    float *xtab = reinterpret_cast<float *>(smem + RING + kTcXbBytes + kTcBarBytes);
    constexpr bool kXFill = N == 16;                                    // the scale warps fill the table
    constexpr bool kXFirst = !kXFill && kPersist && N <= 64;            // first-tile fill through the ring
    const bool xt = (kXFill || kXFirst) && plan.xtab != 0;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    const int ks = plan.ks;
    const int rank = (int)tc_cluster_rank();
    const int p0 = rank * plan.periods / ks, p1 = (rank + 1) * plan.periods / ks;
    const int i0 = 8 * p0, nst = 8 * (p1 - p0);          // this CTA's groups [i0, i0 + nst) of a tile
    // The CTA's tiles: one (blockIdx.x / ks), or with kPersist every
    // gridDim.x-th from blockIdx.x, the roles running on through them without a
    // new start (barrier phases and ring slots count on across tiles).
    const int ntl = kPersist ? (plan.ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 1;
    auto tile_of = [&](int it) { return kPersist ? (int)blockIdx.x + it * (int)gridDim.x : (int)blockIdx.x / ks; };
    const int ntot = ntl * nst;                          // groups this CTA runs through
    const uint32_t bar_s = tc_smem(bars);
    // barrier addresses: full[R] xfree[R] cfree[R] afull[A] aempty[A] dfull[D] dfree[D] xbfull[X] xbfree[X]
    auto full = [=](int s) { return bar_s + 8u * s; };
    auto xfree = [=](int s) { return bar_s + 8u * (R + s); };
    auto cfree = [=](int s) { return bar_s + 8u * (2 * R + s); };
    auto afull = [=](int s) { return bar_s + 8u * (3 * R + s); };
    auto aempty = [=](int s) { return bar_s + 8u * (3 * R + NA + s); };
    auto dfull = [=](int s) { return bar_s + 8u * (3 * R + 2 * NA + s); };
    auto dfree = [=](int s) { return bar_s + 8u * (3 * R + 2 * NA + ND + s); };
    auto xbfull = [=](int s) { return bar_s + 8u * (3 * R + 2 * NA + 2 * ND + s); };
    auto xbfree = [=](int s) { return bar_s + 8u * (3 * R + 2 * NA + 2 * ND + kTcXbSlots + s); };

    // A tile's rows: box A (tile rows 0-63) and box B (64-127) of the whole
    // matrix, how many of each box are valid, and the output column of tile row 0.
    auto tile_info = [&](int tile, int &rowA, int &rowB, int &validA, int &validB, int &col_base) {
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
    };
    int rowA, rowB, validA, validB, col_base;   // the first (or only) tile's
    tile_info(tile_of(0), rowA, rowB, validA, validB, col_base);

    if (threadIdx.x == 0) {
        for (int s = 0; s < R; ++s) {
            tc_mbar_init(full(s), 1);
            tc_mbar_init(xfree(s), 1);
            tc_mbar_init(cfree(s), DW);
        }
        for (int s = 0; s < NA; ++s) {
            tc_mbar_init(afull(s), DW);
            tc_mbar_init(aempty(s), 1);
        }
        for (int s = 0; s < ND; ++s) {
            tc_mbar_init(dfull(s), 1);
            tc_mbar_init(dfree(s), SW);
        }
        for (int s = 0; s < kTcXbSlots; ++s) {
            tc_mbar_init(xbfull(s), 4);
            tc_mbar_init(xbfree(s), SW);
        }
        *fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem(tmem_slot)),
                     "r"(TCOLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        // Per slot (four groups) three copies, each from a lane of its own:
        // lane 0 the activation tiles, lanes 1 and 2 the codes of tile rows
        // 0-63 and 64-127.  A tensor copy holds the thread that issues it for
        // a fixed time, so copies from three lanes overlap where one lane's
        // would queue.
        if (lane < 3) {
            const uint32_t bytes = (uint32_t)SLOT;
            const int nsl = nst / kTcGps;
            int issued = 0;
            int tr_a = rowA, tr_b = rowB;
            for (int j = 0; j < ntl * nsl; ++j) {   // slots over the CTA's tiles
                const int s = j % R;
                if (j > 0 && j % nsl == 0) {   // the next tile's rows
                    int va, vb, cb;
                    tile_info(tile_of(j / nsl), tr_a, tr_b, va, vb, cb);
                }
                bool ok = true;
                if (j >= R) {
                    const uint32_t par = ((j / R) - 1) & 1;
                    ok = tc_wait(xfree(s), par, fail) && tc_wait(cfree(s), par, fail);
                }
                if (!__all_sync(0x7u, ok && !*fail)) {
                    if (lane == 0) *fail = 1;
                    break;
                }
                const int i = i0 + kTcGps * (j % nsl);
                const uint32_t slot = tc_smem(ring + s * SLOT);
                if (lane == 0) tc_expect_tx(full(s), bytes);
                __syncwarp(0x7u);
                if (lane == 0)
                    tc_tma_3d(slot, &xmap, 0, 0, i, full(s));
                else
                    tc_tma_2d(slot + XBYTES + (lane - 1) * (kTcRows / 2) * (kTcGps * kTcK / 2), &cmap,
                              i * (kTcK / 2), lane == 1 ? tr_a : tr_b, full(s));
                issued = j + 1;
            }
            // every copy issued must land before the ring is reused or the CTA exits
            if (lane == 0)
                for (int j = issued - R; j < issued; ++j)
                    if (j >= 0) tc_wait(full(j % R), (j / R) & 1, fail, 1 << 16);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t idesc = tc_idesc(N);
            for (int k = 0; k < ntot / BG; ++k) {   // steps of BG groups
                const int sa = k % NA, sd = k % ND;
                if (!tc_wait(afull(sa), (k / NA) & 1, fail) || (k >= ND && !tc_wait(dfree(sd), ((k / ND) - 1) & 1, fail))) {
                    *fail = 1;
                    break;
                }
                bool ok = true;
#pragma unroll
                for (int g = 0; g < BG; ++g) {
                    const int li = k * BG + g, j = li / kTcGps, gs = li % kTcGps, s = j % R;
                    if (gs == 0 && !tc_wait(full(s), (j / R) & 1, fail)) {   // the slot's first group
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xb = tc_smem(ring + s * SLOT) + (uint32_t)(gs * XG);
                    const uint32_t dt = tmem + (uint32_t)(BG * N * sd + N * g), at = tmem + ACOL + 32u * (BG * sa + g);
#pragma unroll
                    for (int kk = 0; kk < kTcK / 16; ++kk)
                        tc_mma_ts(dt, at + 8 * kk, tc_desc(xb + kk * 32), idesc, kk > 0 ? 1u : 0u);
                    if (gs == kTcGps - 1) tc_commit(xfree(s));   // the slot's last group
                }
                if (!ok) {
                    *fail = 1;
                    break;
                }
                tc_commit(aempty(sa));
                tc_commit(dfull(sd));
            }
        }
    } else if (warp < 2 + DW) {
        // ------------------------------------------- codes -> A stages, and X_g
        // Per step: wait for the A stage; per group wait for the slot (at its
        // first group), turn the row's codes into bf16 pairs and store them into
        // tensor memory; the stage is published (afull) once, after
        // tcgen05.wait::st.  With 8 decoder warps each thread takes half of its
        // row's 64 codes.  The four warps of the first half also form X_g.
        const int q = warp & 3, dh = (warp - 2) >> 2;   // lane quarter; part of the group's codes
        const int t = 32 * q + lane;                    // tile row == TMEM lane; also an activation row
        const uint32_t a_lane = tmem + ((uint32_t)(32 * q) << 16) + ACOL + (uint32_t)(dh * VW);
        const bool xrole = dh == 0;
        uint32_t v[VW];
        for (int k = 0; k < ntot / BG; ++k) {
            const int sa = k % NA, xs = k % XS;
            const bool ring_x = !xt || (!kXFill && k * BG < nst);   // X_g formed here: no table, or its first tile
            bool ok = k < NA || tc_wait(aempty(sa), ((k / NA) - 1) & 1, fail);
            if (__any_sync(0xFFFFFFFFu, !ok)) {
                *fail = 1;
                break;
            }
            tc_fence_after();
            float xsum[BG];
#pragma unroll
            for (int g = 0; g < BG; ++g) {
                const int li = k * BG + g, j = li / kTcGps, gs = li % kTcGps, s = j % R;
                if (gs == 0) {
                    ok = tc_wait(full(s), (j / R) & 1, fail);
                    if (__any_sync(0xFFFFFFFFu, !ok)) break;
                }
                const uint8_t *slot = ring + s * SLOT;
                // row t's 128 bytes of codes, 16-byte chunk c at position c ^ (t & 7)
                // (the copy's swizzle); group gs is chunks 2 gs and 2 gs + 1, so eight
                // neighbouring rows read eight distinct bank quads
                const uint4 *cp = reinterpret_cast<const uint4 *>(slot + XBYTES + 128 * t);
                uint32_t w[VW / 4];
                if (VW == 32) {
                    const uint4 c0 = cp[(2 * gs) ^ (t & 7)], c1 = cp[(2 * gs + 1) ^ (t & 7)];
                    w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w;
                    w[VW / 4 - 4] = c1.x; w[VW / 4 - 3] = c1.y; w[VW / 4 - 2] = c1.z; w[VW / 4 - 1] = c1.w;
                } else {
                    const uint4 c0 = cp[(2 * gs + dh) ^ (t & 7)];
                    w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w;
                }
                xsum[g] = 0.0f;
                if (xrole && ring_x && t < N) {   // X_g of activation row t: 64 values, k ascending (8 chunks of 8)
                    const uint8_t *xrow = slot + gs * XG + t * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 xv = *reinterpret_cast<const uint4 *>(xrow + ((c ^ (t & 7)) << 4));
                        const float cs = tc_add_bf16x2(tc_add_bf16x2(tc_add_bf16x2(tc_add_bf16x2(0.0f, xv.x), xv.y), xv.z), xv.w);
                        xsum[g] = c == 0 ? cs : xsum[g] + cs;
                    }
                }
#pragma unroll
                for (int c = 0; c < VW / 4; ++c) {
                    const uint32_t ws = w[c] >> 4;
                    v[4 * c + 0] = tc_code_pair<0>(w[c], ws);
                    v[4 * c + 1] = tc_code_pair<1>(w[c], ws);
                    v[4 * c + 2] = tc_code_pair<2>(w[c], ws);
                    v[4 * c + 3] = tc_code_pair<3>(w[c], ws);
                }
                __syncwarp();
                if (lane == 0 && gs == kTcGps - 1) tc_arrive(cfree(s));   // the slot's codes are read
                tc_st<VW>(a_lane + 32u * (uint32_t)(BG * sa + g), v);
                tc_wait_st();
            }
            if (__any_sync(0xFFFFFFFFu, !ok)) {
                *fail = 1;
                break;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) tc_arrive(afull(sa));
            if (xrole && ring_x) {
                ok = k < XS || tc_wait(xbfree(xs), ((k / XS) - 1) & 1, fail);
                if (__any_sync(0xFFFFFFFFu, !ok)) {
                    *fail = 1;
                    break;
                }
                if (t < N) {
#pragma unroll
                    for (int g = 0; g < BG; ++g) {
                        xbar[(xs * BG + g) * kTcMaxN + t] = xsum[g];
                        if (!kXFill && xt) xtab[(k * BG + g) * N + t] = xsum[g];   // published by the arrive below
                    }
                }
                __syncwarp();
                if (lane == 0) tc_arrive(xbfull(xs));
            }
        }
    } else {
        // ------------------------------------------------ y += s D_g + b X_g
        const int q = warp & 3, h = (warp - 2 - DW) >> 2;   // lane quarter, block of NT rows
        const int t = 32 * q + lane;                   // tile row == TMEM lane
        const int G = a.K / kGroup;
        const uint32_t d_lane = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * NT);
        const float *xb_h = xbar + h * NT;
        float acc[NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) acc[j] = 0.0f;
        if (kXFill && xt) {   // the X_g table: the same sums, in the same order, as a decoder forms from a slot
            const int ft = threadIdx.x - 32 * (2 + DW);
            for (int e = ft; e < nst * N; e += 32 * SW) {
                const int gl = e / N, tr = e % N;
                float xs = 0.0f;
                if (tr < a.M) {
                    const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + (size_t)tr * a.ldx + (size_t)(i0 + gl) * kTcK);
                    uint4 xv[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) xv[c] = __ldg(xr + c);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float cs =
                            tc_add_bf16x2(tc_add_bf16x2(tc_add_bf16x2(tc_add_bf16x2(0.0f, xv[c].x), xv[c].y), xv[c].z), xv[c].w);
                        xs = c == 0 ? cs : xs + cs;
                    }
                } else {   // a row past M reads as zero in the copies: its sum is +0
                    xs = tc_add_bf16x2(0.0f, 0u);
                }
                xtab[gl * N + tr] = xs;
            }
            asm volatile("bar.sync 1, %0;" ::"r"(32 * SW) : "memory");   // the scale warps only
        }
        int li = 0;   // groups folded so far, over all of the CTA's tiles
        for (int it = 0; it < ntl && !*fail; ++it) {
        const bool ring_x = !xt || (!kXFill && it == 0);   // X_g through the ring (and into the table), else from it
        int lt = 0;                           // group within the tile
        int tra = rowA, trb = rowB, tva = validA, tvb = validB, tcb = col_base;
        if (it > 0) tile_info(tile_of(it), tra, trb, tva, tvb, tcb);
        const bool valid = t < 64 ? t < tva : (t - 64) < tvb;
        const int row = t < 64 ? tra + t : trb + (t - 64);
        const uint16_t *srow = valid ? a.scales + (size_t)row * G : nullptr;
        const uint16_t *brow = valid ? a.biases + (size_t)row * G : nullptr;
#pragma unroll
        for (int j = 0; j < NT; ++j) acc[j] = 0.0f;
        uint4 s8 = make_uint4(0, 0, 0, 0), b8 = s8, sn = s8, bn = s8;
        if (srow) {
            s8 = __ldg(reinterpret_cast<const uint4 *>(srow + 8 * p0));
            b8 = __ldg(reinterpret_cast<const uint4 *>(brow + 8 * p0));
        }
        for (int p = p0; p < p1 && !*fail; ++p) {
            if (srow && p + 1 < p1) {   // next period's eight scales and biases
                sn = __ldg(reinterpret_cast<const uint4 *>(srow + 8 * (p + 1)));
                bn = __ldg(reinterpret_cast<const uint4 *>(brow + 8 * (p + 1)));
            }
// Group J (0..7) of the period; the step's barriers are waited for at its
// first group and released after its last.
#define TC_GROUP(J)                                                                                                 \
    {                                                                                                               \
        const int k = li / BG, sd = k % ND, xs = k % XS, g = (J) % BG;                                              \
        if (g == 0) {                                                                                               \
            const bool ok = tc_wait(dfull(sd), (k / ND) & 1, fail) && (!ring_x || tc_wait(xbfull(xs), (k / XS) & 1, fail)); \
            if (__any_sync(0xFFFFFFFFu, !ok)) {                                                                     \
                *fail = 1;                                                                                          \
                break;                                                                                              \
            }                                                                                                       \
            tc_fence_after();                                                                                       \
        }                                                                                                           \
        /* D holds sum (q - 8) x: y += s D + (b + 8 s) X */                                                       \
        const float sf = tc_pick_bf16<J>(s8), bf = fmaf(8.0f, sf, tc_pick_bf16<J>(b8));                             \
        const float *xg = xt ? xtab + lt * N + h * NT : xb_h + (xs * BG + g) * kTcMaxN;                            \
        _Pragma("unroll") for (int c = 0; c < NT; c += CH) {                                                        \
            uint32_t d[CH];                                                                                         \
            tc_ld<CH>(d_lane + (uint32_t)(BG * N * sd + N * g) + c, d);                                             \
            tc_wait_ld();                                                                                           \
            _Pragma("unroll") for (int j = 0; j < CH; j += 4) {                                                     \
                const float4 xv = *reinterpret_cast<const float4 *>(xg + c + j);                                    \
                tc_fold2(acc[c + j + 0], acc[c + j + 1], sf, __uint_as_float(d[j + 0]), __uint_as_float(d[j + 1]),  \
                         bf, xv.x, xv.y);                                                                           \
                tc_fold2(acc[c + j + 2], acc[c + j + 3], sf, __uint_as_float(d[j + 2]), __uint_as_float(d[j + 3]),  \
                         bf, xv.z, xv.w);                                                                           \
            }                                                                                                       \
        }                                                                                                           \
        if (g == BG - 1) {                                                                                          \
            tc_fence_before();                                                                                      \
            __syncwarp();                                                                                           \
            if (lane == 0) {                                                                                        \
                tc_arrive(dfree(sd));                                                                               \
                if (ring_x) tc_arrive(xbfree(xs));                                                                  \
            }                                                                                                       \
        }                                                                                                           \
        ++li;                                                                                                       \
        ++lt;                                                                                                       \
    }
            do {
                TC_GROUP(0) TC_GROUP(1) TC_GROUP(2) TC_GROUP(3) TC_GROUP(4) TC_GROUP(5) TC_GROUP(6) TC_GROUP(7)
            } while (0);
#undef TC_GROUP
            s8 = sn;
            b8 = bn;
        }
        if (kPersist && valid) {   // the whole K is here: the tile's outputs go straight out
#pragma unroll
            for (int j = 0; j < NT; ++j)
                if (h * NT + j < a.M) a.y[(size_t)(h * NT + j) * a.ldy + tcb + t] = f32_to_bf16_rne(acc[j]);
        }
        }
        // this CTA's partial sums -> shared memory, as part[m][t]
        if (!kPersist) {
#pragma unroll
            for (int j = 0; j < NT; ++j) part[(h * NT + j) * kTcRows + t] = acc[j];
        }
    }
    __syncwarp();
    tc_fence_before();
    tc_cluster_sync();   // every partial sum and failure flag of the cluster is in place

    if (kPersist && warp >= 2 + DW) {
        if (*fail) {   // a wait gave up: every output of the CTA's tiles reads NaN
            const int tid = threadIdx.x - 32 * (2 + DW);
            for (int it = 0; it < ntl; ++it) {
                int ra, rb, va, vb, cb;
                tile_info(tile_of(it), ra, rb, va, vb, cb);
                const int nv = va + vb;
                for (int e = tid; e < nv * a.M; e += 32 * SW) a.y[(size_t)(e / nv) * a.ldy + cb + e % nv] = (uint16_t)TF_NAN_BF16;
            }
        }
    } else if (warp >= 2 + DW) {
        const int tid = threadIdx.x - 32 * (2 + DW);   // 0 .. 32 SW - 1
        constexpr int RT = 32 * SW;                              // reducing threads
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
            const int pr = tid & 63;
            if (pr < validA) {
                for (int m = m0 + (tid >> 6); m < m1; m += RT / 64) {
                    uint16_t out = (uint16_t)TF_NAN_BF16;
                    if (!bad) {
                        const float g = bf16_bits_to_f32(f32_to_bf16_rne(total(m, pr)));
                        const float u = bf16_bits_to_f32(f32_to_bf16_rne(total(m, pr + 64)));
                        out = f32_to_bf16_rne(glu_f32(g, u));
                    }
                    a.y[(size_t)m * a.ldy + col_base + pr] = out;
                }
            }
        } else {
            const int t = tid & 127;
            if (t < validA + validB) {
                for (int m = m0 + (tid >> 7); m < m1; m += RT / 128)
                    a.y[(size_t)m * a.ldy + col_base + t] = bad ? (uint16_t)TF_NAN_BF16 : f32_to_bf16_rne(total(m, t));
            }
        }
    }
    __syncwarp();
    tc_cluster_sync();   // no CTA leaves while another still reads its shared memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS) : "memory");
    }
}

// ------------------------------------------------------------------ host --
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn() {
    if (g_encode) return g_encode;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return nullptr;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return g_encode;
}

static cudaError_t get_encode() { return encode_tiled_fn() ? cudaSuccess : cudaErrorNotSupported; }

// K slices per tile: from K and the whole matrix's row count alone.  The whole
// matrix should give about 512 CTAs; a slice keeps at least four periods of
// eight groups unless the periods divide evenly.
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

template <int N, bool kPersist>
static cudaError_t launch_tc_n(const QmmArgs &a, const CUtensorMap &xmap, const CUtensorMap &cmap, const TcPlan &plan,
                               cudaStream_t stream) {
    static bool smem_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!smem_set[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(qmm_tc_kernel<N, kPersist>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemMax);
        if (e != cudaSuccess) return e;
        smem_set[dev] = true;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    // persistent: one CTA per resident slot, each walking every gridDim.x-th tile
    const int slots = tc_ctas_per_sm(N) * num_sms();
    const int ctas = kPersist ? (plan.ntiles < slots ? plan.ntiles : slots) : plan.ntiles * plan.ks;
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(tc_threads(N));
    cfg.dynamicSmemBytes = tc_smem_bytes(N) + (plan.xtab ? tc_xtab_bytes(N, plan.xgroups) : 0);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)plan.ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, qmm_tc_kernel<N, kPersist>, a, xmap, cmap, plan);
}

template <int N>
static cudaError_t launch_tc_n(const QmmArgs &a, const CUtensorMap &xmap, const CUtensorMap &cmap, const TcPlan &plan,
                               cudaStream_t stream) {
    if (plan.persist) return launch_tc_n<N, true>(a, xmap, cmap, plan, stream);
    return launch_tc_n<N, false>(a, xmap, cmap, plan, stream);
}

cudaError_t launch_qmm_tc(const QmmArgs &a, cudaStream_t stream) {
    cudaError_t e = get_encode();
    if (e != cudaSuccess) return e;
    TcPlan plan;
    std::memset(&plan, 0, sizeof plan);
    plan.ks = qmm_tc_split(a.K, a.n_whole);
    plan.periods = a.K / 512;
    const int n_mma = a.M <= 16 ? 16 : a.M <= 32 ? 32 : a.M <= 64 ? 64 : 128;
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
    // One K slice and plain outputs: CTAs stay resident and walk the tiles.
    plan.persist = plan.ks == 1 && !a.glu;
    // the X_g table where it fits beside the rest, keeping two CTAs per SM where there are two
    plan.xgroups = 8 * ((plan.periods + plan.ks - 1) / plan.ks);
    if (n_mma == 16 || (plan.persist && n_mma <= 64)) {
        const int need = tc_smem_bytes(n_mma) + tc_xtab_bytes(n_mma, plan.xgroups);
        plan.xtab = need <= kTcSmemMax && (tc_ctas_per_sm(n_mma) == 1 || 2 * (need + 1024) <= kTcSmemSM);
    }

    CUtensorMap xmap, cmap;
    {
        // [group][row][64 values]: four groups' activation tiles in one copy,
        // each tile the MMA's B operand as it stands (rows past M read as zero)
        const cuuint64_t dims[3] = {(cuuint64_t)kTcK, (cuuint64_t)a.M, (cuuint64_t)(a.K / kTcK)};
        const cuuint64_t strides[2] = {(cuuint64_t)a.ldx * 2, (cuuint64_t)kTcK * 2};
        const cuuint32_t box[3] = {(cuuint32_t)kTcK, (cuuint32_t)n_mma, (cuuint32_t)kTcGps};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t *>(a.x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(a.K / 2), (cuuint64_t)a.n_whole};
        const cuuint64_t strides[1] = {(cuuint64_t)(a.K / 2)};
        const cuuint32_t box[2] = {(cuuint32_t)(kTcGps * kTcK / 2), 64u};   // four groups' codes of 64 rows
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a.wq), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    switch (n_mma) {
        case 16: return launch_tc_n<16>(a, xmap, cmap, plan, stream);
        case 32: return launch_tc_n<32>(a, xmap, cmap, plan, stream);
        case 64: return launch_tc_n<64>(a, xmap, cmap, plan, stream);
        default: return launch_tc_n<128>(a, xmap, cmap, plan, stream);
    }
}

}  // namespace tf
