// qmm_stream.cu -- M = 1 dequant-GEMV: weights streamed through shared memory by
// bulk asynchronous copies, dot products taken exactly in integer arithmetic.
//
// Why this shape on B200.  At M = 1 every weight byte is used once, and the 148
// SMs must turn ~40 weights per clock each into products to keep up with HBM.
// Two limits meet there:
//   * bytes in flight: ~64 KB per SM are needed to cover HBM latency.  Each warp
//     owns a ring of kStages shared-memory slots that its lanes refill with
//     cp.async.bulk (the TMA engine's 1-D copy), so the copies stay in flight
//     while the warp computes, independent of the register budget;
//   * instructions per weight: floating-point nibble decoding costs 3-4 issue
//     slots per weight, most of them integer-pipe work.  Here a word of 8 codes
//     is split into two words of 4 bytes (2 lop3 + 1 shift) and multiplied with
//     the activations by dp4a, 4 products and their sum per instruction, in exact
//     integer arithmetic.
//
// Exact integer dot (per lane-chunk: the 32 x a lane meets in one 1,024-K chunk).
// The 32 bf16 x are put in fixed point with the chunk's own exponent E (every
// |x| < 2^E, E the smallest such over the chunk): F = RN(x * 2^(23-E)), |F| < 2^23, which is
// exact for every x within 2^15 of the chunk's largest magnitude (smaller ones
// are rounded to 2^(E-24), far below the bf16 resolution of any output).  F is
// kept as three bytes, F = L2*2^16 + L1*2^8 + L0 (L2 signed), and
//     P = sum q_k F_k = 2^16 sum q L2 + 2^8 sum q L1 + sum q L0
// with three int32 dp4a accumulators that cannot overflow (32 * 15 * 255 < 2^17).
// The lane then adds s * 2^(E-23) * P and b * X (X = the fp32 sum of the same 32
// x) to its running sum; w = s q + b, so those two terms are the chunk's x.w.
// A chunk holding NaN or +-Inf gets the scale NaN, so the row's result is NaN.
//
// Order of every operation depends on K alone (chunks ascending, per-lane
// sums, the shuffle tree of qmm_gemv.cu), never on the rows a launch covers:
// split == whole holds bit for bit.
//
// Slot (kRU rows x kKS values of K):
//   [codes of row 0 (kKS/2 B)] .. [codes of row kRU-1] [scales, kKS/32 B per row] [biases]
// A unit is kRU rows: four consecutive output columns (TF_EPI_NONE), or the
// gate and up rows of two consecutive columns (TF_EPI_GLU, rows g0 u0 g1 u1).
#include "qmm_common.cuh"
#include "stream_common.cuh"

namespace tf {

constexpr int kKS = 2048;                                    // K per slot
// slots per warp: two 4-row slots already keep ~90 KB per SM in flight; narrow
// units carry smaller slots, so they keep more of them outstanding
constexpr int stages_for(int ru) { return ru >= 4 ? 2 : (ru == 2 ? 4 : 6); }
constexpr int kSlotQ = kKS / 2;                              // code bytes of one row in a slot
constexpr int kSlotS = kKS / 32;                             // scale (or bias) bytes of one row
constexpr int slot_bytes(int ru) { return ru * (kSlotQ + 2 * kSlotS); }   // 1,152 per row
constexpr int kLimbBytes = 6 * 16;                           // limb words of one lane-chunk
constexpr int kMaxWarps = 20;
constexpr long long kSpinLimit = 1ll << 22;                  // bounded waits, see wait_slot

struct StreamLayout {
    int nch, warps;
    size_t limb_off, X_off, scale_off, bar_off, ring_off, total;
};

__host__ __device__ inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared memory for K and a warp count; the widest that fits is chosen on the host.
__host__ __device__ inline StreamLayout stream_layout(int K, int warps, int ru) {
    StreamLayout L;
    L.nch = (K + kChunk - 1) / kChunk;
    L.warps = warps;
    L.limb_off = 0;
    L.X_off = round_up(L.limb_off + (size_t)L.nch * 32 * kLimbBytes, 128);
    L.scale_off = round_up(L.X_off + (size_t)L.nch * 32 * 4, 128);
    L.bar_off = round_up(L.scale_off + (size_t)L.nch * 32 * 4, 128);
    L.ring_off = round_up(L.bar_off + (size_t)warps * stages_for(ru) * 8, 128);
    L.total = L.ring_off + (size_t)warps * stages_for(ru) * slot_bytes(ru);
    return L;
}

// sum over the lane's 32 codes of q_k * F_k, as a float.  limb[j] (j = limb*2 +
// parity) holds in word w the limb bytes of x[8w+p], x[8w+p+2], x[8w+p+4], x[8w+p+6];
// the even codes of word w are its low nibbles, the odd codes its high nibbles.
__device__ __forceinline__ float lane_chunk_idot(const uint4 &q, const uint4 *limb) {
    int a0 = 0, a1 = 0, a2 = 0;
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
    const uint32_t *L = reinterpret_cast<const uint32_t *>(limb);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t v = words[w];
        const uint32_t ue = v & 0x0F0F0F0Fu, uo = (v >> 4) & 0x0F0F0F0Fu;
        a0 = dp4a_uu(ue, L[0 * 4 + w], a0);
        a0 = dp4a_uu(uo, L[1 * 4 + w], a0);
        a1 = dp4a_uu(ue, L[2 * 4 + w], a1);
        a1 = dp4a_uu(uo, L[3 * 4 + w], a1);
        a2 = dp4a_us(ue, L[4 * 4 + w], a2);
        a2 = dp4a_us(uo, L[5 * 4 + w], a2);
    }
    return fmaf((float)a2, 65536.0f, fmaf((float)a1, 256.0f, (float)a0));
}

// ------------------------------------------------------------------ kernel --
template <int kRU>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) qmm_m1_stream_kernel(QmmArgs a, int units) {
    constexpr int kSlotBytes = slot_bytes(kRU);
    constexpr int kStages = stages_for(kRU);
    extern __shared__ __align__(128) uint8_t smem[];
    const int W = blockDim.x >> 5;
    const StreamLayout L = stream_layout(a.K, W, kRU);
    const int K = a.K, nch = L.nch;
    const int nsl = (K + kKS - 1) / kKS;
    const int G = K / kGroup;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t *limbs = smem + L.limb_off;
    float *Xs = reinterpret_cast<float *>(smem + L.X_off);
    float *Ss = reinterpret_cast<float *>(smem + L.scale_off);
    uint8_t *ring = smem + L.ring_off + (size_t)warp * kStages * kSlotBytes;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar0 = smem_addr(smem + L.bar_off) + (uint32_t)(warp * kStages * 8);

    const long long gw = (long long)blockIdx.x * W + warp;
    const long long nw = (long long)gridDim.x * W;
    const int u0 = (int)(gw * units / nw);
    const int u1 = (int)((gw + 1) * units / nw);
    const int steps = (u1 - u0) * nsl;

    // copy role of this lane: array (lane % 3: codes, scales, biases) of unit row lane / 3
    const int my_r = lane / 3, my_a = lane % 3;
    const bool copier = lane < 3 * kRU;
    const uint8_t *gbase = my_a == 0 ? a.wq
                         : (my_a == 1 ? reinterpret_cast<const uint8_t *>(a.scales)
                                      : reinterpret_cast<const uint8_t *>(a.biases));
    const size_t grow = my_a == 0 ? (size_t)K / 2 : (size_t)G * 2;       // bytes per matrix row
    const int kdiv = my_a == 0 ? 2 : 32;                                 // bytes of a K range = len / kdiv
    const uint32_t doff = my_a == 0 ? my_r * kSlotQ
                        : (my_a == 1 ? kRU * kSlotQ + my_r * kSlotS : kRU * kSlotQ + kRU * kSlotS + my_r * kSlotS);
    constexpr int kCols = kRU / 2 > 0 ? kRU / 2 : 1;   // output columns of a GLU unit
    auto unit_row = [&](int u, int r) {   // whole-matrix row of unit row r, -1 past the end
        const int col = a.glu ? u * kCols + (r >> 1) : u * kRU + r;
        return col < a.seg.ncols ? seg_row(a.seg, col, a.glu, a.glu ? (r & 1) : 0) : -1;
    };
    // rows of a unit that exist (the last unit of a launch may be short)
    auto unit_live_rows = [&](int u) {
        const int cols_left = a.seg.ncols - (a.glu ? u * kCols : u * kRU);
        return a.glu ? 2 * min(kCols, cols_left) : min(kRU, cols_left);
    };
    // issue pointer: unit iu, K-slice ij of the next step whose copies go out
    int iu = u0, ij = 0, it_ = 0;
    int my_row = copier && u0 < u1 ? unit_row(u0, my_r) : -1;
    int live = u0 < u1 ? unit_live_rows(u0) : 0;
    bool failed = false;
    auto issue_next = [&]() {
        const int slot = it_ % kStages;
        const int k0 = ij * kKS, len = min(kKS, K - k0);
        const uint32_t bar = bar0 + 8 * slot;
        if (lane == 0) mbar_expect_tx(bar, (uint32_t)(live * (len / 2 + 2 * (len / 32))));
        __syncwarp();
        if (copier && my_row >= 0)
            bulk_g2s(ring_s + slot * kSlotBytes + doff, gbase + (size_t)my_row * grow + k0 / kdiv, (uint32_t)(len / kdiv),
                     bar);
        if (++ij == nsl) {
            ij = 0;
            ++iu;
            if (iu < u1) {
                my_row = copier ? unit_row(iu, my_r) : -1;
                live = unit_live_rows(iu);
            }
        }
        ++it_;
    };

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    // Wide units send only their first slot's copies before the limb preparation:
    // with every warp queueing its whole ring at once the copy queue fills and the
    // issuing lanes wait, which would hold the preparation back; the rest follow
    // it.  Narrow units, whose warps have few steps, queue their whole ring now.
    constexpr int kPreStages = kRU >= 4 ? 1 : kStages;
    for (int t = 0; t < kPreStages && t < steps; ++t) issue_next();

    // fixed-point limbs of x, one warp per lane-chunk, one lane per value, on the
    // bf16 fields alone: x = sign * M * 2^(e-134), M = 128 + mantissa (e >= 1) or
    // the mantissa (e = 0, subnormal, read with e = 1).  With emax the chunk's
    // largest e, F = x * 2^(23-E), E = emax - 126, is sign * M * 2^(e - emax + 15):
    // a left shift when e >= emax - 15 (exact), else a right shift rounded to nearest even.
    // (loads are issued sixteen lane-chunks at a time so that one L2 round trip
    // covers all of them)
    constexpr int kPrepBatch = 16;
    for (int lc0 = warp; lc0 < nch * 32; lc0 += W * kPrepBatch) {
      uint32_t hb[kPrepBatch];
#pragma unroll
      for (int i = 0; i < kPrepBatch; ++i) {
          const int lc = lc0 + i * W;
          const int k = (lc >> 5) * kChunk + (lc & 31) * 32 + lane;
          hb[i] = (lc < nch * 32 && k < K) ? (uint32_t)a.x[k] : 0u;
      }
#pragma unroll
      for (int i = 0; i < kPrepBatch; ++i) {
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
        int F;
        if (sh >= 0) {
            F = M << sh;
        } else if (sh > -9) {
            const int d = -sh;
            F = (M + (1 << (d - 1)) - 1 + ((M >> d) & 1)) >> d;
        } else {
            F = 0;
        }
        if (h & 0x8000u) F = -F;
        if (bad) F = 0;
        const int w = lane >> 3, p = lane & 1, byte = (lane & 7) >> 1;
        uint8_t *base = limbs + (size_t)(c * 6 * 32 + l) * 16 + w * 4 + byte;
        base[(size_t)(0 * 2 + p) * 32 * 16] = (uint8_t)(F & 0xFF);
        base[(size_t)(1 * 2 + p) * 32 * 16] = (uint8_t)((F >> 8) & 0xFF);
        base[(size_t)(2 * 2 + p) * 32 * 16] = (uint8_t)((F >> 16) & 0xFF);
        float sx = bf16_bits_to_f32(h);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sx += __shfl_down_sync(0xFFFFFFFFu, sx, o);
        if (lane == 0) {
            Xs[lc] = sx;
            // 2^(E-23) = 2^(emax-149); normal for emax >= 23, the exact subnormal below
            Ss[lc] = bad ? __int_as_float(0x7FC00000) : (emax >= 23 ? __int_as_float((emax - 22) << 23) : ldexpf(1.0f, emax - 149));
        }
      }
    }
    __syncthreads();
    for (int t = kPreStages; t < kStages && t < steps; ++t) issue_next();

    float acc[kRU];
#pragma unroll
    for (int r = 0; r < kRU; ++r) acc[r] = 0.0f;
    uint64_t best = 0;   // fused head: the largest argmax key of the rows this warp wrote
    int u = u0, j = 0, slot = 0;
    uint32_t par = 0;
    const uint4 *limb_l = reinterpret_cast<const uint4 *>(limbs) + lane;

    for (int t = 0; t < steps; ++t) {
        const bool ok = __all_sync(0xFFFFFFFFu, wait_slot(bar0 + 8 * slot, par, failed ? 64 : kSpinLimit));
        failed = failed || !ok;
        const uint8_t *sl = ring + slot * kSlotBytes;
        const uint4 *ql = reinterpret_cast<const uint4 *>(sl) + lane;
        const uint16_t *sc16 = reinterpret_cast<const uint16_t *>(sl + kRU * kSlotQ) + (lane >> 1);
#pragma unroll
        for (int cc = 0; cc < kKS / kChunk; ++cc) {
            const int c = j * (kKS / kChunk) + cc;
            if (c * kChunk + lane * 32 >= K) break;   // lanes past the end of a short last chunk
            uint4 lm[6];
#pragma unroll
            for (int q = 0; q < 6; ++q) lm[q] = limb_l[(c * 6 + q) * 32];
            const float X = Xs[c * 32 + lane];
            const float scale = Ss[c * 32 + lane];
#pragma unroll
            for (int r = 0; r < kRU; ++r) {
                const uint4 qv = ql[(r * kSlotQ + cc * (kChunk / 2)) / 16];
                const float s = bf16_bits_to_f32(sc16[r * (kKS / kGroup) + cc * 16]);
                const float b = bf16_bits_to_f32(sc16[kRU * (kKS / kGroup) + r * (kKS / kGroup) + cc * 16]);
                const float P = lane_chunk_idot(qv, lm);
                acc[r] = fmaf(s, P * scale, acc[r]);   // P * 2^(E-23): exact power-of-two scaling
                acc[r] = fmaf(b, X, acc[r]);
            }
        }
        if (++j == nsl) {
            float tot[kRU];
#pragma unroll
            for (int r = 0; r < kRU; ++r) {
                tot[r] = warp_sum_to_lane0(acc[r]);
                acc[r] = 0.0f;
            }
            if (lane == 0) {
                if (a.glu) {
#pragma unroll
                    for (int p = 0; p < kRU / 2; ++p) {
                        const int col = u * kCols + p;
                        if (col < a.seg.ncols) {
                            const float g = bf16_bits_to_f32(f32_to_bf16_rne(tot[2 * p]));
                            const float uu = bf16_bits_to_f32(f32_to_bf16_rne(tot[2 * p + 1]));
                            a.y[col] = failed ? (uint16_t)TF_NAN_BF16 : f32_to_bf16_rne(glu_f32(g, uu));
                        }
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < kRU; ++r) {
                        const int col = u * kRU + r;
                        if (col < a.seg.ncols) {
                            const uint16_t h = failed ? (uint16_t)TF_NAN_BF16 : f32_to_bf16_rne(tot[r]);
                            a.y[col] = h;
                            if (a.cand) best = umax64(best, cand_key(h, a.id_base + (uint32_t)col));
                        }
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
    // every issued slot was waited on above unless a wait gave up; then give the
    // outstanding copies a bounded chance to land before shared memory is released
    if (failed) {
        for (int s2 = 0; s2 < kStages; ++s2) wait_slot(bar0 + 8 * s2, 0, 1024);
    }
    if (a.cand) {
        // fused head: publish this warp's best key; the last CTA to finish reduces all
        // of them into the argmax word (fence, then a ticket: the usual last-block pattern)
        if (lane == 0) a.cand[gw] = best;
        __threadfence();
        __syncthreads();
        __shared__ unsigned int ticket;
        if (tid == 0) ticket = atomicAdd(a.done, 1u);
        __syncthreads();
        if (ticket == gridDim.x - 1) {
            __threadfence();
            const int ncand = (int)(gridDim.x * W);
            uint64_t v = 0;
            for (int i = tid; i < ncand; i += blockDim.x) v = umax64(v, ((volatile uint64_t *)a.cand)[i]);
            v = warp_max64(v);
            __shared__ uint64_t red[32];
            if (lane == 0) red[warp] = v;
            __syncthreads();
            if (warp == 0) {
                v = lane < W ? red[lane] : 0ull;
                v = warp_max64(v);
                if (lane == 0) {
                    *a.word = word_of_key(v, a.y, a.id_base);
                    *a.done = 0u;
                }
            }
        }
    }
}

// The widest warp count whose shared memory fits 227 KB with 1 KB left for the
// kernel's static shared memory.
static int stream_warps(int K, int ru) {
    for (int w = kMaxWarps; w >= 4; --w)
        if (stream_layout(K, w, ru).total <= 226 * 1024) return w;
    return 0;
}

// K % 512 == 0 (every slot piece is a multiple of 16 B) and 16-byte aligned
// code, scale and bias arrays: the bulk copies' requirements.
bool qmm_m1_stream_eligible(const QmmArgs &a) {
    if (a.M != 1 || a.K % 512 != 0) return false;
    if (!aligned(a.scales, 16) || !aligned(a.biases, 16) || !aligned(a.wq, 16)) return false;
    return stream_warps(a.K, 4) > 0;
}

static size_t g_stream_smem_set[64][3];

template <int RU>
static cudaError_t launch_ru(const QmmArgs &a, int ri, cudaStream_t stream) {
    const int W = stream_warps(a.K, RU);
    const StreamLayout L = stream_layout(a.K, W, RU);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (g_stream_smem_set[dev][ri] < L.total) {
        cudaError_t e = cudaFuncSetAttribute(qmm_m1_stream_kernel<RU>, cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
        if (e != cudaSuccess) return e;
        g_stream_smem_set[dev][ri] = 226 * 1024;
    }
    const int units = a.glu ? (a.seg.ncols + RU / 2 - 1) / (RU / 2) : (a.seg.ncols + RU - 1) / RU;
    int blocks = num_sms();
    const int need = (units + W - 1) / W;
    if (need < blocks) blocks = need;
    qmm_m1_stream_kernel<RU><<<blocks, W * 32, L.total, stream>>>(a, units);
    return cudaGetLastError();
}

// Rows per unit only change how often a lane reuses its activation limbs, never a
// row's arithmetic, so the choice may follow N: four rows while every warp of the
// grid still gets two units, fewer when the slice is narrow.
cudaError_t launch_qmm_m1_stream(const QmmArgs &a, cudaStream_t stream) {
    const long long warps = (long long)num_sms() * stream_warps(a.K, 4);
    const long long rows = a.glu ? 2ll * a.seg.ncols : a.seg.ncols;
    if (rows >= 8 * warps) return launch_ru<4>(a, 0, stream);
    if (rows >= 2 * warps || a.glu) return launch_ru<2>(a, 1, stream);
    return launch_ru<1>(a, 2, stream);
}

int qmm_m1_stream_max_cand() { return num_sms() * kMaxWarps; }

}  // namespace tf
