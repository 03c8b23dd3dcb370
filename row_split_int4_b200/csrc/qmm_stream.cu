// qmm_stream.cu -- M = 1 dequant-GEMV: weights streamed through shared memory by
// bulk asynchronous copies, dot products taken exactly in integer arithmetic.
//
// Why this shape on B200.  At M = 1 every weight byte is used once, and the 148
// SMs must turn ~40 weights per clock each into products to keep up with HBM.
// Two limits meet there:
//   * bytes in flight: ~130 KB per SM are needed to cover HBM latency under
//     load.  Copies land in shared-memory rings through the TMA engine, so they
//     stay in flight while the warps compute, independent of the register budget.
//     Wide calls use the tile ring (2-D tensor copies of 16-row tiles filled by
//     producer warps, below); narrow ones a ring per warp refilled by 1-D
//     cp.async.bulk copies, one per row and array;
//   * instructions per weight: floating-point nibble decoding costs 3-4 issue
//     slots per weight, most of them integer-pipe work.  Here a word of 8 codes
//     is split into two words of 4 bytes (2 lop3 + 1 shift) and multiplied with
//     the activations by dp4a, 4 products and their sum per instruction, in exact
//     integer arithmetic.
//
// Integer dot (per lane-chunk: the 32 x a lane meets in one 1,024-K chunk).
// The 32 bf16 x are put in fixed point with the chunk's own exponent E (every
// |x| < 2^E, E the smallest such over the chunk): F = x * 2^(23-E), |F| < 2^23,
// exact for every x within 2^15 of the chunk's largest magnitude and rounded to
// nearest even below (an error under 2^-23 of the largest |x|).  F is kept as
// three bytes, F = L2*2^16 + L1*2^8 + L0 (L2 signed), and with the code written
// as q = (q - 8) + 8 and the weight as w = s (q - 8) + (b + 8 s),
//     P' = sum (q - 8) F = 2^16 sum q L2 + 2^8 sum q L1 + sum q L0 - 8 sum F
// comes from three int32 dp4a accumulators that cannot overflow (32 * 15 * 255 <
// 2^17); |P'| < 2^31, so P' is exact in int32 and is rounded once to fp32.  The
// lane adds s * 2^(E-23) * P' and (b + 8 s) * X, X = 2^(E-23) sum F = the sum of
// the 32 x rounded once.  Taking the code about its middle keeps the two terms
// near the size of their sum for the usual bias b ~ -8 s, where s q and b alone
// would be large terms that cancel.
// A lane-chunk dominated by one or two outliers (at most two nonzero x within
// 2^4 of its largest, and smaller nonzero x beside them) keeps its 32 raw x
// instead of limbs, and the warp takes it element by element: lane j forms
// w_j = s q_j + b and x_j w_j in fp32, a fixed butterfly adds the 32 products,
// and the owning lane adds the sum -- a plain fp32 dot for that lane-chunk, so
// an outlier whose weight is zero adds exactly nothing and sets no grid for the
// others.
// A chunk holding NaN or +-Inf gets the scale NaN, so the row's result is NaN.
//
// Order of every operation depends on K alone, never on the rows a launch
// covers, so split == whole holds bit for bit.  K is cut into slices of chunks
// (slice_chunks: the whole K up to 8 chunks, else 4 chunks = 4,096 K, the last
// one shorter); over a slice each lane adds its lane-chunks' terms in ascending
// chunk order, the shuffle tree of qmm_gemv.cu joins the 32 lanes, and the row
// total is the slices' sums added in ascending order.  A slice is the unit in
// which the narrow-call kernel below shares a row's K among warps.
//
// Slot (kRU rows x kKS values of K):
//   [codes of row 0 (kKS/2 B)] .. [codes of row kRU-1] [scales, kKS/32 B per row] [biases]
// A unit is kRU rows: four consecutive output columns (TF_EPI_NONE), or the
// gate and up rows of two consecutive columns (TF_EPI_GLU, rows g0 u0 g1 u1).
#include "qmm_common.cuh"
#include "stream_common.cuh"
#include "tmap.h"

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
    size_t limb_off, cst_off, wm_off, tot_off, bar_off, ring_off, total;
};

__host__ __device__ inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared memory for K and a warp count; the widest that fits is chosen on the host.
__host__ __device__ inline StreamLayout stream_layout(int K, int warps, int ru) {
    StreamLayout L;
    L.nch = (K + kChunk - 1) / kChunk;
    L.warps = warps;
    L.limb_off = 0;
    L.cst_off = round_up(L.limb_off + (size_t)L.nch * 32 * kLimbBytes, 128);
    L.wm_off = L.cst_off + (size_t)L.nch * 32 * 16;
    L.tot_off = round_up(L.wm_off + (size_t)L.nch * 4, 16);
    L.bar_off = round_up(L.tot_off + (size_t)warps * 4 * 4, 128);
    L.ring_off = round_up(L.bar_off + (size_t)warps * stages_for(ru) * 8, 128);
    L.total = L.ring_off + (size_t)warps * stages_for(ru) * slot_bytes(ru);
    return L;
}

// P' = sum over the lane's 32 codes of (q_k - 8) F_k, exact (see above); sf8 = 8 sum F.
// limb[j] (j = limb*2 + parity) holds in word w the limb bytes of x[8w+p],
// x[8w+p+2], x[8w+p+4], x[8w+p+6]; the even codes of word w are its low nibbles,
// the odd codes its high nibbles.
__device__ __forceinline__ int lane_chunk_pq(const uint4 &q, const uint4 *limb, uint32_t sf8) {
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
    // modulo 2^32; the true value fits int32, so the wrap-around is exact
    return (int)(((uint32_t)a2 << 16) + ((uint32_t)a1 << 8) + (uint32_t)a0 - sf8);
}

// What a lane needs of its lane-chunk c: limbs and the constants the limb
// preparation left in cst (the scale 2^(E-23), X and 8 sum F as one 16-byte
// vector; all three zero for a lane-chunk taken in fp32, NaN scale for a
// non-finite x).
struct LaneChunk {
    uint4 lm[6];
    float scale, X;
    uint32_t sf8;
};
__device__ __forceinline__ void load_lane_chunk(LaneChunk &t, const uint4 *limb_l, const uint4 *cst, int c, int lane) {
#pragma unroll
    for (int q = 0; q < 6; ++q) t.lm[q] = limb_l[(c * 6 + q) * 32];
    const uint4 v = cst[c * 32 + lane];
    t.scale = __uint_as_float(v.x);
    t.X = __uint_as_float(v.y);
    t.sf8 = v.z;
}

// acc += the lane's x.w over lane-chunk t for a row with codes qv, scale s, bias b
// (a lane-chunk taken in fp32 has scale and X zero here and adds nothing).
__device__ __forceinline__ float lane_chunk_fma(float acc, const uint4 &qv, const LaneChunk &t, float s, float b) {
    const int P = lane_chunk_pq(qv, t.lm, t.sf8);
    acc = fmaf(s, __int2float_rn(P) * t.scale, acc);   // P' * 2^(E-23): exact power-of-two scaling
    return fmaf(fmaf(8.0f, s, b), t.X, acc);            // b + 8 s
}

// Element `lane` of the wide lane-chunk (c, l), from the raw bf16 x it keeps in
// place of its limbs (value j in 16-byte vector j / 8 of the lane-chunk).
__device__ __forceinline__ float wide_x(const uint8_t *limbs, int c, int l, int lane) {
    const uint16_t *v = reinterpret_cast<const uint16_t *>(limbs + ((size_t)(c * 6 + (lane >> 3)) * 32 + l) * 16);
    return bf16_bits_to_f32(v[lane & 7]);
}

// The x.w of a wide lane-chunk for one row, lane j taking element j: word = code
// word j / 8 of the lane-chunk, s and b its group's scale and bias.  w = s q + b
// and x w in fp32, then a butterfly over the warp adds the 32 products (every
// lane ends with the same sum, so the order is fixed).
__device__ __forceinline__ float wide_dot(float xj, uint32_t word, int lane, float s, float b) {
    const float q = (float)((word >> (4 * (lane & 7))) & 15u);
    float p = xj * fmaf(s, q, b);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xFFFFFFFFu, p, o);
    return p;
}

// Fixed-point limbs of x for every lane-chunk, on the bf16 fields alone: x = sign *
// M * 2^(e-134), M = 128 + mantissa (e >= 1) or the mantissa (e = 0, subnormal, read
// with e = 1).  With emax the chunk's largest e, F = x * 2^(23-E), E = emax - 126,
// is sign * M * 2^(e - emax + 15): a left shift when e >= emax - 15 (exact), else
// a right shift rounded to nearest even (an error below 2^-23 of the largest |x|,
// the size of an fp32 rounding of a sum that holds the largest product).
// A lane-chunk goes to the fp32 pass (its 32 raw x where its limbs would be, its
// constants zero, its bit set in wmask[c]) when one or two values dominate it --
// at most two nonzero x within 2^4 of the largest and some smaller nonzero x: an
// outlier whose weight may be zero would otherwise set the grid of the others and
// ride in both integer terms.  cst gets (2^(E-23), X = 2^(E-23) sum F, 8 sum F, 0)
// per lane-chunk (|sum F| < 2^28; the scale NaN when the chunk holds a NaN or an
// infinity).
__device__ __forceinline__ void prep_limbs(const uint16_t *x, int K, int nch, uint8_t *limbs, uint4 *cst, uint32_t *wmask,
                                           int W, int warp, int lane) {
    // Four threads per lane-chunk, each with 8 of its values (one 16-byte load, one
    // word of every limb vector), the lane-chunk's largest exponent, counts and sum
    // joined by shuffles within the four; all threads of the CTA take part, so the
    // preparation is short next to the first ring fill.
    const bool x16 = (reinterpret_cast<uintptr_t>(x) & 15) == 0;
    uint8_t *wm8 = reinterpret_cast<uint8_t *>(wmask);   // byte j of chunk c: lane-chunks 8j .. 8j + 7
    const int nu = nch * 128, stride = W * 32;
    // a thread's units in batches of four, each batch's loads issued together
    for (int ub = warp * 32 + lane; ub < nu; ub += 4 * stride) {
        uint32_t xb[4][4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int u = ub + b * stride;
            const int lc = u >> 2, w = u & 3, c = lc >> 5, l = lc & 31;
            const int k0 = c * kChunk + l * 32 + w * 8;
            if (u < nu && x16 && k0 + 8 <= K) {
                const uint4 v = *reinterpret_cast<const uint4 *>(x + k0);
                xb[b][0] = v.x;
                xb[b][1] = v.y;
                xb[b][2] = v.z;
                xb[b][3] = v.w;
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t lo = u < nu && k0 + 2 * i < K ? x[k0 + 2 * i] : 0u;
                    const uint32_t hi = u < nu && k0 + 2 * i + 1 < K ? x[k0 + 2 * i + 1] : 0u;
                    xb[b][i] = lo | (hi << 16);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int u = ub + b * stride;
            if (u >= nu) break;   // warp-uniform: nu is a multiple of 32
            const int lc = u >> 2, w = u & 3, c = lc >> 5, l = lc & 31;
            const uint32_t *hv = xb[b];   // values 8w .. 8w + 7 of the lane-chunk, two per word (zero past K)
            // largest magnitude field of the 8 values: the exponent sits above the
            // mantissa, so the largest field has the largest e (a subnormal reads e = 1)
            uint32_t mx = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) mx = __vmaxu2(mx, hv[i] & 0x7FFF7FFFu);
            mx = max(mx & 0xFFFFu, mx >> 16);
            int emax = mx == 0 ? 0 : max((int)(mx >> 7), 1);
            const int bad = (mx >> 7) == 0xFFu ? 1 : 0;   // an infinity or a NaN
            emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, 1));
            emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, 2));
            // F = x 2^(23-E) = x 2^(149-emax), by two exact power-of-two products in fp32
            // (the first only when 2^(149-emax) would not be a normal fp32), then one
            // conversion rounded to nearest even: exactly the integer shift above for
            // every x (sign * M * 2^sh, |F| < 2^23; below 1/2 when sh <= -9)
            const float pre = emax >= 22 ? 1.0f : __int_as_float(191 << 23);   // 2^64
            const float scl = __int_as_float((emax >= 22 ? 276 - emax : 212 - emax) << 23);
            int F[8];
            // cnt: nonzero x within 2^4 of the largest (bits 0..7), smaller ones (8..15),
            // bad (16..); the sum of F in wrapping arithmetic (an infinity converts to
            // 2^31 - 1; such a lane-chunk's sum is never used)
            int cnt = 0;
            uint32_t sfu = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const uint32_t hw = hv[t >> 1];
                const uint32_t h = (t & 1) ? hw >> 16 : hw & 0xFFFFu;
                const float xf = __uint_as_float((t & 1) ? hw & 0xFFFF0000u : hw << 16);
                F[t] = __float2int_rn((xf * pre) * scl);
                const uint32_t mag = h & 0x7FFFu;
                if (mag != 0) cnt += max((int)(mag >> 7), 1) >= emax - 3 ? 1 : 256;   // sh >= 12
                sfu += (uint32_t)F[t];
            }
            // value 8w + t: byte t >> 1 of word w of limb vectors 2 limb + (t & 1); byte
            // `limb` of the two's complement F
            uint32_t L[6];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint32_t lo = __byte_perm(F[p], F[p + 2], 0x5140), hi = __byte_perm(F[p + 4], F[p + 6], 0x5140);
                const uint32_t lo2 = __byte_perm(F[p], F[p + 2], 0x7362), hi2 = __byte_perm(F[p + 4], F[p + 6], 0x7362);
                L[0 + p] = __byte_perm(lo, hi, 0x5410);
                L[2 + p] = __byte_perm(lo, hi, 0x7632);
                L[4 + p] = __byte_perm(lo2, hi2, 0x5410);
            }
            cnt += bad << 16;
            cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, 1);
            cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, 2);
            sfu += __shfl_xor_sync(0xFFFFFFFFu, sfu, 1);
            sfu += __shfl_xor_sync(0xFFFFFFFFu, sfu, 2);
            const int sf = (int)sfu;
            const bool any_bad = (cnt >> 16) != 0;
            const bool fallback = !any_bad && (cnt & 0xFF) <= 2 && ((cnt >> 8) & 0xFF) > 0;
            uint4 *dst = reinterpret_cast<uint4 *>(limbs) + (size_t)c * 6 * 32 + l;
            if (fallback) {
                dst[w * 32] = make_uint4(hv[0], hv[1], hv[2], hv[3]);   // values 8w .. 8w + 7 in vector w
            } else {
#pragma unroll
                for (int q = 0; q < 6; ++q) reinterpret_cast<uint32_t *>(dst + q * 32)[w] = L[q];
            }
            if (w == 0) {
                if (fallback) {
                    cst[lc] = make_uint4(0u, 0u, 0u, 0u);
                } else {
                    // 2^(E-23) = 2^(emax-149); normal for emax >= 23, the exact subnormal below
                    const float scale = any_bad ? __int_as_float(0x7FC00000)
                                                : (emax >= 23 ? __int_as_float((emax - 22) << 23) : ldexpf(1.0f, emax - 149));
                    const int sfv = any_bad ? 0 : sf;
                    cst[lc] = make_uint4(__float_as_uint(scale), __float_as_uint(__int2float_rn(sfv) * scale),
                                         (uint32_t)sfv << 3, 0u);
                }
            }
            // the warp's 32 threads hold 8 lane-chunks of chunk c (l of lane 0 a multiple of 8)
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, fallback && w == 0);
            if (lane == 0) {
                uint32_t m8 = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) m8 |= ((bal >> (4 * j)) & 1u) << j;
                wm8[c * 4 + (l >> 3)] = (uint8_t)m8;
            }
        }
    }
}

// Fused head: every warp of the grid publishes the largest argmax key of the rows
// it wrote (0 when it wrote none); argmax_keys_kernel turns them into the word.
__device__ __forceinline__ void fused_head_keys(const QmmArgs &a, uint64_t best, int W, int warp, int lane) {
    if (lane == 0) a.cand[(long long)blockIdx.x * W + warp] = best;
}

// The word of one slice from the qmm grid's ncand warp keys: max over them (the
// argmax order is the keys' unsigned order, so any tree gives the same key), the
// winning value read back from the logits.  One CTA of kKeyThreads threads: the
// keys are L2-resident, so the time is a few load latencies, and more threads
// mean fewer of them (measured inside the decode step: 1,024 threads 0.2038
// ms/step against 0.2086 with a 128-thread CTA small enough to sit beside a qmm
// CTA).
constexpr int kKeyThreads = 1024;
__global__ void __launch_bounds__(kKeyThreads) argmax_keys_kernel(const uint64_t *cand, int ncand, const uint16_t *logits,
                                                                  uint32_t id_base, uint64_t *word) {
    pdl_trigger();
    pdl_wait();
    // up to eight loads in flight per thread
    uint64_t v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int i = threadIdx.x;
    for (; i + 7 * kKeyThreads < ncand; i += 8 * kKeyThreads) {
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = umax64(v[u], cand[i + u * kKeyThreads]);
    }
    for (; i < ncand; i += kKeyThreads) v[0] = umax64(v[0], cand[i]);
#pragma unroll
    for (int u = 1; u < 8; ++u) v[0] = umax64(v[0], v[u]);
    uint64_t best = warp_max64(v[0]);
    __shared__ uint64_t red[kKeyThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = best;
    __syncthreads();
    if (warp == 0) {
        best = lane < kKeyThreads / 32 ? red[lane] : 0ull;
        best = warp_max64(best);
        if (lane == 0) *word = word_of_key(best, logits, id_base);
    }
}

// Chunks per K-slice (see the reduction order above).
__host__ __device__ constexpr int slice_chunks(int nch) { return nch <= 8 ? nch : 4; }
__device__ __forceinline__ bool slice_end(int c, int sc, int nch) {
    return c + 1 == nch || (sc == 4 && (c & 3) == 3);   // sc is nch or 4
}
// At the end of a slice: the 32 lanes' sums of the slice by the tree into lane 0,
// which adds them to the row's total (the first slice starts it).  The totals
// live in shared memory, one float per row of the warp, read by lane 0 alone:
// registers are the kernels' scarce resource.
__device__ __forceinline__ void slice_fold(float &acc, float *tot, int c, int sc, int lane) {
    const float v = warp_sum_to_lane0(acc);
    if (lane == 0) *tot = c < sc ? v : *tot + v;
    acc = 0.0f;
}

// acc[r] += the x.w of unit row r over the chunks of one slot: chunk c0 + cc sits
// at position cc of the slot.  A lane whose 32 values start at or past kend (K
// covered by the slot) adds nothing there.  Full slots pass compile-time nc and
// kend, so their bounds fold away.
template <int kRU>
__device__ __forceinline__ void slot_dot(float (&acc)[kRU], const uint8_t *sl, const uint8_t *limbs, const uint4 *cst,
                                         const uint32_t *wms, int c0, int nc, int kend, int lane) {
    const uint4 *ql = reinterpret_cast<const uint4 *>(sl) + lane;
    const uint16_t *sc0 = reinterpret_cast<const uint16_t *>(sl + kRU * kSlotQ);
    const uint16_t *sc16 = sc0 + (lane >> 1);
    const uint4 *limb_l = reinterpret_cast<const uint4 *>(limbs) + lane;
#pragma unroll
    for (int cc = 0; cc < kKS / kChunk; ++cc) {
        if (cc >= nc) break;
        const int c = c0 + cc;
        const bool live = cc * kChunk + lane * 32 < kend;
        LaneChunk t;
        load_lane_chunk(t, limb_l, cst, c, lane);
        const uint32_t wm = wms[c];
        if (live) {
#pragma unroll
            for (int r = 0; r < kRU; ++r) {
                const uint4 qv = ql[(r * kSlotQ + cc * (kChunk / 2)) / 16];
                const float s = bf16_bits_to_f32(sc16[r * (kKS / kGroup) + cc * 16]);
                const float b = bf16_bits_to_f32(sc16[kRU * (kKS / kGroup) + r * (kKS / kGroup) + cc * 16]);
                acc[r] = lane_chunk_fma(acc[r], qv, t, s, b);
            }
        }
        for (uint32_t m = wm; m != 0; m &= m - 1) {   // wide lane-chunks, warp-uniform
            const int l = __ffs(m) - 1;
            const float xj = wide_x(limbs, c, l, lane);
#pragma unroll
            for (int r = 0; r < kRU; ++r) {
                const uint32_t word =
                    reinterpret_cast<const uint32_t *>(sl)[((r * kSlotQ + cc * (kChunk / 2)) / 16 + l) * 4 + (lane >> 3)];
                const float s = bf16_bits_to_f32(sc0[r * (kKS / kGroup) + cc * 16 + (l >> 1)]);
                const float b = bf16_bits_to_f32(sc0[kRU * (kKS / kGroup) + r * (kKS / kGroup) + cc * 16 + (l >> 1)]);
                const float d = wide_dot(xj, word, lane, s, b);
                if (lane == l) acc[r] += d;
            }
        }
    }
}

// ------------------------------------------------------------------ kernel --
// kOne: the whole K is one slice, folded once after the unit's last slot.
template <int kRU, bool kOne>
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
    uint4 *csts = reinterpret_cast<uint4 *>(smem + L.cst_off);
    uint32_t *wms = reinterpret_cast<uint32_t *>(smem + L.wm_off);
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
    const int kshift = my_a == 0 ? 1 : 5;                                // bytes of a K range = len >> kshift
    const uint32_t doff = my_a == 0 ? my_r * kSlotQ
                        : (my_a == 1 ? kRU * kSlotQ + my_r * kSlotS : kRU * kSlotQ + kRU * kSlotS + my_r * kSlotS);
    const int len_last = K - (nsl - 1) * kKS;                            // K of the last slice
    const uint32_t piece_full = (uint32_t)kKS >> kshift, piece_last = (uint32_t)len_last >> kshift;
    constexpr uint32_t kTxFull = kKS / 2 + kKS / 16;                     // bytes of one unit row, full slice
    const uint32_t tx_last = (uint32_t)(len_last / 2 + len_last / 16);
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
    // issue state: unit iu, slice ij go out next, into ring slot islot; csrc is
    // this lane's matrix row of unit iu (null: nothing to copy)
    int iu = u0, ij = 0, islot = 0, issued = 0, live = 0;
    const uint8_t *csrc = nullptr;
    auto set_issue_unit = [&](int uu) {
        const int row = copier ? unit_row(uu, my_r) : -1;
        csrc = row >= 0 ? gbase + (size_t)row * grow : nullptr;
        live = unit_live_rows(uu);
    };
    if (u0 < u1) set_issue_unit(u0);
    bool failed = false;
    auto issue_next = [&]() {
        const bool last = ij == nsl - 1;
        const uint32_t bar = bar0 + 8 * islot;
        if (lane == 0) mbar_expect_tx(bar, (uint32_t)live * (last ? tx_last : kTxFull));
        __syncwarp();
        if (csrc != nullptr)
            bulk_g2s(ring_s + islot * kSlotBytes + doff, csrc + (size_t)ij * piece_full, last ? piece_last : piece_full, bar);
        islot = islot + 1 == kStages ? 0 : islot + 1;
        ++issued;
        if (++ij == nsl) {
            ij = 0;
            if (++iu < u1) set_issue_unit(iu);
        }
    };

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    // While the kernel before this one may still run: the warp's first ring of
    // weights into L2 (never written by the library's kernels; an L2 prefetch
    // cannot see stale data in any case).
    {
        int pu = u0, pj = 0;
        const uint8_t *psrc = csrc;
        for (int i = 0; i < kStages && i < steps; ++i) {
            if (psrc != nullptr)
                l2_prefetch(psrc + (size_t)pj * piece_full, pj == nsl - 1 ? piece_last : piece_full);
            if (++pj == nsl) {
                pj = 0;
                if (++pu >= u1) break;
                const int row = copier ? unit_row(pu, my_r) : -1;
                psrc = row >= 0 ? gbase + (size_t)row * grow : nullptr;
            }
        }
    }
    pdl_wait();
    pdl_trigger();
    // Wide units send only their first slot's copies before the limb preparation:
    // with every warp queueing its whole ring at once the copy queue fills and the
    // issuing lanes wait, which would hold the preparation back; the rest follow
    // it.  Narrow units, whose warps have few steps, queue their whole ring now.
    constexpr int kPreStages = kRU >= 4 ? 1 : kStages;
    while (issued < kPreStages && issued < steps) issue_next();

    prep_limbs(a.x, K, nch, limbs, csts, wms, W, warp, lane);
    __syncthreads();
    while (issued < kStages && issued < steps) issue_next();

    float acc[kRU];
#pragma unroll
    for (int r = 0; r < kRU; ++r) acc[r] = 0.0f;
    float *tot = reinterpret_cast<float *>(smem + L.tot_off) + warp * 4;   // lane 0's row totals
    const int sc = slice_chunks(nch);
    uint64_t best = 0;   // fused head: the largest argmax key of the rows this warp wrote
    int slot = 0;
    uint32_t par = 0;
    const int nc_last = (len_last + kChunk - 1) / kChunk;

    for (int u = u0; u < u1; ++u) {
        for (int j = 0; j < nsl; ++j) {
            const bool ok = __all_sync(0xFFFFFFFFu, wait_slot(bar0 + 8 * slot, par, failed ? 64 : kSpinLimit));
            failed = failed || !ok;
            const uint8_t *sl = ring + slot * kSlotBytes;
            if (j + 1 < nsl)
                slot_dot<kRU>(acc, sl, limbs, csts, wms, j * (kKS / kChunk), kKS / kChunk, kKS, lane);
            else
                slot_dot<kRU>(acc, sl, limbs, csts, wms, j * (kKS / kChunk), nc_last, len_last, lane);
            if (++slot == kStages) {
                slot = 0;
                par ^= 1u;
            }
            __syncwarp();
            if (issued < steps && !failed) issue_next();
            // slices end at slot ends (slots of 2 chunks, slices of 4 or the whole K)
            if (!kOne) {
                const int c_last = min(j * (kKS / kChunk) + kKS / kChunk, nch) - 1;
                if (slice_end(c_last, sc, nch)) {
#pragma unroll
                    for (int r = 0; r < kRU; ++r) slice_fold(acc[r], tot + r, c_last, sc, lane);
                }
            }
        }
        if (kOne) {
#pragma unroll
            for (int r = 0; r < kRU; ++r) slice_fold(acc[r], tot + r, nch - 1, sc, lane);
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
    }
    // every issued slot was waited on above unless a wait gave up; then give the
    // outstanding copies a bounded chance to land before shared memory is released
    if (failed) {
        for (int s2 = 0; s2 < kStages; ++s2) wait_slot(bar0 + 8 * s2, 0, 1024);
    }
    if (a.cand) fused_head_keys(a, best, W, warp, lane);
}

// ---------------------------------------------------------- tile ring --
// The wide M = 1 kernel.  A per-warp ring refilled by one 1-D bulk copy per row
// and array spends ~15 issue slots on every copy instruction, a tenth of all the
// kernel issues at 12 copies per 4-row step, and keeps only half of its shared
// memory in flight.  Here sixteen compute warps form four groups of four; each
// group owns a ring of slots of one tile (16 matrix rows, or 8 GLU columns' gate and
// up rows) by one chunk of K, and a producer warp of its own fills a slot with one
// 2-D tensor copy per array (codes, scales, biases), so three copy instructions
// move 9 KB, and no compute warp ever waits to refill a slot.  The group's four warps take four rows each from every slot, exactly as the
// per-warp kernel takes a unit's rows (the per-lane arithmetic, its order and the
// shuffle tree are the same code, so both kernels give the same bits), and each
// warp frees a slot by one arrival on the slot's empty barrier.  Tiles are
// claimed in order from the CTA's share by a counter in shared memory, so the
// groups stay busy to the end of the share.
// A tile is 4 kWR rows by 4 / kWR chunks of K: kWR = 4 (16 rows by 1,024) for wide
// calls, kWR = 1 (4 rows by 4,096) for calls with few rows (down and attn_out
// halves), so that the four groups of every SM still find tiles.  Every slot
// holds 9,216 bytes, and each compute warp takes kWR rows of it.
constexpr int kTGroups = 4, kTGroupWarps = 4, kTWarps = kTGroups * kTGroupWarps;   // compute warps
constexpr int kTThreads = (kTWarps + kTGroups) * 32;          // and one producer warp per group
constexpr int kTSlotBytes = 16 * (kChunk / 2 + 2 * (kChunk / 32));   // 9,216
template <int kWR> struct TileShape {
    static constexpr int rows = kTGroupWarps * kWR;          // rows of a tile
    static constexpr int cps = 4 / kWR;                      // chunks per slot
    static constexpr int q = cps * (kChunk / 2);             // code bytes of one row in a slot
    static constexpr int sb = cps * (kChunk / 32);           // scale (or bias) bytes of one row
    static constexpr int qelem = q > 1024 ? 8 : 4;           // code element of the tensor map (box <= 256)
    static_assert(rows * (q + 2 * sb) == kTSlotBytes, "slot size");
};
constexpr int kTMaxStages = 6;

struct TileLayout {
    int nch, stages;
    size_t limb_off, cst_off, wm_off, full_off, empty_off, hdr_off, ctl_off, tot_off, ring_off, total;
};

// Shared memory of the tile ring for K, `stages` slots per group and M activation
// rows (limbs, sums and scales of every row, row m at offset m times one row's).
__host__ __device__ inline TileLayout tile_layout(int K, int stages, int M = 1) {
    TileLayout L;
    L.nch = (K + kChunk - 1) / kChunk;
    L.stages = stages;
    L.limb_off = 0;
    L.cst_off = round_up(L.limb_off + (size_t)M * L.nch * 32 * kLimbBytes, 128);
    L.wm_off = L.cst_off + (size_t)M * L.nch * 32 * 16;
    L.full_off = round_up(L.wm_off + (size_t)M * L.nch * 4, 128);
    L.empty_off = L.full_off + (size_t)kTGroups * stages * 8;
    L.hdr_off = L.empty_off + (size_t)kTGroups * stages * 8;    // (tile, chunk) of each slot
    L.ctl_off = L.hdr_off + (size_t)kTGroups * stages * 8;      // claim counter, abort flag
    L.tot_off = L.ctl_off + 16;                                   // row totals: 8 floats per compute warp
    L.ring_off = round_up(L.tot_off + (size_t)kTWarps * 8 * 4, 128);
    L.total = L.ring_off + (size_t)kTGroups * stages * kTSlotBytes;
    return L;
}

// Tiles of a call: segment s (TF_EPI_NONE) owns tiles [tstart[s], tstart[s + 1]),
// tile i of it rows row0[s] + 16 i ...; a GLU call has one run of tiles over its
// columns, 8 columns a tile.
struct TilePlan {
    int tstart[TF_MAX_SEGS + 1];
    int ntiles;
};

__device__ __forceinline__ bool tile_wait(uint32_t bar, uint32_t parity, const volatile int *abort, long long limit) {
    for (long long it = 0; it < limit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255) == 255 && *abort) return false;
    }
    return false;
}

// Slot row of a warp's row r: rows kWR w .. kWR w + kWR - 1 (NONE); for GLU the gate
// rows sit in the first half of the slot and the up rows in the second, and row r
// is member r & 1 of column (kWR / 2) w + (r >> 1), the order the GLU epilogue reads.
template <bool kGlu, int kWR>
__device__ __forceinline__ int tile_row(int w, int r) {
    return kGlu ? (r & 1) * (2 * kWR) + (kWR / 2) * w + (r >> 1) : kWR * w + r;
}

// kOne: the whole K is one slice (at most 8 chunks), so the slice's tree sum is
// the tile's last step and needs no per-slot test.
template <bool kGlu, int kWR, int kM, bool kOne>
__global__ void __launch_bounds__(kTThreads, 1)
    qmm_m1_tile_kernel(QmmArgs a, TilePlan plan, const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap smap, const __grid_constant__ CUtensorMap bmap, int S) {
    extern __shared__ __align__(128) uint8_t smem[];
    const TileLayout L = tile_layout(a.K, S, kM);
    using Sh = TileShape<kWR>;
    static_assert(!kGlu || kWR >= 2, "a GLU column needs its gate and up rows in one warp");
    constexpr int kRows = Sh::rows, kCps = Sh::cps;
    const int K = a.K, nch = L.nch;
    const int nsl = (nch + kCps - 1) / kCps;   // slots of a tile
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool producer = warp >= kTWarps;
    const int grp = producer ? warp - kTWarps : warp / kTGroupWarps, w_in = warp % kTGroupWarps;
    uint8_t *limbs = smem + L.limb_off;
    uint4 *csts = reinterpret_cast<uint4 *>(smem + L.cst_off);
    uint32_t *wms = reinterpret_cast<uint32_t *>(smem + L.wm_off);
    int2 *hdr = reinterpret_cast<int2 *>(smem + L.hdr_off) + grp * S;
    int *claim = reinterpret_cast<int *>(smem + L.ctl_off);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.ctl_off) + 1;
    uint8_t *ring = smem + L.ring_off + (size_t)grp * S * kTSlotBytes;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t full0 = smem_addr(smem + L.full_off) + (uint32_t)(grp * S * 8);
    const uint32_t empty0 = smem_addr(smem + L.empty_off) + (uint32_t)(grp * S * 8);

    // this CTA's share of the tiles
    const int t0 = (int)((long long)blockIdx.x * plan.ntiles / gridDim.x);
    const int t1 = (int)((long long)(blockIdx.x + 1) * plan.ntiles / gridDim.x);

    if (tid == 0) {
        for (int i = 0; i < kTGroups * S; ++i) {
            mbar_init(smem_addr(smem + L.full_off) + 8 * i, 1);
            mbar_init(smem_addr(smem + L.empty_off) + 8 * i, kTGroupWarps);
        }
        claim[0] = 0;
        claim[1] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // first matrix row (both members for GLU) and first output column of tile t
    auto tile_rows = [&](int t, int &r_a, int &r_b, int &col, int &ncol) {
        if (kGlu) {
            r_a = a.seg.row0[0] + (kRows / 2) * t;
            r_b = a.seg.row0[1] + (kRows / 2) * t;
            col = (kRows / 2) * t;
            ncol = min(kRows / 2, a.seg.ncols - col);
        } else {
            // the last segment starting at or before t (selected without a
            // dynamic index into the parameter arrays)
            int ts = plan.tstart[0], row0 = a.seg.row0[0], col0 = a.seg.col0[0], nr = a.seg.nrows[0];
#pragma unroll
            for (int s2 = 1; s2 < TF_MAX_SEGS; ++s2)
                if (s2 < a.seg.nseg && t >= plan.tstart[s2]) {
                    ts = plan.tstart[s2];
                    row0 = a.seg.row0[s2];
                    col0 = a.seg.col0[s2];
                    nr = a.seg.nrows[s2];
                }
            const int i = t - ts;
            r_a = row0 + kRows * i;
            r_b = 0;
            col = col0 + kRows * i;
            ncol = min(kRows, nr - kRows * i);
        }
    };

    // issue state of the group's producer (lane 0): the tile being sent (-1: none
    // left), its next chunk, the slot and its use count
    int it_tile = -2, it_c = nsl, islot = 0, iuse = 0, nissued = 0;
    bool done_issuing = false;
    auto issue_next = [&]() {   // lane 0 of the producer warp only
        if (done_issuing) return;
        if (it_c == nsl) {
            const int t = t0 + atomicAdd(claim, 1);
            it_tile = t < t1 ? t : -1;
            it_c = 0;
        }
        const uint32_t full = full0 + 8 * islot, empty = empty0 + 8 * islot;
        if (iuse > 0 && !tile_wait(empty, (uint32_t)((iuse - 1) & 1), abort_flag, kSpinLimit)) {
            *abort_flag = 1;
            done_issuing = true;
            return;
        }
        hdr[islot] = make_int2(it_tile, it_c);
        if (it_tile >= 0) {
            int r_a, r_b, col, ncol;
            tile_rows(it_tile, r_a, r_b, col, ncol);
            mbar_expect_tx(full, (uint32_t)kTSlotBytes);
            const uint32_t dst = ring_s + islot * kTSlotBytes;
            constexpr uint32_t kS0 = kRows * Sh::q, kB0 = kS0 + kRows * Sh::sb;
            // inner coordinates in the maps' elements: code words, bf16 groups
            const int cq = it_c * (Sh::q / Sh::qelem), cs = it_c * (Sh::sb / 2);
            tma_load_2d(dst, &qmap, cq, r_a, full);
            tma_load_2d(dst + kS0, &smap, cs, r_a, full);
            tma_load_2d(dst + kB0, &bmap, cs, r_a, full);
            if (kGlu) {
                tma_load_2d(dst + (kRows / 2) * Sh::q, &qmap, cq, r_b, full);
                tma_load_2d(dst + kS0 + (kRows / 2) * Sh::sb, &smap, cs, r_b, full);
                tma_load_2d(dst + kB0 + (kRows / 2) * Sh::sb, &bmap, cs, r_b, full);
            }
            ++it_c;
        } else {
            mbar_arrive(full);   // the end marker: no copies, the phase completes at once
            done_issuing = true;
        }
        ++nissued;
        if (++islot == S) {
            islot = 0;
            ++iuse;
        }
    };

    // The first three slots of each ring go out first (one tile-chunk a slot),
    // before the wait for the kernel this one may overlap: the weights are never
    // written by a kernel of the library, and a kernel from elsewhere does not
    // release this one before it ends.  Every CTA's first copies arrive as one
    // burst, and a smaller burst lands each group's first slot sooner (measured:
    // 71.1 -> 69.1 us on the lm_head half against sending the whole ring).  Then
    // all warps prepare the limbs, and the producers keep the rings full.
    if (producer && lane == 0)
        for (int i = 0; i < 3 && i < S; ++i) issue_next();
    __syncwarp();
    pdl_wait();
    pdl_trigger();
    const size_t lc_n = (size_t)nch * 32;   // lane-chunks of one activation row
#pragma unroll
    for (int m = 0; m < kM; ++m)
        prep_limbs(a.x + (size_t)m * a.ldx, K, nch, limbs + m * lc_n * kLimbBytes, csts + m * lc_n, wms + m * nch,
                   kTWarps + kTGroups, warp, lane);
    __syncthreads();
    if (producer) {
        if (lane == 0)
            while (!done_issuing) issue_next();
        __syncwarp();
    }

    static_assert(kWR * kM <= 8, "row totals: 8 floats per warp");
    float acc[kWR][kM];
#pragma unroll
    for (int r = 0; r < kWR; ++r)
#pragma unroll
        for (int m = 0; m < kM; ++m) acc[r][m] = 0.0f;
    float *tot = reinterpret_cast<float *>(smem + L.tot_off) + (producer ? 0 : warp * 8);   // lane 0's, [r][m]
    const int sc = slice_chunks(nch);
    (void)sc;
    uint64_t best = 0;
    int slot = 0;
    uint32_t par = 0;
    const uint4 *limb_l = reinterpret_cast<const uint4 *>(limbs) + lane;
    bool failed = false;
    for (; !producer;) {
        const bool ok = __all_sync(0xFFFFFFFFu, tile_wait(full0 + 8 * slot, par, abort_flag, kSpinLimit));
        if (!ok) {
            failed = true;
            break;
        }
        const int2 h = hdr[slot];
        if (h.x < 0) break;
        const uint8_t *sl = ring + slot * kTSlotBytes;
        const uint4 *ql = reinterpret_cast<const uint4 *>(sl) + lane;
        const uint16_t *sc0 = reinterpret_cast<const uint16_t *>(sl + kRows * Sh::q);
        const uint16_t *sc16 = sc0 + (lane >> 1);
#pragma unroll
        for (int cc = 0; cc < kCps; ++cc) {
            const int c = h.y * kCps + cc;
            if (c >= nch) break;   // chunks past K add nothing
            // nor do lanes past the end of a short last chunk
            const bool live = lane * 32 < K - c * kChunk;
            // the warp's rows: codes, scale and bias (read once per activation row
            // for one row, kept in registers across the rows for more)
            constexpr int kQ = kM == 1 ? 1 : kWR;
            uint4 qv[kQ];
            float sv[kQ], bv[kQ];
            auto row_operands = [&](int r, uint4 &q, float &sr, float &br) {
                const int R = tile_row<kGlu, kWR>(w_in, r);
                q = ql[R * (Sh::q / 16) + cc * (kChunk / 32)];
                sr = bf16_bits_to_f32(sc16[R * (Sh::sb / 2) + cc * (kChunk / 64)]);
                br = bf16_bits_to_f32(sc16[kRows * (Sh::sb / 2) + R * (Sh::sb / 2) + cc * (kChunk / 64)]);
            };
            if (kM > 1) {
#pragma unroll
                for (int r = 0; r < kWR; ++r) row_operands(r, qv[r % kQ], sv[r % kQ], bv[r % kQ]);
            }
#pragma unroll
            for (int m = 0; m < kM; ++m) {
                LaneChunk t;
                load_lane_chunk(t, limb_l + m * lc_n * (kLimbBytes / 16), csts + m * lc_n, c, lane);
                const uint32_t wm = wms[m * nch + c];
                if (live) {
#pragma unroll
                    for (int r = 0; r < kWR; ++r) {
                        if (kM == 1) row_operands(r, qv[0], sv[0], bv[0]);
                        acc[r][m] = lane_chunk_fma(acc[r][m], qv[r % kQ], t, sv[r % kQ], bv[r % kQ]);
                    }
                }
                for (uint32_t mm = wm; mm != 0; mm &= mm - 1) {   // wide lane-chunks, warp-uniform
                    const int l = __ffs(mm) - 1;
                    const float xj = wide_x(limbs + m * lc_n * kLimbBytes, c, l, lane);
#pragma unroll
                    for (int r = 0; r < kWR; ++r) {
                        const int R = tile_row<kGlu, kWR>(w_in, r);
                        const uint32_t word = reinterpret_cast<const uint32_t *>(
                            sl)[(R * (Sh::q / 16) + cc * (kChunk / 32) + l) * 4 + (lane >> 3)];
                        const float s = bf16_bits_to_f32(sc0[R * (Sh::sb / 2) + cc * (kChunk / 64) + (l >> 1)]);
                        const float b =
                            bf16_bits_to_f32(sc0[kRows * (Sh::sb / 2) + R * (Sh::sb / 2) + cc * (kChunk / 64) + (l >> 1)]);
                        const float d = wide_dot(xj, word, lane, s, b);
                        if (lane == l) acc[r][m] += d;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * slot);
        if (++slot == S) {
            slot = 0;
            par ^= 1u;
        }
        // a slice ends only at the end of a slot (slices of 4 chunks, slots of 1, 2
        // or 4), so its tree sum waits until the slot is back with the producer
        if (!kOne) {
            const int c_last = min(h.y * kCps + kCps, nch) - 1;
            if (slice_end(c_last, sc, nch)) {
#pragma unroll
                for (int r = 0; r < kWR; ++r)
#pragma unroll
                    for (int m = 0; m < kM; ++m) slice_fold(acc[r][m], tot + r * kM + m, c_last, sc, lane);
            }
        }
        if (h.y == nsl - 1) {
            if (kOne) {   // the single slice's fold, as slice_fold does it
                float tr[kWR * kM];
#pragma unroll
                for (int r = 0; r < kWR; ++r)
#pragma unroll
                    for (int m = 0; m < kM; ++m) {
                        tr[r * kM + m] = warp_sum_to_lane0(acc[r][m]);
                        acc[r][m] = 0.0f;
                    }
                if (lane == 0) {
#pragma unroll
                    for (int i = 0; i < kWR * kM; ++i) tot[i] = tr[i];
                }
            }
            if (lane == 0) {
                int r_a, r_b, col, ncol;
                tile_rows(h.x, r_a, r_b, col, ncol);
#pragma unroll
                for (int m = 0; m < kM; ++m) {
                    uint16_t *ym = a.y + (size_t)m * a.ldy;
                    if (kGlu) {
#pragma unroll
                        for (int p = 0; p < kWR / 2; ++p) {
                            const int cj = (kWR / 2) * w_in + p;
                            if (cj < ncol) {
                                const float g = bf16_bits_to_f32(f32_to_bf16_rne(tot[(2 * p) * kM + m]));
                                const float uu = bf16_bits_to_f32(f32_to_bf16_rne(tot[(2 * p + 1) * kM + m]));
                                ym[col + cj] = f32_to_bf16_rne(glu_f32(g, uu));
                            }
                        }
                    } else {
#pragma unroll
                        for (int r = 0; r < kWR; ++r) {
                            const int cj = kWR * w_in + r;
                            if (cj < ncol) {
                                const uint16_t hv = f32_to_bf16_rne(tot[r * kM + m]);
                                ym[col + cj] = hv;
                                if (kM == 1 && a.cand) best = umax64(best, cand_key(hv, a.id_base + (uint32_t)(col + cj)));
                            }
                        }
                    }
                }
            }
        }
    }
    if (failed && lane == 0) *abort_flag = 1;
    __syncthreads();
    if (*abort_flag) {
        // a wait gave up: the CTA's whole share of outputs becomes NaN, and the
        // copies still in flight get a bounded chance to land before exit
        for (int t = t0; t < t1; ++t) {
            int r_a, r_b, col, ncol;
            tile_rows(t, r_a, r_b, col, ncol);
            for (int i = tid; i < kM * ncol; i += blockDim.x)
                a.y[(size_t)(i / ncol) * a.ldy + col + i % ncol] = (uint16_t)TF_NAN_BF16;
        }
        if (producer && lane == 0)
            for (int s2 = 0; s2 < S && s2 < nissued; ++s2) {
                const int uses = (nissued - 1 - s2) / S + 1;
                wait_slot(full0 + 8 * s2, (uint32_t)((uses - 1) & 1), 1024);
            }
        best = cand_key((uint16_t)TF_NAN_BF16, 0u);
    }
    if (a.cand) fused_head_keys(a, best, kTWarps + kTGroups, warp, lane);
}

// ---------------------------------------------------------- narrow calls --
// A call with a long K (more than 8 chunks) and too few rows for the 16-row tile
// ring -- down's 2,560-row halves at K = 17,408 -- has about one row per warp of
// the GPU: a warp per row at the full K would run two rounds on a few warps
// while the rest idle.  Here each CTA owns a contiguous run of output columns
// and its warps share the (column, K-slice) pairs of that run, round robin.  A
// pair is one row over one slice (up to 4,096 K: 2 KB of codes), streamed
// through the warp's own ring by one 1-D bulk copy; the scales and biases of
// the CTA's rows come in once, two copies a row, at the start (the copy engine
// takes a fixed time per copy, so many small copies would hold up the rest of
// the CTA's copies).  The warp leaves the slice's tree sum in shared memory,
// and once every pair is done each column's slice sums are added in ascending
// order.  That is the reduction order of every M = 1 kernel (see the top of this
// file), so the bits are theirs.
constexpr int kSWarps = 16;
constexpr int kSMaxStages = 4;
constexpr int kSItemQ = 4 * kChunk / 2;          // code bytes of one row-slice
constexpr int kSSlot = kSItemQ;                  // 2,048

struct SplitLayout {
    int nch, nsl;
    size_t limb_off, cst_off, wm_off, part_off, sb_off, bar_off, ring_off, total;
};

// M activation rows (limbs, sums and scales of each), `stages` slots per warp.
__host__ __device__ inline SplitLayout split_layout(int K, int maxcols, int M, int stages) {
    SplitLayout L;
    L.nch = (K + kChunk - 1) / kChunk;
    L.nsl = (L.nch + 3) / 4;
    L.limb_off = 0;
    L.cst_off = round_up(L.limb_off + (size_t)M * L.nch * 32 * kLimbBytes, 128);
    L.wm_off = L.cst_off + (size_t)M * L.nch * 32 * 16;
    L.part_off = round_up(L.wm_off + (size_t)M * L.nch * 4, 128);
    L.sb_off = round_up(L.part_off + (size_t)maxcols * L.nsl * M * 4, 128);   // [maxcols][G] scales, then biases
    L.bar_off = round_up(L.sb_off + (size_t)2 * maxcols * (K / kGroup) * 2, 128);
    L.ring_off = round_up(L.bar_off + (size_t)(kSWarps * kSMaxStages + 1) * 8, 128);
    L.total = L.ring_off + (size_t)kSWarps * stages * kSSlot;
    return L;
}

template <int kM>
__global__ void __launch_bounds__(kSWarps * 32, 1) qmm_m1_split_kernel(QmmArgs a, int maxcols, int kSStages) {
    extern __shared__ __align__(128) uint8_t smem[];
    const SplitLayout L = split_layout(a.K, maxcols, kM, kSStages);
    const int K = a.K, nch = L.nch, nsl = L.nsl;
    const int G = K / kGroup;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t *limbs = smem + L.limb_off;
    uint4 *csts = reinterpret_cast<uint4 *>(smem + L.cst_off);
    uint32_t *wms = reinterpret_cast<uint32_t *>(smem + L.wm_off);
    float *part = reinterpret_cast<float *>(smem + L.part_off);
    uint8_t *ring = smem + L.ring_off + (size_t)warp * kSStages * kSSlot;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar0 = smem_addr(smem + L.bar_off) + (uint32_t)(warp * kSMaxStages * 8);
    const uint32_t sbar = smem_addr(smem + L.bar_off) + (uint32_t)(kSWarps * kSMaxStages * 8);
    uint16_t *s_all = reinterpret_cast<uint16_t *>(smem + L.sb_off);
    uint16_t *b_all = s_all + (size_t)maxcols * G;

    // this CTA's columns and the warp's (column, slice) pairs: i = warp + t * kSWarps
    const int c0 = (int)((long long)blockIdx.x * a.seg.ncols / gridDim.x);
    const int c1 = (int)((long long)(blockIdx.x + 1) * a.seg.ncols / gridDim.x);
    const int nitems = (c1 - c0) * nsl;
    const int my_items = nitems > warp ? (nitems - warp + kSWarps - 1) / kSWarps : 0;

    // the codes of pair t of warp w into slot t % kSStages of w's ring
    auto issue_for = [&](int w, int t) {
        const int slot = t % kSStages;
        const uint32_t bar = smem_addr(smem + L.bar_off) + (uint32_t)(w * kSMaxStages * 8) + 8 * slot;
        const uint32_t ring_w = smem_addr(smem + L.ring_off + (size_t)w * kSStages * kSSlot);
        const int i = w + t * kSWarps;
        const int col = c0 + i / nsl, j = i % nsl;
        const int len = min(4 * kChunk, K - j * 4 * kChunk);   // K of the slice (a multiple of 512)
        const size_t row = (size_t)seg_row(a.seg, col, 0, 0);
        mbar_expect_tx(bar, (uint32_t)(len / 2));
        bulk_g2s(ring_w + slot * kSSlot, a.wq + row * (size_t)(K / 2) + (size_t)j * kSItemQ, (uint32_t)(len / 2), bar);
    };
    auto issue = [&](int t) { issue_for(warp, t); };   // lane 0 of the pair's warp

    if (lane == 0)
        for (int st = 0; st < kSStages; ++st) mbar_init(bar0 + 8 * st, 1);
    if (tid == 0) {
        mbar_init(sbar, 1);
        fence_mbar_init();
        mbar_expect_tx(sbar, (uint32_t)(2 * (c1 - c0) * G * 2));
    } else if (lane == 0) {
        fence_mbar_init();
    }
    __syncthreads();
    // Weights before the wait for the kernel this one may overlap (the library
    // never writes weights, and a kernel from elsewhere ends before this one
    // starts): the last warp sends the rows' scales and biases and every warp's
    // first pairs (lane w those of warp w), while the other warps prepare the
    // limbs -- the copy engine takes a fixed time per copy, so the copies and the
    // preparation overlap instead of following one another.
    constexpr int kIssuer = kSWarps - 1;
    if (warp == kIssuer) {
        for (int i = lane; i < 2 * (c1 - c0); i += 32) {
            const int col = c0 + (i >> 1);
            const size_t row = (size_t)seg_row(a.seg, col, 0, 0);
            const uint16_t *src = ((i & 1) ? a.biases : a.scales) + row * (size_t)G;
            uint16_t *dst = ((i & 1) ? b_all : s_all) + (size_t)(col - c0) * G;
            bulk_g2s(smem_addr(dst), src, (uint32_t)(G * 2), sbar);
        }
        if (lane < kSWarps) {
            const int items_w = nitems > lane ? (nitems - lane + kSWarps - 1) / kSWarps : 0;
            for (int t = 0; t < kSStages && t < items_w; ++t) issue_for(lane, t);
        }
        __syncwarp();
    }
    pdl_wait();
    pdl_trigger();
    const size_t lc_n = (size_t)nch * 32;   // lane-chunks of one activation row
    if (warp != kIssuer) {
#pragma unroll
        for (int m = 0; m < kM; ++m)
            prep_limbs(a.x + (size_t)m * a.ldx, K, nch, limbs + m * lc_n * kLimbBytes, csts + m * lc_n, wms + m * nch,
                       kSWarps - 1, warp, lane);
    }
    __syncthreads();

    const uint4 *limb_l = reinterpret_cast<const uint4 *>(limbs) + lane;
    bool failed = !__all_sync(0xFFFFFFFFu, wait_slot(sbar, 0, kSpinLimit));
    for (int t = 0; t < my_items; ++t) {
        const int slot = t % kSStages;
        const bool ok = __all_sync(0xFFFFFFFFu, wait_slot(bar0 + 8 * slot, (uint32_t)((t / kSStages) & 1),
                                                          failed ? 64 : kSpinLimit));
        failed = failed || !ok;
        const int i = warp + t * kSWarps;
        const int col = c0 + i / nsl, j = i % nsl;
        const int ch = min(4, nch - 4 * j);
        const uint8_t *sl = ring + slot * kSSlot;
        // the slice's scales and biases of this row: 16 groups a chunk
        const uint16_t *srow = s_all + (size_t)(col - c0) * G + j * (4 * kChunk / kGroup);
        const uint16_t *brow = b_all + (size_t)(col - c0) * G + j * (4 * kChunk / kGroup);
        float acc[kM];
#pragma unroll
        for (int m = 0; m < kM; ++m) acc[m] = 0.0f;
        // one chunk of the pair (a full slice's four unrolled)
        auto chunk = [&](int cc) {
            const int c = 4 * j + cc;
            const bool live = lane * 32 < K - c * kChunk;   // lanes past the end of a short last chunk add nothing
            const uint4 qv = reinterpret_cast<const uint4 *>(sl)[cc * 32 + lane];
            const float sv = bf16_bits_to_f32(srow[cc * 16 + (lane >> 1)]);
            const float bv = bf16_bits_to_f32(brow[cc * 16 + (lane >> 1)]);
#pragma unroll
            for (int m = 0; m < kM; ++m) {
                LaneChunk lc;
                load_lane_chunk(lc, limb_l + m * lc_n * (kLimbBytes / 16), csts + m * lc_n, c, lane);
                const uint32_t wm = wms[m * nch + c];
                if (live) acc[m] = lane_chunk_fma(acc[m], qv, lc, sv, bv);
                for (uint32_t mm = wm; mm != 0; mm &= mm - 1) {   // wide lane-chunks, warp-uniform
                    const int l = __ffs(mm) - 1;
                    const float xj = wide_x(limbs + m * lc_n * kLimbBytes, c, l, lane);
                    const uint32_t word = reinterpret_cast<const uint32_t *>(sl)[(cc * 32 + l) * 4 + (lane >> 3)];
                    const float s = bf16_bits_to_f32(srow[cc * 16 + (l >> 1)]);
                    const float b = bf16_bits_to_f32(brow[cc * 16 + (l >> 1)]);
                    const float d = wide_dot(xj, word, lane, s, b);
                    if (lane == l) acc[m] += d;
                }
            }
        };
        if (ch == 4) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) chunk(cc);
        } else {
            for (int cc = 0; cc < ch; ++cc) chunk(cc);
        }
#pragma unroll
        for (int m = 0; m < kM; ++m) {
            const float v = warp_sum_to_lane0(acc[m]);
            if (lane == 0) part[((col - c0) * nsl + j) * kM + m] = failed ? __int_as_float(0x7FC00000) : v;
        }
        __syncwarp();
        if (lane == 0 && t + kSStages < my_items && !failed) issue(t + kSStages);
    }
    if (failed) {   // copies still in flight get a bounded chance to land before exit
        for (int st = 0; st < kSStages; ++st) wait_slot(bar0 + 8 * st, 0, 1024);
        wait_slot(sbar, 0, 1024);
    }
    __syncthreads();

    // each column and activation row: its slice sums in ascending order
    uint64_t best = 0;
    for (int qm = tid; qm < (c1 - c0) * kM; qm += blockDim.x) {
        const int q = qm / kM, m = qm % kM;
        float tot = part[q * nsl * kM + m];
        for (int j = 1; j < nsl; ++j) tot += part[(q * nsl + j) * kM + m];
        const uint16_t h = f32_to_bf16_rne(tot);
        a.y[(size_t)m * a.ldy + c0 + q] = h;
        if (kM == 1 && a.cand) best = umax64(best, cand_key(h, a.id_base + (uint32_t)(c0 + q)));
    }
    if (kM == 1 && a.cand) {
        best = warp_max64(best);
        fused_head_keys(a, best, kSWarps, warp, lane);
    }
}

// The widest warp count whose shared memory fits 227 KB with 1 KB left for the
// kernel's static shared memory.
static int stream_warps(int K, int ru) {
    for (int w = kMaxWarps; w >= 4; --w)
        if (stream_layout(K, w, ru).total <= 226 * 1024) return w;
    return 0;
}

static bool stream_multi_eligible(const QmmArgs &a);

// K % 512 == 0 (every slot piece is a multiple of 16 B) and 16-byte aligned
// code, scale and bias arrays: the bulk copies' requirements.  One activation
// row, or two to four where their limbs leave room for the rings.
bool qmm_m1_stream_eligible(const QmmArgs &a) {
    if (a.K % 512 != 0) return false;
    if (!aligned(a.scales, 16) || !aligned(a.biases, 16) || !aligned(a.wq, 16)) return false;
    if (a.M == 1) return stream_warps(a.K, 4) > 0;
    return stream_multi_eligible(a);
}

static size_t g_stream_smem_set[64][3];

template <int RU>
static cudaError_t launch_ru(const QmmArgs &a, int ri, cudaStream_t stream, int *ncand) {
    const int W = stream_warps(a.K, RU);
    const StreamLayout L = stream_layout(a.K, W, RU);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (g_stream_smem_set[dev][ri] < L.total) {
        cudaError_t e = cudaFuncSetAttribute(qmm_m1_stream_kernel<RU, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(qmm_m1_stream_kernel<RU, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
        if (e != cudaSuccess) return e;
        g_stream_smem_set[dev][ri] = 226 * 1024;
    }
    constexpr int kCols = RU / 2 > 0 ? RU / 2 : 1;   // output columns of a GLU unit
    const int units = a.glu ? (a.seg.ncols + kCols - 1) / kCols : (a.seg.ncols + RU - 1) / RU;
    int blocks = num_sms();
    const int need = (units + W - 1) / W;
    if (need < blocks) blocks = need;
    if (ncand) *ncand = blocks * W;
    if (slice_chunks(L.nch) == L.nch)
        return launch_pdl(qmm_m1_stream_kernel<RU, true>, dim3(blocks), dim3(W * 32), L.total, stream, a, units);
    return launch_pdl(qmm_m1_stream_kernel<RU, false>, dim3(blocks), dim3(W * 32), L.total, stream, a, units);
}

// ---------------------------------------------------------- tile ring host --
static int tile_stages(int K, int M) {
    for (int st = kTMaxStages; st >= 2; --st)
        if (tile_layout(K, st, M).total <= 226 * 1024) return st;
    return 0;
}

static TilePlan tile_plan(const QmmArgs &a, int rows) {
    TilePlan plan{};
    if (a.glu) {
        plan.ntiles = (a.seg.ncols + rows / 2 - 1) / (rows / 2);
        for (int s = 1; s <= TF_MAX_SEGS; ++s) plan.tstart[s] = plan.ntiles;
    } else {
        int n = 0;
        for (int s = 0; s < a.seg.nseg; ++s) {
            plan.tstart[s] = n;
            n += (a.seg.nrows[s] + rows - 1) / rows;
        }
        for (int s = a.seg.nseg; s <= TF_MAX_SEGS; ++s) plan.tstart[s] = n;
        plan.ntiles = n;
    }
    return plan;
}

// The tile ring takes the call when the driver offers the tensor-map encoder, two
// slots per group fit beside the limbs, and there are tiles enough: 16-row tiles
// with at least two per SM (attn_out's 320 tiles: 15.9 -> 13.8 us against the
// per-warp ring, though half the groups of a CTA get no tile), else (not GLU,
// K >= 8,192) 4-row tiles with at least two per SM; otherwise the per-warp
// kernel's finer units balance better.
// (With a short K the 4-chunk slots run mostly empty -- at K = 5,120 a tile's second
// slot holds one chunk -- and the per-warp ring measured faster there.)  Returns the
// rows per compute warp of the tile shape, 0 for the per-warp kernel.
static int tile_ring_shape(const QmmArgs &a) {
    if (!encode_tiled_fn() || tile_stages(a.K, 1) < 2) return 0;
    if (tile_plan(a, TileShape<4>::rows).ntiles >= 2 * num_sms()) return 4;
    if (!a.glu && a.K >= 8192 && tile_plan(a, TileShape<1>::rows).ntiles >= 2 * num_sms()) return 1;
    return 0;
}

template <bool kGlu, int kWR, int kM>
static cudaError_t launch_tile(const QmmArgs &a, cudaStream_t stream, int *ncand) {
    static bool smem_set[64];
    using Sh = TileShape<kWR>;
    const int S = tile_stages(a.K, kM);
    const TileLayout L = tile_layout(a.K, S, kM);
    const TilePlan plan = tile_plan(a, Sh::rows);
    auto enc = encode_tiled_fn();
    const cuuint32_t box_rows = kGlu ? (cuuint32_t)(Sh::rows / 2) : (cuuint32_t)Sh::rows;
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap qmap, smap, bmap;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(a.K / 2 / Sh::qelem), (cuuint64_t)a.n_whole};
        const cuuint64_t strides[1] = {(cuuint64_t)(a.K / 2)};
        const cuuint32_t box[2] = {(cuuint32_t)(Sh::q / Sh::qelem), box_rows};
        const CUtensorMapDataType qt = Sh::qelem == 8 ? CU_TENSOR_MAP_DATA_TYPE_UINT64 : CU_TENSOR_MAP_DATA_TYPE_UINT32;
        if (enc(&qmap, qt, 2, const_cast<uint8_t *>(a.wq), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const int G = a.K / kGroup;
        const cuuint64_t dims[2] = {(cuuint64_t)G, (cuuint64_t)a.n_whole};
        const cuuint64_t strides[1] = {(cuuint64_t)G * 2};
        const cuuint32_t box[2] = {(cuuint32_t)(Sh::sb / 2), box_rows};
        if (enc(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t *>(a.scales), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            enc(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t *>(a.biases), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!smem_set[dev]) {
        cudaError_t e =
            cudaFuncSetAttribute(qmm_m1_tile_kernel<kGlu, kWR, kM, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(qmm_m1_tile_kernel<kGlu, kWR, kM, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     226 * 1024);
        if (e != cudaSuccess) return e;
        smem_set[dev] = true;
    }
    const int blocks = plan.ntiles < num_sms() ? plan.ntiles : num_sms();
    if (ncand) *ncand = blocks * (kTWarps + kTGroups);
    if (slice_chunks(L.nch) == L.nch)
        return launch_pdl(qmm_m1_tile_kernel<kGlu, kWR, kM, true>, dim3(blocks), dim3(kTThreads), L.total, stream, a, plan,
                          qmap, smap, bmap, S);
    return launch_pdl(qmm_m1_tile_kernel<kGlu, kWR, kM, false>, dim3(blocks), dim3(kTThreads), L.total, stream, a, plan, qmap,
                      smap, bmap, S);
}

// Calls with enough tiles take the tile ring.  Otherwise rows per unit only change
// how often a lane reuses its activation limbs, never a row's arithmetic, so the
// choice may follow N: four rows while every warp of the grid still gets two
// units, fewer when the slice is narrow.
// The narrow-call kernel: no GLU, K longer than 8 chunks, and its layout fits (the
// rings beside the limbs and the slice sums of a CTA's columns): four slots a
// warp for one activation row, two for two.
static int split_maxcols(const QmmArgs &a) {
    const int blocks = a.seg.ncols < num_sms() ? a.seg.ncols : num_sms();
    return blocks > 0 ? (a.seg.ncols + blocks - 1) / blocks : 0;
}
static int split_stages(const QmmArgs &a) {
    if (a.glu || (a.K + kChunk - 1) / kChunk <= 8 || a.M > 2) return 0;
    const int want = a.M == 1 ? kSMaxStages : 2;
    return split_layout(a.K, split_maxcols(a), a.M, want).total <= 226 * 1024 ? want : 0;
}

template <int kM>
static cudaError_t launch_split(const QmmArgs &a, cudaStream_t stream, int *ncand) {
    static bool smem_set[64];
    const int maxcols = split_maxcols(a), S = split_stages(a);
    const SplitLayout L = split_layout(a.K, maxcols, kM, S);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!smem_set[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(qmm_m1_split_kernel<kM>, cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
        if (e != cudaSuccess) return e;
        smem_set[dev] = true;
    }
    const int blocks = a.seg.ncols < num_sms() ? a.seg.ncols : num_sms();
    if (ncand) *ncand = blocks * kSWarps;
    return launch_pdl(qmm_m1_split_kernel<kM>, dim3(blocks), dim3(kSWarps * 32), L.total, stream, a, maxcols, S);
}

// 2 or 3 activation rows on the streaming kernels: each row takes exactly the
// arithmetic it takes alone (the same lane-chunks, order and tree), so its bits
// equal those of an M = 1 call; the codes, scales and biases of a tile are read
// once for all the rows.  Long-K calls take the narrow-call kernel (two rows at
// most: the limbs of more leave too little room for its rings); the others the
// tile ring with as many rows per warp as still give every group a tile
// (four rows by 16 for two activation rows, two by 8 for three).
static int multi_tile_shape(const QmmArgs &a) {
    if (!encode_tiled_fn() || tile_stages(a.K, a.M) < 2) return 0;
    const int big = a.M == 2 ? 4 : 2;
    if (tile_plan(a, 4 * big).ntiles >= 4 * num_sms() || a.glu) return big;
    return 1;
}

static bool stream_multi_eligible(const QmmArgs &a) {
    // four rows measured slower here than on the tensor cores (lm_head half 286 us
    // against 260 us), so the streaming kernels take two and three
    if (a.M < 2 || a.M > 3) return false;
    if (!a.glu && (a.K + kChunk - 1) / kChunk > 8) return split_stages(a) > 0;
    return multi_tile_shape(a) > 0;
}

template <int kM>
static cudaError_t launch_multi(const QmmArgs &a, cudaStream_t stream) {
    if (!a.glu && (a.K + kChunk - 1) / kChunk > 8) {
        if (kM == 2) return launch_split<2>(a, stream, nullptr);
        return cudaErrorInvalidValue;
    }
    constexpr int kBig = kM == 2 ? 4 : 2;
    if (multi_tile_shape(a) == kBig)
        return a.glu ? launch_tile<true, kBig, kM>(a, stream, nullptr) : launch_tile<false, kBig, kM>(a, stream, nullptr);
    return launch_tile<false, 1, kM>(a, stream, nullptr);
}

cudaError_t launch_qmm_m1_stream(const QmmArgs &a, cudaStream_t stream, int *ncand) {
    switch (a.M) {
        case 2: return launch_multi<2>(a, stream);
        case 3: return launch_multi<3>(a, stream);
        default: break;
    }
    const int shape = tile_ring_shape(a);
    if (shape == 4)
        return a.glu ? launch_tile<true, 4, 1>(a, stream, ncand) : launch_tile<false, 4, 1>(a, stream, ncand);
    if (split_stages(a) > 0) return launch_split<1>(a, stream, ncand);
    if (shape == 1) return launch_tile<false, 1, 1>(a, stream, ncand);
    const long long warps = (long long)num_sms() * stream_warps(a.K, 4);
    const long long rows = a.glu ? 2ll * a.seg.ncols : a.seg.ncols;
    if (rows >= 8 * warps) return launch_ru<4>(a, 0, stream, ncand);
    if (rows >= 2 * warps || a.glu) return launch_ru<2>(a, 1, stream, ncand);
    return launch_ru<1>(a, 2, stream, ncand);
}

cudaError_t launch_argmax_keys(const uint64_t *cand, int ncand, const uint16_t *logits, uint32_t id_base, uint64_t *word,
                               cudaStream_t stream) {
    return launch_pdl(argmax_keys_kernel, dim3(1), dim3(kKeyThreads), 0, stream, cand, ncand, logits, id_base, word);
}

int qmm_m1_stream_max_cand() { return num_sms() * kMaxWarps; }

}  // namespace tf
