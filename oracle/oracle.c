/*
 * oracle.c -- plain, slow CPU oracle for the row-split int4 hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline / reference legs may load this library.  It shares no code,
 * header, table or helper with the CUDA library in row_split_int4_b200/, and
 * it never reads anything the CUDA library produced unless a test hands it
 * that data on purpose (the per-stage checks feed each stage the same bf16
 * input the GPU stage took).
 *
 * Everything here is the plain definition, computed in double precision:
 *
 *   qmm      y[m,n] = bf16_RNE( sum_{k<K} x[m,k] * (s[n,k/64]*q[n,k] + b[n,k/64]) )
 *            -- the 4-bit affine, group-64 format of the checkpoint named in
 *               TensorFold PR #1437 (Receipt: "4-bit affine with group 64");
 *               each output row is reduced over the whole K by whoever owns it
 *               (TensorFold PR #1433, step-1 body: the seam exchanges whole
 *               output rows, each rank reduces over the full K).
 *   glu      a = bf16_RNE( g * SiLU(u) ),  SiLU(u) = u / (1 + exp(-u))
 *   gather   whole bf16 rows copied to their offsets, no arithmetic; a missing
 *            half reads as the bf16 NaN 0x7FC0 (PR #1433 step-1 body: a broken
 *            link surfaces as 0x7FC0).
 *   argmax   linear scan, the lower id wins ties, any NaN/+-Inf flags the row
 *            with bit 31 of the id word (PR #1433 step-1 body).
 *   pick     any flagged word -> 0xFFFFFFFF, else the larger value, lower id on
 *            ties (PR #1433 step-1 body; step-2 body: the pick is the better of
 *            the two half-vocab winners).
 *   residual h' = fp32(h + y): a gathered bf16 projection row added to the fp32
 *            residual stream (PR #1433 step-2 body: o_proj and down_proj gather
 *            whole bf16 rows and add in the fp32 stream).
 *   qmm8     y[m,n] = bf16_RNE( s[n] * sum_k x[m,k] q8[n,k] ): the int8 lm_head
 *            with one bf16 scale per row (the b70 lab's "runtime INT8 target
 *            LM-head", bf16 scale).
 *   embed    out[m] = table[id_m], the whole table on every rank, ids checked
 *            against the whole table's bound (PR #1433 step-2 body and the
 *            "Rank-slice the qwen27 family and gather the whole embedding
 *            table" commit: embedBound takes the whole table, refuses a smaller
 *            bound).
 *
 * Readings taken where the pages are silent:
 *   nibble order  element k lives in byte k/2 of its row, low nibble for even k;
 *   q             unsigned 0..15, no separate zero point (the bias carries it);
 *   rounding      round-to-nearest-even straight from double to bf16, NaN -> 0x7FC0;
 *   +-0           compare equal, so they tie and the lower id wins;
 *   flagged word  value bits 0x7FC00000, id word 0x80000000 | first non-finite id.
 *
 * Build:  gcc -O2 -fopenmp -shared -fPIC oracle.c -o liboracle.so -lm
 * (no -ffast-math: the double arithmetic must be IEEE).
 *
 * Planted controls: building with -DORC_PLANT=n makes one deliberate mistake,
 * used only by tests/test_oracle_plants.py to show that the pins catch it:
 *   1 the split rows of half h are the peer's rows      (a stage on the peer's half)
 *   2 gather writes part 0 into every slot              (a gather writing its own half twice)
 *   3 argmax breaks ties to the higher id
 *   4 pick breaks ties to the higher id
 *   5 argmax does not flag non-finite values
 *   6 pick ignores the flag bit
 *   7 dequant drops the bias term
 *   8 dequant swaps the nibble order inside a byte
 *   9 GLU uses SiLU(g)*u instead of g*SiLU(u)
 *  10 the residual add rounds the sum to bf16 instead of fp32
 *  11 the embedding gather checks ids against half of the bound (the shard's width)
 *  12 the int8 head reads its codes as unsigned bytes
 *  13 the top two's second place skips values equal to the winner's (a tie reads as no tie)
 *  14 the top-two merge takes the second place from the winning part only
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#ifndef ORC_PLANT
#define ORC_PLANT 0
#endif

#define ORC_GROUP 64
#define ORC_FLAG 0x80000000u
#define ORC_SENTINEL 0xFFFFFFFFu
#define ORC_NAN_BF16 0x7FC0u

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 bit pattern -> double.  A bf16 is the top half of an fp32, so the
 * widening is exact. */
static double orc_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> bf16, round to nearest, ties to even, in one step (never through
 * fp32, whose own rounding would round twice).  bf16: 1 sign bit, 8 exponent
 * bits (bias 127), 7 stored mantissa bits; subnormals are kept; overflow
 * rounds to +-Inf; NaN becomes 0x7FC0. */
uint16_t orc_bf16_rne(double v)
{
    if (isnan(v))
        return (uint16_t)ORC_NAN_BF16;
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    int e2;
    (void)frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;               /* a = 1.xxx * 2^E */
    if (E < -126)
        E = -126;                 /* subnormal: fixed spacing 2^-133 */
    double scaled = ldexp(a, 7 - E);   /* a / 2^(E-7): exact power-of-two scaling */
    double r = floor(scaled);
    double frac = scaled - r;          /* exact: scaled < 2^9 */
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) == 1.0))
        r += 1.0;
    uint32_t ri = (uint32_t)r;
    if (scaled < 128.0) {
        /* subnormal range: bits are the mantissa count; 128 carries into
         * the smallest normal, whose encoding is also 128 (0x0080). */
        return (uint16_t)(sign | ri);
    }
    if (ri == 256u) {
        E += 1;
        ri = 128u;
    }
    if (E > 127)
        return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | ((uint32_t)(E + 127) << 7) | (ri - 128u));
}

void orc_bf16_rne_array(const double *v, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_bf16_rne(v[i]);
}

/* --------------------------------------------------------------- dequant -- */

/* q of element k of one packed row (byte k/2, low nibble for even k). */
static unsigned orc_nibble(const uint8_t *row, int64_t k)
{
    uint8_t byte = row[k >> 1];
#if ORC_PLANT == 8
    return (k & 1) ? (byte & 0xFu) : (byte >> 4);
#else
    return (k & 1) ? (byte >> 4) : (byte & 0xFu);
#endif
}

/* w[n,k] = s[n,k/64] * q[n,k] + b[n,k/64], all in double.  With a bf16 scale
 * (8 significant bits) and a 4-bit q the product is exact, and so is the sum
 * with the bias whenever their exponents are within ~40 of each other. */
double orc_dequant(const uint8_t *wq, const uint16_t *scales, const uint16_t *biases,
                   int K, int64_t n, int64_t k)
{
    const int64_t G = K / ORC_GROUP;
    double s = orc_bf16_to_f64(scales[n * G + k / ORC_GROUP]);
    double b = orc_bf16_to_f64(biases[n * G + k / ORC_GROUP]);
    double q = (double)orc_nibble(wq + n * (int64_t)(K / 2), k);
#if ORC_PLANT == 7
    (void)b;
    return s * q;
#else
    return s * q + b;
#endif
}

/* ------------------------------------------------------------------- qmm -- */

/* For each activation row m and each listed weight row rows[i]:
 *   y64[m,i]    = sum_k x[m,k] * w[rows[i],k]   (double, ascending k)
 *   absdot[m,i] = sum_k |x[m,k] * w[rows[i],k]|
 *   y[m,i]      = bf16_RNE(y64[m,i])
 * x is bf16 [M][ldx]; wq is [N][K/2]; scales/biases are bf16 [N][K/64].
 * y is [M][ldy]; y64/absdot are [M][nrows] and may be NULL.
 * nthreads > 1 splits the rows over OpenMP threads; every row is still one
 * thread's ascending-k sum, so the result does not depend on nthreads.
 * Returns 0, or -1 on a bad argument. */
int orc_qmm_rows(const uint16_t *x, int M, int K, int64_t ldx,
                 const uint8_t *wq, const uint16_t *scales, const uint16_t *biases,
                 const int64_t *rows, int64_t nrows,
                 uint16_t *y, int64_t ldy, double *y64, double *absdot, int nthreads)
{
    if (M < 0 || K < 0 || K % ORC_GROUP != 0 || nrows < 0 || ldx < K || ldy < nrows)
        return -1;
    const int64_t G = K / ORC_GROUP;
    const int64_t rowbytes = K / 2;
#pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads > 0 ? nthreads : 1) if (nthreads > 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t n = rows[i];
        const uint8_t *qrow = wq + n * rowbytes;
        for (int m = 0; m < M; ++m) {
            const uint16_t *xr = x + (int64_t)m * ldx;
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double s = orc_bf16_to_f64(scales[n * G + k / ORC_GROUP]);
                double b = orc_bf16_to_f64(biases[n * G + k / ORC_GROUP]);
                double q = (double)orc_nibble(qrow, k);
#if ORC_PLANT == 7
                double w = s * q;
                (void)b;
#else
                double w = s * q + b;
#endif
                double p = orc_bf16_to_f64(xr[k]) * w;
                acc += p;
                aacc += fabs(p);
            }
            y[(int64_t)m * ldy + i] = orc_bf16_rne(acc);
            if (y64)
                y64[(int64_t)m * nrows + i] = acc;
            if (absdot)
                absdot[(int64_t)m * nrows + i] = aacc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ qmm8 -- */

/* The int8 head: y[m,i] = bf16_RNE( s[n] * sum_k x[m,k] * q[n,k] ), n = rows[i],
 * with q the signed byte q8[n,k] (row-major [N][K]) and s[n] one bf16 scale per
 * row -- the "runtime INT8 target LM-head" with a bf16 scale of the b70 lab's
 * Qwen3.6 27B profile ("Reproduce Qwen3.6 27B AutoRound Bring-Up", *Reproduce
 * The TP1 One-Replica Result*); the pages give no other detail, so the codes
 * are symmetric (no zero point).  Each product x*q is exact in double and the
 * sum runs over ascending k, as for the 4-bit format.  y64/absdot as there. */
int orc_qmm8_rows(const uint16_t *x, int M, int K, int64_t ldx, const int8_t *q8, const uint16_t *scales,
                  const int64_t *rows, int64_t nrows, uint16_t *y, int64_t ldy, double *y64, double *absdot,
                  int nthreads)
{
    if (M < 0 || K < 0 || nrows < 0 || ldx < K || ldy < nrows)
        return -1;
#pragma omp parallel for schedule(dynamic, 16) num_threads(nthreads > 0 ? nthreads : 1) if (nthreads > 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t n = rows[i];
        const int8_t *qrow = q8 + n * (int64_t)K;
        const double s = orc_bf16_to_f64(scales[n]);
        for (int m = 0; m < M; ++m) {
            const uint16_t *xr = x + (int64_t)m * ldx;
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
#if ORC_PLANT == 12
                const double q = (double)(uint8_t)qrow[k];
#else
                const double q = (double)qrow[k];
#endif
                const double p = orc_bf16_to_f64(xr[k]) * q;
                acc += p;
                aacc += fabs(p);
            }
            y[(int64_t)m * ldy + i] = orc_bf16_rne(s * acc);
            if (y64)
                y64[(int64_t)m * nrows + i] = s * acc;
            if (absdot)
                absdot[(int64_t)m * nrows + i] = fabs(s) * aacc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------- GLU -- */

/* a = bf16_RNE(g * SiLU(u)), SiLU(u) = u / (1 + exp(-u)), in double.  g and u
 * are the bf16-rounded outputs of the gate row and the up row with the same
 * index.  a64 (may be NULL) receives the unrounded double. */
void orc_glu(const uint16_t *g, const uint16_t *u, uint16_t *a, double *a64, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        double gv = orc_bf16_to_f64(g[i]);
        double uv = orc_bf16_to_f64(u[i]);
#if ORC_PLANT == 9
        double r = (gv / (1.0 + exp(-gv))) * uv;
#else
        double r = gv * (uv / (1.0 + exp(-uv)));
#endif
        a[i] = orc_bf16_rne(r);
        if (a64)
            a64[i] = r;
    }
}

/* ---------------------------------------------------------------- gather -- */

/* The row range that half h of nparts owns in a matrix of N rows: contiguous
 * equal spans [h*N/nparts, (h+1)*N/nparts) (TensorFold PR #1433 step-2 body:
 * 2,560 of 5,120, 8,704 of 17,408, 124,160 of 248,320; rank 0 starts at 0).
 * Returns -1 when N does not split evenly. */
int orc_half_rows(int h, int nparts, int64_t N, int64_t *row0, int64_t *nrows)
{
    if (nparts <= 0 || h < 0 || h >= nparts || N < 0 || N % nparts != 0)
        return -1;
    int64_t w = N / nparts;
#if ORC_PLANT == 1
    h = (h + 1) % nparts;
#endif
    *row0 = (int64_t)h * w;
    *nrows = w;
    return 0;
}

/* dst[m, off_h + j] = part_h[m, j] with off_h = widths[0] + ... + widths[h-1];
 * part h is dense [M][widths[h]].  A NULL part fills its columns with the bf16
 * NaN 0x7FC0.  Pure copy, no arithmetic. */
void orc_gather_rows(uint16_t *dst, int64_t ld_dst, const uint16_t *const *parts,
                     const int64_t *widths, int nparts, int M)
{
    int64_t off = 0;
    for (int h = 0; h < nparts; ++h) {
#if ORC_PLANT == 2
        const uint16_t *src = parts[0];
        const int64_t sw = widths[0];
#else
        const uint16_t *src = parts[h];
        const int64_t sw = widths[h];
#endif
        for (int m = 0; m < M; ++m)
            for (int64_t j = 0; j < widths[h]; ++j)
                dst[(int64_t)m * ld_dst + off + j] =
                    src ? src[(int64_t)m * sw + (j < sw ? j : sw - 1)] : (uint16_t)ORC_NAN_BF16;
        off += widths[h];
    }
}

/* -------------------------------------------------------------- residual -- */

/* out[i] = fp32(h[i] + y[i]) for n elements: a gathered bf16 projection row
 * added to the fp32 residual stream (TensorFold PR #1433 step-2 body: o_proj
 * and down_proj stage their rows, gather the peer's as whole bf16 rows and add
 * in the fp32 stream, so no two bf16 partials are summed).  The sum is formed
 * in double and rounded once to fp32 (round to nearest even): every fp32 + bf16
 * sum whose exponents lie within 29 of each other is exact in double, and when
 * they lie further apart the smaller term is far below half an fp32 ulp of the
 * larger, so the one rounding is the fp32 addition's result.  NaN and +-Inf
 * follow IEEE.  out may be h. */
void orc_residual_add(const float *h, const uint16_t *y, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        const double s = (double)h[i] + orc_bf16_to_f64(y[i]);
#if ORC_PLANT == 10
        out[i] = (float)orc_bf16_to_f64(orc_bf16_rne(s));
#else
        out[i] = (float)s;
#endif
    }
}

/* ----------------------------------------------------------------- embed -- */

/* out[m, :H] = table[ids[m], :H]: the embedding rows of M token ids from the
 * whole table, which every rank keeps whole (TensorFold PR #1433 step-2 body:
 * "Embeddings and norms stay whole on every rank", the gather's bound is the
 * whole 248,320-row table; the "Rank-slice the qwen27 family and gather the
 * whole embedding table" commit: embedBound takes the whole table and refuses
 * a bound below it).  Returns -1 and writes nothing when bound differs from the
 * table's row count (below it is the shard-width bug; above it would read past
 * the table).  An id at or past the bound fills its row with the bf16 NaN
 * 0x7FC0, so the error reaches the head and fails closed. */
int orc_embed_rows(const uint16_t *table, int64_t rows, int64_t H, int64_t ld, int64_t bound,
                   const uint32_t *ids, int M, uint16_t *out, int64_t ld_out)
{
    if (bound != rows || H < 0 || ld < H || ld_out < H)
        return -1;
#if ORC_PLANT == 11
    bound = bound / 2;
#endif
    for (int m = 0; m < M; ++m) {
        const uint32_t id = ids[m];
        for (int64_t j = 0; j < H; ++j)
            out[(int64_t)m * ld_out + j] = (int64_t)id < bound ? table[(int64_t)id * ld + j] : (uint16_t)ORC_NAN_BF16;
    }
    return 0;
}

/* ---------------------------------------------------------------- argmax -- */

/* For each row m of bf16 values v[m][0..n): the largest finite value with the
 * lowest index among equals, reported with global id id_base + j.  Any NaN,
 * +Inf or -Inf flags the row.  Word layout (u64):
 *   unflagged: high 32 = id, low 32 = the fp32 bits of the winning bf16 value
 *   flagged:   high 32 = 0x80000000 | (id_base + first non-finite j),
 *              low 32  = 0x7FC00000 (the NaN the pages report)
 * Returns -1 for n < 1. */
int orc_argmax_rows(const uint16_t *v, int M, int64_t n, int64_t ld, uint32_t id_base,
                    uint64_t *words)
{
    if (n < 1 || M < 0 || ld < n)
        return -1;
    for (int m = 0; m < M; ++m) {
        const uint16_t *r = v + (int64_t)m * ld;
        int flagged = 0;
        int64_t first_nf = 0, best = -1;
        double bestv = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double x = orc_bf16_to_f64(r[j]);
            if (!isfinite(x)) {
#if ORC_PLANT != 5
                if (!flagged) {
                    flagged = 1;
                    first_nf = j;
                }
#endif
                continue;
            }
#if ORC_PLANT == 3
            if (best < 0 || x >= bestv) {
#else
            if (best < 0 || x > bestv) {
#endif
                best = j;
                bestv = x;
            }
        }
        if (flagged) {
            uint32_t idw = ORC_FLAG | (id_base + (uint32_t)first_nf);
            words[m] = ((uint64_t)idw << 32) | 0x7FC00000u;
        } else if (best < 0) {
            /* every value was non-finite but flagging is planted away */
            words[m] = ((uint64_t)id_base << 32) | 0x7FC00000u;
        } else {
            uint32_t bits = (uint32_t)r[best] << 16;
            words[m] = ((uint64_t)(id_base + (uint32_t)best) << 32) | bits;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ pick -- */

static double orc_word_value(uint64_t w)
{
    uint32_t bits = (uint32_t)(w & 0xFFFFFFFFu);
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* words is [nparts][M].  For each row: if any part's id word has the flag bit,
 * the pick is 0xFFFFFFFF; otherwise the id of the larger value, the lower id
 * on equal values (+0 and -0 are equal). */
void orc_pick(const uint64_t *words, int nparts, int M, uint32_t *ids)
{
    for (int m = 0; m < M; ++m) {
        int flagged = 0;
        for (int p = 0; p < nparts; ++p) {
            uint32_t idw = (uint32_t)(words[(int64_t)p * M + m] >> 32);
#if ORC_PLANT == 6
            (void)idw;
#else
            if (idw & ORC_FLAG)
                flagged = 1;
#endif
        }
        if (flagged) {
            ids[m] = ORC_SENTINEL;
            continue;
        }
        uint32_t best_id = 0;
        double best_v = 0.0;
        for (int p = 0; p < nparts; ++p) {
            uint64_t w = words[(int64_t)p * M + m];
            uint32_t id = (uint32_t)(w >> 32);
            double v = orc_word_value(w);
#if ORC_PLANT == 4
            if (p == 0 || v > best_v || (v == best_v && id > best_id)) {
#else
            if (p == 0 || v > best_v || (v == best_v && id < best_id)) {
#endif
                best_id = id;
                best_v = v;
            }
        }
        ids[m] = best_id;
    }
}

/* ------------------------------------------------------- merged top two -- */

/* The session keeps the merged top two of the head for its cross-block tie test
 * (TensorFold PR #1433, step-1 and step-2 bodies: session.zig keeps the merged
 * top two and reads the pick's sentinel as a failure).  Reading: for each row,
 * the two highest entries in the argmax's own order -- the larger value first,
 * the lower id among equal values, +0 equal to -0 -- as two argmax words:
 * words2[2m] the winner (orc_argmax_rows' word) and words2[2m+1] the best of the
 * other ids.  A row holding any NaN, +Inf or -Inf is flagged: both words are the
 * argmax's flagged word.  A slice of one element has no second place: the word
 * ORC_TOP2_NONE (id 0x7FFFFFFF with the bits of -Inf, a value no unflagged
 * word carries).  Returns -1 for n < 1. */
#define ORC_TOP2_NONE ((((uint64_t)0x7FFFFFFFu) << 32) | 0xFF800000u)

static uint64_t orc_word_of(const uint16_t *r, int64_t j, uint32_t id_base)
{
    return ((uint64_t)(id_base + (uint32_t)j) << 32) | ((uint32_t)r[j] << 16);
}

int orc_top2_rows(const uint16_t *v, int M, int64_t n, int64_t ld, uint32_t id_base, uint64_t *words2)
{
    if (n < 1 || M < 0 || ld < n)
        return -1;
    for (int m = 0; m < M; ++m) {
        const uint16_t *r = v + (int64_t)m * ld;
        int flagged = 0;
        int64_t first_nf = 0, best = -1, second = -1;
        double bestv = 0.0, secondv = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double x = orc_bf16_to_f64(r[j]);
            if (!isfinite(x)) {
                if (!flagged) {
                    flagged = 1;
                    first_nf = j;
                }
                continue;
            }
            /* strict comparisons: among equal values the earlier (lower) id keeps its place */
            if (best < 0 || x > bestv) {
                second = best;
                secondv = bestv;
                best = j;
                bestv = x;
#if ORC_PLANT == 13
            } else if (x < bestv && (second < 0 || x > secondv)) {
#else
            } else if (second < 0 || x > secondv) {
#endif
                second = j;
                secondv = x;
            }
        }
        uint64_t *o = words2 + 2 * (int64_t)m;
        if (flagged) {
            uint32_t idw = ORC_FLAG | (id_base + (uint32_t)first_nf);
            o[0] = o[1] = ((uint64_t)idw << 32) | 0x7FC00000u;
        } else {
            o[0] = orc_word_of(r, best, id_base);
            o[1] = second < 0 ? ORC_TOP2_NONE : orc_word_of(r, second, id_base);
        }
    }
    return 0;
}

/* a ahead of b in the argmax order (NONE is behind everything) */
static int orc_word_ahead(uint64_t a, uint64_t b)
{
    if (a == ORC_TOP2_NONE)
        return 0;
    if (b == ORC_TOP2_NONE)
        return 1;
    double va = orc_word_value(a), vb = orc_word_value(b);
    return va > vb || (va == vb && (uint32_t)(a >> 32) < (uint32_t)(b >> 32));
}

/* words2 is [nparts][M][2] as orc_top2_rows writes it for slices of one
 * vocabulary.  For each row: if any part is flagged, both merged words are the
 * flagged word of the lowest such part (the pick fails closed on it); otherwise
 * the two highest of all the parts' words in the argmax order. */
void orc_top2_merge(const uint64_t *words2, int nparts, int M, uint64_t *out2)
{
    for (int m = 0; m < M; ++m) {
        uint64_t *o = out2 + 2 * (int64_t)m;
        int done = 0;
        for (int p = 0; p < nparts && !done; ++p) {
            uint64_t w = words2[((int64_t)p * M + m) * 2];
            if ((uint32_t)(w >> 32) & ORC_FLAG) {
                o[0] = o[1] = w;
                done = 1;
            }
        }
        if (done)
            continue;
        uint64_t best = ORC_TOP2_NONE, second = ORC_TOP2_NONE;
#if ORC_PLANT == 14
        int best_part = -1;
        for (int p = 0; p < nparts; ++p) {
            uint64_t w = words2[((int64_t)p * M + m) * 2];
            if (orc_word_ahead(w, best)) {
                best = w;
                best_part = p;
            }
        }
        second = words2[((int64_t)best_part * M + m) * 2 + 1];
#else
        for (int p = 0; p < nparts; ++p)
            for (int i = 0; i < 2; ++i) {
                uint64_t w = words2[((int64_t)p * M + m) * 2 + i];
                if (orc_word_ahead(w, best)) {
                    second = best;
                    best = w;
                } else if (orc_word_ahead(w, second)) {
                    second = w;
                }
            }
#endif
        o[0] = best;
        o[1] = second;
    }
}

/* ------------------------------------------------------------ top-two gap -- */

/* gap[m] = best - (largest value at any other index), on unrounded double
 * logits [M][n]; +Inf when n == 1.  The end-to-end id check only trusts ids
 * whose gap exceeds the stated margin. */
void orc_top2_gap(const double *logits, int M, int64_t n, double *gap)
{
    for (int m = 0; m < M; ++m) {
        const double *r = logits + (int64_t)m * n;
        int64_t best = 0;
        for (int64_t j = 1; j < n; ++j)
            if (r[j] > r[best])
                best = j;
        double second = -INFINITY;
        for (int64_t j = 0; j < n; ++j)
            if (j != best && r[j] > second)
                second = r[j];
        gap[m] = (n == 1) ? INFINITY : r[best] - second;
    }
}
