/*
 * tf.h -- C ABI of libtf.so, the row-split int4 hot path on one NVIDIA B200.
 *
 * The library computes, on the GPU, the steps the TensorFold pair seam is made
 * of (TensorFold PR #1433, "Step 1 of 6" body and step-2 "What this changes"):
 * a 4-bit affine quantized projection over a slice of output rows, each row
 * reduced over the whole K by whoever owns it; a pure copy that joins the
 * slices; the head's argmax over each half of the vocabulary; and the pick
 * between the halves.  The two ranks of the pages are emulated as two row
 * ranges of one matrix on one GPU: no collective, no second device.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers named x, wq, scales, biases, y, dst, parts[], logits, words,
 *    ids and scratch are DEVICE pointers (cudaMalloc'd or torch tensors on
 *    the current device).  Arrays of pointers and sizes (segs, parts, widths)
 *    are HOST arrays, read before the call returns.
 *  - bf16 values are passed as their 16-bit patterns (bf16 = top half of an
 *    IEEE fp32), row-major with the stated leading dimension in elements.
 *  - The caller owns every buffer.  The library allocates nothing, keeps no
 *    pointer after the call returns and never synchronises the stream: work
 *    is enqueued on `stream` (NULL = the legacy default stream) and results
 *    are valid once that stream reaches them.
 *  - Every argument is validated on the host BEFORE anything is enqueued; a
 *    rejected call moves no data ("refuse by name before any state moves",
 *    TensorFold PR #1434 review thread).  The one exception is TF_E_BROKEN,
 *    which is a result, not a refusal (see tf_gather_rows).
 *  - No entry point exits, aborts, traps or prints.  A failed launch returns
 *    TF_E_CUDA (the CUDA error is left for cudaGetLastError to report).
 *  - Kernels are launched with programmatic dependent launch: a kernel may
 *    be scheduled while the kernel before it on the stream still runs, and
 *    waits (griddepcontrol.wait) for that kernel to finish before it reads
 *    any of its arguments' arrays or writes any output, with one exception:
 *    a qmm kernel may read weights (codes, scales, biases) before that wait.
 *    The library never writes weights, and a kernel of the caller's lets the
 *    next kernel start only once it has ended, so weights it wrote are in
 *    place; callers see plain stream order.  Setting the environment
 *    variable TF_PDL=0 before the first call launches without it.
 *  - Outputs must not overlap inputs.
 */
#ifndef TF_H
#define TF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so that callers need no CUDA header. */
typedef struct CUstream_st *tf_stream;

typedef enum {
    TF_OK = 0,
    TF_E_ARG = 1,     /* a NULL pointer, a count or size out of its stated range */
    TF_E_RANGE = 2,   /* a row segment outside [0, N_whole), overlapping segments, or ids past 2^31 */
    TF_E_ALIGN = 3,   /* a pointer or leading dimension without the stated alignment */
    TF_E_WINDOW = 4,  /* a part of a gather is larger than the exchange window */
    TF_E_BROKEN = 5,  /* a gather part was missing: its columns were filled with 0x7FC0 */
    TF_E_CUDA = 6,    /* a kernel launch failed */
    TF_E_UNIMPL = 7   /* a valid request this build does not implement */
} tf_status;

/* Bit 31 of an argmax id word: the row held a NaN or +-Inf
 * (TensorFold PR #1433 step-1 body: "NaN bits with bit 31 set in its id word"). */
#define TF_PAIR_FLAG 0x80000000u
/* tf_pick's result for a flagged row; never a token id
 * (TensorFold PR #1433 step-2 body: the session reads maxInt(u32) as error.PairFailed). */
#define TF_PICK_FAILED 0xFFFFFFFFu
/* the second place of a one-element slice (tf_top2_rows): id 0x7FFFFFFF with the
 * fp32 bits of -Inf, a value no unflagged word carries */
#define TF_TOP2_NONE ((0x7FFFFFFFull << 32) | 0xFF800000ull)
/* The bf16 NaN a missing gather part reads as (TensorFold PR #1433 step-1 body). */
#define TF_NAN_BF16 0x7FC0u
/* Rows one qmm call may carry: chunk(requested) = min(requested, 128)
 * (TensorFold PR #1434, step-3 body: batch_rows = 128). */
#define TF_BATCH_ROWS 128
/* K elements sharing one bf16 scale and one bf16 bias (TensorFold PR #1437 Receipt:
 * "4-bit affine with group 64"). */
#define TF_GROUP 64
#define TF_MAX_K 65536
#define TF_MAX_SEGS 8
#define TF_MAX_PARTS 8
/* Pass as window_bytes to skip the gather's window check. */
#define TF_NO_WINDOW ((size_t)-1)

/* A range of rows of the WHOLE checkpoint matrix: [row0, row0 + nrows). */
typedef struct {
    int32_t row0;
    int32_t nrows;
} tf_seg;

typedef enum {
    TF_EPI_NONE = 0, /* y holds the bf16 qmm outputs of every listed row */
    TF_EPI_GLU = 1   /* two equal segments (gate rows, up rows): y[i] = bf16(g_i * SiLU(u_i)) */
} tf_epi;

/*
 * tf_qmm_rows -- 4-bit affine quantized matrix-vector / matrix product over a
 * slice of output rows, reduced over the full K in fp32.
 *
 * Defines (TensorFold PR #1433 step-1 body: "rank r owns 2,560 of the 5,120
 * output columns ..., reduces over the full K on its own rank"; PR #1437
 * Receipt: 4-bit affine, group 64):
 *     w[n,k]  = s[n, k/64] * q[n,k] + b[n, k/64]
 *     out[m,n] = bf16_RNE( sum_{k<K} x[m,k] * w[n,k] )   (fp32 accumulation)
 * for every row n of the segments, in segment order.  The summation order
 * depends on K alone -- never on the segments, their order, N_whole or a row's
 * position in a chunk -- so a row computed in a slice has the same bits as the
 * same row computed in the whole matrix (PR #1433 review: "a different sk is
 * a different fp32 order").  With M <= 3 (and K % 512 == 0, 16-byte aligned
 * weights) each activation row's outputs are bit for bit those of a call with
 * that row alone; calls of 4 or more rows run on the tensor cores, whose rows
 * agree with one another but not bit for bit with the M <= 3 calls (both meet
 * the same 2-ulp bar).  A 32-value run of x dominated by one or two outliers
 * (no third value within 2^4 of its largest) is summed as a plain fp32 dot,
 * so an outlier whose weight is zero adds exactly nothing.
 *
 *   x       bf16 [M][ldx] activations.  16-byte aligned, ldx % 8 == 0, ldx >= K.
 *   M       rows of x, 0 <= M <= TF_BATCH_ROWS (M == 0: nothing is enqueued).
 *           Callers split larger requests into chunks of TF_BATCH_ROWS.
 *   K       reduction length, 64 <= K <= TF_MAX_K, K % 64 == 0.
 *   wq      uint8 [N_whole][K/2] packed codes of the whole matrix; element k of
 *           a row is byte k/2, low nibble for even k, high nibble for odd k;
 *           q is unsigned 0..15.  16-byte aligned.
 *   scales  bf16 [N_whole][K/64]; biases bf16 [N_whole][K/64].  2-byte aligned.
 *   N_whole rows of the whole matrix (>= 1).
 *   segs    host array of nseg row ranges of the whole matrix, 1 <= nseg <= TF_MAX_SEGS,
 *           inside [0, N_whole) and pairwise disjoint (TF_E_RANGE otherwise).
 *   epi     TF_EPI_NONE: y[m][c] for c < sum(nrows) is the c-th listed row.
 *           TF_EPI_GLU: nseg == 2 with equal nrows F; g and u are the bf16
 *           outputs of row segs[0].row0+i and segs[1].row0+i, and
 *           y[m][i] = bf16_RNE(g * SiLU(u)), SiLU(u) = u / (1 + exp(-u)), in fp32.
 *   y       bf16 [M][ldy], ldy >= the number of output columns.  2-byte aligned.
 * Errors: TF_E_ARG, TF_E_RANGE, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
tf_status tf_qmm_rows(const void *x, int M, int K, int ldx,
                      const uint8_t *wq, const void *scales, const void *biases, int N_whole,
                      const tf_seg *segs, int nseg, tf_epi epi,
                      void *y, int ldy, tf_stream stream);

/*
 * tf_gather_rows -- join row slices into the whole frame by copying whole bf16
 * rows; no arithmetic (TensorFold PR #1433 step-1 body: pair_gather copies
 * whole rows in bf16 without doing any arithmetic; step-2 body: gather copies
 * each rank's half to its own offset).
 *
 *     dst[m][off_h + j] = parts[h][m][j],   off_h = widths[0] + ... + widths[h-1]
 *
 *   dst     bf16 [M][ld_dst], ld_dst >= sum(widths).
 *   parts   host array of nparts device pointers, part h dense bf16 [M][widths[h]];
 *           1 <= nparts <= TF_MAX_PARTS.  A NULL part is a broken link.
 *   widths  host array, widths[h] >= 0.
 *   window_bytes  the exchange window: every part must satisfy
 *           M * widths[h] * 2 <= window_bytes, else TF_E_WINDOW and nothing is
 *           enqueued (PR #1434: seamBytes(rows) = rows * 8,704 * 2 must fit
 *           pairBytes; the cap exists so that the widest seam never exceeds it).
 *           TF_NO_WINDOW skips the check.
 * Result: TF_OK; or TF_E_BROKEN when a part was NULL -- its columns are filled
 * with TF_NAN_BF16 (0x7FC0), the other parts are copied, and everything is
 * enqueued before the call returns (PR #1433: a broken link surfaces as bf16 NaN).
 * Errors: TF_E_ARG, TF_E_WINDOW (before any launch), TF_E_CUDA.
 */
tf_status tf_gather_rows(void *dst, int ld_dst, const void *const *parts, const int *widths,
                         int nparts, int M, size_t window_bytes, tf_stream stream);

/*
 * tf_argmax_rows -- argmax over one slice of the vocabulary for each row
 * (TensorFold PR #1433 step-1 body: pair_argmax; step-2 body: argmax over each
 * rank's 124,160-logit half).
 *
 * For each row m of logits[m][0..n): the largest finite value, the LOWEST id
 * among equal values (+0 and -0 are equal).  Ids are global: id_base + j.  A
 * row holding any NaN, +Inf or -Inf is flagged.  One 64-bit word per row:
 *     unflagged: bits 63..32 = id, bits 31..0 = fp32 bits of the winning bf16
 *                (its bf16 pattern << 16, the sign of a winning -0 kept)
 *     flagged:   bits 63..32 = TF_PAIR_FLAG | (id_base + first non-finite j),
 *                bits 31..0  = 0x7FC00000
 *
 *   logits  bf16 [M][ld], ld >= n, 2-byte aligned (16-byte aligned with
 *           ld % 8 == 0 takes the vector path; both give the same result).
 *   M       0 <= M <= 65535;  n >= 1;  id_base + n <= 2^31 (TF_E_RANGE).
 *   words   uint64 [M].
 *   scratch device buffer of at least tf_argmax_scratch_bytes(M, n) bytes,
 *           8-byte aligned, owned by the caller; its contents on entry do not
 *           matter and on return are unspecified.  Two calls in flight at
 *           the same time need two scratch buffers.
 * Errors: TF_E_ARG, TF_E_RANGE, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
size_t tf_argmax_scratch_bytes(int M, int n);
tf_status tf_argmax_rows(const void *logits, int M, int n, int ld, uint32_t id_base,
                         uint64_t *words, void *scratch, size_t scratch_bytes, tf_stream stream);

/*
 * tf_qmm8_rows -- the int8 head variant: the b70 lab's "runtime INT8 target
 * LM-head" with a bf16 scale ("Reproduce Qwen3.6 27B AutoRound Bring-Up",
 * *Reproduce The TP1 One-Replica Result*; the pages give no other detail).
 *
 * y[m][c] = bf16_RNE( s[n] * sum_{k<K} x[m][k] * q8[n][k] ), n the whole-matrix
 * row of output column c (segments as in tf_qmm_rows, TF_EPI_NONE), the sum in
 * fp32 over the whole K on this device, in an order fixed by K alone.
 *   x       bf16 [M][ldx], 1 <= K <= TF_MAX_K, ldx >= K, 0 <= M <= TF_BATCH_ROWS.
 *   q8      int8 [N_whole][K], row-major, signed codes (no zero point).
 *   scales  bf16 [N_whole], one per row.
 *   y       bf16 [M][ldy], ldy >= the number of columns.
 *   M = 1 with K % 32 == 0 and a 16-byte aligned q8 streams the codes through
 *   shared memory (bulk copies, dp4a); other calls take a plain warp-per-output
 *   kernel.  A row's bits depend on which of the two ran, never on the other rows.
 * Errors: TF_E_ARG, TF_E_RANGE, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
tf_status tf_qmm8_rows(const void *x, int M, int K, int ldx, const int8_t *q8, const void *scales, int N_whole,
                       const tf_seg *segs, int nseg, void *y, int ldy, tf_stream stream);

/*
 * tf_qmm_argmax_rows -- the head of one rank in one call: the logits of one row
 * slice (tf_qmm_rows, TF_EPI_NONE, one segment) and their argmax word
 * (tf_argmax_rows over those logits with ids id_base + j).  The step-1 body of
 * TensorFold PR #1433 has each rank compute its half of the lm_head and then
 * pair_argmax over it; here, at M = 1, every warp of the qmm keeps the best key
 * of the rows it writes and leaves it in scratch, and one single-CTA kernel
 * combines those keys into the word, so the argmax makes no pass over the
 * logits.  The results are bit for bit those of the two separate
 * calls: the logits equal tf_qmm_rows' and the word equals tf_argmax_rows' on
 * them.  For M > 1, or a weight layout the M = 1 streaming kernel does not take,
 * the same two kernels run one after the other.
 *
 *   x, M, K, ldx, wq, scales, biases, N_whole   as tf_qmm_rows.
 *   seg     the slice: whole-matrix rows [row0, row0 + nrows), nrows >= 1.
 *   id_base global id of logit column 0 (usually seg.row0); id_base + nrows
 *           <= 2^31 (TF_E_RANGE).
 *   logits  bf16 [M][ld_logits], ld_logits >= nrows: written, as tf_qmm_rows' y.
 *   words   uint64 [M], the argmax words (format of tf_argmax_rows).
 *   scratch device buffer of at least tf_qmm_argmax_scratch_bytes(M, nrows)
 *           bytes, 8-byte aligned, owned by the caller; contents on entry do not
 *           matter and on return are unspecified.  Calls in flight at the same
 *           time need separate scratch buffers.
 * Errors: TF_E_ARG, TF_E_RANGE, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
size_t tf_qmm_argmax_scratch_bytes(int M, int nrows);
tf_status tf_qmm_argmax_rows(const void *x, int M, int K, int ldx, const uint8_t *wq, const void *scales,
                             const void *biases, int N_whole, tf_seg seg, uint32_t id_base, void *logits,
                             int ld_logits, uint64_t *words, void *scratch, size_t scratch_bytes, tf_stream stream);

/*
 * tf_residual_add -- the fp32 residual stream after a seam (TensorFold PR #1433
 * step-2 body: o_proj and down_proj stage their own output rows, gather the
 * peer's as whole bf16 rows, and add in the fp32 stream, so no two bf16
 * partials are summed).
 *
 * h[m][j] = fp32(h[m][j] + y[m][j]) for m < M, j < n: the IEEE fp32 addition,
 * one rounding to nearest even; NaN and +-Inf follow IEEE.
 *   h   fp32 [M][ld_h], ld_h >= n, 4-byte aligned, updated in place.
 *   y   bf16 [M][ld_y], ld_y >= n, 2-byte aligned (e.g. a tf_gather_rows frame).
 *   16-byte aligned pointers with ld_h % 4 == 0 and ld_y % 8 == 0 take the vector
 *   path; both paths give the same bits.  M == 0 or n == 0 does nothing.
 * Errors: TF_E_ARG, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
tf_status tf_residual_add(float *h, int ld_h, const void *y, int ld_y, int M, int n, tf_stream stream);

/*
 * tf_embed_rows -- the embedding rows of M token ids from the whole table
 * (TensorFold PR #1433 step-2 body: embeddings stay whole on every rank, so a
 * token id means the same thing on both, and the gather's bound stays the whole
 * 248,320-row table; the "Rank-slice the qwen27 family and gather the whole
 * embedding table" commit: embedBound takes the whole table and refuses a bound
 * below it).
 *
 * out[m][:H] = table[ids[m]][:H]; an id >= bound makes row m the bf16 NaN
 * 0x7FC0 everywhere, so the error reaches the head and fails closed.
 *   table  bf16 [rows][ld_table], ld_table >= H, 2-byte aligned.
 *   bound  must equal rows: a smaller bound (the shard's width, e.g. 124,160 of
 *          248,320) is the bug the pages fixed and a larger one would read past
 *          the table; either is refused with TF_E_RANGE before any launch.
 *   ids    uint32 [M] on the device.   out  bf16 [M][ld_out], ld_out >= H.
 *   16-byte aligned table and out with both leading dimensions % 8 == 0 take
 *   the vector path.  M == 0 or H == 0 does nothing.
 * Errors: TF_E_ARG, TF_E_RANGE, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
tf_status tf_embed_rows(const void *table, int rows, int H, int ld_table, int bound, const uint32_t *ids, int M,
                        void *out, int ld_out, tf_stream stream);

/*
 * tf_pick -- the better of the per-slice winners (TensorFold PR #1433 step-1
 * body: pair_pick; the sixth control's test ((am | ap) & PAIR_FLAG) != 0u).
 *
 * words is uint64 [nparts][M] (word of part p for row m at p*M + m), as
 * written by tf_argmax_rows.  For each row: if ANY part's id word has
 * TF_PAIR_FLAG, ids[m] = TF_PICK_FAILED; otherwise the id of the larger value,
 * and on equal values the lower id.  nparts == 1 applies the same flag rule to
 * a whole-vocabulary word.  1 <= nparts <= TF_MAX_PARTS, 0 <= M <= 65535.
 *   ids     uint32 [M].
 * Errors: TF_E_ARG (before any launch), TF_E_CUDA.
 */
tf_status tf_pick(const uint64_t *words, int nparts, int M, uint32_t *ids, tf_stream stream);

/*
 * tf_top2_rows -- the top two of one slice of the vocabulary for each row (the
 * merged top two of TensorFold PR #1433, step-1 and step-2 bodies: the session
 * keeps the merged top two for its cross-block tie test, and reads the pick's
 * sentinel as a failure).
 *
 * For each row m of logits[m][0..n), two words in tf_argmax_rows' format and
 * order (larger value first, the lower id among equal values, +0 equal to -0):
 *     words2[2m]     the winner -- the word tf_argmax_rows writes;
 *     words2[2m + 1] the best of the other ids; an exact tie gives the same
 *                    value with the next id; TF_TOP2_NONE when n == 1.
 * A row holding any NaN, +Inf or -Inf gets its flagged argmax word twice.
 *   logits, M, n, ld, id_base   as tf_argmax_rows (same limits and vector path).
 *   words2  uint64 [M][2].
 *   scratch device buffer of at least tf_top2_scratch_bytes(M, n) bytes, 8-byte
 *           aligned, owned by the caller; contents on entry do not matter.
 * Errors: TF_E_ARG, TF_E_RANGE, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
size_t tf_top2_scratch_bytes(int M, int n);
tf_status tf_top2_rows(const void *logits, int M, int n, int ld, uint32_t id_base, uint64_t *words2, void *scratch,
                       size_t scratch_bytes, tf_stream stream);

/*
 * tf_top2_merge -- the merged top two across slices (the same passage).
 *
 * words2 is uint64 [nparts][M][2] as tf_top2_rows writes it for slices of one
 * vocabulary (part p, row m at (p*M + m)*2).  For each row: if any part's winner
 * is flagged, both merged words are the flagged word of the lowest such part
 * (tf_pick fails closed on the same rows); otherwise the two highest of all the
 * parts' words in the argmax order.  The merged winner's id is tf_pick's id.
 * 1 <= nparts <= TF_MAX_PARTS, 0 <= M <= 65535.
 *   out2    uint64 [M][2] (not overlapping words2).
 * Errors: TF_E_ARG, TF_E_ALIGN (before any launch), TF_E_CUDA.
 */
tf_status tf_top2_merge(const uint64_t *words2, int nparts, int M, uint64_t *out2, tf_stream stream);

/*
 * tf_argmax_rows_static -- tf_argmax_rows for callers that cannot allocate
 * device memory.  The pages have no counterpart of this entry point; it exists
 * for hosts that own every byte of device memory up front (a fixed arena that
 * forbids any other cudaMalloc) and for latency paths where the implicit
 * device synchronisation of cudaMalloc/cudaFree is not acceptable.
 *
 * Same arguments, result and errors as tf_argmax_rows, without the scratch
 * arguments: the per-block partial results go to a device array built into
 * libtf.so (TF_STATIC_SCRATCH_BYTES bytes, present on every GPU that loads the
 * library, for as long as the process lives).  Nothing is allocated and no
 * allocating routine is called.
 *   - TF_E_ARG when tf_argmax_scratch_bytes(M, n) > TF_STATIC_SCRATCH_BYTES
 *     (for example M = 8,193 rows of any length); nothing is enqueued.
 *   - The first call on a device looks up that array's device address
 *     (cudaGetSymbolAddress, with the device current) and keeps it, with the
 *     id of the CUDA context it belongs to; make that first call before any
 *     stream capture.  After cudaDeviceReset (or any other teardown of the
 *     context) the next call finds a new context id and looks the address up
 *     again, so a stale address is never used.  A failed lookup returns
 *     TF_E_CUDA.
 *   - Every call on a device uses the same array, and the array keeps what the
 *     last call left there.  Each call writes every entry it later reads, so no
 *     clearing is needed, but two calls whose kernels overlap on the GPU (other
 *     streams, or other host threads) race on it: order them on one stream, or
 *     use tf_argmax_rows with a scratch buffer per stream.
 */
#define TF_STATIC_SCRATCH_BYTES ((size_t)64 * 1024)
tf_status tf_argmax_rows_static(const void *logits, int M, int n, int ld, uint32_t id_base, uint64_t *words,
                                tf_stream stream);

/*
 * Host arithmetic of the row split (TensorFold PR #1433 step-2 body: the split
 * is by output rows, rank 0's spans start at 0; 2,560 of 5,120, 8,704 of
 * 17,408, 124,160 of 248,320; "the fused gate-up keeps the member split").
 *   tf_split_rows   part h of nparts owns rows [h*N/nparts, (h+1)*N/nparts) of an
 *                   N-row matrix; *seg receives them.  TF_E_ARG unless
 *                   1 <= nparts <= TF_MAX_PARTS, 0 <= h < nparts, N >= 0 and
 *                   N % nparts == 0 (an uneven split is refused, not rounded).
 *   tf_member_segs  for a fused stack [gate(F rows); up(F rows)] (2F rows in all),
 *                   part h owns gate rows [h*F/nparts, +F/nparts) and the same rows
 *                   of up: segs[0] = gate range, segs[1] = up range (offset by F).
 *                   Same errors as tf_split_rows, with F in place of N.
 * Pure host functions; they touch no device.
 */
tf_status tf_split_rows(int N, int nparts, int h, tf_seg *seg);
tf_status tf_member_segs(int F, int nparts, int h, tf_seg segs[2]);

/*
 * Host arithmetic of the seam window (TensorFold PR #1434, step-3 body):
 *   tf_chunk_rows(requested)      = min(requested, TF_BATCH_ROWS)   (requested >= 0)
 *   tf_seam_bytes(rows, width)    = rows * width * 2                 (bf16 bytes of one part)
 * Both are pure functions; they touch no device.
 */
int tf_chunk_rows(int requested);
size_t tf_seam_bytes(int rows, int width);

/* Static name of a status ("TF_OK", "TF_E_ARG", ...); "TF_E_?" for an unknown value. */
const char *tf_status_str(tf_status s);

/* The CUDA runtime's message for the error behind the last TF_E_CUDA that a
 * tf_* call returned on the calling host thread ("no error" before any).  The
 * string has static storage; the call never fails and never returns NULL.
 * Not an operation of the pages: it only makes TF_E_CUDA diagnosable. */
const char *tf_last_cuda_error(void);

/* ABI version of this header; bumped when a signature changes. */
#define TF_ABI_VERSION 1
int tf_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TF_H */
