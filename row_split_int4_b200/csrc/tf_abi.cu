// tf_abi.cu -- the extern "C" entry points of libtf.so (declared in include/tf.h).
//
// Each entry point validates every argument on the host and refuses a bad
// call by status before anything is enqueued (TensorFold PR #1434 review
// thread: refuse by name before the backend moves any state; fail closed).
#include <climits>
#include <cstdlib>
#include <cstring>

#include "tf_common.cuh"
#include "tf_kernels.h"


namespace tf {

// The CUDA error behind the last TF_E_CUDA returned on this host thread.
static thread_local cudaError_t g_last_cuda = cudaSuccess;

tf_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TF_OK;
    g_last_cuda = e;
    return TF_E_CUDA;
}

cudaError_t last_cuda_error() { return g_last_cuda; }

bool pdl_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("TF_PDL");
        return !(v && v[0] == '0');
    }();
    return on;
}

}  // namespace tf

using namespace tf;

extern "C" {

const char *tf_status_str(tf_status s) {
    switch (s) {
    case TF_OK: return "TF_OK";
    case TF_E_ARG: return "TF_E_ARG";
    case TF_E_RANGE: return "TF_E_RANGE";
    case TF_E_ALIGN: return "TF_E_ALIGN";
    case TF_E_WINDOW: return "TF_E_WINDOW";
    case TF_E_BROKEN: return "TF_E_BROKEN";
    case TF_E_CUDA: return "TF_E_CUDA";
    case TF_E_UNIMPL: return "TF_E_UNIMPL";
    }
    return "TF_E_?";
}

int tf_abi_version(void) { return TF_ABI_VERSION; }

tf_status tf_split_rows(int N, int nparts, int h, tf_seg *seg) {
    if (seg == nullptr || nparts < 1 || nparts > TF_MAX_PARTS || h < 0 || h >= nparts || N < 0 || N % nparts != 0)
        return TF_E_ARG;
    const int w = N / nparts;
    seg->row0 = h * w;
    seg->nrows = w;
    return TF_OK;
}

tf_status tf_member_segs(int F, int nparts, int h, tf_seg segs[2]) {
    if (segs == nullptr || F > INT_MAX / 2) return TF_E_ARG;
    tf_seg g;
    const tf_status st = tf_split_rows(F, nparts, h, &g);
    if (st != TF_OK) return st;
    segs[0] = g;
    segs[1].row0 = F + g.row0;
    segs[1].nrows = g.nrows;
    return TF_OK;
}

int tf_chunk_rows(int requested) {
    if (requested < 0) return 0;
    return requested < TF_BATCH_ROWS ? requested : TF_BATCH_ROWS;
}

size_t tf_seam_bytes(int rows, int width) {
    if (rows <= 0 || width <= 0) return 0;
    return (size_t)rows * (size_t)width * 2u;
}

const char *tf_last_cuda_error(void) { return cudaGetErrorString(last_cuda_error()); }

// Validation and argument block shared by tf_qmm_rows and tf_qmm_argmax_rows.
// TF_OK with *empty set means there is nothing to compute.
static tf_status qmm_args(const void *x, int M, int K, int ldx, const uint8_t *wq, const void *scales,
                          const void *biases, int N_whole, const tf_seg *segs, int nseg, tf_epi epi, void *y, int ldy,
                          QmmArgs *out, bool *empty) {
    *empty = false;
    if (M < 0 || M > TF_BATCH_ROWS) return TF_E_ARG;
    if (K < TF_GROUP || K > TF_MAX_K || K % TF_GROUP != 0) return TF_E_ARG;
    if (N_whole < 1) return TF_E_ARG;
    if (segs == nullptr || nseg < 1 || nseg > TF_MAX_SEGS) return TF_E_ARG;
    if (epi != TF_EPI_NONE && epi != TF_EPI_GLU) return TF_E_ARG;
    if (epi == TF_EPI_GLU && (nseg != 2 || segs[0].nrows != segs[1].nrows)) return TF_E_ARG;

    SegTable t;
    std::memset(&t, 0, sizeof t);
    long long cols = 0;
    for (int i = 0; i < nseg; ++i) {
        const long long r0 = segs[i].row0, nr = segs[i].nrows;
        if (r0 < 0 || nr < 0 || r0 + nr > N_whole) return TF_E_RANGE;
        for (int j = 0; j < i; ++j) {
            const long long a0 = segs[j].row0, an = segs[j].nrows;
            if (nr > 0 && an > 0 && r0 < a0 + an && a0 < r0 + nr) return TF_E_RANGE;
        }
        t.row0[i] = (int)r0;
        t.nrows[i] = (int)nr;
        t.col0[i] = (int)cols;
        cols += nr;
    }
    t.nseg = nseg;
    t.ncols = (epi == TF_EPI_GLU) ? segs[0].nrows : (int)cols;
    if (cols > INT_MAX) return TF_E_RANGE;
    if (ldx < K || ldy < t.ncols) return TF_E_ARG;
    if (M == 0 || t.ncols == 0) {
        *empty = true;
        return TF_OK;
    }
    if (!x || !wq || !scales || !biases || !y) return TF_E_ARG;
    if (!aligned(x, 16) || ldx % 8 != 0 || !aligned(wq, 16) || !aligned(scales, 2) || !aligned(biases, 2) ||
        !aligned(y, 2))
        return TF_E_ALIGN;

    QmmArgs &a = *out;
    std::memset(&a, 0, sizeof a);
    a.x = static_cast<const uint16_t *>(x);
    a.M = M;
    a.K = K;
    a.ldx = ldx;
    a.wq = wq;
    a.scales = static_cast<const uint16_t *>(scales);
    a.biases = static_cast<const uint16_t *>(biases);
    a.seg = t;
    a.glu = epi == TF_EPI_GLU;
    a.y = static_cast<uint16_t *>(y);
    a.ldy = ldy;
    a.n_whole = N_whole;
    a.cand = nullptr;
    a.id_base = 0;
    return TF_OK;
}

tf_status tf_qmm_rows(const void *x, int M, int K, int ldx, const uint8_t *wq, const void *scales,
                      const void *biases, int N_whole, const tf_seg *segs, int nseg, tf_epi epi, void *y,
                      int ldy, tf_stream stream) {
    QmmArgs a;
    bool empty = false;
    const tf_status st = qmm_args(x, M, K, ldx, wq, scales, biases, N_whole, segs, nseg, epi, y, ldy, &a, &empty);
    if (st != TF_OK || empty) return st;
    return cuda_status(launch_qmm(a, reinterpret_cast<cudaStream_t>(stream)));
}

tf_status tf_qmm8_rows(const void *x, int M, int K, int ldx, const int8_t *q8, const void *scales, int N_whole,
                       const tf_seg *segs, int nseg, void *y, int ldy, tf_stream stream) {
    if (M < 0 || M > TF_BATCH_ROWS) return TF_E_ARG;
    if (K < 1 || K > TF_MAX_K) return TF_E_ARG;
    if (N_whole < 1) return TF_E_ARG;
    if (segs == nullptr || nseg < 1 || nseg > TF_MAX_SEGS) return TF_E_ARG;
    Qmm8Args a;
    std::memset(&a, 0, sizeof a);
    long long cols = 0;
    for (int i = 0; i < nseg; ++i) {
        const long long r0 = segs[i].row0, nr = segs[i].nrows;
        if (r0 < 0 || nr < 0 || r0 + nr > N_whole) return TF_E_RANGE;
        for (int j = 0; j < i; ++j) {
            const long long a0 = segs[j].row0, an = segs[j].nrows;
            if (nr > 0 && an > 0 && r0 < a0 + an && a0 < r0 + nr) return TF_E_RANGE;
        }
        a.seg.row0[i] = (int)r0;
        a.seg.nrows[i] = (int)nr;
        a.seg.col0[i] = (int)cols;
        cols += nr;
    }
    if (cols > INT_MAX) return TF_E_RANGE;
    a.seg.nseg = nseg;
    a.seg.ncols = (int)cols;
    if (ldx < K || ldy < a.seg.ncols) return TF_E_ARG;
    if (M == 0 || a.seg.ncols == 0) return TF_OK;
    if (!x || !q8 || !scales || !y) return TF_E_ARG;
    if (!aligned(x, 2) || !aligned(scales, 2) || !aligned(y, 2)) return TF_E_ALIGN;
    a.x = static_cast<const uint16_t *>(x);
    a.M = M;
    a.K = K;
    a.ldx = ldx;
    a.q8 = q8;
    a.scales = static_cast<const uint16_t *>(scales);
    a.y = static_cast<uint16_t *>(y);
    a.ldy = ldy;
    return cuda_status(launch_qmm8(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t tf_qmm_argmax_scratch_bytes(int M, int nrows) {
    if (M <= 0 || nrows <= 0) return 0;
    // fused: one key per warp of the grid
    const size_t fused = (size_t)qmm_m1_stream_max_cand() * sizeof(uint64_t);
    const size_t plain = tf_argmax_scratch_bytes(M, nrows);
    return fused > plain ? fused : plain;
}

tf_status tf_qmm_argmax_rows(const void *x, int M, int K, int ldx, const uint8_t *wq, const void *scales,
                             const void *biases, int N_whole, tf_seg seg, uint32_t id_base, void *logits,
                             int ld_logits, uint64_t *words, void *scratch, size_t scratch_bytes, tf_stream stream) {
    if (seg.nrows < 1) return TF_E_ARG;
    if ((unsigned long long)id_base + (unsigned long long)seg.nrows > 0x80000000ull) return TF_E_RANGE;
    QmmArgs a;
    bool empty = false;
    const tf_status st =
        qmm_args(x, M, K, ldx, wq, scales, biases, N_whole, &seg, 1, TF_EPI_NONE, logits, ld_logits, &a, &empty);
    if (st != TF_OK || empty) return st;
    if (!words || !scratch) return TF_E_ARG;
    if (!aligned(words, 8) || !aligned(scratch, 8)) return TF_E_ALIGN;
    if (scratch_bytes < tf_qmm_argmax_scratch_bytes(M, seg.nrows)) return TF_E_ARG;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (M == 1 && qmm_m1_stream_eligible(a)) {
        // fused: the qmm warps leave their best keys in scratch, one small kernel
        // turns them into the word
        a.cand = static_cast<uint64_t *>(scratch);
        a.id_base = id_base;
        int ncand = 0;
        const tf_status q = cuda_status(launch_qmm_m1_stream(a, s, &ncand));
        if (q != TF_OK) return q;
        return cuda_status(launch_argmax_keys(a.cand, ncand, a.y, id_base, words, s));
    }
    // otherwise the two steps: the rows, then the argmax over them
    const tf_status q = cuda_status(launch_qmm(a, s));
    if (q != TF_OK) return q;
    ArgmaxArgs g;
    std::memset(&g, 0, sizeof g);
    g.logits = a.y;
    g.ld = ld_logits;
    g.n = seg.nrows;
    g.id_base = id_base;
    g.M = M;
    g.partial = static_cast<uint64_t *>(scratch);
    g.words = words;
    g.vec = aligned(logits, 16) && (ld_logits % 8 == 0);
    return cuda_status(launch_argmax(g, s));
}

tf_status tf_gather_rows(void *dst, int ld_dst, const void *const *parts, const int *widths, int nparts, int M,
                         size_t window_bytes, tf_stream stream) {
    if (nparts < 1 || nparts > TF_MAX_PARTS || parts == nullptr || widths == nullptr || M < 0) return TF_E_ARG;
    GatherArgs g;
    std::memset(&g, 0, sizeof g);
    long long total = 0;
    bool broken = false;
    bool vec = aligned(dst, 16) && (ld_dst % 8 == 0);
    for (int h = 0; h < nparts; ++h) {
        if (widths[h] < 0) return TF_E_ARG;
        g.off[h] = (int)total;
        total += widths[h];
        if (total > INT_MAX) return TF_E_ARG;
        g.part[h] = static_cast<const uint16_t *>(parts[h]);
        g.width[h] = widths[h];
        if (!parts[h]) broken = true;
        if (widths[h] % 8 != 0 || (parts[h] && !aligned(parts[h], 16))) vec = false;
        if (parts[h] && !aligned(parts[h], 2)) return TF_E_ALIGN;
    }
    g.off[nparts] = (int)total;
    if (ld_dst < total) return TF_E_ARG;
    for (int h = 0; h < nparts; ++h)
        if (window_bytes != TF_NO_WINDOW && (size_t)M * (size_t)widths[h] * 2u > window_bytes) return TF_E_WINDOW;
    if (M == 0 || total == 0) return broken ? TF_E_BROKEN : TF_OK;
    if (!dst) return TF_E_ARG;
    if (!aligned(dst, 2)) return TF_E_ALIGN;
    g.dst = static_cast<uint16_t *>(dst);
    g.ld_dst = ld_dst;
    g.nparts = nparts;
    g.M = M;
    if (cuda_status(launch_gather(g, vec, reinterpret_cast<cudaStream_t>(stream))) != TF_OK) return TF_E_CUDA;
    return broken ? TF_E_BROKEN : TF_OK;
}

size_t tf_argmax_scratch_bytes(int M, int n) {
    if (M <= 0 || n <= 0) return 0;
    return (size_t)M * (size_t)argmax_blocks_per_row(M, n) * sizeof(uint64_t);
}

tf_status tf_argmax_rows(const void *logits, int M, int n, int ld, uint32_t id_base, uint64_t *words, void *scratch,
                         size_t scratch_bytes, tf_stream stream) {
    if (M < 0 || M > 65535 || n < 1 || ld < n) return TF_E_ARG;
    if ((unsigned long long)id_base + (unsigned long long)n > 0x80000000ull) return TF_E_RANGE;
    if (M == 0) return TF_OK;
    if (!logits || !words || !scratch) return TF_E_ARG;
    if (scratch_bytes < tf_argmax_scratch_bytes(M, n)) return TF_E_ARG;
    if (!aligned(logits, 2) || !aligned(words, 8) || !aligned(scratch, 8)) return TF_E_ALIGN;
    ArgmaxArgs a;
    std::memset(&a, 0, sizeof a);
    a.logits = static_cast<const uint16_t *>(logits);
    a.ld = ld;
    a.n = n;
    a.id_base = id_base;
    a.M = M;
    a.partial = static_cast<uint64_t *>(scratch);
    a.words = words;
    a.vec = aligned(logits, 16) && (ld % 8 == 0);
    return cuda_status(launch_argmax(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t tf_top2_scratch_bytes(int M, int n) {
    if (M <= 0 || n <= 0) return 0;
    return (size_t)M * (size_t)argmax_blocks_per_row(M, n) * 2 * sizeof(uint64_t);
}

tf_status tf_top2_rows(const void *logits, int M, int n, int ld, uint32_t id_base, uint64_t *words2, void *scratch,
                       size_t scratch_bytes, tf_stream stream) {
    if (M < 0 || M > 65535 || n < 1 || ld < n) return TF_E_ARG;
    if ((unsigned long long)id_base + (unsigned long long)n > 0x80000000ull) return TF_E_RANGE;
    if (M == 0) return TF_OK;
    if (!logits || !words2 || !scratch) return TF_E_ARG;
    if (scratch_bytes < tf_top2_scratch_bytes(M, n)) return TF_E_ARG;
    if (!aligned(logits, 2) || !aligned(words2, 8) || !aligned(scratch, 8)) return TF_E_ALIGN;
    ArgmaxArgs a;
    std::memset(&a, 0, sizeof a);
    a.logits = static_cast<const uint16_t *>(logits);
    a.ld = ld;
    a.n = n;
    a.id_base = id_base;
    a.M = M;
    a.partial = static_cast<uint64_t *>(scratch);
    a.words = words2;
    a.vec = aligned(logits, 16) && (ld % 8 == 0);
    return cuda_status(launch_top2(a, reinterpret_cast<cudaStream_t>(stream)));
}

tf_status tf_top2_merge(const uint64_t *words2, int nparts, int M, uint64_t *out2, tf_stream stream) {
    if (nparts < 1 || nparts > TF_MAX_PARTS || M < 0 || M > 65535) return TF_E_ARG;
    if (M == 0) return TF_OK;
    if (!words2 || !out2) return TF_E_ARG;
    if (!aligned(words2, 8) || !aligned(out2, 8)) return TF_E_ALIGN;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(words2), a1 = a0 + (size_t)nparts * M * 16;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(out2), b1 = b0 + (size_t)M * 16;
    if (a0 < b1 && b0 < a1) return TF_E_ARG;   // out2 must not overlap the inputs
    return cuda_status(launch_top2_merge(words2, nparts, M, out2, reinterpret_cast<cudaStream_t>(stream)));
}

tf_status tf_residual_add(float *h, int ld_h, const void *y, int ld_y, int M, int n, tf_stream stream) {
    if (M < 0 || n < 0 || ld_h < n || ld_y < n) return TF_E_ARG;
    if (M == 0 || n == 0) return TF_OK;
    if (!h || !y) return TF_E_ARG;
    if (!aligned(h, 4) || !aligned(y, 2)) return TF_E_ALIGN;
    const bool vec = aligned(h, 16) && ld_h % 4 == 0 && aligned(y, 16) && ld_y % 8 == 0;
    return cuda_status(launch_residual_add(h, ld_h, static_cast<const uint16_t *>(y), ld_y, M, n, vec,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

tf_status tf_embed_rows(const void *table, int rows, int H, int ld_table, int bound, const uint32_t *ids, int M,
                        void *out, int ld_out, tf_stream stream) {
    if (rows < 1 || H < 0 || ld_table < H || ld_out < H || M < 0) return TF_E_ARG;
    if (bound != rows) return TF_E_RANGE;   // below: the shard-width bound; above: past the table
    if (M == 0 || H == 0) return TF_OK;
    if (!table || !ids || !out) return TF_E_ARG;
    if (!aligned(table, 2) || !aligned(out, 2) || !aligned(ids, 4)) return TF_E_ALIGN;
    const bool vec = aligned(table, 16) && ld_table % 8 == 0 && aligned(out, 16) && ld_out % 8 == 0;
    return cuda_status(launch_embed_rows(static_cast<const uint16_t *>(table), ld_table, (uint32_t)bound, H, ids, M,
                                         static_cast<uint16_t *>(out), ld_out, vec,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

tf_status tf_pick(const uint64_t *words, int nparts, int M, uint32_t *ids, tf_stream stream) {
    if (nparts < 1 || nparts > TF_MAX_PARTS || M < 0 || M > 65535) return TF_E_ARG;
    if (M == 0) return TF_OK;
    if (!words || !ids) return TF_E_ARG;
    if (!aligned(words, 8) || !aligned(ids, 4)) return TF_E_ALIGN;
    return cuda_status(launch_pick(words, nparts, M, ids, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
