// tf_kernels.h -- launch arguments and host launchers shared by the
// translation units of libtf.so (internal; the public ABI is include/tf.h).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tf.h"

namespace tf {

// Output columns of one qmm call: segment i covers columns [col0[i], col0[i] + nrows[i])
// and whole-matrix rows [row0[i], row0[i] + nrows[i]).
struct SegTable {
    int row0[TF_MAX_SEGS];
    int nrows[TF_MAX_SEGS];
    int col0[TF_MAX_SEGS];
    int nseg;
    int ncols;   // sum of nrows (TF_EPI_NONE) or the common nrows (TF_EPI_GLU)
};

struct QmmArgs {
    const uint16_t *x;
    int M, K, ldx;
    const uint8_t *wq;
    const uint16_t *scales;
    const uint16_t *biases;
    SegTable seg;
    int glu;
    uint16_t *y;
    int ldy;
    int n_whole;   // rows of the whole matrix (the call may cover only some of them)
    // fused head (M = 1 stream kernel only): when cand is set, every warp of the grid
    // writes the largest argmax key of the rows it wrote (ids id_base + column) to
    // cand[warp of the grid] (0 when it wrote none); launch_argmax_keys reduces them
    uint64_t *cand;
    uint32_t id_base;
};

// The int8 head: codes [N][K] int8, one bf16 scale per row.
struct Qmm8Args {
    const uint16_t *x;
    int M, K, ldx;
    const int8_t *q8;
    const uint16_t *scales;
    SegTable seg;
    uint16_t *y;
    int ldy;
};

struct GatherArgs {
    uint16_t *dst;
    long long ld_dst;
    const uint16_t *part[TF_MAX_PARTS];
    int width[TF_MAX_PARTS];
    int off[TF_MAX_PARTS + 1];
    int nparts;
    int M;
};

struct ArgmaxArgs {
    const uint16_t *logits;
    long long ld;
    int n;
    uint32_t id_base;
    int M;
    int blocks_per_row;
    int span;              // elements per block (multiple of 8)
    uint64_t *partial;     // [M][blocks_per_row] keys
    uint64_t *words;       // [M]
    int vec;               // 16-byte loads allowed
};

// top two: ArgmaxArgs with partial [M][blocks_per_row][2] and words [M][2]
cudaError_t launch_top2(ArgmaxArgs a, cudaStream_t stream);
cudaError_t launch_top2_merge(const uint64_t *words2, int nparts, int M, uint64_t *out2, cudaStream_t stream);
cudaError_t launch_qmm(const QmmArgs &a, cudaStream_t stream);
cudaError_t launch_qmm8(const Qmm8Args &a, cudaStream_t stream);
cudaError_t launch_gather(const GatherArgs &a, bool vec, cudaStream_t stream);
cudaError_t launch_argmax(ArgmaxArgs a, cudaStream_t stream);
cudaError_t launch_pick(const uint64_t *words, int nparts, int M, uint32_t *ids, cudaStream_t stream);
bool qmm_m1_stream_eligible(const QmmArgs &a);
bool qmm_tc_eligible(const QmmArgs &a);
cudaError_t launch_qmm_tc(const QmmArgs &a, cudaStream_t stream);
// *ncand (when not null) receives the number of warp keys the launch writes to a.cand
cudaError_t launch_qmm_m1_stream(const QmmArgs &a, cudaStream_t stream, int *ncand = nullptr);
cudaError_t launch_argmax_keys(const uint64_t *cand, int ncand, const uint16_t *logits, uint32_t id_base, uint64_t *word,
                               cudaStream_t stream);
int qmm_m1_stream_max_cand();   // an upper bound of the warps of any stream launch

int argmax_blocks_per_row(int M, int n);
cudaError_t launch_residual_add(float *h, long long ld_h, const uint16_t *y, long long ld_y, int M, int n, bool vec,
                                cudaStream_t stream);
cudaError_t launch_embed_rows(const uint16_t *table, long long ld_table, uint32_t bound, int H, const uint32_t *ids,
                              int M, uint16_t *out, long long ld_out, bool vec, cudaStream_t stream);
// TF_OK for cudaSuccess; otherwise remembers e for tf_last_cuda_error and returns TF_E_CUDA.
tf_status cuda_status(cudaError_t e);
cudaError_t last_cuda_error();
int num_sms();

}  // namespace tf
