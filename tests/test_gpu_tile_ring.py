"""The M = 1 tile ring at the edges of its shapes: a ragged last 1,024-K chunk,
several segments and a partial last tile (16-row tiles), a ragged last slot of
4-row x 4,096-K tiles, and a GLU call whose column count is not a multiple of
the 8-column tile.  Each case is checked against the oracle on sampled columns
(V) and bit for bit against the same rows asked another way (S) -- including
calls small enough to take the per-warp ring, so the two kernels must agree on
every bit of a row."""
import os

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu
NT = os.cpu_count() or 1
SAMPLE = 160


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def qmm(tf, xt, W, segs, epi=0):
    ncols = segs[0][1] if epi else sum(n for _, n in segs)
    y = empty_bf16(1, ncols)
    tf.tf_qmm_rows(xt, *W.t(), segs, y, epi=epi)
    return y


def sampled(orc, x, w, y_bits, rows, K, what, seed=0):
    rng = np.random.default_rng(seed)
    pick = np.sort(rng.choice(len(rows), min(SAMPLE, len(rows)), replace=False))
    pick = np.unique(np.concatenate([pick, [0, len(rows) - 1]]))   # both ends of the call
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), np.asarray(rows)[pick], nthreads=NT, want_f64=True)
    return check_values(y_bits[:, pick], yo, y64, ad, K, what)


def columns_of(segs):
    return np.concatenate([np.arange(r0, r0 + n) for r0, n in segs])


@pytest.mark.parametrize("K,N,seg_sets", [
    # 16-row tiles; K = 5.5 chunks: the last chunk is half empty
    (5632, 9600, [[(0, 3000), (3000, 6600)], [(6000, 3600), (0, 2999), (2999, 3001)]]),
    # 4-row x 4,096-K tiles; K = 17.5 chunks: the last slot holds one and a half chunks;
    # N = 1,203 leaves a partial last tile; a half alone is narrow enough for the per-warp ring
    (17920, 1203, [[(0, 601), (601, 602)], [(1000, 203), (0, 1000)], [(0, 601)], [(601, 602)]]),
])
def test_tile_ring_ragged_and_segments(tf, orc, K, N, seg_sets):
    w = synth.make_weights(N, K, seed=K % 97, tag=synth.TAG_W2)
    W = DevWeights(w)
    x = synth.make_x(1, K, seed=N)
    xt = dev(x)
    whole = qmm(tf, xt, W, [(0, N)])
    torch.cuda.synchronize()
    sampled(orc, x, w, host_bits(whole), np.arange(N), K, f"K={K} N={N} whole")
    for segs in seg_sets:
        y = qmm(tf, xt, W, segs)
        cols = columns_of(segs)
        torch.cuda.synchronize()
        assert bits_equal(y, whole[:, torch.as_tensor(cols, device="cuda")]), segs
        sampled(orc, x, w, host_bits(y), cols, K, f"K={K} N={N} segs={segs}", seed=1)


def test_tile_ring_glu_odd_columns(tf, orc):
    """F = 4,740 GLU columns: 593 tiles of 8 columns (the last one holding 4), at
    K = 5,120; the member-split halves (2,370 columns) take the per-warp ring."""
    F, K = 4740, 5120
    w = synth.make_weights(2 * F, K, seed=31, tag=synth.TAG_W)
    W = DevWeights(w)
    x = synth.make_x(1, K, seed=31)
    xt = dev(x)
    whole = qmm(tf, xt, W, [(0, F), (F, F)], epi=tf.TF_EPI_GLU)
    parts = [qmm(tf, xt, W, tf.tf_member_segs(F, 2, h), epi=tf.TF_EPI_GLU) for h in range(2)]
    joined = empty_bf16(1, F)
    tf.tf_gather_rows(joined, parts, [F // 2, F // 2])
    g = qmm(tf, xt, W, [(0, F)])
    u = qmm(tf, xt, W, [(F, F)])
    torch.cuda.synchronize()
    assert bits_equal(joined, whole), "GLU: member halves != whole"
    check_values(host_bits(whole), orc.glu(host_bits(g), host_bits(u)), what="GLU stage, tile ring")
    sampled(orc, x, w, host_bits(g), np.arange(F), K, "gate rows")
    sampled(orc, x, w, host_bits(u), np.arange(F, 2 * F), K, "up rows", seed=2)


def test_long_k_routes_agree(tf, orc):
    """K = 17,408 (17 chunks: slices of 4, 4, 4, 4 and 1 chunks).  The whole
    9,600-row matrix runs on the 16-row tile ring, which folds each slice's tree
    sum into the row inside the warp; a 2,560-row slice and a short one run on the
    narrow-call kernel, whose warps share the (row, slice) pairs and add the
    slice sums afterwards; a GLU call over 4,800 columns takes the tile ring and
    a 100-column one the per-warp ring.  Every route must give the same bits for
    the same row, and values within the V bar of the oracle."""
    N, K = 9600, 17408
    w = synth.make_weights(N, K, seed=41, tag=synth.TAG_W2)
    W = DevWeights(w)
    x = synth.make_x(1, K, seed=41)
    xt = dev(x)
    whole = qmm(tf, xt, W, [(0, N)])
    torch.cuda.synchronize()
    sampled(orc, x, w, host_bits(whole), np.arange(N), K, "K=17,408 whole (tile ring)")
    for segs in ([(0, 2560)], [(7040, 2560)], [(5000, 37), (100, 3)]):
        y = qmm(tf, xt, W, segs)
        cols = columns_of(segs)
        torch.cuda.synchronize()
        assert bits_equal(y, whole[:, torch.as_tensor(cols, device="cuda")]), segs
    F = N // 2
    glu_whole = qmm(tf, xt, W, [(0, F), (F, F)], epi=tf.TF_EPI_GLU)
    glu_small = qmm(tf, xt, W, [(200, 100), (F + 200, 100)], epi=tf.TF_EPI_GLU)
    torch.cuda.synchronize()
    assert bits_equal(glu_small, glu_whole[:, 200:300])
    check_values(host_bits(glu_whole), orc.glu(host_bits(whole)[:, :F], host_bits(whole)[:, F:]),
                 what="GLU stage at K = 17,408")


@pytest.mark.parametrize("M", [2, 3])
@pytest.mark.parametrize("shape", ["head", "glu", "narrow", "long_k"])
def test_few_rows_equal_one_row_calls(tf, orc, M, shape):
    """Two or three activation rows on the streaming kernels: every row's outputs
    are bit for bit those of a call with that row alone, and within the V bar of
    the oracle on sampled columns.  Shapes: 12,000 rows at K = 5,120 (the tile
    ring's 16-row or 8-row tiles), a GLU call over 4,800 columns, 2,560 rows at
    K = 5,120 (4-row x 4,096-K tiles) and 2,560 rows at K = 17,408 (the narrow-call
    kernel for two rows, the tensor cores for three)."""
    K, N, segs, epi = {
        "head": (5120, 12000, [(0, 12000)], 0),
        "glu": (5120, 9600, [(0, 4800), (4800, 4800)], 1),
        "narrow": (5120, 2560, [(0, 2560)], 0),
        "long_k": (17408, 2560, [(0, 2560)], 0),
    }[shape]
    w = synth.make_weights(N, K, seed=50 + M, tag=synth.TAG_W2)
    W = DevWeights(w)
    x = synth.make_x(M, K, seed=60 + M)
    xt = dev(x)
    ncols = segs[0][1] if epi else sum(n for _, n in segs)
    y = empty_bf16(M, ncols)
    tf.tf_qmm_rows(xt, *W.t(), segs, y, epi=epi)
    ones = []
    for m in range(M):
        o = empty_bf16(1, ncols)
        tf.tf_qmm_rows(xt[m:m + 1], *W.t(), segs, o, epi=epi)
        ones.append(o)
    torch.cuda.synchronize()
    if not (shape == "long_k" and M > 2):   # three long-K rows run on the tensor cores
        assert bits_equal(y, torch.cat(ones)), (shape, M)
    if epi:
        g = empty_bf16(M, ncols)
        u = empty_bf16(M, ncols)
        tf.tf_qmm_rows(xt, *W.t(), [segs[0]], g)
        tf.tf_qmm_rows(xt, *W.t(), [segs[1]], u)
        torch.cuda.synchronize()
        check_values(host_bits(y), orc.glu(host_bits(g), host_bits(u)), what=f"GLU M={M}")
        sampled(orc, x, w, host_bits(g), np.arange(segs[0][0], segs[0][0] + ncols), K, f"gate M={M}")
    else:
        sampled(orc, x, w, host_bits(y), columns_of(segs), K, f"{shape} M={M}")


@pytest.mark.parametrize("M", [1, 2])
def test_narrow_call_many_columns(tf, orc, M):
    """The narrow-call kernel with many (row, slice) pairs per warp: K = 17,920
    (17.5 chunks, slices of 4, 4, 4, 4 and 1.5 chunks) over 4,000 columns from
    three segments, so each CTA's ~27 columns give its warps more pairs than ring
    slots, and a CTA's run of rows can cross a segment boundary.  Every column is
    checked against the oracle, and bit for bit against the same rows on the
    16-row tile ring (the whole 6,000-row matrix) and, for two activation rows,
    against one-row calls."""
    K, N = 17920, 6000
    segs = [(0, 1500), (4000, 1500), (2000, 1000)]
    w = synth.make_weights(N, K, seed=70 + M, tag=synth.TAG_W2)
    W = DevWeights(w)
    x = synth.make_x(M, K, seed=80 + M)
    xt = dev(x)
    cols = columns_of(segs)
    y = empty_bf16(M, len(cols))
    tf.tf_qmm_rows(xt, *W.t(), segs, y)
    whole = empty_bf16(M, N) if M == 1 else None
    if M == 1:
        tf.tf_qmm_rows(xt, *W.t(), [(0, N)], whole)
    ones = []
    for m in range(M if M > 1 else 0):
        o = empty_bf16(1, len(cols))
        tf.tf_qmm_rows(xt[m:m + 1], *W.t(), segs, o)
        ones.append(o)
    torch.cuda.synchronize()
    if M == 1:
        assert bits_equal(y, whole[:, torch.as_tensor(cols, device="cuda")]), "narrow call != tile ring"
    for m, o in enumerate(ones):
        assert bits_equal(y[m:m + 1], o), f"activation row {m}: two-row call != one-row call"
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), cols, nthreads=NT, want_f64=True)
    check_values(host_bits(y), yo, y64, ad, K, f"narrow call M={M}")
