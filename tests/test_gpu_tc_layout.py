"""Tensor-core qmm at row counts that are not multiples of the MMA's N, with
activation rows padded in memory.

The kernel copies four 64-value groups of activations at a time as one 3-D tile
(the activation rows' leading dimension is a stride of the copy, rows past M read
as zero) and the codes four groups wide; these cases check that both copies land
where the MMA and the decoders read them: M from 4 to 128 (N = 16, 32, 64 and 128),
a ragged last 128-row tile, rows padded to ldx = K + 64 (bits equal to the
unpadded call), the fused gate*SiLU(up) epilogue, and more tiles than resident
CTAs with one K slice (persistent CTAs walking several tiles), each against the oracle
(TensorFold PR #1433, step-1 body: each rank reduces its rows over the full K in
fp32; step-2 body: the GLU of the gate and up halves).
"""
import os

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu
NT = os.cpu_count() or 1


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def qmm(tf, xt, W, segs, epi=0):
    ncols = segs[0][1] if epi else sum(n for _, n in segs)
    y = empty_bf16(xt.shape[0], ncols)
    tf.tf_qmm_rows(xt, *W.t(), segs, y, epi=epi)
    return y


def padded(xt, extra=64):
    """The same rows in a buffer whose leading dimension is K + extra."""
    M, K = xt.shape
    buf = torch.zeros(M, K + extra, dtype=torch.bfloat16, device=xt.device)
    buf[:, :K] = xt
    return buf[:, :K]


@pytest.mark.parametrize("M", [4, 5, 13, 17, 33, 100, 128])
def test_tc_odd_rows_padded(tf, orc, M):
    K, N = 2048, 300   # three 128-row tiles, the last one of 44 rows
    w = synth.make_weights(N, K, seed=M)
    W = DevWeights(w)
    x = synth.make_x(M, K, seed=M)
    xt = dev(x)
    xp = padded(xt)
    assert xp.stride(0) == K + 64
    y = qmm(tf, xt, W, [(0, N)])
    yp = qmm(tf, xp, W, [(0, N)])
    torch.cuda.synchronize()
    assert bits_equal(y, yp), "a padded leading dimension changed the bits"
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), np.arange(N), nthreads=NT, want_f64=True)
    check_values(host_bits(y), yo, y64, ad, K, f"tensor cores M={M}")


@pytest.mark.parametrize("M", [6, 40])
def test_tc_glu_odd_rows(tf, orc, M):
    K, F = 1024, 200   # gate rows 0..199, up rows 200..399: two 64-column tiles, the last of 8
    w = synth.make_weights(2 * F, K, seed=100 + M)
    W = DevWeights(w)
    x = synth.make_x(M, K, seed=100 + M)
    xt = padded(dev(x))
    act = qmm(tf, xt, W, [(0, F), (F, F)], epi=tf.TF_EPI_GLU)
    g = qmm(tf, xt, W, [(0, F)])
    u = qmm(tf, xt, W, [(F, F)])
    torch.cuda.synchronize()
    for t, r0 in ((g, 0), (u, F)):
        yo, y64, ad = orc.qmm_rows(x, *w.astuple(), np.arange(r0, r0 + F), nthreads=NT, want_f64=True)
        check_values(host_bits(t), yo, y64, ad, K, f"tensor cores M={M} rows {r0}..")
    check_values(host_bits(act), orc.glu(host_bits(g), host_bits(u)), what=f"tensor cores M={M} GLU")


@pytest.mark.parametrize("M", [16, 33, 64, 128])
def test_tc_persistent_tiles(tf, orc, M):
    """More 128-row tiles than resident CTAs, with the K range in one slice: each
    CTA walks several tiles (every gridDim-th), its copy ring, tensor-memory
    stages and barrier phases running on across them (MMA widths 16, 64 and 128,
    the last with narrower tensor-memory loads).  Two segments with ragged ends
    put tile starts off the 128-row grid of the whole matrix."""
    K = 512
    segs = [(0, 20000), (25000, 19000)]   # 157 + 149 tiles, both segments end in a partial tile
    N = 44000
    w = synth.make_weights(N, K, seed=200 + M)
    W = DevWeights(w)
    x = synth.make_x(M, K, seed=200 + M)
    xt = padded(dev(x))
    y = host_bits(qmm(tf, xt, W, segs))
    torch.cuda.synchronize()
    cols = np.arange(sum(n for _, n in segs))
    whole = np.concatenate([np.arange(r0, r0 + n) for r0, n in segs])
    pick = np.unique(np.concatenate([cols[::5], cols[-300:], cols[19800:20200]]))   # every fifth, both tails
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), whole[pick], nthreads=NT, want_f64=True)
    check_values(y[:, pick], yo, y64, ad, K, f"tensor cores M={M}, persistent")
