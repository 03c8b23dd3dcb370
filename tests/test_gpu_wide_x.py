"""Activations with a wide dynamic range, against the oracle.

Every 32-value run of x (32 consecutive k from a multiple of 32) holds one
value of magnitude 2^10 and 31 small ones; the weights at the large values'
columns are exactly zero in every row (code 8 and bias -8 * scale), so each
output is built from the small values alone.  The method reduces every row in
fp32 over the full K (TensorFold PR #1433, step-1 body), so the outputs must
meet the same value bar as on natural inputs: within 2 bf16 ulps of the fp64
oracle, with no output accepted through the cancellation floor.  (With the
natural weights the large products themselves can cancel, as in any fp32 dot,
so there the floor -- the fp32 accumulation bound -- is allowed and reported;
on the tensor cores the offset7 terms are not separated, see floor_allowed.)

Variants:
  zero     small values 2^-14 .. 2^-10 (a 2^20 .. 2^24 span within a run),
           zero weights at the large values;
  natural  the same x with the natural weights (the large values dominate);
  window   small values 2^-5 .. 2^-4 (within 2^15 of the large value),
           zero weights: the large value's product cancels to exactly zero;
  offset7  as window, but the zero weights are code 7 with bias -7 * scale, so
           any split of w into a code part and a bias part leaves two large
           terms that cancel;
  pair     as zero, with a second outlier of 2^9 (also of weight zero) in every
           run: two dominating values.
Each runs through every route of tf_qmm_rows: the M = 1 tile ring (with and
without the fused GLU), the narrow-call kernel, the per-warp ring, the fp32 M = 1
kernel (K not a multiple of 512), three rows on the streaming kernels, the
tensor-core kernel (M >= 5) and the general kernel; and through tf_qmm8_rows.
"""
import os

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu
NT = os.cpu_count() or 1

VARIANTS = {   # name: (small exponent range, code of the zero weights or None for natural weights)
    "zero": ((-14, -10), 8),
    "natural": ((-14, -10), None),
    "window": ((-5, -4), 8),
    "offset7": ((-5, -4), 7),
    "pair": ((-14, -10), 8),
}

# name: (M, K, whole rows, segments, epilogue) -- the route each one takes is in its comment
ROUTES = {
    "tile16": (1, 5120, 9600, [(0, 9600)], 0),                 # tile ring, 600 16-row tiles
    "split": (1, 17408, 2560, [(0, 2560)], 0),                 # narrow-call kernel, (row, K-slice) pairs
    "tile_glu": (1, 5120, 9600, [(0, 4800), (4800, 4800)], 1),  # tile ring, 8-column GLU tiles
    "warp": (1, 5120, 512, [(0, 512)], 0),                     # per-warp ring
    "warp_glu": (1, 5120, 512, [(0, 256), (256, 256)], 1),     # per-warp ring, GLU
    "m1_fp32": (1, 1088, 512, [(0, 512)], 0),                  # K % 512 != 0: the fp32 M = 1 kernel
    "rows3": (3, 5120, 512, [(0, 512)], 0),                    # three rows on the streaming kernels
    "tc": (8, 5120, 512, [(0, 512)], 0),                       # tensor cores
    "tc_glu": (16, 5120, 512, [(0, 256), (256, 256)], 1),      # tensor cores, GLU
    "generic": (3, 1088, 512, [(0, 512)], 0),                  # K % 512 != 0, M > 1: general kernel
}


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def inputs(variant, M, K, N, seed):
    small, code = VARIANTS[variant]
    pos = synth.wide_positions(K, seed)
    x = synth.make_x_wide(M, K, small_exp=small, seed=seed, positions=pos)
    if variant == "pair":   # a second outlier, 2^9, one place after the first within its run
        pos2 = (pos // 32) * 32 + (pos % 32 + 1) % 32
        x2 = synth.make_x_wide(M, K, big_exp=9, small_exp=small, seed=seed + 1, positions=pos2)
        x[:, pos2] = x2[:, pos2]
        pos = np.concatenate([pos, pos2])
    w = synth.make_weights(N, K, seed=seed, tag=synth.TAG_W2)
    if code is not None:
        w = synth.with_zero_weights(w, pos, offset=code)
    return x, w


def floor_allowed(route, variant):
    """Where an output may pass on the fp32 accumulation bound instead of the
    2-ulp bar: natural weights (large products that cancel among themselves, as
    in any fp32 dot), and the tensor-core path on offset7 (it forms the code and
    bias terms of a 64-value group separately, so a zero weight whose code is
    not 8 leaves two large terms that cancel; the streaming kernels take such a
    run, a lone outlier, as a plain fp32 dot)."""
    return variant == "natural" or (variant == "offset7" and route.startswith("tc"))


def qmm(tf, xt, W, segs, epi, M):
    ncols = segs[0][1] if epi else sum(n for _, n in segs)
    y = empty_bf16(M, ncols)
    tf.tf_qmm_rows(xt, *W.t(), segs, y, epi=epi)
    return y


@pytest.mark.parametrize("variant", sorted(VARIANTS))
@pytest.mark.parametrize("route", list(ROUTES))
def test_wide_range_x(tf, orc, route, variant):
    M, K, N, segs, epi = ROUTES[route]
    x, w = inputs(variant, M, K, N, seed=K % 101 + M)
    W = DevWeights(w)
    xt = dev(x)
    y = qmm(tf, xt, W, segs, epi, M)
    if epi:
        g = qmm(tf, xt, W, [segs[0]], 0, M)
        u = qmm(tf, xt, W, [segs[1]], 0, M)
    torch.cuda.synchronize()
    if epi:
        stats = []
        for t, (r0, n) in ((g, segs[0]), (u, segs[1])):
            yo, y64, ad = orc.qmm_rows(x, *w.astuple(), np.arange(r0, r0 + n), nthreads=NT, want_f64=True)
            st = check_values(host_bits(t), yo, y64, ad, K, f"{route}/{variant} gate-up rows")
            assert st["floor_used"] == 0 or floor_allowed(route, variant), st
            stats.append(st)
        st = check_values(host_bits(y), orc.glu(host_bits(g), host_bits(u)), what=f"{route}/{variant} GLU")
        stats.append(st)
    else:
        rows = np.concatenate([np.arange(r0, r0 + n) for r0, n in segs])
        yo, y64, ad = orc.qmm_rows(x, *w.astuple(), rows, nthreads=NT, want_f64=True)
        st = check_values(host_bits(y), yo, y64, ad, K, f"{route}/{variant}")
        assert st["floor_used"] == 0 or floor_allowed(route, variant), st
        stats = [st]
    print(f"\n{route}/{variant}: {stats}")


@pytest.mark.parametrize("variant", ["zero", "window"])
def test_wide_range_split_equals_whole(tf, variant):
    """The two row halves of the tile-ring layer, each a call of its own, are the
    whole call's rows bit for bit."""
    M, K, N, _, _ = ROUTES["tile16"]
    x, w = inputs(variant, M, K, N, seed=3)
    W = DevWeights(w)
    xt = dev(x)
    whole = qmm(tf, xt, W, [(0, N)], 0, M)
    halves = [qmm(tf, xt, W, [tf.tf_split_rows(N, 2, h)], 0, M) for h in range(2)]
    torch.cuda.synchronize()
    assert bits_equal(torch.cat(halves, dim=1), whole)


@pytest.mark.parametrize("variant", ["zero", "natural"])
@pytest.mark.parametrize("M,K", [(1, 5120), (3, 1024)])
def test_wide_range_x_int8(tf, orc, variant, M, K):
    N = 512
    pos = synth.wide_positions(K, seed=K)
    x = synth.make_x_wide(M, K, seed=K, positions=pos)
    w = synth.make_weights8(N, K, seed=K)
    if variant == "zero":
        w = synth.with_zero_weights8(w, pos)
    q8, sc = synth.weights8_to_device(w)
    y = empty_bf16(M, N)
    tf.tf_qmm8_rows(dev(x), q8, sc, [(0, N)], y)
    torch.cuda.synchronize()
    yo, y64, ad = orc.qmm8_rows(x, *w.astuple(), np.arange(N), nthreads=NT, want_f64=True)
    st = check_values(host_bits(y), yo, y64, ad, K, f"int8 M={M} K={K}/{variant}")
    assert st["floor_used"] == 0 or variant == "natural", st
    print(f"\nint8 M={M} K={K} {variant}: {st}")
