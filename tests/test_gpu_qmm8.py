"""The int8 head (tf_qmm8_rows): int8 codes with one bf16 scale per row, the b70
lab's runtime INT8 target LM-head.  Values within the V tolerance of the fp64
oracle, the row split bit-identical to the whole matrix on both kernels (the
M = 1 stream and the general one), ragged K and an unaligned code array, and
the full 124,160-row half of the head with its argmax against the oracle's scan
of the GPU's own logits.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def q8dev(w):
    return synth.weights8_to_device(w)


def run(tf, x, q8, sc, segs, ncols):
    y = empty_bf16(x.shape[0], ncols)
    tf.tf_qmm8_rows(x, q8, sc, segs, y)
    return y


@pytest.mark.parametrize("M,K", [(1, 1024), (3, 1024), (1, 1056), (2, 1000), (1, 5120)])
def test_qmm8_values_and_split(tf, orc, M, K):
    N = 512
    w = synth.make_weights8(N, K, seed=K + M)
    q8, sc = q8dev(w)
    xb = synth.make_x(M, K, seed=K)
    x = dev(xb)
    whole = run(tf, x, q8, sc, [(0, N)], N)
    halves = [run(tf, x, q8, sc, [tf.tf_split_rows(N, 2, h)], N // 2) for h in range(2)]
    torch.cuda.synchronize()
    assert bits_equal(torch.cat(halves, dim=1), whole)
    yo, y64, ad = orc.qmm8_rows(xb, w.q8, w.scales, np.arange(N), want_f64=True)
    check_values(host_bits(whole), yo, y64, ad, K, f"int8 head M={M} K={K}")


def test_qmm8_unaligned_codes_take_the_general_kernel(tf, orc):
    N, K = 64, 1024
    w = synth.make_weights8(N, K, seed=3)
    buf = torch.zeros(N * K + 16, dtype=torch.int8, device="cuda")
    q8 = buf[1:1 + N * K].view(N, K)                 # 1-byte offset: no bulk copies
    q8.copy_(torch.from_numpy(w.q8).cuda())
    sc = dev(w.scales)
    xb = synth.make_x(1, K, seed=3)
    y = run(tf, dev(xb), q8, sc, [(0, N)], N)
    torch.cuda.synchronize()
    yo, y64, ad = orc.qmm8_rows(xb, w.q8, w.scales, np.arange(N), want_f64=True)
    check_values(host_bits(y), yo, y64, ad, K, "int8 head, unaligned codes")


def test_qmm8_lm_head_half_full_size(tf, orc):
    rows, K = synth.VOCAB // 2, synth.HIDDEN
    w = synth.make_weights8(rows, K, seed=9)
    q8, sc = q8dev(w)
    xb = synth.make_x(1, K, seed=9, tag=5)
    y = run(tf, dev(xb), q8, sc, [(0, rows)], rows)
    words = torch.empty(1, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_argmax_scratch_bytes(1, rows), dtype=torch.uint8, device="cuda")
    tf.tf_argmax_rows(y, rows, words, scratch)       # this half's ids start at 124,160
    torch.cuda.synchronize()
    yo, y64, ad = orc.qmm8_rows(xb, w.q8, w.scales, np.arange(rows), nthreads=8, want_f64=True)
    check_values(host_bits(y), yo, y64, ad, K, "int8 lm_head half")
    assert np.array_equal(host_bits(words), orc.argmax_rows(host_bits(y), rows))
