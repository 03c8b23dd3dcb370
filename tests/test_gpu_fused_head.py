"""tf_qmm_argmax_rows, the fused head: one rank's logits and their argmax word in
one call (TensorFold PR #1433 step-1 body: each rank computes its half of the
lm_head, then pair_argmax over it).

At M = 1 the qmm warps keep the best argmax key of the rows they write and a
one-CTA kernel combines the keys into the word.  The contract is bit-for-bit equality with
the two separate calls (tf_qmm_rows, then tf_argmax_rows on its logits), which
these tests check on natural weights, on weights that make an exact tie across
the halves, a NaN row and an overflowing row, at full lm_head-half size, and
for M > 1 (where the call runs the two kernels one after the other).  The
picked id of the two fused halves must equal the pick over the whole
vocabulary, and the words must equal the oracle's scan of the GPU's logits.
"""
import os

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def unfused(tf, x, W, seg, id_base):
    M = x.shape[0]
    lg = empty_bf16(M, seg[1])
    tf.tf_qmm_rows(x, *W.t(), [seg], lg)
    w = torch.empty(M, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_argmax_scratch_bytes(M, seg[1]), dtype=torch.uint8, device="cuda")
    tf.tf_argmax_rows(lg, id_base, w, scratch)
    return lg, w


def fused(tf, x, W, seg, id_base):
    M = x.shape[0]
    lg = empty_bf16(M, seg[1])
    w = torch.full((M,), -1, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_qmm_argmax_scratch_bytes(M, seg[1]), dtype=torch.uint8, device="cuda")
    tf.tf_qmm_argmax_rows(x, *W.t(), seg, id_base, lg, w, scratch)
    return lg, w


def pick(tf, words):
    ids = torch.empty(words.shape[1], dtype=torch.int32, device="cuda")
    tf.tf_pick(words.contiguous(), ids)
    return host_bits(ids)


def variant(w: synth.QWeights, kind: str, x_bits: np.ndarray) -> synth.QWeights:
    """Weights of the tiny head changed so that the head meets the case."""
    wq, sc, bi = (a.copy() for a in w.astuple())
    V = w.N
    if kind == "tie":
        # copy the row with the largest logit into a row of the other half
        xf = synth.bf16_bits_to_f32(x_bits[0]).astype(np.float64)
        q = np.empty((V, w.K), dtype=np.float64)
        q[:, 0::2] = wq & 0x0F
        q[:, 1::2] = wq >> 4
        s = np.repeat(synth.bf16_bits_to_f32(sc).astype(np.float64), 64, axis=1)
        b = np.repeat(synth.bf16_bits_to_f32(bi).astype(np.float64), 64, axis=1)
        top = int(np.argmax((s * q + b) @ xf))
        other = top + V // 2 + 5 if top < V // 2 else top - V // 2 + 5
        wq[other], sc[other], bi[other] = wq[top], sc[top], bi[top]
    elif kind == "nan":
        sc[100] = 0x7FC0                      # every group scale NaN: the logit is NaN
    elif kind == "inf":
        sc[V // 2 + 300] = 0x7F7F             # the largest finite bf16: the row overflows
        bi[V // 2 + 300] = 0x7F7F
        wq[V // 2 + 300] = 0xFF
    return synth.QWeights(wq, sc, bi)


@pytest.mark.parametrize("kind", ["natural", "tie", "nan", "inf"])
def test_fused_tiny_head_equals_two_calls(tf, orc, kind):
    V, K = synth.TINY_VOCAB, synth.TINY_HEAD_K
    x_bits = synth.make_x(1, K, seed=11, tag=synth.TAG_X)
    w = variant(synth.make_weights(V, K, seed=11, tag=synth.TAG_HEAD), kind, x_bits)
    W = DevWeights(w)
    x = dev(x_bits)
    words_f = torch.empty(2, 1, dtype=torch.int64, device="cuda")
    for h in range(2):
        seg = tf.tf_split_rows(V, 2, h)
        lu, wu = unfused(tf, x, W, seg, seg[0])
        lf, wf = fused(tf, x, W, seg, seg[0])
        torch.cuda.synchronize()
        assert bits_equal(lf, lu), (kind, h)
        assert torch.equal(wf, wu), (kind, h, hex(int(wf[0]) & (2**64 - 1)), hex(int(wu[0]) & (2**64 - 1)))
        # I-kernel: the oracle's scan of the GPU's own logits
        assert np.array_equal(host_bits(wf), orc.argmax_rows(host_bits(lf), seg[0])), (kind, h)
        words_f[h] = wf
    # the pick of the two fused halves equals the pick over the whole vocabulary
    whole_l, whole_w = unfused(tf, x, W, (0, V), 0)
    assert np.array_equal(pick(tf, words_f), pick(tf, whole_w[None, :]))
    ids = pick(tf, words_f)
    if kind in ("nan", "inf"):
        assert ids[0] == tf.TF_PICK_FAILED
    else:
        assert ids[0] != tf.TF_PICK_FAILED
    if kind == "tie":
        # the two halves' winners are equal values; the lower id wins
        w0, w1 = (int(v) & (2**64 - 1) for v in host_bits(words_f)[:, 0])
        assert (w0 & 0xFFFFFFFF) == (w1 & 0xFFFFFFFF)
        assert ids[0] == min(w0 >> 32, w1 >> 32)


def test_fused_more_rows_equal_two_calls(tf):
    V, K = synth.TINY_VOCAB, synth.TINY_HEAD_K
    W = DevWeights(synth.make_weights(V, K, seed=12, tag=synth.TAG_HEAD))
    x = dev(synth.make_x(3, K, seed=12))
    seg = tf.tf_split_rows(V, 2, 1)
    lu, wu = unfused(tf, x, W, seg, seg[0])
    lf, wf = fused(tf, x, W, seg, seg[0])
    torch.cuda.synchronize()
    assert bits_equal(lf, lu) and torch.equal(wf, wu)


def test_fused_lm_head_half_full_size(tf):
    """The 124,160-row half of the 248,320-row head at K = 5,120 (4-row units)."""
    rows, K = synth.VOCAB // 2, synth.HIDDEN
    W = DevWeights(synth.make_weights(rows, K, seed=13, tag=synth.TAG_HEAD))
    x = dev(synth.make_x(1, K, seed=13, tag=5))
    for id_base in (0, rows):
        lu, wu = unfused(tf, x, W, (0, rows), id_base)
        lf, wf = fused(tf, x, W, (0, rows), id_base)
        torch.cuda.synchronize()
        assert bits_equal(lf, lu)
        assert torch.equal(wf, wu)


@pytest.fixture(scope="module")
def whole_head():
    w = synth.make_weights(synth.VOCAB, synth.HIDDEN, seed=14, tag=synth.TAG_HEAD)
    return w, DevWeights(w)


@pytest.mark.parametrize("kind", ["natural", "tie", "nan", "inf"])
def test_fused_full_head_planted(tf, orc, whole_head, kind):
    """Both 124,160-row halves of the 248,320-row head on the tile ring, with a
    planted exact tie across the halves (the top row copied into the other half),
    a NaN row in half 0 or an overflowing row in half 1: each half's word equals
    the oracle's scan of the GPU's own logits, and the pick of the two words is
    the lower id of the tie, or the sentinel."""
    w, W = whole_head
    V, K = synth.VOCAB, synth.HIDDEN
    h = V // 2
    x = dev(synth.make_x(1, K, seed=14, tag=5))
    saved = []

    def plant(row, wq=None, sc=None, bi=None):
        saved.append((row, W.wq[row].clone(), W.scales[row].clone(), W.biases[row].clone()))
        if wq is not None:
            W.wq[row] = wq
        if sc is not None:
            W.scales[row] = sc
        if bi is not None:
            W.biases[row] = bi

    try:
        expect = None
        if kind == "tie":
            lg, _ = unfused(tf, x, W, (0, V), 0)
            f = lg.float()[0]
            top = int(torch.argmax(torch.where(torch.isfinite(f), f, torch.full_like(f, -float("inf")))))
            other = top + h + 5 if top < h else top - h + 5
            plant(other, W.wq[top].clone(), W.scales[top].clone(), W.biases[top].clone())
            expect = min(top, other)
        elif kind == "nan":   # every group scale NaN (0x7FC0): the logit is NaN
            plant(1234, sc=torch.full_like(W.scales[1234].view(torch.int16), 0x7FC0).view(torch.bfloat16))
        elif kind == "inf":   # codes 15, scale and bias the largest finite bf16 (0x7F7F): the row overflows
            r = h + 4321
            big = torch.full_like(W.scales[r].view(torch.int16), 0x7F7F).view(torch.bfloat16)
            plant(r, wq=torch.full_like(W.wq[r], 0xFF), sc=big, bi=big.clone())
        torch.cuda.synchronize()
        words = torch.empty(2, 1, dtype=torch.int64, device="cuda")
        for p in range(2):
            seg = tf.tf_split_rows(V, 2, p)
            lf, wf = fused(tf, x, W, seg, seg[0])
            torch.cuda.synchronize()
            assert np.array_equal(host_bits(wf), orc.argmax_rows(host_bits(lf), seg[0])), (kind, p)
            words[p] = wf
        ids = pick(tf, words)
        if kind in ("nan", "inf"):
            assert ids[0] == tf.TF_PICK_FAILED
            flagged = int(host_bits(words)[0 if kind == "nan" else 1, 0]) >> 32
            assert flagged & 0x80000000
        else:
            assert ids[0] != tf.TF_PICK_FAILED
        if expect is not None:
            assert ids[0] == expect, (ids[0], expect)
    finally:
        for row, a, b, c in reversed(saved):
            W.wq[row], W.scales[row], W.biases[row] = a, b, c
        torch.cuda.synchronize()


@pytest.mark.parametrize("kind", ["natural", "nan"])
def test_fused_narrow_long_k(tf, orc, kind):
    """A head too narrow for the tile ring with a long K (3,000 rows, K = 17,920:
    the narrow-call kernel, whose warps leave the keys): the fused call's logits and words
    equal the unfused call's, for both halves and the whole, with a NaN row
    planted; and the logits are within the V bar of the oracle on sampled rows."""
    V, K = 3000, 17920
    w = synth.make_weights(V, K, seed=15, tag=synth.TAG_HEAD)
    if kind == "nan":
        wq, sc, bi = (a.copy() for a in w.astuple())
        sc[2200] = 0x7FC0
        w = synth.QWeights(wq, sc, bi)
    W = DevWeights(w)
    x_bits = synth.make_x(1, K, seed=15, tag=synth.TAG_X)
    x = dev(x_bits)
    for seg in (tf.tf_split_rows(V, 2, 0), tf.tf_split_rows(V, 2, 1), (0, V)):
        lu, wu = unfused(tf, x, W, seg, seg[0])
        lf, wf = fused(tf, x, W, seg, seg[0])
        torch.cuda.synchronize()
        assert bits_equal(lf, lu) and torch.equal(wf, wu), seg
    rows = np.unique(np.concatenate([np.arange(0, V, 23), [V - 1, 2200]]))
    yo, y64, ad = orc.qmm_rows(x_bits, *w.astuple(), rows, nthreads=os.cpu_count() or 1, want_f64=True)
    check_values(host_bits(lf)[:, rows], yo, y64, ad, K, f"narrow long-K head ({kind})")
