"""Decode workloads at M=1 and full size.

* MLP layer: fused gate+up K=5,120, N=2x17,408 (each half owns 8,704 rows of
  each member), gate*SiLU(up) in fp32 rounded to bf16, then down K=17,408,
  N=5,120 as two 2,560-row halves; split+gather and whole.
* Head: lm_head K=5,120, N=248,320 as 2x124,160, per-half argmax and pick on
  sixteen seeded rows with a tie straddling the half boundary, one +Inf, one
  NaN and one all-equal row.
"""
import os

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu
import head_pipeline as HP

pytestmark = pytest.mark.gpu
NT = os.cpu_count() or 1


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


@pytest.fixture(scope="module")
def mlp_weights():
    H, F = synth.HIDDEN, synth.FFN
    wgu = synth.make_weights(2 * F, H, seed=0, tag=synth.TAG_W)
    wd = synth.make_weights(H, F, seed=0, tag=synth.TAG_W2)
    return wgu, wd


def test_decode_mlp(tf, orc, mlp_weights):
    H, F = synth.HIDDEN, synth.FFN
    wgu, wd = mlp_weights
    Wgu, Wd = DevWeights(wgu), DevWeights(wd)
    x = synth.make_x(1, H, seed=0)
    xt = dev(x)
    window = synth.WINDOW_BYTES

    # whole
    act_w = empty_bf16(1, F)
    tf.tf_qmm_rows(xt, *Wgu.t(), [(0, F), (F, F)], act_w, epi=tf.TF_EPI_GLU)
    y_w = empty_bf16(1, H)
    tf.tf_qmm_rows(act_w, *Wd.t(), [(0, H)], y_w)
    # split + gather
    acts = []
    for h in range(2):
        a = empty_bf16(1, F // 2)
        tf.tf_qmm_rows(xt, *Wgu.t(), tf.tf_member_segs(F, 2, h), a, epi=tf.TF_EPI_GLU)
        acts.append(a)
    act_s = empty_bf16(1, F)
    tf.tf_gather_rows(act_s, acts, [F // 2] * 2, window_bytes=window)
    ys = []
    for h in range(2):
        yh = empty_bf16(1, H // 2)
        tf.tf_qmm_rows(act_s, *Wd.t(), [tf.tf_split_rows(H, 2, h)], yh)
        ys.append(yh)
    y_s = empty_bf16(1, H)
    tf.tf_gather_rows(y_s, ys, [H // 2] * 2, window_bytes=window)
    # unfused gate / up rows: the GLU's inputs
    g = empty_bf16(1, F)
    u = empty_bf16(1, F)
    tf.tf_qmm_rows(xt, *Wgu.t(), [(0, F)], g)
    tf.tf_qmm_rows(xt, *Wgu.t(), [(F, F)], u)
    torch.cuda.synchronize()

    # S
    assert bits_equal(act_s, act_w), "activated frame: split != whole"
    assert bits_equal(y_s, y_w), "down output: split != whole"
    # V, per stage
    go, g64, gad = orc.qmm_rows(x, *wgu.astuple(), np.arange(F), nthreads=NT, want_f64=True)
    uo, u64, uad = orc.qmm_rows(x, *wgu.astuple(), np.arange(F, 2 * F), nthreads=NT, want_f64=True)
    s1 = check_values(host_bits(g), go, g64, gad, H, "gate rows")
    s2 = check_values(host_bits(u), uo, u64, uad, H, "up rows")
    s3 = check_values(host_bits(act_w), orc.glu(host_bits(g), host_bits(u)), what="GLU stage")
    a_bits = host_bits(act_w)
    yo, y64, yad = orc.qmm_rows(a_bits, *wd.astuple(), np.arange(H), nthreads=NT, want_f64=True)
    s4 = check_values(host_bits(y_w), yo, y64, yad, F, "down")
    # end-to-end oracle chain, reported
    a_chain, y_chain = orc.mlp_split(x, wgu.astuple(), wd.astuple(), nthreads=NT)
    d = np.abs(synth.bf16_bits_to_f32(host_bits(y_s)).astype(np.float64) - synth.bf16_bits_to_f32(y_chain))
    print(f"\ndecode MLP: gate {s1} up {s2} glu {s3} down {s4}; end-to-end chain: "
          f"{int((host_bits(y_s) == y_chain).sum())}/{H} outputs bit-equal, max |diff| {d.max():.3g}")


@pytest.fixture(scope="module")
def head_weights():
    return synth.make_weights(synth.VOCAB, synth.HIDDEN, seed=0, tag=synth.TAG_HEAD)


def test_head_sixteen_rows(tf, orc, head_weights):
    W = DevWeights(head_weights)
    x = synth.make_x(16, synth.HIDDEN, seed=0, tag=5)
    plants = synth.head_plants(synth.VOCAB)
    res = HP.check_head(tf, orc, x, head_weights, W, plants, nthreads=NT)
    ids = res["ids"]
    h = synth.VOCAB // 2
    assert ids[0] == h - 1, "the tie straddling the half boundary goes to the lower id"
    assert ids[1] == 0xFFFFFFFF and ids[2] == 0xFFFFFFFF, "+Inf and NaN rows give the sentinel"
    assert ids[3] == 0, "an all-equal row picks id 0"
    print(f"\nhead: {res}")
