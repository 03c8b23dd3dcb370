"""PairDecode on the GPU kernels, as a one-rank NCCL group (every call here gets
one GPU): with one rank the seams' all-gathers return the rank's own rows, so
the step must give exactly the one-GPU whole path -- the fused gate-up with the
GLU, down, the head, argmax and pick -- bit for bit.  Each stage of the step is
also held to the oracle: the gate and up rows and the down and head outputs
within 2 bf16 ulps of the fp64 oracle on the GPU stage's own inputs, the GLU
frame against the oracle's GLU of the GPU's gate and up rows, the word and the
id bit for bit against the oracle's scan and pick of the GPU's logits.  The
exchange between two ranks is checked on CPU ranks in test_pair_seam.py."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_pair_decode_one_rank_equals_whole(orc):
    need_gpu()
    import torch.distributed as dist
    import row_split_int4_b200 as tf
    from row_split_int4_b200.pair import PairDecode, PairSeam

    H, F, V = 1024, 2048, 4096
    hgu = synth.make_weights(2 * F, H, seed=41, tag=synth.TAG_W)
    hd = synth.make_weights(H, F, seed=41, tag=synth.TAG_W2)
    hlm = synth.make_weights(V, H, seed=41, tag=synth.TAG_HEAD)
    wgu, wd, wlm = DevWeights(hgu), DevWeights(hd), DevWeights(hlm)
    xb = synth.make_x(1, H, seed=41)
    x = dev(xb)

    # the one-GPU whole path
    act = empty_bf16(1, F)
    tf.tf_qmm_rows(x, *wgu.t(), [(0, F), (F, F)], act, epi=tf.TF_EPI_GLU)
    y = empty_bf16(1, H)
    tf.tf_qmm_rows(act, *wd.t(), [(0, H)], y)
    logits = empty_bf16(1, V)
    tf.tf_qmm_rows(y, *wlm.t(), [(0, V)], logits)
    word = torch.empty(1, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_argmax_scratch_bytes(1, V), dtype=torch.uint8, device="cuda")
    tf.tf_argmax_rows(logits, 0, word, scratch)
    ids_w = torch.empty(1, dtype=torch.int32, device="cuda")
    tf.tf_pick(word[None, :].contiguous(), ids_w)

    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        dec = PairDecode(PairSeam(), wgu.t(), wd.t(), wlm.t())
        ids = dec.step(x)
        torch.cuda.synchronize()
        assert bits_equal(dec.act, act) and bits_equal(dec.y, y) and bits_equal(dec.logits, logits)
        assert np.array_equal(host_bits(ids), host_bits(ids_w))
        assert host_bits(ids)[0] == int(host_bits(word)[0]) >> 32
    finally:
        dist.destroy_process_group()

    # every stage against the oracle, on the GPU stage's own inputs
    g, u = empty_bf16(1, F), empty_bf16(1, F)
    tf.tf_qmm_rows(x, *wgu.t(), [(0, F)], g)
    tf.tf_qmm_rows(x, *wgu.t(), [(F, F)], u)
    torch.cuda.synchronize()
    for t, rows, what in ((g, np.arange(F), "gate"), (u, np.arange(F, 2 * F), "up")):
        yo, y64, ad = orc.qmm_rows(xb, *hgu.astuple(), rows, want_f64=True)
        check_values(host_bits(t), yo, y64, ad, H, what)
    check_values(host_bits(dec.act), orc.glu(host_bits(g), host_bits(u)), what="GLU frame")
    yo, y64, ad = orc.qmm_rows(host_bits(dec.act), *hd.astuple(), np.arange(H), want_f64=True)
    check_values(host_bits(dec.y), yo, y64, ad, F, "down")
    yo, y64, ad = orc.qmm_rows(host_bits(dec.y), *hlm.astuple(), np.arange(V), want_f64=True)
    check_values(host_bits(dec.logits), yo, y64, ad, H, "head logits")
    o_word = orc.argmax_rows(host_bits(dec.logits), 0)
    assert np.array_equal(host_bits(word), o_word)
    assert np.array_equal(host_bits(ids), orc.pick(o_word[None, :]))
