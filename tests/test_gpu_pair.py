"""PairDecode on the GPU kernels, as a one-rank NCCL group (every call here gets
one GPU): with one rank the seams' all-gathers return the rank's own rows, so
the step must give exactly the one-GPU whole path -- the fused gate-up with the
GLU, down, the head, argmax and pick -- bit for bit.  This checks the step's
composition (shares, buffers, calls); the exchange between two ranks is checked
on CPU ranks in test_pair_seam.py."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_pair_decode_one_rank_equals_whole():
    need_gpu()
    import torch.distributed as dist
    import row_split_int4_b200 as tf
    from row_split_int4_b200.pair import PairDecode, PairSeam

    H, F, V = 1024, 2048, 4096
    wgu = DevWeights(synth.make_weights(2 * F, H, seed=41, tag=synth.TAG_W))
    wd = DevWeights(synth.make_weights(H, F, seed=41, tag=synth.TAG_W2))
    wlm = DevWeights(synth.make_weights(V, H, seed=41, tag=synth.TAG_HEAD))
    x = dev(synth.make_x(1, H, seed=41))

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
