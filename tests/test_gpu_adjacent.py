"""The steps on either side of the seam, on the GPU against the oracle, bit for
bit (a NaN sum only as a NaN: IEEE leaves its payload open): the fp32 residual add of a gathered bf16 row (TensorFold PR #1433 step-2
body: rows are gathered whole and added in the fp32 stream) and the
whole-table embedding gather with its bound (the same body and the embedBound
commit: the bound is the whole 248,320-row table, never the shard's 124,160).
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import dev, host_bits, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def stream_case(M, n, seed):
    rng = np.random.default_rng(seed)
    h = (rng.standard_normal((M, n)) * np.exp2(rng.integers(-24, 24, (M, n)))).astype(np.float32)
    y = synth.to_bf16_bits((rng.standard_normal((M, n)) * np.exp2(rng.integers(-30, 30, (M, n)))).astype(np.float32))
    # IEEE specials and the fp32 round-to-even tie
    h.flat[0], y.flat[0] = np.float32(1.0 + 2.0 ** -23), 0x3380          # + 2^-24: the tie, to even
    h.flat[1], y.flat[1] = np.float32(np.inf), 0xFF80                     # inf + -inf = NaN
    h.flat[2], y.flat[2] = np.float32(1.0), 0x7FC0                        # NaN row value
    h.flat[3], y.flat[3] = np.float32(-0.0), 0x8000                       # -0 + -0 = -0
    return h, y


@pytest.mark.parametrize("M,n,pad_h,pad_y", [(1, 5120, 0, 0), (3, 17408, 0, 0), (2, 8705, 0, 0), (1, 7, 0, 0),
                                              (4, 1000, 1, 0), (2, 1024, 0, 3)])
def test_residual_add_equals_oracle(tf, orc, M, n, pad_h, pad_y):
    h, y = stream_case(M, n, seed=M * 7 + n)
    want = orc.residual_add(h, y)
    hd = torch.zeros(M, n + pad_h, dtype=torch.float32, device="cuda")
    hd[:, :n] = torch.from_numpy(h).cuda()
    yd = torch.zeros(M, n + pad_y, dtype=torch.bfloat16, device="cuda")
    yd[:, :n] = dev(y)
    hv, yv = hd[:, :n], yd[:, :n]
    tf.tf_residual_add(hv, yv)
    torch.cuda.synchronize()
    got = hv.cpu().numpy()
    # bit for bit, except that any NaN matches any NaN (IEEE leaves the payload open)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))
    if pad_h:
        assert torch.all(hd[:, n:] == 0)          # the padding beyond n is untouched


def test_embed_rows_equals_oracle(tf, orc):
    rows, H = 4096, 5120
    rng = np.random.default_rng(5)
    table = synth.to_bf16_bits(rng.standard_normal((rows, H)).astype(np.float32))
    ids = np.array([0, 4095, 17, 2048, 4096, 99999, 3], dtype=np.uint32)
    want = orc.embed_rows(table, ids, rows)
    out = torch.empty(len(ids), H, dtype=torch.bfloat16, device="cuda")
    tf.tf_embed_rows(dev(table), rows, dev(ids.view(np.int32)), out)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), want)
    assert np.all(host_bits(out)[4] == 0x7FC0) and np.all(host_bits(out)[5] == 0x7FC0)


def test_embed_rows_whole_vocabulary_bound(tf, orc):
    """The pages' case: a 248,320-row table, ids on both sides of 124,160; the
    shard's width as the bound is refused before anything runs."""
    V, H = synth.VOCAB, 24                      # narrow rows: the scalar path (H % 8 != 0)
    rng = np.random.default_rng(6)
    table = rng.integers(0, 1 << 16, size=(V, H), dtype=np.uint16)
    ids = np.array([124159, 124160, 200000, 248319, 248320], dtype=np.uint32)
    tdev, idev = dev(table), dev(ids.view(np.int32))
    out = torch.empty(len(ids), H, dtype=torch.bfloat16, device="cuda")
    tf.tf_embed_rows(tdev, V, idev, out)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), orc.embed_rows(table, ids, V))
    assert tf.tf_embed_rows(tdev, V // 2, idev, out, check=False) == tf.TF_E_RANGE
