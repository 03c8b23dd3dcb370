"""Gather, argmax and pick edge cases on the GPU against the oracle."""
import itertools

import numpy as np
import pytest
import torch

import synth
from gpu_util import bits_equal, dev, empty_bf16, host_bits, need_gpu
import head_pipeline as HP

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def rand_bits(rng, shape):
    return synth.to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


@pytest.mark.parametrize("widths,M,ld_extra", [((256, 256), 1, 0), ((8704, 8704), 128, 0), ((5, 7, 1), 3, 0),
                                               ((16, 24, 8), 4, 8), ((2560, 2560), 7, 3)])
def test_gather(tf, orc, widths, M, ld_extra):
    rng = np.random.default_rng(sum(widths) + M)
    parts = [rand_bits(rng, (M, w)) for w in widths]
    tot = sum(widths)
    dst_full = empty_bf16(M, tot + ld_extra)
    dst = dst_full[:, :tot]
    st = tf.tf_gather_rows(dst, [dev(p) for p in parts], widths, check=False)
    torch.cuda.synchronize()
    assert st == tf.TF_OK
    assert np.array_equal(host_bits(dst), orc.gather_rows(parts, M))


def test_gather_broken_part(tf, orc):
    rng = np.random.default_rng(3)
    a = rand_bits(rng, (4, 64))
    dst = empty_bf16(4, 128)
    st = tf.tf_gather_rows(dst, [dev(a), None], [64, 64], check=False)
    torch.cuda.synchronize()
    assert st == tf.TF_E_BROKEN
    want = orc.gather_rows([a, None], 4, widths=[64, 64])
    assert np.array_equal(host_bits(dst), want)
    assert np.all(host_bits(dst)[:, 64:] == 0x7FC0)


ALPHA = [0xBF80, 0x8000, 0x0000, 0x3F80, 0x7FC0, 0x7F80, 0xFF80]


def test_argmax_pick_bruteforce(tf, orc):
    """Every 5-vector over {-1,-0,+0,1,NaN,+Inf,-Inf} at every split point (16,807 rows)."""
    vecs = np.array(list(itertools.product(ALPHA, repeat=5)), dtype=np.uint16)
    M = vecs.shape[0]
    vt = dev(vecs)
    # whole rows (unaligned width 5: scalar path)
    words = torch.empty(1, M, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_argmax_scratch_bytes(M, 5), dtype=torch.uint8, device="cuda")
    tf.tf_argmax_rows(vt, 0, words[0], scratch)
    ids = torch.empty(M, dtype=torch.int32, device="cuda")
    tf.tf_pick(words, ids)
    torch.cuda.synchronize()
    ow = orc.argmax_rows(vecs, 0)
    assert np.array_equal(host_bits(words)[0], ow)
    assert np.array_equal(host_bits(ids), orc.pick(ow[None, :]))
    for cut in range(1, 5):
        a = dev(np.ascontiguousarray(vecs[:, :cut]))
        b = dev(np.ascontiguousarray(vecs[:, cut:]))
        w2, i2 = HP.gpu_head_words(tf, [a, b], [0, cut])
        torch.cuda.synchronize()
        o2, oi = orc.head_split([vecs[:, :cut], vecs[:, cut:]], [0, cut])
        assert np.array_equal(host_bits(w2), o2), cut
        assert np.array_equal(host_bits(i2), oi), cut
        assert np.array_equal(host_bits(i2), host_bits(ids)), f"split at {cut} != whole"


@pytest.mark.parametrize("n,ld,M,base", [(1, 1, 3, 0), (7, 9, 5, 100), (2048, 2048, 8, 2048), (124160, 124160, 2, 124160),
                                         (124161, 124168, 3, 0), (33, 40, 700, 2 ** 31 - 33)])
def test_argmax_shapes(tf, orc, n, ld, M, base):
    rng = np.random.default_rng(n + M)
    full = rand_bits(rng, (M, ld))
    # a few planted specials
    full[0, n // 2] = 0x7F80 if n > 2 else full[0, 0]
    if M > 1:
        full[1, : n] = 0x3F80
    if M > 2:
        full[2, n - 1] = 0x7F7F   # largest finite at the very end
    t = dev(full)[:, :n]
    words = torch.empty(M, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_argmax_scratch_bytes(M, n), dtype=torch.uint8, device="cuda")
    tf.tf_argmax_rows(t, base, words, scratch)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(words), orc.argmax_rows(np.ascontiguousarray(full[:, :n]), base))


def test_pick_many_parts(tf, orc):
    rng = np.random.default_rng(9)
    for nparts in range(1, 9):
        M = 257
        vals = rng.integers(0, 4, (nparts, M))
        words = np.zeros((nparts, M), dtype=np.uint64)
        for p in range(nparts):
            ids = p * 1000 + rng.integers(0, 1000, M)
            bits = np.array([0x3F80, 0x4000, 0x4040, 0x8000], dtype=np.uint64)[vals[p]]
            words[p] = (ids.astype(np.uint64) << np.uint64(32)) | (bits << np.uint64(16))
        flag_rows = rng.choice(M, 20, replace=False)
        words[rng.integers(0, nparts, 20), flag_rows] |= np.uint64(0x80000000) << np.uint64(32)
        ids_t = torch.empty(M, dtype=torch.int32, device="cuda")
        tf.tf_pick(dev(words), ids_t)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(ids_t), orc.pick(words)), nparts
