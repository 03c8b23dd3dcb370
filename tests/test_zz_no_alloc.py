"""tf_argmax_rows_static, the argmax for callers that cannot allocate device
memory (a host that hands the library a fixed arena and forbids any other
cudaMalloc, or a latency path that cannot afford cudaMalloc's implicit device
synchronisation).  Its partial results live in a device array inside libtf.so
instead of a caller buffer.

Checked here, through the C ABI: on two calls in a row it returns the same
words as tf_argmax_rows with a caller scratch buffer (argmax words are integers,
so the comparison is bit for bit); the first call also performs the one-time
address lookup.  A request larger than the built-in array is refused before
anything runs.  This file is collected last so that a run that stops at the
first failure has run every other test before it.
"""
import ctypes

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


def logits_case(M, n, seed):
    rng = np.random.default_rng(seed)
    v = synth.to_bf16_bits(rng.standard_normal((M, n)).astype(np.float32))
    if M > 1:
        v[1, n // 3] = 0x7FC0                    # a NaN row
    if M > 2:
        v[2, [5, n - 5]] = 0x7F00                # an exact tie, lower id wins
    return v


def words_with_scratch(tf, lg, base):
    M, n = lg.shape
    w = torch.empty(M, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_argmax_scratch_bytes(M, n), dtype=torch.uint8, device="cuda")
    assert tf.tf_argmax_rows(lg, base, w, scratch) == tf.TF_OK
    return w


def static_call(tf, lg, base, words):
    """Through the C entry point directly (device pointers and sizes only)."""
    M, n = lg.shape
    return tf.lib.tf_argmax_rows_static(ctypes.c_void_p(lg.data_ptr()), M, n, lg.stride(0), base,
                                        ctypes.c_void_p(words.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,n,base", [(1, 124160, 124160), (16, 124160, 0), (3, 2048, 2048), (700, 33, 7)])
def test_static_scratch_matches_caller_scratch(tf, M, n, base):
    lg = dev(logits_case(M, n, seed=M + n))
    want = words_with_scratch(tf, lg, base)
    for call in range(2):   # two calls in a row: the array keeps the previous call's contents
        got = torch.full((M,), -1, dtype=torch.int64, device="cuda")
        assert static_call(tf, lg, base, got) == tf.TF_OK
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(got), host_bits(want)), f"call {call}"


def test_static_scratch_after_a_different_shape(tf):
    """A large call, then a small one: stale entries of the first must not leak into the second."""
    big = dev(logits_case(64, 124160, seed=1))
    wb = torch.empty(64, dtype=torch.int64, device="cuda")
    assert static_call(tf, big, 0, wb) == tf.TF_OK
    small = dev(logits_case(2, 5000, seed=2))
    ws = torch.empty(2, dtype=torch.int64, device="cuda")
    assert static_call(tf, small, 100, ws) == tf.TF_OK
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(ws), host_bits(words_with_scratch(tf, small, 100)))
    assert np.array_equal(host_bits(wb), host_bits(words_with_scratch(tf, big, 0)))


def test_static_scratch_refuses_oversize(tf):
    M, n = 8193, 4096
    assert tf.tf_argmax_scratch_bytes(M, n) > tf.TF_STATIC_SCRATCH_BYTES
    lg = torch.zeros(1, 8, dtype=torch.bfloat16, device="cuda")   # never read: refused first
    w = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = tf.lib.tf_argmax_rows_static(ctypes.c_void_p(lg.data_ptr()), M, n, n, 0, ctypes.c_void_p(w.data_ptr()), None)
    assert st == tf.TF_E_ARG
