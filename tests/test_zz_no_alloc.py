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


_RESET_CHILD = r"""
import ctypes, sys
import numpy as np
lib = ctypes.CDLL(sys.argv[1])
rt = ctypes.CDLL("libcudart.so.12")   # the runtime instance libtf.so is linked against
lib.tf_argmax_rows_static.restype = ctypes.c_int
M, n = 3, 5000
rng = np.random.default_rng(5)
host = (rng.standard_normal((M, n)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)

def once():
    d_l, d_w = ctypes.c_void_p(), ctypes.c_void_p()
    assert rt.cudaMalloc(ctypes.byref(d_l), ctypes.c_size_t(M * n * 2)) == 0
    assert rt.cudaMalloc(ctypes.byref(d_w), ctypes.c_size_t(M * 8)) == 0
    assert rt.cudaMemcpy(d_l, host.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(M * n * 2), 1) == 0
    st = lib.tf_argmax_rows_static(d_l, M, n, n, ctypes.c_uint32(0), d_w, None)
    assert rt.cudaDeviceSynchronize() == 0
    out = np.zeros(M, dtype=np.uint64)
    assert rt.cudaMemcpy(out.ctypes.data_as(ctypes.c_void_p), d_w, ctypes.c_size_t(M * 8), 2) == 0
    rt.cudaFree(d_l)
    rt.cudaFree(d_w)
    return st, out

st1, w1 = once()
assert rt.cudaDeviceReset() == 0   # a new primary context, the library's module loaded again
st2, w2 = once()
np.save(sys.argv[2], np.stack([w1, w2]))
print(st1, st2)
"""


def test_static_scratch_after_context_reset(tf, orc, tmp_path):
    """After cudaDeviceReset the next call looks its array's address up again in the
    new context (run in a child process that uses only the CUDA runtime, so the
    reset touches no other state of this process)."""
    import os
    import subprocess
    import sys
    out = tmp_path / "words.npy"
    r = subprocess.run([sys.executable, "-c", _RESET_CHILD, os.path.abspath(tf.LIB_PATH), str(out)],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.split() == ["0", "0"], r.stdout
    words = np.load(out)
    rng = np.random.default_rng(5)
    host = (rng.standard_normal((3, 5000)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    want = orc.argmax_rows(host, 0)
    assert np.array_equal(words[0], want) and np.array_equal(words[1], want)
