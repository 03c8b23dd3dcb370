"""tf_top2_rows and tf_top2_merge, the merged top two of the head (TensorFold PR
#1433, step-1 and step-2 bodies: the session keeps the merged top two for its
cross-block tie test and reads the pick's sentinel as a failure).

The words are compared bit for bit with the oracle's on the same logits
(I: the oracle scans the GPU's own inputs); the merge of the two halves' top two
must equal the top two of the whole row (S), its winner must equal
tf_argmax_rows' word over the whole row and its id tf_pick's id over the halves.
Cases: natural rows, exact ties planted inside a half and across the halves,
+0/-0 ties, NaN and Inf rows in either half or both, one-element slices, a
ragged length, an unaligned view (scalar path), and a full lm_head half of real
logits from the synthetic head.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def make_logits(M, n, seed, ties=False, cross_tie=False, nan=(), inf=()):
    x = synth.make_x(M, n, seed=seed, tag=9)
    rng = np.random.default_rng(seed)
    f = synth.bf16_bits_to_f32(x)
    for m in range(M):
        j = int(np.argmax(f[m]))
        if ties and n > 2:
            k = int(rng.integers(0, n - 1))
            x[m, k if k != j else n - 1] = x[m, j]       # an exact tie with the winner
        if cross_tie and n > 2:
            x[m, (j + n // 2) % n] = x[m, j]             # the same value in the other half
    for m, j in nan:
        x[m, j] = 0x7FC0
    for m, j in inf:
        x[m, j] = 0x7F80
    return x


def gpu_top2(tf, lg, id_base):
    M, n = lg.shape
    w = torch.full((M, 2), -1, dtype=torch.int64, device="cuda")
    scratch = torch.empty(max(8, tf.tf_top2_scratch_bytes(M, n)), dtype=torch.uint8, device="cuda")
    tf.tf_top2_rows(lg, id_base, w, scratch)
    return w


def gpu_argmax(tf, lg, id_base):
    M, n = lg.shape
    w = torch.empty(M, dtype=torch.int64, device="cuda")
    scratch = torch.empty(max(8, tf.tf_argmax_scratch_bytes(M, n)), dtype=torch.uint8, device="cuda")
    tf.tf_argmax_rows(lg, id_base, w, scratch)
    return w


def check_split(tf, orc, x):
    """Halves -> top two each -> merge, against the oracle and against the whole row."""
    M, n = x.shape
    h = n // 2
    lg = dev(x)
    parts = torch.stack([gpu_top2(tf, lg[:, :h], 0), gpu_top2(tf, lg[:, h:], h)]).contiguous()
    merged = torch.empty(M, 2, dtype=torch.int64, device="cuda")
    tf.tf_top2_merge(parts, merged)
    whole = gpu_top2(tf, lg, 0)
    torch.cuda.synchronize()
    p_h = host_bits(parts)
    assert np.array_equal(p_h[0], orc.top2_rows(x[:, :h], 0))
    assert np.array_equal(p_h[1], orc.top2_rows(x[:, h:], h))
    assert np.array_equal(host_bits(merged), orc.top2_merge(p_h))
    assert np.array_equal(host_bits(merged), host_bits(whole)), "merge of the halves != top two of the whole row"
    assert np.array_equal(host_bits(whole), orc.top2_rows(x, 0))
    # the winner is the argmax word over the whole row, and its id the pick over the halves
    assert np.array_equal(host_bits(whole)[:, 0], host_bits(gpu_argmax(tf, lg, 0)))
    words = torch.stack([gpu_argmax(tf, lg[:, :h], 0), gpu_argmax(tf, lg[:, h:], h)]).contiguous()
    ids = torch.empty(M, dtype=torch.int32, device="cuda")
    tf.tf_pick(words, ids)
    top_ids = (host_bits(merged)[:, 0] >> np.uint64(32)).astype(np.uint32)
    picked = host_bits(ids)
    flagged = (top_ids & np.uint32(tf.TF_PAIR_FLAG)) != 0
    assert np.array_equal(picked[~flagged], top_ids[~flagged])
    assert (picked[flagged] == tf.TF_PICK_FAILED).all()
    return host_bits(merged)


@pytest.mark.parametrize("n", [2, 8, 4096, 5001, 20000])
def test_top2_split_natural_and_ties(tf, orc, n):
    check_split(tf, orc, make_logits(5, n, seed=n))
    check_split(tf, orc, make_logits(5, n, seed=n + 1, ties=True))
    got = check_split(tf, orc, make_logits(4, n, seed=n + 2, cross_tie=True))
    if n > 2:
        v = got & np.uint64(0xFFFFFFFF)
        assert np.array_equal(v[:, 0], v[:, 1]), "a value in both halves is a tie of the top two"


def test_top2_signed_zero_and_non_finite(tf, orc):
    n = 4096
    x = make_logits(6, n, seed=5, nan=[(1, 3000)], inf=[(2, 10), (3, 100), (3, 3000)])
    x[4, :] = 0x8000           # every value -0 but one +0: ties all the way down
    x[4, 2500] = 0x0000
    x[5, :] = 0xBF80           # -1 everywhere: the top two are the two lowest ids
    got = check_split(tf, orc, x)
    flag = np.uint64(tf.TF_PAIR_FLAG) << np.uint64(32)
    assert (got[1:4] & flag).all() and not (got[[0, 4, 5]] & flag).any()
    assert int(got[3, 0]) >> 32 == tf.TF_PAIR_FLAG | 100           # the first non-finite id of the row
    assert int(got[4, 0]) >> 32 == 0 and int(got[4, 1]) >> 32 == 1
    assert int(got[5, 0]) >> 32 == 0 and int(got[5, 1]) >> 32 == 1


def test_top2_one_element_and_scalar_path(tf, orc):
    x = make_logits(3, 1, seed=7)
    w = gpu_top2(tf, dev(x), 40)
    torch.cuda.synchronize()
    got = host_bits(w)
    assert np.array_equal(got, orc.top2_rows(x, 40))
    assert (got[:, 1] == np.uint64(tf.TF_TOP2_NONE)).all()
    # an unaligned view takes the scalar loads and gives the same words
    x = make_logits(3, 3001, seed=8, ties=True)
    big = dev(np.concatenate([np.zeros((3, 1), dtype=np.uint16), x], axis=1))
    w_scalar = gpu_top2(tf, big[:, 1:], 0)
    w_vec = gpu_top2(tf, dev(x), 0)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(w_scalar), host_bits(w_vec))
    assert np.array_equal(host_bits(w_vec), orc.top2_rows(x, 0))


def test_top2_merge_three_parts_and_lowest_flag(tf, orc):
    x = make_logits(4, 3000, seed=11, nan=[(1, 2500), (2, 10), (2, 2900)])
    lg = dev(x)
    cuts = [0, 700, 2100, 3000]
    parts = torch.stack([gpu_top2(tf, lg[:, a:b], a) for a, b in zip(cuts, cuts[1:])]).contiguous()
    merged = torch.empty(4, 2, dtype=torch.int64, device="cuda")
    tf.tf_top2_merge(parts, merged)
    torch.cuda.synchronize()
    got = host_bits(merged)
    assert np.array_equal(got, orc.top2_merge(host_bits(parts)))
    assert np.array_equal(got, orc.top2_rows(x, 0))
    assert int(got[2, 0]) >> 32 == tf.TF_PAIR_FLAG | 10    # row 2: part 0's flag, not part 2's


def test_top2_lm_head_half_real_logits(tf, orc):
    """The 124,160-row half of the 248,320-row head at K = 5,120: logits from the
    qmm kernel, then the top two of each half and their merge."""
    rows, K = synth.VOCAB // 2, synth.HIDDEN
    W = DevWeights(synth.make_weights(synth.VOCAB, K, seed=17, tag=synth.TAG_HEAD))
    x = dev(synth.make_x(1, K, seed=17, tag=5))
    halves = []
    for h in range(2):
        lg = empty_bf16(1, rows)
        tf.tf_qmm_rows(x, *W.t(), [(h * rows, rows)], lg)
        halves.append(lg)
    parts = torch.stack([gpu_top2(tf, halves[h], h * rows) for h in range(2)]).contiguous()
    merged = torch.empty(1, 2, dtype=torch.int64, device="cuda")
    tf.tf_top2_merge(parts, merged)
    torch.cuda.synchronize()
    lh = np.concatenate([host_bits(halves[0]), host_bits(halves[1])], axis=1)
    assert np.array_equal(host_bits(parts)[0], orc.top2_rows(lh[:, :rows], 0))
    assert np.array_equal(host_bits(parts)[1], orc.top2_rows(lh[:, rows:], rows))
    assert np.array_equal(host_bits(merged), orc.top2_rows(lh, 0))
