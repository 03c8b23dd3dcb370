"""Tiny workload (CPU-seconds): one int4 affine layer K=1,024, N=512 as two
256-row halves, M=1, then a head over a 4,096-entry vocabulary (two halves of
2,048) fed by the layer's 512-wide output, with three planted exact
cross-half ties and one NaN row.  Plus the qmm edge cases: ragged K and N,
odd GLU widths, empty calls, multi-row calls against single-row calls."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu
import head_pipeline as HP

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def qmm(tf, xt, W, segs, epi=0):
    ncols = segs[0][1] if epi else sum(n for _, n in segs)
    y = empty_bf16(xt.shape[0], ncols)
    tf.tf_qmm_rows(xt, *W.t(), segs, y, epi=epi)
    return y


def test_tiny_layer(tf, orc):
    K, N = synth.TINY_K, synth.TINY_N
    w = synth.make_weights(N, K, seed=0)
    W = DevWeights(w)
    x = synth.make_x(1, K, seed=0)
    xt = dev(x)
    whole = qmm(tf, xt, W, [(0, N)])
    halves = [qmm(tf, xt, W, [tf.tf_split_rows(N, 2, h)]) for h in range(2)]
    joined = empty_bf16(1, N)
    tf.tf_gather_rows(joined, halves, [N // 2, N // 2])
    torch.cuda.synchronize()
    assert bits_equal(joined, whole)
    y, y64, ad = orc.qmm_rows(x, *w.astuple(), np.arange(N), want_f64=True)
    st = check_values(host_bits(whole), y, y64, ad, K, "tiny layer")
    assert st["floor_used"] == 0


def test_tiny_head_with_plants(tf, orc):
    """8 seeded rows through the tiny layer (M=1 each), then the split head."""
    K, N = synth.TINY_K, synth.TINY_N
    HK, V = synth.TINY_HEAD_K, synth.TINY_VOCAB
    assert HK == N
    w1 = synth.make_weights(N, K, seed=0)
    wh = synth.make_weights(V, HK, seed=0, tag=synth.TAG_HEAD)
    W1, WH = DevWeights(w1), DevWeights(wh)
    X = synth.make_x(8, K, seed=0)
    hidden = empty_bf16(8, N)
    xt = dev(X)
    for m in range(8):
        tf.tf_qmm_rows(xt[m:m + 1], *W1.t(), [(0, N)], hidden[m:m + 1])
    torch.cuda.synchronize()
    h_bits = host_bits(hidden)
    # the head's per-stage oracle reads the GPU's hidden rows
    plants = synth.tiny_head_plants(V)
    res = HP.check_head(tf, orc, h_bits, wh, WH, plants)
    ids = res["ids"]
    for p in plants:
        if p.kind == "tie":
            assert ids[p.row] == min(p.ids), (p, ids[p.row])
        elif p.kind in ("nan", "inf"):
            assert ids[p.row] == 0xFFFFFFFF
    # the whole chain on the oracle side as well (layer -> head), reported through the same gate
    h_o = orc.qmm_rows(X, *w1.astuple(), np.arange(N))
    chain_res = HP.check_head(tf, orc, h_o, wh, WH, plants)
    assert chain_res["ids"][3] == 0xFFFFFFFF


@pytest.mark.parametrize("K,N", [(64, 7), (192, 33), (1088, 100), (3136, 17), (2048 + 64 * 3, 260)])
def test_ragged_shapes(tf, orc, K, N):
    """K not a multiple of the 1,024-wide chunk, N not a multiple of the 4-row warp unit."""
    w = synth.make_weights(N, K, seed=K)
    W = DevWeights(w)
    x = synth.make_x(3, K, seed=N)
    xt = dev(x)
    for M in (1, 3):
        y = qmm(tf, xt[:M], W, [(0, N)])
        yo, y64, ad = orc.qmm_rows(x[:M], *w.astuple(), np.arange(N), want_f64=True)
        check_values(host_bits(y), yo, y64, ad, K, f"K={K} N={N} M={M}")
    # a row's bits do not depend on the segment layout it is asked in
    segs = [(N - 3, 3), (0, N // 2)] if N > 6 else [(1, N - 1)]
    y1 = qmm(tf, xt[:1], W, [(0, N)])
    y2 = qmm(tf, xt[:1], W, segs)
    cols = np.concatenate([np.arange(r0, r0 + n) for r0, n in segs])
    assert bits_equal(y2, y1[:, torch.as_tensor(cols, device="cuda")])


def test_row_bits_do_not_depend_on_chunk(tf, orc):
    """A row's bits do not depend on where it sits in its chunk: calls of 5 or more
    rows (the tensor cores) agree with one another, and calls of 2 or 3 rows (the
    streaming kernels, each row taking the one-row arithmetic) agree with one-row
    calls; every row is within tolerance of the oracle."""
    K, N = 5120, 96
    w = synth.make_weights(N, K, seed=7)
    W = DevWeights(w)
    x = synth.make_x(16, K, seed=7)
    xt = dev(x)
    y16 = qmm(tf, xt, W, [(0, N)])
    for m0, M in ((3, 5), (9, 7)):
        yM = qmm(tf, xt[m0:m0 + M], W, [(0, N)])
        assert bits_equal(yM, y16[m0:m0 + M]), (m0, M)
    ones = torch.cat([qmm(tf, xt[m:m + 1], W, [(0, N)]) for m in range(16)])
    for m0, M in ((0, 2), (5, 3)):
        yM = qmm(tf, xt[m0:m0 + M], W, [(0, N)])
        assert bits_equal(yM, ones[m0:m0 + M]), (m0, M)
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), np.arange(N), want_f64=True)
    check_values(host_bits(y16), yo, y64, ad, K, "M=16")
    y1 = qmm(tf, xt[:1], W, [(0, N)])
    check_values(host_bits(y1), yo[:1], y64[:1], ad[:1], K, "M=1")


def test_glu_split_whole_and_oracle(tf, orc):
    F, K = 520, 1024     # F/2 = 260 is not a multiple of the 2-column GLU unit
    w = synth.make_weights(2 * F, K, seed=3)
    W = DevWeights(w)
    x = synth.make_x(2, K, seed=3)
    xt = dev(x)
    for M in (1, 2):
        whole = qmm(tf, xt[:M], W, [(0, F), (F, F)], epi=1)
        parts = [qmm(tf, xt[:M], W, tf.tf_member_segs(F, 2, h), epi=1) for h in range(2)]
        joined = empty_bf16(M, F)
        tf.tf_gather_rows(joined, parts, [F // 2, F // 2])
        # the unfused rows give the GLU's inputs
        g = qmm(tf, xt[:M], W, [(0, F)])
        u = qmm(tf, xt[:M], W, [(F, F)])
        torch.cuda.synchronize()
        assert bits_equal(joined, whole)
        # GLU stage on the GPU's own g, u: the fp32 GLU within 2 ulps of the double one
        a_ref = orc.glu(host_bits(g), host_bits(u))
        check_values(host_bits(whole), a_ref, what=f"GLU stage M={M}")
        # g and u themselves against the oracle
        go, g64, gad = orc.qmm_rows(x[:M], *w.astuple(), np.arange(F), want_f64=True)
        check_values(host_bits(g), go, g64, gad, K, "gate rows")


def test_empty_calls(tf):
    K, N = 128, 16
    W = DevWeights(synth.make_weights(N, K, seed=1))
    xt = dev(synth.make_x(1, K, seed=1))
    y = torch.full((1, N), 1.0, dtype=torch.bfloat16, device="cuda")
    assert tf.tf_qmm_rows(xt[:0], *W.t(), [(0, N)], y[:0]) == tf.TF_OK
    assert tf.tf_qmm_rows(xt, *W.t(), [(3, 0)], y[:, :0]) == tf.TF_OK
    torch.cuda.synchronize()
    assert torch.all(y == 1.0)


def test_special_values(tf, orc):
    """Zero weights, very large (finite) scales, and non-finite activations.

    With a NaN or +-Inf in x every output of that row is non-finite on both
    sides; the class may differ (the factorised fp32 sum s*P + b*X can meet
    0*Inf = NaN where the ascending double sum meets +-Inf), and the method
    only acts on non-finite-ness (the argmax flags either)."""
    K, N = 256, 8
    q = np.random.default_rng(0).integers(0, 16, (N, K), dtype=np.uint8)
    sc = np.full((N, K // 64), 0x3C00, dtype=np.uint16)        # 2^-7
    bi = np.full((N, K // 64), 0xBE00, dtype=np.uint16)        # -0.125
    sc[1] = 0x7A00                                              # 2^117: large but finite results
    sc[2] = 0
    bi[2] = 0
    w = synth.QWeights(synth.pack_nibbles(q), sc, bi)
    W = DevWeights(w)
    x = synth.make_x(3, K, seed=5)
    x[1, 10] = 0x7F80          # +Inf in row 1
    x[2, 20] = 0x7FC0          # NaN in row 2
    xt = dev(x)
    y = qmm(tf, xt, W, [(0, N)])
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), np.arange(N), want_f64=True)
    g = host_bits(y)
    assert g[0, 2] == 0, "all-zero weight row gives +0"
    check_values(g[0], yo[0], y64[0], ad[0], K, "finite row")
    for m in (1, 2):
        assert not np.isfinite(synth.bf16_bits_to_f32(g[m])).any()
        assert not np.isfinite(synth.bf16_bits_to_f32(yo[m])).any()
    assert np.all(np.isnan(synth.bf16_bits_to_f32(g[2])))
