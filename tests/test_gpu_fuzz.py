"""Seeded random calls of tf_qmm_rows over every route, against the oracle.

Each case draws its shape from a route's range: the M = 1 tile ring (more than
296 sixteen-row tiles), the narrow-call kernel (K above 8,192, fewer rows), the
per-warp ring (few rows), the tensor cores (M = 4..128), and the fallbacks for a K
that is not a multiple of 512; with one to three row segments of the whole matrix
or the fused gate*SiLU(up) epilogue, and activation rows padded in memory or not.
Every case is checked against the oracle (V: 2 bf16 ulps, or the fp32
accumulation floor where the sum cancels) on all of its columns, or on 384
sampled ones plus both ends of every segment for the larger cases (TensorFold
PR #1433, step-1 body: each rank reduces its rows over the full K; step-2 body:
the GLU of the gate and up halves).  A last set draws fused heads
(tf_qmm_argmax_rows) of random slices: logits against the oracle, the word bit
for bit against the oracle's argmax scan of the GPU's logits (step-1 body:
pair_argmax over each rank's half); random int8 heads (the b70 lab's runtime INT8
LM-head), random argmax calls with planted ties, signed zeros and non-finites, and
random row splits of such logits through the gather, the per-part argmax words and
top twos, the pick and the merged top two (step-1 body: stage, gather,
pair_argmax, pair_pick).
"""
import os

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, check_values, dev, empty_bf16, host_bits, need_gpu

pytestmark = pytest.mark.gpu
NT = os.cpu_count() or 1
ROUTES = ["tile", "split", "warp", "tc", "odd_k", "glu_tile", "glu_tc", "glu_odd_k"]
CASES = 8   # per route


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


def draw(route: str, i: int):
    """(M, K, N_whole, segs, glu, pad) of case i of a route."""
    rng = np.random.default_rng([1433, ROUTES.index(route), i])
    pick = lambda seq: seq[int(rng.integers(len(seq)))]   # noqa: E731
    glu = route.startswith("glu")
    if route in ("tile", "glu_tile"):
        M, K = int(rng.integers(1, 4)), pick([1024, 2048, 3072])
        N = int(rng.integers(4800, 7000)) if not glu else 2 * int(rng.integers(2400, 3600))
    elif route == "split":
        M, K, N = int(rng.integers(1, 3)), pick([9216, 10240, 12800]), int(rng.integers(100, 3000))
    elif route == "warp":
        M, K, N = 1, pick([512, 1536, 4096]), int(rng.integers(1, 2000))
    elif route in ("tc", "glu_tc"):
        M, K = int(rng.integers(4, 129)), pick([512, 2048, 5120])
        N = int(rng.integers(1, 1500)) if not glu else 2 * int(rng.integers(1, 700))
    else:   # K not a multiple of 512
        M, K = int(rng.integers(1, 41)), pick([576, 1088, 2112])
        N = int(rng.integers(1, 800)) if not glu else 2 * int(rng.integers(1, 400))
    if glu:
        F = N // 2
        segs = [(0, F), (F, F)]
    else:
        cuts = np.sort(rng.choice(np.arange(1, N), size=min(2, N - 1), replace=False)) if N > 2 else np.array([], int)
        bounds = [0, *cuts.tolist(), N]
        spans = [(bounds[j], bounds[j + 1] - bounds[j]) for j in range(len(bounds) - 1)]
        nseg = int(rng.integers(1, len(spans) + 1))
        segs = [spans[j] for j in rng.permutation(len(spans))[:nseg]]
    return M, K, N, segs, glu, bool(rng.integers(2))


def planted_logits(rng, M, n):
    """Random bf16 logits [M, n], each row planted with a top tie, a NaN, an
    infinity, all signed zeros, or nothing."""
    v = synth.to_bf16_bits(rng.standard_normal((M, n)).astype(np.float32))
    for m in range(M):
        kind = int(rng.integers(5))
        if kind == 1 and n > 1:
            top = int(np.argmax(synth.bf16_bits_to_f32(v[m])))
            v[m, int(rng.integers(n))] = v[m, top]
        elif kind == 2:
            v[m, int(rng.integers(n))] = 0x7FC0
        elif kind == 3:
            v[m, int(rng.integers(n))] = int(rng.choice([0x7F80, 0xFF80]))
        elif kind == 4:
            v[m, :] = int(rng.choice([0x0000, 0x8000]))
    return v


@pytest.mark.parametrize("route,i", [(r, i) for r in ROUTES for i in range(CASES)])
def test_random_call(tf, orc, route, i):
    M, K, N, segs, glu, pad = draw(route, i)
    w = synth.make_weights(N, K, seed=1000 + 31 * ROUTES.index(route) + i)
    W = DevWeights(w)
    x = synth.make_x(M, K, seed=2000 + 31 * ROUTES.index(route) + i)
    xt = dev(x)
    if pad:   # the same rows with leading dimension K + 64
        buf = torch.zeros(M, K + 64, dtype=torch.bfloat16, device="cuda")
        buf[:, :K] = xt
        xt = buf[:, :K]
    ncols = segs[0][1] if glu else sum(n for _, n in segs)
    y = empty_bf16(M, ncols)
    tf.tf_qmm_rows(xt, *W.t(), segs, y, epi=tf.TF_EPI_GLU if glu else 0)
    torch.cuda.synchronize()
    yb = host_bits(y)
    what = f"{route} case {i}: M={M} K={K} N={N} segs={segs} pad={pad}"
    if glu:
        F = segs[0][1]
        # The GPU's gate and up rows (the unfused calls) are held to V against the
        # oracle, and the fused result to the oracle's GLU of those same rows: the
        # GLU of bf16 values within V of the oracle's may round differently.
        g = empty_bf16(M, F)
        u = empty_bf16(M, F)
        tf.tf_qmm_rows(xt, *W.t(), [segs[0]], g)
        tf.tf_qmm_rows(xt, *W.t(), [segs[1]], u)
        torch.cuda.synchronize()
        for t, r0, part in ((g, 0, "gate"), (u, F, "up")):
            yo, y64, ad = orc.qmm_rows(x, *w.astuple(), np.arange(r0, r0 + F), nthreads=NT, want_f64=True)
            check_values(host_bits(t), yo, y64, ad, K, f"{what} {part} rows")
        check_values(yb, orc.glu(host_bits(g), host_bits(u)), what=what + " GLU")
        return
    cols = np.concatenate([np.arange(r0, r0 + n) for r0, n in segs])
    pos = np.arange(cols.size)
    if M * cols.size * K > 4e8:   # sample: 384 columns plus both ends of every segment
        rng = np.random.default_rng([7, i])
        ends, o = [], 0
        for _, n in segs:
            ends += [o, o + n - 1]
            o += n
        pos = np.unique(np.concatenate([rng.choice(cols.size, 384, replace=False), ends]))
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), cols[pos], nthreads=NT, want_f64=True)
    check_values(yb[:, pos], yo, y64, ad, K, what)


@pytest.mark.parametrize("i", range(CASES))
def test_random_fused_head(tf, orc, i):
    rng = np.random.default_rng([1437, i])
    M, K = int(rng.integers(1, 4)), int(rng.choice([512, 2048, 5120]))
    N = int(rng.integers(2, 9000))
    r0 = int(rng.integers(0, N - 1))
    n = int(rng.integers(1, N - r0 + 1))
    w = synth.make_weights(N, K, seed=3000 + i, tag=synth.TAG_HEAD)
    W = DevWeights(w)
    x = synth.make_x(M, K, seed=3000 + i)
    xt = dev(x)
    logits = empty_bf16(M, n)
    words = torch.full((M,), -1, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_qmm_argmax_scratch_bytes(M, n), dtype=torch.uint8, device="cuda")
    tf.tf_qmm_argmax_rows(xt, *W.t(), (r0, n), r0, logits, words, scratch)
    torch.cuda.synchronize()
    lb = host_bits(logits)
    what = f"fused head case {i}: M={M} K={K} rows {r0}..{r0 + n}"
    assert np.array_equal(host_bits(words), orc.argmax_rows(lb, r0)), what
    pos = np.arange(n) if M * n * K <= 4e8 else np.unique(np.concatenate([rng.choice(n, 384, replace=False), [0, n - 1]]))
    yo, y64, ad = orc.qmm_rows(x, *w.astuple(), r0 + pos, nthreads=NT, want_f64=True)
    check_values(lb[:, pos], yo, y64, ad, K, what)


@pytest.mark.parametrize("i", range(CASES))
def test_random_int8_head(tf, orc, i):
    """tf_qmm8_rows on random slices, K a multiple of 32 or not (the general kernel)."""
    rng = np.random.default_rng([27, i])
    M, K = int(rng.integers(1, 5)), int(rng.choice([512, 1000, 2048, 5120]))
    N = int(rng.integers(2, 6000))
    r0 = int(rng.integers(0, N - 1))
    n = int(rng.integers(1, N - r0 + 1))
    w = synth.make_weights8(N, K, seed=4000 + i)
    q8, sc = synth.weights8_to_device(w)
    x = synth.make_x(M, K, seed=4000 + i)
    y = empty_bf16(M, n)
    tf.tf_qmm8_rows(dev(x), q8, sc, [(r0, n)], y)
    torch.cuda.synchronize()
    pos = np.arange(n) if M * n * K <= 4e8 else np.unique(np.concatenate([rng.choice(n, 384, replace=False), [0, n - 1]]))
    yo, y64, ad = orc.qmm8_rows(x, w.q8, w.scales, r0 + pos, nthreads=NT, want_f64=True)
    check_values(host_bits(y)[:, pos], yo, y64, ad, K, f"int8 head case {i}: M={M} K={K} rows {r0}..{r0 + n}")


@pytest.mark.parametrize("i", range(CASES))
def test_random_argmax(tf, orc, i):
    """tf_argmax_rows on random logits with planted ties, signed zeros and
    non-finites: the words bit for bit against the oracle's scan."""
    rng = np.random.default_rng([33, i])
    M, n = int(rng.integers(1, 20)), int(rng.integers(1, 300000))
    v = planted_logits(rng, M, n)
    id_base = int(rng.integers(0, 2 ** 30))
    words = torch.empty(M, dtype=torch.int64, device="cuda")
    scratch = torch.empty(tf.tf_argmax_scratch_bytes(M, n), dtype=torch.uint8, device="cuda")
    tf.tf_argmax_rows(dev(v), id_base, words, scratch)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(words), orc.argmax_rows(v, id_base)), f"argmax case {i}: M={M} n={n}"


@pytest.mark.parametrize("i", range(CASES))
def test_random_seam(tf, orc, i):
    """A random row split of random logits into 1-4 parts: the gather of the
    parts, each part's argmax word and top two, the pick and the merged top two,
    all bit for bit against the oracle (PR #1433 step-1 body: stage, gather,
    pair_argmax, pair_pick)."""
    rng = np.random.default_rng([1432, i])
    M, n, nparts = int(rng.integers(1, 9)), int(rng.integers(4, 60000)), int(rng.integers(1, 5))
    v = planted_logits(rng, M, n)
    cuts = np.sort(rng.choice(np.arange(1, n), size=nparts - 1, replace=False)) if nparts > 1 else np.array([], int)
    bounds = [0, *cuts.tolist(), n]
    parts = [v[:, bounds[j]:bounds[j + 1]].copy() for j in range(nparts)]
    widths = [p.shape[1] for p in parts]
    dparts = [dev(p) for p in parts]
    dst = empty_bf16(M, n)
    tf.tf_gather_rows(dst, dparts, widths)
    words = torch.empty(nparts, M, dtype=torch.int64, device="cuda")
    tops = torch.empty(nparts, M, 2, dtype=torch.int64, device="cuda")
    for j, p in enumerate(dparts):
        w = torch.empty(M, dtype=torch.int64, device="cuda")
        scr = torch.empty(tf.tf_argmax_scratch_bytes(M, widths[j]), dtype=torch.uint8, device="cuda")
        tf.tf_argmax_rows(p, bounds[j], w, scr)
        words[j] = w
        t2 = torch.empty(M, 2, dtype=torch.int64, device="cuda")
        scr2 = torch.empty(tf.tf_top2_scratch_bytes(M, widths[j]), dtype=torch.uint8, device="cuda")
        tf.tf_top2_rows(p, bounds[j], t2, scr2)
        tops[j] = t2
    ids = torch.empty(M, dtype=torch.int32, device="cuda")
    tf.tf_pick(words, ids)
    merged = torch.empty(M, 2, dtype=torch.int64, device="cuda")
    tf.tf_top2_merge(tops, merged)
    torch.cuda.synchronize()
    what = f"seam case {i}: M={M} n={n} parts={widths}"
    assert np.array_equal(host_bits(dst), orc.gather_rows(parts, M)), what + " gather"
    o_words = np.stack([orc.argmax_rows(p, bounds[j]) for j, p in enumerate(parts)])
    o_tops = np.stack([orc.top2_rows(p, bounds[j]) for j, p in enumerate(parts)])
    assert np.array_equal(host_bits(words), o_words), what + " words"
    assert np.array_equal(host_bits(tops), o_tops), what + " top two"
    assert np.array_equal(host_bits(ids), orc.pick(o_words)), what + " pick"
    assert np.array_equal(host_bits(merged), orc.top2_merge(o_tops)), what + " merged top two"
    assert np.array_equal(orc.pick(o_words), orc.pick(orc.argmax_rows(v, 0)[None, :])), what + " split != whole"
