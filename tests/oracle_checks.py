"""Pins of the CPU oracle, written as plain check functions.

Each check takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with something fixed independently of it: a value the pages
print, a hand-worked case, a closed form, an invariant, brute force on tiny
inputs or an independent library routine.  ``test_oracle_pins.py`` runs them
on the real oracle; ``test_oracle_plants.py`` runs each on a deliberately
broken build and expects it to fail.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NAN = 0x7FC0


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32_bits(v: float) -> int:
    return int(np.array([v], dtype=np.float32).view(np.uint32)[0])


def bf16_val(bits: int) -> float:
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


def bf16_of(v: float) -> int:
    """bf16 bits of a value that is exactly representable (test constants only)."""
    b = f32_bits(v)
    assert b & 0xFFFF == 0, v
    return b >> 16


# ------------------------------------------------------------------ bf16 RNE

RNE_CASES = [
    # (value, expected bits, why)
    (1.0, 0x3F80, "exact"),
    (1.0 + 2.0 ** -8, 0x3F80, "halfway between 1 and 1+2^-7: ties to the even 1.0"),
    (1.0 + 3 * 2.0 ** -8, 0x3F82, "halfway between 1+2^-7 and 1+2^-6: ties to even 0x3F82"),
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81, "just above halfway rounds up (double keeps the 2^-40)"),
    (-(1.0 + 2.0 ** -8), 0xBF80, "sign symmetric"),
    (255.0 / 128.0 * 2.0 ** 127, 0x7F7F, "largest finite bf16"),
    (255.5 / 128.0 * 2.0 ** 127, 0x7F80, "halfway above the largest finite rounds to even = +Inf"),
    (255.25 / 128.0 * 2.0 ** 127, 0x7F7F, "below halfway stays finite"),
    (2.0 ** -133, 0x0001, "smallest subnormal"),
    (2.0 ** -134, 0x0000, "half the smallest subnormal ties to even 0"),
    (3 * 2.0 ** -134, 0x0002, "1.5 subnormal steps ties to even 2"),
    (127.5 * 2.0 ** -133, 0x0080, "subnormal rounding carries into the smallest normal"),
    (2.0 ** -126, 0x0080, "smallest normal"),
    (0.0, 0x0000, "+0"),
    (-0.0, 0x8000, "-0 keeps its sign"),
    (math.inf, 0x7F80, "+Inf"),
    (-math.inf, 0xFF80, "-Inf"),
    (math.nan, NAN, "NaN canonicalised to the pages' 0x7FC0"),
    (1e300, 0x7F80, "double far above bf16 range overflows"),
    (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81, "double rounding trap: through fp32 this would tie to 0x3F80"),
]


def check_bf16_rne_hand(o):
    for v, bits, why in RNE_CASES:
        got = int(o.bf16_rne(v))
        assert got == bits, f"bf16_rne({v!r}) = {got:#06x}, want {bits:#06x} ({why})"


def check_bf16_rne_vs_torch(o, n=200000, seed=1):
    """On fp32-exact inputs a one-step RNE from double equals torch's fp32->bf16."""
    rng = np.random.default_rng(seed)
    u = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    # add exact halfway patterns: low 16 bits = 0x8000
    halves = (u[: n // 4] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    hf = halves.view(np.float32)
    f = np.concatenate([f, hf[np.isfinite(hf)]])
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = o.bf16_rne(f.astype(np.float64))
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches vs torch, first {f[bad[0]]!r}: {got[bad[0]]:#x} vs {want[bad[0]]:#x}"


# ---------------------------------------------------------------- dequant/qmm

def _one_matrix(K, q, scale_bits, bias_bits):
    """A single-row matrix from explicit codes and per-group bf16 bits."""
    q = np.asarray(q, dtype=np.uint8).reshape(1, K)
    wq = synth.pack_nibbles(q)
    G = K // 64
    sc = np.array([scale_bits], dtype=np.uint16).reshape(1, G)
    bi = np.array([bias_bits], dtype=np.uint16).reshape(1, G)
    return wq, sc, bi


def check_hand_cases(o):
    """The hand-worked cases in tests/golden/hand_cases.json."""
    K = 64
    # ramp_ones
    q = np.arange(K) % 16
    wq, sc, bi = _one_matrix(K, q, [0x3F00], [0xBF80])
    x = np.full((1, K), 0x3F80, dtype=np.uint16)
    y = o.qmm_rows(x, wq, sc, bi, [0])
    assert int(y[0, 0]) == 0x4330, f"ramp_ones: {int(y[0,0]):#x}"
    # one_hot_k37 / one_hot_k100
    K = 128
    q = (3 * np.arange(K) + 1) % 16
    wq, sc, bi = _one_matrix(K, q, [0x3E80, 0x3C00], [0xBE00, 0x3D80])
    x = np.zeros((1, K), dtype=np.uint16)
    x[0, 37] = 0x3F80
    assert int(o.qmm_rows(x, wq, sc, bi, [0])[0, 0]) == 0xBE00, "one_hot_k37"
    x = np.zeros((1, K), dtype=np.uint16)
    x[0, 100] = 0x4000
    assert int(o.qmm_rows(x, wq, sc, bi, [0])[0, 0]) == 0x3EA8, "one_hot_k100"
    # byte_0x21: packed bytes written directly
    K = 64
    wq = np.zeros((1, 32), dtype=np.uint8)
    wq[0, 0] = 0x21
    sc = np.array([[0x3F80]], dtype=np.uint16)
    bi = np.array([[0x0000]], dtype=np.uint16)
    x = np.zeros((1, K), dtype=np.uint16)
    x[0, 0] = 0x3F80
    x[0, 1] = 0x4080
    assert int(o.qmm_rows(x, wq, sc, bi, [0])[0, 0]) == 0x4110, "byte_0x21 (nibble order)"
    # the golden file agrees with these constants
    g = {c["name"]: int(c["y_bits"], 16) for c in golden("hand_cases.json")["cases"]}
    assert g == {"ramp_ones": 0x4330, "one_hot_k37": 0xBE00, "one_hot_k100": 0x3EA8, "byte_0x21": 0x4110}


def check_dequant_closed_forms(o):
    K = 128
    rng = np.random.default_rng(5)
    for qv in (0, 15, 7):
        q = np.full(K, qv)
        s = [bf16_of(0.015625), bf16_of(0.75)]
        b = [bf16_of(-0.125), bf16_of(3.0)]
        wq, sc, bi = _one_matrix(K, q, s, b)
        for k in rng.integers(0, K, 8):
            g = int(k) // 64
            want = bf16_val(s[g]) * qv + bf16_val(b[g])
            got = o.dequant(wq, sc, bi, K, 0, int(k))
            assert got == want, f"q={qv} k={k}: {got} != {want}"
    # s = 0 leaves the bias alone whatever q is
    q = rng.integers(0, 16, K)
    wq, sc, bi = _one_matrix(K, q, [0, 0], [bf16_of(1.5), bf16_of(-2.0)])
    for k in range(K):
        assert o.dequant(wq, sc, bi, K, 0, k) == (1.5 if k < 64 else -2.0)


def check_one_hot(o, seed=2):
    """x = c * e_k gives y = bf16(c * w[n, k]) for every row: an exact product."""
    w = synth.make_weights(6, 256, seed=seed)
    q = np.zeros((6, 256), dtype=np.uint8)
    q[:, 0::2] = w.wq & 0xF
    q[:, 1::2] = w.wq >> 4
    s = synth.bf16_bits_to_f32(w.scales).astype(np.float64)
    b = synth.bf16_bits_to_f32(w.biases).astype(np.float64)
    for k in (0, 1, 63, 64, 130, 255):
        x = np.zeros((1, 256), dtype=np.uint16)
        x[0, k] = 0x4000   # 2.0
        y = o.qmm_rows(x, *w.astuple(), range(6))
        wk = s[:, k // 64] * q[:, k] + b[:, k // 64]
        w2 = 2.0 * wk
        exact = w2.astype(np.float32).astype(np.float64) == w2   # no double rounding through fp32
        assert exact.sum() >= 4
        want = synth.to_bf16_bits(w2.astype(np.float32))
        assert np.array_equal(y[0][exact], want[exact]), f"one-hot k={k}"


def check_zero_rows(o):
    """q = 8 everywhere and b = -8 s exactly gives w = 0, so y = +0 for any x."""
    K = 512
    G = K // 64
    s = np.array([bf16_of(2.0 ** -e) for e in range(3, 3 + G)], dtype=np.uint16)
    b = np.array([bf16_of(-8 * 2.0 ** -e) for e in range(3, 3 + G)], dtype=np.uint16)
    wq, sc, bi = _one_matrix(K, np.full(K, 8), s, b)
    x = synth.make_x(3, K, seed=4)
    y, y64, ad = o.qmm_rows(x, wq, sc, bi, [0], want_f64=True)
    assert np.all(y == 0) and np.all(y64 == 0.0) and np.all(ad == 0.0)


def check_constant_q(o):
    """Constant q per row: y = sum_g (s_g q + b_g) * X_g with X_g the group sums of x."""
    K, G = 1024, 16
    rng = np.random.default_rng(8)
    x = synth.make_x(2, K, seed=9)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    X = xf.reshape(2, G, 64).sum(axis=2)
    for qv in (0, 3, 15):
        s = synth.to_bf16_bits(rng.uniform(0.001, 0.02, G).astype(np.float32))
        b = synth.to_bf16_bits(rng.normal(0, 0.05, G).astype(np.float32))
        wq, sc, bi = _one_matrix(K, np.full(K, qv), s, b)
        _, y64, _ = o.qmm_rows(x, wq, sc, bi, [0], want_f64=True)
        w = synth.bf16_bits_to_f32(s).astype(np.float64) * qv + synth.bf16_bits_to_f32(b).astype(np.float64)
        want = X @ w
        assert np.allclose(y64[:, 0], want, rtol=1e-12, atol=1e-12), (qv, y64[:, 0], want)


def numpy_dequant(w: "synth.QWeights") -> np.ndarray:
    """Independent float64 dequantisation with numpy array ops."""
    N, K = w.N, w.K
    q = np.empty((N, K), dtype=np.float64)
    q[:, 0::2] = w.wq & 0xF
    q[:, 1::2] = w.wq >> 4
    s = np.repeat(synth.bf16_bits_to_f32(w.scales).astype(np.float64), 64, axis=1)
    b = np.repeat(synth.bf16_bits_to_f32(w.biases).astype(np.float64), 64, axis=1)
    return s * q + b


def check_vs_numpy_matmul(o, seed=3):
    w = synth.make_weights(40, 640, seed=seed)
    x = synth.make_x(3, 640, seed=seed)
    W = numpy_dequant(w)
    want = synth.bf16_bits_to_f32(x).astype(np.float64) @ W.T
    rows = np.arange(40)
    y, y64, ad = o.qmm_rows(x, *w.astuple(), rows, want_f64=True)
    assert np.allclose(y64, want, rtol=1e-12, atol=1e-13)
    assert np.all(ad >= np.abs(y64))
    # the bf16 outputs round the double results: within half a bf16 step of them
    yf = synth.bf16_bits_to_f32(y).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126))) - 7)
    assert np.all(np.abs(yf - want) <= 0.5 * ulp * (1 + 1e-9))


def check_rows_order_free(o, seed=6):
    """A row's output does not depend on which other rows are asked for, nor
    on their order, nor on the thread count."""
    w = synth.make_weights(64, 256, seed=seed)
    x = synth.make_x(2, 256, seed=seed)
    full = o.qmm_rows(x, *w.astuple(), np.arange(64))
    perm = np.random.default_rng(seed).permutation(64)
    part = o.qmm_rows(x, *w.astuple(), perm, nthreads=4)
    assert np.array_equal(full[:, perm], part)


# ------------------------------------------------------------------------ GLU

def check_glu(o):
    g = np.array([bf16_of(v) for v in (1.0, -3.0, 0.5, 1.0, 2.0, 0.0)], dtype=np.uint16)
    u = np.array([bf16_of(v) for v in (0.0, 0.0, 1.0, 2.0, 300.0, 5.0)], dtype=np.uint16)
    a, a64 = o.glu(g, u, want_f64=True)
    assert a64[0] == 0.0 and a64[1] == 0.0, "SiLU(0) = 0"
    # SiLU(1) = 1/(1+e^-1) = 0.7310585786300049; SiLU(2) = 2/(1+e^-2) = 1.7615941559557646
    assert abs(a64[2] - 0.5 * 0.7310585786300049) < 1e-15
    assert abs(a64[3] - 1.7615941559557646) < 1e-15
    assert a64[4] == 600.0, "SiLU(u) = u once exp(-u) is below half a double ulp"
    assert a64[5] == 0.0 and a[5] == 0
    # odd part: g*SiLU(u) - g*SiLU(-u) = g*u
    rng = np.random.default_rng(11)
    gv = synth.to_bf16_bits(rng.normal(0, 2, 256).astype(np.float32))
    uv = synth.to_bf16_bits(rng.normal(0, 3, 256).astype(np.float32))
    _, p = o.glu(gv, uv, want_f64=True)
    _, m = o.glu(gv, uv ^ np.uint16(0x8000), want_f64=True)
    gu = synth.bf16_bits_to_f32(gv).astype(np.float64) * synth.bf16_bits_to_f32(uv).astype(np.float64)
    assert np.allclose(p - m, gu, rtol=1e-13, atol=1e-300)


# -------------------------------------------------------------- split/gather

def check_spans(o):
    sp = golden("pages_constants.json")["spans"]
    for key in ("o_proj_down_out", "mlp_member", "lm_head"):
        whole, half = sp[key]["whole"], sp[key]["half"]
        assert o.half_rows(0, 2, whole) == (sp["rank0_start"], half)
        assert o.half_rows(1, 2, whole) == (half, half)


def check_gather(o):
    M = 3
    rng = np.random.default_rng(12)
    a = rng.integers(0, 2 ** 16, (M, 5), dtype=np.uint16)
    b = rng.integers(0, 2 ** 16, (M, 7), dtype=np.uint16)
    d = o.gather_rows([a, b], M)
    assert d.shape == (M, 12)
    for m in range(M):
        for j in range(12):
            assert d[m, j] == (a[m, j] if j < 5 else b[m, j - 5])
    d = o.gather_rows([a, None], M, widths=[5, 7])
    assert np.array_equal(d[:, :5], a) and np.all(d[:, 5:] == NAN)


def check_split_equals_whole_mlp(o, seed=13):
    """Row halves joined by gathers give the whole layer's bits."""
    F, H, K = 256, 128, 128
    Wgu = synth.make_weights(2 * F, K, seed=seed).astuple()
    Wd = synth.make_weights(H, F, seed=seed, tag=synth.TAG_W2).astuple()
    x = synth.make_x(2, K, seed=seed)
    a1, y1 = o.mlp_whole(x, Wgu, Wd)
    a2, y2 = o.mlp_split(x, Wgu, Wd)
    assert np.array_equal(a1, a2) and np.array_equal(y1, y2)


# --------------------------------------------------------------- argmax/pick

ALPHABET = [bf16_of(-1.0), 0x8000, 0x0000, bf16_of(1.0), 0x7FC0, 0x7F80, 0xFF80]


def ref_word(vals, base):
    """Reference argmax word by an independent route: min over (flag, -v, id)."""
    fv = [bf16_val(int(b)) for b in vals]
    nf = [j for j, v in enumerate(fv) if not math.isfinite(v)]
    if nf:
        return ((0x80000000 | (base + nf[0])) << 32) | 0x7FC00000
    j = min(range(len(fv)), key=lambda i: (-fv[i], i))
    return ((base + j) << 32) | (int(vals[j]) << 16)


def check_argmax_bruteforce(o):
    vecs = np.array(list(itertools.product(ALPHABET, repeat=5)), dtype=np.uint16)
    got = o.argmax_rows(vecs, 7)
    for i, v in enumerate(vecs):
        assert int(got[i]) == ref_word(v, 7), (v, hex(int(got[i])), hex(ref_word(v, 7)))


def ref_pick(words):
    if any((int(w) >> 32) & 0x80000000 for w in words):
        return 0xFFFFFFFF
    return min(((-bf16_val((int(w) & 0xFFFFFFFF) >> 16), int(w) >> 32) for w in words))[1]


def check_pick_truth_table(o):
    def word(flag, val, id_):
        if flag:
            return ((0x80000000 | id_) << 32) | 0x7FC00000
        return (id_ << 32) | (bf16_of(val) << 16)
    for fa, fb in itertools.product((0, 1), repeat=2):
        for rel in ("<", "=", ">"):
            va, vb = 1.0, {"<": 2.0, "=": 1.0, ">": 0.5}[rel]
            w = np.array([[word(fa, va, 10)], [word(fb, vb, 20)]], dtype=np.uint64)
            got = int(o.pick(w)[0])
            if fa or fb:
                want = 0xFFFFFFFF
            else:
                want = {"<": 20, "=": 10, ">": 10}[rel]
            assert got == want, (fa, fb, rel, hex(got))
    # +0 and -0 tie: the lower id wins in either order
    w = np.array([[word(0, 0.0, 3)], [(9 << 32) | (0x8000 << 16)]], dtype=np.uint64)
    assert int(o.pick(w)[0]) == 3
    w = np.array([[(3 << 32) | (0x8000 << 16)], [word(0, 0.0, 9)]], dtype=np.uint64)
    assert int(o.pick(w)[0]) == 3


def check_split_pick_equals_whole(o):
    """Every split point of every 5-vector: argmax per part + pick == whole argmax + pick."""
    vecs = np.array(list(itertools.product(ALPHABET, repeat=5)), dtype=np.uint16)
    whole = o.pick(o.argmax_rows(vecs, 0)[None, :])
    for cut in range(1, 5):
        w0 = o.argmax_rows(vecs[:, :cut], 0)
        w1 = o.argmax_rows(vecs[:, cut:], cut)
        split = o.pick(np.stack([w0, w1]))
        bad = np.nonzero(split != whole)[0]
        assert bad.size == 0, (cut, vecs[bad[0]], hex(int(split[bad[0]])), hex(int(whole[bad[0]])))
    for i, v in enumerate(vecs[::37]):
        assert int(whole[::37][i]) == ref_pick([ref_word(v, 0)])


def check_top2_gap(o):
    g = o.top2_gap(np.array([[1.0, 3.0, 2.5, 3.0], [0.0, -1.0, 5.0, 4.0]]))
    assert g[0] == 0.0 and g[1] == 1.0
    assert o.top2_gap(np.array([[2.0]]))[0] == math.inf


TOP2_NONE = (0x7FFFFFFF << 32) | 0xFF800000


def ref_top2(vals, base):
    """Reference top two by an independent route: sort the ids by (-value, id)."""
    fv = [bf16_val(int(b)) for b in vals]
    nf = [j for j, v in enumerate(fv) if not math.isfinite(v)]
    if nf:
        w = ((0x80000000 | (base + nf[0])) << 32) | 0x7FC00000
        return [w, w]
    order = sorted(range(len(fv)), key=lambda i: (-fv[i], i))
    words = [((base + j) << 32) | (int(vals[j]) << 16) for j in order[:2]]
    return words + [TOP2_NONE] * (2 - len(words))


def check_top2_hand(o):
    """Hand-worked rows: an exact tie keeps both ids (lower first), +0 ties -0,
    one element has no second place, and any non-finite value flags both words."""
    def w(id_, v):
        return (id_ << 32) | (bf16_of(v) << 16)
    rows = [([1.0, 3.0, 2.5, 3.0], [w(1, 3.0), w(3, 3.0)]),
            ([0.0, -1.0, 5.0, 4.0], [w(2, 5.0), w(3, 4.0)]),
            ([2.0, 1.0, 1.0, -4.0], [w(0, 2.0), w(1, 1.0)])]
    for vals, want in rows:
        got = o.top2_rows(np.array([bf16_of(v) for v in vals], dtype=np.uint16))
        assert [int(g) for g in got[0]] == want, (vals, [hex(int(g)) for g in got[0]])
    got = o.top2_rows(np.array([0x8000, 0x0000], dtype=np.uint16), 100)[0]
    assert [int(g) for g in got] == [(100 << 32) | 0x80000000, 101 << 32]
    got = o.top2_rows(np.array([bf16_of(7.0)], dtype=np.uint16), 5)[0]
    assert [int(g) for g in got] == [w(5, 7.0), TOP2_NONE]
    got = o.top2_rows(np.array([bf16_of(1.0), 0x7FC0, bf16_of(2.0), 0x7F80], dtype=np.uint16), 10)[0]
    flagged = ((0x80000000 | 11) << 32) | 0x7FC00000
    assert [int(g) for g in got] == [flagged, flagged]


def check_top2_bruteforce(o):
    """Every 5-vector over {-1, -0, +0, 1, NaN, +Inf, -Inf} and random shorter rows
    against the sort above; the winner equals the argmax word."""
    vecs = np.array(list(itertools.product(ALPHABET, repeat=5)), dtype=np.uint16)
    got = o.top2_rows(vecs, 3)
    for i in range(0, len(vecs), 7):
        assert [int(g) for g in got[i]] == ref_top2(vecs[i], 3), (vecs[i], [hex(int(g)) for g in got[i]])
    assert np.array_equal(got[:, 0], o.argmax_rows(vecs, 3))
    rng = np.random.default_rng(29)
    vals = [bf16_of(v) for v in (-2.0, -1.0, -0.0, 0.0, 0.5, 1.0, 3.0)]
    for n in (1, 2, 3, 4, 9):
        rows = rng.choice(vals, size=(64, n)).astype(np.uint16)
        got = o.top2_rows(rows, 40)
        for i in range(64):
            assert [int(g) for g in got[i]] == ref_top2(rows[i], 40), (rows[i], [hex(int(g)) for g in got[i]])


def check_top2_merge_split(o):
    """The merge of the slices' top two equals the top two of the whole row, at
    every split into two parts and at every split into three."""
    vecs = np.array(list(itertools.product(ALPHABET, repeat=5)), dtype=np.uint16)
    whole = o.top2_rows(vecs, 0)
    for cut in range(1, 5):
        parts = np.stack([o.top2_rows(vecs[:, :cut], 0), o.top2_rows(vecs[:, cut:], cut)])
        merged = o.top2_merge(parts)
        bad = np.nonzero((merged != whole).any(axis=1))[0]
        assert bad.size == 0, (cut, vecs[bad[0]], [hex(int(g)) for g in merged[bad[0]]])
    for c1, c2 in ((1, 3), (2, 4), (1, 2)):
        parts = np.stack([o.top2_rows(vecs[:, :c1], 0), o.top2_rows(vecs[:, c1:c2], c1),
                          o.top2_rows(vecs[:, c2:], c2)])
        assert np.array_equal(o.top2_merge(parts), whole), (c1, c2)


def check_qmm8(o, seed=23):
    """The int8 head y = bf16(s * sum x q8): one-hot x (an exact product), a
    constant code (closed form s * q * sum x), numpy's float64 matmul, and the
    sign of the codes (-128 and 127 at the ends of the range)."""
    rng = np.random.default_rng(seed)
    N, K = 6, 256
    w = synth.make_weights8(N, K, seed=seed)
    # one-hot x: y = bf16(s_n * c * q[n, k])
    for k in (0, 77, K - 1):
        x = np.zeros((1, K), np.uint16)
        x[0, k] = bf16_of(-1.5)
        y = o.qmm8_rows(x, w.q8, w.scales, range(N))
        # s * -1.5 * q is exact in fp32 (8 + 2 + 8 bits): torch's fp32 -> bf16 rounds it independently
        prod = np.array([synth.bf16_bits_to_f32(w.scales[n]).item() * -1.5 * int(w.q8[n, k]) for n in range(N)], np.float32)
        want = list(synth.to_bf16_bits(prod))
        assert list(y[0]) == want, (k, list(y[0]), want)
    # constant code: y = bf16(s * q * sum x)
    q = np.full((2, K), -128, np.int8)
    q[1] = 127
    sc = np.array([bf16_of(0.25), bf16_of(2.0 ** -7)], np.uint16)
    x = synth.to_bf16_bits(rng.standard_normal((3, K)).astype(np.float32))
    xs = synth.bf16_bits_to_f32(x).astype(np.float64).sum(axis=1)
    y = o.qmm8_rows(x, q, sc, [0, 1])
    # (the rounding of the closed form uses the oracle's bf16_rne, pinned on its own above)
    want = o.bf16_rne(np.stack([0.25 * -128 * xs, 2.0 ** -7 * 127 * xs], axis=1))
    assert np.array_equal(y, want)
    # numpy float64 matmul
    x = synth.to_bf16_bits(rng.standard_normal((4, K)).astype(np.float32))
    y, y64, _ = o.qmm8_rows(x, w.q8, w.scales, range(N), want_f64=True)
    ref = (synth.bf16_bits_to_f32(x).astype(np.float64) @ w.q8.astype(np.float64).T) * \
        synth.bf16_bits_to_f32(w.scales).astype(np.float64)[None, :]
    assert np.allclose(y64, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(y, o.bf16_rne(ref))


def check_residual_add(o, seed=21):
    """fp32(h + y) for an fp32 stream h and a bf16 row y (PR #1433 step-2 body:
    the gathered rows are added in the fp32 stream)."""
    f32 = np.float32
    # exact sums that bf16 could not hold: 1 + 2^-10 and a 24-bit result
    assert o.residual_add(np.array([1.0], f32), np.array([bf16_of(2.0 ** -10)], np.uint16))[0] == f32(1.0 + 2.0 ** -10)
    h = np.array([2.0 ** 23 + 1], f32)
    assert o.residual_add(h, np.array([bf16_of(1.0)], np.uint16))[0] == f32(2.0 ** 23 + 2)
    # a tie at fp32 precision rounds to even: (1 + 2^-23) + 2^-24 -> 1 + 2^-22
    r = o.residual_add(np.array([1.0 + 2.0 ** -23], f32), np.array([bf16_of(2.0 ** -24)], np.uint16))[0]
    assert r == f32(1.0 + 2.0 ** -22)
    # 1 + 2^-24 alone is the tie below, which rounds down to 1
    assert o.residual_add(np.array([1.0], f32), np.array([bf16_of(2.0 ** -24)], np.uint16))[0] == f32(1.0)
    # IEEE specials
    inf = float("inf")
    out = o.residual_add(np.array([inf, inf, 1.0, float("nan"), -0.0], f32),
                         np.array([bf16_of(1.0), 0xFF80, 0x7FC0, bf16_of(1.0), 0x8000], np.uint16))
    assert out[0] == inf and np.isnan(out[1]) and np.isnan(out[2]) and np.isnan(out[3])
    assert out[4] == 0.0 and np.signbit(out[4])   # -0 + -0 = -0
    # against numpy's IEEE float32 addition on random streams and rows
    rng = np.random.default_rng(seed)
    h = (rng.standard_normal(4096) * np.exp2(rng.integers(-20, 20, 4096))).astype(f32)
    y = synth.to_bf16_bits((rng.standard_normal(4096) * np.exp2(rng.integers(-30, 30, 4096))).astype(f32))
    want = h + synth.bf16_bits_to_f32(y)
    assert np.array_equal(o.residual_add(h, y).view(np.uint32), want.view(np.uint32))


def check_embed_rows(o, seed=22):
    """Rows of the whole table by token id; the bound is the whole table (the
    pages' fix: a bound below the table, e.g. the shard's 124,160 of 248,320,
    is refused), and an id at or past it gives a NaN row."""
    rng = np.random.default_rng(seed)
    rows, H = 64, 24
    table = rng.integers(0, 1 << 16, size=(rows, H), dtype=np.uint16)
    ids = np.array([0, 63, 5, 32, 31, 64, 1000, 0xFFFFFFFF], dtype=np.uint32)
    out = o.embed_rows(table, ids, rows)
    for m, i in enumerate(ids):
        want = table[i] if i < rows else np.full(H, NAN, np.uint16)
        assert np.array_equal(out[m], want), (m, int(i))
    for bad in (rows // 2, rows - 1, rows + 1):      # half the table: the shard-width bound
        try:
            o.embed_rows(table, ids, bad)
        except ValueError:
            continue
        raise AssertionError(f"bound {bad} of a {rows}-row table was accepted")
    # the pages' numbers: a 248,320-row table with the shard's 124,160 as the bound
    big = np.zeros((synth.VOCAB, 1), dtype=np.uint16)
    big[200000, 0] = 0x3F80
    got = o.embed_rows(big, np.array([200000], dtype=np.uint32), synth.VOCAB)
    assert got[0, 0] == 0x3F80
    try:
        o.embed_rows(big, np.array([200000], dtype=np.uint32), synth.VOCAB // 2)
        raise AssertionError("the shard width was accepted as the embedding bound")
    except ValueError:
        pass


ALL_CHECKS = [
    check_bf16_rne_hand, check_bf16_rne_vs_torch, check_hand_cases, check_dequant_closed_forms,
    check_one_hot, check_zero_rows, check_constant_q, check_vs_numpy_matmul, check_rows_order_free,
    check_glu, check_spans, check_gather, check_split_equals_whole_mlp, check_argmax_bruteforce,
    check_pick_truth_table, check_split_pick_equals_whole, check_top2_gap, check_residual_add, check_embed_rows, check_qmm8,
    check_top2_hand, check_top2_bruteforce, check_top2_merge_split,
]
