"""Prompt chunks and the M sweep at full size.

* M=128 bf16 rows through attn_out (5,120 x 5,120), gate+up (2 x 17,408, GLU)
  and down (17,408 -> 5,120); M=512 requested and capped into four 128-row
  chunks; each chunk's activated half frame fits 128 * 8,704 * 2 bytes.
* M in {1,2,4,8,16,32,64,128} over the four shapes (lm_head with argmax and
  pick).  Values are checked on sampled columns (all m): 4,096 random columns
  plus every position of the first and the last 128-row tile and the rows on
  either side of the half boundary; ids bit for bit against the oracle's
  argmax/pick on the GPU's own logits.
"""
import os

import numpy as np
import pytest
import torch

import synth
from gpu_util import DevWeights, bits_equal, check_values, dev, empty_bf16, host_bits, need_gpu
import head_pipeline as HP

pytestmark = pytest.mark.gpu
NT = os.cpu_count() or 1
SAMPLE = 4096
TILE = 128   # rows of one tensor-core tile


@pytest.fixture(scope="module")
def tf():
    need_gpu()
    import row_split_int4_b200 as tf
    return tf


@pytest.fixture(scope="module")
def W():
    H, F = synth.HIDDEN, synth.FFN
    w = {
        "attn_out": synth.make_weights(H, H, seed=0, tag=11),
        "gate_up": synth.make_weights(2 * F, H, seed=0, tag=synth.TAG_W),
        "down": synth.make_weights(H, F, seed=0, tag=synth.TAG_W2),
    }
    return {k: (v, DevWeights(v)) for k, v in w.items()}


@pytest.fixture(scope="module")
def W_head():
    w = synth.make_weights(synth.VOCAB, synth.HIDDEN, seed=0, tag=synth.TAG_HEAD)
    return w, DevWeights(w)


def sample_cols(n, seed=0):
    """4,096 random output columns of n, plus every position of the first and the
    last 128-row tile (a wrong row inside a tile shows there) and the two columns
    either side of the middle (the half boundary)."""
    rng = np.random.default_rng(seed)
    pick = rng.choice(n, min(SAMPLE, n), replace=False)
    forced = np.concatenate([np.arange(min(TILE, n)), np.arange(max(0, n - TILE), n),
                             [max(0, n // 2 - 1), n // 2]])
    return np.unique(np.concatenate([pick, forced]))


def sampled_check(orc, x_bits, w, y_bits, cols, K, what, seed=0):
    pick = sample_cols(len(cols), seed)
    yo, y64, ad = orc.qmm_rows(x_bits, *w.astuple(), np.asarray(cols)[pick], nthreads=NT, want_f64=True)
    return check_values(y_bits[:, pick], yo, y64, ad, K, what)


def chunked(tf, x_t, M_req):
    """The cap: a request of M_req rows runs as rounds of tf_chunk_rows(...) rows."""
    out, m0 = [], 0
    while m0 < M_req:
        c = tf.tf_chunk_rows(M_req - m0)
        out.append((m0, c))
        m0 += c
    return out


def test_prompt_chunk_m128(tf, orc, W):
    H, F = synth.HIDDEN, synth.FFN
    x = synth.make_x(512, H, seed=0, tag=21)
    xt = dev(x)
    rounds = chunked(tf, xt, 512)
    assert [c for _, c in rounds] == [128, 128, 128, 128]
    win = synth.WINDOW_BYTES
    assert tf.tf_seam_bytes(128, F // 2) <= win < tf.tf_seam_bytes(512, F // 2)
    wa, Wa = W["attn_out"]
    wgu, Wgu = W["gate_up"]
    wd, Wd = W["down"]
    y_attn = empty_bf16(512, H)
    act = empty_bf16(512, F)
    y_down = empty_bf16(512, H)
    for m0, c in rounds:
        xs = xt[m0:m0 + c]
        tf.tf_qmm_rows(xs, *Wa.t(), [(0, H)], y_attn[m0:m0 + c])
        halves = []
        for h in range(2):
            a = empty_bf16(c, F // 2)
            tf.tf_qmm_rows(xs, *Wgu.t(), tf.tf_member_segs(F, 2, h), a, epi=tf.TF_EPI_GLU)
            halves.append(a)
        tf.tf_gather_rows(act[m0:m0 + c], halves, [F // 2] * 2, window_bytes=win)
        ys = []
        for h in range(2):
            yh = empty_bf16(c, H // 2)
            tf.tf_qmm_rows(act[m0:m0 + c], *Wd.t(), [tf.tf_split_rows(H, 2, h)], yh)
            ys.append(yh)
        tf.tf_gather_rows(y_down[m0:m0 + c], ys, [H // 2] * 2, window_bytes=win)
    # an uncapped 512-row gather would not fit the window
    big = empty_bf16(512, F // 2)
    assert tf.tf_gather_rows(empty_bf16(512, F), [big, big], [F // 2] * 2, window_bytes=win,
                             check=False) == tf.TF_E_WINDOW
    torch.cuda.synchronize()

    # S: the whole path for one chunk, and a different chunking of the same rows
    act_w = empty_bf16(128, F)
    tf.tf_qmm_rows(xt[128:256], *Wgu.t(), [(0, F), (F, F)], act_w, epi=tf.TF_EPI_GLU)
    y_alt = empty_bf16(64, H)
    tf.tf_qmm_rows(xt[160:224], *Wa.t(), [(0, H)], y_alt)
    torch.cuda.synchronize()
    assert bits_equal(act_w, act[128:256]), "GLU frame: split chunk != whole chunk"
    assert bits_equal(y_alt, y_attn[160:224]), "a row's bits depend on its chunk"

    # V on sampled columns of every output (all 512 rows)
    xb = x
    sampled_check(orc, xb, wa, host_bits(y_attn), np.arange(H), H, "attn_out M=128")
    a_bits = host_bits(act)
    # GLU: g/u via the unfused rows of the first chunk
    g = empty_bf16(128, F)
    u = empty_bf16(128, F)
    tf.tf_qmm_rows(xt[:128], *Wgu.t(), [(0, F)], g)
    tf.tf_qmm_rows(xt[:128], *Wgu.t(), [(F, F)], u)
    torch.cuda.synchronize()
    sampled_check(orc, xb[:128], wgu, host_bits(g), np.arange(F), H, "gate M=128")
    check_values(a_bits[:128], orc.glu(host_bits(g), host_bits(u)), what="GLU stage M=128")
    sampled_check(orc, a_bits, wd, host_bits(y_down), np.arange(H), F, "down M=128")
    # one 128-row chunk of attn_out and of down at full width
    yo, y64, ad = orc.qmm_rows(xb[:128], *wa.astuple(), np.arange(H), nthreads=NT, want_f64=True)
    check_values(host_bits(y_attn)[:128], yo, y64, ad, H, "attn_out M=128, every column")
    yo, y64, ad = orc.qmm_rows(a_bits[:128], *wd.astuple(), np.arange(H), nthreads=NT, want_f64=True)
    check_values(host_bits(y_down)[:128], yo, y64, ad, F, "down M=128, every column")


SHAPES = ["attn_out", "gate_up", "down"]


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32, 64, 128])
def test_sweep_projections(tf, orc, W, M):
    for name in SHAPES:
        w, Wd = W[name]
        K = w.K
        x = synth.make_x(M, K, seed=M, tag=31)
        xt = dev(x)
        y = empty_bf16(M, w.N)
        tf.tf_qmm_rows(xt, *Wd.t(), [(0, w.N)], y)
        torch.cuda.synchronize()
        sampled_check(orc, x, w, host_bits(y), np.arange(w.N), K, f"{name} M={M}", seed=M)


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32, 64, 128])
def test_sweep_head(tf, orc, W_head, M):
    w, Wd = W_head
    V, H = synth.VOCAB, synth.HIDDEN
    x = synth.make_x(M, H, seed=M, tag=41)
    xt = dev(x)
    h = V // 2
    parts = []
    for p in range(2):
        o = empty_bf16(M, h)
        tf.tf_qmm_rows(xt, *Wd.t(), [tf.tf_split_rows(V, 2, p)], o)
        parts.append(o)
    words, ids = HP.gpu_head_words(tf, parts, [0, h])
    torch.cuda.synchronize()
    logits = np.concatenate([host_bits(p) for p in parts], axis=1)
    sampled_check(orc, x, w, logits, np.arange(V), H, f"lm_head M={M}", seed=M)
    o_words, o_ids = orc.head_split([logits[:, :h], logits[:, h:]], [0, h])
    assert np.array_equal(host_bits(words), o_words)
    assert np.array_equal(host_bits(ids), o_ids)
