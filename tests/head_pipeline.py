"""The head as the pages run it -- per-half qmm, per-half argmax, pick -- on
the GPU through the C ABI, with the checks against the oracle (used by the
tiny config and the full 248,320-row head)."""
from __future__ import annotations

import numpy as np
import torch

import synth
from gpu_util import bits_equal, check_values, dev, empty_bf16, host_bits


def gpu_logits(tf, x_rows: torch.Tensor, W, nparts: int = 2, whole: bool = False):
    """Per-row M=1 qmm calls: returns a list of half logits [M, V/nparts] (split) or one [M, V]."""
    M = x_rows.shape[0]
    V = W.N
    if whole:
        out = empty_bf16(M, V)
        for m in range(M):
            tf.tf_qmm_rows(x_rows[m:m + 1], *W.t(), [(0, V)], out[m:m + 1])
        return [out]
    outs = []
    for h in range(nparts):
        r0, n = tf.tf_split_rows(V, nparts, h)
        o = empty_bf16(M, n)
        for m in range(M):
            tf.tf_qmm_rows(x_rows[m:m + 1], *W.t(), [(r0, n)], o[m:m + 1])
        outs.append(o)
    return outs


def plant_parts(parts, plants):
    """Apply plants (synth.Plant, whole-vocab ids) to device logits parts in place."""
    host = np.concatenate([host_bits(p) for p in parts], axis=1)
    synth.apply_plants(host, plants)
    off = 0
    for p in parts:
        w = p.shape[1]
        p.copy_(dev(np.ascontiguousarray(host[:, off:off + w])))
        off += w
    return host


def gpu_head_words(tf, parts, bases):
    M = parts[0].shape[0]
    words = torch.empty(len(parts), M, dtype=torch.int64, device="cuda")
    for h, (p, b) in enumerate(zip(parts, bases)):
        scratch = torch.empty(tf.tf_argmax_scratch_bytes(M, p.shape[1]), dtype=torch.uint8, device="cuda")
        tf.tf_argmax_rows(p, b, words[h], scratch)
    ids = torch.empty(M, dtype=torch.int32, device="cuda")
    tf.tf_pick(words, ids)
    return words, ids


def check_head(tf, orc, x_bits: np.ndarray, w: "synth.QWeights", W, plants, nthreads: int = 1,
               gap_margin: float = 1e-2, value_sample: int | None = None, seed: int = 0):
    """Split head vs whole head vs oracle on M rows of x (bf16 bits [M, K]).

    Returns a dict of counts; raises AssertionError on any failed check."""
    M, K = x_bits.shape
    V = W.N
    xt = dev(x_bits)
    parts = gpu_logits(tf, xt, W, 2)
    whole = gpu_logits(tf, xt, W, whole=True)[0]
    torch.cuda.synchronize()
    # S on the logits: the halves are the whole's columns, bit for bit
    assert bits_equal(torch.cat(parts, dim=1), whole), "split logits != whole logits"

    # V on the (unplanted) logits, oracle on the same x
    rng = np.random.default_rng(seed)
    cols = np.arange(V) if value_sample is None else np.sort(rng.choice(V, value_sample, replace=False))
    y_o, y64, ad = orc.qmm_rows(x_bits, *w.astuple(), cols, nthreads=nthreads, want_f64=True)
    logits_host = np.concatenate([host_bits(p) for p in parts], axis=1)
    vstat = check_values(logits_host[:, cols], y_o, y64, ad, K, "head logits")

    # plants, on the split parts and on the whole logits alike
    planted = plant_parts(parts, plants)
    plant_parts([whole], plants)
    h = V // 2
    words, ids = gpu_head_words(tf, parts, [0, h])
    wwords, wids = gpu_head_words(tf, [whole], [0])
    torch.cuda.synchronize()
    g_words = host_bits(words)
    g_ids = host_bits(ids)

    # I-kernel: the oracle's argmax + pick on the GPU's own (planted) logits, bit for bit
    o_words, o_ids = orc.head_split([planted[:, :h], planted[:, h:]], [0, h])
    assert np.array_equal(g_words, o_words), f"argmax words differ: {g_words} vs {o_words}"
    assert np.array_equal(g_ids, o_ids), f"picked ids differ: {g_ids} vs {o_ids}"

    # S on words and ids: whole vocabulary (one word, nparts = 1) == split + pick
    w_ids = host_bits(wids)
    assert np.array_equal(w_ids, g_ids), "whole-vocab ids != split ids"
    w_words = host_bits(wwords)[0]
    for m in range(M):
        if g_ids[m] != 0xFFFFFFFF:
            winner = 0 if g_ids[m] < h else 1
            assert w_words[m] == g_words[winner, m], f"row {m}: whole word != winning half's word"
        else:
            assert (int(w_words[m]) >> 63) == 1, f"row {m}: whole word not flagged"

    # I-end-to-end: the oracle's own logits (same plants), ids where the fp64 gap > margin
    if value_sample is None:
        o_logits, o64 = y_o.copy(), y64
    else:
        o_logits, o64, _ = orc.qmm_rows(x_bits, *w.astuple(), np.arange(V), nthreads=nthreads, want_f64=True)
    synth.apply_plants(o_logits, plants)
    _, e2e_ids = orc.head_split([o_logits[:, :h], o_logits[:, h:]], [0, h])
    gap = orc.top2_gap(o64)
    planted_rows = {p.row for p in plants}
    gated = 0
    for m in range(M):
        if m in planted_rows or gap[m] > gap_margin:
            assert g_ids[m] == e2e_ids[m], f"row {m}: gpu id {g_ids[m]} != oracle id {e2e_ids[m]} (gap {gap[m]})"
        else:
            gated += 1
    return {"values": vstat, "gated_rows": gated, "ids": [int(i) for i in g_ids]}
