"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds none of the method's arithmetic: it only draws random
numbers, rounds them to bf16 with torch's own conversion (round to nearest
even) and packs 4-bit codes two to a byte in the layout both sides decode
independently (element k in byte k/2, low nibble for even k).

Recipe (the configs' distributions; numpy PCG64):
  * every tensor has its own generator ``default_rng([seed, tag])``;
  * a weight matrix [N, K] is drawn in row blocks of ``BLOCK_ROWS`` rows, and
    within each block in this order:
      q      ~ integers(0, 16)                 uint8 [rows, K]
      scale  ~ uniform(0.001, 0.02)            -> bf16  [rows, K/64]
      noise  ~ normal(0, 1e-3)                          [rows, K/64]
      bias   = bf16(-8 * float(scale_bf16) + noise)  (computed in float32)
  * an activation [M, K] is ``standard_normal`` -> bf16.
The same bytes go to the oracle (numpy) and to the GPU (torch tensors).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

GROUP = 64
BLOCK_ROWS = 8192

# generator tags, one per tensor role
TAG_W = 1
TAG_X = 2
TAG_W2 = 3
TAG_HEAD = 4
TAG_ATTN = 6
TAG_HEAD8 = 7


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 bf16 bit patterns (torch's RNE conversion)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """uint8 codes [N, K] (0..15) -> packed bytes [N, K/2], even k in the low nibble."""
    q = np.asarray(q, dtype=np.uint8)
    return np.ascontiguousarray(q[:, 0::2] | (q[:, 1::2] << 4))


@dataclass
class QWeights:
    """A 4-bit affine group-64 matrix: packed codes plus bf16 scale and bias bits."""
    wq: np.ndarray      # uint8  [N, K/2]
    scales: np.ndarray  # uint16 [N, K/64]
    biases: np.ndarray  # uint16 [N, K/64]

    @property
    def N(self) -> int:
        return self.wq.shape[0]

    @property
    def K(self) -> int:
        return self.wq.shape[1] * 2

    def astuple(self):
        return (self.wq, self.scales, self.biases)

    def nbytes(self) -> int:
        return self.wq.nbytes + self.scales.nbytes + self.biases.nbytes


def make_weights(N: int, K: int, seed: int = 0, tag: int = TAG_W) -> QWeights:
    assert K % GROUP == 0 and K > 0
    rng = np.random.default_rng([seed, tag])
    G = K // GROUP
    wq = np.empty((N, K // 2), dtype=np.uint8)
    sc = np.empty((N, G), dtype=np.uint16)
    bi = np.empty((N, G), dtype=np.uint16)
    for r0 in range(0, N, BLOCK_ROWS):
        r1 = min(N, r0 + BLOCK_ROWS)
        q = rng.integers(0, 16, size=(r1 - r0, K), dtype=np.uint8)
        s = to_bf16_bits(rng.uniform(0.001, 0.02, size=(r1 - r0, G)).astype(np.float32))
        noise = rng.normal(0.0, 1e-3, size=(r1 - r0, G)).astype(np.float32)
        b = to_bf16_bits(np.float32(-8.0) * bf16_bits_to_f32(s) + noise)
        wq[r0:r1] = pack_nibbles(q)
        sc[r0:r1] = s
        bi[r0:r1] = b
    return QWeights(wq, sc, bi)


@dataclass
class Q8Weights:
    """An int8 matrix with one bf16 scale per row (the int8 head)."""
    q8: np.ndarray      # int8   [N, K]
    scales: np.ndarray  # uint16 [N]

    @property
    def N(self) -> int:
        return self.q8.shape[0]

    @property
    def K(self) -> int:
        return self.q8.shape[1]

    def astuple(self):
        return (self.q8, self.scales)


def make_weights8(N: int, K: int, seed: int = 0, tag: int = TAG_HEAD8) -> Q8Weights:
    """Symmetric int8 codes, uniform over [-127, 127], and a bf16 row scale
    uniform over [1e-4, 2e-4] (|w| up to ~0.025, the 4-bit head's range)."""
    rng = np.random.default_rng([seed, tag])
    q8 = np.empty((N, K), dtype=np.int8)
    for r0 in range(0, N, BLOCK_ROWS):
        r1 = min(N, r0 + BLOCK_ROWS)
        q8[r0:r1] = rng.integers(-127, 128, size=(r1 - r0, K), dtype=np.int8)
    sc = to_bf16_bits(rng.uniform(1e-4, 2e-4, size=N).astype(np.float32))
    return Q8Weights(q8, sc)


def weights8_to_device(w: Q8Weights, device="cuda"):
    return (torch.from_numpy(w.q8).to(device), to_device(w.scales, device))


def make_x(M: int, K: int, seed: int = 0, tag: int = TAG_X) -> np.ndarray:
    rng = np.random.default_rng([seed, tag])
    return to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))


def to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy array -> torch tensor on ``device`` holding the same bytes."""
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    elif a.dtype == np.uint64:
        t = torch.from_numpy(a.view(np.int64))
    elif a.dtype == np.uint32:
        t = torch.from_numpy(a.view(np.int32))
    else:
        t = torch.from_numpy(a)
    return t.to(device)


def weights_to_device(w: QWeights, device="cuda"):
    return tuple(to_device(a, device) for a in w.astuple())


def bits_of(t: torch.Tensor) -> np.ndarray:
    """torch bf16 / int tensor -> numpy bit patterns (uint16 for bf16)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.int64:
        return t.numpy().view(np.uint64)
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    return t.numpy()


# ------------------------------------------------------------------ workloads
# Shapes of the pages' 27B model (TensorFold PR #1433, step-2 body: 5,120
# hidden, 17,408 MLP rows, 248,320 vocab) and of the tiny CPU-seconds case.

HIDDEN = 5120
FFN = 17408
VOCAB = 248320
TINY_K, TINY_N = 1024, 512
TINY_HEAD_K, TINY_VOCAB = 512, 4096
BATCH_ROWS = 128
WINDOW_BYTES = BATCH_ROWS * (FFN // 2) * 2   # 2,228,224 B per half


@dataclass
class Plant:
    """Edits planted into bf16 logits between the qmm and the argmax."""
    row: int
    kind: str          # "tie", "nan", "inf", "allequal"
    ids: tuple = ()
    value_bits: int = 0


def tiny_head_plants(vocab: int = TINY_VOCAB):
    """Eight logit rows: rows 0-2 get an exact cross-half tie (ids i < vocab/2
    <= j, the expected winner is i), row 3 gets one NaN; rows 4-7 stay natural."""
    h = vocab // 2
    rng = np.random.default_rng([0, 99])
    plants = []
    for r in range(3):
        i = int(rng.integers(0, h))
        j = int(rng.integers(h, vocab))
        plants.append(Plant(r, "tie", (i, j)))
    plants.append(Plant(3, "nan", (int(rng.integers(0, vocab)),), 0x7FC0))
    return plants


def head_plants(vocab: int = VOCAB):
    """Sixteen rows: row 0 a tie straddling the half boundary (ids h-1 and h),
    row 1 one +Inf, row 2 one NaN, row 3 all-equal; rows 4-15 natural."""
    h = vocab // 2
    rng = np.random.default_rng([0, 98])
    return [Plant(0, "tie", (h - 1, h)),
            Plant(1, "inf", (int(rng.integers(0, vocab)),), 0x7F80),
            Plant(2, "nan", (int(rng.integers(0, vocab)),), 0x7FC0),
            Plant(3, "allequal", (), 0x3F80)]


def apply_plants(logits_bits: np.ndarray, plants, bump_bits: int | None = None) -> np.ndarray:
    """Apply plants to a bf16 logits array [rows, vocab] in place (bit edits only).

    A tie sets both ids to a value above the row's finite maximum: the next
    bf16 above it, so the two planted ids are the row's only maximum."""
    for p in plants:
        row = logits_bits[p.row]
        if p.kind == "tie":
            f = bf16_bits_to_f32(row)
            m = np.nanmax(np.where(np.isfinite(f), f, -np.inf))
            top = to_bf16_bits(np.array([m], dtype=np.float32))[0]
            top = int(top) + 1 if m >= 0 else int(top) - 1   # one bf16 step above
            for i in p.ids:
                row[i] = top
        elif p.kind in ("nan", "inf"):
            for i in p.ids:
                row[i] = p.value_bits
        elif p.kind == "allequal":
            row[:] = p.value_bits
    return logits_bits


# ------------------------------------------------------------ wide-range inputs
# Activations whose 32-value runs (the 32 consecutive k starting at a multiple of
# 32) each hold one large value and 31 small ones, and weights that give the
# large values a weight of exactly zero, so that the output is made of the small
# values alone.  A kernel that keeps the small values only to the precision of
# the run's largest one, or that lets the large value's cancelled product swamp
# them, misses the fp32 accuracy the method asks for.

def wide_positions(K: int, seed: int = 0, tag: int = 11) -> np.ndarray:
    """One position per 32-value run of K: the k of its large value."""
    assert K % 32 == 0
    rng = np.random.default_rng([seed, tag])
    return np.arange(0, K, 32) + rng.integers(0, 32, size=K // 32)


def make_x_wide(M: int, K: int, big_exp: int = 10, small_exp=(-14, -10), seed: int = 0, tag: int = 12,
                positions: np.ndarray | None = None) -> np.ndarray:
    """[M, K] bf16 bits: at every position of ``positions`` (default
    ``wide_positions(K, seed)``) +-2^big_exp; elsewhere +-2^u * (1 + f) with u
    uniform over the integers of [small_exp[0], small_exp[1]] and f uniform in
    [0, 1), random signs."""
    rng = np.random.default_rng([seed, tag])
    pos = wide_positions(K, seed) if positions is None else positions
    u = rng.integers(small_exp[0], small_exp[1] + 1, size=(M, K))
    f = rng.uniform(0.0, 1.0, size=(M, K))
    sgn = np.where(rng.integers(0, 2, size=(M, K)) == 1, -1.0, 1.0)
    v = sgn * np.ldexp(1.0 + f, u)
    big_sgn = np.where(rng.integers(0, 2, size=(M, len(pos))) == 1, -1.0, 1.0)
    v[:, pos] = big_sgn * 2.0 ** big_exp
    return to_bf16_bits(v.astype(np.float32))


def with_zero_weights(w: QWeights, positions: np.ndarray, offset: int = 8) -> QWeights:
    """A copy of ``w`` whose weights at columns ``positions`` are exactly zero in
    every row: code ``offset`` there and, in every group holding such a column,
    bias = -offset * scale (exact in bf16 for offset 8, a power of two; for
    other offsets the scale is rounded to 4 significant bits first, so that
    offset * scale still fits bf16)."""
    q = np.empty((w.N, w.K), dtype=np.uint8)
    q[:, 0::2] = w.wq & 0x0F
    q[:, 1::2] = w.wq >> 4
    q[:, positions] = offset
    sc = w.scales.copy()
    bi = w.biases.copy()
    groups = np.unique(np.asarray(positions) // GROUP)
    if offset & (offset - 1):
        sc[:, groups] &= 0xFFF0   # 4 significant bits: offset * scale is exact
    bi[:, groups] = to_bf16_bits(np.float32(-offset) * bf16_bits_to_f32(sc[:, groups]))
    assert np.array_equal(bf16_bits_to_f32(bi[:, groups]).astype(np.float64),
                          -offset * bf16_bits_to_f32(sc[:, groups]).astype(np.float64))
    return QWeights(pack_nibbles(q), sc, bi)


def with_zero_weights8(w: Q8Weights, positions: np.ndarray) -> Q8Weights:
    """A copy of the int8 matrix with code 0 at columns ``positions``."""
    q8 = w.q8.copy()
    q8[:, positions] = 0
    return Q8Weights(q8, w.scales.copy())
