"""CPU oracle for the row-split int4 hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package.  The product (``row_split_int4_b200``)
never imports it and shares no code with it: the arithmetic lives in
``oracle.c`` (plain C, double precision), this module only marshals numpy
arrays into it and composes its primitives the way the pages compose the
seam (TensorFold PR #1433, step-1 and step-2 bodies):

* a projection's half h owns the contiguous output rows
  ``[h*N/2, (h+1)*N/2)`` and reduces them over the whole K;
* the fused gate-up keeps the member split: half h owns gate rows
  ``[h*F/2, +F/2)`` and the same rows of up (``F`` = 17,408 on the pages);
* the halves are joined by a pure copy (gather);
* the head takes the argmax of each half and picks between the two words.

Every function cites the passage it follows in ``oracle.c``.  Parity status of
each function is listed in ``PINS`` below; a function with no pin independent
of the oracle itself says "parity unpinned" there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FLAG = 0x80000000
SENTINEL = 0xFFFFFFFF
NAN_BF16 = 0x7FC0
TOP2_NONE = (0x7FFFFFFF << 32) | 0xFF800000   # "no second place" (a slice of one element)
GROUP = 64

# What pins each oracle function to something other than itself (tests that
# check it are in tests/test_oracle_*.py).
PINS = {
    "bf16_rne": "hand-picked halfway/overflow/subnormal cases; torch fp32->bf16 on fp32-exact inputs",
    "dequant": "closed forms q=0 -> b, q=15 -> 15s+b, s=0 -> b; hand-decoded bytes",
    "qmm_rows": "one-hot x; q=8,b=-8s rows give 0; constant-q closed form; numpy float64 dequant-then-matmul",
    "glu": "SiLU(0)=0; SiLU(u)-SiLU(-u)=u; SiLU(1) to 16 digits; large |u| limits",
    "gather_rows": "brute-force column bookkeeping; NaN fill of a missing part",
    "argmax_rows": "all 7^5 vectors over {-1,-0,+0,1,NaN,+Inf,-Inf} against a Python min(key=...) scan",
    "pick": "exhaustive flag x flag x {<,=,>} truth table; split-then-pick == whole on every split point",
    "half_rows": "the pages' spans 2,560/8,704/124,160 of 5,120/17,408/248,320",
    "top2_gap": "hand cases (ties give 0, n=1 gives inf)",
    "top2_rows": "hand cases (a tie keeps both ids, +-0 tie, one element has no second, NaN flags both); a numpy lexsort of every small row",
    "top2_merge": "merge of the slices' top two == top two of the whole row at every split point; the lowest flagged part wins",
    "qmm8_rows": "one-hot x; constant-code closed form; numpy float64 matmul; the sign of the codes",
    "residual_add": "exact sums bf16 cannot hold; the fp32 round-to-even tie; IEEE specials; numpy float32 addition",
    "embed_rows": "brute-force row lookup; bound refusals incl. the pages' 124,160-of-248,320 shard width; NaN rows past the bound",
    "end_to_end_on_real_weights": "parity unpinned: the pages print no numeric worked example",
}


def build(out: Optional[str] = None, plant: int = 0, quiet: bool = True) -> str:
    """Compile ``oracle.c`` with gcc (-O2, OpenMP, no fast-math).

    ``plant`` > 0 builds one of the deliberately broken variants listed at the
    top of ``oracle.c``; those are only for the planted-control tests."""
    out = out or _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", out, "-lm"]
    if plant:
        cmd.insert(1, f"-DORC_PLANT={int(plant)}")
    subprocess.run(cmd, check=True, capture_output=quiet)
    return out


def _need_build(path: str) -> bool:
    return (not os.path.exists(path)) or os.path.getmtime(path) < os.path.getmtime(_SRC)


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes view of one build of ``oracle.c``."""

    def __init__(self, path: str):
        self.path = path
        L = ctypes.CDLL(path)
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_bf16_rne.argtypes = [ctypes.c_double]
        L.orc_bf16_rne_array.restype = None
        L.orc_bf16_rne_array.argtypes = [_P, _P, _I64]
        L.orc_dequant.restype = ctypes.c_double
        L.orc_dequant.argtypes = [_P, _P, _P, _I32, _I64, _I64]
        L.orc_qmm_rows.restype = _I32
        L.orc_qmm_rows.argtypes = [_P, _I32, _I32, _I64, _P, _P, _P, _P, _I64, _P, _I64, _P, _P, _I32]
        L.orc_glu.restype = None
        L.orc_glu.argtypes = [_P, _P, _P, _P, _I64]
        L.orc_half_rows.restype = _I32
        L.orc_half_rows.argtypes = [_I32, _I32, _I64, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]
        L.orc_gather_rows.restype = None
        L.orc_gather_rows.argtypes = [_P, _I64, _P, _P, _I32, _I32]
        L.orc_argmax_rows.restype = _I32
        L.orc_argmax_rows.argtypes = [_P, _I32, _I64, _I64, ctypes.c_uint32, _P]
        L.orc_pick.restype = None
        L.orc_pick.argtypes = [_P, _I32, _I32, _P]
        L.orc_top2_rows.restype = _I32
        L.orc_top2_rows.argtypes = [_P, _I32, _I64, _I64, ctypes.c_uint32, _P]
        L.orc_top2_merge.restype = None
        L.orc_top2_merge.argtypes = [_P, _I32, _I32, _P]
        L.orc_top2_gap.restype = None
        L.orc_top2_gap.argtypes = [_P, _I32, _I64, _P]
        L.orc_qmm8_rows.restype = _I32
        L.orc_qmm8_rows.argtypes = [_P, _I32, _I32, _I64, _P, _P, _P, _I64, _P, _I64, _P, _P, _I32]
        L.orc_residual_add.restype = None
        L.orc_residual_add.argtypes = [_P, _P, _P, _I64]
        L.orc_embed_rows.restype = _I32
        L.orc_embed_rows.argtypes = [_P, _I64, _I64, _I64, _I64, _P, _I32, _P, _I64]
        self.L = L

    # -- scalar helpers ------------------------------------------------------
    def bf16_rne(self, v) -> np.ndarray:
        """double -> bf16 bits, RNE in one step (NaN -> 0x7FC0)."""
        shape = np.shape(v)
        a = np.ascontiguousarray(np.asarray(v, dtype=np.float64).reshape(-1))
        out = np.empty(a.shape, dtype=np.uint16)
        self.L.orc_bf16_rne_array(_ptr(a), _ptr(out), a.size)
        return out.reshape(shape)

    def dequant(self, wq, scales, biases, K: int, n: int, k: int) -> float:
        return self.L.orc_dequant(_ptr(wq), _ptr(scales), _ptr(biases), K, n, k)

    # -- qmm ------------------------------------------------------------------
    def qmm_rows(self, x: np.ndarray, wq: np.ndarray, scales: np.ndarray, biases: np.ndarray,
                 rows: Sequence[int], nthreads: int = 1, want_f64: bool = False):
        """bf16 outputs of the listed whole-matrix rows for every row of x.

        x: uint16 [M, K] bf16 bits; wq: uint8 [N, K/2]; scales/biases: uint16
        [N, K/64].  Returns y uint16 [M, len(rows)], plus (y64, absdot) double
        arrays when ``want_f64``."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        if x.ndim == 1:
            x = x[None, :]
        M, K = x.shape
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nr = rows.size
        assert wq.dtype == np.uint8 and wq.flags.c_contiguous and wq.shape[1] * 2 == K
        assert scales.dtype == np.uint16 and scales.flags.c_contiguous and scales.shape[1] * GROUP == K
        assert biases.dtype == np.uint16 and biases.flags.c_contiguous and biases.shape == scales.shape
        if nr:
            assert rows.min() >= 0 and rows.max() < wq.shape[0]
        y = np.empty((M, nr), dtype=np.uint16)
        y64 = np.empty((M, nr), dtype=np.float64) if want_f64 else None
        ad = np.empty((M, nr), dtype=np.float64) if want_f64 else None
        rc = self.L.orc_qmm_rows(_ptr(x), M, K, K, _ptr(wq), _ptr(scales), _ptr(biases),
                                 _ptr(rows), nr, _ptr(y), nr, _ptr(y64), _ptr(ad), int(nthreads))
        if rc != 0:
            raise ValueError("orc_qmm_rows: bad arguments")
        return (y, y64, ad) if want_f64 else y

    def glu(self, g: np.ndarray, u: np.ndarray, want_f64: bool = False):
        g = np.ascontiguousarray(g, dtype=np.uint16)
        u = np.ascontiguousarray(u, dtype=np.uint16)
        assert g.shape == u.shape
        a = np.empty(g.shape, dtype=np.uint16)
        a64 = np.empty(g.shape, dtype=np.float64) if want_f64 else None
        self.L.orc_glu(_ptr(g), _ptr(u), _ptr(a), _ptr(a64), g.size)
        return (a, a64) if want_f64 else a

    def qmm8_rows(self, x: np.ndarray, q8: np.ndarray, scales: np.ndarray, rows: Sequence[int],
                  nthreads: int = 1, want_f64: bool = False):
        """The int8 head: bf16 of s[n] * sum_k x q8[n,k] for the listed rows.
        q8: int8 [N, K]; scales: uint16 [N] bf16 bits."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        if x.ndim == 1:
            x = x[None, :]
        M, K = x.shape
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nr = rows.size
        assert q8.dtype == np.int8 and q8.flags.c_contiguous and q8.shape[1] == K
        assert scales.dtype == np.uint16 and scales.shape == (q8.shape[0],)
        if nr:
            assert rows.min() >= 0 and rows.max() < q8.shape[0]
        y = np.empty((M, nr), dtype=np.uint16)
        y64 = np.empty((M, nr), dtype=np.float64) if want_f64 else None
        ad = np.empty((M, nr), dtype=np.float64) if want_f64 else None
        rc = self.L.orc_qmm8_rows(_ptr(x), M, K, K, _ptr(q8), _ptr(np.ascontiguousarray(scales)), _ptr(rows), nr,
                                  _ptr(y), nr, _ptr(y64), _ptr(ad), int(nthreads))
        if rc != 0:
            raise ValueError("orc_qmm8_rows: bad arguments")
        return (y, y64, ad) if want_f64 else y

    # -- residual stream and embedding rows -----------------------------------
    def residual_add(self, h: np.ndarray, y: np.ndarray) -> np.ndarray:
        """fp32(h + y) elementwise: the fp32 residual stream plus a bf16 row."""
        h = np.ascontiguousarray(h, dtype=np.float32)
        y = np.ascontiguousarray(y, dtype=np.uint16)
        assert h.shape == y.shape
        out = np.empty_like(h)
        self.L.orc_residual_add(_ptr(h), _ptr(y), _ptr(out), h.size)
        return out

    def embed_rows(self, table: np.ndarray, ids: np.ndarray, bound: int) -> np.ndarray:
        """Rows of ``table`` (bf16 bits [rows, H]) for token ``ids``; an id at or
        past ``bound`` gives a NaN row.  ValueError when bound != rows."""
        table = np.ascontiguousarray(table, dtype=np.uint16)
        ids = np.ascontiguousarray(ids, dtype=np.uint32)
        rows, H = table.shape
        out = np.empty((ids.size, H), dtype=np.uint16)
        if self.L.orc_embed_rows(_ptr(table), rows, H, H, int(bound), _ptr(ids), ids.size, _ptr(out), H) != 0:
            raise ValueError("orc_embed_rows: the bound must be the whole table's row count")
        return out

    # -- split / gather -------------------------------------------------------
    def half_rows(self, h: int, nparts: int, N: int):
        r0, nr = _I64(), _I64()
        if self.L.orc_half_rows(h, nparts, N, ctypes.byref(r0), ctypes.byref(nr)) != 0:
            raise ValueError("orc_half_rows: N does not split evenly")
        return r0.value, nr.value

    def gather_rows(self, parts: Sequence[Optional[np.ndarray]], M: int,
                    widths: Optional[Sequence[int]] = None) -> np.ndarray:
        """Join dense parts [M, w_h] into [M, sum w_h]; a None part (its width
        given in ``widths``) reads as the bf16 NaN 0x7FC0."""
        if widths is None:
            widths = [p.shape[1] for p in parts]
        return self._gather(parts, np.asarray(widths, dtype=np.int64), M)

    def _gather(self, parts, widths, M):
        keep = [None if p is None else np.ascontiguousarray(p, dtype=np.uint16) for p in parts]
        for p, w in zip(keep, widths):
            if p is not None:
                assert p.shape == (M, w)
        ptrs = (ctypes.c_void_p * len(keep))(*[None if p is None else p.ctypes.data for p in keep])
        dst = np.empty((M, int(widths.sum())), dtype=np.uint16)
        self.L.orc_gather_rows(_ptr(dst), dst.shape[1], ctypes.cast(ptrs, ctypes.c_void_p),
                               _ptr(widths), len(keep), M)
        return dst

    # -- head -----------------------------------------------------------------
    def argmax_rows(self, v: np.ndarray, id_base: int = 0) -> np.ndarray:
        v = np.ascontiguousarray(v, dtype=np.uint16)
        if v.ndim == 1:
            v = v[None, :]
        M, n = v.shape
        words = np.empty(M, dtype=np.uint64)
        if self.L.orc_argmax_rows(_ptr(v), M, n, n, int(id_base), _ptr(words)) != 0:
            raise ValueError("orc_argmax_rows: n must be >= 1")
        return words

    def pick(self, words: np.ndarray) -> np.ndarray:
        """words: uint64 [nparts, M] -> uint32 ids [M]."""
        w = np.ascontiguousarray(words, dtype=np.uint64)
        if w.ndim == 1:
            w = w[:, None]
        nparts, M = w.shape
        ids = np.empty(M, dtype=np.uint32)
        self.L.orc_pick(_ptr(w), nparts, M, _ptr(ids))
        return ids

    def top2_rows(self, v: np.ndarray, id_base: int = 0) -> np.ndarray:
        """bf16 bits [M, n] -> uint64 words [M, 2]: the winner and the second place
        in the argmax order (oracle.c, merged top two)."""
        v = np.ascontiguousarray(v, dtype=np.uint16)
        if v.ndim == 1:
            v = v[None, :]
        M, n = v.shape
        words2 = np.empty((M, 2), dtype=np.uint64)
        if self.L.orc_top2_rows(_ptr(v), M, n, n, int(id_base), _ptr(words2)) != 0:
            raise ValueError("orc_top2_rows: n must be >= 1")
        return words2

    def top2_merge(self, words2: np.ndarray) -> np.ndarray:
        """uint64 [nparts, M, 2] -> uint64 [M, 2]: the merged top two."""
        w = np.ascontiguousarray(words2, dtype=np.uint64)
        if w.ndim == 2:
            w = w[None]
        nparts, M, _ = w.shape
        out = np.empty((M, 2), dtype=np.uint64)
        self.L.orc_top2_merge(_ptr(w), nparts, M, _ptr(out))
        return out

    def top2_gap(self, logits64: np.ndarray) -> np.ndarray:
        a = np.ascontiguousarray(logits64, dtype=np.float64)
        if a.ndim == 1:
            a = a[None, :]
        M, n = a.shape
        gap = np.empty(M, dtype=np.float64)
        self.L.orc_top2_gap(_ptr(a), M, n, _ptr(gap))
        return gap

    # -- compositions (the seam, as the pages compose it) ---------------------
    def split_rows(self, h: int, nparts: int, N: int) -> np.ndarray:
        r0, nr = self.half_rows(h, nparts, N)
        return np.arange(r0, r0 + nr, dtype=np.int64)

    def member_rows(self, h: int, nparts: int, F: int):
        """Fused gate-up [gate(F); up(F)]: half h owns the same rows of both members."""
        g = self.split_rows(h, nparts, F)
        return g, g + F

    def glu_rows(self, x, W, gate_rows, up_rows, nthreads=1):
        g = self.qmm_rows(x, *W, gate_rows, nthreads=nthreads)
        u = self.qmm_rows(x, *W, up_rows, nthreads=nthreads)
        return self.glu(g, u)

    def mlp_whole(self, x, Wgu, Wdown, nthreads=1):
        """act = glu(x . gate, x . up) over all F rows; y = act . down over all rows."""
        F = Wgu[0].shape[0] // 2
        rows = np.arange(F, dtype=np.int64)
        act = self.glu_rows(x, Wgu, rows, rows + F, nthreads)
        y = self.qmm_rows(act, *Wdown, np.arange(Wdown[0].shape[0]), nthreads=nthreads)
        return act, y

    def mlp_split(self, x, Wgu, Wdown, nparts=2, nthreads=1):
        """The same layer as nparts row halves joined by gathers."""
        F = Wgu[0].shape[0] // 2
        M = np.atleast_2d(x).shape[0]
        acts = [self.glu_rows(x, Wgu, *self.member_rows(h, nparts, F), nthreads) for h in range(nparts)]
        act = self.gather_rows(acts, M)
        ND = Wdown[0].shape[0]
        ys = [self.qmm_rows(act, *Wdown, self.split_rows(h, nparts, ND), nthreads=nthreads)
              for h in range(nparts)]
        return act, self.gather_rows(ys, M)

    def head_split(self, logits_parts: Sequence[np.ndarray], bases: Sequence[int]):
        """argmax per part (global ids from bases) then pick."""
        words = np.stack([self.argmax_rows(p, b) for p, b in zip(logits_parts, bases)])
        return words, self.pick(words)


_CACHE = {}


def load(plant: int = 0, path: Optional[str] = None) -> Oracle:
    """Build (when stale) and load the oracle.  ``plant`` builds a broken
    variant into a temporary directory for the planted-control tests."""
    key = (plant, path)
    if key in _CACHE:
        return _CACHE[key]
    if plant:
        d = tempfile.mkdtemp(prefix="orc_plant_")
        p = build(os.path.join(d, f"liboracle_plant{plant}.so"), plant=plant)
    else:
        p = path or _LIB
        if path is None and _need_build(p):
            build(p)
    o = Oracle(p)
    _CACHE[key] = o
    return o
