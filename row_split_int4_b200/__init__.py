"""row_split_int4_b200 -- Python binding of libtf.so, the row-split int4 hot
path on one B200 (see include/tf.h for the C ABI).

The functions here carry the C entry points' names and only marshal
arguments: tensors become device pointers, shapes and strides become sizes
and leading dimensions, and the current torch stream becomes the stream.
Every step of the computation runs in the library's CUDA kernels.  If
libtf.so is missing the import fails; there is no other implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtf.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python row_split_int4_b200/build.py` "
                      "(or __graft_entry__.build()); this package has no other implementation")

lib = ctypes.CDLL(LIB_PATH)

TF_OK, TF_E_ARG, TF_E_RANGE, TF_E_ALIGN, TF_E_WINDOW, TF_E_BROKEN, TF_E_CUDA, TF_E_UNIMPL = range(8)
TF_PAIR_FLAG = 0x80000000
TF_PICK_FAILED = 0xFFFFFFFF
TF_TOP2_NONE = (0x7FFFFFFF << 32) | 0xFF800000   # no second place (a one-element slice)
TF_NAN_BF16 = 0x7FC0
TF_BATCH_ROWS = 128
TF_GROUP = 64
TF_MAX_K = 65536
TF_MAX_SEGS = 8
TF_MAX_PARTS = 8
TF_NO_WINDOW = ctypes.c_size_t(-1).value
TF_STATIC_SCRATCH_BYTES = 64 * 1024
TF_EPI_NONE, TF_EPI_GLU = 0, 1

EXPORTS = ["tf_qmm_rows", "tf_gather_rows", "tf_argmax_scratch_bytes", "tf_argmax_rows", "tf_pick",
           "tf_split_rows", "tf_member_segs", "tf_chunk_rows", "tf_seam_bytes", "tf_status_str", "tf_last_cuda_error",
           "tf_abi_version", "tf_argmax_rows_static", "tf_qmm_argmax_rows", "tf_qmm_argmax_scratch_bytes",
           "tf_residual_add", "tf_embed_rows", "tf_qmm8_rows", "tf_top2_scratch_bytes", "tf_top2_rows", "tf_top2_merge"]


class tf_seg(ctypes.Structure):
    _fields_ = [("row0", ctypes.c_int32), ("nrows", ctypes.c_int32)]


_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
lib.tf_qmm_rows.restype = _i
lib.tf_qmm_rows.argtypes = [_vp, _i, _i, _i, _vp, _vp, _vp, _i, ctypes.POINTER(tf_seg), _i, _i, _vp, _i, _vp]
lib.tf_gather_rows.restype = _i
lib.tf_gather_rows.argtypes = [_vp, _i, ctypes.POINTER(_vp), ctypes.POINTER(_i), _i, _i, _sz, _vp]
lib.tf_argmax_scratch_bytes.restype = _sz
lib.tf_argmax_scratch_bytes.argtypes = [_i, _i]
lib.tf_argmax_rows.restype = _i
lib.tf_argmax_rows.argtypes = [_vp, _i, _i, _i, ctypes.c_uint32, _vp, _vp, _sz, _vp]
lib.tf_top2_scratch_bytes.restype = _sz
lib.tf_top2_scratch_bytes.argtypes = [_i, _i]
lib.tf_top2_rows.restype = _i
lib.tf_top2_rows.argtypes = [_vp, _i, _i, _i, ctypes.c_uint32, _vp, _vp, _sz, _vp]
lib.tf_top2_merge.restype = _i
lib.tf_top2_merge.argtypes = [_vp, _i, _i, _vp, _vp]
lib.tf_qmm_argmax_scratch_bytes.restype = _sz
lib.tf_qmm_argmax_scratch_bytes.argtypes = [_i, _i]
lib.tf_qmm_argmax_rows.restype = _i
lib.tf_qmm_argmax_rows.argtypes = [_vp, _i, _i, _i, _vp, _vp, _vp, _i, tf_seg, ctypes.c_uint32, _vp, _i, _vp, _vp, _sz,
                                   _vp]
lib.tf_qmm8_rows.restype = _i
lib.tf_qmm8_rows.argtypes = [_vp, _i, _i, _i, _vp, _vp, _i, ctypes.POINTER(tf_seg), _i, _vp, _i, _vp]
lib.tf_residual_add.restype = _i
lib.tf_residual_add.argtypes = [_vp, _i, _vp, _i, _i, _i, _vp]
lib.tf_embed_rows.restype = _i
lib.tf_embed_rows.argtypes = [_vp, _i, _i, _i, _i, _vp, _i, _vp, _i, _vp]
lib.tf_argmax_rows_static.restype = _i
lib.tf_argmax_rows_static.argtypes = [_vp, _i, _i, _i, ctypes.c_uint32, _vp, _vp]
lib.tf_pick.restype = _i
lib.tf_pick.argtypes = [_vp, _i, _i, _vp, _vp]
lib.tf_split_rows.restype = _i
lib.tf_split_rows.argtypes = [_i, _i, _i, ctypes.POINTER(tf_seg)]
lib.tf_member_segs.restype = _i
lib.tf_member_segs.argtypes = [_i, _i, _i, ctypes.POINTER(tf_seg)]
lib.tf_chunk_rows.restype = _i
lib.tf_chunk_rows.argtypes = [_i]
lib.tf_seam_bytes.restype = _sz
lib.tf_seam_bytes.argtypes = [_i, _i]
lib.tf_status_str.restype = ctypes.c_char_p
lib.tf_status_str.argtypes = [_i]
lib.tf_last_cuda_error.restype = ctypes.c_char_p
lib.tf_last_cuda_error.argtypes = []
lib.tf_abi_version.restype = _i
lib.tf_abi_version.argtypes = []


class TFError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {tf_status_str(status)}"
        if status == TF_E_CUDA:
            msg += f" ({tf_last_cuda_error()})"
        super().__init__(msg)


def tf_status_str(status: int) -> str:
    return lib.tf_status_str(int(status)).decode()


def tf_last_cuda_error() -> str:
    """The CUDA runtime's message behind the last TF_E_CUDA on this thread."""
    return lib.tf_last_cuda_error().decode()


def tf_split_rows(N: int, nparts: int, h: int) -> Tuple[int, int]:
    """(row0, nrows) of the rows part h of nparts owns in an N-row matrix."""
    seg = tf_seg()
    st = lib.tf_split_rows(int(N), int(nparts), int(h), ctypes.byref(seg))
    _ret(st, "tf_split_rows", True)
    return seg.row0, seg.nrows


def tf_member_segs(F: int, nparts: int, h: int):
    """[(gate row0, n), (up row0, n)] that part h owns in a fused [gate(F); up(F)] stack."""
    segs = (tf_seg * 2)()
    st = lib.tf_member_segs(int(F), int(nparts), int(h), segs)
    _ret(st, "tf_member_segs", True)
    return [(segs[0].row0, segs[0].nrows), (segs[1].row0, segs[1].nrows)]


def tf_chunk_rows(requested: int) -> int:
    return lib.tf_chunk_rows(int(requested))


def tf_seam_bytes(rows: int, width: int) -> int:
    return lib.tf_seam_bytes(int(rows), int(width))


def tf_argmax_scratch_bytes(M: int, n: int) -> int:
    return lib.tf_argmax_scratch_bytes(int(M), int(n))


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream or None
    return int(stream) or None


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else (t.data_ptr() or None)


def _ld(t: torch.Tensor) -> int:
    assert t.dim() == 2 and (t.stride(1) == 1 or t.shape[1] <= 1), "rows must be contiguous"
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


def _ret(status: int, where: str, check: bool) -> int:
    if check and status != TF_OK:
        raise TFError(status, where)
    return status


def tf_qmm_rows(x: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                segs: Sequence[Tuple[int, int]], y: torch.Tensor, epi: int = TF_EPI_NONE,
                stream=None, check: bool = True) -> int:
    """y[M, cols] = the bf16 qmm outputs of the listed whole-matrix rows
    (``segs`` = [(row0, nrows), ...]); see tf.h for TF_EPI_GLU."""
    assert x.dtype == torch.bfloat16 and y.dtype == torch.bfloat16
    assert wq.dtype == torch.uint8 and scales.dtype == torch.bfloat16 and biases.dtype == torch.bfloat16
    arr = (tf_seg * max(1, len(segs)))(*[tf_seg(int(r0), int(n)) for r0, n in segs])
    st = lib.tf_qmm_rows(_ptr(x), x.shape[0], x.shape[1], _ld(x), _ptr(wq), _ptr(scales), _ptr(biases),
                         wq.shape[0], arr, len(segs), int(epi), _ptr(y), _ld(y), _stream(stream))
    return _ret(st, "tf_qmm_rows", check)


def tf_qmm8_rows(x: torch.Tensor, q8: torch.Tensor, scales: torch.Tensor, segs: Sequence[Tuple[int, int]],
                 y: torch.Tensor, stream=None, check: bool = True) -> int:
    """The int8 head: y[M, cols] = bf16(s[n] * x . q8[n]) for the listed rows."""
    assert x.dtype == torch.bfloat16 and y.dtype == torch.bfloat16
    assert q8.dtype == torch.int8 and scales.dtype == torch.bfloat16 and q8.is_contiguous()
    arr = (tf_seg * max(1, len(segs)))(*[tf_seg(int(r0), int(n)) for r0, n in segs])
    st = lib.tf_qmm8_rows(_ptr(x), x.shape[0], x.shape[1], _ld(x), _ptr(q8), _ptr(scales), q8.shape[0], arr,
                          len(segs), _ptr(y), _ld(y), _stream(stream))
    return _ret(st, "tf_qmm8_rows", check)


def tf_qmm_argmax_scratch_bytes(M: int, nrows: int) -> int:
    return lib.tf_qmm_argmax_scratch_bytes(int(M), int(nrows))


def tf_qmm_argmax_rows(x: torch.Tensor, wq: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                       seg: Tuple[int, int], id_base: int, logits: torch.Tensor, words: torch.Tensor,
                       scratch: torch.Tensor, stream=None, check: bool = True) -> int:
    """logits[M, nrows] = the qmm rows of ``seg`` = (row0, nrows) and words[M] their
    argmax words (ids id_base + j), in one call; see tf.h."""
    assert x.dtype == torch.bfloat16 and logits.dtype == torch.bfloat16
    assert wq.dtype == torch.uint8 and scales.dtype == torch.bfloat16 and biases.dtype == torch.bfloat16
    assert words.dtype == torch.int64 and scratch.dtype == torch.uint8
    st = lib.tf_qmm_argmax_rows(_ptr(x), x.shape[0], x.shape[1], _ld(x), _ptr(wq), _ptr(scales), _ptr(biases),
                                wq.shape[0], tf_seg(int(seg[0]), int(seg[1])), int(id_base), _ptr(logits),
                                _ld(logits), _ptr(words), _ptr(scratch), scratch.numel(), _stream(stream))
    return _ret(st, "tf_qmm_argmax_rows", check)


def tf_residual_add(h: torch.Tensor, y: torch.Tensor, stream=None, check: bool = True) -> int:
    """h[M, n] (fp32, in place) += y[M, n] (bf16), each sum rounded once to fp32."""
    assert h.dtype == torch.float32 and y.dtype == torch.bfloat16 and h.shape == y.shape
    M, n = h.shape
    st = lib.tf_residual_add(_ptr(h), _ld(h), _ptr(y), _ld(y), M, n, _stream(stream))
    return _ret(st, "tf_residual_add", check)


def tf_embed_rows(table: torch.Tensor, bound: int, ids: torch.Tensor, out: torch.Tensor, stream=None,
                  check: bool = True) -> int:
    """out[M, H] = table[ids[m]] (bf16 rows); ids past ``bound`` give NaN rows.
    ``bound`` must be the whole table's row count (TF_E_RANGE otherwise)."""
    assert table.dtype == torch.bfloat16 and out.dtype == torch.bfloat16 and ids.dtype == torch.int32
    rows, H = table.shape
    st = lib.tf_embed_rows(_ptr(table), rows, H, _ld(table), int(bound), _ptr(ids), ids.numel(), _ptr(out),
                           _ld(out), _stream(stream))
    return _ret(st, "tf_embed_rows", check)


def tf_gather_rows(dst: torch.Tensor, parts: Sequence[Optional[torch.Tensor]], widths: Sequence[int],
                   window_bytes: int = TF_NO_WINDOW, stream=None, check: bool = True) -> int:
    """dst[M, sum(widths)] = the parts side by side; a None part fills 0x7FC0
    and returns TF_E_BROKEN (raised unless ``check`` is False)."""
    assert dst.dtype == torch.bfloat16
    n = len(parts)
    ptrs = (_vp * max(1, n))(*[_ptr(p) for p in parts])
    ws = (_i * max(1, n))(*[int(w) for w in widths])
    st = lib.tf_gather_rows(_ptr(dst), _ld(dst), ptrs, ws, n, dst.shape[0], int(window_bytes), _stream(stream))
    return _ret(st, "tf_gather_rows", check)


def tf_argmax_rows(logits: torch.Tensor, id_base: int, words: torch.Tensor, scratch: torch.Tensor,
                   stream=None, check: bool = True) -> int:
    """words[M] (int64 tensor holding u64 words) = per-row argmax of logits[M, n]."""
    assert logits.dtype == torch.bfloat16 and words.dtype == torch.int64 and scratch.dtype == torch.uint8
    M, n = logits.shape
    st = lib.tf_argmax_rows(_ptr(logits), M, n, _ld(logits), int(id_base), _ptr(words), _ptr(scratch),
                            scratch.numel(), _stream(stream))
    return _ret(st, "tf_argmax_rows", check)


def tf_argmax_rows_static(logits: torch.Tensor, id_base: int, words: torch.Tensor, stream=None,
                          check: bool = True) -> int:
    """tf_argmax_rows without a scratch buffer, for callers that cannot allocate
    device memory: the library's own TF_STATIC_SCRATCH_BYTES device array holds
    the partial results.  Calls that overlap on the GPU must not share it."""
    assert logits.dtype == torch.bfloat16 and words.dtype == torch.int64
    M, n = logits.shape
    st = lib.tf_argmax_rows_static(_ptr(logits), M, n, _ld(logits), int(id_base), _ptr(words), _stream(stream))
    return _ret(st, "tf_argmax_rows_static", check)


def tf_pick(words: torch.Tensor, ids: torch.Tensor, stream=None, check: bool = True) -> int:
    """ids[M] (int32 tensor holding u32 ids) from words[nparts, M]."""
    assert words.dtype == torch.int64 and ids.dtype == torch.int32 and words.is_contiguous()
    if words.dim() == 1:
        words = words[None, :]
    nparts, M = words.shape
    st = lib.tf_pick(_ptr(words), nparts, M, _ptr(ids), _stream(stream))
    return _ret(st, "tf_pick", check)


def tf_top2_scratch_bytes(M: int, n: int) -> int:
    return lib.tf_top2_scratch_bytes(int(M), int(n))


def tf_top2_rows(logits: torch.Tensor, id_base: int, words2: torch.Tensor, scratch: torch.Tensor,
                 stream=None, check: bool = True) -> int:
    """words2[M, 2] (int64 tensor holding u64 words) = per-row winner and second
    place of logits[M, n] in the argmax order."""
    assert logits.dtype == torch.bfloat16 and words2.dtype == torch.int64 and scratch.dtype == torch.uint8
    assert words2.is_contiguous()
    M, n = logits.shape
    st = lib.tf_top2_rows(_ptr(logits), M, n, _ld(logits), int(id_base), _ptr(words2), _ptr(scratch),
                          scratch.numel(), _stream(stream))
    return _ret(st, "tf_top2_rows", check)


def tf_top2_merge(words2: torch.Tensor, out2: torch.Tensor, stream=None, check: bool = True) -> int:
    """out2[M, 2] = the merged top two of words2[nparts, M, 2]."""
    assert words2.dtype == torch.int64 and out2.dtype == torch.int64
    assert words2.is_contiguous() and out2.is_contiguous()
    if words2.dim() == 2:
        words2 = words2[None]
    nparts, M, _ = words2.shape
    st = lib.tf_top2_merge(_ptr(words2), nparts, M, _ptr(out2), _stream(stream))
    return _ret(st, "tf_top2_merge", check)


def tf_abi_version() -> int:
    return lib.tf_abi_version()
