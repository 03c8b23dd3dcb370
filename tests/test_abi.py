"""The C ABI without a GPU: exports, host arithmetic, and every refusal that
happens on the host before anything is enqueued."""
import ctypes
import os
import re

import pytest

import oracle_checks as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tf.h")


@pytest.fixture(scope="module")
def tf():
    import row_split_int4_b200 as tf
    return tf


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(tf_[a-z_0-9]+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported(tf):
    names = declared_functions()
    assert len(names) >= 10, names
    lib = ctypes.CDLL(tf.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in tf.h but not exported"
    assert set(names) == set(tf.EXPORTS)


def test_abi_version(tf):
    assert tf.tf_abi_version() == 1


def test_status_names(tf):
    names = [tf.tf_status_str(i) for i in range(8)]
    assert names == ["TF_OK", "TF_E_ARG", "TF_E_RANGE", "TF_E_ALIGN", "TF_E_WINDOW", "TF_E_BROKEN", "TF_E_CUDA",
                     "TF_E_UNIMPL"]
    assert tf.tf_status_str(99) == "TF_E_?"


def test_header_constants_match_pages(tf):
    g = C.golden("pages_constants.json")
    assert tf.TF_PAIR_FLAG == g["flag_bits"]["pair_flag"]
    assert tf.TF_PICK_FAILED == g["sentinel"]["pick_failed"]
    assert tf.TF_NAN_BF16 == g["broken_link_nan_bf16"]["bits"]
    assert tf.TF_BATCH_ROWS == g["seam_window"]["batch_rows"]
    hdr = open(HEADER).read()
    for name, val in [("TF_PAIR_FLAG", "0x80000000u"), ("TF_PICK_FAILED", "0xFFFFFFFFu"), ("TF_NAN_BF16", "0x7FC0u"),
                      ("TF_BATCH_ROWS", "128"), ("TF_GROUP", "64")]:
        assert re.search(rf"#define {name} {val}\b", hdr), name


def test_split_spans_match_pages(tf):
    sp = C.golden("pages_constants.json")["spans"]
    for key in ("o_proj_down_out", "mlp_member", "lm_head"):
        whole, half = sp[key]["whole"], sp[key]["half"]
        assert tf.tf_split_rows(whole, 2, 0) == (sp["rank0_start"], half)
        assert tf.tf_split_rows(whole, 2, 1) == (half, half)
    F = sp["mlp_member"]["whole"]
    assert tf.tf_member_segs(F, 2, 0) == [(0, 8704), (17408, 8704)]
    assert tf.tf_member_segs(F, 2, 1) == [(8704, 8704), (17408 + 8704, 8704)]


def test_split_refuses_uneven(tf):
    with pytest.raises(tf.TFError) as e:
        tf.tf_split_rows(5121, 2, 0)
    assert e.value.status == tf.TF_E_ARG
    for bad in [(10, 0, 0), (10, 2, 2), (10, 2, -1), (10, 9, 0), (-2, 2, 0)]:
        with pytest.raises(tf.TFError):
            tf.tf_split_rows(*bad)


def test_seam_window_inequality(tf):
    """seamBytes(chunk(512)) <= window < seamBytes(512) (PR #1434 host test)."""
    g = C.golden("pages_constants.json")["seam_window"]
    window = g["seam_bytes_128"]
    assert tf.tf_chunk_rows(g["prompt_rows_requested"]) == g["chunked_rows"]
    assert tf.tf_seam_bytes(tf.tf_chunk_rows(512), g["seam_width"]) <= window
    assert tf.tf_seam_bytes(512, g["seam_width"]) == g["seam_bytes_512"] > window
    assert tf.tf_chunk_rows(5) == 5 and tf.tf_chunk_rows(0) == 0 and tf.tf_chunk_rows(-3) == 0
    assert tf.tf_seam_bytes(0, 10) == 0


# -- refusals before any launch (fake, never-dereferenced device addresses) ----

A = 1 << 20          # a 16-byte aligned fake address


def qmm(tf, x=A, M=1, K=1024, ldx=1024, wq=A, sc=A, bi=A, N=512, segs=((0, 256),), epi=0, y=A, ldy=256):
    arr = (tf.tf_seg * max(1, len(segs)))(*[tf.tf_seg(a, b) for a, b in segs])
    return tf.lib.tf_qmm_rows(x, M, K, ldx, wq, sc, bi, N, arr, len(segs), epi, y, ldy, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=-1), 1), (dict(M=129), 1), (dict(K=0), 1), (dict(K=100, ldx=100), 1), (dict(K=65536 + 64, ldx=70000), 1),
    (dict(N=0), 1), (dict(segs=()), 1), (dict(epi=2), 1),
    (dict(epi=1, segs=((0, 256),)), 1), (dict(epi=1, segs=((0, 256), (256, 128))), 1),
    (dict(segs=((400, 200),)), 2), (dict(segs=((-1, 10),)), 2), (dict(segs=((0, 100), (50, 100))), 2),
    (dict(ldx=1000), 1), (dict(ldy=100), 1),
    (dict(x=0), 1), (dict(wq=0), 1), (dict(y=0), 1),
    (dict(x=A + 2), 3), (dict(ldx=1028), 3), (dict(wq=A + 8), 3), (dict(sc=A + 1), 3), (dict(y=A + 1), 3),
])
def test_qmm_refusals(tf, kw, status):
    assert qmm(tf, **kw) == status


def test_qmm_empty_is_ok_without_launch(tf):
    assert qmm(tf, M=0) == tf.TF_OK
    assert qmm(tf, segs=((0, 0),)) == tf.TF_OK
    assert qmm(tf, M=0, x=0, y=0) == tf.TF_OK


def gather(tf, dst=A, ld=512, parts=(A, A), widths=(256, 256), M=1, window=None):
    n = len(parts)
    p = (ctypes.c_void_p * max(1, n))(*parts)
    w = (ctypes.c_int * max(1, n))(*widths)
    win = tf.TF_NO_WINDOW if window is None else window
    return tf.lib.tf_gather_rows(dst, ld, p, w, n, M, win, None)


def test_gather_refusals(tf):
    assert gather(tf, ld=500) == tf.TF_E_ARG
    assert gather(tf, widths=(256, -1)) == tf.TF_E_ARG
    assert gather(tf, parts=(), widths=()) == tf.TF_E_ARG
    assert gather(tf, parts=(A,) * 9, widths=(8,) * 9, ld=72) == tf.TF_E_ARG
    assert gather(tf, dst=0) == tf.TF_E_ARG
    assert gather(tf, dst=A + 1) == tf.TF_E_ALIGN
    assert gather(tf, parts=(A, A + 1)) == tf.TF_E_ALIGN
    # the window: M * width * 2 must fit (PR #1434): 128 rows of 8,704 fit 2,228,224 B, 129 do not
    W = 2228224
    assert gather(tf, M=129, widths=(8704, 8704), ld=17408, window=W) == tf.TF_E_WINDOW
    assert gather(tf, M=0, widths=(8704, 8704), ld=17408, window=W) == tf.TF_OK
    assert gather(tf, M=0, parts=(A, 0), widths=(8, 8), ld=16) == tf.TF_E_BROKEN


def test_argmax_refusals(tf):
    L = tf.lib
    assert L.tf_argmax_rows(A, 1, 0, 8, 0, A, A, 1 << 20, None) == tf.TF_E_ARG
    assert L.tf_argmax_rows(A, 1, 16, 8, 0, A, A, 1 << 20, None) == tf.TF_E_ARG
    assert L.tf_argmax_rows(A, -1, 16, 16, 0, A, A, 1 << 20, None) == tf.TF_E_ARG
    assert L.tf_argmax_rows(A, 1, 16, 16, 0x7FFFFFF8, A, A, 1 << 20, None) == tf.TF_E_RANGE
    assert L.tf_argmax_rows(A, 0, 16, 16, 0, 0, 0, 0, None) == tf.TF_OK
    need = tf.tf_argmax_scratch_bytes(4, 124160)
    assert need > 0 and need % 8 == 0
    assert L.tf_argmax_rows(A, 4, 124160, 124160, 0, A, A, need - 8, None) == tf.TF_E_ARG
    assert L.tf_argmax_rows(A, 4, 124160, 124160, 0, A + 4, A, need, None) == tf.TF_E_ALIGN
    assert L.tf_argmax_rows(A, 4, 124160, 124160, 0, 0, A, need, None) == tf.TF_E_ARG
    assert tf.tf_argmax_scratch_bytes(0, 10) == 0 and tf.tf_argmax_scratch_bytes(3, 0) == 0


def test_fused_head_refusals(tf):
    L = tf.lib
    seg = tf.tf_seg(0, 2048)

    def call(M=1, K=512, seg=seg, id_base=0, logits=A, ld=2048, words=A, scratch=A, nbytes=None):
        nb = tf.tf_qmm_argmax_scratch_bytes(max(M, 1), max(seg.nrows, 1)) if nbytes is None else nbytes
        return L.tf_qmm_argmax_rows(A, M, K, K, A, A, A, 4096, seg, id_base, logits, ld, words, scratch, nb, None)

    assert call(seg=tf.tf_seg(0, 0)) == tf.TF_E_ARG                 # an empty slice has no argmax
    assert call(id_base=0x7FFFFFFF - 100) == tf.TF_E_RANGE           # ids past 2^31
    assert call(seg=tf.tf_seg(4000, 200)) == tf.TF_E_RANGE           # rows past the matrix
    assert call(M=129) == tf.TF_E_ARG
    assert call(ld=100) == tf.TF_E_ARG
    assert call(words=0) == tf.TF_E_ARG
    assert call(scratch=0) == tf.TF_E_ARG
    assert call(words=A + 4) == tf.TF_E_ALIGN
    assert call(nbytes=8) == tf.TF_E_ARG
    assert call(M=0, words=0, scratch=0) == tf.TF_OK                # nothing to do, nothing read
    need1 = tf.tf_qmm_argmax_scratch_bytes(1, 124160)
    assert need1 >= tf.tf_argmax_scratch_bytes(1, 124160) and need1 % 8 == 0
    assert tf.tf_qmm_argmax_scratch_bytes(16, 124160) >= tf.tf_argmax_scratch_bytes(16, 124160)
    assert tf.tf_qmm_argmax_scratch_bytes(0, 5) == 0 and tf.tf_qmm_argmax_scratch_bytes(1, 0) == 0


def test_residual_and_embed_refusals(tf):
    L = tf.lib
    assert L.tf_residual_add(A, 8, A, 8, -1, 8, None) == tf.TF_E_ARG
    assert L.tf_residual_add(A, 4, A, 8, 1, 8, None) == tf.TF_E_ARG        # ld_h < n
    assert L.tf_residual_add(0, 8, A, 8, 1, 8, None) == tf.TF_E_ARG
    assert L.tf_residual_add(A + 2, 8, A, 8, 1, 8, None) == tf.TF_E_ALIGN
    assert L.tf_residual_add(A, 8, A + 1, 8, 1, 8, None) == tf.TF_E_ALIGN
    assert L.tf_residual_add(0, 8, 0, 8, 0, 8, None) == tf.TF_OK          # nothing to do
    V, H = 248320, 5120
    # the pages' regression: the shard's 124,160 as the bound of the whole table is refused
    assert L.tf_embed_rows(A, V, H, H, V // 2, A, 1, A, H, None) == tf.TF_E_RANGE
    assert L.tf_embed_rows(A, V, H, H, V + 1, A, 1, A, H, None) == tf.TF_E_RANGE
    assert L.tf_embed_rows(A, 0, H, H, 0, A, 1, A, H, None) == tf.TF_E_ARG
    assert L.tf_embed_rows(A, V, H, H - 1, V, A, 1, A, H, None) == tf.TF_E_ARG
    assert L.tf_embed_rows(A, V, H, H, V, 0, 1, A, H, None) == tf.TF_E_ARG
    assert L.tf_embed_rows(A, V, H, H, V, A + 2, 1, A, H, None) == tf.TF_E_ALIGN
    assert L.tf_embed_rows(A, V, H, H, V, A, 0, A, H, None) == tf.TF_OK


def test_qmm8_refusals(tf):
    L = tf.lib

    def call(x=A, M=1, K=1024, ldx=1024, q=A, sc=A, N=512, segs=((0, 256),), y=A, ldy=256):
        arr = (tf.tf_seg * max(1, len(segs)))(*[tf.tf_seg(a, b) for a, b in segs])
        return L.tf_qmm8_rows(x, M, K, ldx, q, sc, N, arr, len(segs), y, ldy, None)

    assert call(M=129) == tf.TF_E_ARG
    assert call(K=0) == tf.TF_E_ARG
    assert call(ldx=1000) == tf.TF_E_ARG
    assert call(segs=((400, 200),)) == tf.TF_E_RANGE
    assert call(segs=((0, 100), (50, 100))) == tf.TF_E_RANGE
    assert call(ldy=100) == tf.TF_E_ARG
    assert call(q=0) == tf.TF_E_ARG
    assert call(x=A + 1) == tf.TF_E_ALIGN
    assert call(M=0, x=0, q=0, sc=0, y=0) == tf.TF_OK


def test_last_cuda_error_is_static_text(tf):
    assert tf.tf_last_cuda_error() == "no error"


def test_top2_refusals(tf):
    L = tf.lib
    assert L.tf_top2_rows(A, 1, 0, 8, 0, A, A, 1 << 20, None) == tf.TF_E_ARG
    assert L.tf_top2_rows(A, 1, 16, 8, 0, A, A, 1 << 20, None) == tf.TF_E_ARG
    assert L.tf_top2_rows(A, 65536, 16, 16, 0, A, A, 1 << 30, None) == tf.TF_E_ARG
    assert L.tf_top2_rows(A, 1, 16, 16, 0x7FFFFFF8, A, A, 1 << 20, None) == tf.TF_E_RANGE
    assert L.tf_top2_rows(A, 0, 16, 16, 0, 0, 0, 0, None) == tf.TF_OK
    need = tf.tf_top2_scratch_bytes(2, 124160)
    assert need == 2 * tf.tf_argmax_scratch_bytes(2, 124160)
    assert L.tf_top2_rows(A, 2, 124160, 124160, 0, A, A, need - 8, None) == tf.TF_E_ARG
    assert L.tf_top2_rows(A, 2, 124160, 124160, 0, A + 4, A, need, None) == tf.TF_E_ALIGN
    assert L.tf_top2_rows(A + 1, 2, 124160, 124160, 0, A, A, need, None) == tf.TF_E_ALIGN
    assert L.tf_top2_merge(A, 0, 1, A + 4096, None) == tf.TF_E_ARG
    assert L.tf_top2_merge(A, 9, 1, A + 4096, None) == tf.TF_E_ARG
    assert L.tf_top2_merge(A, 2, -1, A + 4096, None) == tf.TF_E_ARG
    assert L.tf_top2_merge(A, 2, 4, A + 64, None) == tf.TF_E_ARG       # out2 overlaps the inputs
    assert L.tf_top2_merge(A + 4, 2, 4, A + 4096, None) == tf.TF_E_ALIGN
    assert L.tf_top2_merge(A, 2, 0, 0, None) == tf.TF_OK
    assert tf.TF_TOP2_NONE == C.TOP2_NONE


def test_pick_refusals(tf):
    L = tf.lib
    assert L.tf_pick(A, 0, 1, A, None) == tf.TF_E_ARG
    assert L.tf_pick(A, 9, 1, A, None) == tf.TF_E_ARG
    assert L.tf_pick(A, 2, -1, A, None) == tf.TF_E_ARG
    assert L.tf_pick(0, 2, 1, A, None) == tf.TF_E_ARG
    assert L.tf_pick(A + 4, 2, 1, A, None) == tf.TF_E_ALIGN
    assert L.tf_pick(A, 2, 0, 0, None) == tf.TF_OK
