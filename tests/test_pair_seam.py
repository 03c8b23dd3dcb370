"""The row split across ranks (row_split_int4_b200.pair), on two CPU ranks (gloo).

Each rank computes its own rows the way the pages split them (TensorFold PR
#1433, step-1 and step-2 bodies) -- its gate and up rows with the GLU, its down
rows, its half of the head's logits -- and the seams exchange them through the
process group: whole bf16 rows joined into the frame, one argmax word per row
picked on every rank, the top-two words merged.  The joining steps are the CPU
oracle's here (no GPU), so this checks the exchange itself: rank order, shapes,
and that every rank ends with the frame, the ids and the merged top two of the
whole layer and head, bit for bit, including a planted cross-half tie and a NaN
row at the head.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import torch
import torch.multiprocessing as mp

H, F, V, M = 256, 512, 4096, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.numpy().view(np.uint16)


def _t16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16))


def _weights():
    import synth
    wgu = synth.make_weights(2 * F, H, seed=3, tag=synth.TAG_W).astuple()
    wd = synth.make_weights(H, F, seed=3, tag=synth.TAG_W2).astuple()
    wlm = synth.make_weights(V, H, seed=3, tag=synth.TAG_HEAD).astuple()
    x = synth.make_x(M, H, seed=3)
    return x, wgu, wd, wlm


def _whole_logits(orc, y):
    """The whole head's logits of y, with a cross-half tie (row 0) and a NaN (row 1)."""
    import synth
    _, _, _, wlm = _weights()
    lg = orc.qmm_rows(y, *wlm, np.arange(V))
    synth.apply_plants(lg, [synth.Plant(0, "tie", (100, V // 2 + 5)), synth.Plant(1, "nan", (3000,), 0x7FC0)])
    return lg


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    import oracle

    orc = oracle.load()
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        _rank_body(rank, orc, q)
    except Exception:
        import traceback
        q.put((rank, "error", traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def _rank_body(rank, orc, q):
    import torch.distributed as dist
    from row_split_int4_b200.pair import PairSeam
    def join(frame, parts, widths, window):
        frame.copy_(_t16(orc.gather_rows([_bits(p) for p in parts], frame.shape[0], widths)))

    def pick(words, ids):
        ids.copy_(torch.from_numpy(orc.pick(words.numpy().view(np.uint64)).view(np.int32)))

    def top2(words2, out2):
        out2.copy_(torch.from_numpy(orc.top2_merge(words2.numpy().view(np.uint64)).view(np.int64)))

    seam = PairSeam(join_rows=join, pick=pick, top2_merge=top2)
    x, wgu, wd, wlm = _weights()
    # layer: this rank's gate and up rows with the GLU, joined; its down rows, joined
    (g0, ng), (u0, nu) = seam.member_segs(F)
    act_half = orc.glu_rows(x, wgu, np.arange(g0, g0 + ng), np.arange(u0, u0 + nu))
    act = torch.empty(M, F, dtype=torch.int16)
    seam.join_rows(_t16(act_half), act)
    d0, nd = seam.rows(H)
    y_half = orc.qmm_rows(_bits(act), *wd, np.arange(d0, d0 + nd))
    y = torch.empty(M, H, dtype=torch.int16)
    seam.join_rows(_t16(y_half), y)
    # head: this rank's half of the (planted) logits, its word, the pick; its top two, merged
    l0, nl = seam.rows(V)
    lg = _whole_logits(orc, _bits(y))[:, l0:l0 + nl]
    word = torch.from_numpy(orc.argmax_rows(lg, l0).view(np.int64))
    ids = torch.empty(M, dtype=torch.int32)
    seam.pick(word, ids)
    w2 = torch.from_numpy(orc.top2_rows(lg, l0).view(np.int64))
    merged = torch.empty(M, 2, dtype=torch.int64)
    seam.top2(w2, merged)
    dist.barrier()
    q.put((rank, _bits(act).copy(), _bits(y).copy(), ids.numpy().view(np.uint32).copy(),
           merged.numpy().view(np.uint64).copy()))


def test_pair_seam_two_gloo_ranks(orc):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted((q.get(timeout=120) for _ in procs), key=lambda r: r[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    errors = [r[2] for r in results if len(r) == 3 and isinstance(r[1], str)]
    assert not errors, errors[0]
    assert all(p.exitcode == 0 for p in procs)
    # the whole layer and head on one process
    x, wgu, wd, wlm = _weights()
    act_w, y_w = orc.mlp_whole(x, wgu, wd)
    lg = _whole_logits(orc, y_w)
    ids_w = orc.pick(orc.argmax_rows(lg, 0)[None, :])
    top2_w = orc.top2_rows(lg, 0)
    assert [r[0] for r in results] == [0, 1]
    for rank, act, y, ids, merged in results:
        assert np.array_equal(act, act_w), f"rank {rank}: joined activations != whole"
        assert np.array_equal(y, y_w), f"rank {rank}: joined down output != whole"
        assert np.array_equal(ids, ids_w), f"rank {rank}: picked ids != whole"
        assert np.array_equal(merged, top2_w), f"rank {rank}: merged top two != whole"
    assert ids_w[0] == 100 and ids_w[1] == 0xFFFFFFFF       # the planted tie and NaN
