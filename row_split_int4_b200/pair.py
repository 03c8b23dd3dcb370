"""row_split_int4_b200.pair -- the row split across devices, one rank per GPU.

TensorFold PR #1433 (step-1 and step-2 bodies) splits every projection by output
rows: rank h computes rows [h N/2, (h+1) N/2) at full K (the fused gate-up: the
same rows of gate and of up), the ranks exchange those rows as whole bf16 rows,
so no two partial sums meet, and the head exchanges one argmax word per row, so
every rank picks the same token -- the better of the half-vocabulary winners,
failing closed on a non-finite logit in either half.

``PairSeam`` moves the tensors between the ranks with the process group's
all-gather (NCCL over NVLink / NVSwitch on B200s) and hands them, in rank order,
to the kernels that join them: ``tf_gather_rows`` into the frame, ``tf_pick``
over the words, ``tf_top2_merge`` over the top-two words.  Each rank thus holds
the frame, the token id and the merged top two that one device computes from
both halves.  Bytes exchanged per row: 2 per activated column and per down
column, 8 at the head (16 for the top two).

The joining steps are arguments so that the exchange itself can be exercised
where no GPU is present (the CPU tests pass the oracle's gather and pick with
the gloo backend); by default they are this package's CUDA kernels, and
``PairDecode`` runs one rank's decode step on them.
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch
import torch.distributed as dist

from . import (TF_EPI_GLU, TF_NO_WINDOW, tf_argmax_rows, tf_argmax_scratch_bytes, tf_gather_rows, tf_member_segs,
               tf_pick, tf_qmm_rows, tf_split_rows, tf_top2_merge)


def _join_rows_gpu(frame: torch.Tensor, parts: List[torch.Tensor], widths: List[int], window_bytes: int) -> None:
    tf_gather_rows(frame, parts, widths, window_bytes=window_bytes)


def _pick_gpu(words: torch.Tensor, ids: torch.Tensor) -> None:
    tf_pick(words, ids)


def _top2_gpu(words2: torch.Tensor, out2: torch.Tensor) -> None:
    tf_top2_merge(words2, out2)


class PairSeam:
    """The seams of one rank: its share of a split and the three exchanges."""

    def __init__(self, group=None, join_rows: Optional[Callable] = None, pick: Optional[Callable] = None,
                 top2_merge: Optional[Callable] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self._join_rows = join_rows or _join_rows_gpu
        self._pick = pick or _pick_gpu
        self._top2 = top2_merge or _top2_gpu

    # -- shares -----------------------------------------------------------
    def rows(self, N: int):
        """(row0, nrows) of this rank's output rows of an N-row projection."""
        return tf_split_rows(N, self.world, self.rank)

    def member_segs(self, F: int):
        """This rank's gate and up rows of a fused [gate(F); up(F)] stack."""
        return tf_member_segs(F, self.world, self.rank)

    # -- exchanges ----------------------------------------------------------
    def exchange(self, t: torch.Tensor) -> List[torch.Tensor]:
        """Every rank's t, in rank order (t has the same shape and dtype on every
        rank).  The bytes travel as uint8, which every backend carries, and are
        viewed back as t's dtype and shape."""
        t = t.contiguous()
        src = t.view(torch.uint8) if t.dim() > 0 else t.reshape(1).view(torch.uint8)
        out = [torch.empty_like(src) for _ in range(self.world)]
        dist.all_gather(out, src, group=self.group)
        return [o.view(t.dtype).view(t.shape) for o in out]

    def join_rows(self, half: torch.Tensor, frame: torch.Tensor, window_bytes: int = TF_NO_WINDOW) -> None:
        """frame[M, sum of widths] = the ranks' halves [M, w_h] side by side, rank order."""
        parts = self.exchange(half)
        self._join_rows(frame, parts, [p.shape[1] for p in parts], window_bytes)

    def pick(self, word: torch.Tensor, ids: torch.Tensor) -> None:
        """ids[M] = the pick over every rank's argmax words word[M] (int64 holding u64)."""
        self._pick(torch.stack(self.exchange(word)).contiguous(), ids)

    def top2(self, words2: torch.Tensor, out2: torch.Tensor) -> None:
        """out2[M, 2] = the merged top two of every rank's words2[M, 2]."""
        self._top2(torch.stack(self.exchange(words2)).contiguous(), out2)


class PairDecode:
    """One rank's decode step at M = 1 on its halves of the layer and the head:
    gate_up rows with the GLU, join, down rows, join, lm_head rows, argmax word
    with global ids, pick.  Weights are (wq, scales, biases) device tensors of the
    WHOLE matrices (the rank reads only its rows); x is the bf16 [1, H] input."""

    def __init__(self, seam: PairSeam, w_gate_up, w_down, w_head, window_bytes: int = TF_NO_WINDOW):
        self.seam = seam
        self.w_gu, self.w_d, self.w_lm = w_gate_up, w_down, w_head
        self.F = w_gate_up[0].shape[0] // 2
        self.H = w_down[0].shape[0]
        self.V = w_head[0].shape[0]
        self.window = window_bytes
        dev = w_down[0].device
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.segs_gu = seam.member_segs(self.F)
        self.rows_d = seam.rows(self.H)
        self.rows_lm = seam.rows(self.V)
        self.act_half = torch.empty(1, self.segs_gu[0][1], **bf)
        self.act = torch.empty(1, self.F, **bf)
        self.y_half = torch.empty(1, self.rows_d[1], **bf)
        self.y = torch.empty(1, self.H, **bf)
        self.logits = torch.empty(1, self.rows_lm[1], **bf)
        self.word = torch.empty(1, dtype=torch.int64, device=dev)
        self.ids = torch.empty(1, dtype=torch.int32, device=dev)
        self.scratch = torch.empty(tf_argmax_scratch_bytes(1, self.rows_lm[1]), dtype=torch.uint8, device=dev)

    def step(self, x: torch.Tensor, x_head: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Returns ids[1] (int32 holding the u32 token id or TF_PICK_FAILED).
        x_head is the head's input row (defaults to the layer's output y)."""
        tf_qmm_rows(x, *self.w_gu, self.segs_gu, self.act_half, epi=TF_EPI_GLU)
        self.seam.join_rows(self.act_half, self.act, self.window)
        tf_qmm_rows(self.act, *self.w_d, [self.rows_d], self.y_half)
        self.seam.join_rows(self.y_half, self.y, self.window)
        head_in = self.y if x_head is None else x_head
        tf_qmm_rows(head_in, *self.w_lm, [self.rows_lm], self.logits)
        tf_argmax_rows(self.logits, self.rows_lm[0], self.word, self.scratch)
        self.seam.pick(self.word, self.ids)
        return self.ids
