#!/usr/bin/env python
"""bench.py -- one decode step of the row-split int4 hot path, timed on B200s.

A step is one pass of every step of the path at M=1 over seeded synthetic
inputs already resident in HBM, with the pages' two-rank split emulated as
two row halves on one GPU (TensorFold PR #1433, step-1 and step-2 bodies):

  gate+up  K=5,120 -> 2 x 17,408 rows, each half owning 8,704 rows of each
           member, g * SiLU(u) fused, 2 calls          (tf_qmm_rows, GLU)
  gather   the two 8,704-wide activated halves         (tf_gather_rows)
  down     K=17,408 -> 5,120 rows as 2 x 2,560          (tf_qmm_rows)
  gather   the two 2,560-wide halves                    (tf_gather_rows)
  head     per half: lm_head K=5,120 -> 124,160 rows and the half's argmax
           word in one call (tf_qmm_argmax_rows: the qmm's warps keep their
           best keys, one small kernel makes the word)
  pick     the better half-winner                       (tf_pick)

Timed regions (CUDA events on the launching stream, after the warm-up):
  1. K steps back to back, events only at the two ends: `value`, ms_per_step.
  2. K steps with an event pair around the head (both halves and the pick):
     lm_head_argmax_us_per_token.
  3. K launches of one lm_head half's qmm alone (tf_qmm_rows, the kernel the
     fused head runs), alternating halves, each in an event pair: the
     roofline's average launch duration.

The metric is the int4 dequant-GEMV HBM throughput (GB/s of algorithmic
bytes: 0.5625 B per weight plus activations in and out), with the
lm_head+argmax+pick time per token beside it.  The weights of one step
(866 MB) exceed the 126 MB L2, so every step reads them from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tf|reference]
  python bench.py --sweep        # M in {1..128} x the four shapes, per-point lines

For N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the step: the path has no exchange that crosses a device here, so
`value` is the sum of all ranks' bytes over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "int4 dequant-GEMV HBM GB/s (% B200 peak) at M=1; lm_head+argmax µs/token"
WORKLOAD = ("decode step M=1, two row halves on one GPU: gate_up 5120x34816 int4 g64 (GLU fused) + gather + "
            "down 17408x5120 + gather + lm_head 5120x248320 + per-half argmax + pick")
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0   # B200 spec sheet


# --------------------------------------------------------------------------- helpers
def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s of this machine's B200s (burst, for a kernel timed alone)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def max_over_ranks(values, world, dist=None, device="cpu"):
    """Element-wise maximum of per-rank times: the slowest rank decides a
    whole-job figure.  With one rank the values come back unchanged."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_value(bytes_per_step, world, steps, elapsed_ms):
    """Whole-job GB/s of `world` independent replicas, each moving
    `bytes_per_step` per step, over the slowest rank's time."""
    return bytes_per_step * world * steps / (elapsed_ms / 1e3) / 1e9


def qmm_bytes(K, rows, M=1, out_cols=None):
    """Algorithmic bytes of one qmm call: 0.5625 B per weight + x read + y written."""
    out_cols = rows if out_cols is None else out_cols
    return int(0.5625 * K * rows) + 2 * M * K + 2 * M * out_cols


def step_bytes():
    H, F, V = 5120, 17408, 248320
    b = {
        "gate_up": 2 * qmm_bytes(H, F, out_cols=F // 2),      # each half: F rows (8,704 gate + 8,704 up)
        "gather_act": 2 * (2 * F),                            # read both halves, write the frame
        "down": 2 * qmm_bytes(F, H // 2),
        "gather_y": 2 * (2 * H),
        "lm_head": 2 * qmm_bytes(H, V // 2),
        "argmax": 2 * V + 2 * 8,
        "pick": 2 * 8 + 4,
    }
    b["total"] = sum(b.values())
    return b


KERNEL_SOURCES = ["row_split_int4_b200/csrc/qmm_stream.cu", "row_split_int4_b200/csrc/qmm_common.cuh",
                  "row_split_int4_b200/csrc/stream_common.cuh", "row_split_int4_b200/csrc/tf_common.cuh",
                  "row_split_int4_b200/csrc/tf_kernels.h", "include/tf.h"]


def device_source_hash():
    """sha256 over the files the M = 1 streaming kernels are compiled from, in
    KERNEL_SOURCES order (profiles record it when their counters are taken)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_from_profiles():
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    only while the kernel's sources are the ones the counters were taken on."""
    path = os.path.join(ROOT, "profiles", "qmm_m1_tile_lm_head_half.md")
    try:
        txt = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", txt)
    s = re.search(r"device_source_sha256:\s*([0-9a-f]{64})", txt)
    if not m or not s:
        return None
    return int(m.group(1)) if device_source_hash() == s.group(1) else None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read only) while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, index, period=0.01):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        self.period, self.index = period, index
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- the step
class DecodeStep:
    """Device buffers and weights of one decode step; run() enqueues it."""

    def __init__(self, tf, synth, seed=0, host_weights=None):
        import torch
        self.tf, self.torch = tf, torch
        H, F, V = synth.HIDDEN, synth.FFN, synth.VOCAB
        self.H, self.F, self.V = H, F, V
        hw = host_weights or make_host_weights(synth, seed)
        self.host = hw
        self.Wgu = synth.weights_to_device(hw["gate_up"])
        self.Wd = synth.weights_to_device(hw["down"])
        self.Wlm = synth.weights_to_device(hw["lm_head"])
        bf = dict(dtype=torch.bfloat16, device="cuda")
        self.x_mlp = synth.to_device(hw["x_mlp"])
        self.x_head = synth.to_device(hw["x_head"])
        self.act_h = [torch.empty(1, F // 2, **bf) for _ in range(2)]
        self.act = torch.empty(1, F, **bf)
        self.y_h = [torch.empty(1, H // 2, **bf) for _ in range(2)]
        self.y = torch.empty(1, H, **bf)
        self.logits = [torch.empty(1, V // 2, **bf) for _ in range(2)]
        self.words = torch.empty(2, 1, dtype=torch.int64, device="cuda")
        self.ids = torch.empty(1, dtype=torch.int32, device="cuda")
        self.head_scratch = [torch.empty(tf.tf_qmm_argmax_scratch_bytes(1, V // 2), dtype=torch.uint8, device="cuda")
                             for _ in range(2)]
        self.member = [tf.tf_member_segs(F, 2, h) for h in range(2)]
        self.down_rows = [tf.tf_split_rows(H, 2, h) for h in range(2)]
        self.head_rows = [tf.tf_split_rows(V, 2, h) for h in range(2)]
        self.window = synth.WINDOW_BYTES
        # gate_up x2, gather, down x2, gather, per half the head's qmm and its key kernel, pick
        self.launches_per_step = 2 + 1 + 2 + 1 + 2 * 2 + 1

    def run(self, stream, head_events=None):
        tf = self.tf
        for h in range(2):
            tf.tf_qmm_rows(self.x_mlp, *self.Wgu, self.member[h], self.act_h[h], epi=tf.TF_EPI_GLU, stream=stream)
        tf.tf_gather_rows(self.act, self.act_h, [self.F // 2] * 2, window_bytes=self.window, stream=stream)
        for h in range(2):
            tf.tf_qmm_rows(self.act, *self.Wd, [self.down_rows[h]], self.y_h[h], stream=stream)
        tf.tf_gather_rows(self.y, self.y_h, [self.H // 2] * 2, window_bytes=self.window, stream=stream)
        if head_events is not None:
            head_events[0].record(stream)
        self.run_head(stream)
        if head_events is not None:
            head_events[1].record(stream)

    def run_head(self, stream):
        """Per half the fused lm_head qmm and argmax word, then the pick."""
        tf = self.tf
        for h in range(2):
            r0, n = self.head_rows[h]
            tf.tf_qmm_argmax_rows(self.x_head, *self.Wlm, (r0, n), r0, self.logits[h], self.words[h],
                                  self.head_scratch[h], stream=stream)
        tf.tf_pick(self.words, self.ids, stream=stream)

    def lm_head_half(self, h, stream):
        """One half of the lm_head qmm alone: the kernel the fused head runs."""
        self.tf.tf_qmm_rows(self.x_head, *self.Wlm, [self.head_rows[h]], self.logits[h], stream=stream)


def capture_graphs(torch, step):
    """CUDA graphs of the decode step, of its head (both fused halves and the pick)
    and of each lm_head half's qmm alone, captured on a side stream after one
    eager pass there."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step.run(side)
    torch.cuda.current_stream().wait_stream(side)
    out = {"step": torch.cuda.CUDAGraph(), "head": torch.cuda.CUDAGraph(),
           "lm": [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]}
    with torch.cuda.graph(out["step"]):
        step.run(torch.cuda.current_stream())
    with torch.cuda.graph(out["head"]):
        step.run_head(torch.cuda.current_stream())
    for h in range(2):
        with torch.cuda.graph(out["lm"][h]):
            step.lm_head_half(h, torch.cuda.current_stream())
    torch.cuda.synchronize()
    return out


def make_host_weights(synth, seed=0):
    H, F, V = synth.HIDDEN, synth.FFN, synth.VOCAB
    return {
        "gate_up": synth.make_weights(2 * F, H, seed=seed, tag=synth.TAG_W),
        "down": synth.make_weights(H, F, seed=seed, tag=synth.TAG_W2),
        "lm_head": synth.make_weights(V, H, seed=seed, tag=synth.TAG_HEAD),
        "x_mlp": synth.make_x(1, H, seed=seed),
        "x_head": synth.make_x(1, H, seed=seed, tag=5),
    }


# --------------------------------------------------------------------------- CPU oracle leg
def oracle_sample(hw, frac, nthreads):
    """Run the oracle on the first `frac` of every matrix's rows of the step
    (M=1), plus argmax/pick over that many logits; return (seconds, bytes)."""
    import numpy as np
    import oracle
    orc = oracle.load()
    H, F, V = 5120, 17408, 248320
    nF = max(8, int(F * frac)) // 2 * 2
    nH = max(2, int(H * frac)) // 2 * 2
    nV = max(16, int(V * frac)) // 2 * 2
    t0 = time.perf_counter()
    gu = hw["gate_up"].astuple()
    g = orc.qmm_rows(hw["x_mlp"], *gu, np.arange(nF), nthreads=nthreads)
    u = orc.qmm_rows(hw["x_mlp"], *gu, np.arange(F, F + nF), nthreads=nthreads)
    a = orc.glu(g, u)
    act = np.zeros((1, F), dtype=np.uint16)
    act[:, :nF] = a
    orc.qmm_rows(act, *hw["down"].astuple(), np.arange(nH), nthreads=nthreads)
    lg = orc.qmm_rows(hw["x_head"], *hw["lm_head"].astuple(), np.arange(nV), nthreads=nthreads)
    h = nV // 2
    orc.head_split([lg[:, :h], lg[:, h:]], [0, h])
    dt = time.perf_counter() - t0
    nbytes = (qmm_bytes(H, 2 * nF, out_cols=nF) + qmm_bytes(F, nH) + qmm_bytes(H, nV) + 2 * nV)
    return dt, nbytes, f"first {frac:.4%} of every matrix's rows (gate_up {2 * nF}, down {nH}, lm_head {nV} rows) at M=1"


def calibrated_oracle(hw, target_s, nthreads):
    frac = 1.0 / 512
    dt, nb, _ = oracle_sample(hw, frac, nthreads)
    frac = min(1.0, frac * max(1.0, target_s / max(dt, 1e-4)))
    return frac


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(hw, target_s=20.0, single_s=5.0):
    """The oracle on all host cores (OpenMP over rows) on a calibrated sample of the
    step, and once more on one thread on a smaller sample."""
    nthreads = os.cpu_count() or 1
    frac = calibrated_oracle(hw, target_s, nthreads)
    tot_t, tot_b, reps, desc = 0.0, 0, 0, ""
    while tot_t < 0.5 * target_s or reps == 0:
        dt, nb, desc = oracle_sample(hw, frac, nthreads)
        tot_t += dt
        tot_b += nb
        reps += 1
    f1 = calibrated_oracle(hw, single_s, 1)
    dt1, nb1, desc1 = oracle_sample(hw, f1, 1)
    return {"value": round(tot_b / tot_t / 1e9, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": desc + f", x{reps}, {tot_t:.1f} s, C fp64 oracle with OpenMP over rows",
            "single_thread": {"value": round(nb1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": desc1 + f", {dt1:.1f} s"}}


# --------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    hw = make_host_weights(synth, args.seed)
    nthreads = os.cpu_count() or 1
    budget = 90.0 / max(1, args.steps + args.warmup)
    frac = calibrated_oracle(hw, budget, nthreads)
    for _ in range(args.warmup):
        oracle_sample(hw, frac, nthreads)
    tot_t, tot_b, desc = 0.0, 0, ""
    for _ in range(args.steps):
        dt, nb, desc = oracle_sample(hw, frac, nthreads)
        tot_t += dt
        tot_b += nb
    value = tot_b / tot_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_per_step": desc},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- one kernel
KERNELS = {   # name: (rows, K, segments, epilogue)
    "lm_head_half": (248320, 5120, [(0, 124160)], 0),
    "gate_up_half": (34816, 5120, [(0, 8704), (17408, 8704)], 1),
    "down_half": (5120, 17408, [(0, 2560)], 0),
    "attn_out": (5120, 5120, [(0, 5120)], 0),
}


ADJACENT = ("residual_add", "embed_rows", "lm_head8_half", "gather_act", "argmax_half", "head_half_fused", "pick",
            "top2_half")


def run_adjacent(args):
    """The steps either side of the seam, --reps times: the fp32 residual add of
    a 5,120-wide bf16 row (10 B per element) and the embedding rows of M token
    ids from the whole 248,320 x 5,120 table (4 B per element)."""
    import torch
    import row_split_int4_b200 as tf
    H, V, M = 5120, 248320, args.M
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    if args.kernel == "residual_add":
        h = torch.randn(M, H, device="cuda", generator=g)
        y = torch.randn(M, H, device="cuda", generator=g).to(torch.bfloat16)
        call, nbytes = (lambda: tf.tf_residual_add(h, y)), 10 * M * H
    elif args.kernel == "lm_head8_half":
        # the int8 head's half: 124,160 rows x 5,120 int8 codes and a bf16 scale per row
        rows = V // 2
        q8 = torch.randint(-128, 128, (rows, H), dtype=torch.int8, device="cuda", generator=g)
        sc = (1e-4 + 1e-4 * torch.rand(rows, device="cuda", generator=g)).to(torch.bfloat16)
        x = torch.randn(M, H, device="cuda", generator=g).to(torch.bfloat16)
        y = torch.empty(M, rows, dtype=torch.bfloat16, device="cuda")
        call, nbytes = (lambda: tf.tf_qmm8_rows(x, q8, sc, [(0, rows)], y)), rows * H + 2 * rows + 2 * M * H + 2 * M * rows
    elif args.kernel == "gather_act":
        # the activated frame's two 8,704-wide halves joined into the 17,408-wide frame
        F = 17408
        parts = [torch.randn(M, F // 2, device="cuda", generator=g).to(torch.bfloat16) for _ in range(2)]
        frame = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
        call, nbytes = (lambda: tf.tf_gather_rows(frame, parts, [F // 2] * 2)), 4 * M * F
    elif args.kernel in ("argmax_half", "top2_half"):
        # one half of the head's logits, 124,160 wide
        n = V // 2
        lg = torch.randn(M, n, device="cuda", generator=g).to(torch.bfloat16)
        if args.kernel == "argmax_half":
            w = torch.empty(M, dtype=torch.int64, device="cuda")
            scr = torch.empty(tf.tf_argmax_scratch_bytes(M, n), dtype=torch.uint8, device="cuda")
            call = lambda: tf.tf_argmax_rows(lg, n, w, scr)   # noqa: E731
        else:
            w = torch.empty(M, 2, dtype=torch.int64, device="cuda")
            scr = torch.empty(tf.tf_top2_scratch_bytes(M, n), dtype=torch.uint8, device="cuda")
            call = lambda: tf.tf_top2_rows(lg, n, w, scr)   # noqa: E731
        nbytes = 2 * M * n + 8 * M
    elif args.kernel == "head_half_fused":
        # one half of the lm_head with its argmax word (the qmm and the key kernel)
        rows = V // 2
        wq = torch.randint(0, 256, (V, H // 2), dtype=torch.uint8, device="cuda", generator=g)
        sc = (0.001 + 0.019 * torch.rand(V, H // 64, device="cuda", generator=g)).to(torch.bfloat16)
        bi = (-8 * sc.float() + 1e-3 * torch.randn(V, H // 64, device="cuda", generator=g)).to(torch.bfloat16)
        x = torch.randn(M, H, device="cuda", generator=g).to(torch.bfloat16)
        lg = torch.empty(M, rows, dtype=torch.bfloat16, device="cuda")
        w = torch.empty(M, dtype=torch.int64, device="cuda")
        scr = torch.empty(tf.tf_qmm_argmax_scratch_bytes(M, rows), dtype=torch.uint8, device="cuda")
        call = lambda: tf.tf_qmm_argmax_rows(x, wq, sc, bi, (rows, rows), rows, lg, w, scr)   # noqa: E731
        nbytes = qmm_bytes(H, rows, M=M)
    elif args.kernel == "pick":
        words = torch.randint(0, 2**40, (2, M), dtype=torch.int64, device="cuda", generator=g)
        ids = torch.empty(M, dtype=torch.int32, device="cuda")
        call, nbytes = (lambda: tf.tf_pick(words, ids)), 16 * M + 4 * M
    else:
        table = torch.randn(V, H, device="cuda", generator=g).to(torch.bfloat16)
        ids = torch.randint(0, V, (M,), device="cuda", generator=g, dtype=torch.int32)
        out = torch.empty(M, H, dtype=torch.bfloat16, device="cuda")
        call, nbytes = (lambda: tf.tf_embed_rows(table, V, ids, out)), 4 * M * H
    call()
    if not args.no_graph:   # one call in a CUDA graph: a replay has no host work per kernel
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            call()
        call = gr.replay
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.reps)]
    for a, b in ev:
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    us = [a.elapsed_time(b) * 1e3 for a, b in ev]
    best = min(us[1:] or us)
    print(json.dumps({"kernel": args.kernel, "M": M, "H": H, "us": [round(u, 2) for u in us[:8]],
                      "best_us": round(best, 2), "GB/s": round(nbytes / best / 1e3, 1), "bytes": nbytes}))
    return 0


def run_kernel(args):
    """One qmm call of the decode step, --reps times, on random bytes (the small
    case the kernel profiles are captured on)."""
    import torch
    import row_split_int4_b200 as tf
    N, K, segs, epi = KERNELS[args.kernel]
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    wq = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device="cuda", generator=g)
    sc = (0.001 + 0.019 * torch.rand(N, K // 64, device="cuda", generator=g)).to(torch.bfloat16)
    bi = (-8 * sc.float() + 1e-3 * torch.randn(N, K // 64, device="cuda", generator=g)).to(torch.bfloat16)
    x = torch.randn(args.M, K, device="cuda", generator=g).to(torch.bfloat16)
    cols = segs[0][1] if epi else sum(n for _, n in segs)
    y = torch.empty(args.M, cols, dtype=torch.bfloat16, device="cuda")

    def call():
        tf.tf_qmm_rows(x, wq, sc, bi, segs, y, epi=epi, stream=torch.cuda.current_stream())
    call()
    if not args.no_graph:   # one call in a CUDA graph: a replay has no host work per kernel
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        call = g.replay
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.reps)]
    for a, b in ev:
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    us = [a.elapsed_time(b) * 1e3 for a, b in ev]
    rows = sum(n for _, n in segs)
    nbytes = qmm_bytes(K, rows, M=args.M, out_cols=cols)
    best = min(us[1:] or us)
    print(json.dumps({"kernel": args.kernel, "M": args.M, "rows": rows, "K": K, "us": [round(u, 2) for u in us],
                      "best_us": round(best, 2), "GB/s": round(nbytes / best / 1e3, 1), "bytes": nbytes}))
    return 0


# --------------------------------------------------------------------------- sweep
SWEEP_M = (1, 2, 4, 8, 16, 32, 64, 128)
SWEEP_SHAPES = {   # name: (whole rows, K, epilogue); every point runs the two row halves
    "attn_out": (5120, 5120, 0),
    "gate_up": (34816, 5120, 1),
    "down": (5120, 17408, 0),
    "lm_head": (248320, 5120, 0),
}
L2_BYTES = 126 * 1024 * 1024


def run_sweep(args):
    """M in {1..128} over the four shapes, each point the two row halves of the
    shape (for lm_head each half through the fused qmm + argmax call, then the pick), --reps back-to-back
    repetitions timed with CUDA events.  The weights stay in HBM; each shape is
    replicated into enough separate buffers to span 3 x L2 and the repetitions
    rotate through them, so a repetition never finds its weights in L2, and a
    512 MB write flushes L2 between shapes.  One JSON line per point."""
    import torch
    import row_split_int4_b200 as tf
    import synth
    torch.cuda.set_device(0)
    peak_hbm, hbm_kind = measured_peak()
    peak_tc, tc_kind = measured_tensor_peak()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    shapes = [s for s in SWEEP_SHAPES if not args.shapes or s in args.shapes.split(",")]
    points = []
    Ms = [int(m) for m in args.sweep_m.split(",")] if args.sweep_m else list(SWEEP_M)
    for name in shapes:
        N, K, epi = SWEEP_SHAPES[name]
        tag = {"attn_out": synth.TAG_ATTN, "gate_up": synth.TAG_W, "down": synth.TAG_W2, "lm_head": synth.TAG_HEAD}[name]
        w = synth.weights_to_device(synth.make_weights(N, K, seed=args.seed, tag=tag))
        wbytes = sum(t.numel() * t.element_size() for t in w)
        nrep = max(1, -(-3 * L2_BYTES // wbytes))
        replicas = [w] + [tuple(t.clone() for t in w) for _ in range(nrep - 1)]
        x = synth.to_device(synth.make_x(max(Ms), K, seed=args.seed, tag=synth.TAG_X))
        if epi:
            segs = [tf.tf_member_segs(N // 2, 2, h) for h in range(2)]
            cols = N // 4
        else:
            segs = [[tf.tf_split_rows(N, 2, h)] for h in range(2)]
            cols = N // 2
        y = [torch.empty(max(Ms), cols, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        head = name == "lm_head"
        if head:
            ids = torch.empty(max(Ms), dtype=torch.int32, device="cuda")
            hscr = [torch.empty(tf.tf_qmm_argmax_scratch_bytes(max(Ms), cols), dtype=torch.uint8, device="cuda")
                    for _ in range(2)]
        for M in Ms:
            if head:
                words = torch.empty(2, M, dtype=torch.int64, device="cuda")   # [half][M], contiguous

            def rep(r):
                wr = replicas[r % nrep]
                if head:   # per half the fused qmm + argmax word, then the pick
                    for h in range(2):
                        r0, n = segs[h][0]
                        tf.tf_qmm_argmax_rows(x[:M], *wr, (r0, n), r0, y[h][:M], words[h], hscr[h], stream=stream)
                    tf.tf_pick(words, ids[:M], stream=stream)
                    return
                for h in range(2):
                    tf.tf_qmm_rows(x[:M], *wr, segs[h], y[h][:M], epi=epi, stream=stream)
            flush.zero_()
            for r in range(max(3, args.warmup)):
                rep(r)
            torch.cuda.synchronize()
            run = rep
            if not args.no_graph:   # one CUDA graph per weight replica, replayed in turn
                gs = []
                for r in range(nrep):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        stream = torch.cuda.current_stream()
                        rep(r)
                    gs.append(g)
                stream = torch.cuda.current_stream()
                run = lambda r: gs[r % nrep].replay()   # noqa: E731
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            sampler = ClockSampler(0)
            with sampler:
                e0.record(stream)
                for r in range(args.reps):
                    run(r)
                e1.record(stream)
                torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / args.reps
            nbytes = 2 * qmm_bytes(K, N // 2, M=M, out_cols=cols) + (2 * M * N + 2 * 8 * M + 4 * M if head else 0)
            flops = 2.0 * M * K * N
            t_hbm, t_tc = nbytes / (peak_hbm * 1e3), flops / (peak_tc * 1e6)   # microseconds
            bound = "hbm" if t_hbm >= t_tc else "tensor"
            pt = {
                "sweep": name, "M": M, "K": K, "rows": N, "reps": args.reps, "us_per_rep": round(us, 3),
                "GB/s": round(nbytes / us / 1e3, 1), "TFLOP/s": round(flops / us / 1e6, 2),
                "hbm_frac": round(nbytes / us / 1e3 / peak_hbm, 4), "tensor_frac": round(flops / us / 1e6 / peak_tc, 4),
                "bound": bound, "roofline_frac": round(max(t_hbm, t_tc) / us, 4),
                "peaks": {"hbm_gbs": peak_hbm, "bf16_tflops": peak_tc, "kind": f"{hbm_kind}/{tc_kind}"},
                "weight_replicas": nrep, "l2": "replicas span 3 x L2; L2 flushed between points",
                "clocks": sampler.summary()}
            points.append(pt)
            print(json.dumps(pt), flush=True)
        del replicas, w, x, y
        torch.cuda.empty_cache()
    if args.sweep_json:
        with open(args.sweep_json, "w") as f:
            json.dump({"gpu": torch.cuda.get_device_name(0), "points": points}, f, indent=1)
    return 0


# --------------------------------------------------------------------------- main arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["tf", "reference"], default="tf")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every call from the host (no CUDA graph)")
    ap.add_argument("--sweep", action="store_true", help="per-point sweep over M and the four shapes")
    ap.add_argument("--reps", type=int, default=1000)
    ap.add_argument("--kernel", choices=sorted(KERNELS) + list(ADJACENT),
                    help="time one call of a step of the path (profiling driver)")
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--shapes", default="", help="sweep: comma-separated subset of " + ",".join(SWEEP_SHAPES))
    ap.add_argument("--sweep-m", default="", help="sweep: comma-separated M values")
    ap.add_argument("--sweep-json", default="", help="sweep: also write every point to this JSON file")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.kernel in ADJACENT:
        return run_adjacent(args)
    if args.kernel:
        return run_kernel(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    import row_split_int4_b200 as tf
    import synth

    hw = make_host_weights(synth, args.seed)
    step = DecodeStep(tf, synth, host_weights=hw)
    stream = torch.cuda.current_stream()
    nb = step_bytes()

    for _ in range(args.warmup):
        step.run(stream)
    barrier()

    K = args.steps

    def ev_pair():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    # The step, the head and one lm_head half, each captured once into a CUDA graph
    # (the same library calls; a replay launches the same kernels with no host
    # work per kernel), so that host launch costs do not starve the GPU.
    graphs, graph_error = None, ""
    if not args.no_graph:
        try:
            graphs = capture_graphs(torch, step)
        except Exception as e:  # noqa: BLE001
            graphs = None
            graph_error = str(e)[:200]

    def run_step():
        if graphs:
            graphs["step"].replay()
        else:
            step.run(stream)

    t0, t1 = ev_pair()
    sampler = ClockSampler(local)
    barrier()
    with sampler:
        # 1. the whole step, K times back to back
        t0.record(stream)
        for i in range(K):
            run_step()
        t1.record(stream)
        barrier()
        elapsed_ms = t0.elapsed_time(t1)
        # 2. the head chain of each step (both halves' qmm + argmax word, the pick)
        hd_ev = [ev_pair() for _ in range(K)]
        for i in range(K):
            if graphs:
                run_step()   # keeps the head's inputs in their place in the step's stream of work
                hd_ev[i][0].record(stream)
                graphs["head"].replay()
                hd_ev[i][1].record(stream)
            else:
                step.run(stream, head_events=hd_ev[i])
        barrier()
        # 3. one lm_head half's qmm alone, halves alternating
        lm_ev = [ev_pair() for _ in range(K)]
        for i in range(K):
            lm_ev[i][0].record(stream)
            if graphs:
                graphs["lm"][i % 2].replay()
            else:
                step.lm_head_half(i % 2, stream)
            lm_ev[i][1].record(stream)
        barrier()
    lm_ms = [a.elapsed_time(b) for (a, b) in lm_ev]
    head_ms = [a.elapsed_time(b) for (a, b) in hd_ev]

    # end to end through the public API: pinned host inputs in, result out, every step
    e2e = None
    if not args.no_e2e:
        xm_h = torch.empty_like(step.x_mlp, device="cpu").pin_memory()
        xh_h = torch.empty_like(step.x_head, device="cpu").pin_memory()
        xm_h.copy_(step.x_mlp)
        xh_h.copy_(step.x_head)
        y_h = torch.empty_like(step.y, device="cpu").pin_memory()
        id_h = torch.empty_like(step.ids, device="cpu").pin_memory()
        Ke = max(3, min(K, 1000))

        def e2e_enqueue(s):
            step.x_mlp.copy_(xm_h, non_blocking=True)
            step.x_head.copy_(xh_h, non_blocking=True)
            step.run(s)
            y_h.copy_(step.y, non_blocking=True)
            id_h.copy_(step.ids, non_blocking=True)

        # A serving loop replays one CUDA graph per step: the copies of the step's
        # inputs from pinned host memory, the library calls, the copies of the
        # result back; the host waits for the result every step.
        e2e_graph = None
        if graphs:
            try:
                e2e_graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(e2e_graph):
                    e2e_enqueue(torch.cuda.current_stream())
                torch.cuda.synchronize()
            except Exception:  # noqa: BLE001
                e2e_graph = None

        def e2e_step():
            if e2e_graph is not None:
                e2e_graph.replay()
            else:
                e2e_enqueue(stream)
            stream.synchronize()

        for _ in range(args.warmup):
            e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(Ke):
            e2e_step()
        e1.record(stream)
        barrier()
        e2e_ms = e0.elapsed_time(e1) / Ke
        e2e = {"e2e_ms": e2e_ms, "h2d": step.x_mlp.numel() * 2 + step.x_head.numel() * 2,
               "d2h": step.y.numel() * 2 + step.ids.numel() * 4, "graph": e2e_graph is not None}

    # max over ranks
    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e["e2e_ms"] if e2e else 0.0], world, dist, device="cuda")

    if rank == 0:
        ms_step = elapsed_ms / K
        value = job_value(nb["total"], world, K, elapsed_ms)
        peak, peak_kind = measured_peak()
        lm_bytes = qmm_bytes(5120, 248320 // 2)
        lm_avg_ms = statistics.fmean(lm_ms)
        achieved = lm_bytes / (lm_avg_ms / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": 1, "bytes_per_step": nb["total"],
                       "l2": "no flush: inputs larger than L2 (866 MB of weights per step vs 126 MB L2)",
                       "parallelism": f"replicas x{world}" if world > 1 else "one GPU, two row halves",
                       "timed_regions": "value: K steps between two events; head: event pair per step around "
                                        "both fused halves and the pick; roofline: K lone lm_head-half qmm "
                                        "launches, each in an event pair",
                       "launch": ("each timed region replays CUDA graphs of the library calls"
                                  if graphs else "every call launched from the host" +
                                  (f" (graph capture failed: {graph_error})" if not args.no_graph else ""))},
            "step_hbm_frac": {"measured": round(value / peak, 4), "spec_8000": round(value / SPEC_HBM_GBS, 4),
                              "peak_kind": peak_kind},
            "lm_head_argmax_us_per_token": round(statistics.fmean(head_ms) * 1e3, 2),
            "tokens_per_s_equiv": round(1e3 / ms_step, 1),
            "roofline": {"bound": "hbm", "kernel": "qmm_m1_tile_kernel (lm_head half, 124,160 x 5,120)",
                         "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "frac_spec_8000": round(achieved / SPEC_HBM_GBS, 4),
                         "traffic": traffic_from_profiles(),
                         "bytes_per_launch": lm_bytes, "avg_launch_us": round(lm_avg_ms * 1e3, 3)},
            "gpu_launches": step.launches_per_step * K,
            "clocks": sampler.summary(),
        }
        if e2e:
            line["e2e"] = {"value": round(job_value(nb["total"], world, 1, e2e_ms), 2), "unit": "GB/s",
                           "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                           "ms_per_step": round(e2e_ms, 5),
                           "launch": "one CUDA graph per step (host copies in, the library calls, result out), "
                                     "host waits every step" if e2e["graph"] else "eager library calls, host waits every step"}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(hw)
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
