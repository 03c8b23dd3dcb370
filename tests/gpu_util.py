"""Helpers for the GPU parity tests: device tensors of the seeded inputs and
the acceptance checks.

V (values): |gpu - r| <= 2 ulp_bf16(r), r = the oracle's double result
    rounded to bf16, ulp taken in r's binade (subnormal spacing 2^-133 below
    2^-126).  Non-finite r must meet the same class on the GPU.  When |r| is
    tiny because the sum cancels, |gpu - y64| <= K * 2^-24 * sum|x_k w_k|
    (the fp32 accumulation bound) is also accepted, and such cases are counted.
I (ids): argmax words and picked ids are compared bit for bit.
S (split == whole): torch.equal on the raw bits.
"""
from __future__ import annotations

import numpy as np
import torch

import synth

TOL_ULPS = 2


def need_gpu():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def bf16_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def ulp_bf16(r: np.ndarray) -> np.ndarray:
    a = np.abs(r)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.exp2(e - 7.0)


def check_values(gpu_bits: np.ndarray, ref_bits: np.ndarray, y64: np.ndarray | None = None,
                 absdot: np.ndarray | None = None, K: int = 0, what: str = "") -> dict:
    """Apply V; returns counts.  Raises AssertionError with the worst cases."""
    g = bf16_f64(gpu_bits)
    r = bf16_f64(ref_bits)
    fin_r = np.isfinite(r)
    # non-finite oracle values: same class on the GPU
    nf = ~fin_r
    if nf.any():
        same = (np.isnan(g[nf]) & np.isnan(r[nf])) | (g[nf] == r[nf])
        assert same.all(), f"{what}: non-finite class mismatch at {np.nonzero(nf)[0][~same][:5]}"
    gf = np.where(fin_r, g, 0.0)
    rf = np.where(fin_r, r, 0.0)
    err = np.abs(gf - rf)
    tol = TOL_ULPS * ulp_bf16(rf)
    ok = err <= tol
    floor_used = 0
    if y64 is not None and absdot is not None and not ok.all():
        floor = K * 2.0 ** -24 * absdot
        ok_floor = np.abs(gf - y64) <= floor
        floor_used = int((~ok & ok_floor & fin_r).sum())
        ok = ok | ok_floor
    ok = ok | nf
    if not ok.all():
        bad = np.nonzero(~ok.reshape(-1))[0]
        worst = bad[np.argsort(-(err.reshape(-1)[bad] / tol.reshape(-1)[bad]))][:5]
        det = [(int(i), float(g.reshape(-1)[i]), float(r.reshape(-1)[i]),
                float(err.reshape(-1)[i] / tol.reshape(-1)[i] * TOL_ULPS)) for i in worst]
        raise AssertionError(f"{what}: {bad.size} of {ok.size} values beyond {TOL_ULPS} bf16 ulps "
                             f"(index, gpu, oracle, ulps): {det}")
    ulps = err / np.where(tol > 0, tol / TOL_ULPS, 1.0)
    return {"n": int(ok.size), "floor_used": floor_used, "max_ulps": float(ulps.max()) if ulps.size else 0.0,
            "exact": int((gpu_bits == ref_bits).sum())}


def dev(a: np.ndarray) -> torch.Tensor:
    return synth.to_device(a, "cuda")


def host_bits(t: torch.Tensor) -> np.ndarray:
    return synth.bits_of(t)


def empty_bf16(*shape) -> torch.Tensor:
    return torch.empty(*shape, dtype=torch.bfloat16, device="cuda")


def bits_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Bit-for-bit equality (NaN payloads included)."""
    if a.shape != b.shape:
        return False
    if a.dtype == torch.bfloat16:
        a, b = a.view(torch.int16), b.view(torch.int16)
    return bool(torch.equal(a, b))


class DevWeights:
    """A QWeights on the device (wq uint8, scales/biases bf16)."""

    def __init__(self, w: "synth.QWeights"):
        self.host = w
        self.wq, self.scales, self.biases = synth.weights_to_device(w)
        self.N, self.K = w.N, w.K

    def t(self):
        return self.wq, self.scales, self.biases
