"""Shared helpers for the GPU parity tests: uploads and the tolerance check.

Tolerance (bf16 output y, fp32 accumulation on the device, fp64 oracle):
  * elementwise |y - y_ref| <= 1e-2 * rms(y_ref) + 1/2 ulp_bf16(y_ref): the stated bound plus the
    final rounding to bf16, which alone exceeds 1e-2*rms for |y| above ~2.6 rms;
  * relative L1 error sum|y - y_ref| / sum|y_ref| <= 2e-3.
The fp32 debug output (no final rounding) must meet the literal 1e-2*rms bound.
"""
from __future__ import annotations

import numpy as np
import torch

MAX_REL_RMS = 1e-2
MEAN_REL = 2e-3


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def f16_bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def host_f64(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 0.5 * np.exp2(e - 7)


def check_close(y: np.ndarray, ref: np.ndarray, bf16_out: bool, what: str = ""):
    rms = float(np.sqrt(np.mean(ref ** 2)))
    d = np.abs(y - ref)
    bound = MAX_REL_RMS * rms + (bf16_half_ulp(ref) if bf16_out else 0.0)
    bad = np.nonzero(d > bound)
    assert bad[0].size == 0, (f"{what}: {bad[0].size} elements over the bound; worst |d|={d.max():.3e} "
                              f"rms={rms:.3e} at {np.unravel_index(np.argmax(d - bound), d.shape)}")
    rel = float(d.sum() / max(np.abs(ref).sum(), 1e-300))
    assert rel <= MEAN_REL, f"{what}: relative L1 error {rel:.3e} > {MEAN_REL}"
    return {"max_abs_over_rms": float(d.max() / rms) if rms else 0.0, "rel_l1": rel,
            "literal_violations": int((d > MAX_REL_RMS * rms).sum())}
