"""Shared helpers for the GPU parity tests: move synthetic inputs to the device, run the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth


def dev_act(values: np.ndarray, bits, dtype: str, device="cuda"):
    """Device tensor holding exactly `values` (bf16 via its bit pattern, else fp32)."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32)).to(device)


def dev_f32(values, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32)).to(device)


def rel_err(got, ref) -> float:
    """max |got - ref| / max |ref| over the whole tensor (the parity metric)."""
    got = got.detach().float().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    num = np.abs(got.astype(np.float64) - ref).max()
    if den == 0:
        return float(num)
    return float(num / den)


def fwd_case(B, T, H, dk, dv, *, kind="ckda", dtype="bf16", h0_std=0.0, seed=0):
    d = synth.fwd_inputs(B, T, H, dk, dv, kind=kind, dtype=dtype, h0_std=h0_std, seed=seed)
    g = dict(q=dev_act(d["q"], d["q_bits"], dtype), k=dev_act(d["k"], d["k_bits"], dtype),
             v=dev_act(d["v"], d["v_bits"], dtype), alpha=dev_f32(d["alpha"]),
             beta=dev_f32(d["beta"]), h0=None if d["h0"] is None else dev_f32(d["h0"]))
    return d, g


def oracle_fwd(d, **kw):
    return oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"], **kw)
