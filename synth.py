"""Seeded synthetic inputs for the CKDA library, its tests and its benchmark.

This module only draws random numbers and rounds them to the storage types; it holds none of the
recurrence's arithmetic, and both the CUDA library's tests and the float64 oracle consume what it
returns.  Draws use numpy's Philox counter-based generator (keyed by seed and tensor id), are
shaped in float64, rounded to float32 (round-to-nearest-even) and, for bf16 tensors, rounded
again to bf16 (round-to-nearest-even on the float32 bit pattern).  The oracle reads exactly the
rounded values.

Workload recipes (gate value distributions of the "Complex KDA" paper summary, "CKDA
Definition": alpha in [-1, 1]^dk, beta in [0, 2]):

  ``tiny``     q, k, v ~ N(0,1); alpha = s*m, s = +-1 (p = 1/2), m ~ U[0.05, 1]; beta ~ U[0, 2]
  ``ckda``     alpha = s*exp(-softplus(z)), z ~ N(0,1), |alpha| >= 1e-3; beta = 2*sigmoid(N(0,1))
  ``kda``      alpha = exp(-softplus(z)) in (0, 1]; beta = sigmoid(N(0,1)) in [0, 1]
  ``longmem``  alpha = s*m, s = +-1 (p = 1/2), m ~ U[0.95, 1]; beta ~ U[1.5, 2] (slow decay and
               strong reflections: the state keeps a memory over many chunks)
  ``orth``     alpha = +-1 (p = 1/2); beta = 2 (every transition orthogonal: the rotation regime
               of the paper summary's Theorem 1, nothing decays)

Gate logits (the optional input form whose activations 2 sigmoid(a) - 1 and 2 sigmoid(b) the
library and the oracle form themselves): a = s * (1 + 2|z|), s = +-1 (p = 1/2), z ~ N(0,1),
rounded to the activation dtype; b ~ N(0,1) in float32.
"""
from __future__ import annotations

import numpy as np

TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "alpha": 4, "beta": 5, "h0": 6, "pos": 7, "dout": 8,
              "dhT": 9}


def _gen(seed: int, tensor: str) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[int(seed) & (2**64 - 1), TENSOR_IDS[tensor]]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(seed, tensor, shape):
    return _gen(seed, tensor).standard_normal(size=shape, dtype=np.float64)


def _softplus(z):
    return np.logaddexp(0.0, z)


def _sigmoid(z):
    return 0.5 * (1.0 + np.tanh(0.5 * z))


def gates(kind: str, shape_alpha, shape_beta, seed: int):
    """(alpha float32 [.., dk], beta float32 [..]) for one of the recipes above."""
    ga, gb = _gen(seed, "alpha"), _gen(seed, "beta")
    if kind == "tiny":
        s = np.where(ga.random(size=shape_alpha) < 0.5, -1.0, 1.0)
        m = ga.uniform(0.05, 1.0, size=shape_alpha)
        alpha = s * m
        beta = gb.uniform(0.0, 2.0, size=shape_beta)
    elif kind == "ckda":
        z = ga.standard_normal(size=shape_alpha)
        s = np.where(ga.random(size=shape_alpha) < 0.5, -1.0, 1.0)
        alpha = s * np.maximum(np.exp(-_softplus(z)), 1e-3)
        beta = 2.0 * _sigmoid(gb.standard_normal(size=shape_beta))
    elif kind == "kda":
        z = ga.standard_normal(size=shape_alpha)
        alpha = np.exp(-_softplus(z))
        beta = _sigmoid(gb.standard_normal(size=shape_beta))
    elif kind == "longmem":
        s = np.where(ga.random(size=shape_alpha) < 0.5, -1.0, 1.0)
        alpha = s * ga.uniform(0.95, 1.0, size=shape_alpha)
        beta = gb.uniform(1.5, 2.0, size=shape_beta)
    elif kind == "orth":
        alpha = np.where(ga.random(size=shape_alpha) < 0.5, -1.0, 1.0)
        beta = np.full(shape_beta, 2.0)
    else:
        raise ValueError(f"unknown gate recipe {kind!r}")
    return alpha.astype(np.float32), beta.astype(np.float32)


def gate_logits(shape_alpha, shape_beta, seed: int, dtype: str):
    """(a float32 values, a bf16 bits or None, b float32) for the gate-logit recipe above."""
    ga, gb = _gen(seed, "alpha"), _gen(seed, "beta")
    s = np.where(ga.random(size=shape_alpha) < 0.5, -1.0, 1.0)
    a = (s * (1.0 + 2.0 * np.abs(ga.standard_normal(size=shape_alpha)))).astype(np.float32)
    bits = None
    if dtype == "bf16":
        bits = f32_to_bf16_bits(a)
        a = bf16_bits_to_f32(bits)
    b = gb.standard_normal(size=shape_beta).astype(np.float32)
    return a, bits, b


def _activation(seed, tensor, shape, dtype):
    x = _normal(seed, tensor, shape).astype(np.float32)
    if dtype == "bf16":
        bits = f32_to_bf16_bits(x)
        return bf16_bits_to_f32(bits), bits
    return x, None


def fwd_inputs(B, T, H, dk, dv, *, kind="ckda", dtype="bf16", h0_std=0.0, seed=0):
    """Inputs of one chunked forward call.

    Returns a dict of numpy arrays: q, k [B,T,H,dk], v [B,T,H,dv] as float32 holding the exact
    values the library reads (bf16-representable when dtype == "bf16"), their bf16 bit patterns
    under q_bits/k_bits/v_bits (bf16 only), alpha [B,T,H,dk] float32, beta [B,T,H] float32 and
    h0 [B,H,dk,dv] float32 (None when h0_std == 0).
    """
    d = {}
    for name, last in (("q", dk), ("k", dk), ("v", dv)):
        val, bits = _activation(seed, name, (B, T, H, last), dtype)
        d[name] = val
        d[name + "_bits"] = bits
    d["alpha"], d["beta"] = gates(kind, (B, T, H, dk), (B, T, H), seed)
    if h0_std > 0:
        d["h0"] = (h0_std * _normal(seed, "h0", (B, H, dk, dv))).astype(np.float32)
    else:
        d["h0"] = None
    d["meta"] = dict(B=B, T=T, H=H, dk=dk, dv=dv, kind=kind, dtype=dtype, seed=seed)
    return d


def bwd_inputs(B, T, H, dk, dv, *, dtype="bf16", dhT_std=0.0, seed=0):
    """Output gradients for a backward call: dout [B,T,H,dv] ~ N(0,1) in the activation dtype
    (float32 values, bf16 bit patterns under dout_bits) and dhT [B,H,dk,dv] ~ N(0, dhT_std^2)
    float32 (None when dhT_std == 0)."""
    val, bits = _activation(seed, "dout", (B, T, H, dv), dtype)
    d = {"dout": val, "dout_bits": bits}
    d["dhT"] = ((dhT_std * _normal(seed, "dhT", (B, H, dk, dv))).astype(np.float32)
                if dhT_std > 0 else None)
    return d


def decode_inputs(N, H, dk, dv, *, kind="ckda", dtype="bf16", state_std=0.0, seed=0,
                  with_pos=False, max_pos=65536):
    """Inputs of one decode step (same conventions as fwd_inputs, without the T axis)."""
    d = fwd_inputs(N, 1, H, dk, dv, kind=kind, dtype=dtype, seed=seed)
    out = {}
    for name in ("q", "k", "v", "alpha"):
        out[name] = d[name][:, 0]
    for name in ("q_bits", "k_bits", "v_bits"):
        out[name] = None if d[name] is None else d[name][:, 0]
    out["beta"] = d["beta"][:, 0]
    if state_std > 0:
        out["state"] = (state_std * _normal(seed, "h0", (N, H, dk, dv))).astype(np.float32)
    else:
        out["state"] = np.zeros((N, H, dk, dv), np.float32)
    out["pos"] = (_gen(seed, "pos").integers(0, max_pos, size=(N,), dtype=np.int64)
                  if with_pos else None)
    return out


# Named workloads: shapes and recipes of the benchmark and parity configurations.
WORKLOADS = {
    # tiny fp32 forward (oracle finishes instantly)
    "tiny_fp32": dict(B=1, T=64, H=2, dk=16, dv=16, chunk=16, kind="tiny", dtype="f32",
                      rope_theta=0.0, h0_std=0.0),
    # 1.3B-layer-shaped forward, CKDA gate range
    "layer_ckda_bf16": dict(B=2, T=2048, H=16, dk=128, dv=128, chunk=64, kind="ckda",
                            dtype="bf16", rope_theta=0.0, h0_std=0.0),
    # same shape, standard KDA gate range
    "layer_kda_bf16": dict(B=2, T=2048, H=16, dk=128, dv=128, chunk=64, kind="kda",
                           dtype="bf16", rope_theta=0.0, h0_std=0.0),
    # long context with RoPE (theta 10000, half-split) and a nonzero initial state
    "long_rope_bf16": dict(B=1, T=65536, H=16, dk=128, dv=128, chunk=64, kind="ckda",
                           dtype="bf16", rope_theta=10000.0, h0_std=0.02),
    # packed sequences of different lengths (ragged ends, one short sequence) with the layer
    # shape's token count and heads
    "packed_bf16": dict(lens=[1536, 1024, 700, 512, 300, 24], H=16, dk=128, dv=128, chunk=64,
                        kind="ckda", dtype="bf16"),
    # batched decode: 256 sequences x 32 heads, 1024 steps
    "decode_bf16": dict(N=256, H=32, dk=128, dv=128, steps=1024, kind="ckda", dtype="bf16"),
}


# ---- device-side generation for benchmark-sized inputs -----------------------------------------
# Same recipes as above, drawn with torch's seeded CUDA generator (Philox) so that multi-GB
# inputs never pass through the host.  Values follow the same distributions but are not the
# same numbers as the numpy stream; parity tests use the numpy path.

def torch_gates(kind, shape_alpha, shape_beta, gen, device):
    import torch
    if kind == "ckda":
        z = torch.randn(shape_alpha, generator=gen, device=device, dtype=torch.float32)
        s = torch.where(torch.rand(shape_alpha, generator=gen, device=device) < 0.5, -1.0, 1.0)
        alpha = s * torch.clamp(torch.exp(-torch.nn.functional.softplus(z)), min=1e-3)
        beta = 2.0 * torch.sigmoid(torch.randn(shape_beta, generator=gen, device=device))
    elif kind == "kda":
        z = torch.randn(shape_alpha, generator=gen, device=device, dtype=torch.float32)
        alpha = torch.exp(-torch.nn.functional.softplus(z))
        beta = torch.sigmoid(torch.randn(shape_beta, generator=gen, device=device))
    elif kind == "tiny":
        s = torch.where(torch.rand(shape_alpha, generator=gen, device=device) < 0.5, -1.0, 1.0)
        alpha = s * (0.05 + 0.95 * torch.rand(shape_alpha, generator=gen, device=device))
        beta = 2.0 * torch.rand(shape_beta, generator=gen, device=device)
    else:
        raise ValueError(kind)
    return alpha.contiguous(), beta.contiguous()


def torch_fwd_inputs(B, T, H, dk, dv, *, kind="ckda", dtype="bf16", h0_std=0.0, seed=0,
                     device="cuda", gate_logits=False):
    """Device-side draws of the same recipes (torch's seeded generator).  With gate_logits,
    alpha and beta hold logits of the gate-logit recipe (alpha in the activation dtype)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = {}
    for name, last in (("q", dk), ("k", dk), ("v", dv)):
        d[name] = torch.randn((B, T, H, last), generator=gen, device=device).to(tdt)
    if gate_logits:
        s = torch.where(torch.rand((B, T, H, dk), generator=gen, device=device) < 0.5, -1.0, 1.0)
        z = torch.randn((B, T, H, dk), generator=gen, device=device)
        d["alpha"] = (s * (1.0 + 2.0 * z.abs())).to(tdt).contiguous()
        d["beta"] = torch.randn((B, T, H), generator=gen, device=device).contiguous()
    else:
        d["alpha"], d["beta"] = torch_gates(kind, (B, T, H, dk), (B, T, H), gen, device)
    d["h0"] = (h0_std * torch.randn((B, H, dk, dv), generator=gen, device=device)
               if h0_std > 0 else None)
    return d


def torch_decode_inputs(steps, N, H, dk, dv, *, kind="ckda", dtype="bf16", seed=0,
                        device="cuda"):
    """Per-step decode inputs for `steps` steps, stacked on a leading axis."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = {}
    for name, last in (("q", dk), ("k", dk), ("v", dv)):
        d[name] = torch.randn((steps, N, H, last), generator=gen, device=device).to(tdt)
    d["alpha"], d["beta"] = torch_gates(kind, (steps, N, H, dk), (steps, N, H), gen, device)
    return d
