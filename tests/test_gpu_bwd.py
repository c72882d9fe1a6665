"""Backward pass on the GPU (ckda_bwd_chunked) vs the float64 oracle's gradients (GPU).

The oracle (ckda_oracle_bwd) backpropagates through the token loop and is pinned to finite
differences of the forward (test_oracle_bwd.py).  The GPU backward evaluates the chunked form in
reverse in fp32 (chunk 16; the stable algebra is restated in float64 in test_chunk_backward.py).
Every gradient -- dq, dk, dv, dalpha, dbeta, dh0 -- is compared element by element with the
parity metric max|g - g_ref| / max|g_ref|.  The backward's arithmetic is fp32 throughout (bf16
inputs are read exactly), so every case is held to the fp32 bound, 1e-4; the measured errors are
5e-7 to 2e-5.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_82_b200 as ck
import oracle
import synth
from helpers import dev_act, dev_f32, fwd_case, rel_err

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dh0")
TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()


def _run(B, T, H, dk, dv, *, dtype, kind="ckda", h0_std=0.05, dhT_std=0.05, G=1, seed=0,
         nthreads=None, **kw):
    """GPU backward and oracle gradients on the same seeded inputs; returns the six errors."""
    d, g = fwd_case(B, T, H, dk, dv, kind=kind, dtype=dtype, h0_std=h0_std, seed=seed)
    if G > 1:   # q and k on H / G heads (value head h reads q/k head h // G)
        Hk = H // G
        for n in ("q", "k"):
            d[n] = np.ascontiguousarray(d[n][:, :, :Hk])
            if dtype == "bf16":
                d[n + "_bits"] = np.ascontiguousarray(d[n + "_bits"][:, :, :Hk])
            g[n] = g[n][:, :, :Hk].contiguous()
    e = synth.bwd_inputs(B, T, H, dk, dv, dtype=dtype, dhT_std=dhT_std, seed=seed + 500)
    dout = dev_act(e["dout"], e["dout_bits"], dtype)
    dhT = None if e["dhT"] is None else dev_f32(e["dhT"])
    got = ck.bwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], dout, dhT,
                         want_dh0=d["h0"] is not None, **kw)
    torch.cuda.synchronize()
    okw = {x: kw[x] for x in ("l2norm", "rope_theta", "rope_convention", "rope_dims",
                              "pos_offset") if x in kw}
    ref = oracle.bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"], e["dout"], e["dhT"],
                     nthreads=nthreads, **okw)
    errs = {}
    for n in NAMES:
        if ref[n] is None:
            continue
        errs[n] = rel_err(got[n], ref[n])
    return errs


def _check(errs, tol):
    print(" ".join(f"{n} {v:.2e}" for n, v in errs.items()))
    for n, v in errs.items():
        assert v < tol, f"{n}: {v:.3e}"


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128)])
def test_bwd_f32_sizes(dk, dv):
    _check(_run(1, 77, 2, dk, dv, dtype="f32", kind="tiny", seed=dk + dv), TOL)


@pytest.mark.parametrize("conv,dims,pos", [(0, 0, 0), (1, 0, 5), (0, 32, 65000), (1, 32, 3)])
def test_bwd_rope(conv, dims, pos):
    _check(_run(1, 50, 2, 64, 32, dtype="f32", kind="ckda", seed=11, rope_theta=10000.0,
                rope_convention=conv, rope_dims=dims, pos_offset=pos), TOL)


def test_bwd_no_norm_no_state():
    _check(_run(2, 40, 2, 32, 32, dtype="f32", kind="tiny", h0_std=0.0, dhT_std=0.0, seed=13,
                l2norm=False), TOL)


@pytest.mark.parametrize("T", [1, 15, 16, 17, 63])
def test_bwd_ragged_lengths(T):
    _check(_run(1, T, 2, 32, 16, dtype="f32", kind="tiny", seed=T), TOL)


def test_bwd_grouped_heads():
    """q, k on 2 heads serving 4 value heads: dq, dk are sums over the value heads."""
    _check(_run(1, 70, 4, 64, 64, dtype="f32", kind="ckda", G=2, seed=17, rope_theta=10000.0),
           TOL)


def test_bwd_exact_zero_and_tiny_gates():
    """Exact-zero gates and long runs of tiny gates: chunks holding them take the exact ratio
    form, which never divides by a gate (the factored form is used only where every channel's
    decay over the chunk stays >= 2^-60), so the gradients stay finite and match the
    token-by-token oracle."""
    B, T, H, dk, dv = 1, 96, 2, 32, 32
    d, g = fwd_case(B, T, H, dk, dv, kind="tiny", dtype="f32", h0_std=0.3, seed=21)
    rng = np.random.default_rng(0)
    a = d["alpha"]
    a[rng.random(a.shape) < 0.1] = 0.0
    a[:, 40:70] = np.sign(a[:, 40:70] + 1e-30) * 1e-3
    g["alpha"] = dev_f32(a)
    e = synth.bwd_inputs(B, T, H, dk, dv, dtype="f32", dhT_std=0.3, seed=22)
    got = ck.bwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"],
                         dev_f32(e["dout"]), dev_f32(e["dhT"]))
    torch.cuda.synchronize()
    ref = oracle.bwd(d["q"], d["k"], d["v"], a, d["beta"], d["h0"], e["dout"], e["dhT"])
    errs = {n: rel_err(got[n], ref[n]) for n in NAMES}
    for n in NAMES:
        assert torch.isfinite(got[n]).all()
    _check(errs, TOL)


def test_bwd_gate_logits():
    """With gate logits the gradients are those of the logits: dalpha * (1 - alpha^2) / 2 and
    dbeta * beta (1 - beta / 2), alpha and beta the activated gates (formed by the oracle)."""
    B, T, H, dk, dv = 1, 60, 2, 32, 32
    d, g = fwd_case(B, T, H, dk, dv, kind="ckda", dtype="f32", h0_std=0.05, seed=31)
    a, _, b = synth.gate_logits((B, T, H, dk), (B, T, H), 31, "f32")
    al, be = oracle.gates(a, b)
    e = synth.bwd_inputs(B, T, H, dk, dv, dtype="f32", dhT_std=0.05, seed=32)
    got = ck.bwd_chunked(g["q"], g["k"], g["v"], dev_f32(a), dev_f32(b), g["h0"],
                         dev_f32(e["dout"]), dev_f32(e["dhT"]), gate_logits=True)
    torch.cuda.synchronize()
    ref = oracle.bwd(d["q"], d["k"], d["v"], al, be, d["h0"], e["dout"], e["dhT"])
    ref["dalpha"] = ref["dalpha"] * 0.5 * (1.0 - al ** 2)
    ref["dbeta"] = ref["dbeta"] * be * (1.0 - 0.5 * be)
    _check({n: rel_err(got[n], ref[n]) for n in NAMES}, TOL)


def test_bwd_bf16_small():
    _check(_run(2, 150, 3, 128, 128, dtype="bf16", kind="ckda", seed=41, rope_theta=10000.0),
           TOL)


def test_bwd_layer_shape():
    """The 1.3B-layer-shaped workload (B=2, T=2048, H=16, dk=dv=128, bf16, CKDA gates) with a
    nonzero h0 and dhT: every gradient compared in full with the oracle's."""
    w = synth.WORKLOADS["layer_ckda_bf16"]
    _check(_run(w["B"], w["T"], w["H"], 128, 128, dtype="bf16", kind=w["kind"], seed=43,
                nthreads=8), TOL)
