"""Gates given as logits (flags.gate_logits): the kernels form alpha = 2 sigma(a) - 1 and
beta = 2 sigma(b) ("Complex KDA" paper summary, Methodology, CKDA Definition); the oracle forms the
same gates in float64 from the same logits (GPU).  Tolerances as for gate values: 1e-2 with bf16
activations, 1e-4 with fp32."""
import numpy as np
import pytest
import torch

import gated_delta_rule_82_b200 as ck
import oracle
import synth
from helpers import dev_act, dev_f32, fwd_case, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()


def logit_case(B, T, H, dk, dv, dtype, seed, h0_std=0.02):
    d, g = fwd_case(B, T, H, dk, dv, kind="ckda", dtype=dtype, h0_std=h0_std, seed=seed)
    a, abits, b = synth.gate_logits((B, T, H, dk), (B, T, H), seed, dtype)
    g["alpha"] = dev_act(a, abits, dtype)
    g["beta"] = dev_f32(b)
    d["alpha"], d["beta"] = oracle.gates(a, b)
    return d, g


def run(g, path, chunk=64, **kw):
    out, hT = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], chunk=chunk,
                             path=path, gate_logits=True, **kw)
    torch.cuda.synchronize()
    return out, hT


@pytest.mark.parametrize("T", [64, 300])
def test_tc_logits(T):
    d, g = logit_case(1, T, 2, 128, 128, "bf16", seed=31 + T)
    out, hT = run(g, "tc")
    o_ref, s_ref = oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"])
    assert rel_err(out, o_ref) < 1e-2
    assert rel_err(hT, s_ref) < 1e-2


def test_tc_logits_layer_shape_with_rope():
    w = synth.WORKLOADS["layer_ckda_bf16"]
    d, g = logit_case(w["B"], w["T"], w["H"], 128, 128, "bf16", seed=37)
    kw = dict(rope_theta=10000.0, rope_convention=0)
    out, hT = run(g, "tc", **kw)
    o_ref, s_ref = oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"], **kw)
    assert rel_err(out, o_ref) < 1e-2
    assert rel_err(hT, s_ref) < 1e-2


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-4), ("bf16", 1e-2)])
def test_simt_logits(dtype, tol):
    d, g = logit_case(2, 100, 3, 64, 32, dtype, seed=41)
    out, hT = run(g, "simt", chunk=32)
    o_ref, s_ref = oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"])
    assert rel_err(out, o_ref) < tol
    assert rel_err(hT, s_ref) < tol


def test_tc_logits_match_gate_values():
    """The same problem with the gates passed as values (formed on the host in float64, rounded to
    fp32) agrees with the logit form to the bf16 tolerance."""
    d, g = logit_case(1, 200, 2, 128, 128, "bf16", seed=43)
    o1, s1 = run(g, "tc")
    o2, s2 = ck.fwd_chunked(g["q"], g["k"], g["v"], dev_f32(d["alpha"]), dev_f32(d["beta"]),
                            g["h0"], chunk=64, path="tc")
    torch.cuda.synchronize()
    assert rel_err(o1, o2.float().cpu().numpy()) < 1e-2
    assert rel_err(s1, s2.cpu().numpy()) < 1e-2


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-4), ("bf16", 4e-3)])
def test_decode_logits(dtype, tol):
    N, H, dk, dv = 3, 4, 64, 128
    d = synth.decode_inputs(N, H, dk, dv, kind="ckda", dtype=dtype, state_std=0.05, seed=47)
    a, abits, b = synth.gate_logits((N, H, dk), (N, H), 47, dtype)
    al, be = oracle.gates(a, b)
    st = dev_f32(d["state"])
    out = ck.decode_step(dev_act(d["q"], d["q_bits"], dtype), dev_act(d["k"], d["k_bits"], dtype),
                         dev_act(d["v"], d["v_bits"], dtype), dev_act(a, abits, dtype), dev_f32(b),
                         st, gate_logits=True)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.decode(d["q"], d["k"], d["v"], al, be, d["state"])
    assert rel_err(out, o_ref) < tol
    assert rel_err(st, s_ref) < 1e-5
