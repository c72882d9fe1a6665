"""The segment-parallel state pass (ckda_fwd_segmented) vs the float64 oracle (GPU).

The serial pass over the chunks is split into segments: a summary pass forms every segment's end
state from zero (from h0 for the first) and its transition F_s (the product of its chunk
transitions A_c = Diag(gamma_C) - K_end^T W), an fp32 scan forms the state entering every
segment, and a second pass runs the segments with their outputs.  The result is the recurrence's
(the "Complex KDA" paper summary, "Background" transition), so every case is held to the bf16
tensor-core bound of the plain forward, max|o - o_ref| / max|o_ref| <= 1e-2 (same for hT).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_82_b200 as ck
import oracle
import synth
from helpers import dev_act, dev_f32, fwd_case, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()


def run_seg(g, segments, **kw):
    out, hT = ck.fwd_segmented(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"],
                               segments=segments, **kw)
    torch.cuda.synchronize()
    assert ck.last_device_status() == 0
    return out, hT


def check(B, T, H, segments, *, kind="ckda", h0_std=0.0, rope=(0.0, 0), seed=0, tol=TOL):
    theta, conv = rope
    d, g = fwd_case(B, T, H, 128, 128, kind=kind, dtype="bf16", h0_std=h0_std, seed=seed)
    out, hT = run_seg(g, segments, rope_theta=theta, rope_convention=conv)
    o_ref, s_ref = oracle_fwd(d, rope_theta=theta, rope_convention=conv)
    eo, es = rel_err(out, o_ref), rel_err(hT, s_ref)
    print(f"segments {segments}: out {eo:.3e} hT {es:.3e}")
    assert eo < tol and es < tol, f"out {eo:.3e} hT {es:.3e}"
    return eo, es


@pytest.mark.parametrize("segments", [2, 3, 8, 64])
def test_segments_parity(segments):
    """64 chunks of two heads in 2, 3 (22 + 22 + 20 chunks), 8 and 64 (one chunk each)
    segments, with RoPE and a nonzero h0."""
    check(1, 4096, 2, segments, h0_std=0.05, rope=(10000.0, 0), seed=segments)


def test_segments_ragged():
    """38 chunks, the last one partial (13 tokens), in segments of 8: 5 segments, the last of 6
    chunks."""
    check(2, 64 * 37 + 13, 2, 5, h0_std=0.05, seed=5)


@pytest.mark.parametrize("T,segments", [(130, 50), (64, 8), (1, 4), (200, 0)])
def test_segments_few_chunks(T, segments):
    """More segments asked for than there are chunks (one chunk per segment, or the single
    fused launch when there is one chunk), and the automatic count (0), without h0."""
    check(1, T, 2, segments, h0_std=0.0, seed=T)


def test_segments_long_memory():
    """Slowly decaying signed gates and strong reflections from a nonzero h0: the state entering
    a segment depends on every earlier one, so the transitions F_s and the scan are exercised."""
    check(1, 8192, 2, 16, kind="longmem", h0_std=0.05, seed=41)


def test_segments_one_equals_fused():
    """segments = 1 runs the single fused launch: bit-identical to ckda_fwd_chunked."""
    d, g = fwd_case(1, 1000, 2, 128, 128, kind="ckda", dtype="bf16", h0_std=0.05, seed=3)
    o1, s1 = run_seg(g, 1)
    o2, s2 = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], chunk=64,
                            path="tc")
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_segments_state_in_place():
    """hT may be h0's own storage: h0 is read by the summary pass and the scan, hT written by the
    last pass."""
    d, g = fwd_case(1, 2048, 2, 128, 128, kind="ckda", dtype="bf16", h0_std=0.05, seed=8)
    o_ref, s_ref = oracle_fwd(d)
    st = g["h0"].clone()
    out, hT = ck.fwd_segmented(g["q"], g["k"], g["v"], g["alpha"], g["beta"], st, segments=4,
                               hT=st)
    torch.cuda.synchronize()
    assert hT.data_ptr() == st.data_ptr()
    assert rel_err(out, o_ref) < TOL and rel_err(st, s_ref) < TOL


def test_segments_grouped_heads_and_logits():
    """q/k on 2 heads serving 4 value heads, gates from bf16 logits, 6 segments."""
    B, T, H, Hk = 1, 3000, 4, 2
    d, g = fwd_case(B, T, H, 128, 128, kind="ckda", dtype="bf16", h0_std=0.02, seed=12)
    for n in ("q", "k"):
        d[n] = np.ascontiguousarray(d[n][:, :, :Hk])
        g[n] = g[n][:, :, :Hk].contiguous()
    a, a_bits, b = synth.gate_logits((B, T, H, 128), (B, T, H), 12, "bf16")
    d["alpha"], d["beta"] = oracle.gates(a, b)
    out, hT = run_seg(dict(g, alpha=dev_act(a, a_bits, "bf16"), beta=dev_f32(b)), 6,
                      gate_logits=True)
    o_ref, s_ref = oracle_fwd(d)
    assert rel_err(out, o_ref) < TOL and rel_err(hT, s_ref) < TOL


def test_segments_long_context_few_heads():
    """One sequence of 65536 tokens on two heads (the long-context workload's length with the
    heads one GPU keeps when the heads are sharded), RoPE and h0, with the model's segment
    count; every output and both final states compared."""
    w = synth.WORKLOADS["long_rope_bf16"]
    P = ck.segments_auto(1, w["T"], 2)
    assert P > 1
    check(1, w["T"], 2, P, kind=w["kind"], h0_std=w["h0_std"], rope=(w["rope_theta"], 0),
          seed=104)


def test_segments_long_context_all_heads():
    """The long-context workload (B=1, T=65536, H=16, RoPE, h0 ~ N(0, 0.02)) in 8 segments,
    compared with the oracle on every head."""
    w = synth.WORKLOADS["long_rope_bf16"]
    check(w["B"], w["T"], w["H"], 8, kind=w["kind"], h0_std=w["h0_std"],
          rope=(w["rope_theta"], 0), seed=105)
