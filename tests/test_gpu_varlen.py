"""Packed sequences of different lengths (cu_seqlens) on the tensor-core and SIMT forwards (GPU),
against the float64 oracle: ragged and exact-multiple lengths, single tokens, empty sequences
(hT = h0 exactly), rotary positions restarting per sequence, grouped value heads, gate logits,
more than one 1024-sequence tile of the chunk-table scan and more than one batch of empty
sequences; and, for equal lengths, bit-for-bit agreement with the batched forward.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_82_b200 as ck
import oracle
import synth
from helpers import dev_act, dev_f32, rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4    # fp32 inputs
TOL_BF16 = 1e-2   # bf16 inputs, tensor-core path


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()


def _case(lens, H, dk, dv, dtype, seed, Hk=None, logits=False):
    """Packed inputs of the given lengths; the numpy arrays drop the batch axis."""
    lens = [int(x) for x in lens]
    T = sum(lens)
    Hk = Hk or H
    d = synth.fwd_inputs(1, T, H, dk, dv, kind="ckda", dtype=dtype, seed=seed)
    g = dict(q=dev_act(d["q"], d["q_bits"], dtype)[:, :, :Hk].contiguous(),
             k=dev_act(d["k"], d["k_bits"], dtype)[:, :, :Hk].contiguous(),
             v=dev_act(d["v"], d["v_bits"], dtype), alpha=dev_f32(d["alpha"]),
             beta=dev_f32(d["beta"]))
    n = dict(q=d["q"][0, :, :Hk], k=d["k"][0, :, :Hk], v=d["v"][0], alpha=d["alpha"][0],
             beta=d["beta"][0])
    if logits:
        a, bits, b = synth.gate_logits((1, T, H, dk), (1, T, H), seed + 1, dtype)
        g["alpha"] = dev_act(a, bits, dtype)
        g["beta"] = dev_f32(b)
        n["alpha"], n["beta"] = oracle.gates(a[0], b[0])
    h0 = (0.02 * np.random.default_rng(seed + 2).standard_normal((len(lens), H, dk, dv))).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return g, n, h0, cu


def _run(g, n, h0, cu, path, chunk=64, **kw):
    cu_dev = torch.from_numpy(cu).cuda()
    h0_dev = dev_f32(h0)
    out, hT = ck.fwd_varlen(g["q"], g["k"], g["v"], g["alpha"], g["beta"], cu_dev, h0_dev,
                            chunk=chunk, path=path, **kw)
    torch.cuda.synchronize()
    kw.pop("gate_logits", None)
    o_ref, s_ref = oracle.fwd_varlen(n["q"], n["k"], n["v"], n["alpha"], n["beta"], cu, h0, **kw)
    return out, hT, o_ref, s_ref


MIXED = [130, 64, 1, 0, 200, 63, 129]


@pytest.mark.parametrize("rope", [(0.0, 0, 0), (10000.0, 0, 17), (10000.0, 1, 0)])
def test_tc_mixed_lengths(rope):
    theta, conv, pos = rope
    g, n, h0, cu = _case(MIXED, 3, 128, 128, "bf16", seed=500 + pos)
    out, hT, o_ref, s_ref = _run(g, n, h0, cu, "tc", rope_theta=theta, rope_convention=conv,
                                 pos_offset=pos)
    assert rel_err(out[0], o_ref) < TOL_BF16
    assert rel_err(hT, s_ref) < TOL_BF16
    assert torch.equal(hT[3].cpu(), torch.from_numpy(h0[3]))   # the empty sequence


def test_tc_gate_logits_and_grouped_heads():
    g, n, h0, cu = _case([100, 37, 256], 4, 128, 128, "bf16", seed=510, Hk=2, logits=True)
    out, hT, o_ref, s_ref = _run(g, n, h0, cu, "tc", gate_logits=True, rope_theta=10000.0)
    assert rel_err(out[0], o_ref) < TOL_BF16 and rel_err(hT, s_ref) < TOL_BF16


def test_tc_equal_lengths_match_the_batched_forward():
    B, T, H = 3, 150, 2
    g, n, h0, cu = _case([T] * B, H, 128, 128, "bf16", seed=520)
    cu_dev = torch.from_numpy(cu).cuda()
    kw = dict(path="tc", rope_theta=10000.0)
    out, hT = ck.fwd_varlen(g["q"], g["k"], g["v"], g["alpha"], g["beta"], cu_dev, dev_f32(h0), **kw)
    bat = {x: g[x].reshape((B, T) + tuple(g[x].shape[2:])) for x in ("q", "k", "v", "alpha", "beta")}
    ob, hb = ck.fwd_chunked(bat["q"], bat["k"], bat["v"], bat["alpha"], bat["beta"], dev_f32(h0), **kw)
    torch.cuda.synchronize()
    assert torch.equal(out.reshape(ob.shape), ob) and torch.equal(hT, hb)


def test_tc_many_short_sequences():
    # 1500 sequences (more than one tile of the table scan), most of them empty (more than one
    # batch of the empty-sequence copy), the others 1..70 tokens
    rng = np.random.default_rng(7)
    lens = np.where(rng.random(1500) < 0.75, 0, rng.integers(1, 71, 1500))
    g, n, h0, cu = _case(lens, 2, 128, 128, "bf16", seed=530)
    out, hT, o_ref, s_ref = _run(g, n, h0, cu, "tc", rope_theta=10000.0)
    assert rel_err(out[0], o_ref) < TOL_BF16 and rel_err(hT, s_ref) < TOL_BF16
    empty = np.flatnonzero(lens == 0)
    assert torch.equal(hT[torch.from_numpy(empty).cuda()].cpu(), torch.from_numpy(h0[empty]))


def test_tc_uneven_lanes():
    # 65 chunks per head: two lanes of whole sequences, 40 and 25 chunks, ragged ends
    g, n, h0, cu = _case([1536, 1024, 700, 512, 300, 24], 2, 128, 128, "bf16", seed=535)
    out, hT, o_ref, s_ref = _run(g, n, h0, cu, "tc", rope_theta=10000.0, rope_convention=1)
    assert rel_err(out[0], o_ref) < TOL_BF16 and rel_err(hT, s_ref) < TOL_BF16


@pytest.mark.parametrize("dk,dv,chunk", [(64, 64, 32), (32, 128, 16), (128, 128, 64)])
def test_simt_mixed_lengths(dk, dv, chunk):
    g, n, h0, cu = _case(MIXED, 2, dk, dv, "f32", seed=540 + dk)
    out, hT, o_ref, s_ref = _run(g, n, h0, cu, "simt", chunk=chunk, rope_theta=10000.0,
                                 rope_convention=1, pos_offset=3)
    assert rel_err(out[0], o_ref) < TOL_F32 and rel_err(hT, s_ref) < TOL_F32
    assert torch.equal(hT[3].cpu(), torch.from_numpy(h0[3]))


def test_simt_grouped_heads_no_batch_axis():
    g, n, h0, cu = _case([33, 0, 90], 4, 64, 64, "f32", seed=550, Hk=1)
    g = {x: t[0] for x, t in g.items()}   # [T, H, ...] without the batch axis
    out, hT, o_ref, s_ref = _run(g, n, h0, cu, "simt", chunk=32)
    assert out.shape == o_ref.shape
    assert rel_err(out, o_ref) < TOL_F32 and rel_err(hT, s_ref) < TOL_F32
