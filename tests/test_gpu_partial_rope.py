"""Partial rotation (rope_dims = dk / 2: the first half of each q/k head rotated as a vector of its
own, the second half carried through, then the L2 norm over the whole head) on every kernel that
reads q and k: the prologue, the SIMT forward, the tensor-core forward and the decode step (GPU),
each against the float64 oracle, for both pairings (half-split and interleaved).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_82_b200 as ck
import oracle
import synth
from helpers import dev_act, dev_f32, fwd_case, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4    # fp32 inputs
TOL_BF16 = 1e-2   # bf16 inputs, tensor-core path


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk", [32, 64, 128])
@pytest.mark.parametrize("conv,pos", [(0, 0), (1, 9), (0, 40000)])
def test_prologue_partial(dtype, dk, conv, pos):
    d = synth.fwd_inputs(2, 37, 3, dk, dk, dtype=dtype, seed=300 + dk + pos)
    q = dev_act(d["q"], d["q_bits"], dtype)
    k = dev_act(d["k"], d["k_bits"], dtype)
    kw = dict(l2norm=True, rope_theta=10000.0, rope_convention=conv, pos_offset=pos,
              rope_dims=dk // 2)
    qo, ko = ck.qk_prologue(q, k, **kw)
    torch.cuda.synchronize()
    tol = 4e-3 if dtype == "bf16" else 2e-6
    assert rel_err(qo, oracle.prologue(d["q"], **kw)) < tol
    assert rel_err(ko, oracle.prologue(d["k"], **kw)) < tol


@pytest.mark.parametrize("dk,chunk", [(32, 16), (64, 32), (128, 64)])
@pytest.mark.parametrize("conv", [0, 1])
def test_simt_forward_partial(dk, chunk, conv):
    d, g = fwd_case(1, 90, 2, dk, dk, kind="ckda", dtype="f32", h0_std=0.02, seed=310 + dk)
    kw = dict(rope_theta=10000.0, rope_convention=conv, pos_offset=5, rope_dims=dk // 2)
    out, hT = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"],
                             chunk=chunk, path="simt", **kw)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_fwd(d, **kw)
    assert rel_err(out, o_ref) < TOL_F32 and rel_err(hT, s_ref) < TOL_F32


@pytest.mark.parametrize("conv,pos", [(0, 0), (1, 0), (0, 1000), (1, 77)])
def test_tc_forward_partial(conv, pos):
    d, g = fwd_case(2, 200, 3, 128, 128, kind="ckda", dtype="bf16", h0_std=0.02, seed=320 + pos)
    kw = dict(rope_theta=10000.0, rope_convention=conv, pos_offset=pos, rope_dims=64)
    out, hT = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"],
                             path="tc", **kw)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_fwd(d, **kw)
    assert rel_err(out, o_ref) < TOL_BF16 and rel_err(hT, s_ref) < TOL_BF16
    # the full rotation gives a different result (the partial one is not silently ignored)
    o_full, _ = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], path="tc",
                               rope_theta=10000.0, rope_convention=conv, pos_offset=pos)
    torch.cuda.synchronize()
    assert rel_err(o_full, o_ref) > 10 * TOL_BF16


@pytest.mark.parametrize("dk", [64, 128])
@pytest.mark.parametrize("conv", [0, 1])
def test_decode_partial(dk, conv):
    N, H, steps = 4, 2, 4
    st_np = synth.decode_inputs(N, H, dk, dk, dtype="f32", state_std=0.1, seed=330)["state"]
    st_dev = dev_f32(st_np)
    st_ref = st_np.astype(np.float64)
    kw = dict(rope_theta=10000.0, rope_convention=conv, rope_dims=dk // 2)
    for s in range(steps):
        d = synth.decode_inputs(N, H, dk, dk, dtype="f32", seed=331 + s, with_pos=True)
        out = ck.decode_step(dev_f32(d["q"]), dev_f32(d["k"]), dev_f32(d["v"]), dev_f32(d["alpha"]),
                             dev_f32(d["beta"]), st_dev, torch.from_numpy(d["pos"]).cuda(), **kw)
        o_ref, st_ref = oracle.decode(d["q"], d["k"], d["v"], d["alpha"], d["beta"], st_ref,
                                      d["pos"], **kw)
        torch.cuda.synchronize()
        assert rel_err(out, o_ref) < TOL_F32
    assert rel_err(st_dev, st_ref) < TOL_F32
