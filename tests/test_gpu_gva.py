"""Grouped value heads (GVA): q and k with Hk heads, v / gates / states / out with H = G Hk heads
(value head h reads q/k head h // G), on the tensor-core forward, the SIMT forward and the decode
step (GPU).  Each grouped call is checked against the float64 oracle, and bit for bit against the
same call on q and k repeated explicitly to H heads (the kernels do the same arithmetic per value
head either way).
"""
import pytest
import torch

import gated_delta_rule_82_b200 as ck
import oracle
from helpers import fwd_case, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()


def _grouped(g, d, G):
    Hk = g["q"].shape[2] // G
    qk = g["q"][:, :, :Hk].contiguous()
    kk = g["k"][:, :, :Hk].contiguous()
    rep = lambda x: torch.repeat_interleave(x, G, dim=2).contiguous()
    return qk, kk, rep(qk), rep(kk), d["q"][:, :, :Hk], d["k"][:, :, :Hk]


@pytest.mark.parametrize("path,dtype,dk,chunk,tol", [("tc", "bf16", 128, 64, 1e-2),
                                                     ("simt", "f32", 64, 32, 1e-4)])
@pytest.mark.parametrize("G", [2, 4])
def test_grouped_forward(path, dtype, dk, chunk, tol, G):
    B, T, H = 2, 150, 4
    d, g = fwd_case(B, T, H, dk, dk, kind="ckda", dtype=dtype, h0_std=0.02, seed=80 + G)
    qk, kk, qr, kr, qk_np, kk_np = _grouped(g, d, G)
    kw = dict(chunk=chunk, path=path, rope_theta=10000.0)
    out, hT = ck.fwd_chunked(qk, kk, g["v"], g["alpha"], g["beta"], g["h0"], **kw)
    out_r, hT_r = ck.fwd_chunked(qr, kr, g["v"], g["alpha"], g["beta"], g["h0"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, out_r) and torch.equal(hT, hT_r)
    o_ref, s_ref = oracle.fwd(qk_np, kk_np, d["v"], d["alpha"], d["beta"], d["h0"],
                              rope_theta=10000.0)
    assert rel_err(out, o_ref) < tol and rel_err(hT, s_ref) < tol


def test_grouped_decode():
    N, H, G, dk = 8, 8, 4, 128
    d, g = fwd_case(N, 1, H, dk, dk, kind="ckda", dtype="bf16", h0_std=0.02, seed=90)
    Hk = H // G
    q = g["q"][:, 0, :Hk].contiguous()
    k = g["k"][:, 0, :Hk].contiguous()
    v, a, b = g["v"][:, 0].contiguous(), g["alpha"][:, 0].contiguous(), g["beta"][:, 0].contiguous()
    st = g["h0"].clone()
    st_r = g["h0"].clone()
    o = ck.decode_step(q, k, v, a, b, st)
    o_r = ck.decode_step(torch.repeat_interleave(q, G, dim=1).contiguous(),
                         torch.repeat_interleave(k, G, dim=1).contiguous(), v, a, b, st_r)
    torch.cuda.synchronize()
    assert torch.equal(o, o_r) and torch.equal(st, st_r)
    o_ref, s_ref = oracle.decode(d["q"][:, 0, :Hk], d["k"][:, 0, :Hk], d["v"][:, 0],
                                 d["alpha"][:, 0], d["beta"][:, 0], d["h0"])
    assert rel_err(o, o_ref) < 1e-2 and rel_err(st, s_ref) < 1e-2
