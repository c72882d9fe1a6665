"""CUDA library vs the float64 oracle, element by element, on seeded synthetic inputs (GPU).

Parity metric: max|got - ref| / max|ref| over the whole tensor.  Bounds: 1e-4 for the fp32
path and 1e-2 for bf16 inputs/outputs with fp32 accumulation (final states are fp32 in both).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_82_b200 as ck
import oracle
import synth
from helpers import dev_act, dev_f32, fwd_case, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()
    torch.cuda.init()


# ---- tensor-core wrapper self-test ----------------------------------------------------------

@pytest.mark.parametrize("M", [64, 128])
@pytest.mark.parametrize("N", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("K", [64, 128, 256])
@pytest.mark.parametrize("mn", [0, 1])
def test_umma_selftest(M, N, K, mn):
    if mn and N % 64 and N != 32:
        pytest.skip("MN-major operand needs N = 32 or N % 64 == 0")
    g = torch.Generator().manual_seed(M * 1000 + N * 10 + K + mn)
    A = torch.randn(M, K, generator=g).bfloat16()
    B = torch.randn(K, N, generator=g).bfloat16() if mn else torch.randn(N, K, generator=g).bfloat16()
    D = ck.selftest_umma(A.cuda(), B.cuda(), b_mn_major=bool(mn))
    torch.cuda.synchronize()
    ref = A.double() @ (B.double() if mn else B.double().T)
    assert rel_err(D, ref.numpy()) < 1e-5


@pytest.mark.parametrize("N", [32, 64, 128])
@pytest.mark.parametrize("K", [64, 128])
@pytest.mark.parametrize("mn", [0, 1])
@pytest.mark.parametrize("how", ["cp", "st"])
def test_umma_selftest_a_in_tmem(N, K, mn, how):
    """A in Tensor Memory, read by the product from there (M = 128): staged by tcgen05.cp (one
    128x256b copy per K-step), or written by the threads with tcgen05.st (row m in lane m, K
    elements 2j and 2j + 1 in column j)."""
    if mn and N % 64 and N != 32:
        pytest.skip("MN-major operand needs N = 32 or N % 64 == 0")
    g = torch.Generator().manual_seed(7000 + N * 10 + K + mn)
    A = torch.randn(128, K, generator=g).bfloat16()
    B = torch.randn(K, N, generator=g).bfloat16() if mn else torch.randn(N, K, generator=g).bfloat16()
    D = ck.selftest_umma(A.cuda(), B.cuda(), b_mn_major=bool(mn), a_tmem=how)
    torch.cuda.synchronize()
    ref = A.double() @ (B.double() if mn else B.double().T)
    assert rel_err(D, ref.numpy()) < 1e-5


# ---- prologue: rotation then L2 norm --------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk", [16, 32, 64, 128])
@pytest.mark.parametrize("rope", [(0.0, 0, 0), (10000.0, 0, 0), (10000.0, 1, 5), (10000.0, 0, 65000)])
def test_prologue(dtype, dk, rope):
    theta, conv, pos = rope
    d = synth.fwd_inputs(2, 37, 3, dk, dk, dtype=dtype, seed=dk + int(theta) + pos)
    q = dev_act(d["q"], d["q_bits"], dtype)
    k = dev_act(d["k"], d["k_bits"], dtype)
    qo, ko = ck.qk_prologue(q, k, l2norm=True, rope_theta=theta, rope_convention=conv, pos_offset=pos)
    torch.cuda.synchronize()
    kw = dict(l2norm=True, rope_theta=theta, rope_convention=conv, pos_offset=pos)
    tol = 4e-3 if dtype == "bf16" else 2e-6
    assert rel_err(qo, oracle.prologue(d["q"], **kw)) < tol
    assert rel_err(ko, oracle.prologue(d["k"], **kw)) < tol


def test_prologue_in_place_and_no_norm():
    d = synth.fwd_inputs(1, 20, 2, 64, 64, dtype="f32", seed=3)
    q = dev_act(d["q"], None, "f32")
    k = dev_act(d["k"], None, "f32")
    ck.qk_prologue(q, k, l2norm=False, rope_theta=500.0, rope_convention=1, pos_offset=11,
                   q_out=q, k_out=k)
    torch.cuda.synchronize()
    kw = dict(l2norm=False, rope_theta=500.0, rope_convention=1, pos_offset=11)
    assert rel_err(q, oracle.prologue(d["q"], **kw)) < 2e-6
    assert rel_err(k, oracle.prologue(d["k"], **kw)) < 2e-6


# ---- decode ---------------------------------------------------------------------------------

def _decode_steps(N, H, dk, dv, steps, dtype, rope=(0.0, 0), seed=0, state_std=0.1):
    theta, conv = rope
    st_np = synth.decode_inputs(N, H, dk, dv, dtype=dtype, state_std=state_std, seed=seed)["state"]
    st_dev = dev_f32(st_np)
    st_ref = st_np.astype(np.float64)
    worst_o, worst_s = 0.0, 0.0
    for s in range(steps):
        d = synth.decode_inputs(N, H, dk, dv, dtype=dtype, seed=seed * 1000 + s + 1,
                                with_pos=theta > 0)
        pos_dev = None if d["pos"] is None else torch.from_numpy(d["pos"]).cuda()
        out = ck.decode_step(dev_act(d["q"], d["q_bits"], dtype), dev_act(d["k"], d["k_bits"], dtype),
                             dev_act(d["v"], d["v_bits"], dtype), dev_f32(d["alpha"]),
                             dev_f32(d["beta"]), st_dev, pos_dev, rope_theta=theta,
                             rope_convention=conv)
        o_ref, st_ref = oracle.decode(d["q"], d["k"], d["v"], d["alpha"], d["beta"], st_ref,
                                      d["pos"], rope_theta=theta, rope_convention=conv)
        torch.cuda.synchronize()
        worst_o = max(worst_o, rel_err(out, o_ref))
        worst_s = max(worst_s, rel_err(st_dev, st_ref))
    return worst_o, worst_s


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 16), (16, 128)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_small(dk, dv, dtype):
    eo, es = _decode_steps(5, 3, dk, dv, 6, dtype, seed=dk + dv)
    assert eo < (TOL_BF16 if dtype == "bf16" else TOL_F32)
    assert es < TOL_F32


@pytest.mark.parametrize("conv", [0, 1])
def test_decode_rope(conv):
    eo, es = _decode_steps(4, 2, 64, 64, 4, "f32", rope=(10000.0, conv), seed=7)
    assert eo < TOL_F32 and es < TOL_F32


def test_decode_batched_full_shape():
    """256 sequences x 32 heads, dk = dv = 128 (the batched-decode workload), 3 steps."""
    eo, es = _decode_steps(256, 32, 128, 128, 3, "bf16", seed=11, state_std=0.05)
    assert eo < TOL_BF16
    assert es < TOL_F32


def test_decode_batched_all_steps():
    """The batched-decode workload in full: 256 sequences x 32 heads, dk = dv = 128, 1024
    sequential steps in place on the caller's fp32 state (512 MiB).  Sequences 0-7 (256 chains of
    all 32 heads) carry seeded inputs that the oracle replays token by token -- T decode steps
    are the forward over T tokens, a pinned identity of the oracle -- and every step's output and
    the final state of those chains are compared.  The other 248 sequences carry random inputs
    that keep every launch at the full shape."""
    wd = synth.WORKLOADS["decode_bf16"]
    N, H, steps, n_chk = wd["N"], wd["H"], wd["steps"], 8
    d = synth.fwd_inputs(n_chk, steps, H, 128, 128, kind=wd["kind"], dtype="bf16", h0_std=0.05,
                         seed=51)
    o_ref, s_ref = oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"])
    step_major = lambda x: torch.from_numpy(np.ascontiguousarray(np.swapaxes(x, 0, 1)))
    chk = {n: step_major(d[n + "_bits"]).view(torch.bfloat16).cuda() for n in ("q", "k", "v")}
    chk["alpha"] = step_major(d["alpha"]).cuda()
    chk["beta"] = step_major(d["beta"]).cuda()
    pool = synth.torch_decode_inputs(4, N, H, 128, 128, kind=wd["kind"], seed=52)
    state = 0.02 * torch.randn((N, H, 128, 128), device="cuda")
    state[:n_chk] = dev_f32(d["h0"])
    outs = torch.empty((steps, n_chk, H, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((N, H, 128), dtype=torch.bfloat16, device="cuda")
    for t in range(steps):
        x = {n: pool[n][t % 4] for n in ("q", "k", "v", "alpha", "beta")}
        for n in x:
            x[n][:n_chk] = chk[n][t]
        ck.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], state, out=out)
        outs[t] = out[:n_chk]
    torch.cuda.synchronize()
    eo = rel_err(outs.permute(1, 0, 2, 3), o_ref)
    es = rel_err(state[:n_chk], s_ref)
    print(f"1024 decode steps: out {eo:.3e} state {es:.3e}")
    assert eo < TOL_BF16
    assert es < TOL_F32


# ---- chunked forward, CUDA-core path --------------------------------------------------------

def _fwd_check(B, T, H, dk, dv, chunk, *, dtype, kind="ckda", rope=(0.0, 0), pos=0, h0_std=0.0,
               path="simt", seed=0, tol_o=None, tol_s=None, want_state=True, plain=False):
    """The CUDA-core path in its record form (the binding gives it its workspace), or with
    plain=True in the form without a workspace (the chunk factors recomputed per column slice)."""
    theta, conv = rope
    d, g = fwd_case(B, T, H, dk, dv, kind=kind, dtype=dtype, h0_std=h0_std, seed=seed)
    kw = {"workspace": torch.empty(0, dtype=torch.uint8, device="cuda")} if plain else {}
    out, hT = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], chunk=chunk,
                             rope_theta=theta, rope_convention=conv, pos_offset=pos, path=path,
                             want_state=want_state, **kw)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_fwd(d, rope_theta=theta, rope_convention=conv, pos_offset=pos)
    eo = rel_err(out, o_ref)
    es = rel_err(hT, s_ref) if want_state else 0.0
    tol_o = tol_o if tol_o is not None else (TOL_BF16 if dtype == "bf16" else TOL_F32)
    tol_s = tol_s if tol_s is not None else (TOL_BF16 if dtype == "bf16" else TOL_F32)
    assert eo < tol_o, f"out rel err {eo:.3e}"
    assert es < tol_s, f"hT rel err {es:.3e}"
    return eo, es


def test_fwd_tiny_fp32():
    """The tiny fp32 workload: B=1, T=64, H=2, dk=dv=16, chunk 16, sign-magnitude gates."""
    w = synth.WORKLOADS["tiny_fp32"]
    _fwd_check(w["B"], w["T"], w["H"], w["dk"], w["dv"], w["chunk"], dtype="f32", kind="tiny")


@pytest.mark.parametrize("plain", [False, True])
@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 16), (16, 128)])
def test_fwd_simt_sizes(chunk, dk, dv, plain):
    _fwd_check(2, 100, 2, dk, dv, chunk, dtype="f32", kind="tiny", h0_std=0.5, seed=chunk + dk,
               plain=plain)


@pytest.mark.parametrize("kind", ["ckda", "kda"])
def test_fwd_simt_bf16(kind):
    _fwd_check(2, 150, 3, 64, 64, 32, dtype="bf16", kind=kind, h0_std=0.02, seed=5)


@pytest.mark.parametrize("plain", [False, True])
@pytest.mark.parametrize("conv,pos", [(0, 0), (1, 17), (0, 65000)])
def test_fwd_simt_rope(conv, pos, plain):
    _fwd_check(1, 77, 2, 32, 32, 16, dtype="f32", kind="ckda", rope=(10000.0, conv), pos=pos,
               h0_std=0.1, seed=9, plain=plain)


def test_fwd_simt_ragged_and_single_token():
    for T in (1, 15, 17, 63, 65):
        for plain in (False, True):
            _fwd_check(1, T, 2, 32, 16, 16, dtype="f32", kind="tiny", h0_std=0.3, seed=T,
                       plain=plain)


def test_fwd_simt_no_state_out():
    _fwd_check(1, 40, 1, 16, 16, 16, dtype="f32", kind="tiny", want_state=False)


def test_fwd_simt_exact_zero_and_unit_gates():
    """alpha with exact zeros and +-1 entries, beta at 0 and 2: exact-zero gates are floored at
    FLT_MIN in the log-magnitude prefix, which must not change the result."""
    d, g = fwd_case(1, 96, 2, 32, 32, kind="tiny", dtype="f32", h0_std=0.5, seed=21)
    rng = np.random.default_rng(0)
    a = d["alpha"]
    mask = rng.random(a.shape)
    a[mask < 0.1] = 0.0
    a[(mask >= 0.1) & (mask < 0.3)] = -1.0
    a[(mask >= 0.3) & (mask < 0.4)] = 1.0
    b = d["beta"]
    bm = rng.random(b.shape)
    b[bm < 0.2] = 0.0
    b[bm > 0.8] = 2.0
    g["alpha"] = dev_f32(a)
    g["beta"] = dev_f32(b)
    out, hT = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], chunk=32,
                             path="simt")
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_fwd(d)
    assert rel_err(out, o_ref) < TOL_F32
    assert rel_err(hT, s_ref) < TOL_F32


def test_fwd_simt_orthogonal_chain_norm():
    """|alpha| = 1, beta in {0, 2}, v = 0: every transition is orthogonal (Theorem 1), so the
    Frobenius norm of each head's state is preserved over 512 tokens."""
    B, T, H, dk, dv = 1, 512, 2, 32, 16
    d, g = fwd_case(B, T, H, dk, dv, kind="tiny", dtype="f32", h0_std=1.0, seed=4)
    rng = np.random.default_rng(1)
    a = rng.choice([-1.0, 1.0], size=d["alpha"].shape).astype(np.float32)
    b = rng.choice([0.0, 2.0], size=d["beta"].shape).astype(np.float32)
    v = np.zeros_like(d["v"])
    out, hT = ck.fwd_chunked(g["q"], g["k"], dev_f32(v), dev_f32(a), dev_f32(b), g["h0"], chunk=64,
                             path="simt")
    torch.cuda.synchronize()
    n0 = np.linalg.norm(d["h0"].reshape(B * H, -1), axis=1)
    n1 = np.linalg.norm(hT.cpu().numpy().reshape(B * H, -1), axis=1)
    assert np.allclose(n0, n1, rtol=1e-4)
