"""The device status word: failures the kernels detect are reported, not hidden (GPU).

The tensor-core forward bounds every wait.  A wait that runs out stops the kernel (it drains its
copies in flight, frees its Tensor Memory and returns), records a code in a per-device status
word, and leaves the context usable; ckda_last_device_status reads and clears the word.  These
tests make a wait run out in the allowed form -- a state pass over a workspace whose ready flags
nothing will ever raise, with the wait limit shortened from 4 s to 20 ms -- and pass packed
offsets whose device copy disagrees with the host copy; no test traps, faults or hangs a GPU.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_82_b200 as ck
from helpers import fwd_case, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()
    ck.last_device_status()   # start from a clear word
    yield
    ck.set_wait_limit_ns(0)


def test_clean_forward_reports_nothing():
    d, g = fwd_case(1, 200, 2, 128, 128, kind="ckda", dtype="bf16", h0_std=0.02, seed=61)
    out, hT = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], path="tc")
    assert ck.last_device_status() == 0
    o_ref, s_ref = oracle_fwd(d)
    assert rel_err(out, o_ref) < TOL and rel_err(hT, s_ref) < TOL


def test_a_wait_that_runs_out_is_reported_and_the_context_survives():
    B, T, H = 1, 192, 2
    d, g = fwd_case(B, T, H, 128, 128, kind="ckda", dtype="bf16", h0_std=0.02, seed=62)
    # a workspace whose ready flags are all zero, and only the state pass (stages = 2): every
    # chain waits for chunk factors that no kernel will produce
    ws = torch.zeros(ck.workspace_bytes(B, T, H, 128, 128), dtype=torch.uint8, device="cuda")
    out = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    hT = torch.full((B, H, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
    ck.set_wait_limit_ns(20_000_000)
    try:
        ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], path="tc", out=out,
                       hT=hT, workspace=ws, stages=2)
        assert ck.last_device_status() == 2      # a wait of the state pass ran out
    finally:
        ck.set_wait_limit_ns(0)
    assert ck.last_device_status() == 0          # read and cleared
    # the kernel gave up before writing anything
    assert torch.isnan(out.float()).all() and torch.isnan(hT).all()
    # the context is intact: a full forward afterwards is correct and reports nothing
    out2, hT2 = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"], path="tc")
    assert ck.last_device_status() == 0
    o_ref, s_ref = oracle_fwd(d)
    assert rel_err(out2, o_ref) < TOL and rel_err(hT2, s_ref) < TOL


def test_packed_offsets_that_disagree_are_reported():
    H = 2
    lens = [100, 200]
    T = sum(lens)
    d, g = fwd_case(1, T, H, 128, 128, kind="ckda", dtype="bf16", h0_std=0.02, seed=63)
    cu_host = torch.tensor([0, 100, 300], dtype=torch.int32)
    cu_dev = torch.tensor([0, 100, 280], dtype=torch.int32, device="cuda")   # ends short of T
    out = torch.full((1, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    ck.fwd_varlen(g["q"], g["k"], g["v"], g["alpha"], g["beta"], cu_dev,
                  g["h0"][:1].expand(2, -1, -1, -1).contiguous(), cu_seqlens_cpu=cu_host,
                  path="tc", out=out)
    assert ck.last_device_status() == 3
    assert ck.last_device_status() == 0
    # the chunk table was emptied: no output row was written
    assert torch.isnan(out.float()).all()
