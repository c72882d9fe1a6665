"""ckda_fwd_chunked_noalloc, through the C ABI (GPU).

Some callers cannot allocate device memory at the point where they run the forward: code running
while a stream is captured into a CUDA graph, runtimes that hand out memory only from a pool
sized at start-up, real-time paths that must not call cudaMalloc or cudaFree.  This entry point
keeps its scratch in a fixed array inside the library instead of taking a workspace.  The tests
check that two calls in a row reproduce ckda_fwd_chunked with a caller-supplied workspace bit
for bit (the same kernels on the same inputs, so any difference would mean stale scratch), and
that a problem needing more scratch than the array holds is refused before anything runs.

This file is collected last on purpose, so that a run stopping at the first failure has already
run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_82_b200 as ck
from helpers import fwd_case

pytestmark = pytest.mark.gpu

LIMIT = 16 << 20            # CKDA_NOALLOC_MAX_WORKSPACE
CKDA_ERR_WORKSPACE = 5


@pytest.fixture(scope="module")
def noalloc():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_82_b200 import build
    build.build()
    lib = ck._load()
    f = lib.ckda_fwd_chunked_noalloc
    P, I, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    f.restype = I
    f.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, ck._Flags, I, LL, P]
    return f


def _call(f, g, out, hT, B, T, H):
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    flags = ck._flags(True, 0.0, 0, 0.0, ck.PATHS["tc"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(p(g["q"]), p(g["k"]), p(g["v"]), p(g["alpha"]), p(g["beta"]), p(g["h0"]), p(out),
             p(hT), B, T, H, 128, 128, 64, flags, 1, 0, stream)


def test_noalloc_matches_the_workspace_entry_point_on_two_calls(noalloc):
    B, T, H = 1, 640, 15  # 15 heads x 10 chunks = 150 chunk-heads, 13.5 MB of scratch
    assert ck.workspace_bytes(B, T, H, 128, 128, 64, torch.bfloat16, "tc") <= LIMIT
    d, g = fwd_case(B, T, H, 128, 128, kind="ckda", dtype="bf16", h0_std=0.02, seed=31)
    ref_out, ref_hT = ck.fwd_chunked(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["h0"],
                                     chunk=64, path="tc")
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        hT = torch.full((B, H, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(noalloc, g, out, hT, B, T, H) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        assert torch.equal(hT, ref_hT)


def test_noalloc_refuses_problems_over_its_scratch(noalloc):
    B, T, H = 2, 2048, 16  # 92 MB of scratch needed
    assert ck.workspace_bytes(B, T, H, 128, 128, 64, torch.bfloat16, "tc") > LIMIT
    _, g = fwd_case(B, T, H, 128, 128, kind="ckda", dtype="bf16", seed=32)
    out = torch.zeros((B, T, H, 128), dtype=torch.bfloat16, device="cuda")
    hT = torch.zeros((B, H, 128, 128), dtype=torch.float32, device="cuda")
    assert _call(noalloc, g, out, hT, B, T, H) == CKDA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(out.abs().sum().item()) == 0  # nothing ran
