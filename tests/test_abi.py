"""The C-ABI library: it loads, exports every entry point its header declares, and validates
arguments on the host.  CPU only: every call below carries at least one invalid argument, so the
library rejects it before any launch (nothing here ever reaches a kernel)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_82_b200 as ck
from gated_delta_rule_82_b200 import build as ckbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ckda.h")

OK, NULL, SHAPE, UNSUP, ALIGN, WORKSPACE, CUDA, ARG, DEVICE_STATUS = range(9)
P = 0x10000  # a 16-byte-aligned fake address; never dereferenced (calls fail validation first)


@pytest.fixture(scope="module")
def lib():
    ckbuild.build()
    return ck._load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ckda_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("ckda_fwd_chunked", "ckda_decode_step", "ckda_fwd_workspace_bytes",
                 "ckda_qk_prologue", "ckda_strerror", "ckda_abi_version", "ckda_fwd_varlen",
                 "ckda_fwd_varlen_workspace_bytes", "ckda_last_device_status",
                 "ckda_set_wait_limit_ns", "ckda_fwd_chunked_noalloc", "ckda_fwd_segmented",
                 "ckda_fwd_segmented_workspace_bytes", "ckda_fwd_segments_auto",
                 "ckda_fwd_simt_workspace_bytes"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in ckda.h but not exported"


def test_only_declared_symbols_are_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ck.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and "ckda" in l}
    assert exported == set(declared_functions())


def test_version_and_strerror(lib):
    assert ck.abi_version() == 7
    for s in range(9):
        assert lib.ckda_strerror(s)
    assert lib.ckda_strerror(99) == b"unknown status"


def flags(**kw):
    f = dict(l2norm=1, rope_theta=0.0, rope_convention=0, scale=0.0, path=0, stages=0,
             gate_logits=0, rope_dims=0, qk_heads=0)
    f.update(kw)
    return ck._Flags(f["l2norm"], f["rope_theta"], f["rope_convention"], f["scale"], f["path"],
                     f["stages"], f["gate_logits"], f["rope_dims"], f["qk_heads"])


def fwd(lib, q=P, k=2 * P, v=3 * P, a=4 * P, b=5 * P, h0=None, out=6 * P, hT=None, B=1, T=8,
        H=1, dk=16, dv=16, chunk=16, fl=None, dtype=1, pos=0, ws=None, wsb=0):
    fl = fl or flags()
    c = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.ckda_fwd_chunked(c(q), c(k), c(v), c(a), c(b), c(h0), c(out), c(hT), B, T, H, dk,
                                dv, chunk, fl, dtype, pos, c(ws), wsb, None)


# each case is invalid in exactly the stated way
@pytest.mark.parametrize("kw,want", [
    (dict(q=None), NULL), (dict(v=None), NULL), (dict(out=None), NULL), (dict(b=None), NULL),
    (dict(T=0), SHAPE), (dict(B=0), SHAPE), (dict(H=-1), SHAPE),
    (dict(dk=24), UNSUP), (dict(dv=256), UNSUP), (dict(chunk=128), UNSUP), (dict(dtype=7), UNSUP),
    (dict(q=P + 8), ALIGN), (dict(a=4 * P + 4), ALIGN), (dict(hT=7 * P + 2), ALIGN),
    (dict(out=P), ARG),                       # out aliases q
    (dict(fl=flags(path=2)), UNSUP),          # tensor-core path needs bf16 128/128/64
    (dict(fl=flags(path=9)), ARG),
    (dict(fl=flags(stages=4)), ARG),
    (dict(fl=flags(rope_theta=1e4, rope_convention=3)), ARG),
    (dict(fl=flags(gate_logits=2)), ARG),
    (dict(fl=flags(qk_heads=-1)), ARG),
    (dict(dk=32, dv=16, fl=flags(rope_theta=1e4, rope_dims=12)), ARG),   # neither dk nor dk / 2
    (dict(fl=flags(rope_theta=1e4, rope_dims=8)), ARG),                  # dk / 2 needs dk >= 32
    (dict(H=4, fl=flags(qk_heads=3)), ARG),   # q/k heads must divide the value heads
    (dict(dk=128, dv=128, chunk=64, T=64, q=P, k=P * 9, v=P * 17, a=P * 25, b=P * 40,
          out=P * 50, ws=None), WORKSPACE),   # tensor-core path without workspace
])
def test_fwd_validation(lib, kw, want):
    assert fwd(lib, **kw) == want


def test_workspace_query(lib):
    n = lib.ckda_fwd_workspace_bytes(2, 2048, 16, 128, 128, 64, 1, 0)
    assert 0 < n < (1 << 40)
    assert lib.ckda_fwd_workspace_bytes(2, 2048, 16, 128, 128, 64, 1, 1) == 0  # SIMT: none
    assert lib.ckda_fwd_workspace_bytes(1, 64, 2, 16, 16, 16, 0, 0) == 0
    bad = ctypes.c_size_t(-1).value
    assert lib.ckda_fwd_workspace_bytes(1, 64, 2, 16, 16, 16, 0, 2) == bad
    assert lib.ckda_fwd_workspace_bytes(1, 0, 2, 16, 16, 16, 0, 0) == bad
    assert lib.ckda_fwd_workspace_bytes(1, 64, 2, 48, 16, 16, 0, 0) == bad


def fwd_seg(lib, q=P, k=9 * P, v=17 * P, a=25 * P, b=40 * P, h0=None, out=50 * P, hT=None, B=1,
            T=256, H=1, dk=128, dv=128, fl=None, dtype=1, pos=0, segments=2, ws=60 * P,
            wsb=1 << 40):
    fl = fl or flags()
    c = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.ckda_fwd_segmented(c(q), c(k), c(v), c(a), c(b), c(h0), c(out), c(hT), B, T, H,
                                  dk, dv, fl, dtype, pos, segments, c(ws), wsb, None)


# each case is invalid in exactly the stated way (nothing is launched: no GPU needed)
@pytest.mark.parametrize("kw,want", [
    (dict(segments=0), ARG), (dict(segments=-3), ARG),
    (dict(dtype=0), UNSUP),                   # fp32: no tensor-core path
    (dict(dk=64, dv=64), UNSUP),
    (dict(fl=flags(path=1)), UNSUP),          # the CUDA-core path has no segments
    (dict(q=None), NULL), (dict(T=0), SHAPE), (dict(q=P + 8), ALIGN),
    (dict(out=P), ARG),                       # out aliases q
    (dict(ws=None, wsb=0), WORKSPACE),
    (dict(wsb=1024), WORKSPACE),
])
def test_segmented_validation(lib, kw, want):
    assert fwd_seg(lib, **kw) == want


def test_simt_workspace_query(lib):
    # the record form of the CUDA-core path: 7056 floats per 16-token chunk and head at dk = 128
    assert lib.ckda_fwd_simt_workspace_bytes(2, 2048, 16, 128, 128) == 2 * 16 * 128 * 7056 * 4
    assert lib.ckda_fwd_simt_workspace_bytes(1, 17, 1, 16, 16) == 2 * (3 * 16 * 16 + 3 * 256 + 16 + 16) * 4
    bad = ctypes.c_size_t(-1).value
    assert lib.ckda_fwd_simt_workspace_bytes(1, 0, 1, 16, 16) == bad
    assert lib.ckda_fwd_simt_workspace_bytes(1, 64, 1, 24, 16) == bad


def test_segmented_workspace_and_count(lib):
    plain = lib.ckda_fwd_workspace_bytes(1, 65536, 2, 128, 128, 64, 1, 0)
    assert lib.ckda_fwd_segmented_workspace_bytes(1, 65536, 2, 128, 128, 1) == plain
    # 1024 chunks in 32 segments of 32: three fp32 arrays of 2 x 32 matrices of 64 KiB beyond it
    n32 = lib.ckda_fwd_segmented_workspace_bytes(1, 65536, 2, 128, 128, 32)
    assert n32 >= plain + 3 * 2 * 32 * 65536 and n32 - plain < 3 * 2 * 32 * 65536 + 256
    # 5 chunks asked for 4 segments: L = 2, so 3 segments
    n4 = lib.ckda_fwd_segmented_workspace_bytes(1, 320, 1, 128, 128, 4)
    assert n4 - lib.ckda_fwd_workspace_bytes(1, 320, 1, 128, 128, 64, 1, 0) < 3 * 3 * 65536 + 256
    bad = ctypes.c_size_t(-1).value
    assert lib.ckda_fwd_segmented_workspace_bytes(1, 256, 1, 64, 128, 2) == bad
    assert lib.ckda_fwd_segmented_workspace_bytes(1, 256, 1, 128, 128, 0) == bad
    # the model: few heads over a long sequence are chain-bound (segments); the layer shape's
    # 32 heads keep every SM busy (one fused launch)
    assert lib.ckda_fwd_segments_auto(1, 65536, 2) > 1
    assert lib.ckda_fwd_segments_auto(2, 2048, 16) == 1
    assert lib.ckda_fwd_segments_auto(1, 64, 1) == 1


def host_offsets(vals):
    return (ctypes.c_int * len(vals))(*vals)


def fwd_varlen(lib, q=P, k=2 * P, v=3 * P, a=4 * P, b=5 * P, h0=None, out=6 * P, hT=None,
               cu=8 * P, cu_host=(0, 5, 8), n=None, H=1, dk=16, dv=16, chunk=16, fl=None, dtype=1,
               ws=None, wsb=0):
    fl = fl or flags()
    c = lambda x: None if x is None else ctypes.c_void_p(x)
    host = None if cu_host is None else host_offsets(cu_host)
    n = (len(cu_host) - 1 if cu_host else 1) if n is None else n
    return lib.ckda_fwd_varlen(c(q), c(k), c(v), c(a), c(b), c(h0), c(out), c(hT), c(cu),
                               None if host is None else ctypes.cast(host, ctypes.c_void_p), n, H,
                               dk, dv, chunk, fl, dtype, 0, c(ws), wsb, None)


# each case is invalid in exactly the stated way
@pytest.mark.parametrize("kw,want", [
    (dict(cu=None), NULL), (dict(cu_host=None), NULL), (dict(q=None), NULL),
    (dict(cu=8 * P + 2), ALIGN),
    (dict(n=0), SHAPE),
    (dict(cu_host=(1, 5, 8)), ARG),          # offsets must start at 0
    (dict(cu_host=(0, 6, 5, 8)), ARG),       # and never decrease
    (dict(dk=24), UNSUP),
    (dict(out=P), ARG),                      # out aliases q
    (dict(fl=flags(qk_heads=-1)), ARG),
    (dict(dk=128, dv=128, chunk=64, cu_host=(0, 70, 100), q=P, k=P * 9, v=P * 17, a=P * 25,
          b=P * 40, out=P * 50, ws=None), WORKSPACE),   # tensor-core path without workspace
])
def test_fwd_varlen_validation(lib, kw, want):
    assert fwd_varlen(lib, **kw) == want


def test_varlen_workspace_query(lib):
    q = lambda vals, H=16, path=0, dk=128: lib.ckda_fwd_varlen_workspace_bytes(
        ctypes.cast(host_offsets(vals), ctypes.c_void_p), len(vals) - 1, H, dk, 128, 64, 1, path)
    bad = ctypes.c_size_t(-1).value
    one = q((0, 64))                            # one chunk per head
    assert 0 < one < (1 << 40)
    # chunks are counted per sequence: 70 + 30 tokens make 2 + 1 chunks, one sequence of 100 two
    assert q((0, 70, 100)) > q((0, 100)) > one
    assert q((0, 64, 64, 128)) == q((0, 128))   # an empty sequence adds no chunk
    assert q((0, 100), path=1) == 0             # SIMT: none
    assert q((0, 100), dk=48) == bad
    assert q((0, 50, 40)) == bad                # decreasing offsets


def dec(lib, q=P, k=2 * P, v=3 * P, a=4 * P, b=5 * P, st=6 * P, out=7 * P, pos=None, N=2, H=2,
        dk=16, dv=16, fl=None, dtype=1):
    fl = fl or flags()
    c = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.ckda_decode_step(c(q), c(k), c(v), c(a), c(b), c(st), c(out), c(pos), N, H, dk,
                                dv, fl, dtype, None)


@pytest.mark.parametrize("kw,want", [
    (dict(st=None), NULL), (dict(q=None), NULL),
    (dict(fl=flags(rope_theta=1e4)), NULL),   # rotation needs positions
    (dict(N=0), SHAPE), (dict(dk=8), UNSUP), (dict(dtype=3), UNSUP),
    (dict(st=6 * P + 4), ALIGN), (dict(out=3 * P), ARG),
    (dict(fl=flags(gate_logits=-1)), ARG),
    (dict(fl=flags(qk_heads=-2)), ARG), (dict(H=2, fl=flags(qk_heads=3)), ARG),
])
def test_decode_validation(lib, kw, want):
    assert dec(lib, **kw) == want


def test_prologue_validation(lib):
    c = ctypes.c_void_p
    f = flags()
    assert lib.ckda_qk_prologue(None, c(P), c(2 * P), c(3 * P), 1, 4, 1, 16, f, 1, 0, None) == NULL
    assert lib.ckda_qk_prologue(c(P), c(2 * P), c(3 * P), c(4 * P), 1, 4, 1, 12, f, 1, 0, None) == UNSUP
    assert lib.ckda_qk_prologue(c(P), c(2 * P), c(3 * P + 2), c(4 * P), 1, 4, 1, 16, f, 1, 0, None) == ALIGN
    assert lib.ckda_qk_prologue(c(P), c(2 * P), c(2 * P), c(4 * P), 1, 4, 1, 16, f, 1, 0, None) == ARG
    assert lib.ckda_qk_prologue(c(P), c(2 * P), c(3 * P), c(4 * P), 0, 4, 1, 16, f, 1, 0, None) == SHAPE


def test_selftest_validation(lib):
    c = ctypes.c_void_p
    assert lib.ckda_selftest_umma(c(P), c(2 * P), None, 64, 64, 64, 0, None) == NULL
    assert lib.ckda_selftest_umma(c(P), c(2 * P), c(3 * P), 32, 64, 64, 0, None) == UNSUP
    assert lib.ckda_selftest_umma(c(P), c(2 * P), c(3 * P), 64, 48, 64, 1, None) == UNSUP
    assert lib.ckda_selftest_umma(c(P), c(2 * P), c(3 * P), 64, 64, 96, 0, None) == UNSUP
    assert lib.ckda_selftest_umma(c(P), c(2 * P), c(3 * P), 64, 64, 64, 2, None) == UNSUP  # A in TMEM: M = 128
    assert lib.ckda_selftest_umma(c(P), c(2 * P), c(3 * P), 64, 64, 64, 4, None) == UNSUP  # A in TMEM: M = 128
    assert lib.ckda_selftest_umma(c(P), c(2 * P), c(3 * P), 128, 64, 64, 6, None) == ARG
    assert lib.ckda_selftest_umma(c(P), c(2 * P), c(3 * P), 128, 64, 64, 8, None) == ARG


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 16)
    with pytest.raises(ValueError, match="CUDA"):
        ck.qk_prologue(x, x)


@pytest.mark.parametrize("stages", [1, 2, 4, -1])
def test_noalloc_refuses_split_stages(lib, stages):
    """The library-owned scratch of ckda_fwd_chunked_noalloc is shared by every call, so the
    profiling stages that split one forward across two calls (and invalid stages) are refused
    before anything else is looked at."""
    f = lib.ckda_fwd_chunked_noalloc
    f.restype = ctypes.c_int
    P_, I_ = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P_] * 8 + [I_] * 6 + [ck._Flags, I_, ctypes.c_longlong, P_]
    c = ctypes.c_void_p
    st = f(c(P), c(2 * P), c(3 * P), c(4 * P), c(5 * P), None, c(6 * P), None, 1, 64, 1, 128,
           128, 64, flags(path=2, stages=stages), 1, 0, None)
    assert st == ARG
