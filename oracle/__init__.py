"""float64 CPU oracle for the Complex KDA (CKDA) recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` leg (and its
``--impl reference`` arm) may import this package.  The CUDA library in
``gated_delta_rule_82_b200`` never imports, links or calls anything here, and this package
never imports the CUDA library: the two share no code.

The arithmetic lives in ``ckda_oracle.c`` (plain sequential C in float64, see its header for the
definition and the passages it follows); this module only compiles it with gcc, loads it with
ctypes and marshals numpy arrays.  ``dense.py`` holds an independent dense-matrix restatement
used to pin the oracle on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ckda_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_libs: dict[int, ctypes.CDLL] = {}
_lock = threading.Lock()


def lib_path(mutant: int = 0) -> str:
    name = "libckda_oracle.so" if mutant == 0 else f"libckda_oracle_mut{mutant}.so"
    return os.path.join(_BUILD, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE double, no fast-math).  Returns the .so path."""
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    os.makedirs(_BUILD, exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           f"-DCKDA_ORACLE_MUTANT={int(mutant)}", "-o", tmp, _SRC, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _load(mutant: int = 0) -> ctypes.CDLL:
    with _lock:
        if mutant in _libs:
            return _libs[mutant]
        lib = ctypes.CDLL(build(mutant))
        D = ctypes.POINTER(ctypes.c_double)
        lib.ckda_oracle_fwd.restype = ctypes.c_int
        lib.ckda_oracle_fwd.argtypes = [D, D, D, D, D, D, D, D] + [ctypes.c_int] * 6 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_longlong,
            ctypes.c_int]
        lib.ckda_oracle_fwd_varlen.restype = ctypes.c_int
        lib.ckda_oracle_fwd_varlen.argtypes = [D, D, D, D, D, D, D, D,
                                               ctypes.POINTER(ctypes.c_longlong)] + [
            ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                 ctypes.c_longlong, ctypes.c_int]
        lib.ckda_oracle_bwd.restype = ctypes.c_int
        lib.ckda_oracle_bwd.argtypes = [D] * 14 + [ctypes.c_int] * 6 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_longlong,
            ctypes.c_int]
        lib.ckda_oracle_decode.restype = ctypes.c_int
        lib.ckda_oracle_decode.argtypes = [D, D, D, D, D, D, D, ctypes.POINTER(ctypes.c_longlong)] + [
            ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_double]
        lib.ckda_oracle_prologue.restype = ctypes.c_int
        lib.ckda_oracle_prologue.argtypes = [D, D] + [ctypes.c_int] * 5 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_longlong]
        lib.ckda_oracle_mutant.restype = ctypes.c_int
        lib.ckda_oracle_gates.restype = ctypes.c_int
        lib.ckda_oracle_gates.argtypes = [D, D, ctypes.c_longlong, D, D, ctypes.c_longlong]
        _libs[mutant] = lib
        return lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_scale(dk: int) -> float:
    """Read-out scale dk^-1/2 of o_t = dk^-1/2 S_t^T q_t."""
    return 1.0 / float(np.sqrt(dk))


def repeat_qk_heads(x, H: int, axis: int):
    """Grouped value heads (GVA): q or k with Hk heads on `axis`, each repeated H / Hk times in
    place, so that value head h reads q/k head h // (H / Hk).  The pages place the L2 norm (and
    with it the rotation) on the key-head axis, above this repeat ("RoPE review", section 7); both
    act per head, so repeating before or after them gives the same values."""
    Hk = x.shape[axis]
    assert H % Hk == 0, "value heads must be a multiple of the q/k heads"
    return x if Hk == H else np.repeat(x, H // Hk, axis=axis)


def fwd(q, k, v, alpha, beta, h0=None, *, l2norm=True, rope_theta=0.0, rope_convention=0,
        rope_dims=0, scale=None, pos_offset=0, want_state=True, nthreads=None, mutant=0):
    """Sequential float64 forward.

    q, k: [B, T, Hk, dk]; alpha: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H]; h0:
    [B, H, dk, dv] or None; H a multiple of Hk (grouped value heads when H > Hk).
    Returns (out [B, T, H, dv], hT [B, H, dk, dv] or None), float64.
    """
    q, k, v, alpha, beta = (_f64(x) for x in (q, k, v, alpha, beta))
    q = np.ascontiguousarray(repeat_qk_heads(q, v.shape[2], 2))
    k = np.ascontiguousarray(repeat_qk_heads(k, v.shape[2], 2))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and alpha.shape == q.shape
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    h0a = None if h0 is None else _f64(h0)
    if h0a is not None:
        assert h0a.shape == (B, H, dk, dv)
    out = np.empty((B, T, H, dv), np.float64)
    hT = np.empty((B, H, dk, dv), np.float64) if want_state else None
    if scale is None:
        scale = default_scale(dk)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load(mutant).ckda_oracle_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(h0a), _ptr(out), _ptr(hT),
        B, T, H, dk, dv, int(bool(l2norm)), float(rope_theta), int(rope_convention), int(rope_dims),
        float(scale), int(pos_offset), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ckda_oracle_fwd failed with code {rc}")
    return out, hT


def fwd_varlen(q, k, v, alpha, beta, cu_seqlens, h0=None, *, l2norm=True, rope_theta=0.0,
               rope_convention=0, rope_dims=0, scale=None, pos_offset=0, want_state=True,
               nthreads=None, mutant=0):
    """Sequential float64 forward over packed sequences of different lengths.

    q, k: [T_total, Hk, dk] (or with a leading batch axis of 1); alpha: [T_total, H, dk];
    v: [T_total, H, dv]; beta: [T_total, H]; cu_seqlens: [n + 1] token offsets (0 first,
    non-decreasing, T_total last); h0: [n, H, dk, dv] or None.  Sequence s is tokens
    cu_seqlens[s] .. cu_seqlens[s+1] - 1 with its own state and rotary positions from
    pos_offset.  Returns (out shaped like v, hT [n, H, dk, dv] or None), float64.
    """
    q, k, v, alpha, beta = (_f64(x) for x in (q, k, v, alpha, beta))
    lead = v.ndim == 4
    if lead:
        assert v.shape[0] == 1, "packed sequences take a batch axis of 1"
        q, k, v, alpha, beta = q[0], k[0], v[0], alpha[0], beta[0]
    q = np.ascontiguousarray(repeat_qk_heads(q, v.shape[1], 1))
    k = np.ascontiguousarray(repeat_qk_heads(k, v.shape[1], 1))
    Tt, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and alpha.shape == q.shape
    assert v.shape == (Tt, H, dv) and beta.shape == (Tt, H)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n = cu.shape[0] - 1
    assert n >= 0 and cu[-1] == Tt
    h0a = None if h0 is None else _f64(h0)
    if h0a is not None:
        assert h0a.shape == (n, H, dk, dv)
    out = np.empty((Tt, H, dv), np.float64)
    hT = np.empty((n, H, dk, dv), np.float64) if want_state else None
    if scale is None:
        scale = default_scale(dk)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load(mutant).ckda_oracle_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(h0a), _ptr(out), _ptr(hT),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)), n, H, dk, dv, int(bool(l2norm)),
        float(rope_theta), int(rope_convention), int(rope_dims), float(scale), int(pos_offset),
        int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ckda_oracle_fwd_varlen failed with code {rc}")
    return (out[None] if lead else out), hT


def bwd(q, k, v, alpha, beta, h0=None, dout=None, dhT=None, *, l2norm=True, rope_theta=0.0,
        rope_convention=0, rope_dims=0, scale=None, pos_offset=0, nthreads=None):
    """float64 gradients of L = <dout, out> + <dhT, hT> for the forward `fwd` (same arguments).

    Returns a dict with dq, dk ([B, T, Hk, dk]: summed over the value heads a grouped q/k head
    serves), dv, dalpha, dbeta and dh0 (None when h0 is None).
    """
    q, k, v, alpha, beta = (_f64(x) for x in (q, k, v, alpha, beta))
    Hk, H = q.shape[2], v.shape[2]
    qr = np.ascontiguousarray(repeat_qk_heads(q, H, 2))
    kr = np.ascontiguousarray(repeat_qk_heads(k, H, 2))
    B, T, _, dk = qr.shape
    dv = v.shape[-1]
    assert kr.shape == qr.shape and alpha.shape == qr.shape
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    h0a = None if h0 is None else _f64(h0)
    do = None if dout is None else _f64(dout)
    dh = None if dhT is None else _f64(dhT)
    g = {n: np.zeros(shape, np.float64) for n, shape in (
        ("dq", qr.shape), ("dk", qr.shape), ("dv", v.shape), ("dalpha", alpha.shape),
        ("dbeta", beta.shape))}
    g["dh0"] = None if h0a is None else np.zeros(h0a.shape, np.float64)
    if scale is None:
        scale = default_scale(dk)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().ckda_oracle_bwd(
        _ptr(qr), _ptr(kr), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(h0a), _ptr(do), _ptr(dh),
        _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dalpha"]), _ptr(g["dbeta"]),
        _ptr(g["dh0"]), B, T, H, dk, dv, int(bool(l2norm)), float(rope_theta),
        int(rope_convention), int(rope_dims), float(scale), int(pos_offset), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"ckda_oracle_bwd failed with code {rc}")
    if Hk != H:   # a q/k head serves H / Hk value heads: its gradient is their sum
        for n in ("dq", "dk"):
            g[n] = g[n].reshape(B, T, Hk, H // Hk, dk).sum(axis=3)
    return g


def gates(a=None, b=None, *, mutant=0):
    """Gates from logits, float64: alpha = 2 sigma(a) - 1 (same shape as a), beta = 2 sigma(b).
    Returns (alpha or None, beta or None)."""
    aa = None if a is None else _f64(a)
    ba = None if b is None else _f64(b)
    al = None if aa is None else np.empty_like(aa)
    be = None if ba is None else np.empty_like(ba)
    rc = _load(mutant).ckda_oracle_gates(_ptr(aa), _ptr(al), 0 if aa is None else aa.size,
                                         _ptr(ba), _ptr(be), 0 if ba is None else ba.size)
    if rc != 0:
        raise RuntimeError(f"ckda_oracle_gates failed with code {rc}")
    return al, be


def decode(q, k, v, alpha, beta, state, pos=None, *, l2norm=True, rope_theta=0.0,
           rope_convention=0, rope_dims=0, scale=None, mutant=0):
    """One float64 decode step.  q, k: [N, Hk, dk] with H a multiple of Hk (grouped value heads
    when H > Hk).  Returns (out [N, H, dv], new state [N, H, dk, dv])."""
    q, k, v, alpha, beta = (_f64(x) for x in (q, k, v, alpha, beta))
    q = np.ascontiguousarray(repeat_qk_heads(q, v.shape[1], 1))
    k = np.ascontiguousarray(repeat_qk_heads(k, v.shape[1], 1))
    N, H, dk = q.shape
    dv = v.shape[-1]
    st = _f64(state).copy()
    assert st.shape == (N, H, dk, dv)
    out = np.empty((N, H, dv), np.float64)
    if scale is None:
        scale = default_scale(dk)
    pp = None
    if pos is not None:
        posa = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
        pp = posa.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong))
    rc = _load(mutant).ckda_oracle_decode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(st), _ptr(out), pp, N, H, dk,
        dv, int(bool(l2norm)), float(rope_theta), int(rope_convention), int(rope_dims), float(scale))
    if rc != 0:
        raise RuntimeError(f"ckda_oracle_decode failed with code {rc}")
    return out, st


def prologue(x, *, l2norm=True, rope_theta=0.0, rope_convention=0, rope_dims=0, pos_offset=0,
             mutant=0):
    """Rotation (if rope_theta > 0) then per-head L2 norm of x [B, T, H, d], float64."""
    x = _f64(x)
    B, T, H, d = x.shape
    y = np.empty_like(x)
    rc = _load(mutant).ckda_oracle_prologue(_ptr(x), _ptr(y), B, T, H, d, int(bool(l2norm)),
                                            float(rope_theta), int(rope_convention),
                                            int(rope_dims), int(pos_offset))
    if rc != 0:
        raise RuntimeError(f"ckda_oracle_prologue failed with code {rc}")
    return y


def mutant_id(mutant: int = 0) -> int:
    return _load(mutant).ckda_oracle_mutant()
