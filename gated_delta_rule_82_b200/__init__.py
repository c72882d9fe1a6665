"""Python binding of the B200 CKDA library (``libckda.so``, C ABI in ``include/ckda.h``).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  There is no CPU fallback: if the
compiled library is missing or no CUDA device is present, the calls raise.

Build the library with ``python -m gated_delta_rule_82_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["CkdaError", "library_path", "abi_version", "qk_prologue", "workspace_bytes",
           "fwd_chunked", "varlen_workspace_bytes", "fwd_varlen", "decode_step", "selftest_umma",
           "last_device_status", "set_wait_limit_ns", "bwd_workspace_bytes", "bwd_chunked",
           "PATHS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libckda.so")
_lib = None

PATHS = {"auto": 0, "simt": 1, "tc": 2}
_F32, _BF16 = 0, 1


class CkdaError(RuntimeError):
    def __init__(self, func, status):
        self.status = status
        msg = _load().ckda_strerror(status).decode()
        super().__init__(f"{func} failed: status {status} ({msg})")


class _Flags(ctypes.Structure):
    _fields_ = [("l2norm", ctypes.c_int), ("rope_theta", ctypes.c_float),
                ("rope_convention", ctypes.c_int), ("scale", ctypes.c_float),
                ("path", ctypes.c_int), ("stages", ctypes.c_int), ("gate_logits", ctypes.c_int),
                ("rope_dims", ctypes.c_int), ("qk_heads", ctypes.c_int)]


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"CKDA CUDA library not built: {_LIB_PATH} is missing "
                           "(run python -m gated_delta_rule_82_b200.build)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    lib.ckda_abi_version.restype = I
    lib.ckda_abi_version.argtypes = []
    lib.ckda_strerror.restype = ctypes.c_char_p
    lib.ckda_strerror.argtypes = [I]
    lib.ckda_qk_prologue.restype = I
    lib.ckda_qk_prologue.argtypes = [P, P, P, P, I, I, I, I, _Flags, I, LL, P]
    lib.ckda_fwd_workspace_bytes.restype = SZ
    lib.ckda_fwd_workspace_bytes.argtypes = [I, I, I, I, I, I, I, I]
    lib.ckda_fwd_chunked.restype = I
    lib.ckda_fwd_chunked.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, _Flags, I, LL, P,
                                     SZ, P]
    lib.ckda_fwd_segmented_workspace_bytes.restype = SZ
    lib.ckda_fwd_segmented_workspace_bytes.argtypes = [I] * 6
    lib.ckda_fwd_segmented.restype = I
    lib.ckda_fwd_segmented.argtypes = [P] * 8 + [I] * 5 + [_Flags, I, LL, I, P, SZ, P]
    lib.ckda_fwd_simt_workspace_bytes.restype = SZ
    lib.ckda_fwd_simt_workspace_bytes.argtypes = [I] * 5
    lib.ckda_fwd_segments_auto.restype = I
    lib.ckda_fwd_segments_auto.argtypes = [I, I, I]
    lib.ckda_fwd_varlen_workspace_bytes.restype = SZ
    lib.ckda_fwd_varlen_workspace_bytes.argtypes = [P, I, I, I, I, I, I, I]
    lib.ckda_fwd_varlen.restype = I
    lib.ckda_fwd_varlen.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, _Flags, I, LL, P,
                                    SZ, P]
    lib.ckda_decode_step.restype = I
    lib.ckda_decode_step.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, _Flags, I, P]
    lib.ckda_selftest_umma.restype = I
    lib.ckda_selftest_umma.argtypes = [P, P, P, I, I, I, I, P]
    lib.ckda_bwd_workspace_bytes.restype = SZ
    lib.ckda_bwd_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.ckda_bwd_chunked.restype = I
    lib.ckda_bwd_chunked.argtypes = [P] * 14 + [I] * 5 + [_Flags, I, LL, P, SZ, P]
    lib.ckda_last_device_status.restype = I
    lib.ckda_last_device_status.argtypes = [P, ctypes.POINTER(I)]
    lib.ckda_set_wait_limit_ns.restype = I
    lib.ckda_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    _lib = lib
    return lib


def abi_version() -> int:
    return _load().ckda_abi_version()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _BF16
    if t.dtype == torch.float32:
        return _F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _check(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _flags(l2norm, rope_theta, rope_convention, scale, path=0, stages=0, gate_logits=False,
           qk_heads=0, rope_dims=0):
    return _Flags(int(bool(l2norm)), float(rope_theta), int(rope_convention), float(scale),
                  int(path), int(stages), int(bool(gate_logits)), int(rope_dims), int(qk_heads))


def _raise(func, status):
    if status != 0:
        raise CkdaError(func, status)


def qk_prologue(q, k, *, l2norm=True, rope_theta=0.0, rope_convention=0, pos_offset=0,
                q_out=None, k_out=None, rope_dims=0):
    """Rotation at positions pos_offset + t, then per-head L2 norm, of q and k [B, T, H, dk]."""
    _check(q, "q")
    _check(k, "k", dtype=q.dtype, shape=q.shape)
    B, T, H, dk = q.shape
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    _check(q_out, "q_out", dtype=q.dtype, shape=q.shape)
    _check(k_out, "k_out", dtype=q.dtype, shape=q.shape)
    st = _load().ckda_qk_prologue(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), B, T, H, dk,
                                  _flags(l2norm, rope_theta, rope_convention, 0.0,
                                         rope_dims=rope_dims),
                                  _dtype_code(q), int(pos_offset), _stream(q.device))
    _raise("ckda_qk_prologue", st)
    return q_out, k_out


def workspace_bytes(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16, path="auto") -> int:
    code = _BF16 if dtype == torch.bfloat16 else _F32
    n = _load().ckda_fwd_workspace_bytes(B, T, H, dk, dv, chunk, code, PATHS[path])
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("unsupported problem for ckda_fwd_chunked")
    return int(n)


def fwd_chunked(q, k, v, alpha, beta, h0=None, *, chunk=64, l2norm=True, rope_theta=0.0,
                rope_convention=0, scale=0.0, pos_offset=0, path="auto", want_state=True,
                out=None, hT=None, workspace=None, stages=0, gate_logits=False, rope_dims=0):
    """Chunked CKDA forward.  Returns (out [B, T, H, dv], hT [B, H, dk, dv] or None).

    q, k: [B, T, Hk, dk] (bf16 or fp32); v: [B, T, H, dv] same dtype, H a multiple of Hk (grouped
    value heads when H > Hk: value head h reads q/k head h // (H // Hk)); alpha: [B, T, H, dk]
    fp32; beta: [B, T, H] fp32; h0: [B, H, dk, dv] fp32 or None.  With gate_logits, alpha holds
    logits a in q's dtype and beta fp32 logits b; the kernels use alpha = 2 sigma(a) - 1 and
    beta = 2 sigma(b).
    """
    _check(q, "q")
    B, T, Hk, dk = q.shape
    _check(v, "v", dtype=q.dtype)
    if v.dim() != 4 or v.shape[:2] != (B, T):
        raise ValueError(f"v: expected [B={B}, T={T}, H, dv], got {tuple(v.shape)}")
    H, dv = v.shape[2], v.shape[3]
    if H % Hk:
        raise ValueError(f"v has {H} heads, not a multiple of q's {Hk}")
    _check(k, "k", dtype=q.dtype, shape=q.shape)
    _check(alpha, "alpha", dtype=q.dtype if gate_logits else torch.float32, shape=(B, T, H, dk))
    _check(beta, "beta", dtype=torch.float32, shape=(B, T, H))
    if h0 is not None:
        _check(h0, "h0", dtype=torch.float32, shape=(B, H, dk, dv))
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", dtype=q.dtype, shape=(B, T, H, dv))
    if want_state and hT is None:
        hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _check(hT, "hT", dtype=torch.float32, shape=(B, H, dk, dv))
    code = _dtype_code(q)
    if workspace is None:   # (a workspace given is checked against the need by the library)
        need = workspace_bytes(B, T, H, dk, dv, chunk, q.dtype, path)
        if need == 0:   # the CUDA-core path: the workspace of its record form
            need = int(_load().ckda_fwd_simt_workspace_bytes(B, T, H, dk, dv))
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _load().ckda_fwd_chunked(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(h0), _ptr(out), _ptr(hT),
        B, T, H, dk, dv, int(chunk), _flags(l2norm, rope_theta, rope_convention, scale,
                                           PATHS[path], stages, gate_logits,
                                           Hk if Hk != H else 0, rope_dims),
        code, int(pos_offset), _ptr(workspace), wbytes, _stream(q.device))
    _raise("ckda_fwd_chunked", st)
    return out, hT


def simt_workspace_bytes(B, T, H, dk, dv) -> int:
    """Bytes of the optional workspace that selects the record form of the CUDA-core path."""
    n = _load().ckda_fwd_simt_workspace_bytes(B, T, H, dk, dv)
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("unsupported problem for the CUDA-core path")
    return int(n)


def segments_auto(B, T, H) -> int:
    """Segment count ckda_fwd_segments_auto picks for a batch of B x H sequences of T tokens on the
    current device (1: the single fused launch is expected to be faster)."""
    return int(_load().ckda_fwd_segments_auto(B, T, H))


def segmented_workspace_bytes(B, T, H, dk, dv, segments) -> int:
    n = _load().ckda_fwd_segmented_workspace_bytes(B, T, H, dk, dv, segments)
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("unsupported problem for ckda_fwd_segmented")
    return int(n)


def fwd_segmented(q, k, v, alpha, beta, h0=None, *, segments=0, l2norm=True, rope_theta=0.0,
                  rope_convention=0, scale=0.0, pos_offset=0, want_state=True, out=None, hT=None,
                  workspace=None, gate_logits=False, rope_dims=0):
    """Tensor-core forward with the segment-parallel state pass (ckda_fwd_segmented): arguments
    and results as fwd_chunked (bf16, dk = dv = 128).  segments = 0 takes segments_auto's count.
    Returns (out, hT)."""
    _check(q, "q")
    B, T, Hk, dk = q.shape
    _check(v, "v", dtype=q.dtype)
    if v.dim() != 4 or v.shape[:2] != (B, T):
        raise ValueError(f"v: expected [B={B}, T={T}, H, dv], got {tuple(v.shape)}")
    H, dv = v.shape[2], v.shape[3]
    if H % Hk:
        raise ValueError(f"v has {H} heads, not a multiple of q's {Hk}")
    _check(k, "k", dtype=q.dtype, shape=q.shape)
    _check(alpha, "alpha", dtype=q.dtype if gate_logits else torch.float32, shape=(B, T, H, dk))
    _check(beta, "beta", dtype=torch.float32, shape=(B, T, H))
    if h0 is not None:
        _check(h0, "h0", dtype=torch.float32, shape=(B, H, dk, dv))
    if segments == 0:
        segments = segments_auto(B, T, H)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", dtype=q.dtype, shape=(B, T, H, dv))
    if want_state and hT is None:
        hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _check(hT, "hT", dtype=torch.float32, shape=(B, H, dk, dv))
    if workspace is None:
        workspace = torch.empty(segmented_workspace_bytes(B, T, H, dk, dv, segments),
                                dtype=torch.uint8, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    st = _load().ckda_fwd_segmented(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(h0), _ptr(out), _ptr(hT),
        B, T, H, dk, dv, _flags(l2norm, rope_theta, rope_convention, scale, PATHS["tc"], 0,
                                gate_logits, Hk if Hk != H else 0, rope_dims),
        _dtype_code(q), int(pos_offset), int(segments), _ptr(workspace), wbytes,
        _stream(q.device))
    _raise("ckda_fwd_segmented", st)
    return out, hT


def _host_offsets(cu_seqlens, cu_seqlens_cpu):
    """int32 offsets on the device (as given) and a host copy (given, or read back: a sync)."""
    _check(cu_seqlens, "cu_seqlens", dtype=torch.int32)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens: expected [n + 1] token offsets, n >= 1")
    host = cu_seqlens.cpu() if cu_seqlens_cpu is None else cu_seqlens_cpu
    host = host.to(torch.int32).contiguous()
    if tuple(host.shape) != tuple(cu_seqlens.shape):
        raise ValueError("cu_seqlens_cpu must have the shape of cu_seqlens")
    return host


def varlen_workspace_bytes(cu_seqlens_cpu, H, dk, dv, chunk, dtype, path="auto") -> int:
    """Device workspace bytes of fwd_varlen for these host offsets (0 when none is needed)."""
    host = cu_seqlens_cpu.to(torch.int32).contiguous()
    code = _BF16 if dtype == torch.bfloat16 else _F32
    n = _load().ckda_fwd_varlen_workspace_bytes(ctypes.c_void_p(host.data_ptr()), host.numel() - 1,
                                                H, dk, dv, chunk, code, PATHS[path])
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("unsupported sizes or invalid offsets for the packed forward")
    return n


def fwd_varlen(q, k, v, alpha, beta, cu_seqlens, h0=None, *, cu_seqlens_cpu=None, chunk=64,
               l2norm=True, rope_theta=0.0, rope_convention=0, scale=0.0, pos_offset=0,
               path="auto", want_state=True, out=None, hT=None, workspace=None, stages=0,
               gate_logits=False, rope_dims=0):
    """Chunked CKDA forward over packed sequences of different lengths.  Returns (out, hT).

    q, k: [1, T, Hk, dk] or [T, Hk, dk]; v: [.., T, H, dv]; alpha: [.., T, H, dk]; beta:
    [.., T, H] (the layouts of fwd_chunked with a batch of 1, or without the batch axis);
    cu_seqlens: int32 [n + 1] on the device, token offsets of the n sequences (0 first,
    non-decreasing, T last); cu_seqlens_cpu: the same offsets on the host (read back from the
    device when omitted); h0 / hT: [n, H, dk, dv] fp32.  Each sequence starts from its own h0,
    ends in its own hT, and its rotary positions start again at pos_offset.
    """
    _check(q, "q")
    lead = q.dim() == 4
    if lead and q.shape[0] != 1:
        raise ValueError("packed sequences take a batch axis of 1 (or none)")
    T, Hk, dk = q.shape[-3:]
    _check(v, "v", dtype=q.dtype)
    if v.dim() != q.dim() or v.shape[-3] != T:
        raise ValueError(f"v: expected [.., T={T}, H, dv], got {tuple(v.shape)}")
    H, dv = v.shape[-2], v.shape[-1]
    if H % Hk:
        raise ValueError(f"v has {H} heads, not a multiple of q's {Hk}")
    pre = (1,) if lead else ()
    _check(k, "k", dtype=q.dtype, shape=q.shape)
    _check(alpha, "alpha", dtype=q.dtype if gate_logits else torch.float32, shape=pre + (T, H, dk))
    _check(beta, "beta", dtype=torch.float32, shape=pre + (T, H))
    host = _host_offsets(cu_seqlens, cu_seqlens_cpu)
    n = host.numel() - 1
    if int(host[-1]) != T:
        raise ValueError(f"cu_seqlens ends at {int(host[-1])}, but the token axis holds {T}")
    if h0 is not None:
        _check(h0, "h0", dtype=torch.float32, shape=(n, H, dk, dv))
    if out is None:
        out = torch.empty(pre + (T, H, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", dtype=q.dtype, shape=pre + (T, H, dv))
    if want_state and hT is None:
        hT = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _check(hT, "hT", dtype=torch.float32, shape=(n, H, dk, dv))
    if workspace is None:   # (a workspace given is checked against the need by the library)
        need = varlen_workspace_bytes(host, H, dk, dv, chunk, q.dtype, path)
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _load().ckda_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(h0), _ptr(out), _ptr(hT),
        _ptr(cu_seqlens), ctypes.c_void_p(host.data_ptr()), n, H, dk, dv, int(chunk),
        _flags(l2norm, rope_theta, rope_convention, scale, PATHS[path], stages, gate_logits,
               Hk if Hk != H else 0, rope_dims),
        _dtype_code(q), int(pos_offset), _ptr(workspace), wbytes, _stream(q.device))
    _raise("ckda_fwd_varlen", st)
    return out, hT


def decode_step(q, k, v, alpha, beta, state, pos=None, *, l2norm=True, rope_theta=0.0,
                rope_convention=0, scale=0.0, out=None, gate_logits=False, rope_dims=0):
    """One decode step, in place on state [N, H, dk, dv] fp32.  Returns out [N, H, dv].
    q, k: [N, Hk, dk] with H a multiple of Hk (grouped value heads when H > Hk).  With
    gate_logits, alpha holds logits a in q's dtype and beta fp32 logits b."""
    _check(q, "q")
    N, Hk, dk = q.shape
    _check(v, "v", dtype=q.dtype)
    if v.dim() != 3 or v.shape[0] != N:
        raise ValueError(f"v: expected [N={N}, H, dv], got {tuple(v.shape)}")
    H, dv = v.shape[1], v.shape[2]
    if H % Hk:
        raise ValueError(f"v has {H} heads, not a multiple of q's {Hk}")
    _check(k, "k", dtype=q.dtype, shape=q.shape)
    _check(alpha, "alpha", dtype=q.dtype if gate_logits else torch.float32, shape=(N, H, dk))
    _check(beta, "beta", dtype=torch.float32, shape=(N, H))
    _check(state, "state", dtype=torch.float32, shape=(N, H, dk, dv))
    if pos is not None:
        _check(pos, "pos", dtype=torch.int64, shape=(N,))
    if out is None:
        out = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _check(out, "out", dtype=q.dtype, shape=(N, H, dv))
    st = _load().ckda_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(out), _ptr(pos),
        N, H, dk, dv, _flags(l2norm, rope_theta, rope_convention, scale, 0, 0, gate_logits,
                             Hk if Hk != H else 0, rope_dims),
        _dtype_code(q),
        _stream(q.device))
    _raise("ckda_decode_step", st)
    return out


def bwd_workspace_bytes(B, T, H, dk, dv) -> int:
    n = _load().ckda_bwd_workspace_bytes(B, T, H, dk, dv)
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("unsupported problem for ckda_bwd_chunked")
    return int(n)


def bwd_chunked(q, k, v, alpha, beta, h0, dout, dhT=None, *, l2norm=True, rope_theta=0.0,
                rope_convention=0, scale=0.0, pos_offset=0, gate_logits=False, rope_dims=0,
                workspace=None, want_dh0=True):
    """Gradients of <dout, out> + <dhT, hT> for fwd_chunked with the same inputs and flags.

    Returns a dict of fp32 tensors: dq, dk ([B, T, Hk, dk]), dv, dalpha, dbeta and dh0 (None
    when want_dh0 is False).  dout has the dtype of q; dhT is fp32 [B, H, dk, dv] or None.
    """
    _check(q, "q")
    B, T, Hk, dk = q.shape
    _check(v, "v", dtype=q.dtype)
    H, dv = v.shape[2], v.shape[3]
    if H % Hk:
        raise ValueError(f"v has {H} heads, not a multiple of q's {Hk}")
    _check(k, "k", dtype=q.dtype, shape=q.shape)
    _check(alpha, "alpha", dtype=q.dtype if gate_logits else torch.float32, shape=(B, T, H, dk))
    _check(beta, "beta", dtype=torch.float32, shape=(B, T, H))
    _check(dout, "dout", dtype=q.dtype, shape=(B, T, H, dv))
    if h0 is not None:
        _check(h0, "h0", dtype=torch.float32, shape=(B, H, dk, dv))
    if dhT is not None:
        _check(dhT, "dhT", dtype=torch.float32, shape=(B, H, dk, dv))
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"dq": torch.empty((B, T, Hk, dk), **f32), "dk": torch.empty((B, T, Hk, dk), **f32),
         "dv": torch.empty((B, T, H, dv), **f32), "dalpha": torch.empty((B, T, H, dk), **f32),
         "dbeta": torch.empty((B, T, H), **f32),
         "dh0": torch.empty((B, H, dk, dv), **f32) if want_dh0 else None}
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(B, T, H, dk, dv), dtype=torch.uint8,
                                device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    st = _load().ckda_bwd_chunked(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(h0), _ptr(dout), _ptr(dhT),
        _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dalpha"]), _ptr(g["dbeta"]),
        _ptr(g["dh0"]), B, T, H, dk, dv,
        _flags(l2norm, rope_theta, rope_convention, scale, 0, 0, gate_logits,
               Hk if Hk != H else 0, rope_dims),
        _dtype_code(q), int(pos_offset), _ptr(workspace), wbytes, _stream(q.device))
    _raise("ckda_bwd_chunked", st)
    return g


def last_device_status(device=None) -> int:
    """Wait for the current stream, then read and clear the library's device status word:
    0 = no failure recorded; 1 / 2 = a bounded wait of the tensor-core forward ran out (factor
    work / state pass); 3 = packed-sequence offsets on the device disagreed with the host copy."""
    code = ctypes.c_int(0)
    st = _load().ckda_last_device_status(_stream(device), ctypes.byref(code))
    if st not in (0, 8):   # CKDA_OK, CKDA_ERR_DEVICE_STATUS
        raise CkdaError("ckda_last_device_status", st)
    return int(code.value)


def set_wait_limit_ns(ns: int = 0) -> None:
    """Upper bound of one wait of the tensor-core forward's state pass on the current device
    (0 restores the default of 4 s).  A diagnostic: a short limit makes a wait give up sooner."""
    _raise("ckda_set_wait_limit_ns", _load().ckda_set_wait_limit_ns(int(ns)))


def selftest_umma(A, B, b_mn_major=False, a_tmem=False):
    """fp32 A @ B^T (b_mn_major=False, B [N, K]) or A @ B (B [K, N]) via the library's tcgen05
    wrappers, for bf16 A [M, K] and B.  a_tmem: False (A from shared memory), True or "cp" (A
    copied into Tensor Memory by tcgen05.cp), "st" (A written into Tensor Memory by tcgen05.st)."""
    _check(A, "A", dtype=torch.bfloat16)
    _check(B, "B", dtype=torch.bfloat16)
    M, K = A.shape
    N = B.shape[1] if b_mn_major else B.shape[0]
    D = torch.empty((M, N), dtype=torch.float32, device=A.device)
    mode = int(bool(b_mn_major)) | (4 if a_tmem == "st" else 2 if a_tmem else 0)
    st = _load().ckda_selftest_umma(_ptr(A), _ptr(B), _ptr(D), M, N, K, mode,
                                    _stream(A.device))
    _raise("ckda_selftest_umma", st)
    return D
