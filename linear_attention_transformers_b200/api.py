"""Thin Python binding of liblinattn (the C ABI in include/la_api.h).

Argument marshalling only: every function checks tensor placement, dtype,
shape and contiguity, allocates the outputs (and the workspace) it is not
given with torch, and calls the C entry point of the same name on the
current CUDA stream.  No arithmetic of the method runs here, and there is no
fallback: if ``liblinattn.so`` is missing or cannot be loaded, every call
raises ``RuntimeError``.

    la_forward(q, k, v, causal=True, phi="elu1", ...)        -> o [, S, z]
    la_backward(q, k, v, dO, causal=True, phi="elu1", ...)   -> dq, dk, dv
    la_decode_step(S, z, q, k, v, phi="elu1", ...)           -> o   (S, z in place)
    la_workspace_size(op, B, H, N, D, causal, dtype, Hkv)    -> bytes
    la_forward_decay(q, k, v, gamma, phi="elu1", ...)        -> o [, S, z]  (causal)
    la_backward_decay(q, k, v, dO, gamma, phi="elu1", ...)   -> dq, dk, dv
    la_decode_step_decay(S, z, q, k, v, gamma, ...)          -> o   (S, z in place)
    la_favor_features(x, omega)                              -> phi(x)  (Performer FAVOR+)
    la_favor_features_backward(x, omega, dphi)               -> dx
    la_forward_mv / la_backward_mv(q, k, v[, dO])            features of length m != D
    la_state_local / la_state_range_sum / la_forward_sp /
    la_backward_sp_dq / la_backward_sp_dkdv                  (one rank's steps of a
                                                              sequence split across ranks)
    la_get_device_error(stream=None)                         -> raises on a device timeout
    LinearAttention.apply(q, k, v, causal, phi)              -> o   (torch autograd)

k and v may have fewer heads than q (grouped-query / multi-query attention:
Hkv key/value heads shared by groups of H / Hkv query heads); the group size
is read from their shapes.  The *_decay calls take one decay factor per head
(gamma, H host values in [0, 1]): S_i = gamma S_{i-1} + phi(k_i) v_i^T.
With phi="identity" q and k are taken as feature vectors already (for
example la_favor_features(q, omega)), and the backward returns their
gradients.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

LA_OK = 0
LA_ERR_INVALID_ARG = 1
LA_ERR_UNSUPPORTED = 2
LA_ERR_CUDA = 3
LA_ERR_WORKSPACE = 4
LA_ERR_DEVICE_TIMEOUT = 5

LA_F32 = 0
LA_BF16 = 1
LA_OP_FORWARD = 0
LA_OP_BACKWARD = 1
PHI = {"elu1": 0, "relu_eps": 1, "identity": 2, 0: 0, 1: 1, 2: 2}
DTYPE = {torch.float32: LA_F32, torch.bfloat16: LA_BF16}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblinattn.so")
_lock = threading.Lock()
_lib = None


class ProfileEntry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double)]


class LinearAttentionError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} failed: {la_status_string(status)} (status {status})"
        if status == LA_ERR_CUDA:
            msg += f" [{la_last_error()}]"
        super().__init__(msg)


def load_library(path: str | None = None):
    """Load liblinattn.so (built in-tree by ``build.py``); raises if absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(
                f"liblinattn.so not found at {p}; build it with "
                "`python -m linear_attention_transformers_b200.build` (there is no fallback)")
        lib = ctypes.CDLL(p)
        vp, i64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        lib.la_workspace_size.argtypes = [ci, i64, i64, i64, i64, ci, ci]
        lib.la_workspace_size.restype = sz
        lib.la_workspace_size_gqa.argtypes = [ci, i64, i64, i64, i64, i64, ci, ci]
        lib.la_workspace_size_gqa.restype = sz
        lib.la_forward_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                       i64, ci, ci, ci, vp, sz, vp]
        lib.la_forward_gqa.restype = ci
        lib.la_backward_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64,
                                        i64, i64, ci, ci, ci, vp, sz, vp]
        lib.la_backward_gqa.restype = ci
        lib.la_decode_step_gqa.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, vp]
        lib.la_decode_step_gqa.restype = ci
        lib.la_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci,
                                   ci, vp, sz, vp]
        lib.la_forward.restype = ci
        lib.la_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64,
                                    i64, ci, ci, ci, vp, sz, vp]
        lib.la_backward.restype = ci
        lib.la_backward_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64,
                                            i64, i64, ci, ci, ci, vp]
        lib.la_backward_noalloc.restype = ci
        lib.la_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, ci, ci, vp]
        lib.la_decode_step.restype = ci
        fp = ctypes.POINTER(ctypes.c_float)
        lib.la_workspace_size_decay.argtypes = [ci, i64, i64, i64, i64, ci]
        lib.la_workspace_size_decay.restype = sz
        lib.la_forward_decay.argtypes = [vp, vp, vp, vp, vp, vp, vp, fp, i64, i64, i64, i64, ci,
                                         ci, vp, sz, vp]
        lib.la_forward_decay.restype = ci
        lib.la_backward_decay.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, fp, i64, i64, i64,
                                          i64, ci, ci, vp, sz, vp]
        lib.la_backward_decay.restype = ci
        lib.la_decode_step_decay.argtypes = [vp, vp, vp, vp, vp, vp, fp, i64, i64, i64, ci, ci, vp]
        lib.la_decode_step_decay.restype = ci
        lib.la_favor_features.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, ci, vp]
        lib.la_favor_features.restype = ci
        lib.la_favor_features_backward.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, ci,
                                                   vp]
        lib.la_favor_features_backward.restype = ci
        lib.la_workspace_size_mv.argtypes = [ci, i64, i64, i64, i64, i64, ci, ci]
        lib.la_workspace_size_mv.restype = sz
        lib.la_forward_mv.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, ci, ci, ci,
                                      vp, sz, vp]
        lib.la_forward_mv.restype = ci
        lib.la_backward_mv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                       i64, ci, ci, ci, vp, sz, vp]
        lib.la_backward_mv.restype = ci
        lib.la_workspace_size_sp.argtypes = [ci, i64, i64, i64, i64, ci, ci]
        lib.la_workspace_size_sp.restype = sz
        lib.la_state_local.argtypes = [vp, vp, vp, i64, i64, i64, i64, ci, ci, ci, vp, sz, vp]
        lib.la_state_local.restype = ci
        lib.la_state_range_sum.argtypes = [vp, i64, i64, i64, vp, i64, i64, i64, vp]
        lib.la_state_range_sum.restype = ci
        lib.la_forward_sp.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, ci, ci, ci,
                                      vp, sz, vp]
        lib.la_forward_sp.restype = ci
        lib.la_backward_sp_dq.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                          ci, ci, ci, vp, sz, vp]
        lib.la_backward_sp_dq.restype = ci
        lib.la_backward_sp_dkdv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                            ci, ci, ci, vp, sz, vp]
        lib.la_backward_sp_dkdv.restype = ci
        lib.la_status_string.argtypes = [ci]
        lib.la_status_string.restype = ctypes.c_char_p
        lib.la_last_error.argtypes = []
        lib.la_last_error.restype = ctypes.c_char_p
        lib.la_get_device_error.argtypes = [vp]
        lib.la_get_device_error.restype = ci
        lib.la_selftest_wait_timeout.argtypes = [ci, vp]
        lib.la_selftest_wait_timeout.restype = ci
        lib.la_version.argtypes = []
        lib.la_version.restype = ci
        lib.la_launch_count.argtypes = []
        lib.la_launch_count.restype = ctypes.c_uint64
        lib.la_profile_enable.argtypes = [ci]
        lib.la_profile_enable.restype = None
        lib.la_profile_collect.argtypes = [ctypes.POINTER(ProfileEntry), ci]
        lib.la_profile_collect.restype = ci
        _lib = lib
        return lib


def la_status_string(status: int) -> str:
    return load_library().la_status_string(int(status)).decode()


def la_last_error() -> str:
    """Detail of the last CUDA failure on this thread ("" if none)."""
    return load_library().la_last_error().decode()


def la_version() -> int:
    return int(load_library().la_version())


def _check(fn: str, status: int) -> None:
    if status != LA_OK:
        raise LinearAttentionError(fn, status)


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _phi(phi) -> int:
    if phi not in PHI:
        raise ValueError(f"phi must be 'elu1', 'relu_eps' or 'identity', got {phi!r}")
    return PHI[phi]


def _check_qkv(name: str, ref: torch.Tensor, *ts: torch.Tensor) -> None:
    if not ref.is_cuda:
        raise ValueError(f"{name}: tensors must be on a CUDA device")
    if ref.dtype not in DTYPE:
        raise ValueError(f"{name}: dtype must be float32 or bfloat16, got {ref.dtype}")
    for t in (ref, *ts):
        if t.device != ref.device or t.dtype != ref.dtype or t.shape != ref.shape:
            raise ValueError(f"{name}: all tensors need the same device, dtype and shape")
        if not t.is_contiguous():
            raise ValueError(f"{name}: tensors must be contiguous")


def la_workspace_size(op: int, B: int, H: int, N: int, D: int, causal: bool,
                      dtype: torch.dtype, Hkv: int | None = None) -> int:
    return int(load_library().la_workspace_size_gqa(int(op), B, H, H if Hkv is None else Hkv, N,
                                                    D, int(bool(causal)), DTYPE[dtype]))


def _check_kv(name: str, q: torch.Tensor, k: torch.Tensor, *ts: torch.Tensor) -> int:
    """k (and v, dk, dv): [B, Hkv, N, D] like q but with Hkv heads dividing
    q's; returns Hkv."""
    _check_qkv(name, k, *ts)
    if q.dim() != k.dim() or q.device != k.device or q.dtype != k.dtype:
        raise ValueError(f"{name}: q and k need the same device, dtype and rank")
    if q.dim() >= 3:
        hq, hk = q.shape[1], k.shape[1]
        if (q.shape[0], *q.shape[2:]) != (k.shape[0], *k.shape[2:]) or hk < 1 or hq % hk != 0:
            raise ValueError(f"{name}: k, v must be [B, Hkv, ...] with Hkv dividing q's heads")
        return int(hk)
    return 1


def _workspace(op, q, causal, workspace, Hkv=None):
    B, H, N, D = q.shape
    need = la_workspace_size(op, B, H, N, D, causal, q.dtype, Hkv)
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    return workspace, workspace.numel() * workspace.element_size()


def la_forward(q, k, v, causal: bool = True, phi="elu1", o=None, return_state=False,
               workspace=None, stream=None, g=None, phi_out=None, state_out=None):
    """o = linear attention of q, k, v [B, H, N, D]; optionally the final (S, z).

    ``g``: optional float32 [B, H, N] tensor that receives the denominators;
    pass it with ``o`` to la_backward to skip the forward recompute there.
    ``phi_out``: optional pair (pq, pk) of tensors shaped and typed like q
    that receive phi(q), phi(k); pass them to la_backward with o and g.
    ``state_out``: optional pair (S, z) of float32 tensors [B, H, D, D] and
    [B, H, D] that receive the final state (instead of allocating them, as
    ``return_state`` does); pass them to la_backward as S, z.
    """
    lib = load_library()
    _check_qkv("la_forward", q)
    if q.dim() != 4:
        raise ValueError("la_forward: q, k, v must be [B, H, N, D]")
    Hkv = _check_kv("la_forward", q, k, v)
    B, H, N, D = q.shape
    if o is None:
        o = torch.empty_like(q)
    else:
        _check_qkv("la_forward", q, o)
    S = z = None
    if state_out is not None:
        S, z = state_out
        for nm, t, shape in (("S", S, (B, Hkv, D, D)), ("z", z, (B, Hkv, D))):
            if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous() \
                    or t.device != q.device:
                raise ValueError(f"la_forward: {nm} must be contiguous float32 {shape} on q's "
                                 "device")
    elif return_state:
        S = torch.empty((B, Hkv, D, D), dtype=torch.float32, device=q.device)
        z = torch.empty((B, Hkv, D), dtype=torch.float32, device=q.device)
    if g is not None and (g.dtype != torch.float32 or tuple(g.shape) != (B, H, N)
                          or not g.is_contiguous() or g.device != q.device):
        raise ValueError("la_forward: g must be contiguous float32 [B, H, N] on q's device")
    pq = pk = None
    if phi_out is not None:
        pq, pk = phi_out
        _check_qkv("la_forward", q, pq, pk)
    ws, ws_bytes = _workspace(LA_OP_FORWARD, q, causal, workspace, Hkv)
    st = lib.la_forward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), _ptr(z), _ptr(g),
                            _ptr(pq), _ptr(pk), B, H, Hkv, N, D, DTYPE[q.dtype],
                            int(bool(causal)), _phi(phi), _ptr(ws), ws_bytes,
                            _stream_handle(stream))
    _check("la_forward", st)
    return (o, S, z) if return_state else o


def _check_saved(name, q, o, g, phi_q=None, phi_k=None):
    if (o is None) != (g is None):
        raise ValueError(f"{name}: pass both o and g (saved forward statistics) or neither")
    if (phi_q is None) != (phi_k is None) or (phi_q is not None and o is None):
        raise ValueError(f"{name}: phi_q and phi_k go together, and only with o and g")
    if phi_q is not None:
        _check_qkv(name, q, phi_q, phi_k)
    if o is not None:
        _check_qkv(name, q, o)
        B, H, N, _ = q.shape
        if g.dtype != torch.float32 or tuple(g.shape) != (B, H, N) or not g.is_contiguous():
            raise ValueError(f"{name}: g must be contiguous float32 [B, H, N]")


def la_backward(q, k, v, dO, causal: bool = True, phi="elu1", dq=None, dk=None, dv=None,
                workspace=None, stream=None, o=None, g=None, phi_q=None, phi_k=None):
    """dq, dk, dv of sum(dO * O) for O = la_forward(q, k, v, causal, phi).

    ``o``, ``g``: the forward's output and denominators (la_forward(..., g=g));
    when given, the backward does not recompute them.  ``phi_q``, ``phi_k``:
    the forward's feature maps (la_forward(..., phi_out=(phi_q, phi_k))),
    only with ``o`` and ``g``; when given, phi is not evaluated again.
    """
    lib = load_library()
    _check_qkv("la_backward", q, dO)
    if q.dim() != 4:
        raise ValueError("la_backward: tensors must be [B, H, N, D]")
    Hkv = _check_kv("la_backward", q, k, v)
    B, H, N, D = q.shape
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    _check_qkv("la_backward", q, dq)
    _check_qkv("la_backward", k, dk, dv)
    _check_saved("la_backward", q, o, g, phi_q, phi_k)
    ws, ws_bytes = _workspace(LA_OP_BACKWARD, q, causal, workspace, Hkv)
    st = lib.la_backward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(o), _ptr(g), _ptr(phi_q),
                             _ptr(phi_k), _ptr(dq), _ptr(dk), _ptr(dv),
                             B, H, Hkv, N, D, DTYPE[q.dtype], int(bool(causal)), _phi(phi),
                             _ptr(ws), ws_bytes, _stream_handle(stream))
    _check("la_backward", st)
    return dq, dk, dv


def la_backward_noalloc(q, k, v, dO, causal: bool = True, phi="elu1", dq=None, dk=None,
                        dv=None, stream=None, o=None, g=None, phi_q=None, phi_k=None):
    """la_backward on the library's static device scratch (no workspace).

    For callers that cannot allocate device memory during the call; see
    la_backward_noalloc in include/la_api.h for the limits (a fixed maximum
    scratch size, one shared scratch array: overlapping calls race).  The
    output tensors dq, dk, dv are required: this wrapper allocates nothing
    either, and raises ValueError when one of them is missing.
    """
    lib = load_library()
    _check_qkv("la_backward_noalloc", q, k, v, dO)
    if q.dim() != 4:
        raise ValueError("la_backward_noalloc: tensors must be [B, H, N, D]")
    if dq is None or dk is None or dv is None:
        raise ValueError("la_backward_noalloc: pass dq, dk and dv (it allocates nothing)")
    B, H, N, D = q.shape
    _check_qkv("la_backward_noalloc", q, dq, dk, dv)
    _check_saved("la_backward_noalloc", q, o, g, phi_q, phi_k)
    st = lib.la_backward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(o), _ptr(g),
                                 _ptr(phi_q), _ptr(phi_k), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N,
                                 D, DTYPE[q.dtype], int(bool(causal)),
                                 _phi(phi), _stream_handle(stream))
    _check("la_backward_noalloc", st)
    return dq, dk, dv


def la_decode_step(S, z, q, k, v, phi="elu1", o=None, stream=None):
    """One in-place recurrent step: S, z (float32) updated, o [B, H, D] returned."""
    lib = load_library()
    _check_qkv("la_decode_step", q)
    if q.dim() != 3:
        raise ValueError("la_decode_step: q, k, v must be [B, H, D]")
    Hkv = _check_kv("la_decode_step", q, k, v)
    B, H, D = q.shape
    for name, t, shape in (("S", S, (B, Hkv, D, D)), ("z", z, (B, Hkv, D))):
        if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous() \
                or t.device != q.device:
            raise ValueError(f"la_decode_step: {name} must be contiguous float32 {shape} "
                             "on the device of q")
    if o is None:
        o = torch.empty_like(q)
    st = lib.la_decode_step_gqa(_ptr(S), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, Hkv,
                                D, DTYPE[q.dtype], _phi(phi), _stream_handle(stream))
    _check("la_decode_step", st)
    return o


# ------------------------------------------------------- decayed (gated) LA
def _gamma(gamma, H: int):
    """Per-head decay factors (host sequence, numpy array or tensor) as a
    ctypes float array of length H; the library checks the range."""
    if isinstance(gamma, torch.Tensor):
        gamma = gamma.detach().to("cpu", torch.float32).reshape(-1).tolist()
    vals = [float(x) for x in gamma]
    if len(vals) != H:
        raise ValueError(f"gamma must hold one factor per head ({H}), got {len(vals)}")
    return (ctypes.c_float * H)(*vals)


def la_workspace_size_decay(op: int, B: int, H: int, N: int, D: int, dtype: torch.dtype) -> int:
    return int(load_library().la_workspace_size_decay(int(op), B, H, N, D, DTYPE[dtype]))


def _workspace_decay(op, q, workspace):
    B, H, N, D = q.shape
    need = la_workspace_size_decay(op, B, H, N, D, q.dtype)
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    return workspace, workspace.numel() * workspace.element_size()


def la_forward_decay(q, k, v, gamma, phi="elu1", o=None, return_state=False, workspace=None,
                     stream=None, g=None):
    """Causal linear attention with a decay factor per head:
    S_i = gamma S_{i-1} + phi(k_i) v_i^T, z_i = gamma z_{i-1} + phi(k_i).
    ``gamma``: H factors in [0, 1] (host values).  ``g``: optional float32
    [B, H, N] tensor receiving the denominators (pass with o to
    la_backward_decay)."""
    lib = load_library()
    _check_qkv("la_forward_decay", q, k, v)
    if q.dim() != 4:
        raise ValueError("la_forward_decay: q, k, v must be [B, H, N, D]")
    B, H, N, D = q.shape
    gm = _gamma(gamma, H)
    o = torch.empty_like(q) if o is None else o
    _check_qkv("la_forward_decay", q, o)
    S = z = None
    if return_state:
        S = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
        z = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    if g is not None and (g.dtype != torch.float32 or tuple(g.shape) != (B, H, N)
                          or not g.is_contiguous() or g.device != q.device):
        raise ValueError("la_forward_decay: g must be contiguous float32 [B, H, N] on q's device")
    ws, ws_bytes = _workspace_decay(LA_OP_FORWARD, q, workspace)
    st = lib.la_forward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), _ptr(z), _ptr(g), gm,
                              B, H, N, D, DTYPE[q.dtype], _phi(phi), _ptr(ws), ws_bytes,
                              _stream_handle(stream))
    _check("la_forward_decay", st)
    return (o, S, z) if return_state else o


def la_backward_decay(q, k, v, dO, gamma, phi="elu1", dq=None, dk=None, dv=None,
                      workspace=None, stream=None, o=None, g=None):
    """dq, dk, dv of sum(dO * O) for O = la_forward_decay(q, k, v, gamma, phi)
    (no gradient with respect to gamma).  ``o``, ``g``: the forward's output
    and denominators, both or neither."""
    lib = load_library()
    _check_qkv("la_backward_decay", q, k, v, dO)
    if q.dim() != 4:
        raise ValueError("la_backward_decay: tensors must be [B, H, N, D]")
    B, H, N, D = q.shape
    gm = _gamma(gamma, H)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    _check_qkv("la_backward_decay", q, dq, dk, dv)
    _check_saved("la_backward_decay", q, o, g)
    ws, ws_bytes = _workspace_decay(LA_OP_BACKWARD, q, workspace)
    st = lib.la_backward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(o), _ptr(g), _ptr(dq),
                               _ptr(dk), _ptr(dv), gm, B, H, N, D, DTYPE[q.dtype], _phi(phi),
                               _ptr(ws), ws_bytes, _stream_handle(stream))
    _check("la_backward_decay", st)
    return dq, dk, dv


def la_decode_step_decay(S, z, q, k, v, gamma, phi="elu1", o=None, stream=None):
    """One decayed in-place step: S = gamma S + phi(k) v^T, z = gamma z +
    phi(k), o = S^T phi(q) / (phi(q) . z); returns o [B, H, D]."""
    lib = load_library()
    _check_qkv("la_decode_step_decay", q, k, v)
    if q.dim() != 3:
        raise ValueError("la_decode_step_decay: q, k, v must be [B, H, D]")
    B, H, D = q.shape
    gm = _gamma(gamma, H)
    for name, t, shape in (("S", S, (B, H, D, D)), ("z", z, (B, H, D))):
        if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous() \
                or t.device != q.device:
            raise ValueError(f"la_decode_step_decay: {name} must be contiguous float32 {shape} "
                             "on the device of q")
    o = torch.empty_like(q) if o is None else o
    st = lib.la_decode_step_decay(_ptr(S), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(o), gm, B, H,
                                  D, DTYPE[q.dtype], _phi(phi), _stream_handle(stream))
    _check("la_decode_step_decay", st)
    return o


# ------------------------------------------------ Performer FAVOR+ features
def _check_omega(name, x, omega):
    m = x.shape[-1]
    if (omega.dtype != x.dtype or omega.device != x.device or omega.dim() != 2
            or omega.shape[1] != x.shape[-1] or not omega.is_contiguous()):
        raise ValueError(f"{name}: omega must be a contiguous [m, D] tensor like x")
    return int(omega.shape[0]) if omega.dim() == 2 else m


def la_favor_features(x, omega, out=None, stream=None):
    """phi(x) = m^-1/2 exp(omega x - |x|^2/2) for x [B, H, N, D] (bf16) and
    omega [m, D]: the Performer's positive random features [B, H, N, m]."""
    lib = load_library()
    _check_qkv("la_favor_features", x)
    if x.dim() != 4:
        raise ValueError("la_favor_features: x must be [B, H, N, D]")
    m = _check_omega("la_favor_features", x, omega)
    B, H, N, D = x.shape
    out = torch.empty((B, H, N, m), dtype=x.dtype, device=x.device) if out is None else out
    if tuple(out.shape) != (B, H, N, m) or out.dtype != x.dtype or not out.is_contiguous():
        raise ValueError("la_favor_features: out must be contiguous [B, H, N, m] like x")
    st = lib.la_favor_features(_ptr(x), _ptr(omega), _ptr(out), B, H, N, D, m, DTYPE[x.dtype],
                               _stream_handle(stream))
    _check("la_favor_features", st)
    return out


def la_favor_features_backward(x, omega, dphi, dx=None, stream=None):
    """dx of sum(dphi * phi(x)) given x, omega and dphi (phi recomputed)."""
    lib = load_library()
    _check_qkv("la_favor_features_backward", x)
    m = _check_omega("la_favor_features_backward", x, omega)
    _check_qkv("la_favor_features_backward", dphi)
    B, H, N, D = x.shape
    if tuple(dphi.shape) != (B, H, N, m) or dphi.dtype != x.dtype:
        raise ValueError("la_favor_features_backward: dphi must be [B, H, N, m] like x")
    dx = torch.empty_like(x) if dx is None else dx
    _check_qkv("la_favor_features_backward", x, dx)
    st = lib.la_favor_features_backward(_ptr(x), _ptr(omega), _ptr(dphi), _ptr(dx), B, H, N, D, m,
                                        DTYPE[x.dtype], _stream_handle(stream))
    _check("la_favor_features_backward", st)
    return dx


# ------------------------------------- feature length m != head size D
def _check_mv(name, q, k, v, *vs):
    _check_qkv(name, q, k)
    _check_qkv(name, v, *vs)
    if q.dim() != 4 or v.dim() != 4 or q.shape[:3] != v.shape[:3] or q.device != v.device \
            or q.dtype != v.dtype:
        raise ValueError(f"{name}: q, k [B, H, N, Dk] and v [B, H, N, Dv] of one device and dtype")


def _workspace_mv(op, q, v, causal, workspace):
    B, H, N, Dk = q.shape
    need = int(load_library().la_workspace_size_mv(int(op), B, H, N, Dk, v.shape[-1],
                                                   int(bool(causal)), DTYPE[q.dtype]))
    if workspace is not None:
        have = workspace.numel() * workspace.element_size()
        if have < need:
            raise ValueError(f"workspace smaller than the {need} bytes needed")
        return workspace, have
    if need == 0:
        return None, 0
    return torch.empty(need, dtype=torch.uint8, device=q.device), need


def la_forward_mv(q, k, v, causal: bool = True, phi="identity", o=None, g=None, workspace=None,
                  stream=None):
    """o [B, H, N, Dv] of attention with features q, k [B, H, N, Dk] (e.g. m
    Performer features) and values v [B, H, N, Dv]."""
    lib = load_library()
    _check_mv("la_forward_mv", q, k, v)
    B, H, N, Dk = q.shape
    Dv = v.shape[-1]
    o = torch.empty_like(v) if o is None else o
    _check_qkv("la_forward_mv", v, o)
    if g is not None and (g.dtype != torch.float32 or tuple(g.shape) != (B, H, N)
                          or not g.is_contiguous()):
        raise ValueError("la_forward_mv: g must be contiguous float32 [B, H, N]")
    ws, ws_bytes = _workspace_mv(LA_OP_FORWARD, q, v, causal, workspace)
    st = lib.la_forward_mv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(g), B, H, N, Dk, Dv,
                           DTYPE[q.dtype], int(bool(causal)), _phi(phi), _ptr(ws), ws_bytes,
                           _stream_handle(stream))
    _check("la_forward_mv", st)
    return o


def la_backward_mv(q, k, v, dO, causal: bool = True, phi="identity", o=None, g=None, dq=None,
                   dk=None, dv=None, workspace=None, stream=None):
    """dq, dk [B, H, N, Dk] and dv [B, H, N, Dv] of sum(dO * O) for
    O = la_forward_mv(q, k, v, causal, phi); o, g optional as in la_backward."""
    lib = load_library()
    _check_mv("la_backward_mv", q, k, v, dO)
    B, H, N, Dk = q.shape
    Dv = v.shape[-1]
    if (o is None) != (g is None):
        raise ValueError("la_backward_mv: pass both o and g or neither")
    if o is not None:
        _check_qkv("la_backward_mv", v, o)
        if g.dtype != torch.float32 or tuple(g.shape) != (B, H, N) or not g.is_contiguous():
            raise ValueError("la_backward_mv: g must be contiguous float32 [B, H, N]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_qkv("la_backward_mv", q, dq, dk)
    _check_qkv("la_backward_mv", v, dv)
    ws, ws_bytes = _workspace_mv(LA_OP_BACKWARD, q, v, causal, workspace)
    st = lib.la_backward_mv(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(o), _ptr(g), _ptr(dq),
                            _ptr(dk), _ptr(dv), B, H, N, Dk, Dv, DTYPE[q.dtype],
                            int(bool(causal)), _phi(phi), _ptr(ws), ws_bytes,
                            _stream_handle(stream))
    _check("la_backward_mv", st)
    return dq, dk, dv


# ------------------------------------------------ sequence split across ranks
def la_workspace_size_sp(op: int, B: int, H: int, N: int, D: int, causal: bool,
                         dtype: torch.dtype) -> int:
    return int(load_library().la_workspace_size_sp(int(op), B, H, N, D, int(bool(causal)),
                                                   DTYPE[dtype]))


def _workspace_sp(op, x, causal, workspace):
    B, H, N, D = x.shape
    need = la_workspace_size_sp(op, B, H, N, D, causal, x.dtype)
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < need:
            raise ValueError(f"workspace smaller than the {need} bytes needed")
        return workspace, workspace.numel() * workspace.element_size()
    if need == 0:
        return None, 0
    workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    return workspace, need


def _state_records(name, t, B, H, D, device, lead=()):
    shape = (*lead, B, H, D * D + D)
    if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous() \
            or t.device != device:
        raise ValueError(f"{name}: state records must be contiguous float32 {shape}")


def la_state_local(k, v, phi="elu1", centred=False, out=None, workspace=None, stream=None):
    """This shard's state record per head, [B, H, D*D + D] float32: S (row =
    key feature) then z, of phi(k) - c (c = 0, or the backward's centring
    constant with ``centred``)."""
    lib = load_library()
    _check_qkv("la_state_local", k, v)
    B, H, N, D = k.shape
    out = torch.empty((B, H, D * D + D), dtype=torch.float32, device=k.device) \
        if out is None else out
    _state_records("la_state_local", out, B, H, D, k.device)
    ws, ws_bytes = _workspace_sp(LA_OP_FORWARD, k, True, workspace)
    st = lib.la_state_local(_ptr(k), _ptr(v), _ptr(out), B, H, N, D, DTYPE[k.dtype], _phi(phi),
                            int(bool(centred)), _ptr(ws), ws_bytes, _stream_handle(stream))
    _check("la_state_local", st)
    return out


def la_state_range_sum(states, lo: int, hi: int, out=None, stream=None):
    """Sum of the records of ranks lo..hi-1 from gathered records [P, B, H, R]."""
    lib = load_library()
    if states.dim() != 4:
        raise ValueError("la_state_range_sum: states must be [P, B, H, D*D + D]")
    P, B, H, R = states.shape
    D = int(round((-1 + (1 + 4 * R) ** 0.5) / 2))
    _state_records("la_state_range_sum", states, B, H, D, states.device, (P,))
    out = torch.empty((B, H, R), dtype=torch.float32, device=states.device) if out is None else out
    _state_records("la_state_range_sum", out, B, H, D, states.device)
    st = lib.la_state_range_sum(_ptr(states), P, int(lo), int(hi), _ptr(out), B, H, D,
                                _stream_handle(stream))
    _check("la_state_range_sum", st)
    return out


def la_forward_sp(q, k, v, state_in, causal: bool = True, phi="elu1", o=None, g=None,
                  state_out=None, workspace=None, stream=None):
    """la_forward on this rank's shard starting from ``state_in`` (the records
    of the shards before it, causal; of every shard, non-causal)."""
    lib = load_library()
    _check_qkv("la_forward_sp", q, k, v)
    B, H, N, D = q.shape
    _state_records("la_forward_sp", state_in, B, H, D, q.device)
    o = torch.empty_like(q) if o is None else o
    _check_qkv("la_forward_sp", q, o)
    if g is not None and (g.dtype != torch.float32 or tuple(g.shape) != (B, H, N)
                          or not g.is_contiguous()):
        raise ValueError("la_forward_sp: g must be contiguous float32 [B, H, N]")
    if state_out is not None:
        _state_records("la_forward_sp", state_out, B, H, D, q.device)
    ws, ws_bytes = _workspace_sp(LA_OP_FORWARD, q, causal, workspace)
    st = lib.la_forward_sp(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state_in), _ptr(state_out),
                           _ptr(g), B, H, N, D, DTYPE[q.dtype], int(bool(causal)), _phi(phi),
                           _ptr(ws), ws_bytes, _stream_handle(stream))
    _check("la_forward_sp", st)
    return o


def la_backward_sp_dq(q, k, v, dO, o, g, state_in, causal: bool = True, phi="elu1", dq=None,
                      state_out=None, workspace=None, stream=None):
    """First local backward step: (dq, this shard's query-side record,
    workspace); pass the workspace on to la_backward_sp_dkdv unchanged."""
    lib = load_library()
    _check_qkv("la_backward_sp_dq", q, k, v, dO, o)
    B, H, N, D = q.shape
    if g.dtype != torch.float32 or tuple(g.shape) != (B, H, N) or not g.is_contiguous():
        raise ValueError("la_backward_sp_dq: g must be contiguous float32 [B, H, N]")
    _state_records("la_backward_sp_dq", state_in, B, H, D, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    _check_qkv("la_backward_sp_dq", q, dq)
    state_out = torch.empty((B, H, D * D + D), dtype=torch.float32, device=q.device) \
        if state_out is None else state_out
    _state_records("la_backward_sp_dq", state_out, B, H, D, q.device)
    ws, ws_bytes = _workspace_sp(LA_OP_BACKWARD, q, causal, workspace)
    st = lib.la_backward_sp_dq(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(o), _ptr(g),
                               _ptr(state_in), _ptr(dq), _ptr(state_out), B, H, N, D,
                               DTYPE[q.dtype], int(bool(causal)), _phi(phi), _ptr(ws), ws_bytes,
                               _stream_handle(stream))
    _check("la_backward_sp_dq", st)
    return dq, state_out, ws


def la_backward_sp_dkdv(q, k, v, dO, g, state_in, workspace, causal: bool = True, phi="elu1",
                        dk=None, dv=None, stream=None):
    """Second local backward step: (dk, dv), with the workspace that
    la_backward_sp_dq filled."""
    lib = load_library()
    _check_qkv("la_backward_sp_dkdv", q, k, v, dO)
    B, H, N, D = q.shape
    _state_records("la_backward_sp_dkdv", state_in, B, H, D, q.device)
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_qkv("la_backward_sp_dkdv", k, dk, dv)
    need = la_workspace_size_sp(LA_OP_BACKWARD, B, H, N, D, causal, q.dtype)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if ws_bytes < need:
        raise ValueError("la_backward_sp_dkdv: pass the workspace la_backward_sp_dq filled")
    st = lib.la_backward_sp_dkdv(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(g), _ptr(state_in),
                                 _ptr(dk), _ptr(dv), B, H, N, D, DTYPE[q.dtype],
                                 int(bool(causal)), _phi(phi), _ptr(workspace), ws_bytes,
                                 _stream_handle(stream))
    _check("la_backward_sp_dkdv", st)
    return dk, dv


def la_get_device_error(stream=None) -> None:
    """Synchronise the stream and raise if a bounded device-side wait gave up."""
    _check("la_get_device_error", load_library().la_get_device_error(_stream_handle(stream)))


def la_selftest_wait_timeout(nthreads: int = 256, stream=None) -> None:
    """Launch the failure-detection self-test (a bounded device wait that is
    made to run out); la_get_device_error then raises with status
    LA_ERR_DEVICE_TIMEOUT."""
    _check("la_selftest_wait_timeout",
           load_library().la_selftest_wait_timeout(int(nthreads), _stream_handle(stream)))


def la_launch_count() -> int:
    """Kernels launched by liblinattn since it was loaded."""
    return int(load_library().la_launch_count())


def la_profile_enable(on: bool = True) -> None:
    """Bracket every library launch with CUDA events on its stream."""
    load_library().la_profile_enable(int(bool(on)))


def la_profile_collect() -> dict:
    """{kernel name: (launches, total ms)} since the last collect (synchronises)."""
    lib = load_library()
    buf = (ProfileEntry * 64)()
    n = lib.la_profile_collect(buf, 64)
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms))
            for i in range(min(n, 64))}


def backward_reads_phi(dtype, D: int) -> bool:
    """True where la_backward reads saved phi(q), phi(k) instead of
    evaluating the feature map (the bf16 head-size-64 passes: phi(q) in
    pass 1, both in pass 2); elsewhere they are ignored and asking the
    forward for them only costs a pass."""
    return dtype == torch.bfloat16 and D == 64


class LinearAttention(torch.autograd.Function):
    """torch autograd wrapper: forward and backward both run in liblinattn."""

    @staticmethod
    def forward(ctx, q, k, v, causal=True, phi="elu1"):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        B, H, N, _ = q.shape
        g = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        pq = pk = None
        if backward_reads_phi(q.dtype, q.shape[-1]) and k.shape[1] == H:
            pq, pk = torch.empty_like(q), torch.empty_like(k)
        o = la_forward(q, k, v, causal, phi, g=g,
                       phi_out=None if pq is None else (pq, pk))
        # the output, its denominators and the feature maps are kept so the
        # backward need not recompute the forward or evaluate phi again
        ctx.save_for_backward(q, k, v, o, g, pq, pk)
        ctx.causal, ctx.phi = causal, phi
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, o, g, pq, pk = ctx.saved_tensors
        dq, dk, dv = la_backward(q, k, v, dO.contiguous(), ctx.causal, ctx.phi, o=o, g=g,
                                 phi_q=pq, phi_k=pk)
        return dq, dk, dv, None, None
