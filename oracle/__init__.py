"""fp64 CPU oracle for kernelized linear attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never touches it, and it shares no code with them.

The arithmetic lives in ``la_oracle.c`` (plain C, double precision, one head
at a time, OpenMP across heads); this module compiles it with gcc on first
use and marshals numpy arrays to it.  Inputs are converted to float64 first,
so a bf16 tensor enters the oracle with exactly the values the GPU reads.

Functions (all arrays [B, H, N, D] contiguous, D innermost):
  forward(q, k, v, causal, phi)            -> o, S_final, z_final
  quadratic(q, k, v, causal, phi)          -> o   (small N only)
  backward(q, k, v, dO, causal, phi)       -> dq, dk, dv
  decode_step(S, z, q, k, v, phi)          -> o   (updates S, z in place)
  phi_map(x, phi), dphi_map(x, phi)        -> elementwise feature map / slope
  forward_gqa / backward_gqa / decode_step_gqa: the same with k, v on fewer
  (key/value) heads, each shared by a group of query heads
  forward_decay(q, k, v, gamma, phi)       -> o, S_final, z_final  (causal)
  quadratic_decay(q, k, v, gamma, phi)     -> o   (small N only)
  backward_decay(q, k, v, dO, gamma, phi)  -> dq, dk, dv
  decode_step_decay(S, z, q, k, v, gamma, phi) -> o  (updates S, z in place)
      the decayed (gated) recurrence S_i = gamma S_{i-1} + b_i v_i^T, z_i =
      gamma z_{i-1} + b_i with one gamma in [0, 1] per head (gamma [H])
  favor_features(x, omega)                 -> phi(x) [..., m]  (Performer)
  favor_features_backward(x, omega, dphi)  -> dx
      the positive random features of the Performer (FAVOR+), phi(x) =
      m^-1/2 exp(-|x|^2/2) [exp(w_1.x), ..., exp(w_m.x)], omega [m, D] the
      random directions; with phi = PHI_IDENTITY the functions above then
      take phi(q), phi(k) as their q, k
  forward_mv(q, k, v, causal, phi)         -> o [..., Dv]
  backward_mv(q, k, v, dO, causal, phi)    -> dq, dk [..., Dk], dv [..., Dv]
      features q, k of length Dk (e.g. m Performer features) and values of
      length Dv: S is Dk x Dv
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

PHI_ELU1 = 0
PHI_RELU_EPS = 1
PHI_IDENTITY = 2  # inputs are feature vectors already (Performer features)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile la_oracle.c into liboracle.so next to it (gcc, -fopenmp)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            ci = ctypes.c_int
            lib.oracle_forward.argtypes = [P, P, P, P, P, P, i64, i64, i64, i64, ci, ci]
            lib.oracle_quadratic.argtypes = [P, P, P, P, i64, i64, i64, i64, ci, ci]
            lib.oracle_backward.argtypes = [P, P, P, P, P, P, P, i64, i64, i64, i64, ci, ci]
            lib.oracle_decode_step.argtypes = [P, P, P, P, P, P, i64, i64, i64, ci]
            lib.oracle_forward_decay.argtypes = [P, P, P, P, P, P, P, i64, i64, i64, i64, ci]
            lib.oracle_quadratic_decay.argtypes = [P, P, P, P, P, i64, i64, i64, i64, ci]
            lib.oracle_backward_decay.argtypes = [P, P, P, P, P, P, P, P, i64, i64, i64, i64, ci]
            lib.oracle_decode_step_decay.argtypes = [P, P, P, P, P, P, P, i64, i64, i64, ci]
            lib.oracle_set_threads.argtypes = [ci]
            lib.oracle_max_threads.restype = ci
            for fn in ("oracle_forward", "oracle_quadratic", "oracle_backward",
                       "oracle_decode_step", "oracle_set_threads", "oracle_forward_decay",
                       "oracle_quadratic_decay", "oracle_backward_decay",
                       "oracle_decode_step_decay"):
                getattr(lib, fn).restype = None
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a (CPU/GPU) torch tensor."""
    if not isinstance(x, np.ndarray):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _shape4(q):
    if q.ndim != 4:
        raise ValueError("expected [B, H, N, D]")
    return q.shape


def forward(q, k, v, causal: bool, phi: int = PHI_ELU1):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = _shape4(q)
    o = np.empty_like(q)
    S = np.empty((B, H, D, D))
    z = np.empty((B, H, D))
    _load().oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), _ptr(z),
                           B, H, N, D, int(bool(causal)), int(phi))
    return o, S, z


def quadratic(q, k, v, causal: bool, phi: int = PHI_ELU1):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = _shape4(q)
    o = np.empty_like(q)
    _load().oracle_quadratic(_ptr(q), _ptr(k), _ptr(v), _ptr(o),
                             B, H, N, D, int(bool(causal)), int(phi))
    return o


def backward(q, k, v, dO, causal: bool, phi: int = PHI_ELU1):
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, D = _shape4(q)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dq), _ptr(dk),
                            _ptr(dv), B, H, N, D, int(bool(causal)), int(phi))
    return dq, dk, dv


def decode_step(S: np.ndarray, z: np.ndarray, q, k, v, phi: int = PHI_ELU1):
    """One in-place step on float64 arrays S [B,H,D,D], z [B,H,D]; q,k,v [B,H,D]."""
    if S.dtype != np.float64 or not S.flags.c_contiguous:
        raise TypeError("S must be a C-contiguous float64 array (updated in place)")
    if z.dtype != np.float64 or not z.flags.c_contiguous:
        raise TypeError("z must be a C-contiguous float64 array (updated in place)")
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, D = q.shape
    o = np.empty_like(q)
    _load().oracle_decode_step(_ptr(S), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                               B, H, D, int(phi))
    return o


# ------------------------------------------------------- decayed (gated) LA
def _gamma(gamma, H: int) -> np.ndarray:
    g = np.ascontiguousarray(np.asarray(gamma, dtype=np.float64).reshape(-1))
    if g.shape != (H,):
        raise ValueError(f"gamma must hold one factor per head ({H})")
    if not ((g >= 0.0) & (g <= 1.0)).all():
        raise ValueError("gamma must lie in [0, 1]")
    return g


def forward_decay(q, k, v, gamma, phi: int = PHI_ELU1):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = _shape4(q)
    g = _gamma(gamma, H)
    o = np.empty_like(q)
    S = np.empty((B, H, D, D))
    z = np.empty((B, H, D))
    _load().oracle_forward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), _ptr(S), _ptr(z),
                                 B, H, N, D, int(phi))
    return o, S, z


def quadratic_decay(q, k, v, gamma, phi: int = PHI_ELU1):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = _shape4(q)
    g = _gamma(gamma, H)
    o = np.empty_like(q)
    _load().oracle_quadratic_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), B, H, N, D,
                                   int(phi))
    return o


def backward_decay(q, k, v, dO, gamma, phi: int = PHI_ELU1):
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, D = _shape4(q)
    g = _gamma(gamma, H)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    _load().oracle_backward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(g), _ptr(dq),
                                  _ptr(dk), _ptr(dv), B, H, N, D, int(phi))
    return dq, dk, dv


def decode_step_decay(S: np.ndarray, z: np.ndarray, q, k, v, gamma, phi: int = PHI_ELU1):
    """One decayed in-place step on float64 S [B,H,D,D], z [B,H,D]; q,k,v [B,H,D]."""
    if S.dtype != np.float64 or not S.flags.c_contiguous:
        raise TypeError("S must be a C-contiguous float64 array (updated in place)")
    if z.dtype != np.float64 or not z.flags.c_contiguous:
        raise TypeError("z must be a C-contiguous float64 array (updated in place)")
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, D = q.shape
    g = _gamma(gamma, H)
    o = np.empty_like(q)
    _load().oracle_decode_step_decay(_ptr(S), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                     _ptr(o), B, H, D, int(phi))
    return o


# ------------------------------------------------ Performer FAVOR+ features
# "Efficient Transformers Survey", Low-Rank Approximations, Performer:
# phi(x) = m^-1/2 exp(-|x|^2/2) [exp(w_1^T x), ..., exp(w_m^T x)], w_i drawn
# from N(0, I_d) (passed in as omega [m, D]); phi(q)^T phi(k) is an unbiased
# estimate of exp(q^T k) (Proposition "Performer Approximation Quality").
# The 1/sqrt(d) of softmax attention is the caller's pre-normalisation of q
# and k (x = q / d^(1/4)), as the page states.

def favor_features(x, omega) -> np.ndarray:
    """phi(x) for x [..., D] and omega [m, D]: float64 [..., m]."""
    x = _f64(x)
    w = _f64(omega)
    m = w.shape[0]
    proj = x @ w.T                                   # w_i^T x
    half_sq = 0.5 * (x * x).sum(axis=-1, keepdims=True)
    return np.exp(proj - half_sq) / np.sqrt(m)


def favor_features_backward(x, omega, dphi) -> np.ndarray:
    """dx of sum(dphi * phi(x)): d phi_i / dx = phi_i (w_i - x), so
    dx = sum_i dphi_i phi_i w_i - x sum_i dphi_i phi_i."""
    x = _f64(x)
    w = _f64(omega)
    g = _f64(dphi) * favor_features(x, w)            # dphi_i phi_i
    return g @ w - x * g.sum(axis=-1, keepdims=True)


# ------------------------------------------- feature length m != head size D
# The Proposition "Linear Attention via Kernel Decomposition" takes phi:
# R^d -> R^m, so S = sum_j phi(k_j) v_j^T is m x D ("Efficient Transformers
# Survey"; with the Performer's m random features, Low-Rank Approximations,
# Performer).  The functions above take one width for q, k and v; these
# widen the narrower side with zero columns and cut the result back, which
# is the same sums: a zero value column gives a zero output column (and dV
# column), a zero feature column adds 0 to every a_i . b_j and to z (given
# features, phi = PHI_IDENTITY, so the zero stays zero).

def _widen(x, w: int) -> np.ndarray:
    x = _f64(x)
    out = np.zeros((*x.shape[:-1], w))
    out[..., :x.shape[-1]] = x
    return out


def forward_mv(q, k, v, causal: bool, phi: int = PHI_IDENTITY) -> np.ndarray:
    """o [B, H, N, Dv] for features q, k [B, H, N, Dk] and values v [..., Dv]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    dk, dv = q.shape[-1], v.shape[-1]
    if dk < dv and phi != PHI_IDENTITY:
        raise ValueError("zero feature columns need the identity map")
    D = max(dk, dv)
    o, _, _ = forward(_widen(q, D), _widen(k, D), _widen(v, D), causal, phi)
    return np.ascontiguousarray(o[..., :dv])


def backward_mv(q, k, v, dO, causal: bool, phi: int = PHI_IDENTITY):
    """dq, dk [B, H, N, Dk] and dv [B, H, N, Dv] of sum(dO * O)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    dk_, dv_ = q.shape[-1], v.shape[-1]
    if dk_ < dv_ and phi != PHI_IDENTITY:
        raise ValueError("zero feature columns need the identity map")
    D = max(dk_, dv_)
    dq, dk, dv = backward(_widen(q, D), _widen(k, D), _widen(v, D), _widen(dO, D), causal, phi)
    return (np.ascontiguousarray(dq[..., :dk_]), np.ascontiguousarray(dk[..., :dk_]),
            np.ascontiguousarray(dv[..., :dv_]))


# ---------------------------------------------------- grouped key/value heads
# Grouped-query / multi-query attention ("Attention Optimization", Advanced
# Techniques: Multi-Query Attention and Grouped-Query Attention): Hkv
# key/value heads, each shared by G = H / Hkv consecutive query heads.  By
# definition this is the per-head attention above with every query head h
# given k, v of head h // G: the functions below expand k, v to one copy
# per query head and call the functions above; the gradient with respect to
# a shared k or v is the sum over the query heads that read it.

def expand_kv(x, H: int) -> np.ndarray:
    """[B, Hkv, ...] -> [B, H, ...], head h taking head h // (H // Hkv)."""
    x = _f64(x)
    hkv = x.shape[1]
    if hkv < 1 or H % hkv:
        raise ValueError("H must be a multiple of the key/value heads")
    return np.ascontiguousarray(np.repeat(x, H // hkv, axis=1))


def group_sum(x, Hkv: int) -> np.ndarray:
    """[B, H, ...] -> [B, Hkv, ...]: the sum over each group of H // Hkv heads."""
    x = np.asarray(x, dtype=np.float64)
    B, H = x.shape[:2]
    return x.reshape(B, Hkv, H // Hkv, *x.shape[2:]).sum(axis=2)


def forward_gqa(q, k, v, causal: bool, phi: int = PHI_ELU1):
    """o [B, H, N, D] and the final state per key/value head."""
    q = _f64(q)
    H, Hkv = q.shape[1], _f64(k).shape[1]
    o, S, z = forward(q, expand_kv(k, H), expand_kv(v, H), causal, phi)
    G = H // Hkv
    return o, np.ascontiguousarray(S[:, ::G]), np.ascontiguousarray(z[:, ::G])


def backward_gqa(q, k, v, dO, causal: bool, phi: int = PHI_ELU1):
    """dq [B, H, N, D]; dk, dv [B, Hkv, N, D] summed over each group."""
    q = _f64(q)
    H, Hkv = q.shape[1], _f64(k).shape[1]
    dq, dk, dv = backward(q, expand_kv(k, H), expand_kv(v, H), dO, causal, phi)
    return dq, group_sum(dk, Hkv), group_sum(dv, Hkv)


def decode_step_gqa(S: np.ndarray, z: np.ndarray, q, k, v, phi: int = PHI_ELU1):
    """One step with per-key/value-head state S [B, Hkv, D, D], z [B, Hkv, D]
    (updated in place); q [B, H, D], k, v [B, Hkv, D]; returns o [B, H, D].
    The state is updated once per key/value head, then every query head of
    the group reads it."""
    q = _f64(q)
    H, Hkv = q.shape[1], S.shape[1]
    G = H // Hkv
    # every query head steps its own copy of its group's state (all copies
    # of a group receive the same update), then one copy per group is kept
    S_x = np.ascontiguousarray(np.repeat(S, G, axis=1))
    z_x = np.ascontiguousarray(np.repeat(z, G, axis=1))
    o = decode_step(S_x, z_x, q, expand_kv(k, H), expand_kv(v, H), phi)
    S[...] = S_x[:, ::G]
    z[...] = z_x[:, ::G]
    return o


def phi_map(x, phi: int = PHI_ELU1) -> np.ndarray:
    """The elementwise feature map on float64 values (elu+1 or relu+1e-6)."""
    x = _f64(x)
    if phi == PHI_ELU1:
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    return np.maximum(x, 0.0) + 1e-6


def dphi_map(x, phi: int = PHI_ELU1) -> np.ndarray:
    x = _f64(x)
    if phi == PHI_ELU1:
        return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))
    return np.where(x > 0, 1.0, 0.0)
