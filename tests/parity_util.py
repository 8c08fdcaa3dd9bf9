"""Tolerances and comparison helpers for GPU-vs-oracle parity tests.

Tolerance reading: an element passes when |gpu - ref| <= atol + rtol*|ref|.
float32 inputs: atol 1e-4, rtol 0.  bfloat16 inputs (float32 accumulation,
bf16 outputs): atol 2e-2, rtol 1e-2.  The oracle is float64 and is never
rounded to the output dtype before the comparison.
"""
import numpy as np
import torch

TOL = {torch.float32: (1e-4, 0.0), torch.bfloat16: (2e-2, 1e-2)}


def compare(gpu, ref, dtype, what=""):
    """Assert elementwise parity; return (max_abs, max_rel, err_rms/ref_rms)."""
    atol, rtol = TOL[dtype]
    g = gpu.detach().to("cpu").double().numpy() if isinstance(gpu, torch.Tensor) else gpu
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    err = np.abs(g - r)
    bound = atol + rtol * np.abs(r)
    bad = err > bound
    max_abs = float(err.max()) if err.size else 0.0
    max_rel = float((err / np.maximum(np.abs(r), 1e-30)).max()) if err.size else 0.0
    rms_ratio = float(np.sqrt((err ** 2).mean()) / max(np.sqrt((r ** 2).mean()), 1e-30)) \
        if err.size else 0.0
    if bad.any():
        idx = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{bad.size} elements out of tolerance "
            f"(atol={atol}, rtol={rtol}); worst at {idx}: gpu={g[idx]!r} ref={r[idx]!r}; "
            f"max_abs={max_abs:.3e} max_rel={max_rel:.3e} err_rms/ref_rms={rms_ratio:.3e}")
    return max_abs, max_rel, rms_ratio
