"""Tolerances and comparison helpers for GPU-vs-oracle parity tests.

Two bounds, both asserted for every compared output:

1. Elementwise (the stated parity tolerance): an element passes when
   |gpu - ref| <= atol + rtol*|ref|.  float32 inputs: atol 1e-4, rtol 0.
   bfloat16 inputs (float32 accumulation, bf16 outputs): atol 2e-2, rtol 1e-2.

2. Normalised: err_rms/ref_rms <= eps_rms and max|err|/max|ref| <= eps_max.
   With inputs drawn at N(0,1)/sqrt(D) the gradients are far smaller than the
   elementwise atol (|dQ| ~ 1e-3), so bound 1 alone would accept an all-zero
   or sign-flipped gradient; bound 2 is scale-free and rejects both (ratio 1
   and 2) and a 10 % scale error (ratio 0.1).

   bfloat16: every value on the GPU path passes through at most five bf16
   roundings (the feature map, dU = dO/g, the masked C x C operand, the bf16
   state operand and the output), each a relative error of at most
   u = 2^-9 and, for round-to-nearest, of rms u/sqrt(3) ~ 2^-9.8.  Added
   independently they give an rms of about sqrt(5)*u/sqrt(3) ~ 2^-8.6, and
   the gradient sums that cancel (dA_i = sum_j b_j (v_j - o_i).du_i) cost
   at most a factor ~2 on top: eps_rms = 2^-6 keeps a 4x margin over that.
   The worst single element of ~1e5-1e7 sits a few rms away from the mean,
   so eps_max = 2^-5.
   float32: u = 2^-24 and the sums run over at most 2^17 tokens with a
   first-order bound of n*u, so eps_rms = 2^-14 and eps_max = 2^-11 (the
   decode step's base-2 exponential adds ~2^-22 relative, far below).

The oracle is float64 and is never rounded to the output dtype before the
comparison.  References that are zero in exact arithmetic (for example dQ
at N = 1, where v_1 - o_1 = 0) carry only float64 rounding residue; for
them (max|ref| below ZERO_REF) the normalised bound is skipped and the
elementwise one decides.

Setting PARITY_LOG=<path> appends one JSON line per comparison (name, dtype,
the four ratios) so that a GPU run can record the worst observed values.
"""
import json
import os

import numpy as np
import torch

TOL = {torch.float32: (1e-4, 0.0), torch.bfloat16: (2e-2, 1e-2)}
NORM = {torch.float32: (2.0 ** -14, 2.0 ** -11), torch.bfloat16: (2.0 ** -6, 2.0 ** -5)}
ZERO_REF = 1e-10


def _log(record):
    path = os.environ.get("PARITY_LOG")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps(record) + "\n")


def ratios(g, r):
    """(err_rms/ref_rms, max|err|/max|ref|, max_abs, max_rel) of arrays g, r."""
    err = np.abs(g - r)
    if err.size == 0:
        return 0.0, 0.0, 0.0, 0.0
    ref_rms = float(np.sqrt((r ** 2).mean()))
    ref_max = float(np.abs(r).max())
    rms_ratio = float(np.sqrt((err ** 2).mean())) / max(ref_rms, 1e-300)
    max_ratio = float(err.max()) / max(ref_max, 1e-300)
    max_rel = float((err / np.maximum(np.abs(r), 1e-30)).max())
    return rms_ratio, max_ratio, float(err.max()), max_rel


def compare(gpu, ref, dtype, what="", elementwise=True):
    """Assert elementwise and normalised parity; return (max_abs, max_rel,
    err_rms/ref_rms, max_err/max_ref).  elementwise=False skips the output
    tolerance (for sums such as the final state, bounded against their own
    scale by the caller)."""
    atol, rtol = TOL[dtype]
    eps_rms, eps_max = NORM[dtype]
    g = gpu.detach().to("cpu").double().numpy() if isinstance(gpu, torch.Tensor) else \
        np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    rms_ratio, max_ratio, max_abs, max_rel = ratios(g, r)
    normalised = r.size > 0 and float(np.abs(r).max()) >= ZERO_REF
    _log({"what": what, "dtype": str(dtype).replace("torch.", ""), "rms_ratio": rms_ratio,
          "max_ratio": max_ratio, "max_abs": max_abs, "normalised": normalised,
          "test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]})
    err = np.abs(g - r)
    bad = err > atol + rtol * np.abs(r)
    summary = (f"max_abs={max_abs:.3e} max_rel={max_rel:.3e} err_rms/ref_rms={rms_ratio:.3e} "
               f"max_err/max_ref={max_ratio:.3e}")
    if elementwise and bad.any():
        idx = np.unravel_index(np.argmax(err - (atol + rtol * np.abs(r))), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{bad.size} elements out of tolerance "
            f"(atol={atol}, rtol={rtol}); worst at {idx}: gpu={g[idx]!r} ref={r[idx]!r}; "
            f"{summary}")
    if normalised and (rms_ratio > eps_rms or max_ratio > eps_max):
        raise AssertionError(
            f"{what}: normalised error above bound (err_rms/ref_rms <= {eps_rms:.3e}, "
            f"max_err/max_ref <= {eps_max:.3e}); {summary}")
    return max_abs, max_rel, rms_ratio, max_ratio


def check_state(S, z, S_ref, z_ref, dtype):
    """Final (S, z): float32 sums over all N tokens.  Elementwise against the
    state's own scale (2e-5 for float32 inputs; for bf16 inputs the tensor
    cores sum phi(k) rounded to bf16, a relative error of at most 2^-9 per
    term that adds up like a random walk, bounded here by 4e-3 of the scale),
    plus the normalised bound of compare() (its elementwise output tolerance
    is an absolute bound for outputs of order one and does not apply to sums
    over N tokens)."""
    rel = 2e-5 if dtype == torch.float32 else 4e-3
    for name, got, ref in (("S", S, S_ref), ("z", z, z_ref)):
        g = got.double().cpu().numpy()
        scale = float(np.abs(ref).max())
        err = np.abs(g - ref)
        assert (err <= rel * scale + 1e-6).all(), \
            f"final {name}: max err {err.max():.3e} vs {rel:.1e} of scale {scale:.3e}"
        compare(got, ref, dtype, f"final {name}", elementwise=False)


def relu_branch_as_kernel(ref, x):
    """The oracle's dQ (x = q) or dK (x = k) for the relu+eps map with the
    branch phi'(x) taken as the bf16 tensor-core kernels take it: from the
    bf16 value phi(x) = bf16(max(x, 0) + 1e-6) they read, 1 where it exceeds
    bf16(1e-6) and 0 otherwise.  The two readings differ only for
    0 < x < ~4e-9 (where max(x, 0) + 1e-6 rounds to the x <= 0 value); there
    the oracle's gradient entry (taken with phi' = 1) becomes 0.  Where
    floating point decides a branch, both sides take it in the same (the
    kernel's) precision; everything else stays the oracle's."""
    xf = (x.detach().to("cpu") if isinstance(x, torch.Tensor) else torch.as_tensor(x)).float()
    phi_b = (torch.clamp(xf, min=0.0) + 1e-6).to(torch.bfloat16).float()
    floor = torch.tensor(1e-6, dtype=torch.float32).to(torch.bfloat16).float()
    mask = ((xf > 0) & (phi_b <= floor)).numpy()
    out = np.array(ref, dtype=np.float64, copy=True)
    out[mask] = 0.0
    return out
