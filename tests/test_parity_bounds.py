"""The parity check itself must be able to fail on a wrong result.

On the inputs of the bf16 backward parity tests (N(0,1)/sqrt(D) draws), the
gradients are much smaller than the elementwise atol: an all-zero or
sign-flipped dQ would pass the elementwise bound alone.  These CPU-only tests
show that compare() (elementwise + normalised bounds) rejects a zeroed, a
sign-flipped and a 10 %-scaled oracle gradient, and still accepts the oracle
rounded to the output dtype.  Nothing here runs GPU code: the "wrong"
results are planted in the oracle's own output on the CPU.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_transformers_b200 import inputs
from parity_util import NORM, TOL, compare, ratios


@pytest.fixture(scope="module")
def backward_refs():
    # the shape and seed of test_backward_small(bf16, D=64, N=777)
    q, k, v, dO = inputs.make_tensors(2, 2, 777, 64, torch.bfloat16, seed=777 * 11 + 64,
                                      with_grad_out=True)
    o, _, _ = oracle.forward(q, k, v, True, oracle.PHI_ELU1)
    dq, dk, dv = oracle.backward(q, k, v, dO, True, oracle.PHI_ELU1)
    return {"o": o, "dq": dq, "dk": dk, "dv": dv}


def test_elementwise_bound_alone_is_blind_here(backward_refs):
    # why the normalised bound exists: zero dQ is inside atol everywhere
    atol, rtol = TOL[torch.bfloat16]
    dq = backward_refs["dq"]
    assert (np.abs(dq) <= atol + rtol * np.abs(dq)).all()


@pytest.mark.parametrize("name", ["o", "dq", "dk", "dv"])
def test_rounded_oracle_passes(backward_refs, name):
    ref = backward_refs[name]
    got = torch.from_numpy(ref).to(torch.bfloat16)
    compare(got, ref, torch.bfloat16, f"bf16-rounded {name}")


@pytest.mark.parametrize("name", ["dq", "dk", "dv", "o"])
@pytest.mark.parametrize("mutation", ["zero", "sign", "scale1.1"])
def test_wrong_results_are_rejected(backward_refs, name, mutation):
    ref = backward_refs[name]
    wrong = {"zero": np.zeros_like(ref), "sign": -ref, "scale1.1": 1.1 * ref}[mutation]
    got = torch.from_numpy(wrong).to(torch.bfloat16)
    with pytest.raises(AssertionError):
        compare(got, ref, torch.bfloat16, f"{mutation} {name}")


def test_float32_bounds_reject_small_relative_errors(backward_refs):
    ref = backward_refs["dq"]
    with pytest.raises(AssertionError):
        compare(torch.from_numpy(ref * (1 + 1e-3)).float(), ref, torch.float32, "fp32 dq")
    compare(torch.from_numpy(ref).float(), ref, torch.float32, "fp32 dq rounded")


def test_ratios_of_planted_errors():
    r = np.array([1.0, -2.0, 3.0, -4.0])
    rms, mx, _, _ = ratios(np.zeros_like(r), r)
    assert rms == pytest.approx(1.0) and mx == pytest.approx(1.0)
    rms, mx, _, _ = ratios(-r, r)
    assert rms == pytest.approx(2.0) and mx == pytest.approx(2.0)
    eps_rms, eps_max = NORM[torch.bfloat16]
    assert eps_rms < 0.1 and eps_max < 0.1  # a 10 % scale error is caught


def test_relu_branch_as_kernel_changes_only_the_rounding_band():
    # bf16 inputs: exactly the x > 0 whose max(x, 0) + 1e-6 rounds to
    # bf16(1e-6) (here x below ~2e-9; 3e-9 already rounds up) take the
    # kernel's phi' = 0; every other entry is kept
    from parity_util import relu_branch_as_kernel
    x = torch.tensor([1.2e-9, 3e-9, 0.0, -1e-9, -1.0, 6e-9, 1e-8, 1e-3]).to(torch.bfloat16)
    out = relu_branch_as_kernel(np.arange(1.0, 9.0), x)
    np.testing.assert_array_equal(out, [0.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0, 8.0])
