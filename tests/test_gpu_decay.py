"""GPU parity for decayed (gated) linear attention, S_i = gamma S_{i-1} +
phi(k_i) v_i^T with one gamma per head: the forward, the backward and the
decode step through the C ABI against the fp64 oracle's decayed functions
(pinned on the CPU in tests/test_oracle_pins.py)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_transformers_b200 import api, inputs
from parity_util import check_state, compare

pytestmark = pytest.mark.gpu

PHIS = {"elu1": oracle.PHI_ELU1, "relu_eps": oracle.PHI_RELU_EPS}


def gammas(H, lo=0.5):
    """H factors spread over [lo, 1], the last exactly 1."""
    return np.linspace(lo, 1.0, H).astype(np.float32)


def tensors(B, H, N, D, dtype, seed, dO=False):
    return [t.cuda() for t in inputs.make_tensors(B, H, N, D, dtype, seed, with_grad_out=dO)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("N", [1, 129, 777])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
def test_decay_forward(dtype, D, N, phi):
    B, H = 2, 4
    q, k, v = tensors(B, H, N, D, dtype, seed=N + D)
    gm = gammas(H, 0.3)
    g = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    o, S, z = api.la_forward_decay(q, k, v, gm, phi, return_state=True, g=g)
    torch.cuda.synchronize()
    api.la_get_device_error()
    o_ref, S_ref, z_ref = oracle.forward_decay(q, k, v, gm.astype(np.float64), PHIS[phi])
    compare(o, o_ref, dtype, "o")
    check_state(S, z, S_ref, z_ref, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [16, 64, 128])
@pytest.mark.parametrize("N", [1, 129, 777])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
@pytest.mark.parametrize("saved", [False, True])
def test_decay_backward(dtype, D, N, phi, saved):
    B, H = 2, 3
    q, k, v, dO = tensors(B, H, N, D, dtype, seed=N + 3 * D, dO=True)
    gm = gammas(H, 0.6)
    if saved:
        g = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
        o = api.la_forward_decay(q, k, v, gm, phi, g=g)
        dq, dk, dv = api.la_backward_decay(q, k, v, dO, gm, phi, o=o, g=g)
    else:
        dq, dk, dv = api.la_backward_decay(q, k, v, dO, gm, phi)
    torch.cuda.synchronize()
    api.la_get_device_error()
    rq, rk, rv = oracle.backward_decay(q, k, v, dO, gm.astype(np.float64), PHIS[phi])
    compare(dq, rq, dtype, "dq")
    compare(dk, rk, dtype, "dk")
    compare(dv, rv, dtype, "dv")


def test_decay_of_one_is_the_causal_call():
    # gamma = 1 everywhere: the decayed call equals the plain causal one (the
    # token-sequential kernels give bitwise the same numbers for float32)
    q, k, v = tensors(1, 2, 300, 32, torch.float32, seed=5)
    o1 = api.la_forward_decay(q, k, v, [1.0, 1.0])
    o0 = api.la_forward(q, k, v, True)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1)


def test_decay_zero_returns_the_values():
    q, k, v = tensors(2, 2, 65, 64, torch.float32, seed=6)
    o = api.la_forward_decay(q, k, v, [0.0, 0.0])
    torch.cuda.synchronize()
    compare(o, v.double().cpu().numpy(), torch.float32, "o = v")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [16, 64, 128])
def test_decay_decode_continues_the_decayed_forward(dtype, D):
    B, H, T0, T1 = 3, 4, 50, 6
    q, k, v = tensors(B, H, T0 + T1, D, dtype, seed=D)
    gm = gammas(H, 0.7)
    _, S, z = api.la_forward_decay(q[:, :, :T0].contiguous(), k[:, :, :T0].contiguous(),
                                   v[:, :, :T0].contiguous(), gm, return_state=True)
    o_ref, S_ref, z_ref = oracle.forward_decay(q, k, v, gm.astype(np.float64))
    for t in range(T0, T0 + T1):
        o_t = api.la_decode_step_decay(S, z, q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                       v[:, :, t].contiguous(), gm)
        compare(o_t, o_ref[:, :, t], dtype, f"decode step {t}")
    check_state(S, z, S_ref, z_ref, dtype)


def test_decay_rejects_bad_factors():
    q, k, v = tensors(1, 2, 16, 64, torch.bfloat16, seed=1)
    for bad in ([0.5, 1.5], [0.5, float("nan")], [-0.1, 0.5]):
        with pytest.raises(api.LinearAttentionError):
            api.la_forward_decay(q, k, v, bad)
    with pytest.raises(ValueError):
        api.la_forward_decay(q, k, v, [0.5])


# ----------------------------------------------- tensor-core decayed forward
# bf16 with D = 64 (128-token chunks) or D = 128 (64-token chunks) and every
# gamma >= 2^(-64/C) runs the chunked tcgen05 kernels with chunk-local decay
# factors; the profile shows which kernels ran.

def _launched(fn):
    api.la_profile_collect()
    api.la_profile_enable(True)
    try:
        out = fn()
        torch.cuda.synchronize()
        return out, api.la_profile_collect()
    finally:
        api.la_profile_enable(False)


CHUNK_GMIN = {64: 2.0 ** -0.5, 128: 0.5}


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", [1, 100, 129, 777, 1000])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
def test_decay_forward_chunked(D, N, phi):
    B, H = 2, 4
    q, k, v = tensors(B, H, N, D, torch.bfloat16, seed=7 * N + D)
    gm = np.array([CHUNK_GMIN[D], 0.9, 0.99, 1.0], dtype=np.float32)
    g = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    (o, S, z), prof = _launched(lambda: api.la_forward_decay(q, k, v, gm, phi, return_state=True,
                                                             g=g))
    api.la_get_device_error()
    assert "chunk_causal" in prof and "fwd_generic" not in prof, prof
    o_ref, S_ref, z_ref = oracle.forward_decay(q, k, v, gm.astype(np.float64), PHIS[phi])
    compare(o, o_ref, torch.bfloat16, "o")
    check_state(S, z, S_ref, z_ref, torch.bfloat16)


@pytest.mark.parametrize("D", [64, 128])
def test_decay_forward_chunked_segments(D):
    # few heads, long sequence: segment states (REDUCE decayed to each
    # segment's end), the decayed exclusive scan, then the causal pass
    B, H, N = 1, 2, 20000
    q, k, v = tensors(B, H, N, D, torch.bfloat16, seed=D + 1)
    gm = np.array([0.97, 0.9995], dtype=np.float32)
    (o, S, z), prof = _launched(lambda: api.la_forward_decay(q, k, v, gm, return_state=True))
    api.la_get_device_error()
    assert "chunk_reduce" in prof and "state_scan" in prof and "chunk_causal" in prof, prof
    o_ref, S_ref, z_ref = oracle.forward_decay(q, k, v, gm.astype(np.float64))
    compare(o, o_ref, torch.bfloat16, "o")
    check_state(S, z, S_ref, z_ref, torch.bfloat16)


def test_decay_below_the_chunked_range_runs_token_sequential():
    q, k, v = tensors(1, 2, 300, 64, torch.bfloat16, seed=9)
    gm = np.array([0.6, 0.99], dtype=np.float32)  # 0.6 < 2^-0.5
    o, prof = _launched(lambda: api.la_forward_decay(q, k, v, gm))
    assert "fwd_generic" in prof and "chunk_causal" not in prof, prof
    compare(o, oracle.forward_decay(q, k, v, gm.astype(np.float64))[0], torch.bfloat16, "o")


def test_decay_chunked_matches_token_sequential_gamma_one():
    # gamma = 1 through the decayed chunked kernels: the undecayed causal
    # result within bf16 rounding (the same arithmetic with unit factors)
    q, k, v = tensors(2, 2, 1000, 64, torch.bfloat16, seed=11)
    o1 = api.la_forward_decay(q, k, v, [1.0, 1.0])
    o0 = api.la_forward(q, k, v, True)
    torch.cuda.synchronize()
    compare(o1, o0.double().cpu().numpy(), torch.bfloat16, "gamma 1 vs plain")


# ---------------------------------------------- tensor-core decayed backward
# bf16, D = 64, every gamma >= 2^(-0.5), one segment per head (fewer than 4
# chunks, or enough heads to fill the GPU): the pipelined dQ and dK/dV
# passes with chunk-local decay factors.

@pytest.mark.parametrize("N", [1, 100, 129, 300, 384])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
@pytest.mark.parametrize("saved", [False, True])
def test_decay_backward_chunked(N, phi, saved):
    B, H, D = 2, 4, 64
    q, k, v, dO = tensors(B, H, N, D, torch.bfloat16, seed=5 * N + 1, dO=True)
    gm = np.array([CHUNK_GMIN[D], 0.9, 0.99, 1.0], dtype=np.float32)

    def run():
        if saved:
            g = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
            o = api.la_forward_decay(q, k, v, gm, phi, g=g)
            return api.la_backward_decay(q, k, v, dO, gm, phi, o=o, g=g)
        return api.la_backward_decay(q, k, v, dO, gm, phi)

    (dq, dk, dv), prof = _launched(run)
    api.la_get_device_error()
    assert "bwd_dq" in prof and "bwd_dkdv" in prof and "bwd_generic" not in prof, prof
    rq, rk, rv = oracle.backward_decay(q, k, v, dO, gm.astype(np.float64), PHIS[phi])
    compare(dq, rq, torch.bfloat16, "dq")
    compare(dk, rk, torch.bfloat16, "dk")
    compare(dv, rv, torch.bfloat16, "dv")


@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
def test_decay_backward_chunked_many_heads(phi):
    # 128 heads keep one segment per head at N = 1000 (8 chunks, ragged
    # tail), with the retention-style factors of the decayed training
    # workload (the chunked range's lower edge is covered at small N above)
    B, H, N, D = 4, 32, 1000, 64
    q, k, v, dO = tensors(B, H, N, D, torch.bfloat16, seed=77, dO=True)
    gm = np.array(inputs.decay_factors(H), dtype=np.float32)
    (dq, dk, dv), prof = _launched(lambda: api.la_backward_decay(q, k, v, dO, gm, phi))
    api.la_get_device_error()
    assert "bwd_dq" in prof and "bwd_generic" not in prof, prof
    rq, rk, rv = oracle.backward_decay(q, k, v, dO, gm.astype(np.float64), PHIS[phi])
    compare(dq, rq, torch.bfloat16, "dq")
    compare(dk, rk, torch.bfloat16, "dk")
    compare(dv, rv, torch.bfloat16, "dv")
