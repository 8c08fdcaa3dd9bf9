"""GPU parity for the Performer's positive random features (FAVOR+) and for
Performer attention (the features through the linear-attention kernels
with the identity map), against the fp64 oracle's favor_features /
favor_features_backward and its attention functions (pinned on the CPU in
tests/test_oracle_pins.py)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_transformers_b200 import api, inputs
from parity_util import compare

pytestmark = pytest.mark.gpu


def qkv(B, H, N, D, seed, dO=False):
    return [t.cuda() for t in inputs.make_tensors(B, H, N, D, torch.bfloat16, seed,
                                                  with_grad_out=dO)]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", [1, 100, 128, 300, 1000])
def test_favor_features(D, N):
    x, _, _ = qkv(2, 3, N, D, seed=N + D)
    omega = inputs.make_favor_directions(D, D, seed=D).cuda()
    phi = api.la_favor_features(x, omega)
    torch.cuda.synchronize()
    api.la_get_device_error()
    ref = oracle.favor_features(x, omega)
    compare(phi, ref, torch.bfloat16, "phi")
    assert (phi > 0).all()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", [1, 129, 1000])
def test_favor_features_backward(D, N):
    x, _, _, dphi = qkv(2, 3, N, D, seed=3 * N + D, dO=True)
    omega = inputs.make_favor_directions(D, D, seed=D + 1).cuda()
    dx = api.la_favor_features_backward(x, omega, dphi)
    torch.cuda.synchronize()
    api.la_get_device_error()
    compare(dx, oracle.favor_features_backward(x, omega, dphi), torch.bfloat16, "dx")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", [129, 777])
@pytest.mark.parametrize("causal", [True, False])
def test_performer_attention_forward_backward(D, N, causal):
    q, k, v, dO = qkv(2, 4, N, D, seed=N + 7 * D, dO=True)
    omega = inputs.make_favor_directions(D, D, seed=2 * D).cuda()
    pq, pk = api.la_favor_features(q, omega), api.la_favor_features(k, omega)
    o = api.la_forward(pq, pk, v, causal, "identity")
    dpq, dpk, dv = api.la_backward(pq, pk, v, dO, causal, "identity")
    dq = api.la_favor_features_backward(q, omega, dpq)
    dk = api.la_favor_features_backward(k, omega, dpk)
    torch.cuda.synchronize()
    api.la_get_device_error()
    Fq, Fk = oracle.favor_features(q, omega), oracle.favor_features(k, omega)
    o_ref, _, _ = oracle.forward(Fq, Fk, v, causal, oracle.PHI_IDENTITY)
    dFq, dFk, dv_ref = oracle.backward(Fq, Fk, v, dO, causal, oracle.PHI_IDENTITY)
    compare(o, o_ref, torch.bfloat16, "o")
    compare(dv, dv_ref, torch.bfloat16, "dv")
    compare(dq, oracle.favor_features_backward(q, omega, dFq), torch.bfloat16, "dq")
    compare(dk, oracle.favor_features_backward(k, omega, dFk), torch.bfloat16, "dk")


def test_favor_rejects_unsupported_sizes():
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.LinearAttentionError):
        api.la_favor_features(x, torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda"))
    xf = torch.zeros(1, 1, 8, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(api.LinearAttentionError):
        api.la_favor_features(xf, torch.zeros(64, 64, dtype=torch.float32, device="cuda"))
