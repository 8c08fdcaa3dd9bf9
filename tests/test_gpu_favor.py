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


DM = [(64, 64), (128, 128), (64, 128), (128, 64)]  # (head size D, features m)


@pytest.mark.parametrize("D,m", DM)
@pytest.mark.parametrize("N", [1, 100, 128, 300, 1000])
def test_favor_features(D, m, N):
    x, _, _ = qkv(2, 3, N, D, seed=N + D)
    omega = inputs.make_favor_directions(m, D, seed=D + m).cuda()
    phi = api.la_favor_features(x, omega)
    torch.cuda.synchronize()
    api.la_get_device_error()
    ref = oracle.favor_features(x, omega)
    assert phi.shape == (2, 3, N, m)
    compare(phi, ref, torch.bfloat16, "phi")
    assert (phi > 0).all()


@pytest.mark.parametrize("D,m", DM)
@pytest.mark.parametrize("N", [1, 129, 1000])
def test_favor_features_backward(D, m, N):
    x, _, _ = qkv(2, 3, N, D, seed=3 * N + D)
    dphi = qkv(2, 3, N, m, seed=5 * N + m)[0] * 8.0
    omega = inputs.make_favor_directions(m, D, seed=D + m + 1).cuda()
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


@pytest.mark.parametrize("D,m", [(64, 128), (128, 64)])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("saved", [False, True])
def test_performer_attention_with_m_features(D, m, causal, saved):
    # m random features of head-size-D queries and keys; values of size D:
    # S is m x D (features and values of two lengths through la_*_mv)
    N = 777
    q, k, v, dO = qkv(2, 3, N, D, seed=N + 3 * D + m, dO=True)
    omega = inputs.make_favor_directions(m, D, seed=D + 2 * m).cuda()
    pq, pk = api.la_favor_features(q, omega), api.la_favor_features(k, omega)
    if saved:
        g = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
        o = api.la_forward_mv(pq, pk, v, causal, "identity", g=g)
        dpq, dpk, dv = api.la_backward_mv(pq, pk, v, dO, causal, "identity", o=o, g=g)
    else:
        o = api.la_forward_mv(pq, pk, v, causal, "identity")
        dpq, dpk, dv = api.la_backward_mv(pq, pk, v, dO, causal, "identity")
    dq = api.la_favor_features_backward(q, omega, dpq)
    dk = api.la_favor_features_backward(k, omega, dpk)
    torch.cuda.synchronize()
    api.la_get_device_error()
    assert o.shape == v.shape and dpq.shape == pq.shape and dv.shape == v.shape
    Fq, Fk = oracle.favor_features(q, omega), oracle.favor_features(k, omega)
    dFq, dFk, dv_ref = oracle.backward_mv(Fq, Fk, v, dO, causal, oracle.PHI_IDENTITY)
    compare(o, oracle.forward_mv(Fq, Fk, v, causal, oracle.PHI_IDENTITY), torch.bfloat16, "o")
    compare(dv, dv_ref, torch.bfloat16, "dv")
    compare(dq, oracle.favor_features_backward(q, omega, dFq), torch.bfloat16, "dq")
    compare(dk, oracle.favor_features_backward(k, omega, dFk), torch.bfloat16, "dk")


@pytest.mark.parametrize("causal", [True, False])
def test_mv_with_a_feature_map_and_shorter_values(causal):
    # q, k of length 128 through elu+1, values of length 64
    N = 300
    q, k, _ = qkv(2, 2, N, 128, seed=31)
    v, _, _, dO = qkv(2, 2, N, 64, seed=32, dO=True)
    o = api.la_forward_mv(q, k, v, causal, "elu1")
    dq, dk, dv = api.la_backward_mv(q, k, v, dO, causal, "elu1")
    torch.cuda.synchronize()
    api.la_get_device_error()
    compare(o, oracle.forward_mv(q, k, v, causal, oracle.PHI_ELU1), torch.bfloat16, "o")
    rq, rk, rv = oracle.backward_mv(q, k, v, dO, causal, oracle.PHI_ELU1)
    compare(dq, rq, torch.bfloat16, "dq")
    compare(dk, rk, torch.bfloat16, "dk")
    compare(dv, rv, torch.bfloat16, "dv")


def test_favor_rejects_unsupported_sizes():
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.LinearAttentionError):
        api.la_favor_features(x, torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda"))
    # features shorter than the values need the identity map
    v = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.LinearAttentionError):
        api.la_forward_mv(x, x, v, True, "elu1")
    xf = torch.zeros(1, 1, 8, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(api.LinearAttentionError):
        api.la_favor_features(xf, torch.zeros(64, 64, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("N", [1, 64, 129])
@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 128)])
def test_mv_short_sequences(N, dk, dv):
    # identity-map attention with feature and value lengths of their own at
    # one token, one chunk and a ragged tail
    g = torch.Generator().manual_seed(N + dk)
    pq = (torch.rand((2, 2, N, dk), generator=g) + 0.05).to(torch.bfloat16).cuda()
    pk = (torch.rand((2, 2, N, dk), generator=g) + 0.05).to(torch.bfloat16).cuda()
    v, _, _, dO = qkv(2, 2, N, dv, seed=N + dv, dO=True)
    for causal in (True, False):
        o = api.la_forward_mv(pq, pk, v, causal, "identity")
        dpq, dpk, dvv = api.la_backward_mv(pq, pk, v, dO, causal, "identity")
        torch.cuda.synchronize()
        api.la_get_device_error()
        compare(o, oracle.forward_mv(pq, pk, v, causal), torch.bfloat16, "o")
        rq, rk, rv = oracle.backward_mv(pq, pk, v, dO, causal)
        compare(dpq, rq, torch.bfloat16, "dq")
        compare(dpk, rk, torch.bfloat16, "dk")
        compare(dvv, rv, torch.bfloat16, "dv")
