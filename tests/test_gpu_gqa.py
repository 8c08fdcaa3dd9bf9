"""GPU parity for grouped key/value heads (grouped-query and multi-query
attention): the forward, the backward (dK, dV summed over each group) and
the decode step through the C ABI against the fp64 oracle's grouped
functions, which are pinned on the CPU (tests/test_oracle_pins.py)."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_transformers_b200 import api, inputs
from parity_util import check_state, compare

pytestmark = pytest.mark.gpu

PHIS = {"elu1": oracle.PHI_ELU1, "relu_eps": oracle.PHI_RELU_EPS}
GROUPS = [(4, 2), (6, 3), (8, 1)]


def gqa(B, H, Hkv, N, D, dtype, seed, dO=False):
    return [t.cuda() for t in inputs.make_gqa_tensors(B, H, Hkv, N, D, dtype, seed,
                                                      with_grad_out=dO)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("N", [129, 777])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("H,Hkv", GROUPS)
def test_gqa_forward(dtype, D, N, causal, H, Hkv):
    q, k, v = gqa(2, H, Hkv, N, D, dtype, seed=N + D + H)
    o, S, z = api.la_forward(q, k, v, causal, "elu1", return_state=True)
    torch.cuda.synchronize()
    api.la_get_device_error()
    o_ref, S_ref, z_ref = oracle.forward_gqa(q, k, v, causal, oracle.PHI_ELU1)
    compare(o, o_ref, dtype, "o")
    check_state(S, z, S_ref, z_ref, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("N", [129, 777])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
@pytest.mark.parametrize("H,Hkv", GROUPS)
@pytest.mark.parametrize("saved", [False, True])
def test_gqa_backward(dtype, D, N, causal, phi, H, Hkv, saved):
    q, k, v, dO = gqa(2, H, Hkv, N, D, dtype, seed=N + 3 * D + H, dO=True)
    if saved:
        g = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
        o = api.la_forward(q, k, v, causal, phi, g=g)
        dq, dk, dv = api.la_backward(q, k, v, dO, causal, phi, o=o, g=g)
    else:
        dq, dk, dv = api.la_backward(q, k, v, dO, causal, phi)
    torch.cuda.synchronize()
    api.la_get_device_error()
    assert dk.shape == k.shape and dv.shape == v.shape
    rq, rk, rv = oracle.backward_gqa(q, k, v, dO, causal, PHIS[phi])
    compare(dq, rq, dtype, "dq")
    compare(dk, rk, dtype, "dk")
    compare(dv, rv, dtype, "dv")


def test_gqa_with_one_group_per_head_is_the_plain_call():
    # Hkv == H takes exactly the plain path: bitwise equal results
    q, k, v, dO = gqa(2, 4, 4, 300, 64, torch.bfloat16, seed=3, dO=True)
    lib = api.load_library()
    o1 = api.la_forward(q, k, v, True)
    o2 = torch.empty_like(q)
    ws = torch.empty(max(256, api.la_workspace_size(api.LA_OP_FORWARD, 2, 4, 300, 64, True,
                                                    q.dtype)), dtype=torch.uint8, device="cuda")
    st = lib.la_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), None, None, None,
                        None, None, 2, 4, 300, 64, api.LA_BF16, 1, 0, ws.data_ptr(), ws.numel(),
                        torch.cuda.current_stream().cuda_stream)
    assert st == api.LA_OK
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [16, 64, 128])
@pytest.mark.parametrize("H,Hkv", [(4, 2), (8, 1), (32, 8)])
def test_gqa_decode_matches_oracle(dtype, D, H, Hkv):
    B, T0, T1 = 3, 40, 6
    q, k, v = gqa(B, H, Hkv, T0 + T1, D, dtype, seed=D + H)
    # prefill with the grouped forward, then decode
    o0, S, z = api.la_forward(q[:, :, :T0].contiguous(), k[:, :, :T0].contiguous(),
                              v[:, :, :T0].contiguous(), True, return_state=True)
    o_ref, _, _ = oracle.forward_gqa(q, k, v, True, oracle.PHI_ELU1)
    compare(o0, o_ref[:, :, :T0], dtype, "prefill")
    for t in range(T0, T0 + T1):
        o_t = api.la_decode_step(S, z, q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                 v[:, :, t].contiguous())
        compare(o_t, o_ref[:, :, t], dtype, f"decode step {t}")
    _, S_ref, z_ref = oracle.forward_gqa(q, k, v, True, oracle.PHI_ELU1)
    check_state(S, z, S_ref, z_ref, torch.float32 if dtype == torch.float32 else dtype)


def test_gqa_decode_full_size_sampled_heads():
    cfg = inputs.DECODE_GQA
    B, H, Hkv, D, steps = cfg["B"], cfg["H"], cfg["Hkv"], cfg["D"], cfg["steps"]
    q, k, v = inputs.make_decode_gqa_inputs(B, H, Hkv, D, steps, cfg["seed"], device="cuda")
    S = torch.zeros(B, Hkv, D, D, device="cuda")
    z = torch.zeros(B, Hkv, D, device="cuda")
    outs = torch.empty(steps, B, H, D, dtype=q.dtype, device="cuda")
    for t in range(steps):
        api.la_decode_step(S, z, q[t], k[t], v[t], o=outs[t])
    torch.cuda.synchronize()
    api.la_get_device_error()
    G = H // Hkv
    for (b, hk) in [(0, 0), (B // 2, Hkv // 2), (B - 1, Hkv - 1)]:
        heads = slice(hk * G, (hk + 1) * G)
        qs = q[:, b, heads].cpu().permute(1, 0, 2)[None]            # [1, G, T, D]
        ks = k[:, b, hk].cpu()[None, None]                          # [1, 1, T, D]
        vs = v[:, b, hk].cpu()[None, None]
        o_ref, S_ref, z_ref = oracle.forward_gqa(qs, ks, vs, True, oracle.PHI_ELU1)
        compare(outs[:, b, heads].permute(1, 0, 2), o_ref[0], q.dtype, f"decode group {(b, hk)}")
        np.testing.assert_allclose(S[b, hk].double().cpu().numpy(), S_ref[0, 0], rtol=0,
                                   atol=2e-5 * np.abs(S_ref).max())


def test_gqa_rejects_bad_groups():
    q, k, v = gqa(1, 4, 2, 16, 64, torch.bfloat16, seed=1)
    k3 = torch.zeros(1, 3, 16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        api.la_forward(q, k3, k3, True)
    pq, pk = torch.empty_like(q), torch.empty_like(q)
    with pytest.raises(api.LinearAttentionError):
        api.la_forward(q, k, v, True, phi_out=(pq, pk))
