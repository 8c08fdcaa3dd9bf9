"""GPU parity: liblinattn (through the C ABI) against the fp64 oracle.

Small cases cover every dtype, head size, mode and feature map with ragged
sequence lengths that span several 128-token chunks plus a tail; the named
workloads run at their full sizes with the oracle evaluated on sampled heads
(heads are independent, so a sampled head is checked exactly).
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_transformers_b200 import api, inputs
from parity_util import check_state, compare

pytestmark = pytest.mark.gpu

DEV = "cuda"
PHIS = {"elu1": oracle.PHI_ELU1, "relu_eps": oracle.PHI_RELU_EPS}


def small(B, H, N, D, dtype, seed, dO=False):
    return [t.to(DEV) for t in inputs.make_tensors(B, H, N, D, dtype, seed, with_grad_out=dO)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("N", [1, 129, 1000])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
def test_forward_small(dtype, D, N, causal, phi):
    q, k, v = small(2, 3, N, D, dtype, seed=N * 7 + D)
    o, S, z = api.la_forward(q, k, v, causal, phi, return_state=True)
    torch.cuda.synchronize()
    o_ref, S_ref, z_ref = oracle.forward(q, k, v, causal, PHIS[phi])
    compare(o, o_ref, dtype, "o")
    check_state(S, z, S_ref, z_ref, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("N", [1, 129, 777])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
@pytest.mark.parametrize("saved", ["none", "o_g", "o_g_phi"])
def test_backward_small(dtype, D, N, causal, phi, saved):
    q, k, v, dO = small(2, 2, N, D, dtype, seed=N * 11 + D, dO=True)
    if saved != "none":
        # the forward's output and denominators (and feature maps) handed to
        # the backward
        g = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
        if saved == "o_g_phi":
            pq, pk = torch.empty_like(q), torch.empty_like(k)
            o = api.la_forward(q, k, v, causal, phi, g=g, phi_out=(pq, pk))
            dq, dk, dv = api.la_backward(q, k, v, dO, causal, phi, o=o, g=g, phi_q=pq, phi_k=pk)
        else:
            o = api.la_forward(q, k, v, causal, phi, g=g)
            dq, dk, dv = api.la_backward(q, k, v, dO, causal, phi, o=o, g=g)
    else:
        dq, dk, dv = api.la_backward(q, k, v, dO, causal, phi)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.backward(q, k, v, dO, causal, PHIS[phi])
    compare(dq, rq, dtype, "dq")
    compare(dk, rk, dtype, "dk")
    compare(dv, rv, dtype, "dv")


@pytest.mark.parametrize("N", [1, 129, 700])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
@pytest.mark.parametrize("with_phi", [False, True])
def test_fwd_bwd_one_segment_per_head(N, phi, with_phi):
    """128 heads put one segment on each head (the timed layout), which runs
    the D = 64 kernels without a segment split; ragged N, both feature maps,
    the forward's o and g (and phi(q), phi(k)) handed to the backward, every
    head checked."""
    q, k, v, dO = small(8, 16, N, 64, torch.bfloat16, seed=N + 5, dO=True)
    g = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
    if with_phi:
        pq, pk = torch.empty_like(q), torch.empty_like(k)
        o = api.la_forward(q, k, v, True, phi, g=g, phi_out=(pq, pk))
        dq, dk, dv = api.la_backward(q, k, v, dO, True, phi, o=o, g=g, phi_q=pq, phi_k=pk)
    else:
        o = api.la_forward(q, k, v, True, phi, g=g)
        dq, dk, dv = api.la_backward(q, k, v, dO, True, phi, o=o, g=g)
    torch.cuda.synchronize()
    api.la_get_device_error()
    o_ref, _, _ = oracle.forward(q, k, v, True, PHIS[phi])
    compare(o, o_ref, torch.bfloat16, "o")
    rq, rk, rv = oracle.backward(q, k, v, dO, True, PHIS[phi])
    compare(dq, rq, torch.bfloat16, "dq")
    compare(dk, rk, torch.bfloat16, "dk")
    compare(dv, rv, torch.bfloat16, "dv")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,H", [(2, 2), (8, 16)])
def test_forward_feature_map_outputs(dtype, D, causal, B, H):
    """phi(q), phi(k) written by the forward (stored from the D = 64 causal
    kernel's own tiles, by an elementwise pass elsewhere) are the oracle's
    feature map rounded to the tensor dtype: within half an ulp of it plus
    the exponential's error."""
    N = 300
    q, k, v = small(B, H, N, D, dtype, seed=D + N)
    pq, pk = torch.empty_like(q), torch.empty_like(k)
    api.la_forward(q, k, v, causal, "elu1", phi_out=(pq, pk))
    torch.cuda.synchronize()
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
    for name, got, x in (("phi(q)", pq, q), ("phi(k)", pk, k)):
        ref = oracle.phi_map(x, oracle.PHI_ELU1)
        err = np.abs(got.double().cpu().numpy() - ref)
        assert (err <= rel * np.abs(ref) + 1e-30).all(), f"{name}: max rel {np.max(err / ref):.3e}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("causal", [True, False])
def test_forward_denominators(dtype, causal):
    # g_i = phi(q_i) . z_i, the row sums of the unnormalised weights
    q, k, v = small(2, 3, 300, 64, dtype, seed=12)
    g = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
    api.la_forward(q, k, v, causal, g=g)
    torch.cuda.synchronize()
    _, S, z = oracle.forward(q, k, v, causal)
    a = oracle.phi_map(q)
    ref = np.einsum("bhnf,bhnf->bhn", a, causal_prefix_z(k) if causal else
                    np.broadcast_to(z[:, :, None, :], a.shape))
    np.testing.assert_allclose(g.double().cpu().numpy(), ref, rtol=1e-2 if dtype ==
                               torch.bfloat16 else 2e-5)


def causal_prefix_z(k):
    return np.cumsum(oracle.phi_map(k), axis=2)


def test_unit_values_give_unit_output_on_gpu():
    q, k, _ = small(2, 4, 300, 64, torch.bfloat16, seed=5)
    v = torch.ones_like(q)
    for causal in (True, False):
        o = api.la_forward(q, k, v, causal)
        torch.cuda.synchronize()
        assert (o.float() - 1).abs().max().item() <= 2e-2


def test_autograd_wrapper_runs_library_backward():
    q, k, v, dO = small(1, 2, 130, 64, torch.bfloat16, seed=6, dO=True)
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = api.LinearAttention.apply(qq, kk, vv, True, "elu1")
    o.backward(dO)
    rq, rk, rv = oracle.backward(q, k, v, dO, True, oracle.PHI_ELU1)
    compare(qq.grad, rq, torch.bfloat16, "dq")
    compare(kk.grad, rk, torch.bfloat16, "dk")
    compare(vv.grad, rv, torch.bfloat16, "dv")


def test_bad_tensors_raise():
    q, k, v = small(1, 1, 16, 64, torch.bfloat16, seed=7)
    with pytest.raises(ValueError):
        api.la_forward(q, k, v.transpose(2, 3).contiguous().transpose(2, 3), True)
    with pytest.raises(api.LinearAttentionError):
        qq = torch.zeros(1, 1, 16, 48, dtype=torch.bfloat16, device=DEV)
        api.la_forward(qq, qq, qq, True)


def test_empty_sequence_gives_zero_state():
    q = torch.empty(2, 3, 0, 64, dtype=torch.bfloat16, device=DEV)
    o, S, z = api.la_forward(q, q, q, True, return_state=True)
    torch.cuda.synchronize()
    assert o.numel() == 0 and S.abs().max().item() == 0 and z.abs().max().item() == 0


# ------------------------------------------------------------------ decode


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_matches_oracle_and_forward_handoff(D, dtype):
    B, H, T0, T1 = 3, 5, 70, 9
    q, k, v = small(B, H, T0 + T1, D, dtype, seed=D + 100)
    # prefill T0 tokens with the forward, hand the state to the decode step
    o0, S, z = api.la_forward(q[:, :, :T0].contiguous(), k[:, :, :T0].contiguous(),
                              v[:, :, :T0].contiguous(), True, return_state=True)
    o_ref, _, _ = oracle.forward(q, k, v, True, oracle.PHI_ELU1)
    for t in range(T0, T0 + T1):
        o_t = api.la_decode_step(S, z, q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                 v[:, :, t].contiguous())
        compare(o_t, o_ref[:, :, t], dtype, f"decode step {t}")
    compare(o0, o_ref[:, :, :T0], dtype, "prefill")


def test_decode_full_size_1024_steps_sampled_heads():
    cfg = inputs.DECODE
    B, H, D, steps = cfg["B"], cfg["H"], cfg["D"], cfg["steps"]
    q, k, v = inputs.make_decode_inputs(B, H, D, steps, cfg["seed"], device=DEV)
    S = torch.zeros(B, H, D, D, device=DEV)
    z = torch.zeros(B, H, D, device=DEV)
    outs = torch.empty(steps, B, H, D, dtype=q.dtype, device=DEV)
    for t in range(steps):
        api.la_decode_step(S, z, q[t], k[t], v[t], o=outs[t])
    torch.cuda.synchronize()
    sample = [(0, 0), (B // 2, H // 3), (B - 1, H - 1)]
    for (b, h) in sample:
        qs, ks, vs = (x[:, b, h].cpu()[None, None] for x in (q, k, v))  # [1,1,T,D]
        o_ref, S_ref, z_ref = oracle.forward(qs, ks, vs, True, oracle.PHI_ELU1)
        compare(outs[:, b, h], o_ref[0, 0], q.dtype, f"decode head {(b, h)}")
        np.testing.assert_allclose(S[b, h].double().cpu().numpy(), S_ref[0, 0],
                                   rtol=0, atol=2e-5 * np.abs(S_ref).max())
        np.testing.assert_allclose(z[b, h].double().cpu().numpy(), z_ref[0, 0], rtol=2e-5)


# ------------------------------------------------------- named workloads


def sampled_heads(B, H):
    heads = {(0, 0), (B - 1, H - 1), (B // 2, H // 2)}
    return sorted(heads)


def run_workload(w, full_check: bool):
    dev_inputs = inputs.make_inputs(w, device=DEV if not full_check else "cpu")
    dev_inputs = [t.to(DEV) for t in dev_inputs]
    q, k, v = dev_inputs[:3]
    # the launch configuration the benchmark times: the forward keeps its
    # denominators and feature maps and the backward uses them with the output
    g = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
    pq, pk = torch.empty_like(q), torch.empty_like(k)
    o = api.la_forward(q, k, v, w.causal, w.phi, g=g, phi_out=(pq, pk))
    grads = None
    if w.backward:
        grads = api.la_backward(q, k, v, dev_inputs[3], w.causal, w.phi, o=o, g=g, phi_q=pq,
                                phi_k=pk)
    torch.cuda.synchronize()
    api.la_get_device_error()
    if full_check:
        o_ref, _, _ = oracle.forward(q, k, v, w.causal, w.phi)
        compare(o, o_ref, w.dtype, f"{w.name} o")
        if grads is not None:
            refs = oracle.backward(q, k, v, dev_inputs[3], w.causal, w.phi)
            for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
                compare(g, r, w.dtype, f"{w.name} {name}")
        return
    for (b, h) in sampled_heads(w.B, w.H):
        sl = lambda t: t[b:b + 1, h:h + 1].cpu()  # noqa: E731
        o_ref, _, _ = oracle.forward(sl(q), sl(k), sl(v), w.causal, w.phi)
        compare(sl(o), o_ref, w.dtype, f"{w.name} o head {(b, h)}")
        if grads is not None:
            refs = oracle.backward(sl(q), sl(k), sl(v), sl(dev_inputs[3]), w.causal, w.phi)
            for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
                compare(sl(g), r, w.dtype, f"{w.name} {name} head {(b, h)}")


@pytest.mark.parametrize("name", ["causal_fwd_b1h1n256d32_f32", "fwd_b4h8n2048d64_bf16",
                                  "ncfwd_b4h8n2048d64_bf16"])
def test_workload_full_check(name):
    run_workload(inputs.WORKLOADS[name], full_check=True)


@pytest.mark.parametrize("name", ["causal_fwdbwd_b8h16n8192d64_bf16",
                                  "causal_fwdbwd_b4h16n4096d128_relu_bf16",
                                  "causal_fwdbwd_b4h16n4096d128_elu_bf16",
                                  "causal_fwd_b1h32n131072d128_bf16"])
def test_workload_sampled_heads(name):
    run_workload(inputs.WORKLOADS[name], full_check=False)


def test_timed_workload_back_to_back_steps():
    """Twenty forward + backward steps of the timed workload back to back, as
    the benchmark runs them: no bounded device wait may give up (a pipeline
    whose hand-offs can fall two phases behind shows up here, not in a single
    call), and the last step still matches the oracle on a sampled head."""
    w = inputs.WORKLOADS["causal_fwdbwd_b8h16n8192d64_bf16"]
    q, k, v, dO = (t.to(DEV) for t in inputs.make_inputs(w, device=DEV))
    g = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
    pq, pk, o = torch.empty_like(q), torch.empty_like(k), torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    for _ in range(20):
        api.la_forward(q, k, v, True, w.phi, o=o, g=g, phi_out=(pq, pk))
        api.la_backward(q, k, v, dO, True, w.phi, dq=dq, dk=dk, dv=dv, o=o, g=g, phi_q=pq,
                        phi_k=pk)
    torch.cuda.synchronize()
    api.la_get_device_error()
    b, h = w.B - 1, w.H // 3
    sl = lambda t: t[b:b + 1, h:h + 1].cpu()  # noqa: E731
    refs = oracle.backward(sl(q), sl(k), sl(v), sl(dO), True, w.phi)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        compare(sl(got), r, w.dtype, f"step 20 {name}")


def test_quadratic_form_small_fp32():
    # the GPU forward against the oracle's quadratic form (the form the
    # associativity identity starts from), small N
    q, k, v = small(1, 2, 100, 32, torch.float32, seed=8)
    for causal in (True, False):
        o = api.la_forward(q, k, v, causal)
        compare(o, oracle.quadratic(q, k, v, causal), torch.float32, "quadratic")


def test_calls_from_another_host_thread():
    # A fresh host thread (as torch's autograd worker is) must work: the
    # library binds the current device's context before its driver calls.
    import threading
    q, k, v, dO = small(1, 2, 200, 64, torch.bfloat16, seed=9, dO=True)
    out = {}

    def worker():
        try:
            out["o"] = api.la_forward(q, k, v, True)
            out["g"] = api.la_backward(q, k, v, dO, True)
            torch.cuda.synchronize()
        except Exception as e:  # surfaced below
            out["err"] = e

    t = threading.Thread(target=worker)
    t.start()
    t.join()
    assert "err" not in out, out.get("err")
    rq, rk, rv = oracle.backward(q, k, v, dO, True, oracle.PHI_ELU1)
    compare(out["o"], oracle.forward(q, k, v, True, oracle.PHI_ELU1)[0], torch.bfloat16, "o")
    for name, g, r in zip(("dq", "dk", "dv"), out["g"], (rq, rk, rv)):
        compare(g, r, torch.bfloat16, name)
