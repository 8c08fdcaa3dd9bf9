"""Pins for the fp64 CPU oracle, independent of the oracle's own formulas.

Each test ties the oracle to something the linear-attention pages or plain
mathematics fix, chosen so that a plausible slip (a dropped term, a wrong
index or sign, a transposed state, an exclusive instead of inclusive prefix,
the wrong feature-map branch) fails at least one of them:

- the recurrence equals the quadratic, row-normalised form (the
  associativity identity of "Efficient Transformers Survey", Proposition
  "Linear Attention via Kernel Decomposition", Intuition and Proof Sketch);
- the feature map matches torch's library elu / relu;
- closed forms: D = 1 reduces attention to a phi(k)-weighted mean of v;
  identical keys reduce it to a plain prefix (or global) mean of v;
- invariants: V = 1 gives O = 1; N = 1 gives o = v; the first causal output
  is v_1; causal outputs ignore later tokens; non-causal outputs ignore the
  order of (k, v) pairs;
- the token-by-token decode recurrence ("Why It Matters": update S and z
  incrementally) reproduces the causal forward and its final state;
- S is D x D and z has D entries (section Exercises, ExerciseCore);
- the backward matches central finite differences of L = sum(dO * O), and
  satisfies the homogeneity / linearity identities of the definition;
- grouped key/value heads: finite differences through the shared k, v;
  multi-query heads are independent single-head attentions; the grouped
  decode continues the grouped forward;
- decayed (gated) recurrence: gamma = 1 is the causal oracle; recurrence ==
  decayed quadratic form; gamma = 0 returns v; identical keys give the
  bias-corrected exponential moving average of v; the final state is the
  gamma^(N-1-j)-weighted sum; finite differences; decode continues it;
- Performer FAVOR+ features: phi(q).phi(k) is an unbiased estimate of
  exp(q.k) (a large Monte Carlo sample within 5 standard errors); x = 0 and
  a zero direction give closed forms; the feature backward matches finite
  differences; with many features the attention approaches softmax
  attention; the identity map is the quadratic form of the given features
  and its backward matches finite differences.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import PHI_ELU1, PHI_RELU_EPS


def rnd(shape, seed, scale=1.0, away_from_zero=False):
    g = np.random.default_rng(seed)
    x = g.standard_normal(shape) * scale
    if away_from_zero:
        # keep the ReLU map differentiable for finite differences
        x = np.where(np.abs(x) < 1e-2, np.sign(x + 1e-300) * (1e-2 + np.abs(x)), x)
    return x


SHAPES = [(1, 1, 1, 4), (1, 2, 7, 3), (2, 1, 16, 8), (1, 1, 33, 16)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("phi", [PHI_ELU1, PHI_RELU_EPS])
def test_recurrence_equals_quadratic_form(shape, causal, phi):
    q, k, v = (rnd(shape, s) for s in (1, 2, 3))
    o_lin, _, _ = oracle.forward(q, k, v, causal, phi)
    o_quad = oracle.quadratic(q, k, v, causal, phi)
    np.testing.assert_allclose(o_lin, o_quad, rtol=1e-12, atol=1e-12)


def test_feature_map_matches_library():
    x = torch.linspace(-6, 6, 1001, dtype=torch.float64)
    elu1 = torch.nn.functional.elu(x, alpha=1.0) + 1.0
    relu = torch.relu(x) + 1e-6
    np.testing.assert_allclose(oracle.phi_map(x, PHI_ELU1), elu1.numpy(), rtol=1e-13, atol=0)
    np.testing.assert_allclose(oracle.phi_map(x, PHI_RELU_EPS), relu.numpy(), rtol=1e-13, atol=0)
    # slope of elu+1: 1 for x > 0, exp(x) for x <= 0 (autograd of the library map)
    xg = x.clone().requires_grad_(True)
    (torch.nn.functional.elu(xg) + 1.0).sum().backward()
    np.testing.assert_allclose(oracle.dphi_map(x, PHI_ELU1), xg.grad.numpy(), rtol=1e-13)


@pytest.mark.parametrize("phi", [PHI_ELU1, PHI_RELU_EPS])
@pytest.mark.parametrize("causal", [True, False])
def test_d1_is_phi_weighted_mean(phi, causal):
    # D = 1: o_i = sum_j phi(k_j) v_j / sum_j phi(k_j); the query cancels.
    N = 9
    q, k, v = (rnd((1, 1, N, 1), s) for s in (4, 5, 6))
    kt = torch.from_numpy(k[0, 0, :, 0])
    w = (torch.nn.functional.elu(kt) + 1.0) if phi == PHI_ELU1 else (torch.relu(kt) + 1e-6)
    w = w.numpy()
    vv = v[0, 0, :, 0]
    if causal:
        expect = np.cumsum(w * vv) / np.cumsum(w)
    else:
        expect = np.full(N, (w * vv).sum() / w.sum())
    o, _, _ = oracle.forward(q, k, v, causal, phi)
    np.testing.assert_allclose(o[0, 0, :, 0], expect, rtol=1e-13, atol=1e-15)
    o2 = oracle.quadratic(q, k, v, causal, phi)
    np.testing.assert_allclose(o2[0, 0, :, 0], expect, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("causal", [True, False])
def test_identical_keys_give_mean_of_values(causal):
    B, H, N, D = 1, 2, 11, 5
    q = rnd((B, H, N, D), 7)
    v = rnd((B, H, N, D), 8)
    k = np.broadcast_to(rnd((B, H, 1, D), 9), (B, H, N, D)).copy()
    o, _, _ = oracle.forward(q, k, v, causal, PHI_ELU1)
    if causal:
        expect = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    else:
        expect = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
    np.testing.assert_allclose(o, expect, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("phi", [PHI_ELU1, PHI_RELU_EPS])
def test_unit_values_give_unit_output(causal, phi):
    shape = (2, 2, 13, 6)
    q, k = rnd(shape, 10), rnd(shape, 11)
    v = np.ones(shape)
    o, _, _ = oracle.forward(q, k, v, causal, phi)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


def test_single_token_and_first_causal_output():
    q, k, v = (rnd((2, 3, 1, 8), s) for s in (12, 13, 14))
    for causal in (True, False):
        o, _, _ = oracle.forward(q, k, v, causal, PHI_ELU1)
        np.testing.assert_allclose(o, v, rtol=1e-14, atol=1e-15)
    q, k, v = (rnd((1, 2, 10, 8), s) for s in (15, 16, 17))
    o, _, _ = oracle.forward(q, k, v, True, PHI_ELU1)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=1e-14, atol=1e-15)


def test_causal_output_ignores_later_tokens():
    shape = (1, 1, 20, 6)
    q, k, v = (rnd(shape, s) for s in (18, 19, 20))
    o, _, _ = oracle.forward(q, k, v, True, PHI_ELU1)
    cut = 8
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, :, cut:] += 3.0
    k2[:, :, cut:] -= 2.0
    v2[:, :, cut:] *= -5.0
    o2, _, _ = oracle.forward(q2, k2, v2, True, PHI_ELU1)
    np.testing.assert_array_equal(o[:, :, :cut], o2[:, :, :cut])
    assert np.abs(o[:, :, cut:] - o2[:, :, cut:]).max() > 1e-3


def test_noncausal_ignores_key_order():
    shape = (1, 2, 15, 4)
    q, k, v = (rnd(shape, s) for s in (21, 22, 23))
    perm = np.random.default_rng(24).permutation(shape[2])
    o, _, _ = oracle.forward(q, k, v, False, PHI_ELU1)
    o2, _, _ = oracle.forward(q, k[:, :, perm], v[:, :, perm], False, PHI_ELU1)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-14)


def test_state_shapes_and_final_state():
    B, H, N, D = 2, 3, 9, 5
    q, k, v = (rnd((B, H, N, D), s) for s in (25, 26, 27))
    for causal in (True, False):
        _, S, z = oracle.forward(q, k, v, causal, PHI_ELU1)
        assert S.shape == (B, H, D, D) and z.shape == (B, H, D)
        # a single extra decode step with v = 1 column: S, z equal the quadratic
        # row sums on the last query (both modes end with the full prefix)
        o_last = oracle.quadratic(q, k, v, True, PHI_ELU1)[:, :, -1]
        a = oracle.phi_map(q[:, :, -1])
        num = np.einsum("bhf,bhfe->bhe", a, S)
        den = np.einsum("bhf,bhf->bh", a, z)
        np.testing.assert_allclose(num / den[..., None], o_last, rtol=1e-12)


@pytest.mark.parametrize("phi", [PHI_ELU1, PHI_RELU_EPS])
def test_decode_recurrence_equals_causal_forward(phi):
    B, H, T, D = 2, 2, 17, 6
    q, k, v = (rnd((B, H, T, D), s) for s in (28, 29, 30))
    o_ref, S_ref, z_ref = oracle.forward(q, k, v, True, phi)
    S = np.zeros((B, H, D, D))
    z = np.zeros((B, H, D))
    for t in range(T):
        o_t = oracle.decode_step(S, z, q[:, :, t], k[:, :, t], v[:, :, t], phi)
        np.testing.assert_allclose(o_t, o_ref[:, :, t], rtol=1e-12, atol=1e-14)
        if t == 0:
            np.testing.assert_allclose(o_t, v[:, :, 0], rtol=1e-14)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(z, z_ref, rtol=1e-12)


# ---------------------------------------------------------------- backward


def fd_grads(q, k, v, dO, causal, phi, h=1e-6):
    """Central differences of L = sum(dO * O) with the (pinned) forward."""
    def loss(qq, kk, vv):
        o, _, _ = oracle.forward(qq, kk, vv, causal, phi)
        return float((o * dO).sum())

    out = []
    for which in range(3):
        base = [q, k, v]
        g = np.zeros_like(base[which])
        it = np.nditer(base[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        out.append(g)
    return out


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("phi", [PHI_ELU1, PHI_RELU_EPS])
@pytest.mark.parametrize("shape", [(1, 1, 1, 3), (1, 1, 6, 4), (1, 2, 11, 5)])
def test_backward_matches_finite_differences(causal, phi, shape):
    relu = phi == PHI_RELU_EPS
    q = rnd(shape, 31, away_from_zero=relu)
    k = rnd(shape, 32, away_from_zero=relu)
    v = rnd(shape, 33)
    dO = rnd(shape, 34)
    dq, dk, dv = oracle.backward(q, k, v, dO, causal, phi)
    for got, ref in zip((dq, dk, dv), fd_grads(q, k, v, dO, causal, phi)):
        scale = max(np.abs(ref).max(), 1e-3)
        assert np.abs(got - ref).max() <= 1e-6 * scale + 1e-9, (np.abs(got - ref).max(), scale)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_identities(causal):
    shape = (2, 2, 14, 6)
    q, k, v, dO = (rnd(shape, s) for s in (35, 36, 37, 38))
    phi = PHI_ELU1
    dq, dk, dv = oracle.backward(q, k, v, dO, causal, phi)
    o, _, _ = oracle.forward(q, k, v, causal, phi)
    # O is linear in V: sum <dV, V> = sum <dO, O>
    np.testing.assert_allclose((dv * v).sum(), (dO * o).sum(), rtol=1e-11)
    # o_i is homogeneous of degree 0 in a_i: <dA_i, a_i> = 0 per query
    A = oracle.phi_map(q)
    dA = dq / oracle.dphi_map(q)
    per_i = (dA * A).sum(-1)
    assert np.abs(per_i).max() < 1e-11 * max(1.0, np.abs(dA * A).max())
    # scaling every phi(k) by one constant leaves O unchanged: sum_j <dB_j, b_j> = 0
    Bm = oracle.phi_map(k)
    dB = dk / oracle.dphi_map(k)
    per_head = (dB * Bm).sum(axis=(-1, -2))
    assert np.abs(per_head).max() < 1e-10 * max(1.0, np.abs(dB * Bm).max())
    # V = 1 makes O = 1 whatever Q and K are: dQ = dK = 0
    dq1, dk1, _ = oracle.backward(q, k, np.ones(shape), dO, causal, phi)
    assert np.abs(dq1).max() < 1e-12 and np.abs(dk1).max() < 1e-12


def test_backward_d1_has_no_query_gradient():
    q, k, v, dO = (rnd((1, 1, 10, 1), s) for s in (39, 40, 41, 42))
    for causal in (True, False):
        dq, _, _ = oracle.backward(q, k, v, dO, causal, PHI_ELU1)
        assert np.abs(dq).max() < 1e-13


# ---------------------------------------------------- grouped key/value heads

def _gqa_inputs(B, H, Hkv, N, D, seed):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, H, N, D)) * 0.5
    k = g.standard_normal((B, Hkv, N, D)) * 0.5
    v = g.standard_normal((B, Hkv, N, D))
    dO = g.standard_normal((B, H, N, D))
    return q, k, v, dO


@pytest.mark.parametrize("causal", [True, False])
def test_gqa_backward_matches_finite_differences(causal):
    # the gradient with respect to a k or v shared by a group is checked
    # against central differences of sum(dO * O) through the grouped forward
    B, H, Hkv, N, D = 1, 4, 2, 6, 3
    q, k, v, dO = _gqa_inputs(B, H, Hkv, N, D, 41)
    dq, dk, dv = oracle.backward_gqa(q, k, v, dO, causal, oracle.PHI_ELU1)
    loss = lambda q_, k_, v_: float((dO * oracle.forward_gqa(q_, k_, v_, causal)[0]).sum())  # noqa
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_mqa_heads_are_independent_single_head_attentions():
    # one key/value head shared by all query heads: each query head's output
    # is the single-head attention of that query against the shared k, v
    B, H, N, D = 2, 3, 9, 4
    q, k, v, _ = _gqa_inputs(B, H, 1, N, D, 42)
    o, S, z = oracle.forward_gqa(q, k, v, True)
    for h in range(H):
        o1, S1, z1 = oracle.forward(q[:, h:h + 1], k, v, True)
        np.testing.assert_allclose(o[:, h:h + 1], o1, rtol=1e-13, atol=0)
    np.testing.assert_allclose(S, S1, rtol=1e-13)
    np.testing.assert_allclose(z, z1, rtol=1e-13)
    # the quadratic form with the shared k, v gives the same outputs
    qd = oracle.quadratic(q, np.repeat(k, H, 1), np.repeat(v, H, 1), True)
    np.testing.assert_allclose(o, qd, rtol=1e-12)


def test_gqa_decode_continues_the_grouped_forward():
    B, H, Hkv, T, D = 2, 4, 2, 7, 3
    q, k, v, _ = _gqa_inputs(B, H, Hkv, T, D, 43)
    o_ref, S_ref, z_ref = oracle.forward_gqa(q, k, v, True)
    S = np.zeros((B, Hkv, D, D))
    z = np.zeros((B, Hkv, D))
    for t in range(T):
        o = oracle.decode_step_gqa(S, z, q[:, :, t], k[:, :, t], v[:, :, t])
        np.testing.assert_allclose(o, o_ref[:, :, t], rtol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12)
    np.testing.assert_allclose(z, z_ref, rtol=1e-12)


# ------------------------------------------------------- decayed (gated) LA
# S_i = gamma S_{i-1} + b_i v_i^T, z_i = gamma z_{i-1} + b_i, one gamma per
# head ("Efficient Transformers Survey", Common Confusions, "Watch Out": the
# gating and decay factors linear-attention models add).

def test_decay_one_is_the_causal_oracle():
    q, k, v, dO = (rnd((2, 3, 37, 8), 300 + i, 0.5) for i in range(4))
    g = np.ones(3)
    o1, S1, z1 = oracle.forward_decay(q, k, v, g)
    o0, S0, z0 = oracle.forward(q, k, v, True)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(S1, S0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(z1, z0, rtol=0, atol=1e-12)
    for a, b in zip(oracle.backward_decay(q, k, v, dO, g), oracle.backward(q, k, v, dO, True)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("phi", [PHI_ELU1, PHI_RELU_EPS])
def test_decay_recurrence_equals_decayed_quadratic_form(phi):
    q, k, v = (rnd((2, 4, 41, 8), 310 + i, 0.6) for i in range(3))
    g = np.array([0.0, 0.35, 0.9, 0.999])
    o, _, _ = oracle.forward_decay(q, k, v, g, phi)
    np.testing.assert_allclose(o, oracle.quadratic_decay(q, k, v, g, phi), rtol=1e-11, atol=1e-13)


def test_decay_zero_returns_the_values():
    # gamma = 0 keeps only j = i: o_i = (a_i . b_i) v_i / (a_i . b_i) = v_i.
    # A normaliser z left undecayed would give a different answer.
    q, k, v = (rnd((1, 2, 23, 8), 320 + i) for i in range(3))
    o, S, z = oracle.forward_decay(q, k, v, np.zeros(2))
    np.testing.assert_allclose(o, v, rtol=1e-13, atol=1e-14)
    # the final state is the last token's b v^T alone
    b = oracle.phi_map(k[:, :, -1])
    np.testing.assert_allclose(S, b[..., :, None] * v[:, :, -1][..., None, :], rtol=1e-13)


@pytest.mark.parametrize("gamma", [0.5, 0.9])
def test_decay_identical_keys_is_the_bias_corrected_moving_average(gamma):
    # Identical keys: a_i . b_j = c_i for all j <= i, so o_i is the
    # exponentially weighted average sum_j gamma^(i-j) v_j over the
    # geometric sum (1 - gamma^(i+1)) / (1 - gamma), the recursion
    # m_i = gamma m_{i-1} + (1 - gamma) v_i divided by 1 - gamma^(i+1).
    N, D = 30, 4
    q = rnd((1, 1, N, D), 330)
    k = np.broadcast_to(rnd((1, 1, 1, D), 331), (1, 1, N, D)).copy()
    v = rnd((1, 1, N, D), 332)
    o, _, _ = oracle.forward_decay(q, k, v, np.array([gamma]))
    m = np.zeros(D)
    for i in range(N):
        m = gamma * m + (1.0 - gamma) * v[0, 0, i]
        np.testing.assert_allclose(o[0, 0, i], m / (1.0 - gamma ** (i + 1)), rtol=1e-12,
                                   atol=1e-13)


def test_decay_final_state_is_the_weighted_sum():
    N, D, gamma = 19, 5, 0.8
    q, k, v = (rnd((1, 1, N, D), 340 + i) for i in range(3))
    _, S, z = oracle.forward_decay(q, k, v, np.array([gamma]))
    b = oracle.phi_map(k)[0, 0]
    w = gamma ** (N - 1 - np.arange(N))
    np.testing.assert_allclose(S[0, 0], (b * w[:, None]).T @ v[0, 0], rtol=1e-12)
    np.testing.assert_allclose(z[0, 0], (b * w[:, None]).sum(0), rtol=1e-12)


def _fd_decay(q, k, v, dO, gamma, phi, h=1e-6):
    def loss(q_, k_, v_):
        return float((oracle.forward_decay(q_, k_, v_, gamma, phi)[0] * dO).sum())
    grads = []
    for which in range(3):
        args = [q, k, v]
        g = np.zeros_like(args[which])
        it = np.nditer(g, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("phi", [PHI_ELU1, PHI_RELU_EPS])
def test_decay_backward_matches_finite_differences(phi):
    q, k, v, dO = (rnd((1, 2, 7, 3), 350 + i, 0.7, away_from_zero=True) for i in range(4))
    gamma = np.array([0.6, 0.95])
    got = oracle.backward_decay(q, k, v, dO, gamma, phi)
    ref = _fd_decay(q, k, v, dO, gamma, phi)
    for name, a, b in zip("qkv", got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-8, err_msg=f"d{name}")


def test_decay_decode_continues_the_decayed_forward():
    B, H, N, D, T0 = 2, 3, 25, 8, 17
    q, k, v = (rnd((B, H, N, D), 360 + i, 0.5) for i in range(3))
    gamma = np.array([0.2, 0.7, 1.0])
    o, S_ref, z_ref = oracle.forward_decay(q, k, v, gamma)
    _, S, z = oracle.forward_decay(q[:, :, :T0], k[:, :, :T0], v[:, :, :T0], gamma)
    for t in range(T0, N):
        o_t = oracle.decode_step_decay(S, z, q[:, :, t], k[:, :, t], v[:, :, t], gamma)
        np.testing.assert_allclose(o_t, o[:, :, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12)
    np.testing.assert_allclose(z, z_ref, rtol=1e-12)


def test_decay_rejects_out_of_range_factors():
    q = rnd((1, 2, 3, 4), 370)
    with pytest.raises(ValueError):
        oracle.forward_decay(q, q, q, np.array([0.5, 1.5]))
    with pytest.raises(ValueError):
        oracle.forward_decay(q, q, q, np.array([0.5]))


# ------------------------------------------------ Performer FAVOR+ features
# "Efficient Transformers Survey", Low-Rank Approximations, Performer, and
# Proposition "Performer Approximation Quality".

def test_favor_features_are_an_unbiased_estimate_of_the_exp_kernel():
    # E[phi(q)^T phi(k)] = exp(q^T k): the sample mean over m draws sits
    # within a few standard errors of the closed form
    g = np.random.default_rng(400)
    D, m = 8, 200000
    q, k = g.standard_normal(D) * 0.3, g.standard_normal(D) * 0.3
    w = g.standard_normal((m, D))
    pq, pk = oracle.favor_features(q, w), oracle.favor_features(k, w)
    est = float(pq @ pk)
    samples = m * pq * pk                      # the m terms whose mean is est
    se = samples.std() / np.sqrt(m)
    assert abs(est - np.exp(q @ k)) < 5 * se, (est, np.exp(q @ k), se)


def test_favor_features_closed_forms():
    g = np.random.default_rng(401)
    w = g.standard_normal((16, 4))
    # x = 0: every feature is m^-1/2
    np.testing.assert_allclose(oracle.favor_features(np.zeros(4), w), np.full(16, 0.25),
                               rtol=1e-15)
    # a zero direction gives exp(-|x|^2/2) / sqrt(m); features are positive
    x = g.standard_normal(4)
    w0 = np.vstack([np.zeros(4), w])
    f = oracle.favor_features(x, w0)
    np.testing.assert_allclose(f[0], np.exp(-0.5 * x @ x) / np.sqrt(17), rtol=1e-14)
    assert (f > 0).all()


def test_favor_features_backward_matches_finite_differences():
    g = np.random.default_rng(402)
    x, w, dphi = g.standard_normal((3, 5)) * 0.5, g.standard_normal((7, 5)), g.standard_normal((3, 7))
    got = oracle.favor_features_backward(x, w, dphi)
    h = 1e-6
    ref = np.zeros_like(x)
    for i in range(x.shape[0]):
        for j in range(x.shape[1]):
            xp, xm = x.copy(), x.copy()
            xp[i, j] += h
            xm[i, j] -= h
            ref[i, j] = ((oracle.favor_features(xp, w) - oracle.favor_features(xm, w)) * dphi).sum() / (2 * h)
    np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-9)


def test_identity_map_is_the_quadratic_form_of_the_given_features():
    g = np.random.default_rng(403)
    a, b = np.exp(g.standard_normal((1, 2, 9, 4))), np.exp(g.standard_normal((1, 2, 9, 4)))
    v = g.standard_normal((1, 2, 9, 4))
    for causal in (True, False):
        o, _, _ = oracle.forward(a, b, v, causal, oracle.PHI_IDENTITY)
        w = np.einsum("bhid,bhjd->bhij", a, b)
        if causal:
            w = np.tril(w)
        ref = np.einsum("bhij,bhje->bhie", w, v) / w.sum(-1, keepdims=True)
        np.testing.assert_allclose(o, ref, rtol=1e-12)


def test_performer_attention_approaches_softmax_attention():
    # with many features, linear attention on phi(q), phi(k) reproduces
    # softmax attention with weights exp(q_i^T k_j) (here x = q / d^(1/4)
    # is already applied: the inputs are the pre-normalised q, k)
    g = np.random.default_rng(404)
    N, D, m = 12, 4, 100000
    q, k, v = (g.standard_normal((1, 1, N, D)) * 0.4 for _ in range(3))
    w = g.standard_normal((m, D))
    pq, pk = oracle.favor_features(q, w), oracle.favor_features(k, w)
    # the core with m-dimensional features: the identity map's quadratic form
    wts = np.tril(np.einsum("bhim,bhjm->bhij", pq, pk))
    o_perf = np.einsum("bhij,bhje->bhie", wts, v) / wts.sum(-1, keepdims=True)
    sm = np.tril(np.exp(np.einsum("bhid,bhjd->bhij", q, k)))
    o_soft = np.einsum("bhij,bhje->bhie", sm, v) / sm.sum(-1, keepdims=True)
    assert np.abs(o_perf - o_soft).max() < 0.02 * np.abs(o_soft).max()


def test_identity_map_backward_matches_finite_differences():
    g = np.random.default_rng(405)
    shape = (1, 1, 6, 3)
    q, k = np.exp(g.standard_normal(shape) * 0.5), np.exp(g.standard_normal(shape) * 0.5)
    v, dO = g.standard_normal(shape), g.standard_normal(shape)
    got = oracle.backward(q, k, v, dO, True, oracle.PHI_IDENTITY)
    ref = fd_grads(q, k, v, dO, True, oracle.PHI_IDENTITY)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-9)


@pytest.mark.parametrize("dk,dv,phi", [(6, 3, PHI_ELU1), (6, 3, oracle.PHI_IDENTITY),
                                       (3, 6, oracle.PHI_IDENTITY)])
@pytest.mark.parametrize("causal", [True, False])
def test_mv_forward_is_the_quadratic_form_with_features_and_values_of_two_lengths(dk, dv, phi,
                                                                                 causal):
    # S = sum_j phi(k_j) v_j^T is dk x dv: the quadratic form of the
    # Proposition with A [N, dk], B [N, dk] and V [N, dv], written directly
    g = np.random.default_rng(406 + dk)
    N = 11
    if phi == oracle.PHI_IDENTITY:
        q, k = np.exp(g.standard_normal((2, 1, N, dk)) * 0.5), np.exp(g.standard_normal((2, 1, N, dk)) * 0.5)
        a, b = q, k
    else:
        q, k = g.standard_normal((2, 1, N, dk)), g.standard_normal((2, 1, N, dk))
        a, b = oracle.phi_map(q, phi), oracle.phi_map(k, phi)
    v = g.standard_normal((2, 1, N, dv))
    w = np.einsum("bhid,bhjd->bhij", a, b)
    if causal:
        w = np.tril(w)
    ref = np.einsum("bhij,bhje->bhie", w, v) / w.sum(-1, keepdims=True)
    o = oracle.forward_mv(q, k, v, causal, phi)
    assert o.shape == (2, 1, N, dv)
    np.testing.assert_allclose(o, ref, rtol=1e-12)


def test_mv_refuses_zero_features_under_a_feature_map():
    x = np.ones((1, 1, 2, 3))
    with pytest.raises(ValueError):
        oracle.forward_mv(x, x, np.ones((1, 1, 2, 6)), True, PHI_ELU1)


@pytest.mark.parametrize("dk,dv", [(5, 3), (3, 5)])
def test_mv_backward_matches_finite_differences(dk, dv):
    g = np.random.default_rng(407 + dk)
    N, h = 7, 1e-6
    q = np.exp(g.standard_normal((1, 1, N, dk)) * 0.5)
    k = np.exp(g.standard_normal((1, 1, N, dk)) * 0.5)
    v, dO = g.standard_normal((1, 1, N, dv)), g.standard_normal((1, 1, N, dv))
    got = oracle.backward_mv(q, k, v, dO, True, oracle.PHI_IDENTITY)
    loss = lambda qq, kk, vv: float((dO * oracle.forward_mv(qq, kk, vv, True)).sum())  # noqa: E731
    for idx, x in enumerate((q, k, v)):
        fd = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[pos] += h
            xm[pos] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[idx], args_m[idx] = xp, xm
            fd[pos] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(got[idx], fd, rtol=1e-6, atol=1e-9)
