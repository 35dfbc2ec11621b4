"""Pins for the fp64 oracle, checked against facts that do not come from the oracle itself.

* alpha == 1 reduces GLA to causal linear attention, (Q K^T . M) V ("Gated Linear Attention
  for Efficient Long Sequences": GLA sits between linear attention and RetNet decay; the
  reference list names "Transformers are RNNs").
* a constant scalar gate reduces it to RetNet's closed-form decay mask gamma^(t-s).
* for any gate the recurrence unrolls to a double sum with exp(b_t - b_s) factors, computed
  here by brute-force loops.
* the backward pass agrees with central finite differences, with linear attention's closed
  form gradients, and with the cumulative-sum identity for the gate gradient.
* the chunked form equals the recurrence for every chunk size ("MS-GLA", section 2.1).
* decode steps continue the parallel form (recurrent inference).
* GSA reduces to known forms for alpha == 1 and for a single slot (m = 1, softmax == 1).
* a few plausible mistakes planted in copies of the recurrence fail these pins.
"""
import math

import numpy as np
import pytest

import oracle as O


def _rand_inputs(rng, B=1, H=2, T=9, dk=3, dv=4, gate="random", h0=True):
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    if gate == "random":
        g = -np.log1p(np.exp(rng.standard_normal((B, H, T, dk))))  # logsigmoid(-x) < 0
    elif gate == "zero":
        g = np.zeros((B, H, T, dk))
    else:
        g = np.full((B, H, T, dk), float(gate))
    s0 = rng.standard_normal((B, H, dk, dv)) if h0 else None
    return q, k, v, g, s0


def _brute_gla(q, k, v, g, h0):
    """o_t = sum_{s<=t} sum_d q_td k_sd exp(b_td - b_sd) v_s + sum_d q_td exp(b_td) h0_d."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    b = np.cumsum(g, axis=2)
    o = np.zeros((B, H, T, dv))
    hT = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for hh in range(H):
            for t in range(T):
                for s in range(t + 1):
                    for d in range(dk):
                        o[bb, hh, t] += q[bb, hh, t, d] * k[bb, hh, s, d] * np.exp(
                            b[bb, hh, t, d] - b[bb, hh, s, d]) * v[bb, hh, s]
                if h0 is not None:
                    for d in range(dk):
                        o[bb, hh, t] += q[bb, hh, t, d] * np.exp(b[bb, hh, t, d]) * h0[bb, hh, d]
            for s in range(T):
                for d in range(dk):
                    hT[bb, hh, d] += np.exp(b[bb, hh, T - 1, d] - b[bb, hh, s, d]) * k[bb, hh, s, d] * v[bb, hh, s]
            if h0 is not None:
                hT[bb, hh] += np.exp(b[bb, hh, T - 1])[:, None] * h0[bb, hh]
    return o, hT


# ---------------------------------------------------------------------------------------
# forward pins
# ---------------------------------------------------------------------------------------
def test_alpha_one_is_causal_linear_attention(rng):
    q, k, v, g, h0 = _rand_inputs(rng, T=11, gate="zero")
    o, hT = O.gla_fwd(q, k, v, g, h0)
    M = np.tril(np.ones((11, 11)))
    ref = (q @ np.swapaxes(k, -1, -2) * M) @ v + q @ h0
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT, h0 + np.swapaxes(k, -1, -2) @ v, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("gamma", [0.9, 0.5, 0.99])
def test_constant_gate_is_retnet_decay_mask(rng, gamma):
    T = 10
    q, k, v, g, h0 = _rand_inputs(rng, T=T, gate=np.log(gamma))
    o, hT = O.gla_fwd(q, k, v, g, h0)
    t = np.arange(T)
    Dm = np.where(t[:, None] >= t[None, :], gamma ** (t[:, None] - t[None, :]).clip(0), 0.0)
    ref = (q @ np.swapaxes(k, -1, -2) * Dm) @ v + (gamma ** (t + 1))[:, None] * (q @ h0)
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-11)
    w = gamma ** (T - 1 - t)
    ref_hT = np.einsum("s,bhsi,bhsj->bhij", w, k, v) + gamma ** T * h0
    np.testing.assert_allclose(hT, ref_hT, rtol=1e-11, atol=1e-11)


def test_general_gate_matches_bruteforce_unrolled_sum(rng):
    q, k, v, g, h0 = _rand_inputs(rng, B=2, H=1, T=7, dk=3, dv=2)
    o, hT = O.gla_fwd(q, k, v, g, h0)
    bo, bhT = _brute_gla(q, k, v, g, h0)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT, bhT, rtol=1e-12, atol=1e-12)


def test_h0_superposition(rng):
    q, k, v, g, h0 = _rand_inputs(rng, T=13)
    o1, _ = O.gla_fwd(q, k, v, g, h0)
    o0, _ = O.gla_fwd(q, k, v, g, None)
    b = np.cumsum(g, axis=2)
    np.testing.assert_allclose(o1, o0 + (q * np.exp(b)) @ h0, rtol=1e-11, atol=1e-11)


def test_near_reset_gate_keeps_only_current_token(rng):
    q, k, v, g, _ = _rand_inputs(rng, T=8, gate=-30.0, h0=False)
    o, _ = O.gla_fwd(q, k, v, g)
    ref = np.sum(q * k, axis=-1, keepdims=True) * v
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-10)


@pytest.mark.parametrize("chunk", [1, 2, 3, 4, 5, 8, 16, 64, 37])
def test_chunked_form_equals_recurrence(rng, chunk):
    q, k, v, g, h0 = _rand_inputs(rng, B=1, H=2, T=37, dk=5, dv=3)
    o, hT = O.gla_fwd(q, k, v, g, h0)
    oc, hTc = O.gla_chunked_fwd(q, k, v, g, h0, chunk=chunk)
    np.testing.assert_allclose(oc, o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hTc, hT, rtol=1e-12, atol=1e-12)


def test_decode_steps_continue_the_sequence(rng):
    q, k, v, g, h0 = _rand_inputs(rng, T=20)
    o, hT = O.gla_fwd(q, k, v, g, h0)
    oa, S = O.gla_chunked_fwd(q[:, :, :12], k[:, :, :12], v[:, :, :12], g[:, :, :12], h0, chunk=4)
    np.testing.assert_allclose(oa, o[:, :, :12], rtol=1e-12, atol=1e-12)
    for t in range(12, 20):
        ot, S = O.gla_decode_step(q[:, :, t], k[:, :, t], v[:, :, t], g[:, :, t], S)
        np.testing.assert_allclose(ot, o[:, :, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, hT, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------
# backward pins
# ---------------------------------------------------------------------------------------
def _fd_grad(f, x, eps=1e-6):
    grad = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + eps
        fp = f()
        x[idx] = old - eps
        fm = f()
        x[idx] = old
        grad[idx] = (fp - fm) / (2 * eps)
    return grad


def test_gla_bwd_matches_finite_differences(rng):
    q, k, v, g, h0 = _rand_inputs(rng, B=1, H=1, T=9, dk=3, dv=4)
    do = rng.standard_normal(q.shape[:3] + (4,))
    dhT = rng.standard_normal(h0.shape)

    def loss():
        o, hT = O.gla_fwd(q, k, v, g, h0)
        return float(np.sum(o * do) + np.sum(hT * dhT))

    dq, dk, dv, dg, dh0 = O.gla_bwd(q, k, v, g, h0, do, dhT, ckpt=4)
    for name, x, an in [("q", q, dq), ("k", k, dk), ("v", v, dv), ("g", g, dg), ("h0", h0, dh0)]:
        num = _fd_grad(loss, x)
        np.testing.assert_allclose(an, num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_gla_bwd_alpha_one_closed_forms(rng):
    q, k, v, g, _ = _rand_inputs(rng, T=12, gate="zero", h0=False)
    do = rng.standard_normal(v.shape)
    dq, dk, dv, _, _ = O.gla_bwd(q, k, v, g, None, do)
    M = np.tril(np.ones((12, 12)))
    dA = do @ np.swapaxes(v, -1, -2) * M
    np.testing.assert_allclose(dq, dA @ k, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(dk, np.swapaxes(dA, -1, -2) @ q, rtol=1e-11, atol=1e-11)
    A = q @ np.swapaxes(k, -1, -2) * M
    np.testing.assert_allclose(dv, np.swapaxes(A, -1, -2) @ do, rtol=1e-11, atol=1e-11)


def test_gate_gradient_identity(rng):
    q, k, v, g, h0 = _rand_inputs(rng, B=2, H=2, T=17, dk=4, dv=3)
    do = rng.standard_normal(v.shape)
    dhT = rng.standard_normal(h0.shape)
    _, hT = O.gla_fwd(q, k, v, g, h0)
    dq, dk, _, dg, _ = O.gla_bwd(q, k, v, g, h0, do, dhT, ckpt=5)
    np.testing.assert_allclose(O.dg_from_identity(q, k, dq, dk, hT, dhT), dg, rtol=1e-10, atol=1e-10)


def test_checkpoint_interval_does_not_change_gradients(rng):
    q, k, v, g, h0 = _rand_inputs(rng, T=23)
    do = rng.standard_normal(v.shape)
    a = O.gla_bwd(q, k, v, g, h0, do, ckpt=1)
    b = O.gla_bwd(q, k, v, g, h0, do, ckpt=7)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------------------
# value-gated pass and GSA pins
# ---------------------------------------------------------------------------------------
def _brute_value_gated(q, k, phi, g, h0):
    """o1_t[s] = sum_{r<=t} (q_t . k_r) phi_r[s] exp(b_t[s]-b_r[s]) + exp(b_t[s]) (q_t h0)[s]."""
    B, H, T, _ = q.shape
    m = phi.shape[-1]
    b = np.cumsum(g, axis=2)
    o = np.zeros((B, H, T, m))
    for bb in range(B):
        for hh in range(H):
            for t in range(T):
                for r in range(t + 1):
                    o[bb, hh, t] += np.dot(q[bb, hh, t], k[bb, hh, r]) * phi[bb, hh, r] * np.exp(
                        b[bb, hh, t] - b[bb, hh, r])
                if h0 is not None:
                    o[bb, hh, t] += np.exp(b[bb, hh, t]) * (q[bb, hh, t] @ h0[bb, hh])
    return o


def test_value_gated_pass_matches_bruteforce(rng):
    q, k, phi, _, _ = _rand_inputs(rng, B=1, H=2, T=8, dk=3, dv=4)
    g = -np.log1p(np.exp(rng.standard_normal(phi.shape)))
    h0 = rng.standard_normal((1, 2, 3, 4))
    o1, _ = O.gla_value_gated_fwd(q, k, phi, g, h0)
    np.testing.assert_allclose(o1, _brute_value_gated(q, k, phi, g, h0), rtol=1e-12, atol=1e-12)


def test_value_gated_bwd_matches_finite_differences(rng):
    q, k, phi, _, _ = _rand_inputs(rng, B=1, H=1, T=7, dk=3, dv=4)
    g = -np.log1p(np.exp(rng.standard_normal(phi.shape)))
    h0 = rng.standard_normal((1, 1, 3, 4))
    do1 = rng.standard_normal(phi.shape)
    dhT = rng.standard_normal(h0.shape)

    def loss():
        o1, hT = O.gla_value_gated_fwd(q, k, phi, g, h0)
        return float(np.sum(o1 * do1) + np.sum(hT * dhT))

    grads = O.gla_value_gated_bwd(q, k, phi, g, h0, do1, dhT)
    for name, x, an in zip(["q", "k", "phi", "g", "h0"], [q, k, phi, g, h0], grads):
        np.testing.assert_allclose(an, _fd_grad(loss, x), rtol=1e-6, atol=1e-7, err_msg=name)


def test_softmax_matches_library(rng):
    import torch
    x = rng.standard_normal((3, 5, 64)) * 4
    np.testing.assert_allclose(O.softmax(x), torch.softmax(torch.from_numpy(x), -1).numpy(),
                               rtol=1e-14, atol=1e-15)


def test_gsa_alpha_one_bruteforce(rng):
    B, H, T, dk, dv, m = 1, 2, 9, 3, 4, 5
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    phi = rng.standard_normal((B, H, T, m))
    g = np.zeros((B, H, T, m))
    o, p, _, _ = O.gsa_fwd(q, k, v, phi, g)
    for t in range(T):
        s = sum((q[:, :, t] * k[:, :, r]).sum(-1, keepdims=True) * phi[:, :, r] for r in range(t + 1))
        e = np.exp(s - s.max(-1, keepdims=True))
        pt = e / e.sum(-1, keepdims=True)
        np.testing.assert_allclose(p[:, :, t], pt, rtol=1e-12, atol=1e-13)
        ot = sum((pt * phi[:, :, r]).sum(-1, keepdims=True) * v[:, :, r] for r in range(t + 1))
        np.testing.assert_allclose(o[:, :, t], ot, rtol=1e-12, atol=1e-12)


def test_gsa_single_slot(rng):
    B, H, T, dk, dv = 1, 1, 10, 3, 4
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    phi = rng.standard_normal((B, H, T, 1))
    g = -np.abs(rng.standard_normal((B, H, T, 1)))
    o, p, _, _ = O.gsa_fwd(q, k, v, phi, g)
    np.testing.assert_allclose(p, 1.0, rtol=0, atol=0)
    b = np.cumsum(g[..., 0], axis=2)
    for t in range(T):
        ot = sum(phi[:, :, r] * np.exp(b[:, :, t] - b[:, :, r])[..., None] * v[:, :, r] for r in range(t + 1))
        np.testing.assert_allclose(o[:, :, t], ot, rtol=1e-12, atol=1e-12)
    do = rng.standard_normal(v.shape)
    dq, dk, *_ = O.gsa_bwd(q, k, v, phi, g, None, None, do)
    np.testing.assert_array_equal(dq, 0.0)
    np.testing.assert_array_equal(dk, 0.0)


def test_gsa_constant_gate_retnet_both_passes(rng):
    B, H, T, dk, dv, m, gamma = 1, 1, 8, 3, 2, 4, 0.8
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    phi = rng.standard_normal((B, H, T, m))
    g = np.full((B, H, T, m), np.log(gamma))
    o, p, _, _ = O.gsa_fwd(q, k, v, phi, g)
    t = np.arange(T)
    Dm = np.where(t[:, None] >= t[None, :], gamma ** (t[:, None] - t[None, :]).clip(0), 0.0)
    o1 = (q @ np.swapaxes(k, -1, -2) * Dm) @ phi
    e = np.exp(o1 - o1.max(-1, keepdims=True))
    pr = e / e.sum(-1, keepdims=True)
    np.testing.assert_allclose(p, pr, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o, (pr @ np.swapaxes(phi, -1, -2) * Dm) @ v, rtol=1e-11, atol=1e-12)


def test_gsa_bwd_matches_finite_differences(rng):
    B, H, T, dk, dv, m = 1, 1, 6, 3, 2, 4
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    phi = rng.standard_normal((B, H, T, m))
    g = -np.log1p(np.exp(rng.standard_normal((B, H, T, m))))
    h1 = rng.standard_normal((B, H, dk, m))
    h2 = rng.standard_normal((B, H, m, dv))
    do = rng.standard_normal((B, H, T, dv))
    d1 = rng.standard_normal(h1.shape)
    d2 = rng.standard_normal(h2.shape)

    def loss():
        o, _, hT1, hT2 = O.gsa_fwd(q, k, v, phi, g, h1, h2)
        return float(np.sum(o * do) + np.sum(hT1 * d1) + np.sum(hT2 * d2))

    grads = O.gsa_bwd(q, k, v, phi, g, h1, h2, do, d1, d2)
    for name, x, an in zip(["q", "k", "v", "phi", "g", "h0_1", "h0_2"], [q, k, v, phi, g, h1, h2], grads):
        np.testing.assert_allclose(an, _fd_grad(loss, x), rtol=1e-6, atol=1e-7, err_msg=name)


# ---------------------------------------------------------------------------------------
# planted mistakes: copies of the recurrence with one plausible error must fail the pins
# ---------------------------------------------------------------------------------------
def _mutant(q, k, v, g, h0, kind):
    B, H, T, dk = q.shape
    S = h0.copy()
    o = np.zeros(q.shape[:3] + (v.shape[-1],))
    for t in range(T):
        a = np.exp(g[:, :, t])
        kv = k[:, :, t, :, None] * v[:, :, t, None, :]
        if kind == "decay_after_write":
            S = a[..., None] * (S + kv)
        elif kind == "exclusive_readout":
            o[:, :, t] = np.einsum("bhi,bhij->bhj", q[:, :, t], S)
            S = a[..., None] * S + kv
            continue
        elif kind == "gate_on_value_axis":
            S = a[..., None, :] * S + kv
        elif kind == "sign":
            S = a[..., None] * S - kv
        S_read = S
        o[:, :, t] = np.einsum("bhi,bhij->bhj", q[:, :, t], S_read)
    return o, S


@pytest.mark.parametrize("kind", ["decay_after_write", "exclusive_readout", "gate_on_value_axis", "sign"])
def test_planted_mistakes_fail_the_bruteforce_pin(rng, kind):
    q, k, v, g, h0 = _rand_inputs(rng, B=1, H=1, T=6, dk=3, dv=3)
    bo, _ = _brute_gla(q, k, v, g, h0)
    mo, _ = _mutant(q, k, v, g, h0, kind)
    assert np.max(np.abs(mo - bo)) > 1e-3


# ---------------------------------------------------------------------------------------
# raw-logit gate: g = logsigmoid(x) / tau and its derivative
# ---------------------------------------------------------------------------------------
def test_gate_logsigmoid_values():
    """logsigmoid(0) = -ln 2; logsigmoid(x) - logsigmoid(-x) = x; -> 0 for large x, -> x for very negative x."""
    tau = 16.0
    assert abs(O.gate_logsigmoid(0.0, tau) * tau + math.log(2.0)) < 1e-15
    x = np.linspace(-30, 30, 121)
    np.testing.assert_allclose((O.gate_logsigmoid(x, 1.0) - O.gate_logsigmoid(-x, 1.0)), x, rtol=0, atol=1e-12)
    assert abs(O.gate_logsigmoid(60.0, 1.0)) < 1e-25
    assert abs(O.gate_logsigmoid(-700.0, 8.0) - (-700.0 / 8.0)) < 1e-12
    assert np.all(np.diff(O.gate_logsigmoid(x, tau)) > 0) and np.all(O.gate_logsigmoid(x, tau) < 0)


def test_gate_logsigmoid_bwd_finite_differences(rng):
    x = rng.normal(size=50) * 4
    dg = rng.normal(size=50)
    tau, h = 8.0, 1e-6
    fd = dg * (O.gate_logsigmoid(x + h, tau) - O.gate_logsigmoid(x - h, tau)) / (2 * h)
    np.testing.assert_allclose(O.gate_logsigmoid_bwd(x, dg, tau), fd, rtol=1e-7, atol=1e-10)
    # sigmoid(-x) + sigmoid(x) = 1
    np.testing.assert_allclose(O.gate_logsigmoid_bwd(x, dg, tau) + O.gate_logsigmoid_bwd(-x, dg, tau), dg / tau,
                               rtol=1e-13, atol=1e-15)


def test_planted_gate_mistake_fails():
    """A gate built as log(sigmoid(x)) * tau (scale applied the wrong way) fails the ln 2 pin."""
    wrong = -math.log1p(math.exp(0.0)) * 16.0
    assert abs(wrong * 16.0 + math.log(2.0)) > 1e-3


# ---------------------------------------------------------------------------------------
# MS-GLA pooling and causal hold
# ---------------------------------------------------------------------------------------
def test_msgla_pool_hand_example():
    """T = 5, s = 2: blocks {1,2}, {3,4}, {5} -> 1.5, 3.5, 5 (the short block averages its one token)."""
    x = np.arange(1.0, 6.0).reshape(1, 1, 5, 1)
    np.testing.assert_array_equal(O.msgla_pool(x, 2).ravel(), [1.5, 3.5, 5.0])
    np.testing.assert_array_equal(O.msgla_pool(x, 5).ravel(), [3.0])
    np.testing.assert_array_equal(O.msgla_pool(x, 1), x)


def test_msgla_hold_hand_example():
    """Pooled outputs [a, b, c] at s = 2, T = 5: token t sees block (t+1)//2 - 1 -> [0, a, a, b, b]."""
    y = np.array([10.0, 20.0, 30.0]).reshape(1, 1, 3, 1)
    np.testing.assert_array_equal(O.msgla_hold(y, 5, 2).ravel(), [0, 10, 10, 20, 20])
    np.testing.assert_array_equal(O.msgla_hold(y, 3, 1).ravel(), [10, 20, 30])


def test_msgla_pool_then_hold_is_causal(rng):
    """hold(pool(x)) at token t depends on x only through tokens <= t, and a block shows up
    exactly at its last token."""
    T, s = 13, 4
    x = rng.normal(size=(1, 2, T, 3))
    base = O.msgla_hold(O.msgla_pool(x, s), T, s)
    for t0 in range(T):
        x2 = x.copy()
        x2[..., t0, :] += 1.0
        diff = np.abs(O.msgla_hold(O.msgla_pool(x2, s), T, s) - base).max(axis=(0, 1, 3))
        changed = np.nonzero(diff > 1e-12)[0]
        if changed.size:
            first = (t0 // s + 1) * s - 1  # last token of t0's block
            assert changed.min() == first and changed.min() >= t0


@pytest.mark.parametrize("T,s", [(13, 4), (8, 8), (7, 1), (5, 9)])
def test_msgla_backward_is_the_adjoint(rng, T, s):
    """<pool(x), dy> = <x, pool_bwd(dy)> and <hold(y), dz> = <y, hold_bwd(dz)>."""
    P = -(-T // s)
    x, dy = rng.normal(size=(2, 1, T, 4)), rng.normal(size=(2, 1, P, 4))
    assert abs((O.msgla_pool(x, s) * dy).sum() - (x * O.msgla_pool_bwd(dy, T, s)).sum()) < 1e-12
    y, dz = rng.normal(size=(2, 1, P, 4)), rng.normal(size=(2, 1, T, 4))
    assert abs((O.msgla_hold(y, T, s) * dz).sum() - (y * O.msgla_hold_bwd(dz, s)).sum()) < 1e-12
