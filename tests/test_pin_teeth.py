"""The oracle's pins have teeth: a plain step recurrence written here on the CPU
passes them, and each plausible mistake planted in a copy of it (the step
order, a dropped decay, a sign, a transposed operand, swapped gates, the
readout taken before the update) fails at least one.

The checks are the ones the oracle is pinned by: the pages' literal product
form (explicit transition matrices), the Complex-KDA rotation closed form
(d_k = 2, alpha = (1, -1), beta = 2, unit k: R(2 theta + pi) per token), and
causal linear attention (RDA with e = 0, alpha = 1)."""
import math

import numpy as np
import pytest

import oracle

MISTAKES = [None, "decay_after_write", "residual_without_decay", "erase_sign", "readout_transposed",
            "gates_swapped", "readout_before_update"]


def step_recurrence(variant, q, k, v, alpha, g1, g2, s0, mistake=None):
    """One sequence and head: q, k, alpha [T, d_k]; v [T, d_v]; gates [T] or [T, d]."""
    T, dk = q.shape
    S = np.zeros((dk, v.shape[1])) if s0 is None else s0.copy()
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        if variant == "kda":
            e, w = g1[t], g1[t]
        else:
            e, w = g1[t], g2[t]
        if mistake == "gates_swapped":
            e, w = w, e
        at, m = e * k[t], w * v[t]
        if mistake == "readout_before_update":
            o[t] = S.T @ q[t]
        if mistake == "decay_after_write":
            S = alpha[t][:, None] * (S + np.outer(k[t], m - S.T @ at))
        else:
            Sp = alpha[t][:, None] * S
            pred = S.T @ at if mistake == "residual_without_decay" else Sp.T @ at
            u = m + pred if mistake == "erase_sign" else m - pred
            S = Sp + np.outer(k[t], u)
        if mistake != "readout_before_update":
            o[t] = S @ q[t] if mistake == "readout_transposed" else S.T @ q[t]
    return o, S


def agrees_with_product_form(mistake):
    rng = np.random.default_rng(11)
    T, d = 9, 4                                   # d_k = d_v so that a transposed operand is well formed
    for variant in ("kda", "rda", "gdn2"):
        q, k, v = rng.standard_normal((3, T, d))
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        alpha = np.tanh(2 * rng.standard_normal((T, d)))
        if variant == "gdn2":
            g1, g2 = rng.uniform(0, 1, (2, T, d))
        else:
            g1, g2 = rng.uniform(0, 2, T), rng.uniform(0, 1, T)
            if variant == "kda":
                g2 = None
        s0 = rng.standard_normal((d, d))
        o, s = step_recurrence(variant, q, k, v, alpha, g1, g2, s0, mistake)
        lead = lambda x: None if x is None else x[None, :, None]
        o_ref, s_ref = oracle.literal_recurrence(variant, lead(q), lead(k), lead(v), lead(alpha), lead(g1),
                                                 lead(g2), s0[None, None])
        if not (np.allclose(o, o_ref[0, :, 0], atol=1e-10) and np.allclose(s, s_ref[0, 0], atol=1e-10)):
            return False
    return True


def agrees_with_rotation(mistake):
    T, th = 7, 0.4
    k = np.tile([math.cos(th), math.sin(th)], (T, 1))
    s0 = np.array([[1.0, 0.3], [-0.2, 0.7]])
    _, s = step_recurrence("kda", np.zeros((T, 2)), k, np.zeros((T, 2)), np.tile([1.0, -1.0], (T, 1)),
                           np.full(T, 2.0), None, s0, mistake)
    phi = T * (2 * th + math.pi)
    R = np.array([[math.cos(phi), -math.sin(phi)], [math.sin(phi), math.cos(phi)]])
    return np.allclose(s, R @ s0, atol=1e-12)


def agrees_with_linear_attention(mistake):
    rng = np.random.default_rng(12)
    T, d = 8, 3
    q, k, v = rng.standard_normal((3, T, d))
    w = rng.uniform(0.5, 1.5, T)
    s0 = rng.standard_normal((d, d))
    o, _ = step_recurrence("rda", q, k, v, np.ones((T, d)), np.zeros(T), w, s0, mistake)
    ref = np.stack([s0.T @ q[t] + sum(w[s] * (q[t] @ k[s]) * v[s] for s in range(t + 1)) for t in range(T)])
    return np.allclose(o, ref, atol=1e-12)


def test_the_faithful_recurrence_passes_every_check():
    assert agrees_with_product_form(None) and agrees_with_rotation(None) and agrees_with_linear_attention(None)


@pytest.mark.parametrize("mistake", MISTAKES[1:])
def test_each_planted_mistake_fails_a_check(mistake):
    passed = [agrees_with_product_form(mistake), agrees_with_rotation(mistake), agrees_with_linear_attention(mistake)]
    assert not all(passed), f"{mistake} slipped through every check"
