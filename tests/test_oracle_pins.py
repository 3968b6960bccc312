"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: the pages' own
product form, a property the pages state, a closed form, or a textbook special
case.  A plausible slip anywhere in the oracle (a dropped term, a wrong sign,
decay applied after the erase instead of before, a transposed state, a readout
on the pre-update state, a gate read at the wrong index) fails at least one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import make_chunk_inputs, tiny_ckda

RNG = np.random.default_rng(1234)


def _small(variant, rng_seed, B=2, T=9, H=2, dk=5, dv=3, gate_range="standard", init="random"):
    return make_chunk_inputs(variant, gate_range, "f32", B=B, T=T, H=H, d_k=dk, d_v=dv,
                             seed=rng_seed, init_state=init, init_std=0.5)


@pytest.mark.parametrize("variant", ["kda", "rda", "gdn2"])
@pytest.mark.parametrize("gate_range", ["standard", "extended"])
def test_step_recurrence_equals_literal_product_form(variant, gate_range):
    """C step recurrence == the update equations exactly as printed
    (Raon-1-mini-preview discussion: KDA, RDA, GDN-2 equations)."""
    inp = _small(variant, 7, gate_range=gate_range)
    o, sf = oracle.recurrence(inp)
    o2, sf2 = oracle.literal_recurrence(variant, inp.q, inp.k, inp.v, inp.alpha, inp.g1, inp.g2,
                                        inp.initial_state)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sf, sf2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("variant", ["kda", "rda", "gdn2"])
def test_step_recurrence_equals_brute_force(variant):
    """Dense unrolled closed form on tiny inputs, recomputed for every t."""
    inp = _small(variant, 11, B=1, T=6, H=1, dk=4, dv=3, gate_range="extended")
    o, sf = oracle.recurrence(inp)
    o2, sf2 = oracle.brute_force(variant, inp.q, inp.k, inp.v, inp.alpha, inp.g1, inp.g2, inp.initial_state)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sf, sf2, rtol=0, atol=1e-12)


def test_rda_reduces_to_kda_when_e_equals_w():
    """'RDA reduces to KDA when e_t = w_t' (Raon-1-mini-preview discussion)."""
    kda = _small("kda", 3, gate_range="extended")
    o_k, s_k = oracle.recurrence(kda)
    o_r, s_r = oracle.recurrence_arrays("rda", kda.q, kda.k, kda.v, kda.alpha, kda.g1, kda.g1,
                                        None, kda.initial_state)
    assert np.array_equal(o_k, o_r) and np.array_equal(s_k, s_r)
    # and a genuinely different w changes the result (the write gate is read)
    o_r2, _ = oracle.recurrence_arrays("rda", kda.q, kda.k, kda.v, kda.alpha, kda.g1, kda.g1 * 0.5,
                                       None, kda.initial_state)
    assert not np.allclose(o_k, o_r2)


def test_gdn2_reduces_to_rda_for_constant_vectors():
    """GDN-2 with b_t = e_t 1 and w_t = w_t 1 is RDA (the two equations on the
    discussion page coincide term by term)."""
    rda = _small("rda", 5, dk=6, dv=4)
    b = rda.g1[..., None].expand(*rda.g1.shape, rda.d_k).contiguous()
    w = rda.g2[..., None].expand(*rda.g2.shape, rda.d_v).contiguous()
    o_r, s_r = oracle.recurrence(rda)
    o_g, s_g = oracle.recurrence_arrays("gdn2", rda.q, rda.k, rda.v, rda.alpha, b, w, None, rda.initial_state)
    np.testing.assert_allclose(o_g, o_r, rtol=0, atol=1e-14)
    np.testing.assert_allclose(s_g, s_r, rtol=0, atol=1e-14)
    # channel-wise gates that are NOT constant give a different answer
    b2 = b.clone()
    b2[..., 0] = 0.0
    o_g2, _ = oracle.recurrence_arrays("gdn2", rda.q, rda.k, rda.v, rda.alpha, b2, w, None, rda.initial_state)
    assert not np.allclose(o_g2, o_r)


def _transitions_from_oracle(k, alpha, beta):
    """Read the oracle's transition matrices: start each sequence from S_0 = I
    (d_v = d_k) with v = 0, run one token; then S_1 = A_1 I = A_1."""
    n, d = k.shape
    z = np.zeros((n, 1, 1, d))
    s0 = np.broadcast_to(np.eye(d), (n, 1, d, d)).copy()
    _, sf = oracle.recurrence_arrays("kda", z, k.reshape(n, 1, 1, d), z, alpha.reshape(n, 1, 1, d),
                                     beta.reshape(n, 1, 1), None, None, s0)
    return sf[:, 0]


def test_ckda_transitions_are_non_expansive():
    """Complex KDA transitions (I - beta k k^T) Diag(alpha) with unit k,
    alpha in [-1,1]^d and beta in [0,2] have spectral norm <= 1 (abstract:
    'transitions that remain diagonal-plus-rank-one and non-expansive')."""
    n, d = 10000, 8
    k = RNG.standard_normal((n, d))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    alpha = RNG.uniform(-1, 1, (n, d))
    alpha[: n // 10] = np.sign(alpha[: n // 10])          # include the orthogonal corner |alpha| = 1
    beta = RNG.uniform(0, 2, n)
    beta[: n // 20] = 2.0
    A = _transitions_from_oracle(k, alpha, beta)
    sv = np.linalg.svd(A, compute_uv=False)[:, 0]
    assert sv.max() <= 1.0 + 1e-12
    assert sv.max() >= 1.0 - 1e-9        # the bound is attained (reflection x sign gate)
    # outside the extended range the bound fails, so the check has teeth
    A_bad = _transitions_from_oracle(k[:2000], alpha[:2000], np.full(2000, 2.5))
    assert np.linalg.svd(A_bad, compute_uv=False)[:, 0].max() > 1.0 + 1e-3


def _rot(phi):
    return np.array([[math.cos(phi), -math.sin(phi)], [math.sin(phi), math.cos(phi)]])


@pytest.mark.parametrize("theta", [0.0, 0.3, 1.1, -2.0, math.pi / 4])
def test_reflection_times_gate_is_exact_2d_rotation(theta):
    """d_k = 2, alpha = (1,-1), beta = 2, k = (cos th, sin th): the delta-rule
    reflection times the sign-flip gate is the rotation R(2 th + pi)
    (abstract: 'realize 2D rotations by combining a single delta-rule
    transformation with a second reflection supplied by its channel-wise
    gate')."""
    k = np.array([[math.cos(theta), math.sin(theta)]])
    A = _transitions_from_oracle(k, np.array([[1.0, -1.0]]), np.array([2.0]))[0]
    np.testing.assert_allclose(A, _rot(2 * theta + math.pi), atol=1e-15)
    np.testing.assert_allclose(A @ A.T, np.eye(2), atol=1e-15)
    assert abs(np.linalg.det(A) - 1.0) < 1e-15
    # many steps with v = 0: S_T = R(T (2 th + pi)) S_0
    T = 37
    s0 = RNG.standard_normal((1, 1, 2, 3))
    z2 = np.zeros((1, T, 1, 2))
    z3 = np.zeros((1, T, 1, 3))
    kk = np.broadcast_to(k, (1, T, 1, 2)).copy()
    al = np.broadcast_to([1.0, -1.0], (1, T, 1, 2)).copy()
    _, sf = oracle.recurrence_arrays("kda", z2, kk, z3, al, np.full((1, T, 1), 2.0), None, None, s0)
    np.testing.assert_allclose(sf[0, 0], _rot(T * (2 * theta + math.pi)) @ s0[0, 0], atol=1e-12)


def test_no_erase_no_decay_keeps_state():
    """beta = 0 and alpha = 1: S_t = S_0 and o_t = S_0^T q_t."""
    inp = _small("kda", 21, init="random")
    inp.alpha = torch.ones_like(inp.alpha)
    inp.g1 = torch.zeros_like(inp.g1)
    o, sf = oracle.recurrence(inp)
    s0 = inp.initial_state.double().numpy()
    np.testing.assert_allclose(sf, s0, atol=0)
    ref = np.einsum("bthi,bhij->bthj", inp.q.double().numpy(), s0)
    np.testing.assert_allclose(o, ref, atol=1e-13)


def test_rda_without_erase_is_causal_linear_attention():
    """RDA with e = 0 and alpha = 1 is plain causal linear attention:
    o = ((Q K^T) (.) causal mask (.) w) V + Q S_0, a dense-matrix formula."""
    inp = _small("rda", 31, B=1, T=23, H=2, dk=6, dv=4)
    inp.alpha = torch.ones_like(inp.alpha)
    inp.g1 = torch.zeros_like(inp.g1)
    o, _ = oracle.recurrence(inp)
    for h in range(inp.H):
        Q, K, V = (x[0, :, h].double().numpy() for x in (inp.q, inp.k, inp.v))
        w = inp.g2[0, :, h].double().numpy()
        L = np.tril(Q @ K.T) * w[None, :]
        ref = L @ V + Q @ inp.initial_state[0, h].double().numpy()
        np.testing.assert_allclose(o[0, :, h], ref, atol=1e-12)


def test_rda_without_erase_is_gated_linear_attention():
    """RDA with e = 0: gated linear attention with channel-wise decay (the
    Lightning-style recurrence without the v - Sk correction):
    o_t = sum_{s<=t} w_s sum_c q_tc (prod_{s<r<=t} alpha_rc) k_sc v_s
          + sum_c q_tc (prod_{r<=t} alpha_rc) S_0[c,:]."""
    inp = _small("rda", 41, B=1, T=12, H=1, dk=5, dv=3, gate_range="extended")
    inp.g1 = torch.zeros_like(inp.g1)
    o, _ = oracle.recurrence(inp)
    Q, K, V, Al = (x[0, :, 0].double().numpy() for x in (inp.q, inp.k, inp.v, inp.alpha))
    w = inp.g2[0, :, 0].double().numpy()
    S0 = inp.initial_state[0, 0].double().numpy()
    T = Q.shape[0]
    for t in range(T):
        acc = np.zeros(V.shape[1])
        for s in range(t + 1):
            lam = np.prod(Al[s + 1:t + 1], axis=0) if t > s else np.ones(K.shape[1])
            acc += w[s] * np.sum(Q[t] * lam * K[s]) * V[s]
        acc += (Q[t] * np.prod(Al[:t + 1], axis=0)) @ S0
        np.testing.assert_allclose(o[0, t, 0], acc, atol=1e-12)


def test_unit_erase_on_one_hot_key_overwrites_row():
    """beta = 1, alpha = 1, k = e_i: row i of the state is replaced by v_t
    exactly, other rows untouched (the notebook analogy on the openarchlab
    page: erase the old number on that line, then write the new one)."""
    dk, dv, T = 6, 4, 5
    s0 = RNG.standard_normal((1, 1, dk, dv))
    idx = [2, 0, 2, 5, 3]
    k = np.zeros((1, T, 1, dk))
    for t, i in enumerate(idx):
        k[0, t, 0, i] = 1.0
    v = RNG.standard_normal((1, T, 1, dv))
    S = s0[0, 0].copy()
    for t in range(T):
        _, sf = oracle.recurrence_arrays("kda", np.zeros((1, t + 1, 1, dk)), k[:, :t + 1], v[:, :t + 1],
                                         np.ones((1, t + 1, 1, dk)), np.ones((1, t + 1, 1)), None, None, s0)
        S[idx[t]] = v[0, t, 0]
        np.testing.assert_allclose(sf[0, 0], S, atol=1e-15)


def test_householder_reflection_preserves_frobenius_norm():
    """beta = 2, alpha = 1, v = 0: each step applies I - 2 k k^T (unit k), an
    orthogonal reflection, so ||S_t||_F = ||S_0||_F."""
    dk, dv, T = 7, 5, 40
    k = RNG.standard_normal((1, T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    s0 = RNG.standard_normal((1, 1, dk, dv))
    _, sf = oracle.recurrence_arrays("kda", np.zeros((1, T, 1, dk)), k, np.zeros((1, T, 1, dv)),
                                     np.ones((1, T, 1, dk)), np.full((1, T, 1), 2.0), None, None, s0)
    assert abs(np.linalg.norm(sf) - np.linalg.norm(s0)) < 1e-12


def test_zero_gate_erases_channel_exactly():
    """alpha_t = 0 wipes the decayed state, so S_t = k_t m_t^T exactly
    (u = m because S' = 0)."""
    inp = _small("gdn2", 51, B=1, T=4, H=1, dk=5, dv=3)
    inp.alpha[0, -1] = 0.0
    _, sf = oracle.recurrence(inp)
    k = inp.k[0, -1, 0].double().numpy()
    m = inp.g2[0, -1, 0].double().numpy() * inp.v[0, -1, 0].double().numpy()
    np.testing.assert_array_equal(sf[0, 0], np.outer(k, m))


def test_state_continuation_and_varlen_packing():
    """Running [0,t) then [t,T) from the carried state equals [0,T); packing
    documents with cu_seqlens equals running them separately (document reset,
    openarchlab page sec. 3)."""
    inp = _small("rda", 61, B=1, T=20, H=3, dk=4, dv=5, gate_range="extended")
    o, sf = oracle.recurrence(inp)
    t = 7
    a = [x[:, :t] for x in (inp.q, inp.k, inp.v, inp.alpha, inp.g1, inp.g2)]
    b = [x[:, t:] for x in (inp.q, inp.k, inp.v, inp.alpha, inp.g1, inp.g2)]
    oa, sa = oracle.recurrence_arrays("rda", *a, None, inp.initial_state)
    ob, sb = oracle.recurrence_arrays("rda", *b, None, sa)
    assert np.array_equal(np.concatenate([oa, ob], axis=1), o) and np.array_equal(sb, sf)
    # varlen: three documents packed along T
    lens = [5, 1, 9]
    pk = make_chunk_inputs("gdn2", "extended", "f32", H=2, d_k=4, d_v=3, seed=71, doc_lens=lens,
                           init_state="random", init_std=0.3)
    o_p, s_p = oracle.recurrence(pk)
    start = 0
    for n, ln in enumerate(lens):
        parts = [x[:, start:start + ln] for x in (pk.q, pk.k, pk.v, pk.alpha, pk.g1, pk.g2)]
        o_n, s_n = oracle.recurrence_arrays("gdn2", *parts, None, pk.initial_state[n:n + 1])
        assert np.array_equal(o_p[:, start:start + ln], o_n)
        assert np.array_equal(s_p[n], s_n[0])
        start += ln


def test_sampled_restriction_matches_full_run():
    pk = make_chunk_inputs("kda", "extended", "f32", H=3, d_k=4, d_v=3, seed=81, doc_lens=[4, 7, 2],
                           init_state="random")
    o, sf = oracle.recurrence(pk)
    o_d, s_d = oracle.recurrence(pk, seqs=[2, 0], heads=[1, 2])
    cu = pk.cu_seqlens.numpy()
    for (n, h), on in o_d.items():
        np.testing.assert_array_equal(on, o[0, cu[n]:cu[n + 1], h])
        np.testing.assert_array_equal(s_d[(n, h)], sf[n, h])


def test_tiny_ckda_inputs_match_recipe():
    """The tiny Complex-KDA workload: shapes, ranges and unit-norm keys."""
    inp = tiny_ckda()
    assert tuple(inp.q.shape) == (1, 64, 2, 16) and inp.chunk_size == 16
    assert inp.q.dtype == torch.float32 and inp.initial_state is None
    assert float(inp.alpha.min()) >= -1 and float(inp.alpha.max()) <= 1 and float(inp.alpha.min()) < 0
    assert float(inp.g1.min()) >= 0 and float(inp.g1.max()) <= 2 and float(inp.g1.max()) > 1
    np.testing.assert_allclose(inp.k.double().norm(dim=-1).numpy(), 1.0, atol=1e-6)


# ---- input preparation (gate logits, L2-normalised k) -------------------------------------

def test_prepare_at_zero_logits():
    """sigmoid(0) = 1/2, exp(-softplus(0)) = 1/2, tanh(0) = 0: the activations' fixed values."""
    z = np.zeros((1, 1, 1, 4))
    zs = np.zeros((1, 1, 1))
    _, a, g1, g2 = oracle.prepare("standard", z + 1.0, z, zs, zs, logits=True)
    assert np.allclose(a, 0.5) and np.allclose(g1, 0.5) and np.allclose(g2, 0.5)
    _, a, g1, g2 = oracle.prepare("extended", z + 1.0, z, zs, zs, logits=True)
    assert np.allclose(a, 0.0) and np.allclose(g1, 1.0) and np.allclose(g2, 1.0)


def test_prepare_inverts_the_activations():
    """Logits written with the inverse functions come back as the gates they encode."""
    rng = np.random.default_rng(11)
    a = rng.uniform(0.01, 0.99, (2, 5, 3, 8))
    g = rng.uniform(0.01, 0.99, (2, 5, 3))
    x = np.log((1.0 - a) / a)                  # exp(-softplus(x)) = 1 / (1 + e^x) = a
    y = np.log(g / (1.0 - g))                  # sigmoid(y) = g
    k = rng.standard_normal((2, 5, 3, 8))
    _, a2, g2, _ = oracle.prepare("standard", k, x, y, None, logits=True)
    assert np.allclose(a2, a, rtol=1e-12, atol=1e-14) and np.allclose(g2, g, rtol=1e-12, atol=1e-14)
    ae = rng.uniform(-0.99, 0.99, (2, 5, 3, 8))
    ge = rng.uniform(0.02, 1.98, (2, 5, 3))
    _, a3, g3, _ = oracle.prepare("extended", k, np.arctanh(ae), np.log((ge / 2) / (1 - ge / 2)), None,
                                  logits=True)
    assert np.allclose(a3, ae, rtol=1e-12, atol=1e-14) and np.allclose(g3, ge, rtol=1e-12, atol=1e-14)
    # GDN-2 vectors take the gate activation elementwise
    b = rng.uniform(0.01, 0.99, (2, 5, 3, 8))
    _, _, b2, w2 = oracle.prepare("standard", k, x, np.log(b / (1 - b)), np.log(b / (1 - b)), logits=True)
    assert np.allclose(b2, b, rtol=1e-12) and np.allclose(w2, b, rtol=1e-12)


def test_prepare_saturates_without_overflow():
    big = np.array([[[[800.0, -800.0]]]])
    with np.errstate(over="raise", invalid="raise", divide="raise"):
        _, a, g, _ = oracle.prepare("standard", big, big, big[..., 0], None, logits=True)
    assert a[0, 0, 0, 0] == 0.0 and a[0, 0, 0, 1] == 1.0 and g[0, 0, 0] == 1.0


def test_prepare_l2_normalises_k():
    rng = np.random.default_rng(12)
    k = rng.standard_normal((2, 7, 3, 16)) * 5.0
    k[0, 0, 0] = 0.0                                       # a zero key stays zero (norm floor)
    kn, a, g1, _ = oracle.prepare("standard", k, np.ones((2, 7, 3, 16)), np.ones((2, 7, 3)), l2norm_k=True)
    n = np.linalg.norm(kn, axis=-1)
    assert np.allclose(n[n > 0], 1.0, rtol=1e-13) and n[0, 0, 0] == 0.0
    assert np.allclose(np.sum(kn * k, axis=-1), np.linalg.norm(k, axis=-1), rtol=1e-12)   # same direction
    assert np.array_equal(a, np.ones((2, 7, 3, 16))) and np.array_equal(g1, np.ones((2, 7, 3)))  # untouched


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "extended"),
                                                ("gdn2", "standard")])
def test_recurrence_with_preparation_equals_prepared_inputs(variant, gate_range):
    """The oracle's prepared path is the recurrence on the activated, normalised inputs."""
    inp = make_chunk_inputs(variant, gate_range, "f32", B=2, T=23, H=2, d_k=8, d_v=4, seed=5,
                              logits=True, raw_k=True, init_state="random", init_std=0.3)
    o1, s1 = oracle.recurrence(inp)
    k, a, g1, g2 = oracle.prepare(gate_range, inp.k, inp.alpha, inp.g1, inp.g2, logits=True, l2norm_k=True,
                                  round_to=inp.dtype)
    o2, s2 = oracle.recurrence_arrays(variant, inp.q, k, inp.v, a, g1, g2, None, inp.initial_state)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)
    # and the raw inputs give a different answer (the preparation is not a no-op)
    o3, _ = oracle.recurrence_arrays(variant, inp.q, inp.k, inp.v, inp.alpha, inp.g1, inp.g2, None,
                                     inp.initial_state)
    assert not np.allclose(o1, o3)


def test_prepare_rounds_to_the_input_dtype():
    """Rounded preparation: bf16-representable values within half a bf16 ulp of the exact ones."""
    rng = np.random.default_rng(13)
    k = rng.standard_normal((1, 9, 2, 16)) * 3
    x = rng.standard_normal((1, 9, 2, 16)) * 2
    y = rng.standard_normal((1, 9, 2))
    ex = oracle.prepare("standard", k, x, y, None, logits=True, l2norm_k=True)
    rd = oracle.prepare("standard", k, x, y, None, logits=True, l2norm_k=True, round_to="bf16")
    for e, r in zip(ex[:3], rd[:3]):
        back = torch.from_numpy(r).to(torch.bfloat16).double().numpy()
        assert np.array_equal(back, r)                                   # representable in bf16
        assert np.all(np.abs(r - e) <= np.abs(e) * 2.0 ** -8 + 1e-300)  # RNE: half an ulp (8 bits)
    f = oracle.prepare("extended", k, x, y, None, logits=True, round_to="f32")
    assert np.array_equal(f[1], f[1].astype(np.float32).astype(np.float64))


def test_chunk_states_are_prefix_runs():
    """The oracle's state after chunk c is the final state of a run over the first 64(c+1) tokens."""
    inp = make_chunk_inputs("gdn2", "extended", "f32", H=2, d_k=8, d_v=4, seed=31, doc_lens=[150, 64, 0, 9],
                            init_state="random", init_std=0.3)
    cs = oracle.chunk_states(inp)
    assert sorted(cs) == [(0, 0), (0, 1), (0, 2), (1, 0), (3, 0)]
    _, s_full = oracle.recurrence(inp)
    for n, c in cs:
        b, t0, ln = inp.seq_bounds(n)
        e = min(ln, 64 * (c + 1))
        cut = make_chunk_inputs("gdn2", "extended", "f32", H=2, d_k=8, d_v=4, seed=31, doc_lens=[150, 64, 0, 9],
                                init_state="random", init_std=0.3)
        _, sp = oracle.recurrence_arrays("gdn2", cut.q[:, t0:t0 + e], cut.k[:, t0:t0 + e], cut.v[:, t0:t0 + e],
                                         cut.alpha[:, t0:t0 + e], cut.g1[:, t0:t0 + e], cut.g2[:, t0:t0 + e],
                                         None, cut.initial_state[n:n + 1])
        assert np.allclose(cs[(n, c)], sp[0], rtol=1e-12, atol=1e-14)
        if 64 * (c + 1) >= ln:                       # the last chunk's state is the final state
            assert np.allclose(cs[(n, c)], s_full[n], rtol=1e-12, atol=1e-14)


# ---- gradients ------------------------------------------------------------------------------

@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "standard"),
                                                ("rda", "extended"), ("gdn2", "standard"), ("gdn2", "extended")])
def test_recurrence_grad_matches_central_differences(variant, gate_range):
    """Every input's gradient against central differences of the forward oracle (float64)."""
    inp = make_chunk_inputs(variant, gate_range, "f32", B=1, T=7, H=1, d_k=4, d_v=3, seed=43,
                            init_state="random", init_std=0.5)
    f = lambda x: x[0, :, 0].double().numpy()
    arrs = {"q": f(inp.q), "k": f(inp.k), "v": f(inp.v), "alpha": f(inp.alpha), "g1": f(inp.g1),
            "g2": None if inp.g2 is None else f(inp.g2)}
    s0 = inp.initial_state[0, 0].double().numpy()
    rng = np.random.default_rng(3)
    do = rng.standard_normal((7, 3))
    dsf = rng.standard_normal((4, 3))

    def loss(a, s):
        o, sf = oracle.recurrence_arrays(variant, *(None if a[n] is None else a[n][None, :, None]
                                                     for n in ("q", "k", "v", "alpha", "g1", "g2")),
                                         None, s[None, None])
        return float(np.sum(o[0, :, 0] * do) + np.sum(sf[0, 0] * dsf))

    g = oracle.recurrence_grad(variant, arrs["q"], arrs["k"], arrs["v"], arrs["alpha"], arrs["g1"], arrs["g2"],
                               s0, do, dsf)
    eps = 1e-6
    for name, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("alpha", "dalpha"), ("g1", "dg1"), ("g2", "dg2")):
        if arrs[name] is None:
            assert g[gname] is None
            continue
        fd = np.zeros_like(arrs[name])
        for idx in np.ndindex(arrs[name].shape):
            a_p = {n: (None if x is None else x.copy()) for n, x in arrs.items()}
            a_m = {n: (None if x is None else x.copy()) for n, x in arrs.items()}
            a_p[name][idx] += eps
            a_m[name][idx] -= eps
            fd[idx] = (loss(a_p, s0) - loss(a_m, s0)) / (2 * eps)
        assert np.allclose(g[gname], fd, rtol=1e-6, atol=1e-7), name
    fd0 = np.zeros_like(s0)
    for idx in np.ndindex(s0.shape):
        sp, sm = s0.copy(), s0.copy()
        sp[idx] += eps
        sm[idx] -= eps
        fd0[idx] = (loss(arrs, sp) - loss(arrs, sm)) / (2 * eps)
    assert np.allclose(g["ds0"], fd0, rtol=1e-6, atol=1e-7)


def test_recurrence_grad_of_linear_attention_closed_form():
    """alpha = 1, beta = 0 (no erase, no write): o_t = S_0^T q_t, so dq_t = S_0 do_t and dS_0 = sum_t q_t do_t^T."""
    rng = np.random.default_rng(4)
    T, dk, dv = 6, 5, 3
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v, s0, do = rng.standard_normal((T, dv)), rng.standard_normal((dk, dv)), rng.standard_normal((T, dv))
    g = oracle.recurrence_grad("kda", q, k, v, np.ones((T, dk)), np.zeros(T), None, s0, do)
    assert np.allclose(g["dq"], do @ s0.T) and np.allclose(g["ds0"], q.T @ do)
    assert np.allclose(g["dv"], 0) and np.allclose(g["dk"], 0)


# ---- rank-2 (DeltaProduct_2-style) steps ----------------------------------------------------

def _rank2_inputs(variant, B=2, T=9, H=2, dk=6, dv=5, seed=51):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = rng.standard_normal((B, T, H, dk))
    k = unit(rng.standard_normal((B, T, 2, H, dk)))
    v = rng.standard_normal((B, T, 2, H, dv))
    alpha = np.tanh(rng.standard_normal((B, T, H, dk)))
    if variant == "gdn2":
        g1, g2 = rng.uniform(0, 1, (B, T, 2, H, dk)), rng.uniform(0, 1, (B, T, 2, H, dv))
    else:
        g1 = rng.uniform(0, 2, (B, T, 2, H))
        g2 = rng.uniform(0, 1, (B, T, 2, H)) if variant == "rda" else None
    s0 = rng.standard_normal((B, H, dk, dv))
    return q, k, v, alpha, g1, g2, s0


@pytest.mark.parametrize("variant", ["kda", "rda", "gdn2"])
def test_rank2_with_silent_second_step_is_rank1(variant):
    """Second sub-step with zero erase and write gates: exactly the rank-1 recurrence on the first."""
    q, k, v, alpha, g1, g2, s0 = _rank2_inputs(variant)
    g1[:, :, 1] = 0
    if g2 is not None:
        g2[:, :, 1] = 0
    o2, s2 = oracle.recurrence_rank2(variant, q, k, v, alpha, g1, g2, initial_state=s0)
    o1, s1 = oracle.recurrence_arrays(variant, q, k[:, :, 0], v[:, :, 0], alpha, g1[:, :, 0],
                                      None if g2 is None else g2[:, :, 0], initial_state=s0)
    assert np.allclose(o2, o1, rtol=1e-12, atol=1e-12) and np.allclose(s2, s1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("variant", ["kda", "rda", "gdn2"])
def test_rank2_equals_two_rank1_tokens_without_decay_in_between(variant):
    """A rank-2 step is two rank-1 steps of the C oracle, the second with alpha = 1, read out after the
    second; packed documents double their offsets."""
    q, k, v, alpha, g1, g2, s0 = _rank2_inputs(variant, B=1, T=11)
    cu = np.array([0, 4, 4, 11])
    s0 = s0[:1].repeat(3, axis=0) * np.array([1.0, -0.5, 2.0])[:, None, None, None]
    o2, s2 = oracle.recurrence_rank2(variant, q, k, v, alpha, g1, g2, cu_seqlens=cu, initial_state=s0)
    B, T, H, dk = q.shape
    inter = lambda x: x.reshape(B, 2 * T, *x.shape[3:])        # [B,T,2,...] is [B,2T,...] in memory
    a2 = np.ones((B, T, 2, H, dk))
    a2[:, :, 0] = alpha
    q2 = np.stack([np.zeros_like(q), q], axis=2)
    o1, s1 = oracle.recurrence_arrays(variant, inter(q2), inter(k), inter(v), inter(a2), inter(g1),
                                      None if g2 is None else inter(g2), cu_seqlens=2 * cu, initial_state=s0)
    assert np.allclose(o2, o1.reshape(B, T, 2, H, -1)[:, :, 1], rtol=1e-12, atol=1e-12)
    assert np.allclose(s2, s1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("a,b", [(0.2, 0.9), (1.1, -0.4)])
def test_rank2_two_reflections_make_a_rotation(a, b):
    """beta = 2 on both sub-steps, unit keys at angles a and b, alpha = 1, v = 0: each step applies the
    Householder reflections H(k1) then H(k2), whose product turns the plane by 2 (b - a); T steps turn
    the state's rows by 2 T (b - a)."""
    T = 5
    k = np.zeros((1, T, 2, 1, 2))
    k[0, :, 0, 0] = [np.cos(a), np.sin(a)]
    k[0, :, 1, 0] = [np.cos(b), np.sin(b)]
    s0 = np.random.default_rng(6).standard_normal((1, 1, 2, 3))
    _, sf = oracle.recurrence_rank2("kda", np.zeros((1, T, 1, 2)), k, np.zeros((1, T, 2, 1, 3)),
                                    np.ones((1, T, 1, 2)), np.full((1, T, 2, 1), 2.0), None, initial_state=s0)
    phi = 2 * T * (b - a)
    R = np.array([[np.cos(phi), -np.sin(phi)], [np.sin(phi), np.cos(phi)]])
    assert np.allclose(sf[0, 0], R @ s0[0, 0], rtol=1e-12, atol=1e-12)


def test_rank2_gradient_is_the_rank1_reverse_mode_over_sub_tokens():
    """The gradient of rank-2 steps equals the rank-1 reverse mode over the 2T sub-tokens (the first carries
    the token's decay and q = 0, the second alpha = 1 and the token's q), mapped back: dq from the second
    sub-tokens, dalpha from the first; k, v and gate gradients keep the sub-token layout.  Checked against
    central differences of ``recurrence_rank2``."""
    rng = np.random.default_rng(21)
    T, dk, dv = 4, 3, 2
    q, alpha = rng.standard_normal((T, dk)), np.tanh(rng.standard_normal((T, dk)))
    k, v = rng.standard_normal((T, 2, dk)), rng.standard_normal((T, 2, dv))
    g1 = rng.uniform(0, 2, (T, 2))
    s0, do, dsf = rng.standard_normal((dk, dv)), rng.standard_normal((T, dv)), rng.standard_normal((dk, dv))

    def loss(q_, k_, v_, a_, g_):
        o, sf = oracle.recurrence_rank2("kda", q_[None, :, None], k_[None, :, :, None], v_[None, :, :, None],
                                        a_[None, :, None], g_[None, :, :, None], None, initial_state=s0[None, None])
        return float(np.sum(o[0, :, 0] * do) + np.sum(sf[0, 0] * dsf))

    q2 = np.stack([np.zeros_like(q), q], axis=1).reshape(2 * T, dk)
    a2 = np.stack([alpha, np.ones_like(alpha)], axis=1).reshape(2 * T, dk)
    do2 = np.stack([np.zeros_like(do), do], axis=1).reshape(2 * T, dv)
    g = oracle.recurrence_grad("kda", q2, k.reshape(2 * T, dk), v.reshape(2 * T, dv), a2, g1.reshape(2 * T),
                               None, s0, do2, dsf)
    mapped = {"q": g["dq"].reshape(T, 2, dk)[:, 1], "alpha": g["dalpha"].reshape(T, 2, dk)[:, 0],
              "k": g["dk"].reshape(T, 2, dk), "v": g["dv"].reshape(T, 2, dv), "g1": g["dg1"].reshape(T, 2)}
    args = {"q": q, "k": k, "v": v, "alpha": alpha, "g1": g1}
    eps = 1e-6
    for name, x in args.items():
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            a_p = {**args, name: xp}
            a_m = {**args, name: xm}
            fd[idx] = (loss(a_p["q"], a_p["k"], a_p["v"], a_p["alpha"], a_p["g1"])
                       - loss(a_m["q"], a_m["k"], a_m["v"], a_m["alpha"], a_m["g1"])) / (2 * eps)
        assert np.allclose(mapped[name], fd, rtol=1e-6, atol=1e-7), name
