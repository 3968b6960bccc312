"""Rank-2 steps (kda_chunk_fwd_rank2) vs the float64 oracle's rank-2 recurrence
(``oracle.recurrence_rank2``: decay once per token, two erase/write sub-steps,
readout after the second), on the tensor-core path (bf16, d = 128, both forms)
and on the token scan (fp32, other head sizes).  Tolerances as for the rank-1
forward: 2e-2 (bf16 inputs) and 1e-4 (fp32) of max(1, ||ref||_inf) per token
and per state.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import assert_state_close, assert_tokens_close, tol_for

pytestmark = pytest.mark.gpu


def _run(inp, flags=0):
    import linear_rnn_delta_b200 as kda
    dev = torch.device("cuda")
    c = lambda t: None if t is None else t.to(dev).contiguous()
    o, sf = kda.kda_chunk_fwd_rank2(inp.variant, inp.gate_range, c(inp.q), c(inp.k), c(inp.v), c(inp.alpha),
                                    c(inp.g1), c(inp.g2), cu_seqlens=c(inp.cu_seqlens),
                                    initial_state=c(inp.initial_state), flags=flags)
    torch.cuda.synchronize()
    return o, sf


def _ref(inp):
    return oracle.recurrence_rank2(inp.variant, inp.q, inp.k, inp.v, inp.alpha, inp.g1, inp.g2,
                                   cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state)


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "standard"),
                                                ("gdn2", "extended")])
def test_rank2_tensor_core_path(variant, gate_range):
    inp = W.make_rank2_inputs(variant, gate_range, "bf16", B=2, T=100, H=2, d_k=128, d_v=128, seed=91,
                              init_state="random", init_std=0.1)
    o, sf = _run(inp)
    o_ref, s_ref = _ref(inp)
    tol = tol_for("bf16")
    assert_tokens_close(o, o_ref, tol)
    assert_state_close(sf, s_ref, tol)


def test_rank2_forms_agree_bitwise_varlen():
    inp = W.make_rank2_inputs("kda", "extended", "bf16", H=2, d_k=128, d_v=128, seed=93,
                              doc_lens=[70, 0, 1, 33], init_state="random", init_std=0.1)
    of, sff = _run(inp, flags=4)
    os_, sfs = _run(inp, flags=8)
    assert torch.equal(of, os_) and torch.equal(sff, sfs)
    o_ref, s_ref = _ref(inp)
    assert_tokens_close(of, o_ref, tol_for("bf16"))
    assert_state_close(sff, s_ref, tol_for("bf16"))


@pytest.mark.parametrize("variant", ["kda", "rda", "gdn2"])
def test_rank2_token_scan_fp32_varlen(variant):
    inp = W.make_rank2_inputs(variant, "extended", "f32", H=3, d_k=64, d_v=32, seed=95,
                              doc_lens=[37, 0, 1, 70], init_state="random", init_std=0.3)
    o, sf = _run(inp)
    o_ref, s_ref = _ref(inp)
    assert_tokens_close(o, o_ref, tol_for("f32"))
    assert_state_close(sf, s_ref, tol_for("f32"))


def test_rank2_reflections_rotate_fp32():
    """Keys in span(e1, e2) at angles a and b, beta = 2, alpha = 1, v = 0: each token turns rows 1-2 of
    the state by 2 (b - a); rows 3..d_k stay bitwise put."""
    import linear_rnn_delta_b200 as kda
    T, dk, dv, a, b = 40, 16, 16, 0.3, 1.0
    dev = torch.device("cuda")
    k = torch.zeros(1, T, 2, 1, dk)
    k[0, :, 0, 0, 0], k[0, :, 0, 0, 1] = math.cos(a), math.sin(a)
    k[0, :, 1, 0, 0], k[0, :, 1, 0, 1] = math.cos(b), math.sin(b)
    s0 = torch.from_numpy(np.random.default_rng(8).standard_normal((1, 1, dk, dv)).astype(np.float32))
    o, sf = kda.kda_chunk_fwd_rank2("kda", "extended", torch.zeros(1, T, 1, dk, device=dev), k.to(dev),
                                    torch.zeros(1, T, 2, 1, dv, device=dev), torch.ones(1, T, 1, dk, device=dev),
                                    torch.full((1, T, 2, 1), 2.0, device=dev), initial_state=s0.to(dev))
    torch.cuda.synchronize()
    phi = 2 * T * (b - a)
    R = np.array([[math.cos(phi), -math.sin(phi)], [math.sin(phi), math.cos(phi)]])
    s = sf.cpu().double().numpy()[0, 0]
    ref = s0.double().numpy()[0, 0]
    np.testing.assert_allclose(s[:2], R @ ref[:2], atol=1e-4 * max(1.0, np.abs(ref).max()))
    assert np.array_equal(s[2:], ref[2:])


def test_rank2_empty_batch_passes_state_through():
    inp = W.make_rank2_inputs("rda", "standard", "bf16", B=2, T=0, H=2, d_k=128, d_v=128, seed=97,
                              init_state="random")
    o, sf = _run(inp)
    assert o.numel() == 0 and torch.equal(sf.cpu(), inp.initial_state)


# ---- gradients of rank-2 steps (kda_chunk_bwd_rank2) --------------------------------------------

GRAD_TOL = 1e-3   # fp32 arithmetic throughout, as for the rank-1 backward


def _grad_close(g, r, what):
    g2 = g.reshape(-1, g.shape[-1]) if g.ndim > 1 else g.reshape(-1, 1)
    r2 = r.reshape(-1, r.shape[-1]) if r.ndim > 1 else r.reshape(-1, 1)
    assert np.all(np.isfinite(g2)), f"{what}: non-finite"
    if g2.size == 0:
        return
    err = np.abs(g2 - r2).max(axis=1)
    scale = np.maximum(1.0, np.abs(r2).max(axis=1))
    worst = int(np.argmax(err / scale))
    assert err[worst] <= GRAD_TOL * scale[worst], \
        f"{what}: row {worst} error {err[worst]:.3e} > {GRAD_TOL} * {scale[worst]:.3e}"


def _rank2_grad_ref(inp, d_o, dsf, n, h):
    """The oracle's reverse mode over the 2T sub-tokens of (sequence n, head h), mapped back."""
    f64 = lambda t: None if t is None else t.double().numpy()
    b, t0, ln = inp.seq_bounds(n)
    s0 = None if inp.initial_state is None else f64(inp.initial_state[n, h])
    if ln == 0:   # an empty sequence hands dL/dS_final straight to its initial state
        return {"ds0": np.zeros((inp.d_k, inp.d_v)) if dsf is None else f64(dsf[n, h])}
    sl = slice(t0, t0 + ln)
    q, al, do = f64(inp.q[b, sl, h]), f64(inp.alpha[b, sl, h]), f64(d_o[b, sl, h])
    def sub(t):   # [B,T,2,H,(d)] -> the sequence's 2 ln sub-tokens of head h
        if t is None:
            return None
        x = f64(t[b, sl, :, h])
        return x.reshape((2 * ln,) + x.shape[2:])
    k2, v2, g12, g22 = sub(inp.k), sub(inp.v), sub(inp.g1), sub(inp.g2)
    q2 = np.stack([np.zeros_like(q), q], axis=1).reshape(2 * ln, -1)
    a2 = np.stack([al, np.ones_like(al)], axis=1).reshape(2 * ln, -1)
    do2 = np.stack([np.zeros_like(do), do], axis=1).reshape(2 * ln, -1)
    g = oracle.recurrence_grad(inp.variant, q2, k2, v2, a2, g12, g22, s0, do2, None if dsf is None else f64(dsf[n, h]))
    pair = lambda x: None if x is None else x.reshape((ln, 2) + x.shape[1:])
    return {"dq": g["dq"][1::2], "dalpha": g["dalpha"][0::2], "dk": pair(g["dk"]), "dv": pair(g["dv"]),
            "dg1": pair(g["dg1"]), "dg2": pair(g["dg2"]), "ds0": g["ds0"]}


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "standard"),
                                                ("gdn2", "extended")])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 32, 64)])
def test_rank2_backward_matches_the_oracle(variant, gate_range, dtype, dk, dv):
    import linear_rnn_delta_b200 as kda
    inp = W.make_rank2_inputs(variant, gate_range, dtype, H=2, d_k=dk, d_v=dv, seed=93, doc_lens=[70, 0, 1, 33],
                              init_state="random", init_std=0.2)
    d_o, dsf = W.grad_outputs(inp, seed=93)
    c = lambda t: None if t is None else t.cuda().contiguous()
    got = kda.kda_chunk_bwd_rank2(inp.variant, inp.gate_range, c(inp.q), c(inp.k), c(inp.v), c(inp.alpha),
                                  c(inp.g1), c(inp.g2), c(d_o), c(dsf), cu_seqlens=c(inp.cu_seqlens),
                                  initial_state=c(inp.initial_state))
    torch.cuda.synchronize()
    names = ("dq", "dk", "dv", "dalpha", "dg1", "dg2", "ds0")
    got = {nm: (None if t is None else t.double().cpu().numpy()) for nm, t in zip(names, got)}
    for n in range(inp.num_seqs):
        b, t0, ln = inp.seq_bounds(n)
        for h in range(inp.H):
            ref = _rank2_grad_ref(inp, d_o, dsf, n, h)
            _grad_close(got["ds0"][n, h], ref["ds0"], f"ds0[{n},{h}]")
            if ln == 0:
                continue
            for nm in ("dq", "dalpha"):
                _grad_close(got[nm][b, t0:t0 + ln, h], ref[nm], f"{nm}[{n},{h}]")
            for nm in ("dk", "dv", "dg1", "dg2"):
                if ref[nm] is not None:
                    _grad_close(got[nm][b, t0:t0 + ln, :, h], ref[nm], f"{nm}[{n},{h}]")


def test_rank2_backward_fixed_length_without_final_gradient():
    import linear_rnn_delta_b200 as kda
    inp = W.make_rank2_inputs("rda", "extended", "bf16", B=2, T=45, H=3, d_k=64, d_v=64, seed=94)
    d_o, _ = W.grad_outputs(inp, seed=94, d_final=False)
    c = lambda t: None if t is None else t.cuda().contiguous()
    got = kda.kda_chunk_bwd_rank2(inp.variant, inp.gate_range, c(inp.q), c(inp.k), c(inp.v), c(inp.alpha),
                                  c(inp.g1), c(inp.g2), c(d_o), None, d_initial_state=False)
    torch.cuda.synchronize()
    assert got[6] is None
    for n in range(inp.B):
        for h in range(inp.H):
            ref = _rank2_grad_ref(inp, d_o, None, n, h)
            _grad_close(got[0][n, :, h].double().cpu().numpy(), ref["dq"], "dq")
            _grad_close(got[3][n, :, h].double().cpu().numpy(), ref["dalpha"], "dalpha")
            _grad_close(got[1][n, :, :, h].double().cpu().numpy(), ref["dk"], "dk")
            _grad_close(got[5][n, :, :, h].double().cpu().numpy(), ref["dg2"], "dg2")
