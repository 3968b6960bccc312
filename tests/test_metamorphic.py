"""Invariants of the recurrence checked on the GPU path without the oracle's
values: chunked kernel vs the token scan, state continuation, varlen packing
vs separate runs, chunked forward vs repeated decode steps, the exact 2D
rotation embedded in d_k = 128, and run-to-run determinism."""
import math

import numpy as np
import pytest
import torch

import workloads as W
from parity import assert_state_close, assert_tokens_close, cuda_inputs, run_chunk

pytestmark = pytest.mark.gpu
FORCE_SCAN = 2


def _np(x):
    return x.detach().float().cpu().double().numpy()


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "standard"),
                                                ("gdn2", "extended")])
def test_chunked_kernel_matches_token_scan(variant, gate_range):
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", B=2, T=333, H=2, d_k=128, d_v=128, seed=31,
                              init_state="random", init_std=0.2)
    o1, s1 = run_chunk(inp)
    o2, s2 = run_chunk(inp, flags=FORCE_SCAN)
    assert_tokens_close(o1, _np(o2), 2e-2)
    assert_state_close(s1, _np(s2), 2e-2)


def test_state_continuation():
    """[0,T) in one call == [0,t) then [t,T) with the final state fed back."""
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=256, H=2, d_k=128, d_v=128, seed=41,
                              init_state="random", init_std=0.2)
    d = cuda_inputs(inp)
    o, s = kda.kda_chunk_fwd("kda", "extended", d["q"], d["k"], d["v"], d["alpha"], d["g1"], None,
                             initial_state=d["initial_state"])
    t = 128
    sl = lambda x, a, b: x[:, a:b].contiguous()
    oa, sa = kda.kda_chunk_fwd("kda", "extended", *(sl(d[n], 0, t) for n in ("q", "k", "v", "alpha", "g1")), None,
                               initial_state=d["initial_state"])
    ob, sb = kda.kda_chunk_fwd("kda", "extended", *(sl(d[n], t, 256) for n in ("q", "k", "v", "alpha", "g1")), None,
                               initial_state=sa)
    torch.cuda.synchronize()
    assert_tokens_close(torch.cat([oa, ob], dim=1), _np(o), 2e-2)
    assert_state_close(sb, _np(s), 2e-2)


def test_varlen_equals_separate_runs():
    import linear_rnn_delta_b200 as kda
    lens = [100, 64, 7, 190]
    inp = W.make_chunk_inputs("gdn2", "extended", "bf16", H=2, d_k=128, d_v=128, seed=51, doc_lens=lens,
                              init_state="random", init_std=0.2)
    o, s = run_chunk(inp)
    d = cuda_inputs(inp)
    start = 0
    for n, ln in enumerate(lens):
        part = {k: d[k][:, start:start + ln].contiguous() for k in ("q", "k", "v", "alpha", "g1", "g2")}
        on, sn = kda.kda_chunk_fwd("gdn2", "extended", part["q"], part["k"], part["v"], part["alpha"], part["g1"],
                                   part["g2"], initial_state=d["initial_state"][n:n + 1].contiguous())
        torch.cuda.synchronize()
        # identical per-document work: bitwise equal
        assert torch.equal(on, o[:, start:start + ln]), f"doc {n}"
        assert torch.equal(sn[0], s[n])
        start += ln


def test_chunked_forward_equals_decode_steps():
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("rda", "extended", "bf16", B=3, T=70, H=2, d_k=128, d_v=128, seed=61,
                              init_state="random", init_std=0.2)
    o, s = run_chunk(inp)
    d = cuda_inputs(inp)
    state = d["initial_state"].clone()
    outs = []
    for t in range(inp.T):
        outs.append(kda.kda_decode_step("rda", "extended", *(d[n][:, t].contiguous() for n in
                                                             ("q", "k", "v", "alpha", "g1", "g2")), state))
    torch.cuda.synchronize()
    assert_tokens_close(torch.stack(outs, dim=1), _np(o), 2e-2)
    assert_state_close(state, _np(s), 2e-2)


def _rotation_inputs(theta, T, dk, dtype):
    k = torch.zeros(1, T, 1, dk)
    k[..., 0], k[..., 1] = math.cos(theta), math.sin(theta)
    al = torch.ones(1, T, 1, dk)
    al[..., 1] = -1.0
    beta = torch.full((1, T, 1), 2.0)
    z = torch.zeros(1, T, 1, dk)
    s0 = (0.5 * torch.randn(1, 1, dk, dk, generator=torch.Generator().manual_seed(0))).float()
    cast = (lambda x: x.to(torch.bfloat16)) if dtype == "bf16" else (lambda x: x.float())
    return [cast(x).cuda() for x in (z, k, z, al, beta)], s0


@pytest.mark.parametrize("theta", [0.3, 1.1, -2.0])
def test_rotation_closed_form_fp32_d128(theta):
    """Complex-KDA abstract: one delta-rule reflection (beta = 2, unit k) times the
    sign-flip gate alpha = (1, -1, 1, ...) is a 2D rotation.  With k in span(e1, e2)
    and v = 0 the state's rows 1-2 turn by R(T (2 theta + pi)) and rows 3..d_k stay
    put: checked against the closed form at the fp32 tolerance (token scan path)."""
    import linear_rnn_delta_b200 as kda
    T, dk = 40, 128
    (q, k, v, al, beta), s0 = _rotation_inputs(theta, T, dk, "f32")
    o, s = kda.kda_chunk_fwd("kda", "extended", q, k, v, al, beta, None, initial_state=s0.cuda())
    torch.cuda.synchronize()
    s = s.cpu().double()[0, 0]
    phi = T * (2 * theta + math.pi)
    R = torch.tensor([[math.cos(phi), -math.sin(phi)], [math.sin(phi), math.cos(phi)]], dtype=torch.float64)
    ref = s0.double()[0, 0]
    np.testing.assert_allclose(s[:2].numpy(), (R @ ref[:2]).numpy(), atol=1e-4 * max(1.0, float(ref.abs().max())))
    assert torch.equal(s[2:], ref[2:])


@pytest.mark.parametrize("form", ["fused", "split"])
@pytest.mark.parametrize("T", [4, 64, 128, 256])
def test_rotation_tensor_core_path_bf16(T, form):
    """The same construction through the bf16 tensor-core kernel, over one to
    four whole chunks of identical, non-decaying reflections: rows 3..d_k are
    bitwise unchanged (zero key channels, unit gates), and rows 1-2 match the
    oracle within the bf16 tolerance however many chunks the rotation runs."""
    import linear_rnn_delta_b200 as kda
    import oracle
    dk = 128
    (q, k, v, al, beta), s0 = _rotation_inputs(0.3, T, dk, "bf16")
    o, s = kda.kda_chunk_fwd("kda", "extended", q, k, v, al, beta, None, initial_state=s0.cuda(),
                             flags={"fused": 4, "split": 8}[form])
    torch.cuda.synchronize()
    _, s_ref = oracle.recurrence_arrays("kda", q.cpu(), k.cpu(), v.cpu(), al.cpu(), beta.cpu(), None, None, s0)
    assert torch.equal(s.cpu()[0, 0, 2:], s0[0, 0, 2:])
    assert_state_close(s, s_ref, 2e-2)


def test_deterministic():
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=200, H=2, d_k=128, d_v=128, seed=71,
                              init_state="random")
    o1, s1 = run_chunk(inp)
    o2, s2 = run_chunk(inp)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
