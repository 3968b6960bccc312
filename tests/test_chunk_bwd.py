"""Backward pass (kda_chunk_bwd) vs the float64 oracle's reverse mode
(``oracle.recurrence_grad``, itself pinned by central differences).

The backward computes in fp32 throughout (bf16 inputs are widened exactly), so
one tolerance serves both input dtypes: per token and per gradient tensor,
max |g_gpu - g_ref| <= 1e-3 * max(1, ||g_ref[t]||_inf).  fp32 rounding (unit
6e-8) accumulated over a few hundred steps of d-term sums stays orders of
magnitude below that; a dropped term, a wrong sign or a wrong index moves the
result by O(1).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import cuda_inputs

pytestmark = pytest.mark.gpu

GRAD_TOL = 1e-3


def _bwd(inp, d_o, dsf, want_ds0=True):
    import linear_rnn_delta_b200 as kda
    d = cuda_inputs(inp)
    out = kda.kda_chunk_bwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                            d_o.cuda(), None if dsf is None else dsf.cuda(), cu_seqlens=d["cu_seqlens"],
                            initial_state=d["initial_state"], d_initial_state=want_ds0)
    torch.cuda.synchronize()
    names = ("dq", "dk", "dv", "dalpha", "dg1", "dg2", "ds0")
    return {n: (None if t is None else t.double().cpu().numpy()) for n, t in zip(names, out)}


def _close(g, r, what):
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


def _check(inp, got, d_o, dsf):
    f64 = lambda t: None if t is None else t.double().numpy()
    for n in range(inp.num_seqs):
        b, t0, ln = inp.seq_bounds(n)
        sl = slice(t0, t0 + ln)
        for h in range(inp.H):
            pick = lambda t: None if t is None else f64(t[b, sl, h])
            s0 = None if inp.initial_state is None else f64(inp.initial_state[n, h])
            ref = oracle.recurrence_grad(inp.variant, pick(inp.q), pick(inp.k), pick(inp.v), pick(inp.alpha),
                                         pick(inp.g1), pick(inp.g2), s0, pick(d_o),
                                         None if dsf is None else f64(dsf[n, h]))
            for name in ("dq", "dk", "dv", "dalpha", "dg1", "dg2"):
                if ref[name] is None:
                    assert got[name] is None
                    continue
                _close(got[name][b, sl, h], ref[name], f"{name} seq {n} head {h}")
            if got["ds0"] is not None:
                _close(got["ds0"][n, h], ref["ds0"], f"ds0 seq {n} head {h}")


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "standard"),
                                                ("rda", "extended"), ("gdn2", "standard"), ("gdn2", "extended")])
def test_bwd_fixed_length_bf16_d128(variant, gate_range):
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", B=2, T=150, H=2, d_k=128, d_v=128, seed=61,
                              init_state="random", init_std=0.2)
    d_o, dsf = W.grad_outputs(inp, seed=61)
    _check(inp, _bwd(inp, d_o, dsf), d_o, dsf)


@pytest.mark.parametrize("variant", ["kda", "rda", "gdn2"])
def test_bwd_varlen_f32_small_heads(variant):
    inp = W.make_chunk_inputs(variant, "extended", "f32", H=3, d_k=64, d_v=32, seed=67,
                              doc_lens=[70, 0, 1, 129, 64], init_state="random", init_std=0.3)
    d_o, dsf = W.grad_outputs(inp, seed=67)
    _check(inp, _bwd(inp, d_o, dsf), d_o, dsf)


@pytest.mark.parametrize("dk,dv", [(16, 128), (128, 16), (32, 64), (64, 64)])
def test_bwd_head_dims_no_initial_state(dk, dv):
    inp = W.make_chunk_inputs("gdn2", "standard", "f32", B=1, T=97, H=2, d_k=dk, d_v=dv, seed=71)
    d_o, _ = W.grad_outputs(inp, seed=71, d_final=False)
    _check(inp, _bwd(inp, d_o, None), d_o, None)


@pytest.mark.parametrize("dk", [16, 32, 64, 128])
@pytest.mark.parametrize("dv", [16, 32, 64, 128])
def test_bwd_every_head_size(dk, dv):
    """Every (d_k, d_v): the checkpoint scan's states-only variant in each lane-group shape, and both
    adjoint kernels (shared-memory at d_k = 16, cluster rows otherwise), over three checkpointed chunks
    of packed documents."""
    inp = W.make_chunk_inputs("kda", "extended", "f32", H=1, d_k=dk, d_v=dv, seed=90 + dk + dv,
                              doc_lens=[130, 0, 21], init_state="random", init_std=0.2)
    d_o, dsf = W.grad_outputs(inp, seed=90 + dk + dv)
    _check(inp, _bwd(inp, d_o, dsf), d_o, dsf)


def test_bwd_long_sequence_one_head():
    """1024 tokens (16 checkpointed chunks) on the KDA gates at d = 128."""
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=1, T=1024, H=1, d_k=128, d_v=128, seed=73,
                              init_state="random", init_std=0.1)
    d_o, dsf = W.grad_outputs(inp, seed=73)
    _check(inp, _bwd(inp, d_o, dsf), d_o, dsf)


def test_bwd_empty_sequence_passes_final_gradient_through():
    inp = W.make_chunk_inputs("rda", "standard", "bf16", B=2, T=0, H=2, d_k=128, d_v=128, seed=79,
                              init_state="random")
    d_o, dsf = W.grad_outputs(inp, seed=79)
    got = _bwd(inp, d_o, dsf)
    assert np.array_equal(got["ds0"], dsf.double().numpy())   # S_T = S_0: dL/dS_0 = dL/dS_T exactly
    assert got["dq"].size == 0


def test_autograd_function_matches_direct_call():
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("gdn2", "extended", "f32", B=2, T=80, H=2, d_k=32, d_v=32, seed=83,
                              init_state="random", init_std=0.2)
    d_o, dsf = W.grad_outputs(inp, seed=83)
    d = cuda_inputs(inp)
    leaves = {n: d[n].clone().requires_grad_(True) for n in ("q", "k", "v", "alpha", "g1", "g2", "initial_state")}
    o, sf = kda.KdaChunkFunction.apply(inp.variant, inp.gate_range, leaves["q"], leaves["k"], leaves["v"],
                                       leaves["alpha"], leaves["g1"], leaves["g2"], None, leaves["initial_state"])
    ((o * d_o.cuda()).sum() + (sf * dsf.cuda()).sum()).backward()
    direct = kda.kda_chunk_bwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                               d_o.cuda(), dsf.cuda(), initial_state=d["initial_state"])
    for name, ref in zip(("q", "k", "v", "alpha", "g1", "g2", "initial_state"), direct):
        assert torch.equal(leaves[name].grad, ref), name


def test_bwd_rejects_flags_and_small_workspace():
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("kda", "standard", "bf16", B=1, T=64, H=1, d_k=128, d_v=128, seed=89)
    d = cuda_inputs(inp)
    d_o = W.grad_outputs(inp)[0].cuda()
    g = [torch.empty(t.shape, dtype=torch.float32, device="cuda") for t in (d["q"], d["k"], d["v"], d["alpha"],
                                                                          d["g1"])]
    need = kda.lib.kda_chunk_bwd_workspace_size(0, 1, 64, 1, 128, 128, 0, 1)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    P = lambda t: None if t is None else t.data_ptr()
    args = [0, 0, 0, 1, 64, 1, 128, 128, P(d["q"]), P(d["k"]), P(d["v"]), P(d["alpha"]), P(d["g1"]), None, None,
            1, None, P(d_o), None] + [P(x) for x in g] + [None, None]
    assert kda.lib.kda_chunk_bwd(*args, P(ws), need - 16, 0, None) != 0       # workspace too small
    assert kda.lib.kda_chunk_bwd(*args, P(ws), need, 1 << 4, None) != 0       # flags not taken
    assert kda.lib.kda_chunk_bwd(*args, P(ws), need, 0, None) == 0
    torch.cuda.synchronize()
