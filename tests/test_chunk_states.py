"""State snapshots after every 64 tokens (``chunk_states`` of kda_chunk_fwd_ws)
vs the float64 oracle's piecewise runs, on every path that writes them: the
fused and split tensor-core forms and the token scan.  The slot of chunk c of
sequence n is n + floor(first row / 64) + c; the last chunk's snapshot is the
final state itself.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import assert_state_close, cuda_inputs, tol_for

pytestmark = pytest.mark.gpu

FORMS = {"fused": 4, "split": 8, "scan": 2}


def _run(inp, flags):
    import linear_rnn_delta_b200 as kda
    d = cuda_inputs(inp)
    o, sf, cs = kda.kda_chunk_fwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"],
                                  d["g2"], cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"],
                                  chunk_size=inp.chunk_size, flags=flags, chunk_states=True)
    torch.cuda.synchronize()
    return o, sf, cs


def _row0(inp, n):
    b, t0, _ = inp.seq_bounds(n)
    return t0 if inp.cu_seqlens is not None else n * inp.T


@pytest.mark.parametrize("variant,gate_range", [("kda", "extended"), ("rda", "standard"), ("gdn2", "extended")])
@pytest.mark.parametrize("form", ["fused", "split", "scan"])
def test_chunk_states_match_prefix_runs(variant, gate_range, form):
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", H=2, d_k=128, d_v=128, seed=37,
                              doc_lens=[200, 64, 0, 1, 129], init_state="random", init_std=0.2)
    _, sf, cs = _run(inp, FORMS[form])
    ref = oracle.chunk_states(inp)
    tol = tol_for(inp.dtype)
    cs_h = cs.double().cpu().numpy()
    for (n, c), s_ref in ref.items():
        slot = kda.chunk_slot(n, c, _row0(inp, n))
        assert_state_close(cs_h[slot], s_ref, tol, f"state after chunk {c} of sequence {n}")
    for n in range(inp.num_seqs):          # the last chunk's snapshot is the final state, bit for bit
        _, _, ln = inp.seq_bounds(n)
        if ln:
            last = kda.chunk_slot(n, (ln - 1) // 64, _row0(inp, n))
            assert torch.equal(cs[last], sf[n])


def test_chunk_states_fixed_length_and_forms_agree():
    inp = W.make_chunk_inputs("kda", "standard", "bf16", B=3, T=150, H=2, d_k=128, d_v=128, seed=41,
                              init_state="random", init_std=0.1)
    _, _, cf = _run(inp, FORMS["fused"])
    _, _, cs = _run(inp, FORMS["split"])
    import linear_rnn_delta_b200 as kda
    ref = oracle.chunk_states(inp)
    slots = [kda.chunk_slot(n, c, n * inp.T) for (n, c) in ref]
    assert torch.equal(cf[slots], cs[slots])    # both forms, identical bits
    for (n, c), s_ref in ref.items():
        assert_state_close(cf[kda.chunk_slot(n, c, n * inp.T)].double().cpu().numpy(), s_ref, 2e-2)
