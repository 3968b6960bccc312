"""Input preparation inside the kernels (KDA_FLAG_GATE_LOGITS, KDA_FLAG_L2NORM_K)
vs the float64 oracle, which applies the same preparation (``oracle.prepare``:
activations and L2 norm in float64, rounded to the input dtype as a separate
preparation pass would store them) before the recurrence.

Every path that reads inputs is covered: the tensor-core chunked forward in
both forms, the token scan (fp32, and bf16 forced), and the decode step.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import assert_state_close, assert_tokens_close, run_chunk, sampled_pairs, tol_for

pytestmark = pytest.mark.gpu

LOGITS, L2K = 16, 32
FORMS = {"fused": 4, "split": 8, "scan": 2}


def _check(inp, flags):
    o, sf = run_chunk(inp, flags=flags)
    o_ref, s_ref = oracle.recurrence(inp)
    tol = tol_for(inp.dtype)
    assert_tokens_close(o, o_ref, tol)
    assert_state_close(sf, s_ref, tol)


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "standard"),
                                                ("rda", "extended"), ("gdn2", "standard"), ("gdn2", "extended")])
@pytest.mark.parametrize("form", ["fused", "split", "scan"])
def test_chunk_logits_and_raw_keys_bf16(variant, gate_range, form):
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", H=3, d_k=128, d_v=128, seed=17,
                              doc_lens=[150, 64, 1, 0, 97], init_state="random", init_std=0.2,
                              logits=True, raw_k=True)
    _check(inp, LOGITS | L2K | FORMS[form])


@pytest.mark.parametrize("logits,raw_k", [(True, False), (False, True)])
@pytest.mark.parametrize("form", ["fused", "split"])
def test_chunk_each_preparation_alone(logits, raw_k, form):
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=205, H=2, d_k=128, d_v=128, seed=19,
                              init_state="random", init_std=0.2, logits=logits, raw_k=raw_k)
    _check(inp, (LOGITS if logits else 0) | (L2K if raw_k else 0) | FORMS[form])


@pytest.mark.parametrize("variant", ["kda", "gdn2"])
def test_chunk_preparation_fp32_scan(variant):
    inp = W.make_chunk_inputs(variant, "extended", "f32", B=2, T=77, H=2, d_k=64, d_v=32, seed=23,
                              init_state="random", init_std=0.3, logits=True, raw_k=True)
    _check(inp, LOGITS | L2K)


def test_chunk_preparation_forms_agree_bitwise():
    inp = W.make_chunk_inputs("rda", "extended", "bf16", H=2, d_k=128, d_v=128, seed=29,
                              doc_lens=[300, 65, 2], logits=True, raw_k=True)
    of, sff = run_chunk(inp, flags=LOGITS | L2K | FORMS["fused"])
    os_, sfs = run_chunk(inp, flags=LOGITS | L2K | FORMS["split"])
    assert torch.equal(of, os_) and torch.equal(sff, sfs)


@pytest.mark.parametrize("variant,gate_range", [("kda", "extended"), ("rda", "standard"), ("gdn2", "extended")])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_logits_and_raw_keys(variant, gate_range, dtype):
    import linear_rnn_delta_b200 as kda
    N, H, dk, dv, steps = 4, 3, 128, 128, 12
    state0 = W.decode_initial_state(N, H, dk, dv, seed=7, std=0.3)
    state = state0.cuda()
    names = ("q", "k", "v", "alpha", "g1", "g2")
    kept = {nm: [] for nm in names}
    outs = []
    for s in range(steps):
        st = W.decode_step_inputs(s, variant, gate_range, dtype, N, H, dk, dv, seed=7, logits=True, raw_k=True)
        d = [None if getattr(st, nm) is None else getattr(st, nm).cuda() for nm in names]
        outs.append(kda.kda_decode_step(variant, gate_range, *d, state, flags=LOGITS | L2K).float().cpu())
        for nm in names:
            t = getattr(st, nm)
            if t is not None:
                kept[nm].append(t.reshape(N * H, *t.shape[2:]).double())
    torch.cuda.synchronize()
    arr = {nm: (torch.stack(v, dim=1).unsqueeze(2).numpy() if v else None) for nm, v in kept.items()}
    o_ref, s_ref = oracle.recurrence_arrays(variant, arr["q"], arr["k"], arr["v"], arr["alpha"], arr["g1"],
                                            arr["g2"], None, state0.reshape(N * H, dk, dv).double().numpy()[:, None],
                                            gate_range=gate_range, logits=True, l2norm_k=True, round_to=dtype)
    o_gpu = torch.stack(outs, dim=2).reshape(N * H, steps, dv).double().numpy()
    tol = tol_for(dtype)
    assert_tokens_close(o_gpu, o_ref[:, :, 0], tol, "decode o")
    assert_state_close(state.reshape(N * H, dk, dv).double().cpu().numpy(), s_ref[:, 0], tol, "decode state")
