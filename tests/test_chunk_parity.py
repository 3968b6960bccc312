"""Chunked forward (kda_chunk_fwd) vs the float64 CPU oracle, element by element.

Small cases span several 64-token chunks and a ragged tail; the full-size
workloads (KDA 4x16x4096, Complex KDA 8x16x8192, RDA/GDN-2 varlen with 16
documents) run in the same launch configuration the benchmark times and are
checked on a seeded sample of (sequence, head) pairs over their full length.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import (assert_state_close, assert_tokens_close, check_sampled, run_chunk, sampled_pairs,
                    tol_for)

pytestmark = pytest.mark.gpu

FORCE_SCAN = 2
# the two forms of the tensor-core path (bf16, d = 128, chunk 64)
FORMS = {"fused": 4, "split": 8}


def _full_check(inp, flags=0):
    o, sf = run_chunk(inp, flags=flags)
    o_ref, s_ref = oracle.recurrence(inp)
    tol = tol_for(inp.dtype)
    eo = assert_tokens_close(o, o_ref, tol)
    es = assert_state_close(sf, s_ref, tol)
    return eo, es


def test_tiny_complex_kda_fp32():
    """B=1, H=2, T=64, d=16, chunk 16, alpha ~ U[-1,1], beta ~ U[0,2], fp32: 1e-4."""
    _full_check(W.tiny_ckda(0))


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "standard"),
                                                ("rda", "extended"), ("gdn2", "standard"), ("gdn2", "extended")])
@pytest.mark.parametrize("dtype,form", [("bf16", "fused"), ("bf16", "split"), ("f32", "fused")])
@pytest.mark.parametrize("init", ["zero", "random"])
def test_fixed_length_d128(variant, gate_range, dtype, form, init):
    """Several chunks plus a ragged tail (T = 3*64 + 13) at d = 128."""
    inp = W.make_chunk_inputs(variant, gate_range, dtype, B=2, T=205, H=3, d_k=128, d_v=128, seed=5,
                              init_state=init, chunk_size=64)
    _full_check(inp, FORMS[form])


@pytest.mark.parametrize("variant", ["kda", "rda", "gdn2"])
@pytest.mark.parametrize("dtype,form", [("bf16", "fused"), ("bf16", "split"), ("f32", "fused")])
def test_varlen_d128(variant, dtype, form):
    """Packed documents: shorter than a chunk, exactly a chunk, chunk +- 1, empty, long."""
    lens = [5, 64, 63, 65, 0, 1, 200, 128, 17]
    inp = W.make_chunk_inputs(variant, "extended", dtype, H=2, d_k=128, d_v=128, seed=9, doc_lens=lens,
                              init_state="random", init_std=0.3)
    _full_check(inp, FORMS[form])


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 16), (16, 128), (64, 64)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_other_head_dims(dk, dv, dtype):
    inp = W.make_chunk_inputs("gdn2", "extended", dtype, B=2, T=77, H=2, d_k=dk, d_v=dv, seed=13,
                              init_state="random", chunk_size=32)
    _full_check(inp)


@pytest.mark.parametrize("dk", [16, 32, 64, 128])
@pytest.mark.parametrize("dv", [16, 32, 64, 128])
def test_token_scan_every_head_size(dk, dv):
    """Every (d_k, d_v) the token scan is instantiated for (its lane groups take 4, 8 or 16 lanes and 2
    or 4 value columns, one or two CTAs per head), packed documents with a ragged tail, at 1e-4."""
    inp = W.make_chunk_inputs("rda", "extended", "f32", H=2, d_k=dk, d_v=dv, seed=14 + dk + dv,
                              doc_lens=[37, 0, 70], init_state="random", init_std=0.3)
    _full_check(inp, FORCE_SCAN)


@pytest.mark.parametrize("form", ["fused", "split"])
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 129])
def test_awkward_lengths_bf16(T, form):
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=1, T=T, H=2, d_k=128, d_v=128, seed=T,
                              init_state="random", init_std=0.1)
    _full_check(inp, FORMS[form])


@pytest.mark.parametrize("form", ["fused", "split"])
def test_empty_sequence_passes_state_through(form):
    """T = 0: nothing to read or write except final_state = initial_state."""
    inp = W.make_chunk_inputs("rda", "standard", "bf16", B=2, T=0, H=2, d_k=128, d_v=128, seed=1,
                              init_state="random")
    o, sf = run_chunk(inp, flags=FORMS[form])
    assert o.numel() == 0
    assert torch.equal(sf.cpu(), inp.initial_state)


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "extended"),
                                                ("gdn2", "extended")])
def test_split_and_fused_forms_agree_bitwise(variant, gate_range):
    """Both forms run the same arithmetic in the same order: identical bits, varlen and ragged."""
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", H=3, d_k=128, d_v=128, seed=31,
                              doc_lens=[300, 1, 64, 0, 129, 77], init_state="random", init_std=0.2)
    of, sff = run_chunk(inp, flags=FORMS["fused"])
    os_, sfs = run_chunk(inp, flags=FORMS["split"])
    assert torch.equal(of, os_)
    assert torch.equal(sff, sfs)


@pytest.mark.parametrize("form", ["fused", "split"])
def test_final_state_may_alias_initial_state(form):
    import linear_rnn_delta_b200 as kda
    from parity import cuda_inputs
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=150, H=2, d_k=128, d_v=128, seed=3,
                              init_state="random")
    d = cuda_inputs(inp)
    s = d["initial_state"].clone()
    o, sf = kda.kda_chunk_fwd("kda", "extended", d["q"], d["k"], d["v"], d["alpha"], d["g1"], None,
                              initial_state=s, final_state=s, flags=FORMS[form])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.recurrence(inp)
    assert_tokens_close(o, o_ref, 2e-2)
    assert_state_close(s, s_ref, 2e-2)


def test_scan_path_matches_oracle_bf16_d128():
    """The token-by-token CUDA scan on the shape the tensor-core kernel serves."""
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=130, H=2, d_k=128, d_v=128, seed=21,
                              init_state="random")
    o, sf = run_chunk(inp, flags=FORCE_SCAN)
    o_ref, s_ref = oracle.recurrence(inp)
    assert_tokens_close(o, o_ref, 2e-2)
    assert_state_close(sf, s_ref, 2e-2)


# ---- full-size workloads, sampled (sequence, head) pairs -----------------------------------

@pytest.mark.slow
@pytest.mark.parametrize("form", ["fused", "split"])
def test_full_kda_bf16_4x16x4096_sampled(form):
    inp = W.kda_bf16(0)
    o, sf = run_chunk(inp, flags=FORMS[form])
    check_sampled(inp, o, sf, sampled_pairs(inp.num_seqs, inp.H, 12), 2e-2)


@pytest.mark.slow
def test_full_complex_kda_bf16_8x16x8192_sampled():
    inp = W.ckda_bf16(0)
    o, sf = run_chunk(inp)
    check_sampled(inp, o, sf, sampled_pairs(inp.num_seqs, inp.H, 10), 2e-2)


@pytest.mark.slow
@pytest.mark.parametrize("variant", ["rda", "gdn2"])
def test_full_varlen_16_docs_sampled(variant):
    inp = W.varlen_bf16(variant, 0)
    o, sf = run_chunk(inp)
    check_sampled(inp, o, sf, sampled_pairs(inp.num_seqs, inp.H, 12), 2e-2)
