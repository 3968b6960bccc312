"""The chunked kernel's division-free (anchored) branch, forced by planted gates.

A chunk whose gates all satisfy |alpha| <= 1 and whose per-channel chunk
products stay at or above 2^-110 takes the fast branch (one tensor-core GEMM
for A and P, one division by the chunk product).  Every other chunk -- an
exact zero gate, a run of tiny gates whose product underflows, a gate above 1
-- takes the anchored branch, which forms the decay products forward from
anchors and never divides ("Complex KDA" arXiv abstract: gates in [-1, 1],
so zeros and sign changes are part of the method's range).  Random draws
from the benchmark recipes almost never reach it, so these tests plant such
gates (``workloads.plant_gates``) and compare the tensor-core path with the
float64 oracle element by element, for every variant and gate range, both
forms of the tensor-core path, packed documents with ragged tails and
fixed-length batches.  A white-box check reads the split form's workspace to
confirm that the planted chunks really took the anchored branch.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import assert_state_close, assert_tokens_close, cuda_inputs, run_chunk

pytestmark = pytest.mark.gpu

FORMS = {"fused": 4, "split": 8}
COMBOS = [("kda", "standard"), ("kda", "extended"), ("rda", "standard"), ("rda", "extended"),
          ("gdn2", "standard"), ("gdn2", "extended")]
DOCS = [200, 64, 1, 0, 130, 77]   # ragged tails, a one-token and an empty document


def _check(inp, flags):
    o, sf = run_chunk(inp, flags=flags)
    o_ref, s_ref = oracle.recurrence(inp)
    assert_tokens_close(o, o_ref, 2e-2)
    assert_state_close(sf, s_ref, 2e-2)


@pytest.mark.parametrize("kind", W.PLANT_KINDS)
@pytest.mark.parametrize("variant,gate_range", COMBOS)
@pytest.mark.parametrize("form", ["fused", "split"])
def test_planted_gates_packed_documents(kind, variant, gate_range, form):
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", H=2, d_k=128, d_v=128, seed=101, doc_lens=DOCS,
                              init_state="random", init_std=0.2)
    _check(W.plant_gates(inp, kind, seed=7), FORMS[form])


@pytest.mark.parametrize("kind", W.PLANT_KINDS)
@pytest.mark.parametrize("variant,gate_range", [("kda", "extended"), ("rda", "standard"), ("gdn2", "extended")])
@pytest.mark.parametrize("form", ["fused", "split"])
def test_planted_gates_fixed_length(kind, variant, gate_range, form):
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", B=2, T=3 * 64 + 13, H=3, d_k=128, d_v=128, seed=102,
                              init_state="random", init_std=0.2)
    _check(W.plant_gates(inp, kind, seed=8), FORMS[form])


def test_all_gates_zero_erase_the_state():
    """alpha = 0 everywhere: S_t = k_t m_t^T after every token, whatever came before
    (the oracle pins the same identity); the kernel must give it chunk after chunk."""
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=1, T=150, H=2, d_k=128, d_v=128, seed=103,
                              init_state="random", init_std=0.5)
    inp.alpha = torch.zeros_like(inp.alpha)
    for form in ("fused", "split"):
        _check(inp, FORMS[form])


# ---- which branch ran: the split form's slot status words ---------------------------------------

SLOT_BYTES = 82944             # bytes of one (chunk slot, head) operand image in the split workspace
META_STATUS = 65536 + 512      # int status word: bit 0 fast branch, bit 1 slot complete
META_FAST, META_OK = 1, 2


def _split_statuses(inp):
    """Run the split form through kda_chunk_fwd_ws with a workspace of our own and
    return {(n, h, c): status word} for every chunk."""
    import linear_rnn_delta_b200 as kda
    d = cuda_inputs(inp)
    N, H = inp.num_seqs, inp.H
    ws_bytes = kda.lib.kda_chunk_fwd_workspace_size(0, inp.B, inp.T, H, 128, 128, int(inp.cu_seqlens is not None),
                                                    N, 64, FORMS["split"])
    assert ws_bytes > 0
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    o = torch.empty((inp.B, inp.T, H, 128), dtype=torch.bfloat16, device="cuda")
    sf = torch.empty((N, H, 128, 128), dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = kda.lib.kda_chunk_fwd_ws(kda.VARIANTS[inp.variant], kda.RANGES[inp.gate_range], 0, inp.B, inp.T, H, 128,
                                  128, p(d["q"]), p(d["k"]), p(d["v"]), p(d["alpha"]), p(d["g1"]), p(d["g2"]),
                                  p(d["cu_seqlens"]), N, p(d["initial_state"]), p(sf), None, p(o), 64, p(ws),
                                  ws_bytes, FORMS["split"], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, kda.lib.kda_last_error_detail()
    torch.cuda.synchronize()
    words = ws.view(-1, SLOT_BYTES)[:, META_STATUS:META_STATUS + 4].contiguous().view(torch.int32).cpu()
    out = {}
    for n in range(N):
        b, t0, ln = inp.seq_bounds(n)
        row0 = b * inp.T + t0
        for c in range((ln + 63) // 64):
            slot = kda.chunk_slot(n, c, row0)
            for h in range(H):
                out[(n, h, c)] = int(words[slot * H + h])
    return out, (o, sf)


def _min_log2_chunk_product(inp, n, h, c):
    b, t0, ln = inp.seq_bounds(n)
    a = inp.alpha[b, t0 + 64 * c:t0 + min(64 * c + 64, ln), h].double().numpy()
    if np.abs(a).max() > 1:
        return -np.inf
    with np.errstate(divide="ignore"):
        return float(np.log2(np.abs(a).prod(axis=0)).min())


@pytest.mark.parametrize("kind", W.PLANT_KINDS)
def test_planted_chunks_take_the_anchored_branch(kind):
    inp = W.make_chunk_inputs("kda", "standard", "bf16", H=2, d_k=128, d_v=128, seed=104, doc_lens=DOCS,
                              init_state="random", init_std=0.2)
    planted = W.plant_gates(inp, kind, seed=9)
    status, (o, sf) = _split_statuses(planted)
    n_anchored = n_fast = 0
    for (n, h, c), word in status.items():
        assert word & META_OK, f"slot of chunk {(n, h, c)} not completed"
        lg = _min_log2_chunk_product(planted, n, h, c)
        if lg < -110:
            assert not word & META_FAST, f"chunk {(n, h, c)}: product 2^{lg:.1f} but the fast branch ran"
            n_anchored += 1
        elif lg > -100:
            assert word & META_FAST, f"chunk {(n, h, c)}: product 2^{lg:.1f} but the anchored branch ran"
            n_fast += 1
    assert n_anchored > 0
    if kind == "mixed":
        assert n_fast > 0
    o_ref, s_ref = oracle.recurrence(planted)
    assert_tokens_close(o, o_ref, 2e-2)
    assert_state_close(sf, s_ref, 2e-2)
