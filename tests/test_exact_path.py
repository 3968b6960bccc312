"""The chunked kernel's exact path for ill-conditioned chunks.

Runs of strong, barely decaying reflections on correlated keys -- the
dynamics the Complex KDA abstract builds its expressivity on (beta near 2,
|alpha| near 1: a reflection times a sign-flipping gate is a 2D rotation) --
make the UT transform T = (I + A)^-1 of a chunk large, and the bf16 rounding
of the WY operands then cancels badly in K^T T (.); aligned keys with erase
gates near 1 make A itself large, and the readout sums many nearly cancelling
terms.  The preparation step measures the largest row sums of |T| (weighted
by the gates) and of |A|; above fixed bounds the chain computes that chunk
token by token in fp32 instead.  These tests
plant such chunks (``workloads.plant_reflections``) next to ordinary ones and
compare with the float64 oracle element by element on every variant, both
gate ranges, both forms, packed documents, input preparation and state
snapshots; a white-box check reads the split form's slot status words to
confirm which chunks took the exact path.
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
DOCS = [200, 64, 1, 0, 130, 77]


def _check(inp, flags):
    o, sf = run_chunk(inp, flags=flags)
    o_ref, s_ref = oracle.recurrence(inp)
    assert_tokens_close(o, o_ref, 2e-2)
    assert_state_close(sf, s_ref, 2e-2)


@pytest.mark.parametrize("variant,gate_range", [("kda", "extended"), ("kda", "standard"), ("rda", "extended"),
                                                ("rda", "standard"), ("gdn2", "extended"), ("gdn2", "standard")])
@pytest.mark.parametrize("form", ["fused", "split"])
def test_reflection_runs_packed_documents(variant, gate_range, form):
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", H=2, d_k=128, d_v=128, seed=201, doc_lens=DOCS,
                              init_state="random", init_std=0.3)
    _check(W.plant_reflections(inp, seed=1), FORMS[form])


@pytest.mark.parametrize("form", ["fused", "split"])
@pytest.mark.parametrize("every", [1, 3])
def test_reflection_runs_fixed_length(form, every):
    """Every chunk exact (every = 1), or one in three, over 5 chunks and a tail."""
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=5 * 64 + 21, H=3, d_k=128, d_v=128, seed=202,
                              init_state="random", init_std=0.3)
    _check(W.plant_reflections(inp, seed=2, every=every), FORMS[form])


@pytest.mark.parametrize("form", ["fused", "split"])
def test_reflection_runs_from_logits_and_raw_keys(form):
    """The exact path applies the same input preparation as the tensor-core path."""
    for variant in ("kda", "gdn2"):
        inp = W.make_chunk_inputs(variant, "extended", "bf16", H=2, d_k=128, d_v=128, seed=203, doc_lens=[150, 70],
                                  init_state="random", init_std=0.3, logits=True, raw_k=True)
        inp = W.plant_reflections(inp, seed=3)
        _check(inp, FORMS[form] | 16 | 32)


@pytest.mark.parametrize("form", ["fused", "split"])
def test_reflection_runs_state_snapshots(form):
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("rda", "extended", "bf16", H=2, d_k=128, d_v=128, seed=204, doc_lens=[190, 64, 3],
                              init_state="random", init_std=0.3)
    inp = W.plant_reflections(inp, seed=4)
    d = cuda_inputs(inp)
    o, sf, cs = kda.kda_chunk_fwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                                  cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"],
                                  flags=FORMS[form], chunk_states=True)
    torch.cuda.synchronize()
    snaps = oracle.chunk_states(inp)
    for (n, c), ref in snaps.items():
        b, t0, _ = inp.seq_bounds(n)
        slot = kda.chunk_slot(n, c, b * inp.T + t0)
        assert_state_close(cs[slot], ref, 2e-2, f"snapshot of sequence {n}, chunk {c}")


# ---- which chunks took the exact path -----------------------------------------------------------

SLOT_BYTES = 82944
META_STATUS = 65536 + 512
META_EXACT = 4


def _norms(inp, n, c, h):
    """Largest row sums of |T_{r,s}| max(|e_s|, |w_s|) (T = (I + A)^-1) and of |A_{r,s}|, in float64."""
    b, t0, ln = inp.seq_bounds(n)
    s, e = t0 + 64 * c, t0 + min(ln, 64 * c + 64)
    f = lambda x: x[b, s:e, h].double().numpy()
    k, al = f(inp.k), f(inp.alpha)
    L = e - s
    if inp.variant == "gdn2":
        eg = wg = np.ones(L)
        bv = f(inp.g1)
    else:
        eg = f(inp.g1)
        wg = eg if inp.variant == "kda" else f(inp.g2)
        bv = np.ones_like(k)
    A = np.zeros((L, L))
    for r in range(L):
        lam = np.ones(k.shape[1])
        for s2 in range(r - 1, -1, -1):
            lam = lam * al[s2 + 1]
            A[r, s2] = eg[r] * np.dot(bv[r] * k[r] * lam, k[s2])
    T = np.linalg.inv(np.eye(L) + A)
    return (float((np.abs(T) * np.maximum(np.abs(eg), np.abs(wg))[None, :]).sum(1).max()),
            float(np.abs(A).sum(1).max()))


@pytest.mark.parametrize("gate_range", ["extended", "standard"])
def test_planted_chunks_take_the_exact_path(gate_range):
    """Chunks well past either bound (|T| row sums 6, |A| row sums 3) are run
    exactly; chunks well under both stay on the tensor cores."""
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("kda", gate_range, "bf16", H=2, d_k=128, d_v=128, seed=205, doc_lens=DOCS,
                              init_state="random", init_std=0.3)
    inp = W.plant_reflections(inp, seed=5)
    d = cuda_inputs(inp)
    N, H = inp.num_seqs, inp.H
    ws_bytes = kda.lib.kda_chunk_fwd_workspace_size(0, inp.B, inp.T, H, 128, 128, 1, N, 64, FORMS["split"])
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    o = torch.empty((inp.B, inp.T, H, 128), dtype=torch.bfloat16, device="cuda")
    sf = torch.empty((N, H, 128, 128), dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = kda.lib.kda_chunk_fwd_ws(0, kda.RANGES[gate_range], 0, inp.B, inp.T, H, 128, 128, p(d["q"]), p(d["k"]),
                                  p(d["v"]), p(d["alpha"]), p(d["g1"]), None, p(d["cu_seqlens"]), N,
                                  p(d["initial_state"]), p(sf), None, p(o), 64, p(ws), ws_bytes, FORMS["split"],
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, kda.lib.kda_last_error_detail()
    torch.cuda.synchronize()
    words = ws.view(-1, SLOT_BYTES)[:, META_STATUS:META_STATUS + 4].contiguous().view(torch.int32).cpu()
    n_exact = n_tc = 0
    for n in range(N):
        b, t0, ln = inp.seq_bounds(n)
        for c in range((ln + 63) // 64):
            for h in range(H):
                word = int(words[kda.chunk_slot(n, c, t0) * H + h])
                tn, an = _norms(inp, n, c, h)
                if tn > 8 or an > 4.5:
                    assert word & META_EXACT, f"chunk {(n, c, h)}: norms {tn:.1f}, {an:.1f}; tensor cores ran it"
                    n_exact += 1
                elif tn < 4 and an < 2:
                    assert not word & META_EXACT, f"chunk {(n, c, h)}: norms {tn:.1f}, {an:.1f}; exact path ran"
                    n_tc += 1
    assert n_exact > 0 and n_tc > 0
    o_ref, s_ref = oracle.recurrence(inp)
    assert_tokens_close(o, o_ref, 2e-2)
    assert_state_close(sf, s_ref, 2e-2)


def test_benchmark_recipe_never_takes_the_exact_path():
    """Random Complex-KDA chunks (the largest benchmark workload's recipe) stay on the tensor cores."""
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=1024, H=4, d_k=128, d_v=128, seed=206)
    d = cuda_inputs(inp)
    ws_bytes = kda.lib.kda_chunk_fwd_workspace_size(0, 2, 1024, 4, 128, 128, 0, 2, 64, FORMS["split"])
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    o = torch.empty((2, 1024, 4, 128), dtype=torch.bfloat16, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = kda.lib.kda_chunk_fwd_ws(0, 1, 0, 2, 1024, 4, 128, 128, p(d["q"]), p(d["k"]), p(d["v"]), p(d["alpha"]),
                                  p(d["g1"]), None, None, 2, None, None, None, p(o), 64, p(ws), ws_bytes,
                                  FORMS["split"], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    words = ws.view(-1, SLOT_BYTES)[:, META_STATUS:META_STATUS + 4].contiguous().view(torch.int32).cpu()
    used = [int(words[kda.chunk_slot(n, c, n * 1024) * 4 + h]) for n in range(2) for c in range(16) for h in range(4)]
    assert all(w & 2 for w in used)
    assert not any(w & META_EXACT for w in used)
