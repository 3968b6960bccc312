"""kda_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate
device memory at call time (an engine that owns all of HBM through its own
allocator, a fixed device-memory budget, a loop that cannot take cudaMalloc's
latency or synchronisation).  Its workspace is a fixed 64 MiB array inside the
library.  It runs the split form of the tensor-core path, so its results must
equal, bit for bit, those of the allocating entry point forced to the split
form, on two calls in a row over different slot layouts of the same array (any
leftover of the first call read by the second would change bits); both are
also checked against the float64 oracle.

This file is collected last on purpose: a failure here comes after every other
test has run.
"""
import ctypes
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads as W  # noqa: E402

_vp, _i = ctypes.c_void_p, ctypes.c_int
OK, INVALID, UNSUPPORTED = 0, 1, 2
SCRATCH_SLOT_HEADS = (64 << 20) // 82944   # (chunk slot, head) pairs the fixed array holds


def _lib():
    import linear_rnn_delta_b200 as kda
    lib = kda.lib
    lib.kda_chunk_fwd_noalloc.restype = _i
    lib.kda_chunk_fwd_noalloc.argtypes = [_i] * 8 + [_vp] * 6 + [_vp, _i, _vp, _vp, _vp, ctypes.c_uint, _vp]
    return lib


def _noalloc(lib, inp, d, o, sf, stream):
    var = {"kda": 0, "rda": 1, "gdn2": 2}[inp.variant]
    rng = {"standard": 0, "extended": 1}[inp.gate_range]
    p = lambda t: None if t is None else t.data_ptr()
    return lib.kda_chunk_fwd_noalloc(var, rng, 0, inp.B, inp.T, inp.H, inp.d_k, inp.d_v, p(d["q"]), p(d["k"]),
                                     p(d["v"]), p(d["alpha"]), p(d["g1"]), p(d["g2"]), p(d["cu_seqlens"]),
                                     inp.num_seqs, p(d["initial_state"]), p(sf), p(o), 0, stream)


def _close(got, ref, tol, what):
    """Per row: max |got - ref| <= tol * max(1, max |ref|) (rows = tokens or state rows)."""
    g = got.float().cpu().double().numpy().reshape(-1, got.shape[-1])
    r = ref.float().cpu().double().numpy().reshape(-1, ref.shape[-1])
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    if g.size == 0:
        return
    ratio = np.abs(g - r).max(axis=1) / np.maximum(1.0, np.abs(r).max(axis=1))
    assert ratio.max() <= tol, f"{what}: error ratio {ratio.max():.3e} > {tol}"


@pytest.mark.gpu
def test_noalloc_matches_the_allocating_entry_point_on_two_calls_in_a_row():
    import linear_rnn_delta_b200 as kda
    lib = _lib()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [  # a varlen batch, then a fixed-length one: different slot layouts over the same array
        W.make_chunk_inputs("kda", "extended", "bf16", H=3, d_k=128, d_v=128, seed=41,
                            doc_lens=[300, 1, 64, 0, 129, 77], init_state="random", init_std=0.2),
        W.make_chunk_inputs("rda", "standard", "bf16", B=2, T=333, H=4, d_k=128, d_v=128, seed=42,
                            init_state="random", init_std=0.1),
    ]
    for inp in cases:
        d = {n: (None if getattr(inp, n) is None else getattr(inp, n).cuda())
             for n in ("q", "k", "v", "alpha", "g1", "g2", "cu_seqlens", "initial_state")}
        o = torch.empty((inp.B, inp.T, inp.H, inp.d_v), dtype=torch.bfloat16, device="cuda")
        sf = torch.empty((inp.num_seqs, inp.H, inp.d_k, inp.d_v), dtype=torch.float32, device="cuda")
        assert _noalloc(lib, inp, d, o, sf, stream) == OK, lib.kda_last_error_detail()
        o_ws, sf_ws = kda.kda_chunk_fwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"],
                                        d["g1"], d["g2"], cu_seqlens=d["cu_seqlens"],
                                        initial_state=d["initial_state"], flags=kda.FLAG_FORCE_SPLIT)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ws), "o differs from the split form's"
        assert torch.equal(sf, sf_ws), "final state differs from the split form's"
        o_ref, s_ref = oracle.recurrence(inp)
        _close(o, torch.from_numpy(o_ref), 2e-2, "o")
        _close(sf, torch.from_numpy(s_ref), 2e-2, "final state")


# A fake, 16-byte-aligned, never-dereferenced device address: the checks below
# return before anything touches the GPU.
P = ctypes.c_void_p(0x10000)


def _fake_call(lib, B, T, H, dtype=0, dk=128, flags=0):
    return lib.kda_chunk_fwd_noalloc(0, 0, dtype, B, T, H, dk, 128, P, P, P, P, P, None, None, 0, None, None, P,
                                     flags, None)


def test_noalloc_rejects_problems_beyond_the_fixed_array():
    lib = _lib()
    # (N + ceil(B*T/64)) * H slot-heads: 4 + 256 = 260 slots x 16 heads = 4160 > 809
    assert _fake_call(lib, 4, 4096, 16) == UNSUPPORTED
    assert "needs" in lib.kda_last_error_detail().decode()
    # one slot-head over the limit (only rejected calls here: the fake pointers must never reach a kernel)
    assert _fake_call(lib, 1, 64 * SCRATCH_SLOT_HEADS, 1) == UNSUPPORTED   # 1 + 809 slots x 1 head
    assert _fake_call(lib, 1, 64 * 404, 2) == UNSUPPORTED                  # (1 + 404) x 2 = 810


def test_noalloc_rejects_other_shapes_and_flags():
    lib = _lib()
    assert _fake_call(lib, 1, 64, 1, dtype=1) == UNSUPPORTED   # fp32
    assert _fake_call(lib, 1, 64, 1, dk=64) == UNSUPPORTED     # d_k = 64
    assert _fake_call(lib, 1, 64, 1, flags=8) == INVALID       # no flags taken
