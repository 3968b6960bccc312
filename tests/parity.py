"""Helpers for GPU-vs-oracle parity tests.

Tolerance rule (per token t, per (sequence, head) state):
    max_j |o_gpu[t] - o_ref[t]|  <=  tol * max(1, ||o_ref[t]||_inf)
    max   |S_gpu - S_ref|        <=  tol * max(1, ||S_ref||_inf)
tol = 2e-2 for bf16 inputs (fp32 accumulation, fp32 state, o rounded to
bf16) and 1e-4 for fp32 inputs.
"""
import numpy as np
import torch

TOL = {"bf16": 2e-2, "f32": 1e-4}


def tol_for(dtype: str) -> float:
    return TOL[dtype]


def cuda_inputs(inp, device="cuda"):
    d = {}
    for name in ("q", "k", "v", "alpha", "g1", "g2"):
        t = getattr(inp, name)
        d[name] = None if t is None else t.to(device).contiguous()
    d["cu_seqlens"] = None if inp.cu_seqlens is None else inp.cu_seqlens.to(device)
    d["initial_state"] = None if inp.initial_state is None else inp.initial_state.to(device).contiguous()
    return d


def run_chunk(inp, flags=0, chunk_size=None, device="cuda"):
    import linear_rnn_delta_b200 as kda
    d = cuda_inputs(inp, device)
    o, sf = kda.kda_chunk_fwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                              cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"],
                              chunk_size=inp.chunk_size if chunk_size is None else chunk_size, flags=flags)
    torch.cuda.synchronize()
    return o, sf


def token_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    """Per-token max abs error and per-token scale max(1, ||o_ref||_inf), rows = tokens."""
    g = o_gpu.reshape(-1, o_gpu.shape[-1]).astype(np.float64)
    r = o_ref.reshape(-1, o_ref.shape[-1])
    err = np.abs(g - r).max(axis=1) if g.size else np.zeros(0)
    scale = np.maximum(1.0, np.abs(r).max(axis=1)) if r.size else np.zeros(0)
    return err, scale


def assert_tokens_close(o_gpu, o_ref, tol, what="o"):
    if hasattr(o_gpu, "detach"):
        o_gpu = o_gpu.detach().float().cpu().double().numpy()
    err, scale = token_errors(o_gpu, o_ref)
    if err.size == 0:
        return 0.0
    ratio = err / scale
    worst = int(np.argmax(ratio))
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite values"
    assert ratio[worst] <= tol, f"{what}: token row {worst} error {err[worst]:.3e} > {tol} * {scale[worst]:.3e}"
    return float(ratio.max())


def assert_state_close(s_gpu, s_ref, tol, what="state"):
    if hasattr(s_gpu, "detach"):
        s_gpu = s_gpu.detach().cpu().double().numpy()
    s_gpu = np.asarray(s_gpu, dtype=np.float64)
    assert np.all(np.isfinite(s_gpu)), f"{what}: non-finite values"
    flat_g = s_gpu.reshape(-1, s_gpu.shape[-2] * s_gpu.shape[-1])
    flat_r = s_ref.reshape(-1, s_ref.shape[-2] * s_ref.shape[-1])
    err = np.abs(flat_g - flat_r).max(axis=1)
    scale = np.maximum(1.0, np.abs(flat_r).max(axis=1))
    ratio = err / scale
    worst = int(np.argmax(ratio))
    assert ratio[worst] <= tol, f"{what}: head {worst} error {err[worst]:.3e} > {tol} * {scale[worst]:.3e}"
    return float(ratio.max())


def sampled_pairs(n_seqs, H, count, seed=0):
    """A fixed, seeded sample of (sequence, head) pairs, always including the
    first and last sequence and head."""
    rng = np.random.default_rng(seed)
    pairs = {(0, 0), (n_seqs - 1, H - 1)}
    while len(pairs) < min(count, n_seqs * H):
        pairs.add((int(rng.integers(n_seqs)), int(rng.integers(H))))
    return sorted(pairs)


def check_sampled(inp, o_gpu, sf_gpu, pairs, tol, threads=0):
    """Compare a full GPU run with the oracle on sampled (sequence, head) pairs."""
    import oracle
    seqs = sorted({n for n, _ in pairs})
    heads = sorted({h for _, h in pairs})
    o_d, s_d = oracle.recurrence(inp, seqs=seqs, heads=heads, threads=threads)
    o_gpu = o_gpu.detach().float().cpu()
    worst_o = worst_s = 0.0
    for (n, h) in pairs:
        b, t0, ln = inp.seq_bounds(n)
        worst_o = max(worst_o, assert_tokens_close(o_gpu[b, t0:t0 + ln, h].double().numpy(), o_d[(n, h)], tol,
                                                   f"o[seq {n}, head {h}]"))
        if sf_gpu is not None:
            worst_s = max(worst_s, assert_state_close(sf_gpu[n, h][None], s_d[(n, h)][None], tol,
                                                      f"S[seq {n}, head {h}]"))
    return worst_o, worst_s
