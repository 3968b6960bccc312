"""Single-token decode (kda_decode_step) vs the float64 CPU oracle.

A run of decode steps on one (sequence, head) is the recurrence over those
tokens, so the oracle reproduces every step's output and the final state by
stacking the per-step inputs along T.  The full decode workload (256 x 32
heads, d = 128, fp32 state 512 MiB, 1024 consecutive steps, Complex-KDA
range) is checked at every step on a seeded sample of heads.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import assert_state_close, assert_tokens_close, sampled_pairs, tol_for

pytestmark = pytest.mark.gpu


def _run_decode(variant, gate_range, dtype, N, H, dk, dv, n_steps, pairs, seed=0, state_std=0.02):
    import linear_rnn_delta_b200 as kda
    state0 = W.decode_initial_state(N, H, dk, dv, seed=seed, std=state_std)
    state = state0.cuda()
    names = ("q", "k", "v", "alpha", "g1", "g2")
    idx_n = torch.tensor([n for n, _ in pairs])
    idx_h = torch.tensor([h for _, h in pairs])
    kept = {nm: [] for nm in names}       # sampled heads only, per step
    outs = []
    for s in range(n_steps):
        st = W.decode_step_inputs(s, variant, gate_range, dtype, N, H, dk, dv, seed=seed)
        d = [None if getattr(st, nm) is None else getattr(st, nm).cuda() for nm in names]
        o = kda.kda_decode_step(variant, gate_range, *d, state)
        for nm in names:
            t = getattr(st, nm)
            if t is not None:
                kept[nm].append(t[idx_n, idx_h].double())
        outs.append(o[idx_n.cuda(), idx_h.cuda()].float().cpu())
    torch.cuda.synchronize()
    # [pairs, T, 1, ...] float64: one sequence of n_steps tokens per sampled head
    arrays = {nm: (torch.stack(v, dim=1).unsqueeze(2).numpy() if v else None) for nm, v in kept.items()}
    s0 = state0[idx_n, idx_h].double().numpy()[:, None]
    o_ref, s_ref = oracle.recurrence_arrays(variant, arrays["q"], arrays["k"], arrays["v"], arrays["alpha"],
                                            arrays["g1"], arrays["g2"], None, s0)
    o_gpu = torch.stack(outs, dim=1).double().numpy()          # [pairs, T, dv]
    s_gpu = state[idx_n.cuda(), idx_h.cuda()].double().cpu().numpy()
    tol = tol_for(dtype)
    assert_tokens_close(o_gpu, o_ref[:, :, 0], tol, "decode o")
    assert_state_close(s_gpu, s_ref[:, 0], tol, "decode state")


@pytest.mark.parametrize("variant,gate_range", [("kda", "standard"), ("kda", "extended"), ("rda", "extended"),
                                                ("gdn2", "standard")])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_small_d128(variant, gate_range, dtype):
    N, H = 5, 3
    pairs = [(n, h) for n in range(N) for h in range(H)]
    _run_decode(variant, gate_range, dtype, N, H, 128, 128, 20, pairs, seed=3, state_std=0.3)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 128), (128, 16), (64, 64), (16, 64)])
def test_decode_other_dims(dk, dv):
    N, H = 3, 2
    pairs = [(n, h) for n in range(N) for h in range(H)]
    _run_decode("gdn2", "extended", "f32", N, H, dk, dv, 9, pairs, seed=4, state_std=0.3)


@pytest.mark.slow
def test_decode_full_complex_kda_256x32_1024_steps_sampled():
    """The full decode workload: every one of 1024 steps checked on 24 heads."""
    pairs = sampled_pairs(256, 32, 24, seed=7)
    _run_decode("kda", "extended", "bf16", 256, 32, 128, 128, 1024, pairs, seed=0)
