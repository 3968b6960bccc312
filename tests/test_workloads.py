"""The seeded input recipe (CPU): gate ranges per variant, the signed and
near-zero gates Complex KDA needs to exercise the sign-safe paths, unit-norm
keys, and reproducibility from the seed."""
import numpy as np
import pytest
import torch

import workloads as W


def _f(t):
    return t.double().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_kda_standard_range(dtype):
    inp = W.make_chunk_inputs("kda", "standard", dtype, B=2, T=300, H=4, d_k=32, d_v=16, seed=3)
    a, b = _f(inp.alpha), _f(inp.g1)
    assert a.min() > 0 and a.max() <= 1 and b.min() > 0 and b.max() < 1
    assert inp.g2 is None and inp.g1.shape == (2, 300, 4)


def test_complex_kda_range_has_signed_small_and_large_gates():
    inp = W.make_chunk_inputs("kda", "extended", "bf16", B=2, T=300, H=4, d_k=32, d_v=16, seed=3)
    a, b = _f(inp.alpha), _f(inp.g1)
    assert a.min() >= -1 and a.max() <= 1
    assert (a < 0).mean() > 0.3                 # negative gates (reflections)
    assert (np.abs(a) < 0.05).mean() > 0.01     # near-zero gates (the anchored path's case)
    assert b.min() > 0 and b.max() < 2 and (b > 1).mean() > 0.3


@pytest.mark.parametrize("variant", ["rda", "gdn2"])
def test_rda_gdn2_gates(variant):
    inp = W.make_chunk_inputs(variant, "standard", "bf16", B=1, T=200, H=3, d_k=32, d_v=16, seed=4)
    g1, g2 = _f(inp.g1), _f(inp.g2)
    assert g1.min() > 0 and g1.max() < 1 and g2.min() > 0 and g2.max() < 1
    shape1, shape2 = ((1, 200, 3, 32), (1, 200, 3, 16)) if variant == "gdn2" else ((1, 200, 3), (1, 200, 3))
    assert g1.shape == shape1 and g2.shape == shape2
    assert not np.array_equal(g1.reshape(-1)[:50], g2.reshape(-1)[:50])   # drawn independently


def test_keys_are_unit_norm_unless_raw():
    inp = W.make_chunk_inputs("kda", "standard", "f32", B=1, T=50, H=2, d_k=64, d_v=16, seed=5)
    np.testing.assert_allclose(np.linalg.norm(_f(inp.k), axis=-1), 1.0, atol=1e-6)
    raw = W.make_chunk_inputs("kda", "standard", "f32", B=1, T=50, H=2, d_k=64, d_v=16, seed=5, raw_k=True)
    assert np.abs(np.linalg.norm(_f(raw.k), axis=-1) - 1.0).max() > 0.5
    r2 = W.make_rank2_inputs("gdn2", "extended", "bf16", B=1, T=40, H=2, d_k=64, d_v=16, seed=6)
    np.testing.assert_allclose(np.linalg.norm(_f(r2.k), axis=-1), 1.0, atol=1e-2)   # per sub-step, bf16


def test_same_seed_same_inputs_other_seed_other_inputs():
    a = W.make_chunk_inputs("gdn2", "extended", "bf16", H=2, d_k=32, d_v=32, seed=8, doc_lens=[30, 0, 70],
                            init_state="random")
    b = W.make_chunk_inputs("gdn2", "extended", "bf16", H=2, d_k=32, d_v=32, seed=8, doc_lens=[30, 0, 70],
                            init_state="random")
    c = W.make_chunk_inputs("gdn2", "extended", "bf16", H=2, d_k=32, d_v=32, seed=9, doc_lens=[30, 0, 70],
                            init_state="random")
    for name in ("q", "k", "v", "alpha", "g1", "g2", "initial_state"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert not torch.equal(getattr(a, name), getattr(c, name)), name
    assert a.cu_seqlens.tolist() == [0, 30, 30, 100]


def test_decode_steps_regenerate_independently():
    s5 = W.decode_step_inputs(5, N=4, H=2, d_k=32, d_v=16)
    again = W.decode_step_inputs(5, N=4, H=2, d_k=32, d_v=16)
    s6 = W.decode_step_inputs(6, N=4, H=2, d_k=32, d_v=16)
    assert torch.equal(s5.q, again.q) and torch.equal(s5.alpha, again.alpha)
    assert not torch.equal(s5.q, s6.q)


def test_varlen_lengths_follow_the_recipe():
    lens = W.varlen_doc_lens(seed=0)
    assert len(lens) == 16 and min(lens) >= 512 and max(lens) <= 4096
    assert lens == W.varlen_doc_lens(seed=0)


def test_grad_outputs_shapes_and_scale():
    inp = W.make_chunk_inputs("rda", "standard", "bf16", B=2, T=500, H=2, d_k=32, d_v=16, seed=10)
    d_o, dsf = W.grad_outputs(inp, seed=10)
    assert d_o.shape == (2, 500, 2, 16) and d_o.dtype == torch.bfloat16
    assert dsf.shape == (2, 2, 32, 16) and dsf.dtype == torch.float32
    assert 0.9 < float(d_o.float().std()) < 1.1 and 0.08 < float(dsf.std()) < 0.12
    assert W.grad_outputs(inp, seed=10, d_final=False)[1] is None
