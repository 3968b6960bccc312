"""Python binding argument checks that need no GPU: shape, dtype and device
errors are raised before the library is called."""
import pytest
import torch


@pytest.fixture(scope="module")
def kda():
    import linear_rnn_delta_b200 as k
    return k


def _inputs(B=1, T=8, H=2, dk=16, dv=16, dtype=torch.float32, rank2=False):
    sub = (2,) if rank2 else ()
    return dict(q=torch.zeros(B, T, H, dk, dtype=dtype), k=torch.zeros(B, T, *sub, H, dk, dtype=dtype),
                v=torch.zeros(B, T, *sub, H, dv, dtype=dtype), alpha=torch.ones(B, T, H, dk, dtype=dtype),
                g1=torch.zeros(B, T, *sub, H, dtype=dtype))


def test_chunk_bwd_needs_cuda_tensors(kda):
    x = _inputs()
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_chunk_bwd("kda", "standard", x["q"], x["k"], x["v"], x["alpha"], x["g1"], None,
                          torch.zeros(1, 8, 2, 16))


def test_chunk_bwd_rejects_bad_names_and_dtypes(kda):
    x = _inputs(dtype=torch.float16)
    with pytest.raises(ValueError):
        kda.kda_chunk_bwd("kda", "standard", x["q"], x["k"], x["v"], x["alpha"], x["g1"], None, x["v"])
    x = _inputs()
    with pytest.raises(ValueError):
        kda.kda_chunk_bwd("nope", "standard", x["q"], x["k"], x["v"], x["alpha"], x["g1"], None, x["v"])
    with pytest.raises(ValueError):
        kda.kda_chunk_bwd("kda", "wide", x["q"], x["k"], x["v"], x["alpha"], x["g1"], None, x["v"])
    with pytest.raises(ValueError):   # q must be 4-D
        kda.kda_chunk_bwd("kda", "standard", x["q"][0], x["k"], x["v"], x["alpha"], x["g1"], None, x["v"])


def test_rank2_needs_the_sub_step_axis(kda):
    x = _inputs()   # rank-1 shapes: k is 4-D
    with pytest.raises(ValueError, match="2,H"):
        kda.kda_chunk_fwd_rank2("kda", "standard", x["q"], x["k"], x["v"], x["alpha"], x["g1"])


def test_rank2_needs_cuda_tensors_and_write_gate(kda):
    x = _inputs(rank2=True)
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_chunk_fwd_rank2("kda", "standard", x["q"], x["k"], x["v"], x["alpha"], x["g1"])
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd_rank2("kda", "standard", x["q"].half(), x["k"], x["v"], x["alpha"], x["g1"])


def test_autograd_function_is_exported(kda):
    assert issubclass(kda.KdaChunkFunction, torch.autograd.Function)
    for name in ("kda_chunk_bwd", "kda_chunk_fwd_rank2", "KdaChunkFunction"):
        assert name in kda.__all__


def test_chunk_slots_are_unique_increasing_and_in_range(kda):
    """Slot of chunk c of sequence n (first packed row R_n): n + floor(R_n / 64) + c.  For random packings,
    every (sequence, chunk) gets its own slot, slots increase within a sequence and stay below
    num_chunk_slots(B, T, N) = N + ceil(B*T / 64)."""
    import numpy as np
    rng = np.random.default_rng(5)
    for _ in range(200):
        lens = rng.integers(0, 300, size=int(rng.integers(1, 12)))
        rows = np.concatenate([[0], np.cumsum(lens)])
        N, total = len(lens), int(rows[-1])
        seen = set()
        for n, ln in enumerate(lens):
            slots = [kda.chunk_slot(n, c, int(rows[n])) for c in range((int(ln) + 63) // 64)]
            assert slots == sorted(slots) and len(set(slots)) == len(slots)
            seen.update(slots)
            assert all(0 <= s < kda.num_chunk_slots(1, total, N) for s in slots)
        assert len(seen) == sum((int(ln) + 63) // 64 for ln in lens)
    # fixed-length batches: sequence n starts at row n*T
    B, T = 3, 130
    slots = [kda.chunk_slot(n, c, n * T) for n in range(B) for c in range(3)]
    assert len(set(slots)) == len(slots) and max(slots) < kda.num_chunk_slots(B, T, B)
