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
