"""Checks of device-resident inputs and the report of device-side failures.

* kda_check_gates counts gates outside the declared range ("Complex KDA"
  arXiv abstract: alpha in [-1, 1], beta in [0, 2]; KDA: alpha in (0, 1],
  beta in [0, 1]) and NaN, on planted values.
* kda_check_seqlens counts violations of the packed-document contract
  (cu[0] = 0, non-decreasing, cu[N] = total tokens: the document reset of the
  openarchlab page on GDN/KDA state updates, sec. 3).  A broken array only
  ever goes through the check itself.
* KDA_FLAG_VALIDATE_RANGE refuses a call with bad gates or offsets before
  anything is launched, and changes nothing for good inputs.
* A bounded wait that runs out is reported by kda_device_status: the
  test-only KDA_FLAG_DEBUG_STALL makes one chain CTA wait for a load that was
  never issued; the kernel gives up after about 1 ms, drains what it did
  issue, poisons that pair's final state and exits; every other pair is
  unaffected and the context stays usable.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity import assert_state_close, assert_tokens_close, cuda_inputs, run_chunk

pytestmark = pytest.mark.gpu

FORCE_SPLIT, VALIDATE, DEBUG_STALL = 8, 1, 64
KDA_OK, INVALID, RANGE, DEVICE_TIMEOUT = 0, 1, 3, 5


@pytest.fixture(autouse=True)
def _clear_status():
    import linear_rnn_delta_b200 as kda
    kda.kda_device_status()
    yield


@pytest.mark.parametrize("gate_range", ["standard", "extended"])
@pytest.mark.parametrize("variant", ["kda", "gdn2"])
def test_check_gates_counts_planted_violations(variant, gate_range):
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs(variant, gate_range, "bf16", B=2, T=100, H=3, d_k=128, d_v=128, seed=301)
    alpha, g1 = inp.alpha.clone(), inp.g1.clone()
    assert kda.kda_check_gates(variant, gate_range, alpha.cuda(), g1.cuda()) == 0
    ext = gate_range == "extended"
    a = alpha.view(-1)
    a[5] = 1.5                       # above 1 in both ranges
    a[77] = -1.25 if ext else -0.5   # below the range
    a[900] = float("nan")
    if not ext:
        a[1234] = 0.0                # the KDA range excludes 0
    g = g1.view(-1)
    g[3] = 2.5 if ext else 1.5       # above the range's maximum
    g[40] = -0.125
    g[41] = float("nan")
    expect = (4 if not ext else 3) + 3
    assert kda.kda_check_gates(variant, gate_range, alpha.cuda(), g1.cuda()) == expect


def test_check_seqlens_counts_violations():
    import linear_rnn_delta_b200 as kda
    good = torch.tensor([0, 5, 5, 70, 200], dtype=torch.int32, device="cuda")
    assert kda.kda_check_seqlens(good, 200) == 0
    assert kda.kda_check_seqlens(good, 199) == 1                                     # cu[N] != total
    bad = torch.tensor([3, 5, 4, 70, 60, 200], dtype=torch.int32, device="cuda")
    assert kda.kda_check_seqlens(bad, 200) == 3                                      # cu[0], two descents
    long = torch.arange(0, 5001, dtype=torch.int32, device="cuda") * 2
    long[2500] = 0
    assert kda.kda_check_seqlens(long, 10000) == 1


def test_validate_flag_refuses_bad_inputs_and_launches_nothing():
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("kda", "standard", "bf16", H=2, d_k=128, d_v=128, seed=302, doc_lens=[100, 40],
                              init_state="random", init_std=0.1)
    d = cuda_inputs(inp)
    o = torch.full((1, inp.T, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    # gates: one alpha above 1 -> KDA_ERR_RANGE, o untouched
    bad_alpha = d["alpha"].clone()
    bad_alpha[0, 10, 1, 3] = 1.5
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd("kda", "standard", d["q"], d["k"], d["v"], bad_alpha, d["g1"], None,
                          cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"], o=o, flags=VALIDATE)
    assert e.value.code == RANGE
    # offsets: not ending at the token count -> KDA_ERR_INVALID_ARG, o untouched
    bad_cu = torch.tensor([0, 100, 120], dtype=torch.int32, device="cuda")
    with pytest.raises(kda.KdaError) as e:
        kda.kda_chunk_fwd("kda", "standard", d["q"], d["k"], d["v"], d["alpha"], d["g1"], None, cu_seqlens=bad_cu,
                          initial_state=d["initial_state"], o=o, flags=VALIDATE)
    assert e.value.code == INVALID
    torch.cuda.synchronize()
    assert bool((o.float() == 7.0).all())
    # good inputs: the same bits as without the flag
    o1, s1 = kda.kda_chunk_fwd("kda", "standard", d["q"], d["k"], d["v"], d["alpha"], d["g1"], None,
                               cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"], flags=VALIDATE)
    o2, s2 = kda.kda_chunk_fwd("kda", "standard", d["q"], d["k"], d["v"], d["alpha"], d["g1"], None,
                               cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_validate_flag_on_decode():
    import linear_rnn_delta_b200 as kda
    st = W.decode_step_inputs(0, "kda", "extended", "bf16", N=4, H=2, d_k=128, d_v=128)
    state = W.decode_initial_state(4, 2, 128, 128).cuda()
    beta = st.g1.clone()
    beta[1, 1] = 2.5
    with pytest.raises(kda.KdaError) as e:
        kda.kda_decode_step("kda", "extended", st.q.cuda(), st.k.cuda(), st.v.cuda(), st.alpha.cuda(), beta.cuda(),
                            None, state, flags=VALIDATE)
    assert e.value.code == RANGE
    before = state.clone()
    kda.kda_decode_step("kda", "extended", st.q.cuda(), st.k.cuda(), st.v.cuda(), st.alpha.cuda(), st.g1.cuda(),
                        None, state, flags=VALIDATE)
    torch.cuda.synchronize()
    assert not torch.equal(state, before)


def test_status_is_clear_after_normal_calls():
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs("rda", "extended", "bf16", H=2, d_k=128, d_v=128, seed=303, doc_lens=[130, 3])
    for form in (4, 8):
        run_chunk(inp, flags=form)
    assert kda.kda_device_status() == (KDA_OK, 0)


@pytest.mark.parametrize("variant", ["kda", "gdn2"])
def test_expired_wait_is_reported_and_the_rest_is_computed(variant):
    import linear_rnn_delta_b200 as kda
    inp = W.make_chunk_inputs(variant, "extended", "bf16", B=2, T=200, H=2, d_k=128, d_v=128, seed=304,
                              init_state="random", init_std=0.2)
    o, sf = run_chunk(inp, flags=FORCE_SPLIT | DEBUG_STALL)
    code, bits = kda.kda_device_status()
    assert code == DEVICE_TIMEOUT and bits & kda.DEVICE_WAIT_TIMEOUT
    assert kda.kda_device_status() == (KDA_OK, 0)        # read and cleared
    s = sf.cpu()
    assert bool(torch.isnan(s[0, 0]).all())              # the stalled pair's state is poisoned
    o_ref, s_ref = oracle.recurrence(inp)
    assert_state_close(s[0, 1:], s_ref[0, 1:], 2e-2)     # every other pair is intact
    assert_state_close(s[1], s_ref[1], 2e-2)
    assert_tokens_close(o[0, :, 1], o_ref[0, :, 1], 2e-2)
    assert_tokens_close(o[1], o_ref[1], 2e-2)
    # the context is still usable: a normal call right after is correct and reports nothing
    o2, sf2 = run_chunk(inp, flags=FORCE_SPLIT)
    assert_tokens_close(o2, o_ref, 2e-2)
    assert_state_close(sf2, s_ref, 2e-2)
    assert kda.kda_device_status() == (KDA_OK, 0)
