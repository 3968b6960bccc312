"""Host-side accounting of bench.py (CPU): algorithmic bytes and flops, the
committed DRAM-traffic table, and the clock-sample parser that decides whether
a timed run is kept."""
import json
import os

import pytest

import bench
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_chunk_bytes_and_flops_by_hand():
    # KDA, bf16, one head, one 64-token chunk, d = 128, zero initial state
    inp = W.make_chunk_inputs("kda", "standard", "bf16", B=1, T=64, H=1, d_k=128, d_v=128, seed=0)
    alg = bench.chunk_algorithmic(inp)
    q_k_v_alpha = 4 * 64 * 128 * 2
    beta = 64 * 2
    o = 64 * 128 * 2
    final_state = 128 * 128 * 4
    assert alg["bytes"] == q_k_v_alpha + beta + o + final_state
    assert alg["head_tokens"] == 64 and alg["tokens"] == 64
    assert alg["flops"] == pytest.approx(64 * (6 * 128 * 128 + 2 * 64 * 256 + 64 * 64 / 3.0))


def test_chunk_bytes_count_the_initial_state_and_vector_gates():
    base = W.make_chunk_inputs("gdn2", "standard", "bf16", B=2, T=32, H=3, d_k=64, d_v=32, seed=1)
    with_s0 = W.make_chunk_inputs("gdn2", "standard", "bf16", B=2, T=32, H=3, d_k=64, d_v=32, seed=1,
                                  init_state="random")
    a, b = bench.chunk_algorithmic(base), bench.chunk_algorithmic(with_s0)
    assert b["bytes"] - a["bytes"] == 2 * 3 * 64 * 32 * 4          # the initial states, read once
    # GDN-2 reads its erase vector b (d_k) and write vector w (d_v) per head-token
    per_ht = (2 * 64 + 32 + 64) * 2 + (64 + 32) * 2 + 32 * 2     # q, k, alpha; v; b, w; o
    assert a["bytes"] == 2 * 32 * 3 * per_ht + 2 * 3 * 64 * 32 * 4


def test_decode_bytes_match_the_bench_workload():
    # Complex-KDA decode, N=256 sequences x H=32 heads, d=128: the fp32 state read and
    # written once, q, k, alpha (d_k each), v, beta in and o out, bf16
    alg = bench.decode_algorithmic(256, 32, 128, 128)
    state = 2 * 256 * 32 * 128 * 128 * 4
    per_head = (3 * 128 + 128) * 2 + 2 + 128 * 2
    assert alg["bytes"] == state + 256 * 32 * per_head == 1084243968
    assert alg["tokens"] == 256


def test_decode_bytes_per_variant():
    kda = bench.decode_algorithmic(1, 1, 16, 16, variant="kda")["bytes"]
    rda = bench.decode_algorithmic(1, 1, 16, 16, variant="rda")["bytes"]
    gdn2 = bench.decode_algorithmic(1, 1, 16, 16, variant="gdn2")["bytes"]
    assert rda - kda == 2                  # one more scalar gate
    assert gdn2 - kda == (16 + 16) * 2 - 2  # two vectors instead of one scalar


def test_backward_flops_are_one_forward_pass_and_the_adjoint():
    inp = W.make_chunk_inputs("kda", "standard", "bf16", B=2, T=48, H=2, d_k=32, d_v=64, seed=2)
    alg = bench.backward_algorithmic(inp)
    assert alg["tokens"] == 96
    assert alg["flops"] == (2 * 2 + 2 * 7.5) * 32 * 64 * 2 * 48 * 2


def test_traffic_table_is_consistent():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    for name, e in table.items():
        assert len(e["source_sha256"]) == 64, name
        assert e["dram_bytes_per_launch"] > 0, name
        assert os.path.exists(os.path.join(ROOT, e["capture"])), name
        if "per_kernel" in e:
            assert abs(sum(e["per_kernel"].values()) - e["dram_bytes_per_launch"]) <= 1, name


def test_traffic_is_dropped_when_the_sources_change(monkeypatch):
    name = "chunk_fwd_ckda_8x16x8192_split"
    monkeypatch.setattr(bench, "source_digest", lambda paths: "0" * 64)
    assert bench.measured_traffic(name, bench.CHUNK_SOURCES) == {}


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampled(tmp_path, rows):
    p = tmp_path / "clocks.csv"
    p.write_text("".join(", ".join(r) + "\n" for r in rows))
    s = bench.ClockSampler(0)
    s.proc, s.path = _DoneProc(), str(p)
    return s.stop()


def test_clock_sampler_median_of_loaded_samples(tmp_path):
    idle = ["0", "345", "1965", "120.0", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"]
    busy = ["0", "1965", "1965", "900.0", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"]
    r = _sampled(tmp_path, [idle, busy, busy, busy])
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == [] and r["samples"] == 4


def test_clock_sampler_reports_throttle_reasons(tmp_path):
    row = ["0", "1500", "1965", "1000.0", "0x4", "Not Active", "Active", "Not Active", "Active"]
    r = _sampled(tmp_path, [row, row])
    assert r["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert r["sm_mhz"] == 1500


def test_clock_sampler_without_samples(tmp_path):
    r = _sampled(tmp_path, [])
    assert r["sm_mhz"] is None and r["reasons"] == ["no samples"]
