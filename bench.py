"""Benchmark of the gated delta-rule recurrence on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--extra]

A step is one pass of the hot path over one batch of synthetic input: one
chunked forward (``kda_chunk_fwd``) over the Complex-KDA bf16 workload
B=8, H=16, T=8192, d_k=d_v=128, chunk 64 (alpha = tanh(2 N(0,1)), beta =
2 sigmoid(N(0,1)); seeded inputs resident in HBM) -- the largest of the
chunked workloads and the one with signed gates.  In the same run, each with
its own roofline and end-to-end figures, "also" times the KDA-range workload
B=4, H=16, T=4096 and the RDA and GDN-2 packed workloads (16 documents of
U[512, 4096] tokens, H=32); "decode" times the single-token step (256 x 32
heads, d=128, fp32 state 512 MiB in place, Complex-KDA range) and
"backward" the gradients of the KDA-range workload.  --extra adds the forward
from gate logits and raw keys, with state snapshots, and rank-2 steps.

Multi-GPU (torchrun): every rank runs its own independent batch (different
seed): the work shards over (sequence, head) units with no collective on the
data path, so scaling is weak; ranks only meet at barriers and at the final
max-over-ranks of the device times.

Rank 0 prints one JSON line.  All device times come from CUDA events on the
launching stream; clocks are sampled with nvidia-smi during the timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "chunked fwd tokens/s & % tensor-core peak; decode step HBM GB/s (1×B200)"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# Algorithmic work per workload (bytes and flops the path must move / do)
# ---------------------------------------------------------------------------

def chunk_algorithmic(inp) -> dict:
    """Bytes: every input read once, o written once, states read/written once.
    Flops: WY chunk form per head-token, triangles counted as half:
    6*dk*dv + 2*C*(dk+dv) + C^2/3."""
    head_tokens = inp.B * inp.T * inp.H
    C, dk, dv = inp.chunk_size, inp.d_k, inp.d_v
    in_bytes = inp.nbytes()
    o_bytes = inp.B * inp.T * inp.H * dv * inp.q.element_size()
    n_states = inp.num_seqs * inp.H
    state_bytes = n_states * dk * dv * 4 * (2 if inp.initial_state is not None else 1)
    flops = head_tokens * (6 * dk * dv + 2 * C * (dk + dv) + C * C / 3.0)
    return {"bytes": in_bytes + o_bytes + state_bytes, "flops": flops, "head_tokens": head_tokens,
            "tokens": inp.B * inp.T}


def decode_algorithmic(N, H, dk, dv, elem=2, variant="kda") -> dict:
    state = 2 * N * H * dk * dv * 4
    per_head_in = (3 * dk + dv) * elem + (elem if variant != "gdn2" else (dk + dv) * elem)
    if variant == "rda":
        per_head_in += elem
    io = N * H * (per_head_in + dv * elem)
    return {"bytes": state + io, "flops": N * H * 7 * dk * dv, "tokens": N}


# ---------------------------------------------------------------------------
# Device helpers
# ---------------------------------------------------------------------------

# fp32 FMA peak of the SIMT cores: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_algorithmic(inp) -> dict:
    """Arithmetic the backward needs per head-token: one forward pass for the
    states (u and the state update: 2 d_k d_v FMAs) and the adjoint step
    (G += q do^T, the row sums S do, G u, S dS', S du, the column sum k^T G,
    dS' and G <- Diag(alpha) dS': 7.5 d_k d_v FMAs), i.e. 19 d_k d_v flops.
    Recomputation is not counted: neither the replay of each chunk from its
    checkpoint nor the states between stored ones."""
    heads_tokens = inp.B * inp.T * inp.H
    return {"tokens": inp.B * inp.T, "flops": 19.0 * inp.d_k * inp.d_v * heads_tokens}


def source_digest(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


CHUNK_SOURCES = ["linear_rnn_delta_b200/csrc/chunk_fwd_sm100.cu", "linear_rnn_delta_b200/csrc/sm100.cuh",
                 "linear_rnn_delta_b200/csrc/common.cuh"]
DECODE_SOURCES = ["linear_rnn_delta_b200/csrc/decode_step.cu", "linear_rnn_delta_b200/csrc/common.cuh"]
BWD_SOURCES = ["linear_rnn_delta_b200/csrc/scan_fwd.cu", "linear_rnn_delta_b200/csrc/scan_bwd.cu",
               "linear_rnn_delta_b200/csrc/scan_bwd.cuh", "linear_rnn_delta_b200/csrc/common.cuh"]


def measured_traffic(name: str, sources) -> dict:
    """DRAM bytes per launch from a committed ncu summary (profiles/traffic.json),
    only while the kernel's sources still hash to what was profiled."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    with open(p) as f:
        d = json.load(f).get(name)
    if not d or d.get("source_sha256") != source_digest(sources):
        return {}
    return d


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        """Start sampling and wait until the first sample is written, so that
        nvidia-smi's start-up never overlaps the timed region."""
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 20.0:
                if os.path.getsize(self.path) > 0:
                    break
                time.sleep(0.05)
            time.sleep(0.2)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Slowest rank's time: the job finishes when every rank has."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload_seed(rank: int) -> int:
    """Weak scaling: every rank owns an independent batch of (sequence, head)
    units drawn with its own seed; no data crosses ranks."""
    return rank


# ---------------------------------------------------------------------------
# Timed regions
# ---------------------------------------------------------------------------

def time_launches(fn, steps: int, warmup: int, world: int, stream):
    """W untimed steps, then K steps bracketed by barrier + synchronize; per-launch
    CUDA events on the launching stream.  Returns (total_s, per_launch_s list)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start_all = torch.cuda.Event(enable_timing=True)
    end_all = torch.cuda.Event(enable_timing=True)
    start_all.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    end_all.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total = start_all.elapsed_time(end_all) / 1e3
    per = [a.elapsed_time(b) / 1e3 for a, b in ev]
    return total, per


def pct(xs, p):
    return float(np.percentile(np.asarray(xs), p))


FORM_FLAGS = {"auto": 0, "fused": 4, "split": 8}


def chunk_form(inp, flags=0) -> str:
    """Which form of the tensor-core path the library runs for this workload:
    it needs a workspace exactly when it runs the split form."""
    import linear_rnn_delta_b200 as kda
    ws = kda.lib.kda_chunk_fwd_workspace_size(0 if inp.dtype == "bf16" else 1, inp.B, inp.T, inp.H, inp.d_k,
                                              inp.d_v, int(inp.cu_seqlens is not None), inp.num_seqs,
                                              inp.chunk_size, flags)
    return "split" if ws else "fused"


def run_chunk_workload(inp, steps, warmup, world, peaks, sampler=None, e2e=True, flags=0, states=False):
    import linear_rnn_delta_b200 as kda
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    d = {n: (None if getattr(inp, n) is None else getattr(inp, n).to(dev)) for n in
         ("q", "k", "v", "alpha", "g1", "g2")}
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    s0 = None if inp.initial_state is None else inp.initial_state.to(dev)
    N = inp.num_seqs
    o = torch.empty((inp.B, inp.T, inp.H, inp.d_v), dtype=d["q"].dtype, device=dev)
    sf = torch.empty((N, inp.H, inp.d_k, inp.d_v), dtype=torch.float32, device=dev)
    cs = None
    if states:   # state snapshots after every 64 tokens
        cs = torch.empty((kda.num_chunk_slots(inp.B, inp.T, N), inp.H, inp.d_k, inp.d_v), dtype=torch.float32,
                         device=dev)

    def step():
        kda.kda_chunk_fwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                          cu_seqlens=cu, initial_state=s0, final_state=sf, o=o, chunk_size=inp.chunk_size,
                          flags=flags, stream=stream, chunk_states=cs)

    if sampler:
        sampler.start()
    total, per = time_launches(step, steps, warmup, world, stream)
    clocks = sampler.stop() if sampler else None
    total = max_over_ranks(total, world)
    alg = chunk_algorithmic(inp)
    avg = sum(per) / len(per)
    form = chunk_form(inp, flags)
    res = {"tokens_per_step": alg["tokens"], "total_s": total, "avg_launch_s": avg, "form": form,
           "kernels_per_step": 2 if form == "split" else 1,
           "p50_ms": pct(per, 50) * 1e3, "p95_ms": pct(per, 95) * 1e3, "p99_ms": pct(per, 99) * 1e3,
           "alg": alg, "clocks": clocks}
    gbs = alg["bytes"] / avg / 1e9
    tfs = alg["flops"] / avg / 1e12
    res["hbm"] = {"achieved": gbs, "peak": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"]}
    res["tensor"] = {"achieved": tfs, "peak": peaks["bf16_tflops"], "frac": tfs / peaks["bf16_tflops"]}
    if e2e:
        res["e2e"] = chunk_e2e(inp, d, cu, s0, o, sf, steps, warmup, world, stream, flags)
    return res


def chunk_e2e(inp, d, cu, s0, o, sf, steps, warmup, world, stream, flags=0):
    """Same step through the public API with pinned host buffers: H2D of the
    step's inputs, the kernel, D2H of o and the final state, all timed."""
    import linear_rnn_delta_b200 as kda
    host = {n: (None if getattr(inp, n) is None else getattr(inp, n).pin_memory()) for n in
            ("q", "k", "v", "alpha", "g1", "g2")}
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    sf_h = torch.empty(sf.shape, dtype=sf.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    d2h = o.numel() * o.element_size() + sf.numel() * sf.element_size()

    def step():
        for n, t in host.items():
            if t is not None:
                d[n].copy_(t, non_blocking=True)
        kda.kda_chunk_fwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                          cu_seqlens=cu, initial_state=s0, final_state=sf, o=o, chunk_size=inp.chunk_size,
                          flags=flags, stream=stream)
        o_h.copy_(o, non_blocking=True)
        sf_h.copy_(sf, non_blocking=True)

    total, _ = time_launches(step, steps, max(1, warmup), world, stream)
    total = max_over_ranks(total, world)
    return {"total_s": total, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def run_decode_workload(steps, warmup, world, peaks, rank, N=256, H=32, dk=128, dv=128, e2e=True):
    import linear_rnn_delta_b200 as kda
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    state = W.decode_initial_state(N, H, dk, dv, seed=rank).to(dev)
    n_inputs = 8   # distinct per-step inputs cycled through the timed steps
    inputs = []
    for s in range(n_inputs):
        st = W.decode_step_inputs(s, "kda", "extended", "bf16", N, H, dk, dv, seed=rank)
        inputs.append([None if t is None else t.to(dev) for t in (st.q, st.k, st.v, st.alpha, st.g1, st.g2)])
    o = torch.empty((N, H, dv), dtype=torch.bfloat16, device=dev)
    it = [0]

    def step():
        x = inputs[it[0] % n_inputs]
        it[0] += 1
        kda.kda_decode_step("kda", "extended", *x, state, o=o, stream=stream)

    total, per = time_launches(step, steps, warmup, world, stream)
    total = max_over_ranks(total, world)
    alg = decode_algorithmic(N, H, dk, dv)
    avg = sum(per) / len(per)
    gbs = alg["bytes"] / avg / 1e9
    res = {"value": N * world * steps / total, "unit": "tokens/s", "workload":
           f"decode Complex-KDA N={N} H={H} d_k=d_v={dk} fp32 state in place, bf16 inputs",
           "ms_per_step": total / steps * 1e3, "p50_ms": pct(per, 50) * 1e3, "p95_ms": pct(per, 95) * 1e3,
           "p99_ms": pct(per, 99) * 1e3,
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"],
                        "traffic": measured_traffic("decode_ckda_256x32", DECODE_SOURCES).get("dram_bytes_per_launch"),
                        "peak_source": peaks["source"]},
           "bytes_per_step": alg["bytes"], "gpu_launches": steps}
    if e2e:
        host = [None if t is None else t.cpu().pin_memory() for t in inputs[0]]
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host if t is not None)

        def step_e2e():
            x = inputs[0]
            for dst, src in zip(x, host):
                if src is not None:
                    dst.copy_(src, non_blocking=True)
            kda.kda_decode_step("kda", "extended", *x, state, o=o, stream=stream)
            o_h.copy_(o, non_blocking=True)

        tot_e2e, _ = time_launches(step_e2e, steps, warmup, world, stream)
        tot_e2e = max_over_ranks(tot_e2e, world)
        res["e2e"] = {"value": N * world * steps / tot_e2e, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": o.numel() * o.element_size()}
    return res


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline and reference arm)
# ---------------------------------------------------------------------------

def run_backward_workload(inp, steps, warmup, world, rank):
    """kda_chunk_bwd over the chunked workload with seeded d_o and dL/dS_final."""
    import linear_rnn_delta_b200 as kda
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    d = {n: (None if getattr(inp, n) is None else getattr(inp, n).to(dev)) for n in
         ("q", "k", "v", "alpha", "g1", "g2")}
    d_o, dsf = W.grad_outputs(inp, seed=rank_workload_seed(rank))
    d_o, dsf = d_o.to(dev), dsf.to(dev)

    def step():
        kda.kda_chunk_bwd(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"], d_o,
                          dsf, stream=stream)

    total, per = time_launches(step, steps, warmup, world, stream)
    total = max_over_ranks(total, world)
    alg = backward_algorithmic(inp)
    avg = sum(per) / len(per)
    tfs = alg["flops"] / avg / 1e12
    return {"workload": "backward (all gradients) of the KDA-range chunked workload B=4 H=16 T=4096 d=128 bf16 "
                        "inputs, fp32 arithmetic; seeded d_o ~ N(0,1), dL/dS_final ~ N(0, 0.01)",
            "value": alg["tokens"] * world * steps / total, "unit": UNIT, "ms_per_step": total / steps * 1e3,
            "p50_ms": pct(per, 50) * 1e3, "kernels_per_step": 2, "gpu_launches": 2 * steps,
            "roofline": {"bound": "alu", "achieved": tfs, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                         "frac": tfs / FP32_ALU_TFLOPS,
                         "traffic": measured_traffic("backward_kda_4x16x4096", BWD_SOURCES).get("dram_bytes_per_launch"),
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz",
                         "alg_flops_per_launch": alg["flops"],
                         "kernel": "kda_chunk_bwd: checkpoint scan + cluster adjoint scan timed as one call"}}


def run_rank2_workload(inp, steps, warmup, world):
    """kda_chunk_fwd_rank2 (two sub-steps per token) over a rank-2 workload."""
    import linear_rnn_delta_b200 as kda
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    d = {n: (None if getattr(inp, n) is None else getattr(inp, n).to(dev)) for n in
         ("q", "k", "v", "alpha", "g1", "g2")}
    o = torch.empty((inp.B, inp.T, inp.H, inp.d_v), dtype=d["q"].dtype, device=dev)
    sf = torch.empty((inp.B, inp.H, inp.d_k, inp.d_v), dtype=torch.float32, device=dev)

    def step():
        kda.kda_chunk_fwd_rank2(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                                final_state=sf, o=o, stream=stream)

    total, per = time_launches(step, steps, warmup, world, stream)
    total = max_over_ranks(total, world)
    return {"tokens_per_step": inp.B * inp.T, "total_s": total, "avg_launch_s": sum(per) / len(per)}


def run_rank2_backward_workload(inp, steps, warmup, world, rank):
    """kda_chunk_bwd_rank2 (gradients of rank-2 steps) with seeded d_o ~ N(0,1), dL/dS_final ~ N(0, 0.01)."""
    import linear_rnn_delta_b200 as kda
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    d = {n: (None if getattr(inp, n) is None else getattr(inp, n).to(dev)) for n in
         ("q", "k", "v", "alpha", "g1", "g2")}
    g = torch.Generator().manual_seed(rank_workload_seed(rank) * 7 + 3)
    d_o = torch.randn((inp.B, inp.T, inp.H, inp.d_v), generator=g).to(dev, d["q"].dtype)
    dsf = (0.1 * torch.randn((inp.B, inp.H, inp.d_k, inp.d_v), generator=g)).to(dev)

    def step():
        kda.kda_chunk_bwd_rank2(inp.variant, inp.gate_range, d["q"], d["k"], d["v"], d["alpha"], d["g1"], d["g2"],
                                d_o, dsf, stream=stream)

    total, per = time_launches(step, steps, warmup, world, stream)
    total = max_over_ranks(total, world)
    return {"tokens_per_step": inp.B * inp.T, "total_s": total, "avg_launch_s": sum(per) / len(per)}


def host_cores() -> int:
    """Cores this process may run on (its CPU affinity)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:   # pragma: no cover
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_block(inp, n_pairs: int):
    """A block of about n_pairs (sequence, head) pairs, whole sequences: the
    first heads, then as many of the first sequences as it takes."""
    heads = list(range(min(inp.H, max(1, n_pairs))))
    seqs = list(range(min(inp.num_seqs, -(-max(1, n_pairs) // len(heads)))))
    return seqs, heads


def time_oracle(inp, seqs, heads, threads: int):
    """Seconds and head-tokens of the float64 oracle over every (sequence, head)
    of the block."""
    import oracle
    t0 = time.perf_counter()
    oracle.recurrence(inp, seqs=seqs, heads=heads, threads=threads)
    dt = time.perf_counter() - t0
    return dt, sum(inp.seq_bounds(n)[2] for n in seqs) * len(heads)


def oracle_sample_rate(inp, target_s=10.0):
    """Tokens/s of the float64 oracle, as it stands, on a bounded sample of the
    workload (whole sequences of a block of (sequence, head) pairs), on every
    core this process may use; a token is a position of the batch across all
    H heads, so the rate is head-tokens / H / seconds.  A one-thread time of
    one (sequence, head) sizes the sample and is reported beside it."""
    cores = host_cores()
    one_s, one_ht = time_oracle(inp, [0], [0], threads=1)
    seqs, heads = oracle_block(inp, int(max(cores, target_s * cores / max(one_s, 1e-4))))
    dt, ht = time_oracle(inp, seqs, heads, threads=cores)
    return {"value": ht / inp.H / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(seqs)} sequences x {len(heads)} heads of the workload, whole sequences ({ht} "
                      f"head-tokens, {dt:.1f} s of float64 work on {cores} threads); tokens = head-tokens / H",
            "cpu_model": cpu_model(), "affinity_cores": cores,
            "single_thread": {"value": one_ht / inp.H / one_s, "unit": "tokens/s",
                              "sample": f"sequence 0, head 0 ({one_ht} head-tokens, {one_s:.2f} s, 1 thread)"}}


HEADLINE = "Complex-KDA chunked forward B=8 H=16 T=8192 d_k=d_v=128 chunk=64 bf16, fp32 state, zero initial state"


def reference_arm(args, world, rank):
    """The oracle, as it stands, on the host cores: the headline workload, metric
    and unit.  A reference step is the float64 recurrence over a fixed sample of
    the workload -- as many whole (sequence, head) pairs as there are cores, so
    that each step takes about a second -- and it is timed whole: ms_per_step is
    the wall time of one such step, value = head-tokens / H / seconds."""
    if rank != 0:
        return
    inp = W.ckda_bf16(0)
    cores = host_cores()
    seqs, heads = oracle_block(inp, cores)
    head_tokens = None
    times = []
    for i in range(args.warmup + args.steps):
        dt, head_tokens = time_oracle(inp, seqs, heads, threads=cores)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = head_tokens * len(times) / inp.H / total
    sample = (f"{len(seqs)} sequences x {len(heads)} heads of the workload per step, whole sequences "
              f"({head_tokens} head-tokens, float64 on {cores} threads, {cpu_model()}); tokens = head-tokens / H")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy, cast to bf16; the oracle reads the same values in float64)",
            "config": {"workload": HEADLINE, "global_batch": inp.B, "seq_len": inp.T, "heads": inp.H,
                       "parallelism": "host cores", "step": "a bounded sample of the workload (see cpu_baseline)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def chunk_line(name, inp, r, world, steps, traffic_key=None):
    """The JSON fields of one timed chunked workload."""
    value = r["tokens_per_step"] * world * steps / r["total_s"]
    line = {"workload": name, "value": value, "unit": UNIT, "ms_per_step": r["total_s"] / steps * 1e3,
            "p50_ms": r["p50_ms"], "p95_ms": r["p95_ms"], "p99_ms": r["p99_ms"], "form": r["form"],
            "gpu_launches": steps * r["kernels_per_step"],
            "roofline": {"bound": "hbm", "achieved": r["hbm"]["achieved"], "peak": r["hbm"]["peak"], "unit": "GB/s",
                         "frac": r["hbm"]["frac"],
                         "traffic": (measured_traffic(traffic_key, CHUNK_SOURCES).get("dram_bytes_per_launch")
                                     if traffic_key else None),
                         "kernel": ("kda_chunk_fwd, split form: preparation + chain kernels timed as one call"
                                    if r["form"] == "split" else "kda_chunk_fwd, fused form: one kernel"),
                         "alg_bytes_per_launch": r["alg"]["bytes"]},
            "tensor": {"achieved": r["tensor"]["achieved"], "peak": r["tensor"]["peak"], "unit": "TFLOP/s",
                       "frac": r["tensor"]["frac"], "alg_flops_per_launch": r["alg"]["flops"]}}
    if "e2e" in r:
        e = r["e2e"]
        line["e2e"] = {"value": r["tokens_per_step"] * world * steps / e["total_s"], "unit": UNIT,
                       "h2d_bytes_per_step": e["h2d_bytes_per_step"], "d2h_bytes_per_step": e["d2h_bytes_per_step"]}
    return line


# ---------------------------------------------------------------------------

ONLY = {
    "ckda": (HEADLINE, lambda seed: W.ckda_bf16(seed)),
    "kda": ("KDA-range chunked forward B=4 H=16 T=4096 d=128 chunk=64 bf16", lambda seed: W.kda_bf16(seed)),
    "rda": ("RDA packed documents: 16 docs of U[512,4096] tokens, H=32", lambda seed: W.varlen_bf16("rda", seed)),
    "gdn2": ("GDN-2 packed documents: 16 docs of U[512,4096] tokens, H=32",
             lambda seed: W.varlen_bf16("gdn2", seed)),
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--extra", action="store_true",
                    help="also time the forward from gate logits and raw keys, with state snapshots, and rank-2 steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--backward-steps", type=int, default=20)
    ap.add_argument("--form", choices=sorted(FORM_FLAGS), default="auto",
                    help="form of the tensor-core chunked path (auto = the library's shape-based choice)")
    ap.add_argument("--only", choices=sorted(ONLY) + ["backward", "decode"], default=None,
                    help="time one workload alone (no e2e, no other workloads, no CPU baseline; for profiler "
                         "captures) and print its line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world, rank, local = dist_setup() if args.impl == "ours" else (int(os.environ.get("WORLD_SIZE", "1")),
                                                                   int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return

    import linear_rnn_delta_b200  # noqa: F401  (fails loudly if the library is missing)
    peaks = load_peaks()
    seed = rank_workload_seed(rank)
    fflags = FORM_FLAGS[args.form]
    if args.only == "backward":
        r = run_backward_workload(W.kda_bf16(seed), args.backward_steps, args.warmup, world, rank)
        if rank == 0:
            print(json.dumps(r))
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.only == "decode":
        r = run_decode_workload(args.decode_steps, args.warmup, world, peaks, rank, e2e=False)
        if rank == 0:
            print(json.dumps(r))
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.only:
        name, mk = ONLY[args.only]
        x = mk(seed)
        r = run_chunk_workload(x, args.steps, args.warmup, world, peaks, e2e=False, flags=fflags)
        if rank == 0:
            print(json.dumps(chunk_line(name, x, r, world, args.steps)))
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    sampler = ClockSampler(local) if rank == 0 else None
    # the headline: Complex KDA, B=8 H=16 T=8192
    inp = W.ckda_bf16(seed)
    main_res = run_chunk_workload(inp, args.steps, args.warmup, world, peaks, sampler=sampler, flags=fflags)
    head = chunk_line(HEADLINE, inp, main_res, world, args.steps, f"chunk_fwd_ckda_8x16x8192_{main_res['form']}")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample_rate(inp)
    del inp
    # the other chunked workloads, each with its own roofline and end-to-end figures
    also = []
    for name, mk, key in (
            ("KDA-range chunked forward B=4 H=16 T=4096 d=128 chunk=64 bf16, zero initial state",
             lambda: W.kda_bf16(seed), "chunk_fwd_kda_4x16x4096"),
            ("RDA packed documents: 16 docs of U[512,4096] tokens, H=32 d=128 bf16, random initial states",
             lambda: W.varlen_bf16("rda", seed), "chunk_fwd_rda_varlen"),
            ("GDN-2 packed documents: 16 docs of U[512,4096] tokens, H=32 d=128 bf16, random initial states",
             lambda: W.varlen_bf16("gdn2", seed), "chunk_fwd_gdn2_varlen")):
        x = mk()
        r = run_chunk_workload(x, args.steps, args.warmup, world, peaks, flags=fflags)
        also.append(chunk_line(name, x, r, world, args.steps, f"{key}_{r['form']}"))
        del x
    decode = run_decode_workload(args.decode_steps, args.warmup, world, peaks, rank)
    bwd_inp = W.kda_bf16(seed)
    backward = run_backward_workload(bwd_inp, args.backward_steps, args.warmup, world, rank)
    del bwd_inp
    if args.extra:
        prep = lambda: W.make_chunk_inputs("kda", "standard", "bf16", B=4, T=4096, H=16, d_k=128, d_v=128,
                                           seed=seed, logits=True, raw_k=True)
        for name, mk, xflags in (
                ("KDA B=4 H=16 T=4096 bf16 from gate logits and raw keys (in-kernel activations, L2 norm)",
                 prep, 16 | 32),
                ("KDA B=4 H=16 T=4096 bf16 with fp32 state snapshots after every 64 tokens",
                 lambda: W.kda_bf16(seed), "states")):
            x = mk()
            r = run_chunk_workload(x, args.steps, args.warmup, world, peaks, e2e=False,
                                   flags=fflags | (xflags if xflags != "states" else 0), states=xflags == "states")
            also.append(chunk_line(name, x, r, world, args.steps))
            del x
        x = W.make_rank2_inputs("kda", "standard", "bf16", B=4, T=2048, H=16, d_k=128, d_v=128, seed=seed)
        r = run_rank2_workload(x, args.steps, args.warmup, world)
        also.append({"workload": "KDA rank-2 steps (two sub-steps per token) B=4 H=16 T=2048 d=128 bf16: "
                                 "q/alpha expansion + chunked forward over 4096 sub-tokens + o gather",
                     "value": r["tokens_per_step"] * world * args.steps / r["total_s"], "unit": UNIT,
                     "ms_per_step": r["total_s"] / args.steps * 1e3})
        r = run_rank2_backward_workload(x, args.backward_steps, args.warmup, world, rank)
        also.append({"workload": "gradients of KDA rank-2 steps B=4 H=16 T=2048 d=128 bf16 inputs, fp32 "
                                 "arithmetic: d_o spread + rank-1 backward over 4096 sub-tokens + dq/dalpha gathers",
                     "value": r["tokens_per_step"] * world * args.backward_steps / r["total_s"], "unit": UNIT,
                     "ms_per_step": r["total_s"] / args.backward_steps * 1e3})
        del x
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy draws, bf16; per-rank seed)",
        "config": {"workload": HEADLINE, "global_batch": 8 * world, "seq_len": 8192, "heads": 16,
                   "parallelism": f"dp{world}", "l2": "inputs 1.08 GB per step > L2 126 MB, no flush"},
        "p50_ms": head["p50_ms"], "p95_ms": head["p95_ms"], "p99_ms": head["p99_ms"],
        "roofline": dict(head["roofline"], peak_source=peaks["source"], form=head["form"]),
        "tensor": head["tensor"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": main_res["clocks"],
        "also": also,
        "decode": decode,
        "backward": backward,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
