"""Seeded synthetic inputs for the gated delta-rule recurrence.

This module only draws random numbers and shapes them into the workloads the
recurrence is exercised on (KDA, Complex KDA, RDA, GDN-2; chunked forward and
single-token decode).  It holds none of the recurrence's arithmetic: the GPU
library and the CPU oracle both consume what it returns, and neither is
imported here.

Recipe (all draws float32 from ``numpy.random.default_rng``, fixed order
q, k, v, alpha-pre-activation, gate pre-activations; then k is L2-normalised
per token and head; then everything is cast to the run dtype with
round-to-nearest-even).  Both sides read the SAME cast values: bf16 -> float64
is exact, so the oracle sees exactly what the kernels see.

Gate activations per workload (Complex KDA arXiv abstract, "gates in [-1,1]
and beta in [0,2]"; KDA/RDA/GDN-2 equations on the Raon-1-mini-preview
discussion page):

* KDA range:      alpha = exp(-softplus(x)) = sigmoid(-x) in (0,1),
                  beta = sigmoid(y) in (0,1)
* Complex KDA:    alpha = tanh(2x) in [-1,1] (negative values and values
                  near zero included), beta = 2*sigmoid(y) in (0,2)
* RDA:            alpha = sigmoid(-x); e, w = sigmoid(.) drawn independently
* GDN-2:          alpha = sigmoid(-x); b in R^{d_k}, w in R^{d_v}, each
                  sigmoid(.) per channel
* tiny CKDA:      alpha ~ U[-1,1], beta ~ U[0,2], fp32

Gate tensors follow the library's argument convention: ``g1`` is beta (KDA),
e (RDA) or the vector b (GDN-2); ``g2`` is None (KDA), w (RDA) or the vector
w (GDN-2).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

VARIANTS = {"kda": 0, "rda": 1, "gdn2": 2}
RANGES = {"standard": 0, "extended": 1}
DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


@dataclasses.dataclass
class ChunkInputs:
    """One chunked-forward problem, all tensors on the host in the run dtype.

    Layouts: q, k, alpha [B,T,H,d_k]; v [B,T,H,d_v]; gates [B,T,H] (scalar)
    or [B,T,H,d_k] / [B,T,H,d_v] (GDN-2 vectors).  With ``cu_seqlens`` B is 1
    and the documents are packed along T.  ``initial_state`` is fp32
    [N,H,d_k,d_v] or None (zeros).
    """
    variant: str
    gate_range: str
    dtype: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    alpha: torch.Tensor
    g1: torch.Tensor
    g2: Optional[torch.Tensor]
    cu_seqlens: Optional[torch.Tensor]
    initial_state: Optional[torch.Tensor]
    chunk_size: int = 64
    logits: bool = False     # alpha and gates are stored as logits (KDA_FLAG_GATE_LOGITS)
    l2norm_k: bool = False   # k is stored unnormalised (KDA_FLAG_L2NORM_K)

    @property
    def num_seqs(self) -> int:
        return self.B if self.cu_seqlens is None else int(self.cu_seqlens.numel() - 1)

    def seq_bounds(self, n: int) -> tuple[int, int, int]:
        """(batch row, first token, token count) of sequence n."""
        if self.cu_seqlens is None:
            return n, 0, self.T
        c = self.cu_seqlens
        return 0, int(c[n]), int(c[n + 1] - c[n])

    def tensors(self):
        return [t for t in (self.q, self.k, self.v, self.alpha, self.g1, self.g2) if t is not None]

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.tensors())


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _l2norm_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    n = np.maximum(n, 1e-12)
    return (x / n).astype(np.float32)


def _cast(x: Optional[np.ndarray], dtype: str) -> Optional[torch.Tensor]:
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(DTYPES[dtype])


def _alpha_gates(rng, variant, gate_range, lead, d_k, d_v, uniform_tiny=False, logits=False):
    """Draw alpha and the variant's gates for leading shape ``lead``.  With
    ``logits`` the same draws are returned as logits (alpha's logit x with
    alpha = exp(-softplus(x)), or tanh(x) for the extended range; gate logits
    y with gate = sigmoid(y), or 2 sigmoid(y) extended)."""
    a_pre = rng.standard_normal(lead + (d_k,), dtype=np.float32)
    if logits:
        if uniform_tiny:
            raise ValueError("uniform_tiny draws have no logits")
        ext = gate_range == "extended"
        x = (2.0 * a_pre if ext else a_pre).astype(np.float32)
        if variant == "kda":
            return x, rng.standard_normal(lead, dtype=np.float32), None
        if variant == "rda":
            return x, rng.standard_normal(lead, dtype=np.float32), rng.standard_normal(lead, dtype=np.float32)
        if variant == "gdn2":
            return (x, rng.standard_normal(lead + (d_k,), dtype=np.float32),
                    rng.standard_normal(lead + (d_v,), dtype=np.float32))
        raise ValueError(f"unknown variant {variant!r}")
    if uniform_tiny:
        alpha = rng.uniform(-1.0, 1.0, lead + (d_k,)).astype(np.float32)
        g1 = rng.uniform(0.0, 2.0, lead).astype(np.float32)
        return alpha, g1, None
    if variant == "kda":
        g_pre = rng.standard_normal(lead, dtype=np.float32)
        if gate_range == "extended":
            alpha = np.tanh(2.0 * a_pre).astype(np.float32)
            g1 = 2.0 * _sigmoid(g_pre)
        else:
            alpha = _sigmoid(-a_pre)          # exp(-softplus(x)) == sigmoid(-x)
            g1 = _sigmoid(g_pre)
        return alpha, g1, None
    if variant == "rda":
        e_pre = rng.standard_normal(lead, dtype=np.float32)
        w_pre = rng.standard_normal(lead, dtype=np.float32)
        alpha = np.tanh(2.0 * a_pre).astype(np.float32) if gate_range == "extended" else _sigmoid(-a_pre)
        return alpha, _sigmoid(e_pre), _sigmoid(w_pre)
    if variant == "gdn2":
        b_pre = rng.standard_normal(lead + (d_k,), dtype=np.float32)
        w_pre = rng.standard_normal(lead + (d_v,), dtype=np.float32)
        alpha = np.tanh(2.0 * a_pre).astype(np.float32) if gate_range == "extended" else _sigmoid(-a_pre)
        return alpha, _sigmoid(b_pre), _sigmoid(w_pre)
    raise ValueError(f"unknown variant {variant!r}")


def make_chunk_inputs(variant: str = "kda", gate_range: str = "standard", dtype: str = "bf16",
                      B: int = 1, T: int = 64, H: int = 2, d_k: int = 16, d_v: int = 16,
                      seed: int = 0, chunk_size: int = 64, doc_lens=None,
                      init_state: str = "zero", init_std: float = 0.02,
                      uniform_tiny: bool = False, logits: bool = False, raw_k: bool = False) -> ChunkInputs:
    """Draw one chunked-forward problem.

    ``doc_lens`` packs documents of those lengths along T (B must be 1) and
    returns the matching ``cu_seqlens`` (int32, exclusive prefix sum).
    ``init_state`` is "zero" (None is passed, the library starts from 0) or
    "random" (fp32 N(0, init_std) per sequence and head).  ``logits`` stores
    alpha and the gates as logits, ``raw_k`` stores k unnormalised (the
    library's input preparation turns them into the recurrence's inputs).
    """
    rng = np.random.default_rng(seed)
    cu = None
    if doc_lens is not None:
        doc_lens = [int(x) for x in doc_lens]
        B, T = 1, int(sum(doc_lens))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(doc_lens)]).astype(np.int32))
    lead = (B, T, H)
    q = rng.standard_normal(lead + (d_k,), dtype=np.float32)
    k = rng.standard_normal(lead + (d_k,), dtype=np.float32)
    v = rng.standard_normal(lead + (d_v,), dtype=np.float32)
    alpha, g1, g2 = _alpha_gates(rng, variant, gate_range, lead, d_k, d_v, uniform_tiny, logits)
    if not raw_k:
        k = _l2norm_rows(k)
    n_seqs = B if cu is None else len(doc_lens)
    s0 = None
    if init_state == "random":
        s0 = torch.from_numpy(
            (init_std * rng.standard_normal((n_seqs, H, d_k, d_v), dtype=np.float32)).astype(np.float32))
    elif init_state != "zero":
        raise ValueError(init_state)
    return ChunkInputs(variant, gate_range, dtype, B, T, H, d_k, d_v,
                       _cast(q, dtype), _cast(k, dtype), _cast(v, dtype), _cast(alpha, dtype),
                       _cast(g1, dtype), _cast(g2, dtype), cu, s0, chunk_size, logits, raw_k)


def grad_outputs(inp: ChunkInputs, seed: int = 0, d_final: bool = True):
    """Incoming gradients for a backward pass over ``inp``: d_o [B,T,H,d_v]
    ~ N(0,1) in the run dtype and dL/dS_final fp32 [N,H,d_k,d_v] ~ N(0, 0.1^2)
    (None unless ``d_final``), from ``default_rng((seed, 7))``."""
    rng = np.random.default_rng((seed, 7))
    d_o = _cast(rng.standard_normal((inp.B, inp.T, inp.H, inp.d_v), dtype=np.float32), inp.dtype)
    dsf = None
    if d_final:
        dsf = torch.from_numpy(0.1 * rng.standard_normal((inp.num_seqs, inp.H, inp.d_k, inp.d_v),
                                                         dtype=np.float32))
    return d_o, dsf


@dataclasses.dataclass
class Rank2Inputs(ChunkInputs):
    """A rank-2 (two sub-steps per token) problem.  q, alpha [B,T,H,d_k] per
    token; k [B,T,2,H,d_k], v [B,T,2,H,d_v] and the gates ([B,T,2,H] scalars
    or [B,T,2,H,d] GDN-2 vectors) carry the sub-step axis after T."""


def make_rank2_inputs(variant: str = "kda", gate_range: str = "standard", dtype: str = "bf16",
                      B: int = 1, T: int = 64, H: int = 2, d_k: int = 16, d_v: int = 16, seed: int = 0,
                      doc_lens=None, init_state: str = "zero", init_std: float = 0.02) -> Rank2Inputs:
    """Draw one rank-2 problem with the rank-1 recipe: q, then k and v of both
    sub-steps, then alpha per token, then the gates per sub-step (same
    distributions as ``make_chunk_inputs``); keys L2-normalised per sub-step;
    from ``default_rng((seed, 2))``."""
    rng = np.random.default_rng((seed, 2))
    cu = None
    if doc_lens is not None:
        doc_lens = [int(x) for x in doc_lens]
        B, T = 1, int(sum(doc_lens))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(doc_lens)]).astype(np.int32))
    q = rng.standard_normal((B, T, H, d_k), dtype=np.float32)
    k = _l2norm_rows(rng.standard_normal((B, T, 2, H, d_k), dtype=np.float32))
    v = rng.standard_normal((B, T, 2, H, d_v), dtype=np.float32)
    alpha, _, _ = _alpha_gates(rng, variant, gate_range, (B, T, H), d_k, d_v)
    _, g1, g2 = _alpha_gates(rng, variant, gate_range, (B, T, 2, H), d_k, d_v)
    n_seqs = B if cu is None else len(doc_lens)
    s0 = None
    if init_state == "random":
        s0 = torch.from_numpy(init_std * rng.standard_normal((n_seqs, H, d_k, d_v), dtype=np.float32))
    elif init_state != "zero":
        raise ValueError(init_state)
    return Rank2Inputs(variant, gate_range, dtype, B, T, H, d_k, d_v, _cast(q, dtype), _cast(k, dtype),
                       _cast(v, dtype), _cast(alpha, dtype), _cast(g1, dtype), _cast(g2, dtype), cu, s0)


# ---------------------------------------------------------------------------
# The named workloads (shapes and distributions of the recurrence's benchmark
# configurations).  Each returns ChunkInputs; the decode workload is separate.
# ---------------------------------------------------------------------------

def tiny_ckda(seed: int = 0) -> ChunkInputs:
    """Tiny Complex-KDA case: B=1, H=2, T=64, d=16, fp32, chunk 16."""
    return make_chunk_inputs("kda", "extended", "f32", B=1, T=64, H=2, d_k=16, d_v=16,
                             seed=seed, chunk_size=16, uniform_tiny=True)


def kda_bf16(seed: int = 0, B: int = 4, T: int = 4096, H: int = 16) -> ChunkInputs:
    """KDA range, bf16: B=4, H=16, T=4096, d=128, chunk 64, zero initial state."""
    return make_chunk_inputs("kda", "standard", "bf16", B=B, T=T, H=H, d_k=128, d_v=128,
                             seed=seed, chunk_size=64)


def ckda_bf16(seed: int = 0, B: int = 8, T: int = 8192, H: int = 16) -> ChunkInputs:
    """Complex KDA full range, bf16: B=8, H=16, T=8192, d=128, chunk 64."""
    return make_chunk_inputs("kda", "extended", "bf16", B=B, T=T, H=H, d_k=128, d_v=128,
                             seed=seed, chunk_size=64)


def varlen_doc_lens(seed: int = 0, n_docs: int = 16, lo: int = 512, hi: int = 4096):
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi + 1, n_docs)]


def varlen_bf16(variant: str, seed: int = 0, H: int = 32, doc_lens=None) -> ChunkInputs:
    """RDA or GDN-2 varlen, bf16: 16 packed documents with lengths U[512,4096],
    H=32, d=128, random fp32 initial state N(0, 0.02), alpha in (0,1)."""
    assert variant in ("rda", "gdn2")
    if doc_lens is None:
        doc_lens = varlen_doc_lens(seed)
    return make_chunk_inputs(variant, "standard", "bf16", H=H, d_k=128, d_v=128, seed=seed,
                             chunk_size=64, doc_lens=doc_lens, init_state="random")


@dataclasses.dataclass
class DecodeInputs:
    """One decode step for N sequences: q,k,alpha [N,H,d_k]; v [N,H,d_v]; gates [N,H](,d)."""
    variant: str
    gate_range: str
    dtype: str
    N: int
    H: int
    d_k: int
    d_v: int
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    alpha: torch.Tensor
    g1: torch.Tensor
    g2: Optional[torch.Tensor]
    logits: bool = False
    l2norm_k: bool = False

    def tensors(self):
        return [t for t in (self.q, self.k, self.v, self.alpha, self.g1, self.g2) if t is not None]

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.tensors())


def decode_initial_state(N: int = 256, H: int = 32, d_k: int = 128, d_v: int = 128,
                         seed: int = 0, std: float = 0.02) -> torch.Tensor:
    """fp32 decode state [N,H,d_k,d_v] ~ N(0, std)."""
    rng = np.random.default_rng((seed, 1 << 20))
    return torch.from_numpy(std * rng.standard_normal((N, H, d_k, d_v), dtype=np.float32))


def decode_step_inputs(step: int, variant: str = "kda", gate_range: str = "extended",
                       dtype: str = "bf16", N: int = 256, H: int = 32, d_k: int = 128,
                       d_v: int = 128, seed: int = 0, logits: bool = False, raw_k: bool = False) -> DecodeInputs:
    """Per-step decode inputs from ``default_rng((seed, step))`` so any step can be
    regenerated independently (Complex KDA range by default)."""
    rng = np.random.default_rng((seed, step))
    lead = (N, H)
    q = rng.standard_normal(lead + (d_k,), dtype=np.float32)
    k = rng.standard_normal(lead + (d_k,), dtype=np.float32)
    v = rng.standard_normal(lead + (d_v,), dtype=np.float32)
    alpha, g1, g2 = _alpha_gates(rng, variant, gate_range, lead, d_k, d_v, logits=logits)
    if not raw_k:
        k = _l2norm_rows(k)
    return DecodeInputs(variant, gate_range, dtype, N, H, d_k, d_v, _cast(q, dtype), _cast(k, dtype),
                        _cast(v, dtype), _cast(alpha, dtype), _cast(g1, dtype), _cast(g2, dtype), logits, raw_k)


# ---------------------------------------------------------------------------
# Planted gates: inputs that force the chunked kernel's division-free
# (anchored) branch.  That branch serves every chunk in which some channel's
# chunk product of gates vanishes or underflows; random draws almost never
# produce one.  Each kind rewrites alpha of an existing problem in place of
# its draws (same seed -> same planting); nothing else changes.
# ---------------------------------------------------------------------------

PLANT_KINDS = ("zero", "tiny", "mixed", "negative")
TINY_GATE = 2.0 ** -6   # 19 such factors already fall below 2^-110; a chunk of 64 underflows fp32


def plant_gates(inp: ChunkInputs, kind: str, seed: int = 0, chunk: int = 64) -> ChunkInputs:
    """A copy of ``inp`` with alpha rewritten so that chosen 64-token chunks
    of every sequence contain vanishing gates:

    * "zero": alpha = 0 exactly at 3% of the (token, head, channel) entries of
      every chunk (erases those channels, as the recurrence defines);
    * "tiny": |alpha| = 2^-6 over whole chunks in 8 channels per head (signs
      random in the extended range), so their chunk products underflow;
    * "mixed": "zero" only in the odd chunks of each sequence, so fast and
      anchored chunks alternate within one sequence;
    * "negative": runs of 16 tokens with alpha = -1 or -0.999 in a quarter of
      the channels, plus one exact zero per chunk and head (extended range;
      in the standard range the runs use +1 and +0.999).
    Returns a new ChunkInputs; alpha keeps the run dtype (all planted values
    are bf16-representable except -0.999 / 0.999, rounded like any input)."""
    if kind not in PLANT_KINDS:
        raise ValueError(f"unknown planting {kind!r}; expected one of {PLANT_KINDS}")
    rng = np.random.default_rng((seed, 31))
    a = inp.alpha.float().numpy().copy()          # [B,T,H,d_k]
    B, T, H, dk = a.shape
    ext = inp.gate_range == "extended"
    starts = []
    for n in range(inp.num_seqs):
        b, t0, ln = inp.seq_bounds(n)
        for c in range((ln + chunk - 1) // chunk):
            starts.append((b, t0 + c * chunk, min(chunk, ln - c * chunk), c))
    for b, s, ln, c in starts:
        blk = a[b, s:s + ln]                       # view [ln, H, d_k]
        if kind in ("zero", "mixed"):
            if kind == "mixed" and c % 2 == 0:
                continue
            blk[rng.random(blk.shape) < 0.03] = 0.0
        elif kind == "tiny":
            for h in range(H):
                ch = rng.choice(dk, 8, replace=False)
                sign = rng.choice([-1.0, 1.0], (ln, 8)) if ext else np.ones((ln, 8))
                blk[:, h, ch] = sign * TINY_GATE
        else:   # negative
            mag = np.where(rng.random(blk.shape) < 0.5, 1.0, 0.999)
            run = np.zeros(blk.shape, dtype=bool)
            for h in range(H):
                ch = rng.choice(dk, dk // 4, replace=False)
                r0 = int(rng.integers(0, max(1, ln - 15)))
                run[r0:r0 + 16, h, ch] = True
            blk[run] = ((-1.0 if ext else 1.0) * mag)[run]
            for h in range(H):
                blk[int(rng.integers(ln)), h, int(rng.integers(dk))] = 0.0
    out = dataclasses.replace(inp)
    out.alpha = _cast(a, inp.dtype)
    return out


def plant_reflections(inp: ChunkInputs, seed: int = 0, chunk: int = 64, every: int = 2) -> ChunkInputs:
    """A copy of ``inp`` in which every ``every``-th 64-token chunk of each
    sequence (starting with the first) is rewritten into a run of strong,
    barely decaying reflections on correlated keys: k_t = normalise(c + 0.05
    n_t) around one direction c per (sequence, head), |alpha| in [0.97, 1]
    (random signs in the extended range), and erase gates near their top
    (beta / e, or every channel of GDN-2's b, in [0.9, 1] x the range's
    maximum).  The
    exact result is close to an orthogonal map; the bf16 WY form of such a
    chunk amplifies its operands' rounding, which is the case the chunked
    kernel hands to its exact token-by-token path.  Other chunks keep their
    draws.  Inputs stored as logits (``inp.logits``) get logits of such gates,
    raw keys (``inp.l2norm_k``) keep a random norm."""
    rng = np.random.default_rng((seed, 37))
    k = inp.k.float().numpy().copy()
    a = inp.alpha.float().numpy().copy()
    g1 = inp.g1.float().numpy().copy()
    B, T, H, dk = k.shape
    ext = inp.gate_range == "extended"
    top = 2.0 if ext else 1.0
    for n in range(inp.num_seqs):
        b, t0, ln = inp.seq_bounds(n)
        for c in range(0, (ln + chunk - 1) // chunk, every):
            s, e = t0 + c * chunk, t0 + min(ln, (c + 1) * chunk)
            L = e - s
            for h in range(H):
                cdir = rng.standard_normal(dk)
                kk = cdir[None, :] + 0.05 * rng.standard_normal((L, dk))
                kk /= np.linalg.norm(kk, axis=1, keepdims=True)
                if inp.l2norm_k:
                    kk *= rng.uniform(0.5, 3.0, (L, 1))
                k[b, s:e, h] = kk
                mag = rng.uniform(0.97, 1.0, (L, dk))
                sign = np.where(rng.random((L, dk)) < 0.3, -1.0, 1.0) if ext else np.ones((L, dk))
                al = mag * sign
                if inp.variant == "gdn2":
                    gate = top * rng.uniform(0.9, 1.0, (L, dk))
                else:
                    gate = top * rng.uniform(0.9, 1.0, L)
                if inp.logits:   # the logits of these gates (the library's activations inverted)
                    al = np.arctanh(np.clip(al, -0.9999, 0.9999)) if ext else np.log((1.0 - al + 1e-4) / al)
                    x = gate / top
                    gate = np.log(x / (1.0 - x + 1e-4))
                a[b, s:e, h] = al
                g1[b, s:e, h] = gate
    out = dataclasses.replace(inp)
    out.k, out.alpha, out.g1 = _cast(k, inp.dtype), _cast(a, inp.dtype), _cast(g1, inp.dtype)
    return out
