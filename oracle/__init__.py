"""CPU oracle for the gated delta-rule recurrence (KDA / Complex KDA / RDA / GDN-2).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py``.  The GPU library never
imports it and it never imports the GPU library; the two share only the seeded
input generators in ``workloads``.

Three independent formulations, all float64:

* ``recurrence`` -- the plain-C step recurrence in ``kda_oracle.c`` (decay,
  residual u = m - S'^T a~, rank-one write, readout o_t = S_t^T q_t), OpenMP
  over (sequence, head).  This is THE oracle the GPU path is compared with.
* ``literal_recurrence`` -- NumPy, the state updates exactly as the
  Raon-1-mini-preview discussion page prints them: explicit d_k x d_k
  transition matrices (I - beta k k^T) Diag(alpha), (I - e k k^T) Diag(alpha),
  (I - k (b (.) k)^T) Diag(alpha) and write terms beta k v^T, w k v^T,
  k (w (.) v)^T.  Small inputs only.
* ``brute_force`` -- NumPy dense closed form of the unrolled recurrence,
  S_t = (prod_{s<=t} A_s) S_0 + sum_{s<=t} (prod_{s<r<=t} A_r) W_s, evaluated
  from scratch for every t.  Tiny inputs only.
* ``prepare`` -- the optional input preparation (gate activations from
  logits, L2 normalisation of k) in float64, applied before ``recurrence``
  when a problem stores logits or raw keys.
* ``recurrence_grad`` -- NumPy reverse mode of the step recurrence (every
  gradient of one sequence and head).
* ``recurrence_rank2`` -- NumPy rank-2 (DeltaProduct_2-style) steps: the
  decay once per token, then two erase/write sub-steps with their own keys,
  values and gates, then the readout.

Every function is pinned by ``tests/test_oracle_pins.py`` against properties
the pages fix (RDA = KDA when e = w; GDN-2 = RDA for constant vectors;
non-expansive Complex-KDA transitions; the exact 2D rotation) and textbook
special cases (causal linear attention, gated linear attention, overwrite
memory, Householder reflection).  No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

VARIANT_CODE = {"kda": 0, "rda": 1, "gdn2": 2}


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (float64, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-shared", "-fPIC", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_recurrence.restype = ctypes.c_int
        lib.oracle_recurrence.argtypes = [ctypes.c_int] * 6 + [dp] * 6 + [ip, ctypes.c_int] + [dp] * 3 + [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f64(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact upcast of bf16 / fp32
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _sigmoid(y: np.ndarray) -> np.ndarray:
    # 1 / (1 + e^-y) without overflow for large |y|
    e = np.exp(-np.abs(y))
    return np.where(y >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def _round_to(x, dtype: Optional[str]):
    if x is None or dtype is None:
        return x
    if dtype == "bf16":   # round to nearest even, as the input dtype stores it
        import torch
        return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


def prepare(gate_range: str, k, alpha, g1, g2=None, logits: bool = False, l2norm_k: bool = False,
            round_to: Optional[str] = None):
    """Input preparation on request, float64, from the stored values.

    ``logits``: alpha, g1, g2 hold logits.  Standard range: alpha =
    exp(-softplus(x)) and every gate (beta, e, w, GDN-2's b and w) =
    sigmoid(y); extended (Complex-KDA) range: alpha = tanh(x), gate =
    2 sigmoid(y) -- the gates' ranges (0,1] / [-1,1] and [0,1] / [0,2].
    ``l2norm_k``: k_t / max(||k_t||_2, 1e-6) along the last axis.
    ``round_to`` ("bf16" / "f32"): the prepared values are rounded to the
    input dtype, as a separate preparation pass would store them.
    Returns (k, alpha, g1, g2) as float64 arrays (g2 may be None).
    """
    k, alpha, g1, g2 = (_f64(x) for x in (k, alpha, g1, g2))
    if logits:
        ext = gate_range == "extended"
        alpha = np.tanh(alpha) if ext else np.exp(-np.logaddexp(0.0, alpha))
        scale = 2.0 if ext else 1.0
        g1 = scale * _sigmoid(g1)
        g2 = None if g2 is None else scale * _sigmoid(g2)
        alpha, g1, g2 = (_round_to(x, round_to) for x in (alpha, g1, g2))
    if l2norm_k:
        norm = np.sqrt(np.sum(k * k, axis=-1, keepdims=True))
        k = _round_to(k / np.maximum(norm, 1e-6), round_to)
    return k, alpha, g1, g2


def recurrence_arrays(variant: str, q, k, v, alpha, g1, g2=None, cu_seqlens=None,
                      initial_state=None, threads: int = 0, gate_range: str = "standard",
                      logits: bool = False, l2norm_k: bool = False, round_to: Optional[str] = None):
    """Step recurrence on float64 arrays with the library's layouts.

    q,k,alpha [B,T,H,dk]; v [B,T,H,dv]; g1/g2 per the variant; cu_seqlens
    optional int offsets (B must be 1); initial_state [N,H,dk,dv] or None.
    ``logits`` / ``l2norm_k`` run ``prepare`` first (``gate_range`` picks the
    activations, ``round_to`` the stored dtype of the prepared values).
    Returns (o [B,T,H,dv], final_state [N,H,dk,dv]) float64.
    """
    q, k, v, alpha, g1, g2 = (_f64(x) for x in (q, k, v, alpha, g1, g2))
    if logits or l2norm_k:
        k, alpha, g1, g2 = prepare(gate_range, k, alpha, g1, g2, logits, l2norm_k, round_to)
    s0 = _f64(initial_state)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    cu = None
    N = B
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                                             dtype=np.int32))
        N = cu.size - 1
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    sf = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().oracle_recurrence(
        VARIANT_CODE[variant], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(g1), _ptr(g2),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int)) if cu is not None else ctypes.POINTER(ctypes.c_int)(),
        N, _ptr(s0), _ptr(sf), _ptr(o), int(threads))
    if rc != 0:
        raise ValueError("oracle_recurrence rejected its arguments")
    return o, sf


def recurrence(inp, seqs: Optional[Sequence[int]] = None, heads: Optional[Sequence[int]] = None,
               threads: int = 0):
    """Oracle on a ``workloads.ChunkInputs`` problem, optionally restricted to
    some sequences and heads (they are independent, so a restriction is exact).

    Returns (o, final_state) float64.  Without a restriction o is [B,T,H,dv]
    and final_state [N,H,dk,dv]; with one, o is a dict {(n, h): [len, dv]} and
    final_state a dict {(n, h): [dk, dv]}.
    """
    pk = dict(gate_range=inp.gate_range, logits=getattr(inp, "logits", False),
              l2norm_k=getattr(inp, "l2norm_k", False), round_to=inp.dtype)
    if seqs is None and heads is None:
        return recurrence_arrays(inp.variant, inp.q, inp.k, inp.v, inp.alpha, inp.g1, inp.g2,
                                 inp.cu_seqlens, inp.initial_state, threads, **pk)
    seqs = list(range(inp.num_seqs)) if seqs is None else list(seqs)
    heads = list(range(inp.H)) if heads is None else list(heads)
    # gather every requested (sequence, head) as its own batch row, padded to the
    # longest length (padding rows are never read: cu_seqlens bounds them)
    parts = []
    for n in seqs:
        b, t0, ln = inp.seq_bounds(n)
        for h in heads:
            parts.append((n, h, b, t0, ln))
    lens = [p[4] for p in parts]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    tot = int(cu[-1])

    def gather(x, last):
        if x is None:
            return None
        out = np.zeros((1, tot, 1) + ((last,) if last else ()), dtype=np.float64)
        for i, (n, h, b, t0, ln) in enumerate(parts):
            sl = x[b, t0:t0 + ln, h]
            out[0, cu[i]:cu[i + 1], 0] = sl.detach().cpu().double().numpy() if hasattr(sl, "detach") else sl
        return out

    dk, dv = inp.d_k, inp.d_v
    g_last1 = dk if inp.variant == "gdn2" else 0
    g_last2 = dv if inp.variant == "gdn2" else 0
    s0 = None
    if inp.initial_state is not None:
        s0 = np.stack([inp.initial_state[n, h].double().numpy() for (n, h, *_r) in parts])[:, None]
    o, sf = recurrence_arrays(inp.variant, gather(inp.q, dk), gather(inp.k, dk), gather(inp.v, dv),
                              gather(inp.alpha, dk), gather(inp.g1, g_last1), gather(inp.g2, g_last2),
                              cu, s0, threads, **pk)
    o_d, s_d = {}, {}
    for i, (n, h, *_r) in enumerate(parts):
        o_d[(n, h)] = o[0, cu[i]:cu[i + 1], 0]
        s_d[(n, h)] = sf[i, 0]
    return o_d, s_d


# ---------------------------------------------------------------------------
# Literal product form and brute force (small inputs)
# ---------------------------------------------------------------------------

def transition_and_write(variant: str, k, v, alpha, g1, g2):
    """The pages' transition A_t (d_k x d_k) and write term W_t (d_k x d_v) for
    one token, exactly as the three update equations print them."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    D = np.diag(np.asarray(alpha, dtype=np.float64))
    I = np.eye(k.size)
    if variant == "kda":        # S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T
        beta = float(g1)
        return (I - beta * np.outer(k, k)) @ D, beta * np.outer(k, v)
    if variant == "rda":        # S_t = (I - e k k^T) Diag(alpha) S_{t-1} + w k v^T
        e, w = float(g1), float(g2)
        return (I - e * np.outer(k, k)) @ D, w * np.outer(k, v)
    if variant == "gdn2":       # S_t = (I - k (b (.) k)^T) Diag(alpha) S_{t-1} + k (w (.) v)^T
        b, w = np.asarray(g1, dtype=np.float64), np.asarray(g2, dtype=np.float64)
        return (I - np.outer(k, b * k)) @ D, np.outer(k, w * v)
    raise ValueError(variant)


def _tok(x, b, t, h):
    if x is None:
        return None
    y = x[b, t, h]
    return y.detach().cpu().double().numpy() if hasattr(y, "detach") else np.asarray(y, dtype=np.float64)


def literal_recurrence(variant: str, q, k, v, alpha, g1, g2=None, initial_state=None):
    """Fixed-length batches only.  Returns (o [B,T,H,dv], S_T [B,H,dk,dv])."""
    B, T, H, dk = tuple(q.shape)
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if initial_state is None else _f64(initial_state[b, h])
            for t in range(T):
                A, W = transition_and_write(variant, _tok(k, b, t, h), _tok(v, b, t, h), _tok(alpha, b, t, h),
                                            _tok(g1, b, t, h), _tok(g2, b, t, h))
                S = A @ S + W
                o[b, t, h] = S.T @ _tok(q, b, t, h)
            sf[b, h] = S
    return o, sf


def brute_force(variant: str, q, k, v, alpha, g1, g2=None, initial_state=None):
    """Dense unrolled form, recomputed from scratch at every t.  Returns (o, S_T)."""
    B, T, H, dk = tuple(q.shape)
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S0 = np.zeros((dk, dv)) if initial_state is None else _f64(initial_state[b, h])
            mats = [transition_and_write(variant, _tok(k, b, t, h), _tok(v, b, t, h), _tok(alpha, b, t, h),
                                         _tok(g1, b, t, h), _tok(g2, b, t, h)) for t in range(T)]
            for t in range(T):
                # S_t = (A_t ... A_0) S_0 + sum_s (A_t ... A_{s+1}) W_s
                P = np.eye(dk)
                for r in range(t + 1):
                    P = mats[r][0] @ P
                St = P @ S0
                for s in range(t + 1):
                    Q = np.eye(dk)
                    for r in range(s + 1, t + 1):
                        Q = mats[r][0] @ Q
                    St = St + Q @ mats[s][1]
                o[b, t, h] = St.T @ _tok(q, b, t, h)
                if t == T - 1:
                    sf[b, h] = St
    return o, sf


def chunk_states(inp, every: int = 64, threads: int = 0):
    """State after every ``every`` tokens of each sequence and after its last
    token, by running the step recurrence piece by piece from the previous
    piece's final state (continuation is exact).  Returns a dict
    {(n, c): [H, dk, dv] float64} for chunk c of sequence n.
    """
    names = ("q", "k", "v", "alpha", "g1", "g2")
    out = {}
    for n in range(inp.num_seqs):
        b, t0, ln = inp.seq_bounds(n)
        s = None if inp.initial_state is None else inp.initial_state[n:n + 1]
        for c in range((ln + every - 1) // every):
            a, e = t0 + c * every, t0 + min(ln, (c + 1) * every)
            piece = {nm: (None if getattr(inp, nm) is None else getattr(inp, nm)[b:b + 1, a:e]) for nm in names}
            _, sf = recurrence_arrays(inp.variant, piece["q"], piece["k"], piece["v"], piece["alpha"],
                                      piece["g1"], piece["g2"], None, s, threads, gate_range=inp.gate_range,
                                      logits=getattr(inp, "logits", False), l2norm_k=getattr(inp, "l2norm_k", False),
                                      round_to=inp.dtype)
            out[(n, c)] = sf[0]
            s = sf
    return out


# ---------------------------------------------------------------------------
# Gradients (reverse mode of the step recurrence)
# ---------------------------------------------------------------------------

def _gates(variant, k, v, g1, g2):
    """Erase direction a~ and written value m of every token (float64)."""
    if variant == "kda":
        return g1[..., None] * k, g1[..., None] * v
    if variant == "rda":
        return g1[..., None] * k, g2[..., None] * v
    return g1 * k, g2 * v


def recurrence_grad(variant: str, q, k, v, alpha, g1, g2, initial_state, do, dsf=None):
    """Gradients of L = sum(do * o) + sum(dsf * S_T) for ONE sequence and head.

    q, k, alpha [T, dk]; v [T, dv]; g1 / g2 per the variant ([T] scalars or
    [T, d] vectors, g2 None for KDA); initial_state [dk, dv] or None; do
    [T, dv]; dsf [dk, dv] or None.  Reverse mode of the step recurrence
      S' = Diag(alpha) S,  u = m - S'^T a~,  S = S' + k u^T,  o = S^T q,
    taken step by step backwards (the adjoint of each step written out).
    Returns a dict of float64 arrays: dq, dk, dv, dalpha, dg1, dg2 (None for
    KDA), ds0.
    """
    q, k, v, alpha, g1, g2, do = (_f64(x) for x in (q, k, v, alpha, g1, g2, do))
    T, dk = q.shape
    dv = v.shape[-1]
    at, m = _gates(variant, k, v, g1, g2)
    S = np.zeros((dk, dv)) if initial_state is None else _f64(initial_state).copy()
    states, us = [S.copy()], []
    for t in range(T):                                   # forward, keeping S_{t-1} and u_t
        Sp = alpha[t][:, None] * S
        u = m[t] - Sp.T @ at[t]
        S = Sp + np.outer(k[t], u)
        states.append(S.copy())
        us.append(u)
    G = np.zeros((dk, dv)) if dsf is None else _f64(dsf).copy()
    dq, dk_, dv_, da = (np.zeros_like(x) for x in (q, k, v, alpha))
    dat, dm = np.zeros_like(at), np.zeros_like(m)
    for t in range(T - 1, -1, -1):
        S_prev, S_t, u = states[t], states[t + 1], us[t]
        G = G + np.outer(q[t], do[t])                    # o_t = S_t^T q_t
        dq[t] = S_t @ do[t]
        du = G.T @ k[t]                                  # S_t = S' + k u^T
        dk_[t] = G @ u
        dSp = G - np.outer(at[t], du)                    # u = m - S'^T a~
        dm[t] = du
        Sp = alpha[t][:, None] * S_prev
        dat[t] = -(Sp @ du)
        da[t] = np.sum(S_prev * dSp, axis=1)             # S' = Diag(alpha) S_{t-1}
        G = alpha[t][:, None] * dSp
    if variant == "kda":
        dg1 = np.sum(k * dat, axis=1) + np.sum(v * dm, axis=1)
        dk_ += g1[:, None] * dat
        dv_ = g1[:, None] * dm
        dg2 = None
    elif variant == "rda":
        dg1 = np.sum(k * dat, axis=1)
        dg2 = np.sum(v * dm, axis=1)
        dk_ += g1[:, None] * dat
        dv_ = g2[:, None] * dm
    else:
        dg1 = k * dat
        dg2 = v * dm
        dk_ += g1 * dat
        dv_ = g2 * dm
    return {"dq": dq, "dk": dk_, "dv": dv_, "dalpha": da, "dg1": dg1, "dg2": dg2, "ds0": G}


def recurrence_rank2(variant: str, q, k, v, alpha, g1, g2=None, cu_seqlens=None, initial_state=None):
    """Rank-2 steps (two delta-rule transitions composed in one recurrent
    update, named as prior work in the Complex KDA arXiv abstract), with the
    channel-wise decay applied once per token, before the first sub-step:

      S <- Diag(alpha_t) S
      for s in (1, 2):  u = m_{t,s} - S^T a~_{t,s};  S <- S + k_{t,s} u^T
      o_t = S^T q_t

    (a~, m) per sub-step as in the rank-1 variants.  Layouts: q, alpha
    [B,T,H,dk]; k [B,T,2,H,dk]; v [B,T,2,H,dv]; g1 [B,T,2,H] (KDA beta, RDA e)
    or [B,T,2,H,dk] (GDN-2 b); g2 None (KDA), [B,T,2,H] (RDA w) or
    [B,T,2,H,dv] (GDN-2 w); cu_seqlens optional (B = 1); initial_state
    [N,H,dk,dv] or None.  Returns (o [B,T,H,dv], final_state [N,H,dk,dv]).
    Small inputs only (NumPy loop over tokens).
    """
    q, k, v, alpha, g1, g2 = (_f64(x) for x in (q, k, v, alpha, g1, g2))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        cu = [int(x) for x in np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens)]
        seqs = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    else:
        seqs = [(b, 0, T) for b in range(B)]
    s0 = _f64(initial_state)
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((len(seqs), H, dk, dv))
    for n, (b, t0, t1) in enumerate(seqs):
        S = np.zeros((H, dk, dv)) if s0 is None else s0[n].copy()
        for t in range(t0, t1):
            S = alpha[b, t][:, :, None] * S                                 # decay, once per token
            for sub in range(2):
                kk, vv = k[b, t, sub], v[b, t, sub]                         # [H, dk], [H, dv]
                if variant == "kda":
                    at, m = g1[b, t, sub][:, None] * kk, g1[b, t, sub][:, None] * vv
                elif variant == "rda":
                    at, m = g1[b, t, sub][:, None] * kk, g2[b, t, sub][:, None] * vv
                else:
                    at, m = g1[b, t, sub] * kk, g2[b, t, sub] * vv
                u = m - np.einsum("hij,hi->hj", S, at)                      # residual
                S = S + kk[:, :, None] * u[:, None, :]                      # rank-one write
            o[b, t] = np.einsum("hij,hi->hj", S, q[b, t])                   # readout after both sub-steps
        sf[n] = S
    return o, sf
