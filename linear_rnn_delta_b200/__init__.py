"""B200 (sm_100a) library for the gated delta-rule recurrence with channel-wise
decay: KDA, Complex KDA, RDA and GDN-2.

This module is a thin ctypes binding over the C ABI in ``include/kda.h``
(``libkda.so``, built in-tree by ``python linear_rnn_delta_b200/build.py``).
It only marshals arguments: it reads shapes and device pointers off torch
tensors, picks the caller's current CUDA stream, and allocates outputs the
caller did not pass.  Every step of the recurrence runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback, and importing this module
fails if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Union

import torch

__all__ = ["kda_chunk_fwd", "kda_chunk_bwd", "KdaChunkFunction", "kda_chunk_fwd_rank2", "kda_chunk_bwd_rank2",
           "kda_decode_step",
           "kda_check_gates", "kda_check_seqlens", "kda_device_status", "kda_error_string", "kda_version",
           "KdaError", "VARIANTS", "RANGES", "LIB_PATH", "FLAG_VALIDATE_RANGE", "FLAG_FORCE_SCAN",
           "FLAG_FORCE_FUSED", "FLAG_FORCE_SPLIT", "FLAG_GATE_LOGITS", "FLAG_L2NORM_K", "FLAG_DEBUG_STALL",
           "DEVICE_WAIT_TIMEOUT", "DEVICE_SLOT_MISSING", "num_chunk_slots", "chunk_slot"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")

VARIANTS = {"kda": 0, "rda": 1, "gdn2": 2}
RANGES = {"standard": 0, "extended": 1}
_DTYPES = {torch.bfloat16: 0, torch.float32: 1}
FLAG_VALIDATE_RANGE = 1  # check gates and cu_seqlens on the device first (synchronous); refuse on a violation
FLAG_FORCE_SCAN = 2    # token-by-token CUDA scan even where the tensor-core path applies
FLAG_FORCE_FUSED = 4   # tensor-core path, single fused kernel
FLAG_FORCE_SPLIT = 8   # tensor-core path, preparation kernel + chain kernel
FLAG_GATE_LOGITS = 16  # alpha and gates given as logits; the kernels apply the activations
FLAG_L2NORM_K = 32     # k given unnormalised; the kernels L2-normalise it per token and head
FLAG_DEBUG_STALL = 64  # testing aid (with FLAG_FORCE_SPLIT): one chain CTA's first wait runs out
DEVICE_WAIT_TIMEOUT = 1   # kda_device_status bits
DEVICE_SLOT_MISSING = 2

_vp = ctypes.c_void_p
_i = ctypes.c_int


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python linear_rnn_delta_b200/build.py` "
                          "(the recurrence has no implementation other than its CUDA kernels)")
    lib = ctypes.CDLL(LIB_PATH)
    for name in ("kda_chunk_fwd", "kda_chunk_fwd_ws", "kda_chunk_fwd_workspace_size", "kda_chunk_bwd",
                 "kda_chunk_bwd_workspace_size", "kda_chunk_fwd_rank2", "kda_chunk_fwd_rank2_workspace_size",
                 "kda_chunk_bwd_rank2", "kda_chunk_bwd_rank2_workspace_size",
                 "kda_decode_step", "kda_check_gates", "kda_check_seqlens", "kda_device_status", "kda_error_string",
                 "kda_last_error_detail", "kda_version"):
        if not hasattr(lib, name):
            raise ImportError(f"{LIB_PATH} lacks {name}: it is stale, rebuild it with "
                              "`python linear_rnn_delta_b200/build.py`")
    lib.kda_chunk_fwd.restype = _i
    lib.kda_chunk_fwd.argtypes = [_i] * 8 + [_vp] * 6 + [_vp, _i, _vp, _vp, _vp, _i, ctypes.c_uint, _vp]
    lib.kda_chunk_fwd_ws.restype = _i
    lib.kda_chunk_fwd_ws.argtypes = ([_i] * 8 + [_vp] * 6 + [_vp, _i, _vp, _vp, _vp, _vp, _i, _vp, ctypes.c_size_t,
                                                            ctypes.c_uint, _vp])
    lib.kda_chunk_fwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_chunk_fwd_workspace_size.argtypes = [_i] * 9 + [ctypes.c_uint]
    lib.kda_chunk_bwd.restype = _i
    lib.kda_chunk_bwd.argtypes = ([_i] * 8 + [_vp] * 6 + [_vp, _i, _vp] + [_vp, _vp] + [_vp] * 7 +
                                  [_vp, ctypes.c_size_t, ctypes.c_uint, _vp])
    lib.kda_chunk_bwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_chunk_bwd_workspace_size.argtypes = [_i] * 8
    lib.kda_chunk_fwd_rank2.restype = _i
    lib.kda_chunk_fwd_rank2.argtypes = ([_i] * 8 + [_vp] * 6 + [_vp, _i, _vp, _vp, _vp, _i, _vp, ctypes.c_size_t,
                                         ctypes.c_uint, _vp])
    lib.kda_chunk_fwd_rank2_workspace_size.restype = ctypes.c_size_t
    lib.kda_chunk_fwd_rank2_workspace_size.argtypes = [_i] * 9 + [ctypes.c_uint]
    lib.kda_chunk_bwd_rank2.restype = _i
    lib.kda_chunk_bwd_rank2.argtypes = lib.kda_chunk_bwd.argtypes
    lib.kda_chunk_bwd_rank2_workspace_size.restype = ctypes.c_size_t
    lib.kda_chunk_bwd_rank2_workspace_size.argtypes = [_i] * 8
    lib.kda_decode_step.restype = _i
    lib.kda_decode_step.argtypes = [_i] * 7 + [_vp] * 6 + [_vp, _vp, ctypes.c_uint, _vp]
    lib.kda_check_gates.restype = _i
    lib.kda_check_gates.argtypes = [_i, _i, _i, ctypes.c_longlong, _i, _vp, _vp, _vp, _vp]
    lib.kda_check_seqlens.restype = _i
    lib.kda_check_seqlens.argtypes = [_vp, _i, ctypes.c_longlong, _vp, _vp]
    lib.kda_device_status.restype = _i
    lib.kda_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint)]
    lib.kda_error_string.restype = ctypes.c_char_p
    lib.kda_error_string.argtypes = [_i]
    lib.kda_last_error_detail.restype = ctypes.c_char_p
    lib.kda_last_error_detail.argtypes = []
    lib.kda_version.restype = _i
    lib.kda_version.argtypes = []
    return lib


lib = _load()


class KdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = lib.kda_last_error_detail().decode(errors="replace")
        super().__init__(f"{where}: {lib.kda_error_string(code).decode()} -- {detail}")


def kda_error_string(code: int) -> str:
    return lib.kda_error_string(int(code)).decode()


def kda_version() -> int:
    return int(lib.kda_version())


def _code(table, x, what):
    if isinstance(x, str):
        if x not in table:
            raise ValueError(f"unknown {what} {x!r}; expected one of {sorted(table)}")
        return table[x]
    return int(x)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else _vp(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return _vp(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(t: Optional[torch.Tensor], name: str, dtype, shape, device):
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def kda_chunk_fwd(variant: Union[str, int], gate_range: Union[str, int], q: torch.Tensor, k: torch.Tensor,
                  v: torch.Tensor, alpha: torch.Tensor, g1: torch.Tensor, g2: Optional[torch.Tensor] = None,
                  cu_seqlens: Optional[torch.Tensor] = None, initial_state: Optional[torch.Tensor] = None,
                  final_state: Union[torch.Tensor, bool, None] = True, o: Optional[torch.Tensor] = None,
                  chunk_size: int = 64, flags: int = 0, stream=None,
                  chunk_states: Union[torch.Tensor, bool, None] = None):
    """Chunked forward of the recurrence over whole sequences (C: kda_chunk_fwd_ws,
    with the split form's workspace taken from torch's caching allocator).

    q, k, alpha [B,T,H,d_k]; v [B,T,H,d_v]; g1/g2 per variant (KDA: beta
    [B,T,H], g2 None; RDA: e, w [B,T,H]; GDN-2: b [B,T,H,d_k], w [B,T,H,d_v]);
    cu_seqlens int32 [N+1] (B == 1) or None; initial_state fp32 [N,H,d_k,d_v]
    or None.  ``final_state`` True allocates it, a tensor is written in place,
    None/False skips it.  ``chunk_states`` (True allocates fp32
    [num_chunk_slots(B, T, N), H, d_k, d_v]) receives the state after every 64
    tokens of each sequence and after its last token, at ``chunk_slot``.
    Returns (o, final_state or None), plus chunk_states when requested.
    """
    var = _code(VARIANTS, variant, "variant")
    rng = _code(RANGES, gate_range, "gate_range")
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,d_k]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"dtype {dt} unsupported (bf16 or fp32)")
    _check(q, "q", dt, (B, T, H, dk), dev)
    _check(k, "k", dt, (B, T, H, dk), dev)
    _check(v, "v", dt, (B, T, H, dv), dev)
    _check(alpha, "alpha", dt, (B, T, H, dk), dev)
    if var == 2:
        _check(g1, "g1 (b)", dt, (B, T, H, dk), dev)
        _check(g2, "g2 (w)", dt, (B, T, H, dv), dev)
    else:
        _check(g1, "g1", dt, (B, T, H), dev)
        if var == 1:
            _check(g2, "g2 (w)", dt, (B, T, H), dev)
    if var != 0 and g2 is None:
        raise ValueError("RDA and GDN-2 need g2 (write gate)")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    _check(initial_state, "initial_state", torch.float32, (N, H, dk, dv), dev)
    if final_state is True:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif final_state is False:
        final_state = None
    _check(final_state, "final_state", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _check(o, "o", dt, (B, T, H, dv), dev)
    want_states = chunk_states is not None and chunk_states is not False
    if chunk_states is True:
        chunk_states = torch.empty((num_chunk_slots(B, T, N), H, dk, dv), dtype=torch.float32, device=dev)
    elif chunk_states is False:
        chunk_states = None
    _check(chunk_states, "chunk_states", torch.float32, (num_chunk_slots(B, T, N), H, dk, dv), dev)
    # workspace of the split form, from torch's caching allocator (no per-call device allocation)
    ws_bytes = lib.kda_chunk_fwd_workspace_size(_DTYPES[dt], B, T, H, dk, dv, int(cu_seqlens is not None), N,
                                                int(chunk_size), int(flags))
    ws = None
    if ws_bytes:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        if stream is not None and stream != torch.cuda.current_stream(dev):
            ws.record_stream(stream)
    rc = lib.kda_chunk_fwd_ws(var, rng, _DTYPES[dt], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                              _ptr(g1), _ptr(g2), _ptr(cu_seqlens), N, _ptr(initial_state), _ptr(final_state),
                              _ptr(chunk_states), _ptr(o), int(chunk_size), _ptr(ws),
                              ws_bytes if ws is not None else 0, int(flags), _stream(stream, dev))
    if rc != 0:
        raise KdaError(rc, "kda_chunk_fwd")
    if want_states:
        return o, final_state, chunk_states
    return o, final_state


def kda_chunk_bwd(variant: Union[str, int], gate_range: Union[str, int], q: torch.Tensor, k: torch.Tensor,
                  v: torch.Tensor, alpha: torch.Tensor, g1: torch.Tensor, g2: Optional[torch.Tensor], d_o: torch.Tensor,
                  d_final_state: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
                  initial_state: Optional[torch.Tensor] = None, d_initial_state: bool = True, stream=None):
    """Gradients of the forward recurrence (C: kda_chunk_bwd), for a loss with
    dL/do = d_o ([B,T,H,d_v], the inputs' dtype) and dL/dS_final =
    d_final_state (fp32 [N,H,d_k,d_v] or None for zero).  Inputs as for
    kda_chunk_fwd (no flags).  Returns fp32 (dq, dk, dv, dalpha, dg1, dg2,
    d_initial_state) shaped like q, k, v, alpha, g1, g2 (None for KDA) and the
    state (None unless ``d_initial_state``)."""
    var = _code(VARIANTS, variant, "variant")
    rng = _code(RANGES, gate_range, "gate_range")
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,d_k]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"dtype {dt} unsupported (bf16 or fp32)")
    for t, name, shape in ((q, "q", (B, T, H, dk)), (k, "k", (B, T, H, dk)), (v, "v", (B, T, H, dv)),
                           (alpha, "alpha", (B, T, H, dk)), (d_o, "d_o", (B, T, H, dv)),
                           (g1, "g1", (B, T, H, dk) if var == 2 else (B, T, H))):
        _check(t, name, dt, shape, dev)
    if var != 0:
        if g2 is None:
            raise ValueError("RDA and GDN-2 need g2 (write gate)")
        _check(g2, "g2", dt, (B, T, H, dv) if var == 2 else (B, T, H), dev)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    _check(initial_state, "initial_state", torch.float32, (N, H, dk, dv), dev)
    _check(d_final_state, "d_final_state", torch.float32, (N, H, dk, dv), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = [torch.empty(t.shape, **f32) for t in (q, k, v, alpha, g1)]
    grads.append(torch.empty(g2.shape, **f32) if var != 0 else None)
    grads.append(torch.empty((N, H, dk, dv), **f32) if d_initial_state else None)
    ws_bytes = lib.kda_chunk_bwd_workspace_size(_DTYPES[dt], B, T, H, dk, dv, int(cu_seqlens is not None), N)
    if ws_bytes == 0:
        raise KdaError(1, "kda_chunk_bwd_workspace_size")
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if stream is not None and stream != torch.cuda.current_stream(dev):
        ws.record_stream(stream)
    rc = lib.kda_chunk_bwd(var, rng, _DTYPES[dt], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                           _ptr(g1), _ptr(g2), _ptr(cu_seqlens), N, _ptr(initial_state), _ptr(d_o),
                           _ptr(d_final_state), *[_ptr(x) for x in grads], _ptr(ws), ws_bytes, 0,
                           _stream(stream, dev))
    if rc != 0:
        raise KdaError(rc, "kda_chunk_bwd")
    return tuple(grads)


class KdaChunkFunction(torch.autograd.Function):
    """Differentiable forward: ``KdaChunkFunction.apply(variant, gate_range, q,
    k, v, alpha, g1, g2, cu_seqlens, initial_state)`` returns (o, final_state)
    from kda_chunk_fwd; the backward calls kda_chunk_bwd and casts each
    gradient to its input's dtype."""

    @staticmethod
    def forward(ctx, variant, gate_range, q, k, v, alpha, g1, g2=None, cu_seqlens=None, initial_state=None):
        o, sf = kda_chunk_fwd(variant, gate_range, q, k, v, alpha, g1, g2, cu_seqlens=cu_seqlens,
                              initial_state=initial_state)
        ctx.save_for_backward(q, k, v, alpha, g1, g2, cu_seqlens, initial_state)
        ctx.kda = (variant, gate_range)
        return o, sf

    @staticmethod
    def backward(ctx, d_o, d_sf):
        q, k, v, alpha, g1, g2, cu_seqlens, initial_state = ctx.saved_tensors
        d_o = q.new_zeros(*q.shape[:3], v.shape[-1]) if d_o is None else d_o.contiguous()
        grads = kda_chunk_bwd(*ctx.kda, q, k, v, alpha, g1, g2, d_o.to(q.dtype),
                              None if d_sf is None else d_sf.float().contiguous(), cu_seqlens, initial_state,
                              d_initial_state=initial_state is not None and ctx.needs_input_grad[9])
        casts = [None if g is None else g.to(x.dtype)
                 for g, x in zip(grads, (q, k, v, alpha, g1, g2, initial_state))]
        return (None, None, *casts[:6], None, casts[6])


def kda_chunk_fwd_rank2(variant: Union[str, int], gate_range: Union[str, int], q: torch.Tensor, k: torch.Tensor,
                        v: torch.Tensor, alpha: torch.Tensor, g1: torch.Tensor, g2: Optional[torch.Tensor] = None,
                        cu_seqlens: Optional[torch.Tensor] = None, initial_state: Optional[torch.Tensor] = None,
                        final_state: Union[torch.Tensor, bool, None] = True, o: Optional[torch.Tensor] = None,
                        chunk_size: int = 64, flags: int = 0, stream=None):
    """Rank-2 steps (C: kda_chunk_fwd_rank2): per token the decay alpha_t,
    then two erase/write sub-steps, then o_t = S_t^T q_t.  q, alpha
    [B,T,H,d_k]; k [B,T,2,H,d_k]; v [B,T,2,H,d_v]; g1 / g2 with the sub-step
    axis after T ([B,T,2,H] or GDN-2's [B,T,2,H,d]).  Other arguments as for
    kda_chunk_fwd (no gate logits).  Returns (o, final_state or None)."""
    var = _code(VARIANTS, variant, "variant")
    rng = _code(RANGES, gate_range, "gate_range")
    if q.dim() != 4 or k.dim() != 5:
        raise ValueError("q must be [B,T,H,d_k] and k [B,T,2,H,d_k]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"dtype {dt} unsupported (bf16 or fp32)")
    _check(q, "q", dt, (B, T, H, dk), dev)
    _check(alpha, "alpha", dt, (B, T, H, dk), dev)
    _check(k, "k", dt, (B, T, 2, H, dk), dev)
    _check(v, "v", dt, (B, T, 2, H, dv), dev)
    _check(g1, "g1", dt, (B, T, 2, H, dk) if var == 2 else (B, T, 2, H), dev)
    if var != 0:
        if g2 is None:
            raise ValueError("RDA and GDN-2 need g2 (write gate)")
        _check(g2, "g2", dt, (B, T, 2, H, dv) if var == 2 else (B, T, 2, H), dev)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    _check(initial_state, "initial_state", torch.float32, (N, H, dk, dv), dev)
    if final_state is True:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif final_state is False:
        final_state = None
    _check(final_state, "final_state", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _check(o, "o", dt, (B, T, H, dv), dev)
    ws_bytes = lib.kda_chunk_fwd_rank2_workspace_size(_DTYPES[dt], B, T, H, dk, dv, int(cu_seqlens is not None), N,
                                                      int(chunk_size), int(flags))
    if ws_bytes == 0:
        raise KdaError(1, "kda_chunk_fwd_rank2_workspace_size")
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if stream is not None and stream != torch.cuda.current_stream(dev):
        ws.record_stream(stream)
    rc = lib.kda_chunk_fwd_rank2(var, rng, _DTYPES[dt], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                 _ptr(g1), _ptr(g2), _ptr(cu_seqlens), N, _ptr(initial_state), _ptr(final_state),
                                 _ptr(o), int(chunk_size), _ptr(ws), ws_bytes, int(flags), _stream(stream, dev))
    if rc != 0:
        raise KdaError(rc, "kda_chunk_fwd_rank2")
    return o, final_state


def kda_chunk_bwd_rank2(variant: Union[str, int], gate_range: Union[str, int], q: torch.Tensor, k: torch.Tensor,
                        v: torch.Tensor, alpha: torch.Tensor, g1: torch.Tensor, g2: Optional[torch.Tensor],
                        d_o: torch.Tensor, d_final_state: Optional[torch.Tensor] = None,
                        cu_seqlens: Optional[torch.Tensor] = None, initial_state: Optional[torch.Tensor] = None,
                        d_initial_state: bool = True, stream=None):
    """Gradients of rank-2 steps (C: kda_chunk_bwd_rank2).  Inputs as for
    kda_chunk_fwd_rank2, d_o [B,T,H,d_v] in their dtype, d_final_state fp32
    [N,H,d_k,d_v] or None.  Returns fp32 (dq, dk, dv, dalpha, dg1, dg2,
    d_initial_state) shaped like q, k, v, alpha, g1, g2 (None for KDA) and the
    state (None unless ``d_initial_state``)."""
    var = _code(VARIANTS, variant, "variant")
    rng = _code(RANGES, gate_range, "gate_range")
    if q.dim() != 4 or k.dim() != 5:
        raise ValueError("q must be [B,T,H,d_k] and k [B,T,2,H,d_k]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"dtype {dt} unsupported (bf16 or fp32)")
    for t, name, shape in ((q, "q", (B, T, H, dk)), (alpha, "alpha", (B, T, H, dk)), (d_o, "d_o", (B, T, H, dv)),
                           (k, "k", (B, T, 2, H, dk)), (v, "v", (B, T, 2, H, dv)),
                           (g1, "g1", (B, T, 2, H, dk) if var == 2 else (B, T, 2, H))):
        _check(t, name, dt, shape, dev)
    if var != 0:
        if g2 is None:
            raise ValueError("RDA and GDN-2 need g2 (write gate)")
        _check(g2, "g2", dt, (B, T, 2, H, dv) if var == 2 else (B, T, 2, H), dev)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    _check(initial_state, "initial_state", torch.float32, (N, H, dk, dv), dev)
    _check(d_final_state, "d_final_state", torch.float32, (N, H, dk, dv), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = [torch.empty(t.shape, **f32) for t in (q, k, v, alpha, g1)]
    grads.append(torch.empty(g2.shape, **f32) if var != 0 else None)
    grads.append(torch.empty((N, H, dk, dv), **f32) if d_initial_state else None)
    ws_bytes = lib.kda_chunk_bwd_rank2_workspace_size(_DTYPES[dt], B, T, H, dk, dv, int(cu_seqlens is not None), N)
    if ws_bytes == 0:
        raise KdaError(1, "kda_chunk_bwd_rank2_workspace_size")
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if stream is not None and stream != torch.cuda.current_stream(dev):
        ws.record_stream(stream)
    rc = lib.kda_chunk_bwd_rank2(var, rng, _DTYPES[dt], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                 _ptr(g1), _ptr(g2), _ptr(cu_seqlens), N, _ptr(initial_state), _ptr(d_o),
                                 _ptr(d_final_state), *[_ptr(x) for x in grads], _ptr(ws), ws_bytes, 0,
                                 _stream(stream, dev))
    if rc != 0:
        raise KdaError(rc, "kda_chunk_bwd_rank2")
    return tuple(grads)


def num_chunk_slots(B: int, T: int, N: int) -> int:
    """Chunk slots of a [B, T] token layout with N sequences: N + ceil(B*T / 64)."""
    return N + (B * T + 63) // 64


def chunk_slot(n: int, c: int, row0: int) -> int:
    """Slot of chunk c (tokens [64c, 64c+64)) of sequence n whose first token
    is row ``row0`` of the packed token order (cu_seqlens[n], or n*T)."""
    return n + row0 // 64 + c


def kda_decode_step(variant: Union[str, int], gate_range: Union[str, int], q: torch.Tensor, k: torch.Tensor,
                    v: torch.Tensor, alpha: torch.Tensor, g1: torch.Tensor, g2: Optional[torch.Tensor],
                    state: torch.Tensor, o: Optional[torch.Tensor] = None, flags: int = 0, stream=None):
    """One decode step for N sequences (C: kda_decode_step); ``state`` fp32
    [N,H,d_k,d_v] is updated in place.  q, k, alpha [N,H,d_k]; v [N,H,d_v].
    Returns o [N,H,d_v]."""
    var = _code(VARIANTS, variant, "variant")
    rng = _code(RANGES, gate_range, "gate_range")
    if q.dim() != 3:
        raise ValueError("q must be [N,H,d_k]")
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"dtype {dt} unsupported (bf16 or fp32)")
    _check(q, "q", dt, (N, H, dk), dev)
    _check(k, "k", dt, (N, H, dk), dev)
    _check(v, "v", dt, (N, H, dv), dev)
    _check(alpha, "alpha", dt, (N, H, dk), dev)
    if var == 2:
        _check(g1, "g1 (b)", dt, (N, H, dk), dev)
        _check(g2, "g2 (w)", dt, (N, H, dv), dev)
    else:
        _check(g1, "g1", dt, (N, H), dev)
        if var == 1:
            _check(g2, "g2 (w)", dt, (N, H), dev)
    if var != 0 and g2 is None:
        raise ValueError("RDA and GDN-2 need g2 (write gate)")
    _check(state, "state", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((N, H, dv), dtype=dt, device=dev)
    _check(o, "o", dt, (N, H, dv), dev)
    rc = lib.kda_decode_step(var, rng, _DTYPES[dt], N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                             _ptr(g1), _ptr(g2), _ptr(state), _ptr(o), int(flags), _stream(stream, dev))
    if rc != 0:
        raise KdaError(rc, "kda_decode_step")
    return o


def kda_check_gates(variant: Union[str, int], gate_range: Union[str, int], alpha: torch.Tensor,
                    g1: torch.Tensor, stream=None) -> int:
    """Number of gate values outside the declared range (C: kda_check_gates).
    Synchronises the stream to read the count back."""
    var = _code(VARIANTS, variant, "variant")
    rng = _code(RANGES, gate_range, "gate_range")
    dk = alpha.shape[-1]
    n_tok = alpha.numel() // dk
    dev = alpha.device
    count = torch.empty((1,), dtype=torch.int32, device=dev)
    st = _stream(stream, dev)
    rc = lib.kda_check_gates(var, rng, _DTYPES[alpha.dtype], n_tok, dk, _ptr(alpha.contiguous()),
                             _ptr(g1.contiguous()), _ptr(count), st)
    if rc != 0:
        raise KdaError(rc, "kda_check_gates")
    return int(count.item())


def kda_check_seqlens(cu_seqlens: torch.Tensor, total_tokens: int, stream=None) -> int:
    """Number of violations of the cu_seqlens contract (cu[0] = 0,
    non-decreasing, cu[N] = total_tokens), counted on the device (C:
    kda_check_seqlens).  Synchronises the stream to read the count back."""
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
    dev = cu_seqlens.device
    count = torch.empty((1,), dtype=torch.int32, device=dev)
    cu = cu_seqlens.contiguous()
    rc = lib.kda_check_seqlens(_ptr(cu), cu.numel() - 1, int(total_tokens), _ptr(count), _stream(stream, dev))
    if rc != 0:
        raise KdaError(rc, "kda_check_seqlens")
    return int(count.item())


def kda_device_status(stream=None, device=None):
    """(status code, failure bits) of the library's kernels on the current
    device since the previous query (C: kda_device_status): waits for
    ``stream``, then reads and clears the word.  Code 0 = no failure, 5 =
    KDA_ERR_DEVICE_TIMEOUT (bits DEVICE_WAIT_TIMEOUT, DEVICE_SLOT_MISSING)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    bits = ctypes.c_uint(0)
    rc = lib.kda_device_status(_stream(stream, dev), ctypes.byref(bits))
    if rc not in (0, 5):
        raise KdaError(rc, "kda_device_status")
    return rc, int(bits.value)
