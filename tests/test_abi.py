"""C-ABI surface checks that need no GPU.

The library loads without a driver, exports every function include/kda.h
declares, and rejects bad arguments on the host before any launch.  Every
call below is built so that validation fails first: fake pointers are never
dereferenced and nothing reaches the device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("linear_rnn_delta_b200_build",
                                                  os.path.join(ROOT, "linear_rnn_delta_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)   # by path: importing the package loads the library being built
    build.build()
    import linear_rnn_delta_b200 as k
    return k.lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(kda_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("kda_chunk_fwd", "kda_decode_step", "kda_error_string", "kda_version"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libkda.so does not export {name}"


def test_version_and_error_strings(lib):
    assert lib.kda_version() >= 100
    for code in range(6):
        s = lib.kda_error_string(code).decode()
        assert s.startswith("KDA_")
    assert "unknown" in lib.kda_error_string(99).decode()


# A fake, 16-byte-aligned, never-dereferenced device address.
P = ctypes.c_void_p(0x10000)
BAD = ctypes.c_void_p(0x10008)  # misaligned


def fwd(lib, **kw):
    a = dict(variant=0, gate_range=0, dtype=0, B=1, T=8, H=1, dk=128, dv=128, q=P, k=P, v=P, alpha=P, g1=P,
             g2=None, cu=None, nseq=0, s0=None, sf=None, o=P, chunk=64, flags=0, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd(a["variant"], a["gate_range"], a["dtype"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                             a["q"], a["k"], a["v"], a["alpha"], a["g1"], a["g2"], a["cu"], a["nseq"], a["s0"],
                             a["sf"], a["o"], a["chunk"], a["flags"], a["stream"])


def fwd_ws(lib, ws=None, ws_bytes=0, **kw):
    a = dict(variant=0, gate_range=0, dtype=0, B=1, T=8, H=1, dk=128, dv=128, q=P, k=P, v=P, alpha=P, g1=P,
             g2=None, cu=None, nseq=0, s0=None, sf=None, o=P, chunk=64, flags=0, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd_ws(a["variant"], a["gate_range"], a["dtype"], a["B"], a["T"], a["H"], a["dk"],
                                a["dv"], a["q"], a["k"], a["v"], a["alpha"], a["g1"], a["g2"], a["cu"], a["nseq"],
                                a["s0"], a["sf"], a.get("cs"), a["o"], a["chunk"], ws, ws_bytes, a["flags"],
                                a["stream"])


SLOT_BYTES = 82944


@pytest.mark.parametrize("args,expect", [
    ((0, 4, 4096, 16, 128, 128, 0, 0, 64), (4 + 4 * 4096 // 64) * 16 * SLOT_BYTES),   # fixed length: N = B
    ((0, 1, 1000, 32, 128, 128, 1, 16, 64), (16 + 16) * 32 * SLOT_BYTES),           # varlen: N = num_seqs
    ((0, 2, 65, 3, 128, 128, 0, 0, 64), (2 + 3) * 3 * SLOT_BYTES),                    # ragged: ceil(130 / 64)
    ((0, 2, 0, 3, 128, 128, 0, 0, 64), 2 * 3 * SLOT_BYTES),                           # T = 0
    ((1, 4, 4096, 16, 128, 128, 0, 0, 64), 0),      # fp32: token scan, no workspace
    ((0, 4, 4096, 16, 64, 128, 0, 0, 64), 0),       # d_k = 64: token scan
    ((0, 4, 4096, 16, 128, 128, 0, 0, 32), 0),      # chunk 32: token scan
    ((0, 2, 64, 2, 128, 128, 1, 3, 64), 0),         # cu_seqlens with B != 1
    ((0, 0, 64, 2, 128, 128, 0, 0, 64), 0),         # B = 0
])
def test_workspace_size_of_the_split_form(lib, args, expect):
    assert lib.kda_chunk_fwd_workspace_size(*args, 8) == expect


def test_workspace_size_other_forms(lib):
    args = (0, 4, 4096, 16, 128, 128, 0, 0, 64)
    assert lib.kda_chunk_fwd_workspace_size(*args, 4) == 0       # fused forced
    assert lib.kda_chunk_fwd_workspace_size(*args, 2) == 0       # scan forced
    assert lib.kda_chunk_fwd_workspace_size(*args, 4 | 8) == 0   # contradictory flags


def test_forced_split_needs_a_workspace(lib):
    need = lib.kda_chunk_fwd_workspace_size(0, 1, 8, 1, 128, 128, 0, 0, 64, 8)
    assert fwd_ws(lib, flags=8) == INVALID                          # none
    assert fwd_ws(lib, ws=P, ws_bytes=need - 16, flags=8) == INVALID  # too small
    assert fwd_ws(lib, ws=BAD, ws_bytes=need, flags=8) == INVALID     # misaligned
    assert fwd_ws(lib, ws=P, ws_bytes=need, flags=4 | 8) == INVALID   # both forms forced
    assert fwd_ws(lib, flags=1 << 9) == INVALID
    assert fwd_ws(lib, cs=BAD) == INVALID                            # misaligned chunk_states


def dec(lib, **kw):
    a = dict(variant=0, gate_range=1, dtype=0, N=4, H=2, dk=128, dv=128, q=P, k=P, v=P, alpha=P, g1=P, g2=None,
             state=P, o=P, flags=0, stream=None)
    a.update(kw)
    return lib.kda_decode_step(a["variant"], a["gate_range"], a["dtype"], a["N"], a["H"], a["dk"], a["dv"],
                               a["q"], a["k"], a["v"], a["alpha"], a["g1"], a["g2"], a["state"], a["o"],
                               a["flags"], a["stream"])


INVALID, UNSUPPORTED = 1, 2


@pytest.mark.parametrize("kw,code", [
    (dict(variant=3), INVALID), (dict(variant=-1), INVALID), (dict(gate_range=2), INVALID),
    (dict(dtype=5), INVALID), (dict(B=0), INVALID), (dict(T=-1), INVALID), (dict(H=0), INVALID),
    (dict(dk=48), UNSUPPORTED), (dict(dv=256), UNSUPPORTED), (dict(dk=0), INVALID),
    (dict(q=None), INVALID), (dict(k=None), INVALID), (dict(o=None), INVALID), (dict(g1=None), INVALID),
    (dict(alpha=BAD), INVALID), (dict(v=BAD), INVALID),
    (dict(variant=1), INVALID),             # RDA without g2
    (dict(variant=2, g2=BAD), INVALID),     # GDN-2 with misaligned g2
    (dict(chunk=48), UNSUPPORTED), (dict(chunk=256), UNSUPPORTED),
    (dict(flags=1 << 7), INVALID),
    (dict(flags=4 | 8), INVALID),           # fused and split forms both forced
    (dict(cu=P, nseq=2, B=2), INVALID),     # cu_seqlens needs B == 1
    (dict(cu=P, nseq=0), INVALID),
    (dict(cu=ctypes.c_void_p(0x10002), nseq=1), INVALID),
    (dict(s0=BAD), INVALID), (dict(sf=BAD), INVALID),
])
def test_chunk_fwd_rejects_bad_arguments(lib, kw, code):
    assert fwd(lib, **kw) == code
    assert len(lib.kda_last_error_detail()) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(N=0), INVALID), (dict(H=0), INVALID), (dict(variant=9), INVALID), (dict(dk=24), UNSUPPORTED),
    (dict(state=None), INVALID), (dict(state=BAD), INVALID), (dict(o=None), INVALID),
    (dict(variant=1), INVALID), (dict(flags=1 << 8), INVALID), (dict(q=BAD), INVALID),
])
def test_decode_step_rejects_bad_arguments(lib, kw, code):
    assert dec(lib, **kw) == code


def test_check_gates_rejects_bad_arguments(lib):
    assert lib.kda_check_gates(0, 0, 0, 10, 128, P, P, None, None) == INVALID
    assert lib.kda_check_gates(0, 3, 0, 10, 128, P, P, P, None) == INVALID
    assert lib.kda_check_gates(0, 0, 0, -1, 128, P, P, P, None) == INVALID


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    """The Python binding has no fallback: a missing libkda.so is an ImportError."""
    import importlib.util
    src = os.path.join(ROOT, "linear_rnn_delta_b200", "__init__.py")
    pkg = tmp_path / "kda_copy"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("kda_copy", str(pkg / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


# ---- rank-2 steps ---------------------------------------------------------------------------

def test_rank2_workspace_size(lib):
    # fp32 (token scan: no chunk workspace): q2, alpha2 [1,200,3,64], o2 [1,200,3,32], doubled cu_seqlens
    up = lambda x: (x + 255) // 256 * 256
    expect = 2 * up(600 * 64 * 4) + up(600 * 32 * 4) + up(5 * 4)
    assert lib.kda_chunk_fwd_rank2_workspace_size(1, 1, 100, 3, 64, 32, 1, 4, 64, 0) == expect
    assert lib.kda_chunk_fwd_rank2_workspace_size(1, 2, 100, 3, 64, 32, 1, 4, 64, 0) == 0    # cu_seqlens, B != 1
    assert lib.kda_chunk_fwd_rank2_workspace_size(1, 1, -1, 3, 64, 32, 0, 1, 64, 0) == 0
    assert lib.kda_chunk_fwd_rank2_workspace_size(1, 1, 8, 3, 48, 32, 0, 1, 64, 0) == 0      # d_k = 48
    assert lib.kda_chunk_fwd_rank2_workspace_size(0, 1, 8, 3, 128, 128, 0, 1, 64, 4 | 8) == 0


def r2(lib, **kw):
    a = dict(variant=0, gate_range=0, dtype=1, B=1, T=8, H=2, dk=64, dv=32, q=P, k=P, v=P, alpha=P, g1=P, g2=None,
             cu=None, nseq=1, s0=None, sf=None, o=P, chunk=64, ws=P, ws_bytes=0, flags=0, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd_rank2(a["variant"], a["gate_range"], a["dtype"], a["B"], a["T"], a["H"], a["dk"],
                                   a["dv"], a["q"], a["k"], a["v"], a["alpha"], a["g1"], a["g2"], a["cu"], a["nseq"],
                                   a["s0"], a["sf"], a["o"], a["chunk"], a["ws"], a["ws_bytes"], a["flags"],
                                   a["stream"])


# As for the backward: the default workspace is too small, and the detail names the check that fired.
@pytest.mark.parametrize("kw,code,detail", [
    (dict(flags=16), UNSUPPORTED, b"logits"),   # the second sub-step's alpha = 1 has no logit
    (dict(T=-1), INVALID, b"T=-1"), (dict(B=0), INVALID, b"B=0"), (dict(dtype=7), INVALID, b"dtype"),
    (dict(dk=48), UNSUPPORTED, b"d_k=48"),
    (dict(q=None), INVALID, b"q is NULL"), (dict(alpha=BAD), INVALID, b"alpha"), (dict(o=None), INVALID, b"o is"),
    (dict(cu=ctypes.c_void_p(0x10002), nseq=1), INVALID, b"cu_seqlens"),
    (dict(ws=None), INVALID, b"workspace"),
    (dict(ws_bytes=16), INVALID, b"workspace"),
])
def test_rank2_rejects_bad_arguments(lib, kw, code, detail):
    assert r2(lib, **kw) == code
    assert detail in lib.kda_last_error_detail()


# ---- backward -------------------------------------------------------------------------------

def test_bwd_workspace_size(lib):
    # checkpoints: (N + ceil(B*T/64)) slots x H x d_k x d_v fp32, u_t: B*T*H*d_v fp32,
    # plus N*H*16*d_k*d_v fp32 replay states
    assert lib.kda_chunk_bwd_workspace_size(0, 2, 100, 3, 128, 128, 0, 2) == \
        (2 + 4) * 3 * 128 * 128 * 4 + 2 * 100 * 3 * 128 * 4 + 2 * 3 * 16 * 128 * 128 * 4
    assert lib.kda_chunk_bwd_workspace_size(1, 1, 10, 1, 16, 32, 1, 3) == \
        (3 + 1) * 1 * 16 * 32 * 4 + 10 * 32 * 4 + 3 * 1 * 64 * 16 * 32 * 4     # d_k = 16: every state of a chunk
    assert lib.kda_chunk_bwd_workspace_size(0, 2, 100, 3, 48, 128, 0, 2) == 0
    assert lib.kda_chunk_bwd_workspace_size(0, 2, 100, 3, 128, 128, 1, 2) == 0   # cu_seqlens needs B == 1


def bwd(lib, **kw):
    a = dict(variant=0, gate_range=0, dtype=0, B=1, T=8, H=2, dk=128, dv=128, q=P, k=P, v=P, alpha=P, g1=P,
             g2=None, cu=None, nseq=1, s0=None, d_o=P, dsf=None, dq=P, dk_=P, dv_=P, dalpha=P, dg1=P, dg2=None,
             ds0=None, ws=P, ws_bytes=16, flags=0, stream=None)
    a.update(kw)
    return lib.kda_chunk_bwd(a["variant"], a["gate_range"], a["dtype"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                             a["q"], a["k"], a["v"], a["alpha"], a["g1"], a["g2"], a["cu"], a["nseq"], a["s0"],
                             a["d_o"], a["dsf"], a["dq"], a["dk_"], a["dv_"], a["dalpha"], a["dg1"], a["dg2"],
                             a["ds0"], a["ws"], a["ws_bytes"], a["flags"], a["stream"])


# Every call keeps a far too small workspace, so nothing could launch even if a check were missing;
# the error detail shows which check fired.
@pytest.mark.parametrize("kw,code,detail", [
    (dict(flags=16), INVALID, b"flags"), (dict(d_o=None), INVALID, b"d_o"), (dict(d_o=BAD), INVALID, b"o is not"),
    (dict(dq=None), INVALID, b"dq"), (dict(dalpha=BAD), INVALID, b"dalpha"),
    (dict(variant=1, g2=P), INVALID, b"dg2"),        # RDA without dg2
    (dict(dsf=BAD), INVALID, b"d_final_state"), (dict(ds0=BAD), INVALID, b"d_initial_state"),
    (dict(dk=48), UNSUPPORTED, b"d_k"), (dict(T=-1), INVALID, b"T=-1"),
    (dict(ws=None), INVALID, b"workspace"), (dict(ws=BAD), INVALID, b"workspace"),
    (dict(ws_bytes=16), INVALID, b"workspace"),
])
def test_bwd_rejects_bad_arguments(lib, kw, code, detail):
    assert bwd(lib, **kw) == code
    assert detail in lib.kda_last_error_detail()


def test_debug_stall_needs_the_split_form(lib):
    """The failure-path testing aid only exists in the split form: other forms refuse it on the host."""
    assert fwd(lib, flags=64) == 1                     # no FORCE_SPLIT
    assert fwd(lib, flags=64 | 4) == 1                 # fused
    assert fwd(lib, flags=64 | 8 | 2) == 1             # scan
    assert "DEBUG_STALL" in lib.kda_last_error_detail().decode()
    assert fwd_ws(lib, flags=64 | 8, dtype=1) == 1     # fp32 runs the scan


def test_validate_flag_is_refused_where_it_has_no_meaning(lib):
    r2 = lib.kda_chunk_fwd_rank2
    r2.restype = ctypes.c_int
    assert r2(0, 0, 0, 1, 8, 1, 128, 128, P, P, P, P, P, None, None, 0, None, None, P, 64, P, 1 << 30, 1,
              None) == 2


def test_check_seqlens_rejects_bad_arguments(lib):
    lib.kda_check_seqlens.restype = ctypes.c_int
    assert lib.kda_check_seqlens(None, 2, 10, P, None) == 1
    assert lib.kda_check_seqlens(P, 0, 10, P, None) == 1
    assert lib.kda_check_seqlens(P, 2, -1, P, None) == 1
    assert lib.kda_check_seqlens(P, 2, 10, None, None) == 1
    assert lib.kda_check_seqlens(ctypes.c_void_p(0x10002), 2, 10, P, None) == 1


def test_rank2_bwd_rejects_bad_arguments(lib):
    """Every check happens before anything is launched (fake pointers never reach a kernel)."""
    f = lib.kda_chunk_bwd_rank2
    f.restype = ctypes.c_int

    def call(flags=0, q=P, d_o=P, dq=P, ws=P, ws_bytes=1 << 30, dk=128):
        return f(0, 0, 0, 1, 8, 1, dk, 128, q, P, P, P, P, None, None, 0, None, d_o, None, dq, P, P, P, P, None,
                 None, ws, ctypes.c_size_t(ws_bytes), flags, None)
    assert call(flags=1) == INVALID
    assert call(q=None) == INVALID
    assert call(d_o=BAD) == INVALID
    assert call(dq=None) == INVALID
    assert call(ws_bytes=16) == INVALID
    assert call(ws=BAD) == INVALID
    assert call(dk=48) == UNSUPPORTED
    lib.kda_chunk_bwd_rank2_workspace_size.restype = ctypes.c_size_t
    need = lib.kda_chunk_bwd_rank2_workspace_size(0, 1, 8, 1, 128, 128, 0, 1)
    assert need > lib.kda_chunk_bwd_workspace_size(0, 1, 16, 1, 128, 128, 0, 1)
