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
    from linear_rnn_delta_b200 import build
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
    for code in range(5):
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
    (dict(variant=1), INVALID), (dict(flags=1), INVALID), (dict(q=BAD), INVALID),
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
