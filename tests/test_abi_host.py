"""Host-only checks of the C ABI: the library loads, exports every function
include/fa.h declares, and rejects bad arguments with the documented status
before launching anything (no GPU needed: every case below fails validation)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fa():
    import exact_io_aware_75_b200 as fa
    return fa


def header_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


def test_exports_match_header(fa):
    names = header_functions()
    assert names == sorted(fa.EXPORTS)
    lib = fa.library()
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(fa):
    for code in range(0, -7, -1):
        assert fa.status_string(code) != "unknown status"
    assert fa.status_string(-99) == "unknown status"
    assert fa.version() >= 100


P = 1 << 20   # a 16-byte aligned fake device address; never dereferenced


def fwd(fa, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=0, B=1, Hq=2, Hkv=2, N=128, d=64, causal=0, window=0,
             scale=0.125, o_dtype=0)
    a.update(kw)
    return fa.library().fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"],
                               a["Hkv"], a["N"], a["d"], a["causal"], a["window"],
                               a["scale"], a["o_dtype"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3, Hkv=2), -1), (dict(Hkv=0), -1), (dict(scale=0.0), -1),
    (dict(scale=float("inf")), -1), (dict(scale=float("nan")), -1), (dict(causal=2), -1),
    (dict(o_dtype=7), -1), (dict(d=96), -2), (dict(d=256), -2), (dict(window=5), -2),
    (dict(q=0), -1), (dict(o=0), -1), (dict(k=P + 8), -3), (dict(lse=P + 2), -3),
    (dict(B=-1), -1), (dict(N=-1), -1)])
def test_fwd_rejects(fa, kw, status):
    assert fwd(fa, **kw) == status


def test_fwd_empty_is_noop(fa):
    assert fwd(fa, N=0, q=0, k=0, v=0, o=0) == 0
    assert fwd(fa, B=0) == 0


def varlen(fa, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=0, cu=P, S=2, T=300, maxL=200, Hq=4, Hkv=2, d=128,
             causal=1, window=0, scale=0.1, o_dtype=0)
    a.update(kw)
    return fa.library().fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"],
                                      a["S"], a["T"], a["maxL"], a["Hq"], a["Hkv"], a["d"],
                                      a["causal"], a["window"], a["scale"], a["o_dtype"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(cu=0), -1), (dict(S=-1), -1), (dict(T=-5), -1), (dict(maxL=-1), -1),
    (dict(cu=P + 2), -3), (dict(Hq=5), -1), (dict(d=32), -2), (dict(causal=0, window=9), -2)])
def test_varlen_rejects(fa, kw, status):
    assert varlen(fa, **kw) == status


def test_varlen_empty_is_noop(fa):
    assert varlen(fa, S=0) == 0 and varlen(fa, T=0) == 0


def dec(fa, **kw):
    a = dict(q=P, kc=P, vc=P, bt=P, sl=P, o=P, lse=0, S=4, P=100, Hq=32, Hkv=8, d=128, ps=16,
             maxp=10, scale=0.1, ws=P, wsb=1 << 30)
    a.update(kw)
    return fa.library().fa_decode_paged(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["o"],
                                        a["lse"], a["S"], a["P"], a["Hq"], a["Hkv"], a["d"],
                                        a["ps"], a["maxp"], a["scale"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(ps=32), -2), (dict(d=80), -2), (dict(Hq=30), -1), (dict(bt=0), -1), (dict(sl=0), -1),
    (dict(ws=0), -4), (dict(wsb=16), -4), (dict(ws=P + 16), -3), (dict(q=P + 4), -3),
    (dict(maxp=0), -1), (dict(P=0), -1), (dict(S=-2), -1)])
def test_decode_rejects(fa, kw, status):
    assert dec(fa, **kw) == status


def test_decode_workspace_formula(fa):
    # partial O (fp32) and partial LSE per (sequence, chunk of 16 pages, head),
    # each region rounded up to 256 bytes
    S, Hq, d, maxp = 64, 32, 128, 2037
    chunks = -(-maxp // 16)
    rows = S * chunks * Hq
    r256 = lambda x: (x + 255) // 256 * 256
    assert fa.decode_workspace_bytes(S, Hq, d, 16, maxp) == r256(rows * d * 4) + r256(rows * 4)
    assert fa.decode_workspace_bytes(S, Hq, d, 8, maxp) == 0
    assert fa.decode_workspace_bytes(0, Hq, d, 16, maxp) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    """Importing the binding with the shared library absent raises, rather
    than falling back to anything else."""
    import subprocess
    import sys
    import shutil
    pkg = tmp_path / "exact_io_aware_75_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "exact_io_aware_75_b200", "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import exact_io_aware_75_b200"],
                       cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0 and "missing" in r.stderr
