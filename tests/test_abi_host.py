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
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


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


def bwd(fa, **kw):
    a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, B=1, Hq=4, Hkv=2, N=256, d=128,
             causal=1, window=0, scale=0.125, ws=P, wsb=1 << 30)
    a.update(kw)
    return fa.library().fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"],
                               a["dk"], a["dv"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                               a["causal"], a["window"], a["scale"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3), -1), (dict(scale=-1.0), -1), (dict(causal=3), -1), (dict(d=96), -2),
    (dict(d=80), -2), (dict(window=8, causal=0), -2), (dict(do=0), -1), (dict(lse=0), -1),
    (dict(dq=0), -1), (dict(dv=P + 4), -3), (dict(lse=P + 1), -3), (dict(ws=0), -4),
    (dict(wsb=1000), -4), (dict(ws=P + 16), -3), (dict(B=-2), -1)])
def test_bwd_rejects(fa, kw, status):
    assert bwd(fa, **kw) == status


def test_bwd_empty_is_noop(fa):
    assert bwd(fa, B=0, q=0, ws=0) == 0
    assert bwd(fa, N=0, q=0, ws=0) == 0


def test_bwd_sinks_rejects(fa):
    lib = fa.library()
    head = [P] * 6                    # q, k, v, o, dout, lse
    tail = [1, 4, 2, 256, 128, 1, 0, 0.125, P, 1 << 30, None]
    assert lib.fa_bwd_sinks(*head, None, P, P, P, P, *tail) == -1          # sinks NULL
    assert lib.fa_bwd_sinks(*head, P, P, P, P, None, *tail) == -1          # dsinks NULL
    assert lib.fa_bwd_sinks(*head, P + 2, P, P, P, P, *tail) == -3
    assert lib.fa_bwd_varlen_sinks(*head, P, P, P, P, P + 1, P, 2, 100, 60, 4, 2, 128, 1, 0,
                                   0.1, P, 1 << 30, None) == -3


def test_bwd_varlen_rejects(fa):
    lib = fa.library()
    args = [P] * 9
    # cu_seqlens missing, then misaligned
    assert lib.fa_bwd_varlen(*args, None, 2, 100, 60, 4, 2, 128, 1, 0, 0.1, P, 1 << 30, None) == -1
    assert lib.fa_bwd_varlen(*args, P + 2, 2, 100, 60, 4, 2, 128, 1, 0, 0.1, P, 1 << 30,
                             None) == -3
    assert lib.fa_bwd_varlen(*args, P, 0, 0, 0, 4, 2, 128, 1, 0, 0.1, None, 0, None) == 0


def test_bwd_workspace_formula(fa):
    r256 = lambda x: (x + 255) // 256 * 256
    T, Hq = 4096, 32
    assert fa.bwd_workspace_bytes(T, Hq, 128) == r256(T * Hq * 128 * 4) + r256(T * Hq * 4)
    assert fa.bwd_workspace_bytes(T, Hq, 64) == r256(T * Hq * 64 * 4) + r256(T * Hq * 4)
    assert fa.bwd_workspace_bytes(T, Hq, 96) == 0


def test_sinks_entry_points_reject(fa):
    lib = fa.library()
    # fa_fwd_sinks: sinks NULL, then misaligned
    assert lib.fa_fwd_sinks(P, P, P, P, 0, None, 1, 2, 2, 128, 64, 0, 0, 0.1, 0, None) == -1
    assert lib.fa_fwd_sinks(P, P, P, P, 0, P + 2, 1, 2, 2, 128, 64, 0, 0, 0.1, 0, None) == -3
    # otherwise the same validation as fa_fwd
    assert lib.fa_fwd_sinks(P, P, P, P, 0, P, 1, 3, 2, 128, 64, 0, 0, 0.1, 0, None) == -1
    assert lib.fa_fwd_varlen_sinks(P, P, P, P, 0, None, P, 2, 100, 60, 2, 2, 64, 1, 0, 0.1, 0,
                                   None) == -1
    assert lib.fa_decode_paged_sinks(P, P, P, P, P, P, 0, None, 4, 100, 32, 8, 128, 16, 64, 0.1,
                                     P, 1 << 30, None) == -1
    assert lib.fa_decode_paged_sinks(P, P, P, P, P, P, 0, P + 1, 4, 100, 32, 8, 128, 16, 64,
                                     0.1, P, 1 << 30, None) == -3


def test_fp8_decode_rejects(fa):
    lib = fa.library()
    base = [P, P, P]
    tail = [P, P, P, 0, None, 4, 100, 32, 8, 128, 16, 64, 0.1, P, 1 << 30, None]
    assert lib.fa_decode_paged_fp8(*base, None, P, *tail) == -1          # k_scale NULL
    assert lib.fa_decode_paged_fp8(*base, P, None, *tail) == -1          # v_scale NULL
    assert lib.fa_decode_paged_fp8(*base, P + 2, P, *tail) == -3         # misaligned scale
    t2 = list(tail)
    t2[3] = P + 1                                                        # misaligned sinks
    assert lib.fa_decode_paged_fp8(*base, P, P, *t2) == -3
    t3 = list(tail)
    t3[10] = 8                                                           # page size 8
    assert lib.fa_decode_paged_fp8(*base, P, P, *t3) == -2


def paged_fwd(fa, **kw):
    a = dict(q=P, kc=P, vc=P, bt=P, cu=P, sl=P, o=P, lse=0, sinks=0, S=2, Tq=100, maxq=64,
             npages=40, Hq=8, Hkv=2, d=128, ps=16, maxp=8, causal=1, window=0, scale=0.1,
             od=0)
    a.update(kw)
    return fa.library().fa_fwd_paged(a["q"], a["kc"], a["vc"], a["bt"], a["cu"], a["sl"],
                                     a["o"], a["lse"], a["sinks"], a["S"], a["Tq"], a["maxq"],
                                     a["npages"], a["Hq"], a["Hkv"], a["d"], a["ps"], a["maxp"],
                                     a["causal"], a["window"], a["scale"], a["od"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3), -1), (dict(ps=8), -2), (dict(d=96), -2), (dict(window=4, causal=0), -2),
    (dict(npages=0), -1), (dict(bt=0), -1), (dict(cu=0), -1), (dict(sl=0), -1), (dict(q=0), -1),
    (dict(kc=P + 8), -3), (dict(cu=P + 2), -3), (dict(sinks=P + 1), -3), (dict(lse=P + 2), -3),
    (dict(maxp=0), -1), (dict(S=-1), -1), (dict(od=5), -1)])
def test_fwd_paged_rejects(fa, kw, status):
    assert paged_fwd(fa, **kw) == status


def test_fwd_paged_empty_is_noop(fa):
    assert paged_fwd(fa, S=0, q=0) == 0
    assert paged_fwd(fa, Tq=0, q=0) == 0


def test_fwd_doc_rejects(fa):
    lib = fa.library()
    assert lib.fa_fwd_doc(P, P, P, P, 0, None, 1, 2, 2, 128, 64, 1, 0, 0.1, 0, None) == -1
    assert lib.fa_fwd_doc(P, P, P, P, 0, P + 2, 1, 2, 2, 128, 64, 1, 0, 0.1, 0, None) == -3
    assert lib.fa_fwd_doc(P, P, P, P, 0, P, 1, 3, 2, 128, 64, 1, 0, 0.1, 0, None) == -1
    assert lib.fa_fwd_doc(P, P, P, P, 0, P, 0, 2, 2, 128, 64, 1, 0, 0.1, 0, None) == 0


def fp8_prep(fa, **kw):
    a = dict(q=P, k=P, v=P, signs=P, q8=P, k8=P, vt8=P, qs=P, ks=P, vs=P, B=1, N=300, Hq=4,
             Hkv=2, d=128, ws=P, wsb=1 << 20)
    a.update(kw)
    return fa.library().fa_fp8_prepare(a["q"], a["k"], a["v"], a["signs"], a["q8"], a["k8"],
                                       a["vt8"], a["qs"], a["ks"], a["vs"], a["B"], a["N"],
                                       a["Hq"], a["Hkv"], a["d"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3), -1), (dict(Hkv=0), -1), (dict(d=64), -2), (dict(d=96), -1), (dict(B=-1), -1),
    (dict(q=0), -1), (dict(vt8=0), -1), (dict(vs=0), -1), (dict(ws=0), -4), (dict(wsb=8), -4),
    (dict(q=P + 8), -3), (dict(vt8=P + 4), -3), (dict(signs=P + 4), -3), (dict(qs=P + 2), -3),
    (dict(ws=P + 2), -3)])
def test_fp8_prepare_rejects(fa, kw, status):
    assert fp8_prep(fa, **kw) == status


def test_fp8_prepare_empty_and_workspace(fa):
    assert fp8_prep(fa, N=0, q=0) == 0
    assert fp8_prep(fa, B=0, ws=0) == 0
    # one fp32 block maximum per (batch, KV head, 128-token block)
    assert fa.fp8_workspace_bytes(3, 300, 2) == 3 * 2 * 3 * 4
    assert fa.fp8_workspace_bytes(1, 128, 8) == 8 * 4
    assert fa.fp8_workspace_bytes(0, 128, 8) == 0


def fwd8(fa, **kw):
    a = dict(q8=P, k8=P, vt8=P, qs=P, ks=P, vs=P, o=P, lse=0, B=1, Hq=4, Hkv=2, N=300, d=128,
             causal=1, window=0, scale=0.1, od=0)
    a.update(kw)
    return fa.library().fa_fwd_fp8(a["q8"], a["k8"], a["vt8"], a["qs"], a["ks"], a["vs"],
                                   a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                                   a["causal"], a["window"], a["scale"], a["od"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3), -1), (dict(d=64), -2), (dict(d=96), -2), (dict(window=5, causal=0), -2),
    (dict(scale=0.0), -1), (dict(od=3), -1), (dict(q8=0), -1), (dict(ks=0), -1),
    (dict(o=0), -1), (dict(k8=P + 8), -3), (dict(vt8=P + 1), -3), (dict(vs=P + 2), -3),
    (dict(lse=P + 2), -3), (dict(B=-1), -1)])
def test_fwd_fp8_rejects(fa, kw, status):
    assert fwd8(fa, **kw) == status


def test_fwd_fp8_empty_is_noop(fa):
    assert fwd8(fa, B=0, q8=0) == 0
    assert fwd8(fa, N=0, q8=0) == 0


def test_fwd_sink_tokens_rejects(fa):
    lib = fa.library()
    ok = [P, P, P, P, 0, 1, 4, 2, 300, 128]
    assert lib.fa_fwd_sink_tokens(*ok, 0, 4, 0.1, 0, None) == -1        # no window
    assert lib.fa_fwd_sink_tokens(*ok, 64, -1, 0.1, 0, None) == -1      # negative sinks
    assert lib.fa_fwd_sink_tokens(P, P, P, P, 0, 1, 3, 2, 300, 128, 64, 4, 0.1, 0, None) == -1
    assert lib.fa_fwd_sink_tokens(P, P, P, P, 0, 1, 4, 2, 300, 96, 64, 4, 0.1, 0, None) == -2
    assert lib.fa_fwd_sink_tokens(P + 8, P, P, P, 0, 1, 4, 2, 300, 128, 64, 4, 0.1, 0, None) == -3
    assert lib.fa_fwd_sink_tokens(0, P, P, P, 0, 0, 4, 2, 300, 128, 64, 4, 0.1, 0, None) == 0


def test_fwd_varlen_sink_tokens_rejects(fa):
    lib = fa.library()
    ok = [P, P, P, P, 0, P, 3, 600, 300, 4, 2, 128]
    assert lib.fa_fwd_varlen_sink_tokens(*ok, 0, 4, 0.1, 0, None) == -1      # no window
    assert lib.fa_fwd_varlen_sink_tokens(*ok, 64, -2, 0.1, 0, None) == -1    # negative sinks
    bad_cu = [P, P, P, P, 0, 0, 3, 600, 300, 4, 2, 128]
    assert lib.fa_fwd_varlen_sink_tokens(*bad_cu, 64, 4, 0.1, 0, None) == -1
    mis_cu = [P, P, P, P, 0, P + 2, 3, 600, 300, 4, 2, 128]
    assert lib.fa_fwd_varlen_sink_tokens(*mis_cu, 64, 4, 0.1, 0, None) == -3
    assert lib.fa_fwd_varlen_sink_tokens(P, P, P, P, 0, P, 0, 0, 0, 4, 2, 128, 64, 4, 0.1, 0,
                                         None) == 0


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


def test_noalloc_checks_arguments_before_size(fa):
    """fa_decode_paged_noalloc: an oversized request (64 sequences x 2048
    pages) with another bad argument reports that argument, as
    fa_decode_paged would, not the size; with valid arguments, the size."""
    lib = fa.library()

    def call(q=P, Hq=32, page=16):
        return lib.fa_decode_paged_noalloc(q, P, P, P, P, P, 0, 64, 100, Hq, 8, 128, page,
                                           2048, 0.1, None)
    assert call(Hq=30) == fa.FA_ERR_INVALID_ARG        # Hq not a multiple of Hkv
    assert call(page=32) == fa.FA_ERR_UNSUPPORTED       # page size other than 16
    assert call(q=P + 2) == fa.FA_ERR_ALIGNMENT         # misaligned query pointer
    assert call() == fa.FA_ERR_WORKSPACE                # valid, but needs > 32 MiB
