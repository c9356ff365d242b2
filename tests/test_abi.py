"""The C-ABI library: it loads, exports every entry point ``include/kda.h``
declares, and rejects bad arguments on the host before anything is launched.

Calls below pass fake (never dereferenced) addresses, so each must fail
validation; they are skipped on a machine with a GPU, where a validation bug
would otherwise launch a kernel on them.
"""
import ctypes
import os
import re

import pytest
import torch

import gated_delta_rule_125_b200 as kda
from gated_delta_rule_125_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake-pointer calls only without a GPU")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"kda_prefill", "kda_decode_step", "kda_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(kda.EXPORTED_SYMBOLS)
    assert "kda_device_error" in names


def test_status_strings_and_version(lib):
    for code in range(7):
        s = kda.kda_status_string(code)
        assert s.startswith("KDA_")
    assert kda.kda_status_string(99) == "KDA_ERR_UNKNOWN"
    assert kda.kda_version() >= 100


def test_workspace_queries(lib):
    f = lib.kda_prefill_workspace_size
    m = lib.kda_prefill_workspace_min
    # valid: recommended >= minimum; the exact (fp32) path's minimum grows with heads
    a = f(1, 8192, 8192, 32, 128, 128, 1, 64, 0)
    b = m(1, 8192, 8192, 32, 128, 128, 1, 64, 0)
    assert a >= b > 0
    assert m(1, 8192, 8192, 16, 128, 128, 0, 64, 0) < m(1, 8192, 8192, 32, 128, 128, 0, 64, 0)
    # tensor-core path: a planning launch and one persistent launch; the ring of
    # each stream holds at most its chunks and at most 16 slots, so a short
    # problem needs less and a long one no more than a 16-chunk problem
    assert lib.kda_prefill_launches(1, 8192, 8192, 32, 128, 128, 1, 64, 0, a) == 2
    assert lib.kda_prefill_launches(1, 8192, 8192, 32, 128, 128, 1, 64, 0, b) == 2
    assert lib.kda_prefill_launches(1, 8192, 8192, 32, 128, 128, 1, 64, 0, b - 1) == -1
    assert f(1, 128, 128, 32, 128, 128, 1, 64, 0) < f(1, 8192, 8192, 32, 128, 128, 1, 64, 0)
    assert f(1, 1024, 1024, 32, 128, 128, 1, 64, 0) == a == f(1, 1 << 20, 1 << 20, 32, 128, 128, 1, 64, 0)
    assert m(1, 1 << 20, 1 << 20, 32, 128, 128, 1, 64, 0) == b < a
    # single-chunk problems need no state carry
    assert m(1, 64, 64, 4, 64, 64, 0, 64, 0) == m(1, 1, 1, 4, 64, 64, 0, 64, 0)
    # invalid / unsupported -> 0
    assert f(0, 10, 10, 1, 128, 128, 1, 64, 0) == 0
    assert f(1, 10, 10, 1, 96, 128, 1, 64, 0) == 0
    assert f(1, 10, 10, 1, 128, 128, 1, 32, 0) == 0
    assert f(1, 10, 10, 1, 128, 128, 7, 64, 0) == 0
    assert f(1, 10, 10, 1, 128, 128, 1, 64, 0x80) == 0
    # the scalar-gate flag (log_alpha [T][H]) is a known flag
    assert f(1, 8192, 8192, 32, 128, 128, 1, 64, kda.KDA_FLAG_SCALAR_GATE) > 0
    assert f(1, 10, 10, 1, 64, 64, 0, 64, kda.KDA_FLAG_SCALAR_GATE | kda.KDA_FLAG_EXACT) > 0


A = 0x10000  # fake 16-byte-aligned address, never dereferenced


def prefill(lib, **over):
    args = dict(q=A, k=A, v=A, la=A, beta=A, S0=None, cu=None, N=1, T=128, L=128, H=2, dk=64,
                dv=64, dt=1, chunk=64, flags=0, o=A, ST=A, ws=A, wsb=1 << 30, stream=None)
    args.update(over)
    a = args
    return lib.kda_prefill(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S0"], a["cu"], a["N"],
                           a["T"], a["L"], a["H"], a["dk"], a["dv"], a["dt"], a["chunk"],
                           a["flags"], a["o"], a["ST"], a["ws"], a["wsb"], a["stream"])


def decode(lib, **over):
    a = dict(q=A, k=A, v=A, la=A, beta=A, S=A, N=4, H=2, dk=128, dv=128, dt=1, flags=0, o=A,
             stream=None)
    a.update(over)
    return lib.kda_decode_step(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S"], a["N"],
                               a["H"], a["dk"], a["dv"], a["dt"], a["flags"], a["o"], a["stream"])


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=None), kda.KDA_ERR_INVALID_ARG),
    (dict(o=None), kda.KDA_ERR_INVALID_ARG),
    (dict(N=0), kda.KDA_ERR_INVALID_ARG),
    (dict(N=3), kda.KDA_ERR_INVALID_ARG),          # several sequences need cu_seqlens
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=256), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dt=5), kda.KDA_ERR_INVALID_ARG),
    (dict(flags=0x100), kda.KDA_ERR_INVALID_ARG),
    (dict(q=A + 8), kda.KDA_ERR_MISALIGNED),
    (dict(la=A + 4), kda.KDA_ERR_MISALIGNED),
    (dict(beta=A + 2), kda.KDA_ERR_MISALIGNED),
    (dict(S0=A + 2), kda.KDA_ERR_MISALIGNED),
    (dict(cu=A + 4, N=2), kda.KDA_ERR_MISALIGNED),
    (dict(ST=A + 12), kda.KDA_ERR_MISALIGNED),
    (dict(ws=None), kda.KDA_ERR_WORKSPACE),
    (dict(wsb=1024), kda.KDA_ERR_WORKSPACE),
])
def test_prefill_rejects(lib, over, code):
    assert prefill(lib, **over) == code


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(S=None), kda.KDA_ERR_INVALID_ARG),
    (dict(N=0), kda.KDA_ERR_INVALID_ARG),
    (dict(H=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(dt=2), kda.KDA_ERR_INVALID_ARG),
    (dict(flags=0x8), kda.KDA_ERR_INVALID_ARG),
    (dict(v=A + 2), kda.KDA_ERR_MISALIGNED),
    (dict(S=A + 8), kda.KDA_ERR_MISALIGNED),
    (dict(o=A + 4), kda.KDA_ERR_MISALIGNED),
    (dict(beta=A + 1), kda.KDA_ERR_MISALIGNED),
])
def test_decode_rejects(lib, over, code):
    assert decode(lib, **over) == code


def test_binding_refuses_host_tensors(lib):
    q = torch.zeros(4, 2, 64)
    with pytest.raises(ValueError):
        kda.kda_decode_step(q, q, q, q, torch.zeros(4, 2), torch.zeros(4, 2, 64, 64))


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(kda, "_lib", None)
    monkeypatch.setenv("KDA_LIBRARY", "/nonexistent/libkda.so")
    with pytest.raises(OSError):
        kda.load_library()


# ------------------------------------------------ the next rows' entry points ----

def test_short_conv_launch_counts(lib):
    f = lib.kda_short_conv_launches
    assert f(4, 1, 16) == 2 and f(4, 0, 16) == 1 and f(1, 1, 16) == 1
    assert f(4, 1, 0) == 1 and f(4, 0, 0) == 0
    assert f(0, 0, 16) == -1 and f(9, 0, 16) == -1 and f(4, 0, -1) == -1


def short_conv(lib, width=4, weight=A, sin=None, sout=None, **over):
    a = dict(x=A, y=A + (1 << 24), cu=None, N=1, T=64, C=256, dt=1, stream=None)
    a.update(over)
    c = kda.ShortConv(width, weight, sin, sout)
    return lib.kda_short_conv_swish(a["x"], a["y"], ctypes.byref(c), a["cu"], a["N"], a["T"], a["C"],
                                    a["dt"], a["stream"])


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(width=0), kda.KDA_ERR_UNSUPPORTED),
    (dict(width=9), kda.KDA_ERR_UNSUPPORTED),
    (dict(C=12), kda.KDA_ERR_INVALID_ARG),
    (dict(C=0), kda.KDA_ERR_INVALID_ARG),
    (dict(N=2), kda.KDA_ERR_INVALID_ARG),            # several sequences need cu_seqlens
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dt=3), kda.KDA_ERR_INVALID_ARG),
    (dict(weight=None), kda.KDA_ERR_INVALID_ARG),
    (dict(x=None), kda.KDA_ERR_INVALID_ARG),
    (dict(x=A + 8), kda.KDA_ERR_MISALIGNED),
    (dict(sin=A + 4), kda.KDA_ERR_MISALIGNED),
    (dict(sout=A + 2), kda.KDA_ERR_MISALIGNED),
    (dict(weight=A + 2), kda.KDA_ERR_MISALIGNED),
    (dict(y=A + 512), kda.KDA_ERR_INVALID_ARG),     # y overlaps x (64 x 256 bf16 = 32 KiB)
])
def test_short_conv_rejects(lib, over, code):
    assert short_conv(lib, **over) == code


@no_gpu
@pytest.mark.parametrize("conv,dt,d,code", [
    (kda.ShortConv(4, A, A, A), 0, 128, kda.KDA_ERR_UNSUPPORTED),      # fp32: the CUDA-core path has no fused form
    (kda.ShortConv(4, A, A, A), 1, 64, kda.KDA_ERR_UNSUPPORTED),       # d = 64: likewise
    (kda.ShortConv(5, A, A, A), 1, 128, kda.KDA_ERR_UNSUPPORTED),      # windows up to 4
    (kda.ShortConv(0, A, A, A), 1, 128, kda.KDA_ERR_UNSUPPORTED),
    (kda.ShortConv(4, None, A, A), 1, 128, kda.KDA_ERR_INVALID_ARG),
    (kda.ShortConv(4, A + 2, A, A), 1, 128, kda.KDA_ERR_MISALIGNED),
    (kda.ShortConv(4, A, A + 8, A), 1, 128, kda.KDA_ERR_MISALIGNED),
    (kda.ShortConv(4, A, A, A + 4), 1, 128, kda.KDA_ERR_MISALIGNED),
])
def test_prefill_conv_rejects(lib, conv, dt, d, code):
    """kda_prefill_conv validates its convolutions on the host, before any launch."""
    call = lambda cq, ck, cv: lib.kda_prefill_conv(A, A, A, A, A, None, None, 1, 128, 128, 2, d, d, dt, 64, 0,
                                                   cq, ck, cv, None, A, A, A, 1 << 30, None)
    assert call(ctypes.byref(conv), None, None) == code
    assert call(None, None, ctypes.byref(conv)) == code


@no_gpu
def test_decode_conv_rejects(lib):
    ok = kda.ShortConv(4, A, A, A)
    wide = kda.ShortConv(5, A, A, A)  # the fused decode takes windows up to 4
    odd = kda.ShortConv(4, A, A + 8, A)
    call = lambda cq: lib.kda_decode_step_conv(A, A, A, A, A, A, 4, 2, 128, 128, 1, 0, cq, None, None,
                                               None, A, None)
    assert call(ctypes.byref(wide)) == kda.KDA_ERR_UNSUPPORTED
    assert call(ctypes.byref(odd)) == kda.KDA_ERR_MISALIGNED
    assert lib.kda_decode_step_conv(None, A, A, A, A, A, 4, 2, 128, 128, 1, 0, ctypes.byref(ok), None, None,
                                    None, A, None) == kda.KDA_ERR_INVALID_ARG


def test_backward_workspace_queries(lib):
    f = lib.kda_backward_workspace_size
    a = f(1, 8192, 8192, 32, 128, 128, 1, 64, 0)
    assert a > 0
    assert f(1, 1024, 1024, 32, 128, 128, 1, 64, 0) < a  # per-chunk scratch grows with the chunks
    assert f(2, 8192, 4096, 32, 128, 128, 1, 64, 0) > 0
    # one gate per head: the same scratch
    assert f(1, 10, 10, 1, 128, 128, 1, 64, kda.KDA_FLAG_SCALAR_GATE) == f(1, 10, 10, 1, 128, 128, 1, 64, 0) > 0
    # the chunk slots follow the sequences' own lengths: a varlen batch needs no slots for the
    # longest sequence's length times the batch (16 sequences of at most 8192 tokens, 62,337 in all)
    assert f(16, 62337, 8192, 32, 128, 128, 1, 64, 0) < f(1, 62337 + 16 * 64, 62337 + 16 * 64, 32, 128, 128, 1, 64, 0)
    assert f(16, 62337, 8192, 32, 128, 128, 1, 64, 0) < 16 * f(1, 8192, 8192, 32, 128, 128, 1, 64, 0) / 2
    assert f(1, 10, 10, 1, 96, 128, 1, 64, 0) == 0
    assert f(0, 10, 10, 1, 128, 128, 1, 64, 0) == 0


def backward(lib, **over):
    a = dict(q=A, k=A, v=A, la=A, beta=A, S0=None, cu=None, N=1, T=128, L=128, H=2, dk=64, dv=64, dt=1,
             chunk=64, flags=0, do=A, dST=None, dq=A, dk_=A, dv_=A, dla=A, db=A, dS0=None, ws=A,
             wsb=1 << 30, stream=None)
    a.update(over)
    return lib.kda_backward(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S0"], a["cu"], a["N"], a["T"],
                            a["L"], a["H"], a["dk"], a["dv"], a["dt"], a["chunk"], a["flags"], a["do"],
                            a["dST"], a["dq"], a["dk_"], a["dv_"], a["dla"], a["db"], a["dS0"], a["ws"],
                            a["wsb"], a["stream"])


@no_gpu
@pytest.mark.parametrize("over,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(do=None), kda.KDA_ERR_INVALID_ARG),
    (dict(db=None), kda.KDA_ERR_INVALID_ARG),
    (dict(N=3), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(ws=None), kda.KDA_ERR_WORKSPACE),
    (dict(wsb=4096), kda.KDA_ERR_WORKSPACE),
    (dict(ws=A + 4), kda.KDA_ERR_MISALIGNED),
])
def test_backward_rejects(lib, over, code):
    assert backward(lib, **over) == code


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/kda.h is a C header (C99, no C++ or torch types) and a C program links against
    libkda.so and calls it (version and status strings need no GPU)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use_kda.c"
    src.write_text('#include "kda.h"\n#include <stdio.h>\n#include <string.h>\n'
                   'int main(void) {\n'
                   '    if (kda_version() <= 0) return 1;\n'
                   '    if (strlen(kda_status_string(KDA_ERR_WORKSPACE)) == 0) return 2;\n'
                   '    printf("%d\\n", (int)kda_version());\n'
                   '    return 0;\n}\n')
    libdir = os.path.dirname(kda.library_path())
    exe = tmp_path / "use_kda"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(root, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lkda", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    assert int(out) == lib.kda_version()
