"""The C ABI without a GPU: the library builds and loads, exports every
function include/nattn.h declares, and rejects bad arguments on the host
before anything is launched."""

import ctypes
import os
import re

import pytest

from tests._util import ensure_built

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "nattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nattn_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    ensure_built()
    from alternative_normalizers_b200 import binding
    return binding


def test_exports_every_declared_symbol(L):
    names = _header_functions()
    assert "nattn_fwd" in names and "nattn_fwd_ex" in names
    so = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(so, n), n


def test_version_and_errors(L):
    assert L.nattn_version() == 100
    assert L.nattn_strerror(0) == "ok"
    for code in range(-8, 0):
        assert L.nattn_strerror(code) not in ("ok", "unknown error")


def _args(L, **kw):
    a = L.NattnArgs()
    base = dict(B=1, Hq=4, Hkv=2, Tq=64, Tk=64, d=128, dv=128, scale=0.1,
                normalizer=0, causal=1, window=0, softcap=0.0)
    base.update(kw)
    for k, v in base.items():
        setattr(a, k, v)
    for p in ("q", "k", "v", "out"):
        if getattr(a, p) is None:
            setattr(a, p, 4096)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(Hkv=3), -1), (dict(Hkv=0), -1), (dict(d=300), -2), (dict(dv=12), -2),
    (dict(scale=float("nan")), -1), (dict(scale=float("inf")), -1),
    (dict(softcap=-1.0), -1), (dict(window=-2), -1), (dict(normalizer=4), -1),
    (dict(causal=2), -1), (dict(B=-1), -1), (dict(q=4100), -8),
    (dict(row_stat=4098), -8), (dict(row_nnz=4098), -8), (dict(d=12), -2),
    (dict(dv=264), -2),
])
def test_host_validation(L, kw, code):
    a = _args(L, **kw)
    assert L.nattn_fwd_ex(a) == code
    assert L.nattn_workspace_size(a) == 0


def test_null_pointers(L):
    a = _args(L)
    a.k = None
    assert L.nattn_fwd_ex(a) == -1


def test_empty_problem_is_a_noop(L):
    for kw in (dict(B=0), dict(Tq=0), dict(Hq=0)):
        a = _args(L, **kw)
        assert L.nattn_fwd_ex(a) == 0


def test_weights_size_limit(L):
    a = _args(L, B=64, Hq=32, Tq=4096, Tk=4096, Hkv=8)
    a.weights = 4096
    assert L.nattn_fwd_ex(a) == -3


def test_paged_requires_lengths_and_rejects_weights(L):
    a = _args(L, Tq=1, Tk=1024)
    a.block_table = 4096
    a.page_size, a.block_table_stride, a.num_pages = 64, 16, 100
    assert L.nattn_fwd_ex(a) == -1          # seqlens missing
    a.seqlens = 4096
    a.weights = 4096
    assert L.nattn_fwd_ex(a) == -2


def test_workspace_sizes(L):
    # online prefill needs no scratch; sparse prefill keeps tau + overflow list
    a = _args(L, B=2, Hq=32, Hkv=8, Tq=4096, Tk=4096)
    assert L.nattn_workspace_size(a) == 0
    a.normalizer = 2
    ws = L.nattn_workspace_size(a)
    rows = 2 * 32 * 4096
    assert ws >= rows * 8
    a.workspace, a.workspace_bytes = 4096, ws - 1
    assert L.nattn_fwd_ex(a) == -4
    # paged decode: split partials
    p = _args(L, B=64, Hq=32, Hkv=8, Tq=1, Tk=32768)
    p.block_table, p.seqlens = 4096, 4096
    p.page_size, p.block_table_stride, p.num_pages = 64, 512, 20000
    w0 = L.nattn_workspace_size(p)
    assert w0 > 0
    p.normalizer = 3                     # sparse decode also stores scores
    assert L.nattn_workspace_size(p) > w0 + 64 * 32 * 32768 * 4 - 1


def test_short_form_paged_needs_device_allocations(L):
    """nattn_fwd in paged mode bounds the page pool by the device
    allocations holding k and v; pointers outside any device allocation of
    this process are refused on the host (NATTN_EINVAL) before any launch."""
    import ctypes as C
    rc = L.nattn_fwd(4096, 8192, 12288, 16384, None, 2, 8, 2, 1, 256, 128, 128,
                     0.088, 0, 1, 0, 0.0, 20480, 24576, None)
    assert rc == -1


def test_sinks_only_with_softmax_and_aligned(L):
    a = _args(L)
    a.sinks = 4096
    assert L.nattn_workspace_size(a) == 0          # softmax: valid, no scratch
    for n in (1, 2, 3):                            # softmax1 / sparse: refused
        a.normalizer = n
        assert L.nattn_fwd_ex(a) == -2
    a.normalizer = 0
    a.sinks = 4098
    assert L.nattn_fwd_ex(a) == -8


def test_args_struct_layout_matches_c(tmp_path):
    """The ctypes mirror of nattn_args has the C struct's size and field
    offsets (checked with a small C program built against the header)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("needs gcc")
    from alternative_normalizers_b200.binding import NattnArgs
    names = [f[0] for f in NattnArgs._fields_]
    src = tmp_path / "layout.c"
    body = "".join(f'  printf("%zu\\n", offsetof(nattn_args, {n}));\n' for n in names)
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"nattn.h\"\n"
                   "int main(void) {\n  printf(\"%zu\\n\", sizeof(nattn_args));\n"
                   + body + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe)], check=True)
    out = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert out[0] == ctypes.sizeof(NattnArgs)
    assert out[1:] == [getattr(NattnArgs, n).offset for n in names]
