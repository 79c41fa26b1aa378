"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_429_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 0x100000  # aligned non-null address; never dereferenced by these calls


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"PA_API[^;(]*?\b(pa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_decode", "pa_reshape_and_cache", "pa_copy_blocks",
                     "pa_decode_workspace_size", "pa_status_string",
                     "pa_pool_create", "pa_pool_append", "pa_pool_fork"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_exactly_the_header():
    assert sorted(_lib.SIGNATURES) == declared_functions()


def test_status_strings():
    lib = _lib.lib()
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.pa_status_string(code).decode() == name
    assert lib.pa_status_string(99).decode() == "PA_ERR_UNKNOWN"


def test_workspace_size_formula():
    lib = _lib.lib()
    # 8 seqs, 64 heads, d128, 131072 tokens, 512-token partitions
    P = 131072 // 512
    floats = 8 * 64 * P * (128 + 2)
    expect = (floats * 4 + 512 + 255) // 256 * 256
    assert lib.pa_decode_workspace_size(8, 64, 128, 131072, 512) == expect
    assert lib.pa_decode_workspace_size(8, 64, 128, 131072, -1) == expect
    assert lib.pa_decode_workspace_size(8, 64, 128, 131072, 0) == 0
    assert lib.pa_decode_workspace_size(8, 64, 128, 131072, 100) == 0


def decode_args(**kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, dtype=0, ks=1.0, vs=1.0, bt=FAKE,
             maxb=8, cl=FAKE, maxctx=128, S=2, Hq=8, Hkv=8, D=128, B=16, NB=64,
             scale=0.1, psize=512, ws=None, wsb=0, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(S=0), OK),                       # empty batch: nothing to launch
    (dict(B=8), UNSUPPORTED),
    (dict(D=96), UNSUPPORTED),
    (dict(Hq=12, Hkv=8), UNSUPPORTED),     # not a whole group
    (dict(Hq=32, Hkv=1), UNSUPPORTED),     # group 32 > 16
    (dict(out=None), INVALID),
    (dict(q=FAKE + 2), INVALID),           # misaligned
    (dict(dtype=1, ks=0.0), INVALID),      # fp8 needs positive scales
    (dict(dtype=1, vs=float("inf")), INVALID),
    (dict(dtype=5), INVALID),
    (dict(psize=100), INVALID),            # not a multiple of 16
    (dict(psize=-2), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(NB=0), INVALID),
    (dict(psize=512, ws=None), WORKSPACE),  # forced split, no workspace
    (dict(psize=512, ws=FAKE, wsb=1024), WORKSPACE),
    (dict(psize=512, ws=FAKE + 16, wsb=1 << 30), WORKSPACE),  # not 256-aligned
])
def test_decode_rejects_bad_arguments_on_host(kw, expect):
    assert _lib.lib().pa_decode(*decode_args(**kw)) == expect


def no_alloc_args(**kw):
    a = decode_args(**kw)
    del a[-3:-1]   # no workspace pointer or size
    return a


@pytest.mark.parametrize("kw,expect", [
    (dict(S=0), OK),                       # empty batch: nothing to launch
    # with no sequence the call still rejects what pa_decode rejects
    (dict(S=0, B=32), UNSUPPORTED),
    (dict(S=0, D=96), UNSUPPORTED),
    (dict(S=0, Hq=12, Hkv=8), UNSUPPORTED),
    (dict(S=0, dtype=1, ks=0.0), INVALID),
    (dict(S=0, scale=float("nan")), INVALID),
    (dict(S=0, NB=0), INVALID),
    (dict(psize=0), INVALID),              # the split path is the only one
    (dict(psize=-1), INVALID),
    (dict(psize=100), INVALID),
    (dict(maxctx=-1), INVALID),
    # more scratch than the fixed array holds: 16 MiB / (64 * 8 * 130 * 4) partitions
    (dict(S=64, maxb=1 << 20, maxctx=1 << 20), WORKSPACE),
])
def test_decode_no_alloc_rejects_bad_arguments_on_host(kw, expect):
    assert _lib.lib().pa_decode_no_alloc(*no_alloc_args(**kw)) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(T=0), OK),
    (dict(B=32), UNSUPPORTED),
    (dict(D=80), UNSUPPORTED),
    (dict(key=None), INVALID),
    (dict(slots=None), INVALID),
    (dict(dtype=1, ks=-1.0), INVALID),
    (dict(k=FAKE + 8), INVALID),
])
def test_reshape_rejects_bad_arguments_on_host(kw, expect):
    a = dict(key=FAKE, value=FAKE, k=FAKE, v=FAKE, slots=FAKE, T=4, Hkv=8, D=128,
             B=16, NB=64, dtype=0, ks=1.0, vs=1.0, stream=None)
    a.update(kw)
    assert _lib.lib().pa_reshape_and_cache(*a.values()) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(n=0), OK),
    (dict(pairs=None), INVALID),
    (dict(bb=1000), INVALID),   # not a multiple of 16
    (dict(bb=0), INVALID),
    (dict(k=FAKE + 4), INVALID),
])
def test_copy_rejects_bad_arguments_on_host(kw, expect):
    a = dict(k=FAKE, v=FAKE, pairs=FAKE, n=3, bb=4096, NB=64, stream=None)
    a.update(kw)
    assert _lib.lib().pa_copy_blocks(*a.values()) == expect


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libpa.so"))
    with pytest.raises(_lib.LibraryNotBuilt):
        _lib.lib()


@pytest.mark.parametrize("kw,expect", [
    (dict(n=0), OK),
    (dict(pairs=None), INVALID),
    (dict(dk=None), INVALID),
    (dict(bb=24), INVALID),
    (dict(sk=FAKE + 4), INVALID),
    (dict(snb=0), INVALID),
])
def test_swap_rejects_bad_arguments_on_host(kw, expect):
    a = dict(dk=FAKE, dv=FAKE, sk=FAKE, sv=FAKE, pairs=FAKE, n=3, bb=4096, snb=8,
             dnb=8, stream=None)
    a.update(kw)
    assert _lib.lib().pa_swap_blocks(*a.values()) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(T=0), OK),                        # nothing to launch
    (dict(S=0), OK),
    (dict(maxq=0), OK),
    (dict(dtype=1), UNSUPPORTED),           # fp8 caches: decode only
    (dict(dtype=7), INVALID),
    (dict(B=8), UNSUPPORTED),
    (dict(D=96), UNSUPPORTED),
    (dict(Hq=12, Hkv=8), UNSUPPORTED),      # not a whole group
    (dict(Hq=32, Hkv=1), UNSUPPORTED),      # group 32 > 16
    (dict(scale=float("inf")), INVALID),
    (dict(NB=0), INVALID),
    (dict(maxb=-1), INVALID),
    (dict(out=None), INVALID),
    (dict(qs=None), INVALID),
    (dict(out=FAKE + 4), INVALID),          # misaligned
    (dict(k=FAKE + 8), INVALID),
])
def test_prefill_rejects_bad_arguments_on_host(kw, expect):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, dtype=0, bt=FAKE, maxb=8, qs=FAKE, cl=FAKE,
             maxq=64, maxctx=128, S=2, T=100, Hq=8, Hkv=2, D=128, B=16, NB=64, scale=0.1,
             stream=None)
    a.update(kw)
    assert _lib.lib().pa_prefill(*a.values()) == expect


def declared_arity():
    """Parameter count of every PA_API function in the header."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"PA_API[^;(]*?\b(pa_\w+)\s*\(([^)]*)\)\s*;", text):
        params = [p for p in m.group(2).split(",") if p.strip()]
        out[m.group(1)] = 0 if params == ["void"] or [p.strip() for p in params] == ["void"] \
            else len(params)
    return out


def test_binding_argument_counts_match_the_header():
    arity = declared_arity()
    for name, (_, args) in _lib.SIGNATURES.items():
        assert len(args) == arity[name], (name, len(args), arity[name])


def test_product_never_reaches_the_oracle():
    """The oracle is test infrastructure: no module of the package imports
    it and no CUDA/C++ source includes anything from it."""
    import ast
    pkg = os.path.dirname(_lib.LIB_PATH)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith(".py"):
                tree = ast.parse(open(path, encoding="utf-8").read(), path)
                for node in ast.walk(tree):
                    if isinstance(node, ast.Import):
                        names = [a.name for a in node.names]
                    elif isinstance(node, ast.ImportFrom):
                        names = [node.module or ""]
                    else:
                        continue
                    assert not any(n.split(".")[0] == "oracle" for n in names), (path, names)
            elif f.endswith((".cu", ".cuh", ".cpp", ".h")):
                src = open(path, encoding="utf-8").read()
                assert not re.search(r'#\s*include\s*[<"][^>"]*oracle', src), path


def test_oracle_never_reaches_the_product():
    """The oracle shares no code with the CUDA path: it neither imports the
    package nor includes its headers or sources."""
    import ast
    root = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")
    for dirpath, _, files in os.walk(root):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith(".py"):
                tree = ast.parse(open(path, encoding="utf-8").read(), path)
                for node in ast.walk(tree):
                    if isinstance(node, ast.Import):
                        names = [a.name for a in node.names]
                    elif isinstance(node, ast.ImportFrom):
                        names = [node.module or ""]
                    else:
                        continue
                    assert not any(n.split(".")[0] == "paged_kv_cache_429_b200" for n in names), \
                        (path, names)
            elif f.endswith((".c", ".h", ".cpp")):
                src = open(path, encoding="utf-8").read()
                for inc in re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', src):
                    assert inc in {"stdint.h", "stddef.h", "stdlib.h", "string.h", "math.h",
                                   "stdio.h", "float.h", "limits.h"} or inc.startswith("oracle"), \
                        (path, inc)
