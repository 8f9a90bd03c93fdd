"""The C ABI library loads and exports every entry point of include/pivot.h;
host-side argument checks answer before any device work (no GPU needed)."""
import ctypes
import os
import re

import pytest

import query_group_top_b200 as qg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "pivot.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_]+)\s*\(", text)) - {"if", "sizeof"})


@pytest.fixture(scope="module")
def lib():
    from query_group_top_b200 import build
    build.build()
    return qg.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert set(names) == set(qg.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_sizes_are_host_arithmetic(lib):
    a = lib.pivot_workspace_size(131072, 16, 128, 16, 2048, 4096, qg.REFINE)
    b = lib.pivot_workspace_size(131072, 16, 128, 16, 2048, 4096, qg.REUSE)
    c = lib.dense_workspace_size(8192, 16, 128, 256)
    d = lib.pivot_decode_workspace_size(64, 16, 128, 2, 2048, 4096, qg.REFINE, 131074)
    assert a > b > 0 and c > 0 and d > 0
    # the Refine candidate set alone: H * G * Kc int32
    assert a - b >= 16 * 8192 * 4096 * 4
    assert lib.pivot_workspace_size(0, 16, 128, 16, 2048, 4096, 0) == 0
    # the per-member scan holds one candidate row per position (H * L * Kc
    # int32) and the proxies copied to every position (L * H * d * (4 + 6) B)
    L, H, d, g, k, Kc = 8192, 16, 128, 8, 256, 512
    e = lib.pivot_workspace_size(L, H, d, g, k, Kc, qg.REFINE | qg.PER_MEMBER_SCAN)
    f = lib.pivot_workspace_size(L, H, d, g, k, Kc, qg.REFINE)
    assert e - f >= H * L * Kc * 4 - H * (L // g) * Kc * 4 + L * H * d * 10
    # the bf16-proxy option changes no buffer size
    assert lib.pivot_workspace_size(L, H, d, g, k, Kc, qg.REFINE | qg.PROXY_BF16) == f


def test_argument_errors_before_device_work(lib):
    buf = ctypes.create_string_buffer(64)
    p = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 16
    rc = lib.pivot_index(None, p, 16, 1, 64, 4, 2, 4, 0, p, None)
    assert rc == 1 and b"null" in lib.pivot_last_error()
    assert lib.pivot_index(p, p, 16, 1, 96, 4, 2, 4, 0, p, None) == 2          # d not 64/128
    assert lib.pivot_index(p, p, 16, 1, 64, 4, 5, 4, 0, p, None) == 1          # top_k > Kc
    assert lib.pivot_index(p, p, 16, 1, 64, 4, 2, 8192, 0, p, None) == 1       # Kc > 4096
    assert lib.pivot_index(p, p, 16, 1, 64, 4, 2, 4, 7, p, None) == 1          # bad mode
    assert lib.pivot_index(p + 2, p, 16, 1, 64, 4, 2, 4, 0, p, None) == 1      # misaligned
    assert lib.dense_index(p, p, 16, 1, 64, 0, p, None) == 1
    assert lib.pivot_decode_index(p, p, None, 1, 1, 64, 2, 2, 4, 0, 16, p, None) == 1
    # the per-member scan is a Refine variant of the prefill entry points
    assert lib.pivot_index(p, p, 16, 1, 64, 4, 2, 4, 1 | 0x200, p, None) == 1   # with Reuse
    cu = (ctypes.c_int32 * 2)(0, 16)
    assert lib.pivot_decode_index_ws(p, p, ctypes.addressof(cu), 1, 1, 64, 2, 2, 4, 0x200, 16, p, None, p, 1 << 20,
                                     None) == 1
    # paged cache: the page size must be a power of two, and the pages must cover max_seqlen
    assert lib.pivot_decode_index_paged(p, p, p, p, 1, 1, 64, 2, 24, 4, 2, 4, 0, 16, p, None, p, 1 << 20, None) == 1
    assert lib.pivot_decode_index_paged(p, p, p, p, 1, 1, 64, 2, 16, 1, 2, 4, 0, 17, p, None, p, 1 << 20, None) == 1
    assert lib.pivot_decode_index_paged(p, p, None, p, 1, 1, 64, 2, 16, 4, 2, 4, 0, 16, p, None, p, 1 << 20, None) == 1


def test_no_device_means_unsupported(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    buf = ctypes.create_string_buffer(64)
    p = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 16
    assert lib.pivot_index(p, p, 16, 1, 64, 4, 2, 4, 0, p, None) == 2
    assert b"sm_100" in lib.pivot_last_error() or b"device" in lib.pivot_last_error()


def header_declarations():
    """{name: (return kind, [parameter kinds])} from include/pivot.h, kinds
    'p' (pointer), 'i' (int), 'z' (size_t)."""
    text = open(os.path.join(ROOT, "include", "pivot.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    decls = {}
    for ret, name, params in re.findall(r"\b(int|size_t|const char\s*\*)\s*([a-z_]+)\s*\(([^)]*)\)\s*;", text, re.S):
        kinds = []
        for prm in params.split(","):
            prm = prm.strip()
            if not prm or prm == "void":
                continue
            # size_t and unsigned long long are the same 64-bit unsigned kind here
            kinds.append("p" if "*" in prm else ("z" if ("size_t" in prm or "long long" in prm) else "i"))
        decls[name] = ("p" if "*" in ret else ("z" if ret == "size_t" else "i"), kinds)
    return decls


def ctypes_kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (t is not None and hasattr(t, "_type_") and t.__name__.startswith("LP_")):
        return "p"
    if t is ctypes.c_size_t:
        return "z"
    if t is ctypes.c_int:
        return "i"
    return repr(t)


def test_binding_signatures_match_the_header(lib):
    """Every entry point is called with the argument kinds, count and return
    type that include/pivot.h declares (a drift here would pass a size_t
    where an int is read, or drop an argument)."""
    decls = header_declarations()
    assert set(decls) == set(qg.EXPORTED)
    for name, (ret, kinds) in decls.items():
        f = getattr(lib, name)
        assert [ctypes_kind(t) for t in f.argtypes] == kinds, name
        assert ctypes_kind(f.restype) == ret, name
