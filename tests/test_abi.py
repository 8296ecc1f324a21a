"""The C ABI without a GPU: the library loads, exports every function that
include/fa.h declares, and rejects bad arguments on the host before any
launch."""
import ctypes
import os
import re

import pytest

import exact_io_aware_65_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(fa.SIGNATURES)


def test_library_exports_every_declared_symbol():
    L = fa.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def test_debug_build_has_the_same_abi():
    """The index-checking debug build (libfa_debug.so, built by
    ``__graft_entry__.build()``) exports the same functions and rejects bad
    arguments the same way."""
    from exact_io_aware_65_b200 import build
    if not os.path.exists(build.DEBUG_LIB):
        pytest.skip("debug build not present (python -m exact_io_aware_65_b200.build --debug-bounds)")
    L = ctypes.CDLL(build.DEBUG_LIB)
    for name in declared_functions():
        assert hasattr(L, name), name
    f = L.fa_status_string
    f.restype, f.argtypes = ctypes.c_char_p, [ctypes.c_int]
    assert f(6) and f(6) != fa.lib().fa_status_string(99)
    g = L.fa_bwd_workspace_size
    g.restype, g.argtypes = ctypes.c_size_t, [ctypes.c_int] * 4
    assert g(2, 4, 4096, 128) == fa.bwd_workspace_size(2, 4, 4096, 128)


def test_status_strings():
    L = fa.lib()
    for code in range(7):
        assert L.fa_status_string(code)
    assert L.fa_status_string(0) == b"ok"


def test_workspace_size_is_linear_in_sequence_length():
    s1 = fa.bwd_workspace_size(2, 4, 4096, 128)
    s2 = fa.bwd_workspace_size(2, 4, 8192, 128)
    assert s1 > 0 and abs(s2 / s1 - 2.0) < 1e-3
    assert fa.bwd_workspace_size(1, 1, 100, 96) == 0
    assert fa.bwd_workspace_size(0, 1, 100, 64) == 0
    assert fa.bwd_workspace_size(1 << 20, 1 << 10, 1 << 10, 64) == 0   # B*H*N > 2^37
    assert fa.bwd_workspace_size(1 << 10, 1 << 10, 1 << 17, 64) > 0     # B*H*N = 2^37


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced


@pytest.mark.parametrize("args,code", [
    (dict(Q=0), 1),                     # null pointer
    (dict(N=0), 1),                     # empty sequence
    (dict(B=-1), 1),
    (dict(scale=0.0), 1),
    (dict(scale=float("inf")), 1),
    (dict(scale=float("nan")), 1),
    (dict(mask=7), 1),                  # unknown mask kind
    (dict(mask=2, bm=0), 1),            # block mask missing
    (dict(Q=FAKE + 8), 1),              # misaligned
    (dict(d=96), 2),                    # head size not supported
    (dict(B=1 << 20, H=1 << 10, N=1 << 10), 2),   # B*H*N beyond 32-bit work-item counts
])
def test_fwd_rejects_bad_arguments_on_host(args, code):
    a = dict(Q=FAKE, K=FAKE, V=FAKE, B=1, H=1, N=128, d=64, mask=0, bm=0, scale=0.125, O=FAKE, L=FAKE)
    a.update(args)
    rc = fa.lib().fa_fwd(a["Q"], a["K"], a["V"], a["B"], a["H"], a["N"], a["d"], a["mask"], a["bm"] or None,
                         a["scale"], a["O"], a["L"], None)
    assert rc == code


def test_bwd_rejects_small_workspace_on_host():
    L = fa.lib()
    need = fa.bwd_workspace_size(1, 1, 128, 64)
    rc = L.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, None, 0.125,
                  FAKE, FAKE, FAKE, FAKE, need - 1, None)
    assert rc == 4
    rc = L.fa_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, None, 0.125,
                  FAKE, FAKE, FAKE, FAKE + 16, need, None)   # misaligned workspace
    assert rc == 4
    rc = L.fa_bwd(FAKE, FAKE, FAKE, FAKE, 0, FAKE, 1, 1, 128, 64, 0, None, 0.125,
                  FAKE, FAKE, FAKE, FAKE, need, None)        # null dO
    assert rc == 1


def test_selftests_reject_bad_arguments_on_host():
    L = fa.lib()
    assert L.fa_selftest_bounded_wait(0, None) == 1
    assert L.fa_selftest_mma_tile(FAKE, FAKE, FAKE, 96, 64, 0, None) == 1
    assert L.fa_selftest_mma_tile(FAKE, FAKE, FAKE, 64, 64, 2, None) == 1
