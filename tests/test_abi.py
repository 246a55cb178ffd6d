"""The C-ABI library loads and exports every entry point that include/csld.h declares, and its
host-side validation rejects bad arguments before launching anything (no GPU needed)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csld.h")


def _build_lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "csld_build", os.path.join(ROOT, "compressed_sparse_long_decode_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def lib():
    return C.CDLL(_build_lib())


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"CSLD_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_five_path_calls():
    names = set(declared_functions())
    for n in ("csa_compress", "hca_compress", "indexer_topk", "hybrid_decode_attention", "kv_cache_append"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in csld.h but not exported"


def test_abi_version_and_strings(lib):
    lib.csld_abi_version.restype = C.c_int
    assert lib.csld_abi_version() == 1
    lib.csld_status_string.restype = C.c_char_p
    lib.csld_status_string.argtypes = [C.c_int]
    assert lib.csld_status_string(0) == b"ok"
    assert b"workspace" in lib.csld_status_string(7)


def test_host_validation_without_launch(lib):
    lib.csld_last_error.restype = C.c_char_p
    P, I, I64, F, S = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
    f = lib.hybrid_decode_attention
    f.restype = I
    f.argtypes = [P, I, P, I64, I, P, I, P, I, P, I, F, P, P, P, S, P, P]
    # 8 heads: not implemented by the library -> CSLD_ERR_UNSUPPORTED, nothing launched
    assert f(1, 8, 16, 64, 4, None, 0, 16, 4, 16, 1, 0.05, 16, None, 16, 1 << 20, None, None) == 6
    assert b"heads" in lib.csld_last_error()
    # NULL q -> CSLD_ERR_ARG
    assert f(None, 16, 16, 64, 4, None, 0, 16, 4, 16, 1, 0.05, 16, None, 16, 1 << 20, None, None) == 1
    # window beyond the maximum -> CSLD_ERR_ARG
    assert f(16, 16, 16, 64, 4, None, 0, 16, 5000, 16, 1, 0.05, 16, None, 16, 1 << 20, None, None) == 1
    # misaligned cache pointer -> CSLD_ERR_ALIGN
    assert f(16, 16, 17, 64, 4, None, 0, 16, 4, 16, 1, 0.05, 16, None, 16, 1 << 20, None, None) == 3
    # non-finite scale -> CSLD_ERR_ARG
    assert f(16, 16, 16, 64, 4, None, 0, 16, 4, 16, 1, float("nan"), 16, None, 16, 1 << 20, None, None) == 1
    g = lib.indexer_topk
    g.restype = I
    g.argtypes = [P, P, I64, P, I, P, P, I, I, P, P, S, P, P]
    assert g(16, 16, 63, 16, 4, 16, 16, 1, 8, 16, 256, 1 << 20, None, None) == 3   # odd cap
    assert g(16, 16, 64, 16, 4, 16, 16, 1, 4096, 16, 256, 1 << 20, None, None) == 1  # k > 2048
    assert g(16, 16, 64, 16, 4, 16, 16, 1, 8, 16, None, 0, None, None) == 7         # no workspace
    h = lib.csld_compress
    h.restype = I
    h.argtypes = [P, P, P, I, P, I64, P, P, P, P]
    assert h(16, 16, 16, 0, None, 64, 16, None, None, None) == 1                   # ratio 0
    assert h(16, 16, 16, 4, 16, 64, 16, None, None, None) == 1                     # keys missing
    assert h(None, None, None, 4, None, 3, None, None, None, None) == 0            # T < m: no-op


class _Cache(C.Structure):
    _fields_ = [("ratio", C.c_int32), ("window", C.c_int32), ("batch", C.c_int32),
                ("has_indexer", C.c_int32), ("capacity", C.c_int64)] + \
               [(n, C.c_void_p) for n in ("comp_kv", "ikeys", "iscales", "win_kv", "tail_kv",
                                          "tail_gate", "seq_len", "pos_bias", "w_idx")]


def test_cache_validation(lib):
    f = lib.kv_cache_append
    f.restype = C.c_int
    f.argtypes = [C.POINTER(_Cache), C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    c = _Cache(4, 8, 2, 1, 11, 16, 16, 16, 16, 16, 16, 16, 16, 16)
    assert f(C.byref(c), 16, 16, None, None) == 3          # odd capacity with indexer keys
    c.capacity = 12
    c.ratio = 200
    assert f(C.byref(c), 16, 16, None, None) == 1          # ratio above 128
    c.ratio = 4
    c.ikeys = None
    assert f(C.byref(c), 16, 16, None, None) == 1          # indexer arrays missing
    assert f(None, 16, 16, None, None) == 1


def test_indexer_key_storage_swap_is_an_involution_on_entries_4_to_7_of_8():
    """The key cache stores logical byte c of entry s at s*32 + (c ^ 16*((s >> 2) & 1))."""
    import numpy as np
    import synth
    rng = np.random.default_rng(5)
    a = rng.integers(0, 256, (3, 21, 32), dtype=np.uint8)
    b = synth.ikeys_swap_halves(a)
    assert np.array_equal(synth.ikeys_swap_halves(b), a)
    for s in range(21):
        for c in range(32):
            assert np.array_equal(b[:, s, c ^ (16 * ((s >> 2) & 1))], a[:, s, c])
