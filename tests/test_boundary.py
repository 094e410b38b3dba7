"""The C-ABI library loads and exports every entry point include/li.h
declares (no GPU needed: nothing is called that touches a device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "li.h")
LIB = os.path.join(ROOT, "cross_layer_latent_b200", "libli.so")


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^LI_API\s+[\w\s\*]+?\b(li_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import __graft_entry__
        __graft_entry__._builder().build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_decode_path_entry_points():
    syms = declared_symbols()
    for name in ("li_append_latent", "li_append_latent_ex", "li_absorb_query", "li_absorb_query_group",
                 "li_score_topk", "li_hs_anchor_candidates", "li_hs_follower_refine", "li_dsa_score_topk", "li_topk",
                 "li_device_status", "li_attention_recall"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"libli.so does not export {name}"


def test_binding_covers_every_declared_symbol():
    import cross_layer_latent_b200 as li
    assert set(declared_symbols()) == set(li.EXPORTED)


def test_status_strings_and_null_context(lib):
    lib.li_status_string.restype = ctypes.c_char_p
    assert lib.li_status_string(0) == b"ok"
    assert b"timeout" in lib.li_status_string(8) or b"wait" in lib.li_status_string(8)
    # every entry point rejects a NULL context without touching a device
    lib.li_set_wait_limit.argtypes = [ctypes.c_void_p, ctypes.c_uint64]
    assert lib.li_set_wait_limit(None, 5) == 1
    lib.li_profile_enable.argtypes = [ctypes.c_void_p, ctypes.c_int]
    assert lib.li_profile_enable(None, 1) == 1
    lib.li_score_topk.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_size_t, ctypes.c_void_p]
    assert lib.li_score_topk(None, None, None, None, None, None, None, None, 0, None) == 1


def test_workspace_bytes_grow_with_the_problem(lib):
    lib.li_workspace_bytes.restype = ctypes.c_size_t
    lib.li_workspace_bytes.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 6
    small = lib.li_workspace_bytes(None, 1, 1, 8192, 64, 2048, 4096)
    big = lib.li_workspace_bytes(None, 4, 1, 131072, 64, 2048, 8192)
    assert 0 < small < big
    # the scores and candidate list of every row fit: rows * n * (4 + 8) bytes at least
    assert big >= 4 * 131072 * 12
    assert lib.li_workspace_bytes(None, 1, 1024, 65536, 32, 2048, 0) >= 1024 * 65536 * 12
