"""CPU checks of the C ABI: the library builds, loads and exports every symbol of include/stree.h.

No compute call is made here; calls with a NULL context only exercise the
host-side argument checks, which return before touching the device.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "stree.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(stree_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib_path():
    from hybrid_packed_tree_b200.build import build
    return build()


def test_header_declares_the_expected_entry_points():
    names = _declared()
    for n in ("stree_build_tree", "stree_tree_scan", "stree_commit", "stree_tree_scan_commit",
              "stree_sync_check", "stree_ctx_create", "stree_ctx_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(lib_path):
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (stree_[a-z_]+)\b", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(lib_path)
    for n in _declared():
        assert hasattr(lib, n)


def test_binding_lists_every_declared_symbol(lib_path):
    from hybrid_packed_tree_b200 import stree
    assert sorted(stree.EXPORTS) == _declared()
    for n in _declared():
        assert callable(getattr(stree, n))


def test_status_strings_and_version(lib_path):
    from hybrid_packed_tree_b200 import stree
    assert stree.stree_status_string(0) == "ok"
    assert "tree" in stree.stree_status_string(3)
    assert stree.stree_status_string(99) == "unknown status"
    assert stree.stree_version() >= 100


def test_null_context_is_rejected_on_the_host(lib_path):
    lib = ctypes.CDLL(lib_path)
    lib.stree_build_tree.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int] * 2 + [ctypes.c_void_p] * 3
    assert lib.stree_build_tree(None, None, 4, 1, None, None, None) == 1
    lib.stree_sync_check.argtypes = [ctypes.c_void_p] * 3
    assert lib.stree_sync_check(None, None, None) == 1
    lib.stree_ctx_destroy.argtypes = [ctypes.c_void_p]
    assert lib.stree_ctx_destroy(None) == 0
    lib.stree_ctx_create.argtypes = [ctypes.c_void_p]
    assert lib.stree_ctx_create(None) == 1


def test_library_does_not_load_the_oracle(lib_path):
    out = subprocess.run(["nm", "-D", lib_path], capture_output=True, text=True, check=True).stdout
    assert "oracle" not in out
    src_dir = os.path.join(ROOT, "hybrid_packed_tree_b200")
    for dirpath, _, files in os.walk(src_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), f
                assert "liboracle" not in text and "stree_oracle" not in text, f


def _decl_arg_counts():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(stree_[a-z_]+)\s*\(([^;{]*?)\)\s*;", text):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argtypes_match_header(lib_path):
    """Every binding prototype has the header's argument count, and a NULL context
    is rejected on the host with STREE_ERR_INVALID_ARG (no device work)."""
    from hybrid_packed_tree_b200 import stree
    counts = _decl_arg_counts()
    assert set(counts) == set(stree.EXPORTS)
    for name, n in counts.items():
        fn = getattr(stree._lib, name)
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
        if name.startswith("stree_") and fn.argtypes and name not in (
                "stree_status_string", "stree_ctx_create", "stree_ctx_destroy"):
            args = [0 if t is ctypes.c_int else None for t in fn.argtypes]
            # NULL context / zero sizes: rejected on the host before any device work.
            assert fn(*args) in (1, 2), name


def test_noalloc_rejects_oversized_scratch_on_the_host(lib_path):
    """Sizes whose tree scratch exceeds the fixed 8 MiB array fail before any device call."""
    from hybrid_packed_tree_b200 import stree
    fn = stree._lib.stree_tree_scan_commit_noalloc
    fake = 0x10000                                    # aligned, never dereferenced
    args = [fake] * 8 + [256, 1 << 16, 8, 64, 128, 1, 1] + [fake, fake, 256, fake, fake, None, None]
    assert fn(*args) == 2
