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
            args = [0 if t in (ctypes.c_int, ctypes.c_uint64, ctypes.c_float) else None for t in fn.argtypes]
            # NULL context / zero sizes: rejected on the host before any device work.
            assert fn(*args) in (1, 2), name


def test_noalloc_rejects_oversized_scratch_on_the_host(lib_path):
    """Sizes whose tree scratch exceeds the fixed 8 MiB array fail before any device call."""
    from hybrid_packed_tree_b200 import stree
    fn = stree._lib.stree_tree_scan_commit_noalloc
    fake = 0x10000                                    # aligned, never dereferenced
    args = [fake] * 8 + [256, 1 << 16, 8, 64, 128, 1, 1] + [fake, fake, 256, fake, fake, None, None]
    assert fn(*args) == 2


def test_unrolled_and_accept_host_checks(lib_path):
    """Shape, dtype, pointer and alignment checks of stree_unrolled_scan and
    stree_accept_greedy happen on the host, before any device work."""
    from hybrid_packed_tree_b200 import stree
    un = stree._lib.stree_unrolled_scan
    ok = 0x10000                                      # aligned, never dereferenced
    # x, dt, A, B, C, D, h0, paths, path_len; T, batch, n_paths, max_depth, H, P, N, G, dtype; y, h, err, stream
    base = [ok] * 9 + [15, 1, 6, 4, 80, 64, 128, 1, 1] + [ok, ok, None, None]

    def call(fn, args, **over):
        a = list(args)
        for i, v in over.items():
            a[int(i[1:])] = v
        return fn(*a)

    assert call(un, base, i9=0) == 2                  # n_nodes 0
    assert call(un, base, i11=0) == 2                 # n_paths 0
    assert call(un, base, i15=120) == 2               # dstate not a multiple of 16
    assert call(un, base, i16=3) == 2                 # 80 heads over 3 groups
    assert call(un, base, i17=7) == 2                 # unknown dtype
    assert call(un, base, i18=ok + 4) == 5            # y misaligned
    assert call(un, base, i0=None) == 1               # x missing
    assert call(un, base, i0=ok + 8) == 5             # x misaligned
    assert call(un, base, i10=0) == 0                 # batch 0: nothing to do
    acc = stree._lib.stree_accept_greedy
    # logits, dtype, V, tokens, parent, T, batch, maxlen, pred, path, len, bonus, err, stream
    abase = [ok, 1, 50280, ok, ok, 15, 1, 15, ok, ok, ok, ok, None, None]
    assert call(acc, abase, i5=257) == 2              # more than 256 nodes
    assert call(acc, abase, i1=5) == 2                # unknown logits dtype
    assert call(acc, abase, i7=0) == 2                # maxlen 0
    assert call(acc, abase, i9=None) == 1             # no path buffer
    assert call(acc, abase, i0=ok + 1) == 5           # bf16 logits on an odd address
    assert call(acc, abase, i6=0) == 0                # batch 0: nothing to do
