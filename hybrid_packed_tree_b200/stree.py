"""Thin ctypes binding of ``libstree.so`` (the C ABI declared in include/stree.h).

Argument marshalling only: shapes are read from the torch tensors, pointers are
passed as they are, and every step of the scan runs in the library's CUDA
kernels.  Importing this module loads the library and raises ImportError when it
has not been built (``python -m hybrid_packed_tree_b200.build``); there is no
fallback of any kind.

The functions carry the C names.  Tensors must be contiguous CUDA tensors in the
layouts of the header: x [b,T,H,P], dt [b,T,H], A/D [H] fp32, B/C [b,T,G,N],
h0/h_new [b,H,P,N] fp32, y like x, parent [b,T] int32, path [b,maxlen] int32,
path_len [b] int32.  ``stream`` defaults to torch's current stream.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB

if not os.path.exists(LIB):
    raise ImportError(f"libstree.so is not built ({LIB}); run `python -m hybrid_packed_tree_b200.build`")

_lib = ctypes.CDLL(LIB)

STREE_OK = 0
STATUS_NAMES = {
    0: "STREE_OK", 1: "STREE_ERR_INVALID_ARG", 2: "STREE_ERR_UNSUPPORTED", 3: "STREE_ERR_BAD_TREE",
    4: "STREE_ERR_BAD_PATH", 5: "STREE_ERR_MISALIGNED", 6: "STREE_ERR_CUDA", 7: "STREE_ERR_TIMEOUT",
    8: "STREE_ERR_NO_TREE",
}
STREE_F32, STREE_BF16 = 0, 1
KERNELS = {"auto": 0, "simt": 1, "tc": 2, "small": 3}

# Every exported symbol of include/stree.h.
EXPORTS = (
    "stree_ctx_create", "stree_ctx_destroy", "stree_ctx_set_kernel", "stree_ctx_launch_count",
    "stree_ctx_last_kernel", "stree_ctx_set_wait_limit", "stree_ctx_set_test_fault",
    "stree_build_tree",
    "stree_tree_scan", "stree_commit", "stree_tree_scan_commit", "stree_tree_scan_commit_noalloc",
    "stree_resolve_path", "stree_unrolled_scan", "stree_accept_greedy", "stree_accept_sampling",
    "stree_gdn_tree_scan_commit", "stree_tree_attention", "stree_tree_attention_workspace_size",
    "stree_sync_check", "stree_status_string", "stree_version",
)

_vp, _i, _ip = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int32)
_lib.stree_ctx_create.argtypes = [ctypes.POINTER(_vp)]
_lib.stree_ctx_destroy.argtypes = [_vp]
_lib.stree_ctx_set_kernel.argtypes = [_vp, _i]
_lib.stree_ctx_launch_count.argtypes = [_vp, ctypes.POINTER(ctypes.c_int64)]
_lib.stree_ctx_last_kernel.argtypes = [_vp, ctypes.POINTER(ctypes.c_int)]
_lib.stree_ctx_set_wait_limit.argtypes = [_vp, ctypes.c_uint64]
_lib.stree_ctx_set_test_fault.argtypes = [_vp, _i]
_lib.stree_build_tree.argtypes = [_vp, _vp, _i, _i, _vp, _vp, _vp]
_lib.stree_tree_scan.argtypes = [_vp] * 9 + [_i] * 7 + [_vp, _vp]
_lib.stree_commit.argtypes = [_vp, _vp, _vp, _i, _vp, _vp]
_lib.stree_tree_scan_commit.argtypes = [_vp] * 9 + [_i] * 7 + [_vp, _vp, _i, _vp, _vp, _vp]
_lib.stree_tree_scan_commit_noalloc.argtypes = [_vp] * 8 + [_i] * 7 + [_vp, _vp, _i, _vp, _vp, _vp, _vp]
_lib.stree_resolve_path.argtypes = [_vp, _vp, _vp, _i, _vp, _vp]
_lib.stree_unrolled_scan.argtypes = [_vp] * 9 + [_i] * 9 + [_vp, _vp, _vp, _vp]
_lib.stree_accept_greedy.argtypes = [_vp, _i, _i, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.stree_accept_sampling.argtypes = [_vp, _vp, _i, _i, _vp, _vp, _i, _i, ctypes.c_float, _vp, _vp, _i, _vp,
                                        _vp, _vp, _vp, _vp]
_lib.stree_gdn_tree_scan_commit.argtypes = [_vp] * 8 + [_i] * 7 + [_vp, _vp, _i, _vp, _vp, _vp, _vp]
_lib.stree_tree_attention.argtypes = [_vp] * 7 + [_i] * 6 + [ctypes.c_float, _i, _vp, _vp, ctypes.c_size_t, _vp, _vp]
_lib.stree_tree_attention_workspace_size.argtypes = [_i] * 6 + [ctypes.POINTER(ctypes.c_size_t)]
_lib.stree_sync_check.argtypes = [_vp, _vp, _ip]
_lib.stree_status_string.argtypes = [_i]
_lib.stree_status_string.restype = ctypes.c_char_p
_lib.stree_version.argtypes = []
for _name in EXPORTS:
    if _name not in ("stree_status_string",):
        getattr(_lib, _name).restype = ctypes.c_int


class StreeError(RuntimeError):
    def __init__(self, status: int, where: str, info=None):
        self.status = int(status)
        self.info = info
        msg = f"{where}: {STATUS_NAMES.get(status, status)} ({stree_status_string(status)})"
        if info is not None:
            msg += f" info={list(info)}"
        super().__init__(msg)


def _check(st: int, where: str):
    if st != STREE_OK:
        raise StreeError(st, where)


def stree_status_string(status: int) -> str:
    return _lib.stree_status_string(int(status)).decode()


def stree_version() -> int:
    return int(_lib.stree_version())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t, name, dtypes=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return ctypes.c_void_p(t.data_ptr())


def _io_dtype(x):
    if x.dtype == torch.bfloat16:
        return STREE_BF16
    if x.dtype == torch.float32:
        return STREE_F32
    raise TypeError(f"x has dtype {x.dtype}; fp32 and bf16 are supported")


class Ctx:
    """Owns one ``stree_ctx``; closed by ``stree_ctx_destroy`` (or garbage collection)."""

    def __init__(self):
        h = ctypes.c_void_p()
        _check(_lib.stree_ctx_create(ctypes.byref(h)), "stree_ctx_create")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            _lib.stree_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def stree_ctx_create() -> Ctx:
    return Ctx()


def stree_ctx_destroy(ctx: Ctx):
    ctx.close()


def stree_ctx_set_kernel(ctx: Ctx, kernel="auto"):
    k = KERNELS[kernel] if isinstance(kernel, str) else int(kernel)
    _check(_lib.stree_ctx_set_kernel(ctx.handle, k), "stree_ctx_set_kernel")


def stree_ctx_launch_count(ctx: Ctx) -> int:
    n = ctypes.c_int64(0)
    _check(_lib.stree_ctx_launch_count(ctx.handle, ctypes.byref(n)), "stree_ctx_launch_count")
    return int(n.value)


def stree_ctx_last_kernel(ctx: Ctx) -> str:
    """Name ("simt", "tc" or "small") of the kernel that ran the last scan; "auto" before any."""
    k = ctypes.c_int(0)
    _check(_lib.stree_ctx_last_kernel(ctx.handle, ctypes.byref(k)), "stree_ctx_last_kernel")
    return {v: n for n, v in KERNELS.items()}[int(k.value)]


def stree_ctx_set_wait_limit(ctx: Ctx, ns: int = 0):
    """Bounded-wait limit of the tensor-core kernel in ns (0: the default, about 1 s)."""
    _check(_lib.stree_ctx_set_wait_limit(ctx.handle, int(ns)), "stree_ctx_set_wait_limit")


def stree_ctx_set_test_fault(ctx: Ctx, fault: int = 0):
    """Failure-path test hook: 1 makes a bounded wait of the tensor-core kernel run out."""
    _check(_lib.stree_ctx_set_test_fault(ctx.handle, int(fault)), "stree_ctx_set_test_fault")


def stree_build_tree(ctx: Ctx, parent, anc_out=None, depth_out=None, stream=None):
    batch, T = parent.shape
    _check(_lib.stree_build_tree(ctx.handle, _ptr(parent, "parent", (torch.int32,)), T, batch,
                                 _ptr(anc_out, "anc_out", (torch.int32,)),
                                 _ptr(depth_out, "depth_out", (torch.int32,)), _stream(stream)),
           "stree_build_tree")


def _scan_ptrs(x, dt, A, B, C, D, h0, y):
    io = (x.dtype,)
    return [_ptr(x, "x", (torch.float32, torch.bfloat16)), _ptr(dt, "dt", io), _ptr(A, "A", (torch.float32,)),
            _ptr(B, "B", io), _ptr(C, "C", io), _ptr(D, "D", (torch.float32,)),
            _ptr(h0, "h0", (torch.float32,))], _ptr(y, "y", io)


def _dims(x, B):
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return [T, batch, H, P, N, G]


def stree_tree_scan(ctx: Ctx, x, dt, A, B, C, D, h0, parent, y, stream=None):
    """y <- packed tree scan.  parent=None reuses the context's current tree."""
    ins, yp = _scan_ptrs(x, dt, A, B, C, D, h0, y)
    st = _lib.stree_tree_scan(ctx.handle, *ins, _ptr(parent, "parent", (torch.int32,)),
                              *_dims(x, B), _io_dtype(x), yp, _stream(stream))
    _check(st, "stree_tree_scan")
    return y


def stree_commit(ctx: Ctx, path, path_len, h_new, stream=None):
    """h_new <- activation replay of the accepted paths over the last scan's inputs."""
    st = _lib.stree_commit(ctx.handle, _ptr(path, "path", (torch.int32,)),
                           _ptr(path_len, "path_len", (torch.int32,)), path.shape[1],
                           _ptr(h_new, "h_new", (torch.float32,)), _stream(stream))
    _check(st, "stree_commit")
    return h_new


def stree_tree_scan_commit(ctx: Ctx, x, dt, A, B, C, D, h0, parent, path, path_len, y, h_new, stream=None):
    """(y, h_new) <- fused scan + commit (h0 read once)."""
    ins, yp = _scan_ptrs(x, dt, A, B, C, D, h0, y)
    st = _lib.stree_tree_scan_commit(ctx.handle, *ins, _ptr(parent, "parent", (torch.int32,)),
                                     *_dims(x, B), _io_dtype(x),
                                     _ptr(path, "path", (torch.int32,)),
                                     _ptr(path_len, "path_len", (torch.int32,)), path.shape[1],
                                     yp, _ptr(h_new, "h_new", (torch.float32,)), _stream(stream))
    _check(st, "stree_tree_scan_commit")
    return y, h_new


def stree_tree_scan_commit_noalloc(x, dt, A, B, C, D, h0, parent, path, path_len, y, h_new, err_out=None,
                                   stream=None):
    """(y, h_new) <- fused scan + commit with no context and no allocation.

    Scratch comes from the library's fixed device array; err_out (device int32[4])
    receives this call's error word.  Calls on one device must not overlap.
    """
    ins, yp = _scan_ptrs(x, dt, A, B, C, D, h0, y)
    st = _lib.stree_tree_scan_commit_noalloc(*ins, _ptr(parent, "parent", (torch.int32,)), *_dims(x, B),
                                             _io_dtype(x), _ptr(path, "path", (torch.int32,)),
                                             _ptr(path_len, "path_len", (torch.int32,)), path.shape[1], yp,
                                             _ptr(h_new, "h_new", (torch.float32,)),
                                             _ptr(err_out, "err_out", (torch.int32,)), _stream(stream))
    _check(st, "stree_tree_scan_commit_noalloc")
    return y, h_new


def stree_unrolled_scan(x, dt, A, B, C, D, h0, paths, path_len, y_paths, h_paths, err_out=None, stream=None):
    """(y_paths, h_paths) <- every path scanned as its own sequence (the unrolled-tree baseline).

    paths [b, n_paths, max_depth] int32, path_len [b, n_paths] int32,
    y_paths [b, n_paths, max_depth, H, P] in x's dtype, h_paths [b, n_paths, H, P, N] fp32.
    """
    ins, yp = _scan_ptrs(x, dt, A, B, C, D, h0, y_paths)
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    st = _lib.stree_unrolled_scan(*ins[:7], _ptr(paths, "paths", (torch.int32,)),
                                  _ptr(path_len, "path_len", (torch.int32,)), T, batch, paths.shape[1],
                                  paths.shape[2], H, P, N, G, _io_dtype(x), yp,
                                  _ptr(h_paths, "h_paths", (torch.float32,)),
                                  _ptr(err_out, "err_out", (torch.int32,)), _stream(stream))
    _check(st, "stree_unrolled_scan")
    return y_paths, h_paths


def stree_accept_greedy(logits, draft_tokens, parent, pred, accepted_path, path_len, bonus_token, err_out=None,
                        stream=None):
    """Greedy tree verification: (pred, accepted_path, path_len, bonus_token) from the
    target's logits [b, T, V] (fp32 or bf16) and the draft tokens [b, T]."""
    batch, T, V = logits.shape
    st = _lib.stree_accept_greedy(_ptr(logits, "logits", (torch.float32, torch.bfloat16)), _io_dtype(logits), V,
                                  _ptr(draft_tokens, "draft_tokens", (torch.int32,)),
                                  _ptr(parent, "parent", (torch.int32,)), T, batch, accepted_path.shape[1],
                                  _ptr(pred, "pred", (torch.int32,)), _ptr(accepted_path, "accepted_path", (torch.int32,)),
                                  _ptr(path_len, "path_len", (torch.int32,)),
                                  _ptr(bonus_token, "bonus_token", (torch.int32,)),
                                  _ptr(err_out, "err_out", (torch.int32,)), _stream(stream))
    _check(st, "stree_accept_greedy")
    return pred, accepted_path, path_len, bonus_token


def stree_accept_sampling(target_logits, draft_logits, draft_tokens, parent, temperature, u_accept, u_bonus,
                          accepted_path, path_len, bonus_token, err_out=None, stream=None):
    """Stochastic tree verification by multi-step speculative sampling: (accepted_path,
    path_len, bonus_token) from the target's and the draft's logits [b, T, V] (fp32 or
    bf16, same dtype), the draft tokens [b, T] and the uniforms u_accept [b, T] and
    u_bonus [b] (fp32)."""
    batch, T, V = target_logits.shape
    if draft_logits.shape != target_logits.shape or draft_logits.dtype != target_logits.dtype:
        raise ValueError("draft_logits must match target_logits in shape and dtype")
    st = _lib.stree_accept_sampling(_ptr(target_logits, "target_logits", (torch.float32, torch.bfloat16)),
                                    _ptr(draft_logits, "draft_logits", (target_logits.dtype,)),
                                    _io_dtype(target_logits), V, _ptr(draft_tokens, "draft_tokens", (torch.int32,)),
                                    _ptr(parent, "parent", (torch.int32,)), T, batch, float(temperature),
                                    _ptr(u_accept, "u_accept", (torch.float32,)),
                                    _ptr(u_bonus, "u_bonus", (torch.float32,)), accepted_path.shape[1],
                                    _ptr(accepted_path, "accepted_path", (torch.int32,)),
                                    _ptr(path_len, "path_len", (torch.int32,)),
                                    _ptr(bonus_token, "bonus_token", (torch.int32,)),
                                    _ptr(err_out, "err_out", (torch.int32,)), _stream(stream))
    _check(st, "stree_accept_sampling")
    return accepted_path, path_len, bonus_token


def stree_gdn_tree_scan_commit(q, k, v, alpha, beta, S0, parent, o, path=None, path_len=None, S_new=None,
                               err_out=None, stream=None, erase=None):
    """Gated delta rule over the packed tree: o [b, T, Hv, dv] for every node and, when
    path / path_len / S_new are given, the accepted path's state S_new [b, Hv, dv, dk].
    q, k [b, T, Hk, dk] and v [b, T, Hv, dv] in one dtype (fp32 or bf16); alpha, beta
    [b, T, Hv] and S0 fp32; erase [b, T, Hv] fp32 (None: erase = beta; zeros: gated
    linear attention)."""
    batch, T, Hk, dk = k.shape
    Hv, dv = v.shape[2], v.shape[3]
    io = (v.dtype,)
    st = _lib.stree_gdn_tree_scan_commit(
        _ptr(q, "q", io), _ptr(k, "k", io), _ptr(v, "v", (torch.float32, torch.bfloat16)),
        _ptr(alpha, "alpha", (torch.float32,)), _ptr(beta, "beta", (torch.float32,)),
        _ptr(erase, "erase", (torch.float32,)), _ptr(S0, "S0", (torch.float32,)), _ptr(parent, "parent", (torch.int32,)), T, batch, Hv, Hk, dk, dv,
        _io_dtype(v), _ptr(path, "path", (torch.int32,)), _ptr(path_len, "path_len", (torch.int32,)),
        path.shape[1] if path is not None else 0, _ptr(o, "o", io), _ptr(S_new, "S_new", (torch.float32,)),
        _ptr(err_out, "err_out", (torch.int32,)), _stream(stream))
    _check(st, "stree_gdn_tree_scan_commit")
    return o, S_new


def stree_tree_attention_workspace_size(n_nodes, batch, ctx_cap, heads_q, heads_kv, head_dim=128) -> int:
    """Bytes of the workspace stree_tree_attention splits into on the current device (0: no split)."""
    n = ctypes.c_size_t(0)
    _check(_lib.stree_tree_attention_workspace_size(int(n_nodes), int(batch), int(ctx_cap), int(heads_q),
                                                    int(heads_kv), int(head_dim), ctypes.byref(n)),
           "stree_tree_attention_workspace_size")
    return int(n.value)


def stree_tree_attention(q, k_ctx, v_ctx, k_tree, v_tree, ctx_len, parent, o, scale, err_out, workspace=None,
                         stream=None):
    """Tree-masked attention: o [b, T, Hq, 128] (bf16) from q [b, T, Hq, 128], the
    context cache k_ctx / v_ctx [b, S, Hkv, 128] (S may be 0), the tree's own k_tree /
    v_tree [b, T, Hkv, 128], ctx_len [b] and parent [b, T].  workspace: a device
    uint8 tensor of stree_tree_attention_workspace_size() bytes, or None (no split)."""
    batch, T, Hq, d = q.shape
    S, Hkv = k_ctx.shape[1], k_ctx.shape[2]
    bf = (torch.bfloat16,)
    ws = _ptr(workspace, "workspace", (torch.uint8,)) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    st = _lib.stree_tree_attention(_ptr(q, "q", bf), _ptr(k_ctx, "k_ctx", bf) if S else None,
                                   _ptr(v_ctx, "v_ctx", bf) if S else None, _ptr(k_tree, "k_tree", bf),
                                   _ptr(v_tree, "v_tree", bf), _ptr(ctx_len, "ctx_len", (torch.int32,)),
                                   _ptr(parent, "parent", (torch.int32,)), T, batch, S, Hq, Hkv, d, float(scale),
                                   STREE_BF16, _ptr(o, "o", bf), ws, ws_bytes,
                                   _ptr(err_out, "err_out", (torch.int32,)), _stream(stream))
    _check(st, "stree_tree_attention")
    return o


def stree_resolve_path(ctx: Ctx, path, path_len, leaf_out, stream=None):
    st = _lib.stree_resolve_path(ctx.handle, _ptr(path, "path", (torch.int32,)),
                                 _ptr(path_len, "path_len", (torch.int32,)), path.shape[1],
                                 _ptr(leaf_out, "leaf_out", (torch.int32,)), _stream(stream))
    _check(st, "stree_resolve_path")
    return leaf_out


def stree_sync_check(ctx: Ctx, stream=None, raise_on_error: bool = True):
    """Synchronise, read and clear the device error word; returns (status, info[4])."""
    info = (ctypes.c_int32 * 4)()
    st = _lib.stree_sync_check(ctx.handle, _stream(stream), info)
    if st != STREE_OK and raise_on_error:
        raise StreeError(st, "stree_sync_check", list(info))
    return st, list(info)
