"""Helpers shared by the GPU tests: upload a workload, run the library, compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

from hybrid_packed_tree_b200 import workloads as wl

TOL = {"f32": 1e-4, "bf16": 2e-2}        # max-abs error <= TOL * max|ref|, per output tensor


def to_dev(a, dtype: str, device="cuda"):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def i32(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def upload_layer(w: wl.Workload, layer: int = 0, device="cuda") -> dict:
    L = w.layers[layer]
    d = {k: to_dev(getattr(L, k), w.dtype, device) for k in ("x", "dt", "B", "C")}
    for k in ("A", "D", "h0"):
        d[k] = to_dev(getattr(L, k), "f32", device)
    return d


def upload_tree(w: wl.Workload, device="cuda") -> dict:
    return {"parent": i32(w.parent, device), "path": i32(w.path, device), "path_len": i32(w.path_len, device)}


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: {np.count_nonzero(~np.isfinite(got))} NaN/Inf values"
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    tol = TOL[dtype] * scale
    assert err <= tol, f"{what}: max|err| {err:.3e} > {TOL[dtype]:g} * max|ref| = {tol:.3e}"
    return err, scale
