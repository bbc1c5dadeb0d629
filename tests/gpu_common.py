"""Shared helpers of the GPU parity tests: run the CUDA path through the Python
binding of the C ABI, run the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

# tolerances (bf16: max |dy| <= 1e-2 max |y_ref| and relative L2 <= 5e-3;
# fp32: relative L2 <= 1e-5)
BF16_MAX_REL = 1e-2
BF16_REL_L2 = 5e-3
F32_REL_L2 = 1e-5


def require_cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected on a machine without CUDA")
    import chunk_sparse_moe_b200 as bffn
    return bffn


def dev(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def tdtype(w: wl.Workload) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def run_gpu(w: wl.Workload, workspace=None):
    """Forward on the GPU; returns (y fp64, gates used fp64)."""
    bffn = require_cuda()
    dt = tdtype(w)
    x, W_in, W_out = dev(w.x, dt), dev(w.W_in, dt), dev(w.W_out, dt)
    if w.uses_router:
        W_r = dev(w.W_r, dt)
        gamma = dev(w.gamma, torch.float32)
        b_r = None if w.b_r is None else dev(w.b_r, torch.float32)
        y = bffn.forward(x, W_in, W_out, w.n, W_r=W_r, b_r=b_r, gamma=gamma, eps=w.eps,
                         workspace=workspace)
        gates = bffn.route(x, W_r, gamma, w.eps, b_r=b_r)
    else:
        gates = dev(w.gates, torch.float32)
        y = bffn.forward(x, W_in, W_out, w.n, gates=gates, workspace=workspace)
    torch.cuda.synchronize()
    return to_np64(y), to_np64(gates)


def rel_l2(a, b) -> float:
    den = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / den if den > 0 else float(np.linalg.norm(a))


def assert_close(y, y_ref, dtype: str, what: str = ""):
    assert y.shape == y_ref.shape
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    if not np.any(y_ref):
        assert not np.any(y), f"{what}: expected exact zeros"
        return
    r = rel_l2(y, y_ref)
    m = float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)))
    if dtype == "bf16":
        assert m <= BF16_MAX_REL and r <= BF16_REL_L2, f"{what}: max {m:.3e} relL2 {r:.3e}"
    else:
        assert r <= F32_REL_L2, f"{what}: relL2 {r:.3e}"
    # rows of tokens without an active expert are exact zeros
    zero_rows = ~np.any(y_ref != 0, axis=1)
    assert not np.any(y[zero_rows]), f"{what}: masked rows not zero"


def oracle_y(w: wl.Workload, gates64: np.ndarray, tokens=None):
    """Oracle output on whole chunks; ``tokens`` selects chunk-aligned token ranges."""
    if tokens is None:
        return oracle.forward_chunk_union(w.x, gates64, w.W_in, w.W_out, w.n)
    return oracle.forward_chunk_union(w.x[tokens], gates64[tokens], w.W_in, w.W_out, w.n)


def chunk_tokens(w: wl.Workload, chunks) -> np.ndarray:
    idx = []
    for c in chunks:
        idx.extend(range(c * w.n, min(w.T, c * w.n + w.n)))
    return np.array(idx, dtype=np.int64)


def router_mask_band(w: wl.Workload) -> np.ndarray:
    """Per (token, expert) rounding band of an fp32-accumulated logit:
    gamma_K * sum_k |W_r[e,k] x[t,k]| (+|b|), K = d_h + 1 (Higham's bound)."""
    K = w.d_h + 1
    u = 2.0 ** -24
    gK = K * u / (1 - K * u)
    mag = np.abs(w.x.astype(np.float64)) @ np.abs(w.W_r.astype(np.float64)).T
    if w.b_r is not None:
        mag = mag + np.abs(w.b_r.astype(np.float64))[None, :]
    return gK * mag
