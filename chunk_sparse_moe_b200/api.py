"""Thin torch-facing wrappers of the C ABI (argument marshalling only)."""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import lib


class BlockFFNError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.blockffn_status_string(status).decode()
        detail = lib.blockffn_last_error_message().decode()
        super().__init__(f"{where}: {msg}" + (f" ({detail})" if detail else ""))
        self.status = status


def _check(status: int, where: str) -> None:
    if status != _lib.OK:
        raise BlockFFNError(status, where)


_DT = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}: use float32 or bfloat16")
    return _DT[t.dtype]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def version() -> int:
    return lib.blockffn_version()


def num_sms() -> int:
    return lib.blockffn_num_sms()


def set_wait_limit_ns(ns: int) -> None:
    """Bound of every in-kernel spin-wait (nanoseconds) for later launches."""
    lib.blockffn_set_wait_limit_ns(int(ns))


def debug_skip_flag(unit: int) -> None:
    """Failure-test support: the finisher of expert-in unit ``unit`` never publishes
    its ready flag (-1 turns this off); see include/blockffn.h."""
    lib.blockffn_debug_skip_flag(int(unit))


def debug_set_trace(buf: Optional[torch.Tensor]) -> None:
    """Attach (or detach with None) a zeroed int64 CUDA tensor of num_sms()*64
    entries that later bf16 forward launches fill with per-block timestamps."""
    if buf is not None and (buf.dtype != torch.int64 or buf.numel() < 64 * num_sms()):
        raise ValueError("trace buffer: int64 tensor of at least num_sms()*64 entries")
    lib.blockffn_debug_set_trace(None if buf is None else _ptr(buf))


def route(x: torch.Tensor, W_r: torch.Tensor, gamma: torch.Tensor, eps: float,
          b_r: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """gates [T, E] fp32 = RMSNorm(ReLU(x W_r^T + b_r)) over the experts."""
    T, d_h = x.shape
    E = W_r.shape[0]
    if out is None:
        out = torch.empty((T, E), dtype=torch.float32, device=x.device)
    st = lib.blockffn_route(_ptr(x), _ptr(W_r), _ptr(b_r), _ptr(gamma), float(eps), T, d_h, E,
                            _dtype_code(x), _ptr(out), _stream())
    _check(st, "blockffn_route")
    return out


def residual_layernorm(y: torch.Tensor, x: torch.Tensor, ln_gamma: torch.Tensor,
                       ln_beta: Optional[torch.Tensor], eps: float = 1e-5,
                       out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out [T, d_h] = LayerNorm(y + x) over d_h (scale ln_gamma, shift ln_beta or none, fp32)."""
    T, d_h = x.shape
    if out is None:
        out = torch.empty_like(x)
    st = lib.blockffn_residual_layernorm(_ptr(y), _ptr(x), _ptr(ln_gamma), _ptr(ln_beta), float(eps),
                                         T, d_h, _dtype_code(x), _ptr(out), _stream())
    _check(st, "blockffn_residual_layernorm")
    return out


def chunk_union(gates: torch.Tensor, n: int):
    """Per-chunk union of active experts: (counts [C], idx [C,E], tmask [C,E] as int32)."""
    T, E = gates.shape
    C = (T + n - 1) // n
    dev = gates.device
    counts = torch.empty(C, dtype=torch.int32, device=dev)
    idx = torch.empty((C, E), dtype=torch.int32, device=dev)
    tmask = torch.empty((C, E), dtype=torch.int32, device=dev)  # bits of a uint32
    st = lib.blockffn_chunk_union(_ptr(gates), T, E, n, _ptr(counts), _ptr(idx), _ptr(tmask),
                                  _stream())
    _check(st, "blockffn_chunk_union")
    return counts, idx, tmask


def workspace_bytes(T: int, d_h: int, E: int, d_e: int, n: int, dtype: torch.dtype,
                    with_router: bool, with_bias: bool = False) -> int:
    flags = (_lib.WS_ROUTER if with_router else 0) | (_lib.WS_EXPERT_BIAS if with_bias else 0)
    return int(lib.blockffn_forward_workspace_bytes(T, d_h, E, d_e, n, _DT[dtype], flags))


class Workspace:
    """Device scratch for ``forward`` (zeroed once; the library keeps state in it)."""

    def __init__(self, nbytes: int, device=None):
        self.buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8,
                               device=device or torch.device("cuda"))
        self.reset()

    @property
    def nbytes(self) -> int:
        return self.buf.numel()

    def reset(self) -> None:
        _check(lib.blockffn_workspace_reset(self.buf.data_ptr(), self.nbytes, _stream()),
               "blockffn_workspace_reset")

    @classmethod
    def for_shapes(cls, T, d_h, E, d_e, n, dtype, with_router, device=None,
                   with_bias: bool = False) -> "Workspace":
        nb = workspace_bytes(T, d_h, E, d_e, n, dtype, with_router, with_bias)
        if nb == 0:
            raise BlockFFNError(_lib.ERR_INVALID_ARG, "blockffn_forward_workspace_bytes")
        return cls(nb, device)


def forward(x: torch.Tensor, W_in: torch.Tensor, W_out: torch.Tensor, n: int,
            gates: Optional[torch.Tensor] = None, W_r: Optional[torch.Tensor] = None,
            b_r: Optional[torch.Tensor] = None, gamma: Optional[torch.Tensor] = None,
            eps: float = 2.0 ** -23, y: Optional[torch.Tensor] = None,
            workspace: Optional[Workspace] = None, union=None,
            b_in: Optional[torch.Tensor] = None, b_out: Optional[torch.Tensor] = None,
            ln_weight: Optional[torch.Tensor] = None, ln_bias: Optional[torch.Tensor] = None,
            ln_eps: float = 1e-5) -> torch.Tensor:
    """y [T, d_h] = sum over each chunk's union experts of
    gate * (W_out_e Swish(W_in_e x + b_in_e) + b_out_e), then LayerNorm(y + x) when
    ``ln_weight`` is given.

    ``union``: optional (counts, idx, tmask) as ``chunk_union`` returns them for
    these gates and n; the forward then uses them instead of forming the union.
    ``b_in`` [E, d_e], ``b_out`` [E, d_h], ``ln_weight``/``ln_bias`` [d_h]: fp32,
    optional (a workspace for ``b_out`` is sized with ``with_bias=True``)."""
    T, d_h = x.shape
    E, d_e, _ = W_in.shape
    if y is None:
        y = torch.empty((T, d_h), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = Workspace.for_shapes(T, d_h, E, d_e, n, x.dtype, gates is None, x.device,
                                         with_bias=b_out is not None)
    counts, idx, tmask = union if union is not None else (None, None, None)
    opts = None
    if b_in is not None or b_out is not None or ln_weight is not None:
        opts = ctypes.byref(_lib.LayerOpts(_ptr(b_in), _ptr(b_out), _ptr(ln_weight), _ptr(ln_bias),
                                           float(ln_eps)))
    st = lib.blockffn_forward(_ptr(x), _ptr(gates), _ptr(W_r), _ptr(b_r), _ptr(gamma), float(eps),
                              _ptr(counts), _ptr(idx), _ptr(tmask),
                              _ptr(W_in), _ptr(W_out), T, d_h, E, d_e, n, _dtype_code(x), opts,
                              _ptr(y), workspace.buf.data_ptr(), workspace.nbytes, _stream())
    _check(st, "blockffn_forward")
    return y


def device_status(workspace: Workspace):
    """(status, detail) of the workspace's device status word (synchronizes the stream)."""
    detail = ctypes.c_int32(0)
    st = lib.blockffn_get_device_status(workspace.buf.data_ptr(), _stream(), ctypes.byref(detail))
    return int(st), int(detail.value)
