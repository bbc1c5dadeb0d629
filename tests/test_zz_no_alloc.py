"""The no-allocation forward entry point (blockffn_forward_noalloc).

Some callers cannot hand the library a workspace: they run where cudaMalloc is
not allowed (memory planned up front, regions that must not synchronize the
device, plug-ins given only their input and output buffers).  For them the
library keeps its own fixed scratch array.  These tests call that entry point
directly through the C ABI and check that it gives the same output as the
ordinary forward (which uses a caller workspace) on two calls in a row -- the
second with different inputs, so nothing left in the shared scratch by the
first call leaks into the second -- and that shapes too large for the scratch
are refused before anything runs.

This file is named to be collected last, so a failure here does not hide the
other tests' results; it passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from gpu_common import BF16_MAX_REL, BF16_REL_L2, dev, oracle_y, rel_l2, require_cuda

pytestmark = pytest.mark.gpu

OK, ERR_UNSUPPORTED = 0, 2


def _noalloc(lib, x, g, W_in, W_out, n, y):
    T, d_h = x.shape
    E, d_e, _ = W_in.shape
    return lib.blockffn_forward_noalloc(x.data_ptr(), g.data_ptr(), W_in.data_ptr(), W_out.data_ptr(),
                                        T, d_h, E, d_e, n, y.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("T,n,d_e", [(32, 32, 128), (8, 8, 128), (5, 32, 128), (32, 32, 256)])
def test_noalloc_matches_forward_on_two_calls(T, n, d_e):
    """Full chunks, the 16-token variant (n <= 16), a short chunk and wider
    experts, each on two calls in a row with different inputs."""
    bffn = require_cuda()
    from chunk_sparse_moe_b200 import _lib
    d_h, E = 2048, 64
    base = wl.make_injected("noalloc", T, n, d_h, E, d_e, "bf16", "markov80", seed=T + n + d_e)
    weights = (base.W_in, base.W_out)
    W_in, W_out = dev(base.W_in, torch.bfloat16), dev(base.W_out, torch.bfloat16)
    for call, x_seed in enumerate((3, 5)):
        w = wl.make_injected("noalloc", T, n, d_h, E, d_e, "bf16", "markov80", seed=T + n + d_e,
                             weights=weights, x_seed=x_seed)
        x, g = dev(w.x, torch.bfloat16), dev(w.gates, torch.float32)
        y_ref = bffn.forward(x, W_in, W_out, w.n, gates=g)          # caller workspace
        y = torch.full_like(y_ref, float("nan"))
        st = _noalloc(_lib.lib, x, g, W_in, W_out, w.n, y)
        assert st == OK, _lib.lib.blockffn_last_error_message().decode()
        torch.cuda.synchronize()
        a = y.double().cpu().numpy()
        b = y_ref.double().cpu().numpy()
        assert np.all(np.isfinite(a)), f"call {call}: output not fully written"
        m = float(np.max(np.abs(a - b)) / np.max(np.abs(b)))
        assert m <= BF16_MAX_REL and rel_l2(a, b) <= BF16_REL_L2, f"call {call}: max {m:.2e}"
        # and against the oracle directly
        ref = oracle_y(w, w.gates.astype(np.float64))
        assert rel_l2(a, ref) <= BF16_REL_L2


def test_noalloc_empty_union_writes_zeros():
    """All gates zero after a call that left h' and counters in the shared
    scratch: y is written as exact zeros, then a normal call is correct again."""
    require_cuda()
    from chunk_sparse_moe_b200 import _lib
    w = wl.chunk32()
    x, W_in, W_out = (dev(a, torch.bfloat16) for a in (w.x, w.W_in, w.W_out))
    g = dev(w.gates, torch.float32)
    y = torch.empty((w.T, w.d_h), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(_lib.lib, x, g, W_in, W_out, w.n, y) == OK
    y0 = torch.full_like(y, float("nan"))
    assert _noalloc(_lib.lib, x, torch.zeros_like(g), W_in, W_out, w.n, y0) == OK
    torch.cuda.synchronize()
    assert not torch.any(y0 != 0) and not torch.any(torch.isnan(y0))
    y1 = torch.full_like(y, float("nan"))
    assert _noalloc(_lib.lib, x, g, W_in, W_out, w.n, y1) == OK
    torch.cuda.synchronize()
    assert torch.equal(y1, y)


def test_noalloc_refuses_what_does_not_fit():
    require_cuda()
    from chunk_sparse_moe_b200 import _lib
    # E * d_e too large for the fixed scratch: refused on the host, nothing launched
    st = _lib.lib.blockffn_forward_noalloc(16, 16, 16, 16, 32, 2048, 256, 512, 32, 16,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == ERR_UNSUPPORTED
    assert b"scratch" in _lib.lib.blockffn_last_error_message()
    # more than one chunk: refused
    st = _lib.lib.blockffn_forward_noalloc(16, 16, 16, 16, 64, 2048, 64, 128, 32, 16,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == ERR_UNSUPPORTED
