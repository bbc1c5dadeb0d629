"""Failure detection on the GPU without faulting it.

A forward launch is told (test knob) never to announce one expert-in unit's
result (the multi-chunk kernel: its activations; the single-chunk kernel: one
block's partial sum).  The blocks that need it spin for a bounded time (50 ms
here), record BLOCKFFN_ERR_TIMEOUT in the workspace status word and return; the launch ends, the CUDA context stays usable, the
error is sticky until the workspace is reset, and the next call after a reset
is correct again.  No trap, no device assert, no endless loop.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from gpu_common import assert_close, dev, oracle_y, require_cuda, run_gpu

pytestmark = pytest.mark.gpu

ERR_TIMEOUT = 4
# the wait that runs out first is one on another thread block's result
WAIT_ON_PEERS = (6, 9)


@pytest.fixture()
def bffn():
    m = require_cuda()
    yield m
    m.debug_skip_flag(-1)
    m.set_wait_limit_ns(2_000_000_000)


def test_missing_flag_times_out_and_is_reported(bffn):
    w = wl.chunk32()
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, torch.bfloat16, False)
    x, W_in, W_out = dev(w.x, torch.bfloat16), dev(w.W_in, torch.bfloat16), dev(w.W_out, torch.bfloat16)
    g = dev(w.gates, torch.float32)
    bffn.set_wait_limit_ns(50_000_000)
    bffn.debug_skip_flag(0)
    bffn.forward(x, W_in, W_out, w.n, gates=g, workspace=ws)
    st, detail = bffn.device_status(ws)
    assert st == ERR_TIMEOUT and detail in WAIT_ON_PEERS
    bffn.debug_skip_flag(-1)
    # sticky: a launch on the failed workspace does nothing and keeps the status
    y = torch.full((w.T, w.d_h), 7.0, dtype=torch.bfloat16, device="cuda")
    bffn.forward(x, W_in, W_out, w.n, gates=g, y=y, workspace=ws)
    assert bffn.device_status(ws)[0] == ERR_TIMEOUT
    assert torch.all(y == 7.0)
    # the context is still usable and a reset workspace computes correctly
    assert float(torch.ones(4, device="cuda").sum()) == 4.0
    ws.reset()
    y2, gg = run_gpu(w, ws)
    assert_close(y2, oracle_y(w, gg), "bf16", "after reset")
    assert bffn.device_status(ws) == (0, 0)


def test_multichunk_missing_flag(bffn):
    w = wl.make_injected("mc", 96, 32, 512, 16, 128, "bf16", "markov80", seed=9)
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, torch.bfloat16, False)
    bffn.set_wait_limit_ns(50_000_000)
    bffn.debug_skip_flag(1)
    run_gpu(w, ws)
    st, detail = bffn.device_status(ws)
    assert st == ERR_TIMEOUT and detail in WAIT_ON_PEERS
    bffn.debug_skip_flag(-1)
    ws.reset()
    y, g = run_gpu(w, ws)
    assert_close(y, oracle_y(w, g), "bf16", "multichunk after reset")
