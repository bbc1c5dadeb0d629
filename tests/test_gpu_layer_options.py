"""GPU parity of the layer's optional parts: the experts' fc1/fc2 biases and the
closing LayerNorm(y + x), on every kernel path, against the fp64 oracle.

Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
Deployment", Router Architecture Setup (each expert's fc1 and fc2 are
nn.Linear layers, bias on by default) and Full BlockFFN Layer with Combined
Losses (the gate multiplies the whole expert output; the expert sum plus the
input goes through nn.LayerNorm over the hidden dimension).

Paths: the single-chunk kernel (N = 32 and N = 16, ragged chunks, the empty
union, the routed step, 64 row tiles), the group kernel with the per-token bias
sums, and the fp32 path; the LayerNorm kernel follows each of them.
Tolerances as everywhere: bf16 max |dy| <= 1e-2 max |y_ref| and relative L2
<= 5e-3; fp32 relative L2 <= 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_common import assert_close, dev, require_cuda, tdtype, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bffn():
    return require_cuda()


def _params(w, seed, biases=True, ln=True, scale=4.0, shift=True):
    b_in, b_out = wl.expert_biases(seed, w.E, w.d_e, w.d_h, scale) if biases else (None, None)
    lw, lb = wl.layernorm_params(seed, w.d_h) if ln else (None, None)
    if not shift:
        lb = None
    return b_in, b_out, lw, lb


def _run(bffn, w, b_in, b_out, lw, lb, eps=1e-5, workspace=None):
    """The forward with options through the binding; returns (y fp64, gates fp64)."""
    dt = tdtype(w)
    x, W_in, W_out = dev(w.x, dt), dev(w.W_in, dt), dev(w.W_out, dt)
    f32 = lambda a: None if a is None else dev(a, torch.float32)
    kw = dict(b_in=f32(b_in), b_out=f32(b_out), ln_weight=f32(lw), ln_bias=f32(lb), ln_eps=eps,
              workspace=workspace)
    if w.uses_router:
        W_r, gamma = dev(w.W_r, dt), dev(w.gamma, torch.float32)
        b_r = None if w.b_r is None else dev(w.b_r, torch.float32)
        y = bffn.forward(x, W_in, W_out, w.n, W_r=W_r, b_r=b_r, gamma=gamma, eps=w.eps, **kw)
        gates = bffn.route(x, W_r, gamma, w.eps, b_r=b_r)
    else:
        gates = dev(w.gates, torch.float32)
        y = bffn.forward(x, W_in, W_out, w.n, gates=gates, **kw)
    torch.cuda.synchronize()
    return to_np64(y), to_np64(gates)


def _ref(w, g, b_in, b_out, lw, lb, eps=1e-5):
    y = oracle.forward_chunk_union(w.x, g, w.W_in, w.W_out, w.n, b_in, b_out)
    if lw is not None:
        y = oracle.residual_layernorm(y, w.x, lw, np.zeros(w.d_h) if lb is None else lb, eps)
    return y


def _check(bffn, w, seed, what, **opt):
    p = _params(w, seed, **opt)
    y, g = _run(bffn, w, *p)
    assert_close(y, _ref(w, g, *p), w.dtype, what)
    return y, g, p


# ------------------------------------------------- single-chunk kernel --

@pytest.mark.parametrize("biases,ln", [(True, True), (True, False), (False, True)])
def test_chunk32_options(bffn, biases, ln):
    """The decode step of the benchmark's workload (N = 32): biases, the
    LayerNorm, and both."""
    _check(bffn, wl.chunk32(), 11, f"chunk32 biases={biases} ln={ln}", biases=biases, ln=ln)


@pytest.mark.parametrize("T,n,d_h,E,d_e,regime", [
    (8, 8, 1024, 32, 256, "markov80"),     # N = 16 tokens per MMA, two row tiles per expert
    (20, 32, 512, 16, 128, "markov80"),    # short chunk: rows past T are not stored
    (1, 1, 256, 8, 128, "bern0.2"),        # one token
    (32, 32, 4096, 32, 128, "all_on"),     # 32 row tiles
])
def test_single_chunk_options_shapes(bffn, T, n, d_h, E, d_e, regime):
    w = wl.make_injected("opts", T, n, d_h, E, d_e, "bf16", regime, seed=T + d_h)
    _check(bffn, w, T + 5, f"single chunk T{T} n{n} d_h{d_h} E{E} d_e{d_e}")


def test_single_chunk_layernorm_without_shift(bffn):
    w = wl.make_injected("noshift", 32, 32, 1024, 16, 128, "bf16", "markov80", seed=3)
    _check(bffn, w, 3, "LayerNorm without shift", biases=False, shift=False)


def test_single_chunk_options_many_row_tiles(bffn):
    """64 row tiles of y: clusters own two each (biases in both), and the
    LayerNorm's rows exceed what its one-pass variant holds in registers."""
    w = wl.make_injected("wide_dh", 32, 32, 8192, 16, 128, "bf16", "markov80", seed=41)
    _check(bffn, w, 41, "d_h 8192 with options")


def test_empty_union_with_options(bffn):
    """No active expert: the expert sum and the gated biases are zero, so y is
    LayerNorm(x), or exact zeros without it."""
    w = wl.make_injected("off", 32, 32, 1024, 16, 128, "bf16", "all_off", seed=2)
    y, g, p = _check(bffn, w, 2, "empty union, LayerNorm")
    y0, _ = _run(bffn, w, p[0], p[1], None, None)
    assert not np.any(y0), "gated biases of inactive experts must not appear"


def test_routed_single_chunk_with_options(bffn):
    """The routed decode step with biases and the LayerNorm, given the GPU's
    gates (whose masks the router tests check)."""
    w = wl.make_routed("routed_opts", 32, 32, 2048, 64, 128, "bf16", seed=31, bias_shift=-0.8)
    _check(bffn, w, 31, "routed with options")


def test_options_deterministic(bffn):
    """Two calls give the same bits: the bias sums and the LayerNorm statistics
    are added in fixed orders."""
    w = wl.chunk32(seed=5)
    p = _params(w, 5)
    y1, _ = _run(bffn, w, *p)
    y2, _ = _run(bffn, w, *p)
    assert np.array_equal(y1, y2)


@pytest.mark.parametrize("T", [32, 300])
def test_options_alternating_on_one_workspace(bffn, T):
    """One workspace (sized for fc2 biases), calls with and without biases and the
    LayerNorm in turn: the layout and the per-launch counters stay in step."""
    w = wl.make_injected("alt", T, 32, 2048 if T == 32 else 512, 64, 128, "bf16", "markov80", seed=6)
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, torch.bfloat16, False, "cuda",
                                   with_bias=True)
    p = _params(w, 6)
    for k in range(6):
        use_ln, use_b = k % 2 == 0, k % 3 != 2
        q = (p[0] if use_b else None, p[1] if use_b else None, p[2] if use_ln else None,
             p[3] if use_ln else None)
        y, g = _run(bffn, w, *q, workspace=ws)
        assert_close(y, _ref(w, g, *q), "bf16", f"call {k}")
    assert bffn.device_status(ws) == (0, 0)


# -------------------------------------------------------- group kernel --

@pytest.mark.parametrize("T,n,d_h,E,d_e,regime", [
    (300, 32, 512, 64, 128, "markov80"),   # 10 chunks in two groups, ragged tail
    (70, 8, 256, 16, 256, "bern0.2"),      # short chunks, N = 128, wide experts
    (96, 32, 1024, 64, 128, "markov90"),
])
def test_group_kernel_options(bffn, T, n, d_h, E, d_e, regime):
    w = wl.make_injected("group_opts", T, n, d_h, E, d_e, "bf16", regime, seed=T + n)
    _check(bffn, w, T, f"group T{T} n{n} d_h{d_h} E{E} d_e{d_e}")


def test_batch16_with_biases(bffn):
    """The batch16 workload (16 chunks, one group of 256 tokens x 2) with biases."""
    w = wl.batch16()
    _check(bffn, w, 16, "batch16 biases", ln=False, scale=1.0)


def test_group_bias_needs_a_sized_workspace(bffn):
    """fc2 biases on the multi-chunk path need the per-token bias sums: a workspace
    sized without BLOCKFFN_WS_EXPERT_BIAS is refused on the host."""
    w = wl.make_injected("ws", 96, 32, 512, 16, 128, "bf16", "markov80", seed=9)
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, torch.bfloat16, False, "cuda")
    b_in, b_out, _, _ = _params(w, 9, ln=False)
    with pytest.raises(bffn.BlockFFNError) as ei:
        _run(bffn, w, b_in, b_out, None, None, workspace=ws)
    assert ei.value.status == 5   # BLOCKFFN_ERR_WORKSPACE


# ------------------------------------------------------------ fp32 path --

@pytest.mark.parametrize("T,n", [(32, 32), (70, 16)])
def test_f32_path_options(bffn, T, n):
    w = wl.make_injected("f32_opts", T, n, 256, 16, 64, "f32", "markov80", seed=T)
    _check(bffn, w, T, f"fp32 T{T} n{n}")


def test_f32_routed_with_options(bffn):
    _check(bffn, wl.tiny_f32(), 1, "fp32 routed with options")
