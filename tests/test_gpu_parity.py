"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

* chunk union: bit-exact counts / index lists / token masks;
* router: gate-zero masks bit-exact outside the fp32 rounding band of the logit,
  gate values to fp32 accuracy;
* forward: bf16 max |dy| <= 1e-2 max|y_ref| and relative L2 <= 5e-3, fp32
  relative L2 <= 1e-5; rows of tokens with no active expert exactly zero;
* the five workloads at full size (whole outputs where the oracle is quick,
  whole sampled chunks where it is not), small shapes that span several tiles
  with ragged tails, and the degenerate cases (empty union, one expert, all
  experts, T = 0, one token);
* determinism and workspace reuse.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_common import (assert_close, chunk_tokens, dev, oracle_y, require_cuda,
                        router_mask_band, run_gpu, to_np64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bffn():
    return require_cuda()


# ------------------------------------------------------------ chunk union --

def _union_case(seed, T, E, n, p_on=0.3):
    rng = np.random.default_rng(seed)
    g = np.where(rng.random((T, E)) < p_on, rng.standard_normal((T, E)), 0.0).astype(np.float32)
    g[rng.random((T, E)) < 0.05] = -0.0      # negative zero counts as inactive
    return g


@pytest.mark.parametrize("T,E,n", [(32, 64, 32), (70, 16, 32), (1, 1, 1), (33, 256, 32),
                                   (100, 128, 8), (7, 3, 7), (4096, 64, 32), (257, 40, 31),
                                   (64, 64, 1)])
def test_chunk_union_bit_exact(bffn, T, E, n):
    g = _union_case(T * 1000 + E + n, T, E, n)
    counts, idx, tmask = bffn.chunk_union(dev(g, torch.float32), n)
    rc, ri, rt = oracle.chunk_union(g, n)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(idx.cpu().numpy(), ri)
    assert np.array_equal(tmask.cpu().numpy().view(np.uint32), rt)


def test_chunk_union_markov_workload(bffn):
    w = wl.chunk32()
    counts, idx, tmask = bffn.chunk_union(dev(w.gates, torch.float32), w.n)
    rc, ri, rt = oracle.chunk_union(w.gates, w.n)
    assert np.array_equal(counts.cpu().numpy(), rc) and np.array_equal(idx.cpu().numpy(), ri)
    assert np.array_equal(tmask.cpu().numpy().view(np.uint32), rt)


# ----------------------------------------------------------------- router --

def _check_route(bffn, w):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    x, W_r = dev(w.x, dt), dev(w.W_r, dt)
    b = None if w.b_r is None else dev(w.b_r, torch.float32)
    g = to_np64(bffn.route(x, W_r, dev(w.gamma, torch.float32), w.eps, b_r=b))
    logits, g_ref = oracle.route(w.x, w.W_r, w.gamma, w.eps, b_r=w.b_r)
    band = router_mask_band(w)
    sure = np.abs(logits) > band
    # outside the worst-case fp32 rounding band of the logit the mask is bit-exact
    assert np.array_equal((g != 0)[sure], (g_ref != 0)[sure]), "gate-zero mask differs"
    # inside it either bit is a correct rounding of the fp32 sum; typical errors are
    # ~1000x below the worst-case band, so flips stay rare
    flips = int(np.sum((g != 0)[~sure] != (g_ref != 0)[~sure]))
    assert flips <= max(3, int(1e-5 * g.size)), f"{flips} mask flips inside the band"
    # values: fp32 accumulation and normalisation
    both = (g != 0) & (g_ref != 0)
    err = np.max(np.abs(g - g_ref)[both]) if np.any(both) else 0.0
    assert err <= 1e-4 * max(1.0, float(np.max(np.abs(g_ref)))), f"gate values off by {err}"
    return g


def test_route_tiny_f32(bffn):
    _check_route(bffn, wl.tiny_f32())


def test_route_seq4096_bf16(bffn):
    _check_route(bffn, wl.seq4096())


@pytest.mark.parametrize("T,d_h,E,bias", [
    (45, 512, 192, -0.8),    # two 128-expert tiles, d_h in 2 slices, ragged last token tile
    (7, 4096, 256, None),    # fewer tokens than a tile, two 256-wide k-groups per slice
    (70, 2304, 64, -0.5),    # d_h 9 x 256: one slice of nine k-groups
    (33, 320, 48, None),     # d_h not a multiple of 256: the CUDA-core router
    (1100, 1024, 48, -0.8),  # long input: 128 tokens per cluster of 4, ragged last tile
    (2000, 512, 128, None),  # long input, d_h in 2 slices, all 128 expert rows
])
def test_route_bf16_shapes(bffn, T, d_h, E, bias):
    w = wl.make_routed("route_shape", T, 32, d_h, E, 1, "bf16", seed=T + E, bias_shift=bias)
    _check_route(bffn, w)


def test_route_edge_rows(bffn):
    """A row whose logits are all <= 0 gives zero gates; negative gamma keeps the sign."""
    w = wl.make_routed("edge", 40, 8, 128, 16, 128, "bf16", seed=3, bias_shift=-0.8)
    w.x[0] = 0.0                     # logits = bias < 0 -> all gates 0
    w.gamma = np.linspace(-1.0, 1.5, 16).astype(np.float32)
    g = _check_route(bffn, w)
    assert not np.any(g[0])


# ---------------------------------------------------------------- forward --

def test_forward_tiny_f32_router(bffn):
    w = wl.tiny_f32()
    y, g = run_gpu(w)
    assert_close(y, oracle.forward_dense(w.x, g, w.W_in, w.W_out), "f32", "tiny_f32")


@pytest.mark.parametrize("T,n,d_h,E,d_e,regime", [
    (32, 32, 128, 1, 128, "all_on"),       # one expert, one tile each way
    (32, 32, 256, 4, 128, "markov80"),
    (70, 32, 512, 16, 128, "markov80"),    # 3 chunks, ragged 6-token tail
    (70, 32, 512, 16, 256, "bern0.2"),     # two 128-row tiles per expert
    (45, 8, 384, 16, 128, "markov80"),     # N = 16 tokens per MMA, ragged
    (5, 1, 256, 8, 128, "bern0.2"),        # one-token chunks
    (1, 32, 256, 8, 128, "all_on"),        # one token in a 32-token chunk
    (96, 32, 1024, 64, 128, "markov90"),
    (40, 17, 256, 32, 384, "markov80"),    # d_e = 384, n = 17 (N = 32)
    (32, 32, 8192, 16, 128, "markov80"),   # one chunk, 64 row tiles: clusters own two each
    (32, 32, 16384, 8, 128, "all_on"),     # one chunk, 128 row tiles: clusters own four each
])
def test_forward_bf16_small(bffn, T, n, d_h, E, d_e, regime):
    w = wl.make_injected("small", T, n, d_h, E, d_e, "bf16", regime, seed=T + d_h + E)
    y, g = run_gpu(w)
    assert_close(y, oracle_y(w, g), "bf16", f"T{T} n{n} d_h{d_h} E{E} d_e{d_e} {regime}")


def test_forward_bf16_dense_matches_dense_definition(bffn):
    """All gates on: the union is every expert; compare with the dense definition."""
    w = wl.make_injected("dense", 32, 32, 256, 8, 128, "bf16", "all_on", seed=4)
    y, g = run_gpu(w)
    assert_close(y, oracle.forward_dense(w.x, g, w.W_in, w.W_out), "bf16", "all_on dense")


def test_forward_empty_union_is_zero(bffn):
    for T, n in ((32, 32), (70, 32)):
        w = wl.make_injected("off", T, n, 256, 16, 128, "bf16", "all_off", seed=1)
        y, _ = run_gpu(w)
        assert not np.any(y)


def test_forward_partly_empty_chunks(bffn):
    w = wl.make_injected("mixed", 96, 32, 256, 16, 128, "bf16", "markov80", seed=2)
    w.gates[32:64] = 0.0            # middle chunk has an empty union
    y, g = run_gpu(w)
    assert not np.any(y[32:64])
    assert_close(y, oracle_y(w, g), "bf16", "mixed")


@pytest.mark.parametrize("bias", [-0.8, None])
def test_forward_routed_single_chunk_bf16(bffn, bias):
    """The routed decode step: tensor-core router, then the single-chunk kernel
    launched as its programmatic dependent reading the gates from the workspace
    (T = n = 32, d_h 2048, E 64).  Masks as in the router tests; y against the
    oracle given the GPU's gates."""
    w = wl.make_routed("routed32", 32, 32, 2048, 64, 128, "bf16", seed=31, bias_shift=bias)
    g_chk = _check_route(bffn, w)
    y, g = run_gpu(w)
    assert np.array_equal(g, g_chk), "the forward's router and blockffn_route disagree"
    assert_close(y, oracle_y(w, g), "bf16", f"routed single chunk bias {bias}")


@pytest.mark.parametrize("T,n,d_h,E,d_e", [
    (32, 32, 256, 16, 256),     # two 128-row tiles per expert (MT = 2)
    (20, 32, 512, 16, 512),     # MT = 4, short chunk
    (32, 32, 2048, 16, 384),    # MT = 3 at the benchmark's d_h
    (8, 8, 1024, 32, 256),      # N = 16 tokens per MMA, MT = 2
])
def test_forward_single_chunk_wide_experts(bffn, T, n, d_h, E, d_e):
    """The single-chunk kernel (T <= n, d_h % 256 == 0) with d_e > 128: several
    expert-in row tiles per expert and several k-block pairs per expert-out tile."""
    w = wl.make_injected("wide", T, n, d_h, E, d_e, "bf16", "markov80", seed=T + d_e)
    y, g = run_gpu(w)
    assert_close(y, oracle_y(w, g), "bf16", f"single chunk T{T} n{n} d_h{d_h} E{E} d_e{d_e}")


@pytest.mark.parametrize("T,n,d_h,E,d_e,dt", [
    (32, 32, 2048, 64, 128, "bf16"),    # one chunk: the single-chunk kernel reads the tables
    (300, 32, 512, 64, 128, "bf16"),    # several groups: the group plan reads the token masks
    (70, 8, 256, 16, 256, "bf16"),      # short chunks, N = 128 groups, wide experts
    (40, 16, 256, 16, 64, "f32"),       # the fp32 path
])
def test_forward_with_caller_union_tables(bffn, T, n, d_h, E, d_e, dt):
    """blockffn_chunk_union's tables fed to blockffn_forward: the same bits as the
    forward that forms the union itself, and the oracle's result."""
    w = wl.make_injected("tables", T, n, d_h, E, d_e, dt, "markov80", seed=T + n)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    x, W_in, W_out = dev(w.x, tdt), dev(w.W_in, tdt), dev(w.W_out, tdt)
    g = dev(w.gates, torch.float32)
    tables = bffn.chunk_union(g, n)
    y_tab = bffn.forward(x, W_in, W_out, n, gates=g, union=tables)
    y_own = bffn.forward(x, W_in, W_out, n, gates=g)
    torch.cuda.synchronize()
    assert torch.equal(y_tab, y_own), "tables given vs formed: results differ"
    assert_close(to_np64(y_tab), oracle_y(w, w.gates.astype(np.float64)), dt, f"tables T{T} n{n}")


@pytest.mark.parametrize("T", [32, 300])
def test_forward_refuses_inconsistent_union_tables(bffn, T):
    """An index list that disagrees with its token masks is refused on the device
    (status BLOCKFFN_ERR_INVALID_ARG, detail 11) and nothing is written."""
    w = wl.make_injected("badtab", T, 32, 512 if T > 32 else 2048, 64, 128, "bf16", "markov80", seed=5)
    x, W_in, W_out = dev(w.x, torch.bfloat16), dev(w.W_in, torch.bfloat16), dev(w.W_out, torch.bfloat16)
    g = dev(w.gates, torch.float32)
    counts, idx, tmask = bffn.chunk_union(g, 32)
    idx = idx.clone()
    idx[0, 0] = (idx[0, 0] + 1) % w.E           # names the wrong expert
    ws = bffn.Workspace.for_shapes(T, w.d_h, w.E, w.d_e, 32, torch.bfloat16, False)
    y = torch.full((T, w.d_h), 5.0, dtype=torch.bfloat16, device="cuda")
    bffn.forward(x, W_in, W_out, 32, gates=g, y=y, workspace=ws, union=(counts, idx, tmask))
    assert bffn.device_status(ws) == (1, 11)
    assert torch.all(y == 5.0)


def test_workspace_bound_to_its_shapes(bffn):
    """A workspace is bound to the shapes and gating mode of its first call after a
    reset: a call with other shapes is refused on the device (status
    BLOCKFFN_ERR_WORKSPACE, detail 10) and writes nothing; after a reset the new
    shapes compute correctly."""
    ERR_WORKSPACE, SHAPE_KEY = 5, 10
    big = wl.make_routed("bind", 96, 32, 2048, 64, 128, "bf16", seed=7, bias_shift=-0.8)
    small = wl.chunk32()
    nb = max(bffn.workspace_bytes(96, 2048, 64, 128, 32, torch.bfloat16, True),
             bffn.workspace_bytes(32, 2048, 64, 128, 32, torch.bfloat16, False))
    ws = bffn.Workspace(nb)
    y, g = run_gpu(big, ws)
    assert_close(y, oracle_y(big, g), "bf16", "first binding")
    assert bffn.device_status(ws) == (0, 0)
    x = dev(small.x, torch.bfloat16)
    W_in, W_out = dev(small.W_in, torch.bfloat16), dev(small.W_out, torch.bfloat16)
    yy = torch.full((32, 2048), 3.0, dtype=torch.bfloat16, device="cuda")
    bffn.forward(x, W_in, W_out, 32, gates=dev(small.gates, torch.float32), y=yy, workspace=ws)
    assert bffn.device_status(ws) == (ERR_WORKSPACE, SHAPE_KEY)
    assert torch.all(yy == 3.0)
    ws.reset()
    y2, g2 = run_gpu(small, ws)
    assert_close(y2, oracle_y(small, g2), "bf16", "after reset")
    assert bffn.device_status(ws) == (0, 0)


def test_forward_router_bf16_small(bffn):
    w = wl.make_routed("r", 100, 32, 256, 16, 128, "bf16", seed=5, bias_shift=-0.8, ar_rho=0.95)
    y, g = run_gpu(w)
    assert_close(y, oracle_y(w, g), "bf16", "router small")


def test_forward_zero_tokens(bffn):
    W_in = torch.zeros((4, 128, 256), dtype=torch.bfloat16, device="cuda")
    W_out = torch.zeros((4, 256, 128), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((0, 4), dtype=torch.float32, device="cuda")
    y = bffn.forward(x, W_in, W_out, 32, gates=g, workspace=bffn.Workspace(256))
    assert y.shape == (0, 256)


def test_deterministic_and_workspace_reuse(bffn):
    w = wl.chunk32()
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, torch.bfloat16, False)
    y1, g = run_gpu(w, ws)
    y2, _ = run_gpu(w, ws)
    assert np.array_equal(y1, y2), "two calls differ"
    w2 = wl.chunk32(weights=(w.W_in, w.W_out), x_seed=77)
    y3, g3 = run_gpu(w2, ws)
    assert_close(y3, oracle_y(w2, g3), "bf16", "reuse")
    y4, _ = run_gpu(w, ws)
    assert np.array_equal(y1, y4)
    assert bffn.device_status(ws) == (0, 0)


def test_repeated_calls_alternating_inputs(bffn):
    """Many single-chunk launches on fresh and reused workspaces, two inputs in
    turn: every output matches the oracle and no launch records an error.  (A
    barrier-phase mistake in the expert-out copies showed up here as an
    intermittent timeout, in about one trial of three, never in one call.)"""
    w = wl.chunk32()
    w2 = wl.chunk32(weights=(w.W_in, w.W_out), x_seed=77)
    refs = {id(w): oracle_y(w, w.gates.astype(np.float64)), id(w2): oracle_y(w2, w2.gates.astype(np.float64))}
    for trial in range(12):
        ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, torch.bfloat16, False)
        for k, ww in enumerate((w, w2, w2, w, w2)):
            y, _ = run_gpu(ww, ws)
            assert_close(y, refs[id(ww)], "bf16", f"trial {trial} call {k}")
        assert bffn.device_status(ws) == (0, 0)


def test_chained_launches_read_the_previous_output(bffn):
    """Each forward's input is the previous forward's output, launched back to back
    on one stream with no host synchronisation: the single-chunk kernel may begin
    before its predecessor finishes (programmatic dependent launch) and must not
    read x, the gates or the workspace before it has.  Bit-identical to the same
    chain with a device synchronisation after every call."""
    w = wl.chunk32()
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, torch.bfloat16, False)
    x0 = dev(w.x, torch.bfloat16)
    W_in, W_out = dev(w.W_in, torch.bfloat16), dev(w.W_out, torch.bfloat16)
    g = dev(w.gates, torch.float32)

    def chain(sync):
        xs = [x0]
        for _ in range(6):
            xs.append(bffn.forward(xs[-1], W_in, W_out, w.n, gates=g, workspace=ws))
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return [t.float().cpu().numpy() for t in xs[1:]]

    ref = chain(True)
    for _ in range(3):
        got = chain(False)
        for k, (a, b) in enumerate(zip(got, ref)):
            assert np.array_equal(a, b), f"link {k} differs"
    assert np.any(ref[0]) and np.all(np.isfinite(ref[-1]))
    assert bffn.device_status(ws) == (0, 0)


# ------------------------------------------------- residual + LayerNorm --

def test_residual_layernorm_after_the_decode_step(bffn):
    """out = LayerNorm(y + x) on the decode step's own output: against the oracle
    given the GPU's y (the step alone) and given the oracle's y (the layer)."""
    w = wl.chunk32()
    y, g = run_gpu(w)
    rng = np.random.default_rng(8)
    lg = rng.uniform(0.5, 1.5, w.d_h).astype(np.float32)
    lb = (0.1 * rng.standard_normal(w.d_h)).astype(np.float32)
    x = dev(w.x, torch.bfloat16)
    out = to_np64(bffn.residual_layernorm(dev(y, torch.bfloat16), x, dev(lg, torch.float32),
                                          dev(lb, torch.float32), 1e-5))
    assert_close(out, oracle.residual_layernorm(y, w.x, lg, lb, 1e-5), "bf16", "layernorm step")
    y_ref = oracle.forward_dense(w.x, g, w.W_in, w.W_out)
    assert_close(out, oracle.residual_layernorm(y_ref, w.x, lg, lb, 1e-5), "bf16", "layer")


@pytest.mark.parametrize("T,d_h,dt", [(5, 300, "f32"), (1, 7, "f32"), (33, 2048, "bf16"), (3, 4096, "bf16"),
                                      (2, 8200, "bf16"), (3, 12, "bf16"), (2, 5000, "f32")])
def test_residual_layernorm_shapes(bffn, T, d_h, dt):
    rng = np.random.default_rng(T * 7 + d_h)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    y = wl.bf16_round(3.0 * rng.standard_normal((T, d_h))) if dt == "bf16" else rng.standard_normal((T, d_h))
    x = wl.bf16_round(rng.standard_normal((T, d_h))) if dt == "bf16" else rng.standard_normal((T, d_h))
    lg = rng.uniform(-2.0, 2.0, d_h).astype(np.float32)
    lb = rng.standard_normal(d_h).astype(np.float32)
    out = to_np64(bffn.residual_layernorm(dev(y, tdt), dev(x, tdt), dev(lg, torch.float32),
                                          dev(lb, torch.float32), 1e-5))
    assert_close(out, oracle.residual_layernorm(y, x, lg, lb, 1e-5), dt, f"layernorm {T}x{d_h}")


def test_residual_layernorm_in_place_and_edge_rows(bffn):
    """Writing over y gives the same bits; a row whose y + x is constant gives the
    shift exactly; no rows is a no-op."""
    rng = np.random.default_rng(21)
    T, d_h = 4, 2048
    y = dev(wl.bf16_round(rng.standard_normal((T, d_h))), torch.bfloat16)
    x = dev(wl.bf16_round(rng.standard_normal((T, d_h))), torch.bfloat16)
    lg = dev(rng.uniform(0.5, 2.0, d_h).astype(np.float32), torch.float32)
    lb_np = wl.bf16_round(rng.standard_normal(d_h)).astype(np.float32)
    lb = dev(lb_np, torch.float32)
    ref = bffn.residual_layernorm(y, x, lg, lb, 1e-5).clone()
    y2 = y.clone()
    bffn.residual_layernorm(y2, x, lg, lb, 1e-5, out=y2)
    torch.cuda.synchronize()
    assert torch.equal(y2, ref)
    yc = torch.full((2, d_h), 0.75, dtype=torch.bfloat16, device="cuda")
    xc = torch.full((2, d_h), -0.25, dtype=torch.bfloat16, device="cuda")
    oc = bffn.residual_layernorm(yc, xc, lg, lb, 1e-5)
    assert np.array_equal(to_np64(oc), np.broadcast_to(lb_np.astype(np.float64), (2, d_h)))
    e = torch.empty((0, d_h), dtype=torch.bfloat16, device="cuda")
    assert bffn.residual_layernorm(e, e, lg, lb, 1e-5).shape == (0, d_h)


# ----------------------------------------------- the five workloads, full size --

def test_workload_tiny_f32(bffn):
    w = wl.tiny_f32()
    y, g = run_gpu(w)
    assert_close(y, oracle.forward_dense(w.x, g, w.W_in, w.W_out), "f32", "tiny_f32")


def test_workload_chunk32_full(bffn):
    w = wl.chunk32()
    y, g = run_gpu(w)
    assert_close(y, oracle.forward_dense(w.x, g, w.W_in, w.W_out), "bf16", "chunk32")


def test_workload_batch16_all_chunks(bffn):
    w = wl.batch16()
    y, g = run_gpu(w)
    assert_close(y, oracle_y(w, g), "bf16", "batch16")
    for c in range(w.C):   # and chunk by chunk, so one bad chunk cannot hide in the norm
        tok = chunk_tokens(w, [c])
        assert_close(y[tok], oracle_y(w, g, tok), "bf16", f"batch16 chunk {c}")


def test_workload_seq4096_all_chunks(bffn):
    """Router + union + forward over 4096 tokens; every chunk against the oracle
    (which visits only each chunk's union experts), given the GPU's gates."""
    w = wl.seq4096()
    y, g = run_gpu(w)
    ref = oracle_y(w, g)
    assert_close(y, ref, "bf16", "seq4096")
    for c in range(w.C):
        tok = chunk_tokens(w, [c])
        assert_close(y[tok], ref[tok], "bf16", f"seq4096 chunk {c}")
    # every row: zero exactly where no expert is active
    assert np.array_equal(np.any(y != 0, axis=1), np.any(g != 0, axis=1))


@pytest.mark.parametrize("n", wl.SWEEP_CHUNKS)
@pytest.mark.parametrize("regime", wl.SWEEP_REGIMES)
def test_workload_sweep_chunks(bffn, n, regime):
    """d_h=4096, E=128: decode-step calls (one chunk each, as the sweep runs them)
    on chunks spread over the first 1024 tokens of the sequence."""
    T = 1024
    w = wl.sweep(n, regime, T=T)
    C = (T + n - 1) // n
    W_in, W_out = dev(w.W_in, torch.bfloat16), dev(w.W_out, torch.bfloat16)
    ws = bffn.Workspace.for_shapes(n, w.d_h, w.E, w.d_e, n, torch.bfloat16, False)
    for c in sorted({0, C // 3, (2 * C) // 3, C - 1}):
        sl = slice(c * n, (c + 1) * n)
        y = bffn.forward(dev(w.x[sl], torch.bfloat16), W_in, W_out, n,
                         gates=dev(w.gates[sl], torch.float32), workspace=ws)
        torch.cuda.synchronize()
        ref = oracle.forward_chunk_union(w.x[sl], w.gates[sl].astype(np.float64), w.W_in, w.W_out, n)
        assert_close(to_np64(y), ref, "bf16", f"sweep n{n} {regime} chunk {c}")
    assert bffn.device_status(ws) == (0, 0)
