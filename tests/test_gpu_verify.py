"""GPU: the synthetic speculative-verification driver (a stack of layers over
one draft chunk: each layer one forward with expert biases and the closing
residual + LayerNorm, chained on one stream).

The oracle chain mirrors the dataflow: every layer consumes the previous
layer's output as stored (bf16); within a layer the expert sum stays unrounded
into the LayerNorm, whose output is rounded to bf16, each step in fp64
(oracle.forward_chunk_union with the biases, oracle.residual_layernorm).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_common import assert_close, dev, require_cuda, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bffn():
    return require_cuda()


def _stack(bffn, L, n, d_h, E, d_e, seed=0):
    from chunk_sparse_moe_b200.verify import Layer
    raw = wl.layer_stack(L, n, d_h, E, d_e, "bf16", seed=seed)
    for i, r in enumerate(raw):
        r["b_in"], r["b_out"] = wl.expert_biases(seed * 100 + i, E, d_e, d_h)
    layers = [Layer(W_in=dev(r["W_in"], torch.bfloat16), W_out=dev(r["W_out"], torch.bfloat16),
                    ln_gamma=dev(r["ln_gamma"], torch.float32), ln_beta=dev(r["ln_beta"], torch.float32),
                    gates=dev(r["gates"], torch.float32), b_in=dev(r["b_in"], torch.float32),
                    b_out=dev(r["b_out"], torch.float32)) for r in raw]
    return raw, layers


def test_layer_stack_matches_the_oracle_chain(bffn):
    from chunk_sparse_moe_b200.verify import Verifier
    n, d_h, E, d_e = 32, 256, 16, 128
    raw, layers = _stack(bffn, 3, n, d_h, E, d_e)
    x = wl.bf16_round(np.random.default_rng(4).standard_normal((n, d_h)))
    v = Verifier(layers, n)
    h = to_np64(v.step(dev(x, torch.bfloat16)))
    ref = x.astype(np.float64)
    for r in raw:
        y = oracle.forward_chunk_union(ref, r["gates"], r["W_in"], r["W_out"], n, r["b_in"], r["b_out"])
        ref = wl.bf16_round(oracle.residual_layernorm(y, ref, r["ln_gamma"], r["ln_beta"], 1e-5))
    assert_close(h, ref.astype(np.float64), "bf16", "3-layer chain")


def test_chained_steps_equal_synchronised_layers(bffn):
    """The whole stack issued back to back (each kernel a programmatic dependent
    of the previous one) gives the same bits as one layer at a time with a
    device synchronisation in between; two steps on the same draft agree."""
    from chunk_sparse_moe_b200.verify import Verifier
    n, d_h, E, d_e = 32, 2048, 64, 128
    raw, layers = _stack(bffn, 4, n, d_h, E, d_e, seed=1)
    x = dev(wl.bf16_round(np.random.default_rng(5).standard_normal((n, d_h))), torch.bfloat16)
    v = Verifier(layers, n)
    a = v.step(x).clone()
    b = v.step(x).clone()
    torch.cuda.synchronize()
    h = x
    for i, L in enumerate(layers):
        h = bffn.forward(h, L.W_in, L.W_out, n, gates=L.gates, workspace=v.ws[i], b_in=L.b_in, b_out=L.b_out,
                         ln_weight=L.ln_gamma, ln_bias=L.ln_beta, ln_eps=1e-5)
        torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(a, h)
    for ws in v.ws:
        assert bffn.device_status(ws) == (0, 0)


def test_run_reports_tokens(bffn):
    from chunk_sparse_moe_b200.verify import Verifier, run
    n, d_h, E, d_e = 32, 256, 16, 128
    _, layers = _stack(bffn, 2, n, d_h, E, d_e, seed=2)
    drafts = [dev(wl.bf16_round(np.random.default_rng(10 + k).standard_normal((n, d_h))), torch.bfloat16)
              for k in range(4)]
    acc = wl.accept_lengths(0, 16, n, 0.8)
    r = run(Verifier(layers, n), drafts, acc)
    assert r["steps"] == 16 and r["layers"] == 2
    assert r["mean_accepted"] == pytest.approx(float(acc.mean()))
    assert r["us_per_step"] > 0 and r["accepted_tokens_per_s"] <= r["drafted_tokens_per_s"] * 33 / 32
