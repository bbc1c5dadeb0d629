"""The seeded generators against closed forms and library routines.

* bf16 rounding equals torch's float32 -> bfloat16 conversion (round to nearest
  even);
* Markov masks reproduce the stationary chain's closed-form TLS and CLS
  (tests/golden/markov_closed_forms.json), which are the pages' sparsity
  figures: over 80 % TLS and about 70 % 8-token CLS;
* Bernoulli masks: union fraction of an n-token chunk is 1 - (1-p)^n;
* the long-sequence router workload lands near 79 % TLS (P(z > 0.8));
* generation is deterministic in the seed.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 65504.0,
                                  1e-30, -1e-38, 3.3895314e38], np.float32)])
    ours = wl.bf16_round(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("chain", [0, 1])
def test_markov_mask_closed_forms(chain):
    with open(os.path.join(GOLDEN, "markov_closed_forms.json")) as f:
        spec = json.load(f)["chains"][chain]
    a, b = spec["a"], spec["b"]
    T, E = 20000, 64
    m = wl.markov_mask(123, 5, T, E, a, b)
    g = m.astype(np.float64)
    tls, cls8 = oracle.sparsity(g, 8)
    _, cls32 = oracle.sparsity(g, 32)
    # standard error is well under 0.01 at this size (long chains are correlated)
    assert abs(tls - spec["tls"]) < 0.01
    assert abs(cls8 - spec["cls8"]) < 0.01
    assert abs(cls32 - spec["cls32"]) < 0.015
    assert abs((1 - cls32) - spec["union32"]) < 0.015
    cf = wl.markov_closed_forms(a, b, 8)
    assert abs(cf["tls"] - spec["tls"]) < 1e-4 and abs(cf["cls"] - spec["cls8"]) < 1e-4


def test_markov80_meets_pages_targets():
    with open(os.path.join(GOLDEN, "markov_closed_forms.json")) as f:
        tgt = json.load(f)["pages_targets"]
    cf = wl.markov_closed_forms(*wl.MARKOV80, 8)
    assert cf["tls"] >= tgt["tls_min"] - 1e-9
    assert abs(cf["cls"] - tgt["cls8_min"]) < 0.01


def test_bernoulli_union_fraction():
    T, E, p = 32 * 400, 64, 0.2
    m = wl.bernoulli_mask(1, 5, T, E, p).astype(np.float64)
    tls, cls32 = oracle.sparsity(m, 32)
    assert abs(tls - (1 - p)) < 0.005
    assert abs((1 - cls32) - (1 - (1 - p) ** 32)) < 0.005


def test_gate_values_nonzero_exactly_on_mask():
    m = wl.markov_mask(3, 5, 256, 64, *wl.MARKOV80)
    g = wl.gate_values(3, 6, m)
    assert np.array_equal(g != 0, m)
    assert np.all(g >= 0)


def test_deterministic():
    a = wl.make_injected("t", 40, 32, 128, 8, 128, "bf16", "markov80", seed=5)
    b = wl.make_injected("t", 40, 32, 128, 8, 128, "bf16", "markov80", seed=5)
    for k in ("x", "W_in", "W_out", "gates"):
        assert np.array_equal(getattr(a, k), getattr(b, k))
    c = wl.make_injected("t", 40, 32, 128, 8, 128, "bf16", "markov80", seed=6)
    assert not np.array_equal(a.x, c.x)


def test_ar1_is_stationary_and_correlated():
    x = wl.ar1_tokens(0, 1, 4096, 256, 0.95)
    assert abs(float(np.var(x)) - 1.0) < 0.1
    r = float(np.mean(x[1:] * x[:-1]) / np.mean(x * x))
    assert abs(r - 0.95) < 0.01


@pytest.mark.slow
def test_seq4096_router_sparsity():
    """Router bias -0.8*sigma_e: TLS near P(z > 0.8) = 0.788 over 4096 tokens."""
    w = wl.seq4096()
    _, g = oracle.route(w.x[:1024], w.W_r, w.gamma, w.eps, b_r=w.b_r)
    tls, cls8 = oracle.sparsity(g, 8)
    p_on = 0.5 * math.erfc(0.8 / math.sqrt(2.0))
    assert abs(tls - (1 - p_on)) < 0.03
    # neighbouring tokens share experts: CLS is far above the i.i.d. value
    assert cls8 > (1 - p_on) ** 8 + 0.2


def test_accept_lengths_match_their_closed_form():
    """The synthetic verification outcomes: 1 .. n + 1 tokens per step, mean
    1 + sum_k p^k (accepted prefix of a geometric run plus the verifier's own
    token)."""
    for n, p in [(32, 0.8), (8, 0.5), (32, 0.0)]:
        a = wl.accept_lengths(3, 100_000, n, p)
        assert a.min() >= 1 and a.max() <= n + 1
        m = wl.accept_mean(n, p)
        sd = max(float(a.std()), 1e-12)
        assert abs(a.mean() - m) <= 4.0 * sd / np.sqrt(a.size) + 1e-12, (n, p, a.mean(), m)
    assert np.all(wl.accept_lengths(0, 10, 32, 0.0) == 1)
    assert np.all(wl.accept_lengths(0, 10, 32, 1.0) == 33)


def test_expert_biases_and_layernorm_params():
    """Bias generators: nn.Linear's initial U(-1/sqrt(fan_in), 1/sqrt(fan_in)) times
    the scale, fp32, seeded; LayerNorm scale in [0.5, 1.5], small shifts."""
    E, d_e, d_h = 6, 128, 512
    b_in, b_out = wl.expert_biases(3, E, d_e, d_h)
    assert b_in.shape == (E, d_e) and b_out.shape == (E, d_h)
    assert b_in.dtype == np.float32 and b_out.dtype == np.float32
    assert np.max(np.abs(b_in)) <= 1.0 / np.sqrt(d_h) and np.max(np.abs(b_out)) <= 1.0 / np.sqrt(d_e)
    # uniform: the spread fills most of the interval
    assert np.max(b_out) > 0.9 / np.sqrt(d_e) and np.min(b_out) < -0.9 / np.sqrt(d_e)
    b_in2, b_out2 = wl.expert_biases(3, E, d_e, d_h, scale=4.0)
    assert np.allclose(b_in2, 4.0 * b_in) and np.allclose(b_out2, 4.0 * b_out)
    assert np.array_equal(wl.expert_biases(3, E, d_e, d_h)[0], b_in)
    lw, lb = wl.layernorm_params(5, d_h)
    assert lw.shape == lb.shape == (d_h,) and lw.dtype == lb.dtype == np.float32
    assert np.all((lw >= 0.5) & (lw <= 1.5)) and abs(float(np.std(lb)) - 0.1) < 0.02
