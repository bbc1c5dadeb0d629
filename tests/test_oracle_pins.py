"""Pins for the fp64 oracle: facts that hold independently of its code.

Each ``pin_*`` function takes an oracle module and returns the worst deviation
from a fact the pages or mathematics fix:

* all gates on  == one dense two-layer MLP over the concatenated experts
  (numpy matmul, a library routine);
* one active expert == that expert's MLP times its gate;
* all gates zero == zero output and an empty union;
* union-then-mask == dense definition == per-token sparse sum;
* pure-Python brute force on tiny shapes, and an exhaustive enumeration of
  every mask of a tiny chunk for the union lists;
* the router equals torch's own ``rms_norm`` of ``relu(W_r x + b)``;
* hand-derived worked examples (tests/golden/hand_examples.json);
* the residual LayerNorm equals torch's ``layer_norm`` of y + x, and its closed
  forms (constant row -> shift, unit moments, scale invariance);
* with expert biases: the concatenated-expert MLP with biases (numpy), the
  x = 0 closed form, and the pages' expert module built from torch nn.Linear.

``test_pins_catch_planted_mistakes`` compiles mutated copies of the oracle
(a dropped expert, a sign flip in Swish, a transposed weight index, the wrong
token's gate, a wrong RMS mean, a shifted token bit, a scrambled union list, a
LayerNorm without the residual, a sample variance, an fc1 bias after the
activation or from the wrong expert, a dropped or ungated fc2 bias)
and checks that at least one pin fails for each.
"""
from __future__ import annotations

import importlib.util
import json
import math
import os
import shutil
import sys

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _rand_problem(seed, T=7, d_h=24, E=5, d_e=6):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d_h))
    W_in = rng.standard_normal((E, d_e, d_h)) / math.sqrt(d_h)
    W_out = rng.standard_normal((E, d_h, d_e)) / math.sqrt(d_e)
    return x, W_in, W_out


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


# ---------------------------------------------------------------- pins ------

def pin_all_on_dense_mlp(orc) -> float:
    """Gates all non-zero: y = W_out_cat (g_rep * Swish(W_in_cat x)), a plain MLP."""
    worst = 0.0
    for seed in range(3):
        x, W_in, W_out = _rand_problem(seed)
        E, d_e, d_h = W_in.shape
        rng = np.random.default_rng(100 + seed)
        gates = np.ones((x.shape[0], E)) if seed == 0 else rng.uniform(0.1, 2.0, (x.shape[0], E))
        W_in_cat = W_in.reshape(E * d_e, d_h)                      # [E*d_e, d_h]
        W_out_cat = np.concatenate(list(W_out), axis=1)            # [d_h, E*d_e]
        hidden = _silu(x @ W_in_cat.T) * np.repeat(gates, d_e, axis=1)
        y_ref = hidden @ W_out_cat.T
        worst = max(worst, _rel(orc.forward_dense(x, gates, W_in, W_out), y_ref))
    return worst


def pin_one_active_expert(orc) -> float:
    worst = 0.0
    x, W_in, W_out = _rand_problem(7)
    T, E = x.shape[0], W_in.shape[0]
    for e in range(E):
        gates = np.zeros((T, E))
        gates[:, e] = np.linspace(0.5, 1.5, T)
        y_ref = gates[:, e:e + 1] * (_silu(x @ W_in[e].T) @ W_out[e].T)
        worst = max(worst, _rel(orc.forward_dense(x, gates, W_in, W_out), y_ref))
    return worst


def pin_all_zero(orc) -> float:
    x, W_in, W_out = _rand_problem(3)
    T, E = x.shape[0], W_in.shape[0]
    gates = np.zeros((T, E))
    y = orc.forward_dense(x, gates, W_in, W_out)
    yu = orc.forward_chunk_union(x, gates, W_in, W_out, 3)
    counts, idx, tmask = orc.chunk_union(gates, 3)
    bad = float(np.max(np.abs(y)) + np.max(np.abs(yu)))
    bad += float(np.sum(counts != 0) + np.sum(idx != -1) + np.sum(tmask != 0))
    return bad


def pin_union_then_mask(orc) -> float:
    """Union-then-mask == dense == per-token sparse (numpy), on random masks."""
    worst = 0.0
    for seed, n in [(11, 3), (12, 4), (13, 1), (14, 7)]:
        x, W_in, W_out = _rand_problem(seed, T=10)
        T, E = x.shape[0], W_in.shape[0]
        rng = np.random.default_rng(seed)
        gates = np.where(rng.random((T, E)) < 0.35, rng.uniform(-1.5, 1.5, (T, E)), 0.0)
        yd = orc.forward_dense(x, gates, W_in, W_out)
        yu = orc.forward_chunk_union(x, gates, W_in, W_out, n)
        ys = np.zeros_like(yd)
        for t in range(T):
            for e in range(E):
                if gates[t, e] != 0:
                    ys[t] += gates[t, e] * (W_out[e] @ _silu(W_in[e] @ x[t]))
        # the dense definition and the union schedule add exactly the same
        # non-zero terms in the same order, so they agree bit for bit
        exact = 0.0 if np.array_equal(yd, yu) else 1.0
        worst = max(worst, exact, _rel(yd, ys))
    return worst


def _rand_biases(seed, E, d_e, d_h, scale=0.5):
    rng = np.random.default_rng(500 + seed)
    return scale * rng.standard_normal((E, d_e)), scale * rng.standard_normal((E, d_h))


def pin_bias_all_on_mlp(orc) -> float:
    """Expert biases, gates all non-zero: the layer is one MLP over the
    concatenated experts, y = W_out_cat (g_rep * Swish(W_in_cat x + b_in_cat))
    + g B_out (numpy matmuls), in the dense definition and the union schedule."""
    worst = 0.0
    for seed in range(3):
        x, W_in, W_out = _rand_problem(seed, d_e=5)
        T, E, d_e, d_h = x.shape[0], W_in.shape[0], W_in.shape[1], W_in.shape[2]
        b_in, b_out = _rand_biases(seed, E, d_e, d_h)
        rng = np.random.default_rng(300 + seed)
        gates = rng.uniform(0.1, 2.0, (T, E))
        W_in_cat = W_in.reshape(E * d_e, d_h)
        W_out_cat = np.concatenate(list(W_out), axis=1)
        hidden = _silu(x @ W_in_cat.T + b_in.reshape(-1)) * np.repeat(gates, d_e, axis=1)
        y_ref = hidden @ W_out_cat.T + gates @ b_out
        worst = max(worst, _rel(orc.forward_dense(x, gates, W_in, W_out, b_in, b_out), y_ref))
        worst = max(worst, _rel(orc.forward_chunk_union(x, gates, W_in, W_out, 4, b_in, b_out), y_ref))
    return worst


def pin_bias_zero_input(orc) -> float:
    """x = 0: every expert outputs W_out_e Swish(b_in_e) + b_out_e, so
    y_t = sum_e g_te (W_out_e Swish(b_in_e) + b_out_e) (closed form)."""
    x, W_in, W_out = _rand_problem(21, d_e=3)
    x = np.zeros_like(x)
    T, E, d_e, d_h = x.shape[0], W_in.shape[0], W_in.shape[1], W_in.shape[2]
    b_in, b_out = _rand_biases(21, E, d_e, d_h, scale=1.0)
    rng = np.random.default_rng(22)
    gates = np.where(rng.random((T, E)) < 0.5, rng.uniform(-1.0, 2.0, (T, E)), 0.0)
    per_expert = np.stack([W_out[e] @ _silu(b_in[e]) + b_out[e] for e in range(E)])   # [E, d_h]
    y_ref = gates @ per_expert
    worst = _rel(orc.forward_dense(x, gates, W_in, W_out, b_in, b_out), y_ref)
    return max(worst, _rel(orc.forward_chunk_union(x, gates, W_in, W_out, 2, b_in, b_out), y_ref))


def pin_bias_torch_modules(orc) -> float:
    """The expert as the pages build it -- fc1 = nn.Linear(d_h, d_e), SiLU,
    fc2 = nn.Linear(d_e, d_h), biases on -- in torch fp64, gated and summed over
    the experts with sparse gates; against both oracle schedules.  Zero biases
    give the bias-free forward exactly."""
    import torch
    worst = 0.0
    for seed, n in [(31, 3), (32, 5)]:
        x, W_in, W_out = _rand_problem(seed, T=11, d_h=16, E=4, d_e=6)
        T, E, d_e, d_h = x.shape[0], W_in.shape[0], W_in.shape[1], W_in.shape[2]
        b_in, b_out = _rand_biases(seed, E, d_e, d_h)
        rng = np.random.default_rng(seed)
        gates = np.where(rng.random((T, E)) < 0.4, rng.uniform(0.2, 1.5, (T, E)), 0.0)
        xt = torch.from_numpy(x)
        y_ref = torch.zeros(T, d_h, dtype=torch.float64)
        for e in range(E):
            fc1 = torch.nn.Linear(d_h, d_e).double()
            fc2 = torch.nn.Linear(d_e, d_h).double()
            with torch.no_grad():
                fc1.weight.copy_(torch.from_numpy(W_in[e]))
                fc1.bias.copy_(torch.from_numpy(b_in[e]))
                fc2.weight.copy_(torch.from_numpy(W_out[e]))
                fc2.bias.copy_(torch.from_numpy(b_out[e]))
                y_ref += torch.from_numpy(gates[:, e:e + 1]) * fc2(torch.nn.functional.silu(fc1(xt)))
        y_ref = y_ref.numpy()
        worst = max(worst, _rel(orc.forward_dense(x, gates, W_in, W_out, b_in, b_out), y_ref))
        worst = max(worst, _rel(orc.forward_chunk_union(x, gates, W_in, W_out, n, b_in, b_out), y_ref))
        z_in, z_out = np.zeros_like(b_in), np.zeros_like(b_out)
        same = np.array_equal(orc.forward_chunk_union(x, gates, W_in, W_out, n, z_in, z_out),
                              orc.forward_chunk_union(x, gates, W_in, W_out, n))
        worst = max(worst, 0.0 if same else 1.0)
    return worst


def _py_forward(x, gates, W_in, W_out):
    T, d_h = len(x), len(x[0])
    E, d_e = len(W_in), len(W_in[0])
    y = [[0.0] * d_h for _ in range(T)]
    for t in range(T):
        for e in range(E):
            h = []
            for j in range(d_e):
                z = sum(W_in[e][j][k] * x[t][k] for k in range(d_h))
                h.append(z / (1.0 + math.exp(-z)))
            for i in range(d_h):
                y[t][i] += gates[t][e] * sum(W_out[e][i][j] * h[j] for j in range(d_e))
    return y


def _py_union(gates, n):
    T, E = len(gates), len(gates[0])
    C = (T + n - 1) // n
    counts, idx, tmask = [], [], []
    for c in range(C):
        toks = [t for t in range(c * n, min(T, c * n + n))]
        bits = [sum(1 << (t - c * n) for t in toks if gates[t][e] != 0) for e in range(E)]
        active = sorted(e for e in range(E) if any(gates[t][e] != 0 for t in toks))
        counts.append(len(active))
        idx.append(active + [-1] * (E - len(active)))
        tmask.append(bits)
    return counts, idx, tmask


def pin_bruteforce_tiny(orc) -> float:
    """d_h=4, E=3, d_e=2: pure-Python forward; every 2^(n*E) mask for the union."""
    worst = 0.0
    rng = np.random.default_rng(5)
    for n in (1, 2, 3):
        T = 5
        x, W_in, W_out = _rand_problem(20 + n, T=T, d_h=4, E=3, d_e=2)
        gates = np.where(rng.random((T, 3)) < 0.5, rng.uniform(0.2, 1.0, (T, 3)), 0.0)
        y_py = _py_forward(x.tolist(), gates.tolist(), W_in.tolist(), W_out.tolist())
        worst = max(worst, _rel(orc.forward_dense(x, gates, W_in, W_out), y_py))
        worst = max(worst, _rel(orc.forward_chunk_union(x, gates, W_in, W_out, n), y_py))
    # exhaustive masks of a single chunk: n tokens x E experts
    E = 3
    for n in (1, 2, 3):
        for bits in range(1 << (n * E)):
            g = [[(1.0 if (bits >> (t * E + e)) & 1 else 0.0) for e in range(E)]
                 for t in range(n)]
            counts, idx, tmask = orc.chunk_union(np.array(g), n)
            pc, pi, pt = _py_union(g, n)
            if (counts.tolist() != pc or idx.tolist() != pi or tmask.tolist() != pt):
                return 1.0
    # ragged tail: T not a multiple of n
    for T, n in ((5, 2), (7, 3), (33, 32), (64, 32), (65, 32)):
        g = (rng.random((T, 4)) < 0.3).astype(np.float64)
        counts, idx, tmask = orc.chunk_union(g, n)
        pc, pi, pt = _py_union(g.tolist(), n)
        if (counts.tolist() != pc or idx.tolist() != pi or tmask.tolist() != pt):
            return 1.0
    return worst


def pin_router_torch(orc) -> float:
    """Router == torch.nn.functional.rms_norm(relu(x W_r^T + b), gamma, eps) in fp64."""
    import torch
    worst = 0.0
    rng = np.random.default_rng(9)
    for E, bias in ((16, False), (64, True), (5, True)):
        T, d_h = 40, 32
        x = rng.standard_normal((T, d_h))
        W_r = rng.standard_normal((E, d_h)) / math.sqrt(d_h)
        b_r = -0.5 * np.ones(E) if bias else None
        gamma = rng.uniform(0.5, 1.5, E)
        eps = 2.0 ** -23
        logits, gates = orc.route(x, W_r, gamma, eps, b_r=b_r)
        lt = torch.from_numpy(x) @ torch.from_numpy(W_r).T
        if bias:
            lt = lt + torch.from_numpy(b_r)
        gt = torch.nn.functional.rms_norm(torch.relu(lt), (E,), torch.from_numpy(gamma), eps)
        worst = max(worst, _rel(logits, lt.numpy()), _rel(gates, gt.numpy()))
        # the gate is zero exactly where ReLU zeroed the logit
        if not np.array_equal(gates != 0, lt.numpy() > 0):
            return 1.0
    return worst


def pin_rms_identity(orc) -> float:
    """gamma=1, eps=0: every row with an active expert has mean_e g^2 == 1;
    an all-negative row gives exact zeros (no 0/0)."""
    rng = np.random.default_rng(4)
    T, d_h, E = 30, 16, 12
    x = rng.standard_normal((T, d_h))
    W_r = rng.standard_normal((E, d_h))
    x[0] = 0.0  # logits exactly 0 -> r = 0 for every expert
    _, g = orc.route(x, W_r, np.ones(E), 0.0)
    dev = 0.0
    for t in range(T):
        if np.any(g[t] != 0):
            dev = max(dev, abs(np.mean(g[t] ** 2) - 1.0))
        elif not np.all(g[t] == 0):
            return 1.0
    if not np.all(g[0] == 0):
        return 1.0
    # negative gamma keeps the sign: still active (mask is g != 0)
    gam = np.ones(E)
    gam[0] = -2.0
    _, g2 = orc.route(x, W_r, gam, 1e-6)
    act = g2[:, 0] != 0
    if not np.all(g2[act, 0] < 0):
        return 1.0
    return dev


def pin_hand_examples(orc) -> float:
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        spec = json.load(f)
    worst = 0.0
    for ex in spec["examples"]:
        x, W_r, gamma = np.array(ex["x"]), np.array(ex["W_r"]), np.array(ex["gamma"])
        W_in, W_out = np.array(ex["W_in"]), np.array(ex["W_out"])
        exp = ex["expected"]
        logits, gates = orc.route(x, W_r, gamma, ex["eps"])
        counts, idx, tmask = orc.chunk_union(gates, ex["n"])
        if (counts.tolist() != exp["counts"] or idx.tolist() != exp["idx"]
                or tmask.tolist() != exp["tmask"]):
            return 1.0
        y = orc.forward_dense(x, gates, W_in, W_out)
        yu = orc.forward_chunk_union(x, gates, W_in, W_out, ex["n"])
        for got, want in ((logits, exp["logits"]), (gates, exp["gates"]), (y, exp["y"]),
                          (yu, exp["y"])):
            worst = max(worst, float(np.max(np.abs(np.asarray(got) - np.asarray(want)))))
    return worst


def pin_sparsity(orc) -> float:
    """TLS / CLS_L against brute-force counting, including a ragged last window."""
    rng = np.random.default_rng(8)
    worst = 0.0
    for T, E, L in ((37, 5, 8), (64, 3, 8), (10, 4, 3)):
        g = (rng.random((T, E)) < 0.25).astype(np.float64)
        tls, cls = orc.sparsity(g, L)
        C = (T + L - 1) // L
        z = sum(1 for t in range(T) for e in range(E) if g[t, e] == 0)
        off = sum(1 for c in range(C) for e in range(E)
                  if all(g[t, e] == 0 for t in range(c * L, min(T, c * L + L))))
        worst = max(worst, abs(tls - z / (T * E)), abs(cls - off / (C * E)))
    return worst


def pin_residual_layernorm_torch(orc) -> float:
    """LayerNorm(y + x) equals torch's own layer_norm of the sum (fp64, a library
    routine), for a ragged width, random scale/shift and two eps values."""
    import torch
    worst = 0.0
    for seed, (T, d_h, eps) in enumerate([(5, 300, 1e-5), (3, 64, 0.25), (1, 7, 1e-5)]):
        rng = np.random.default_rng(300 + seed)
        y, x = rng.standard_normal((T, d_h)) * 3.0, rng.standard_normal((T, d_h))
        g, b = rng.uniform(-2.0, 2.0, d_h), rng.standard_normal(d_h)
        ref = torch.nn.functional.layer_norm(torch.from_numpy(y + x), (d_h,), torch.from_numpy(g),
                                             torch.from_numpy(b), eps).numpy()
        worst = max(worst, _rel(orc.residual_layernorm(y, x, g, b, eps), ref))
    return worst


def pin_residual_layernorm_closed_forms(orc) -> float:
    """Closed forms: a constant row gives exactly the shift; with unit scale and
    zero shift a row has mean 0 and mean square var / (var + eps); scaling y + x
    by a > 0 (eps = 0) leaves the output unchanged."""
    rng = np.random.default_rng(11)
    d_h = 96
    worst = 0.0
    b = rng.standard_normal(d_h)
    c = np.full((2, d_h), 0.75)
    out = orc.residual_layernorm(c, -0.25 * np.ones((2, d_h)), rng.uniform(0.5, 2, d_h), b, 1e-5)
    worst = max(worst, float(np.max(np.abs(out - b))))
    y, x = rng.standard_normal((4, d_h)), rng.standard_normal((4, d_h))
    eps = 0.1
    out = orc.residual_layernorm(y, x, np.ones(d_h), np.zeros(d_h), eps)
    v = y + x
    var = np.mean((v - v.mean(1, keepdims=True)) ** 2, axis=1)
    worst = max(worst, float(np.max(np.abs(out.mean(1)))))
    worst = max(worst, float(np.max(np.abs((out ** 2).mean(1) - var / (var + eps)))))
    o1 = orc.residual_layernorm(y, x, np.ones(d_h), np.zeros(d_h), 0.0)
    o2 = orc.residual_layernorm(3.5 * y, 3.5 * x, np.ones(d_h), np.zeros(d_h), 0.0)
    worst = max(worst, _rel(o2, o1))
    return worst


PINS = {
    "all_on_dense_mlp": (pin_all_on_dense_mlp, 1e-12),
    "one_active_expert": (pin_one_active_expert, 1e-12),
    "all_zero": (pin_all_zero, 0.0),
    "union_then_mask": (pin_union_then_mask, 1e-12),
    "bruteforce_tiny": (pin_bruteforce_tiny, 1e-12),
    "router_torch": (pin_router_torch, 1e-13),
    "rms_identity": (pin_rms_identity, 1e-13),
    "hand_examples": (pin_hand_examples, 1e-15),
    "sparsity": (pin_sparsity, 0.0),
    "residual_layernorm_torch": (pin_residual_layernorm_torch, 1e-13),
    "residual_layernorm_closed_forms": (pin_residual_layernorm_closed_forms, 1e-12),
    "bias_all_on_mlp": (pin_bias_all_on_mlp, 1e-12),
    "bias_zero_input": (pin_bias_zero_input, 1e-12),
    "bias_torch_modules": (pin_bias_torch_modules, 1e-12),
}


def _failing_pins(orc):
    failed = []
    for name, (fn, tol) in PINS.items():
        try:
            dev = fn(orc)
        except Exception:  # a crashing mutant fails the pin too
            dev = float("inf")
        if not (dev <= tol):
            failed.append(name)
    return failed


@pytest.mark.parametrize("name", list(PINS))
def test_pin(name):
    fn, tol = PINS[name]
    dev = fn(oracle)
    assert dev <= tol, f"{name}: deviation {dev} > {tol}"


# ------------------------------------------------- planted mistakes ------

MUTANTS = {
    # a dropped term: the last expert never contributes
    "drop_last_expert": ("for (int e = 0; e < E; ++e) {\n            double g = gates",
                         "for (int e = 0; e < E - 1; ++e) {\n            double g = gates"),
    # a wrong sign in Swish
    "swish_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    # a transposed operand in fc1
    "transpose_w_in": ("s += Wi[(size_t)j * d_h + k] * xt[k];",
                       "s += Wi[(size_t)k * d_e + j] * xt[k];"),
    # the union schedule reads the chunk's first token's gate for every token
    # (skipping the post-hoc mask alone is an equivalent mutant for finite
    # inputs: a zero gate already zeroes the term)
    "wrong_token_gate": ("int keep = (int)((bits >> j) & 1u);\n            double g = gates[(size_t)t * E + e];",
                         "int keep = (int)((bits >> j) & 1u);\n            double g = gates[(size_t)(c * n) * E + e];"),
    # RMS over the wrong count (sum instead of mean)
    "rms_sum": ("ms /= (double)E;", "ms /= 1.0;"),
    # union bitmask off by one token
    "union_shift": ("bits |= (1u << j);", "bits |= (1u << (j + 1 < n ? j + 1 : j));"),
    # union ignores the ragged tail guard
    "wrong_idx_order": ("if (bits != 0u) idx[(size_t)c * E + cnt++] = e;",
                        "if (bits != 0u) idx[(size_t)c * E + cnt++] = E - 1 - e;"),
    # the residual dropped from the LayerNorm's input
    "ln_no_residual": ("for (int k = 0; k < d_h; ++k) mu += yr[k] + xr[k];",
                       "for (int k = 0; k < d_h; ++k) mu += yr[k];"),
    # the sample (n - 1) variance instead of nn.LayerNorm's population variance
    "ln_sample_variance": ("var /= (double)d_h;", "var /= (double)(d_h - 1);"),
    # the fc1 bias added after the activation instead of before it
    "bias_in_after_swish": ("if (b_in) s += b_in[(size_t)e * d_e + j];\n        h[j] = silu(s);",
                            "h[j] = silu(s);\n        if (b_in) h[j] += b_in[(size_t)e * d_e + j];"),
    # every expert reads expert 0's fc1 bias
    "bias_in_wrong_expert": ("if (b_in) s += b_in[(size_t)e * d_e + j];", "if (b_in) s += b_in[j];"),
    # the fc2 bias dropped
    "bias_out_dropped": ("if (b_out) s += b_out[(size_t)e * d_h + i];", "if (b_out) s += 0.0;"),
    # the fc2 bias added once per token outside the gate (ungated), not per expert
    "bias_out_ungated": ("for (int i = 0; i < d_h; ++i) yt[i] += g * o[i];",
                         "for (int i = 0; i < d_h; ++i) yt[i] += g * o[i] + (b_out ? b_out[(size_t)e * d_h + i] * (1.0 - g) : 0.0);"),
}


def _load_mutant(tmpdir, name, old, new):
    src_dir = os.path.dirname(oracle.__file__)
    dst = os.path.join(tmpdir, f"oracle_mut_{name}")
    os.makedirs(dst, exist_ok=True)
    shutil.copy(os.path.join(src_dir, "__init__.py"), dst)
    with open(os.path.join(src_dir, "blockffn_oracle.c")) as f:
        code = f.read()
    assert old in code, f"mutation anchor for {name} not found"
    with open(os.path.join(dst, "blockffn_oracle.c"), "w") as f:
        f.write(code.replace(old, new, 1))
    spec = importlib.util.spec_from_file_location(f"oracle_mut_{name}",
                                                  os.path.join(dst, "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_planted_mistakes(name, tmp_path):
    old, new = MUTANTS[name]
    mod = _load_mutant(str(tmp_path), name, old, new)
    failed = _failing_pins(mod)
    assert failed, f"mutant {name} passed every pin"
