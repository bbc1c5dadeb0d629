"""Seeded synthetic inputs for the BlockFFN chunk-union forward.

This module is shared by the oracle side (tests, CPU baseline) and the GPU side
(tests, bench).  It holds none of the layer's arithmetic: it only draws random
numbers, rounds them to bf16 where the workload is bf16, and lays out masks.

Workloads (shapes and structure stand in for the pages' end-side settings: the
pages measure trained models, which are not available, so every tensor is drawn
from the distributions below):

* ``tiny_f32``     -- one chunk, n=32, d_h=256, E=16, d_e=64, fp32, gates from the
                      router (no bias, gamma=1).
* ``chunk32``      -- one verification chunk, n=32, d_h=2048, E=64, d_e=128, bf16,
                      injected gates: per-expert two-state Markov chain along tokens
                      (off->on 0.019, on->off 0.076), active values |N(0,1)|.
* ``batch16``      -- 16 independent 32-token chunks, each with its own x and mask
                      (seed 1000+b), weights as ``chunk32``.
* ``seq4096``      -- 4096 tokens = 128 chunks, router with per-expert bias
                      -0.8*sigma_e, x an AR(1) sequence (rho=0.95), gamma=1.
* ``sweep``        -- d_h=4096, E=128, d_e=128, n in {1,8,32}, T=4096, regimes
                      all-on / Bernoulli(0.2) / Markov(0.019,0.076) / Markov(0.008,0.072).

Distributions: x ~ N(0,1); weights ~ N(0, 1/fan_in) (W_r, W_in: 1/d_h; W_out:
1/d_e); every value rounded once to bf16 (round-to-nearest-even) for bf16
workloads, so the oracle and the GPU read identical numbers.

sigma_e (router bias of ``seq4096``): the standard deviation of logit_e = W_r[e].x
over the token distribution given the weights.  x has i.i.d. unit-variance
coordinates (the AR(1) chain is started in its stationary law), so
sigma_e = ||W_r[e]||_2.  P(z > 0.8) = 0.212 then gives about 79 % token-level
sparsity.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# RMSNorm epsilon used by every workload: the fp32 machine epsilon, the value
# nn.RMSNorm(E) picks for fp32 when eps is left unset.
RMS_EPS = float(2.0 ** -23)

MARKOV80 = (0.019, 0.076)
MARKOV90 = (0.008, 0.072)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream)])


def normal(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    z = _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        z *= np.float32(std)
    return z


def markov_mask(seed: int, stream: int, T: int, E: int, a: float, b: float) -> np.ndarray:
    """Per-expert two-state chain along tokens: P(off->on)=a, P(on->off)=b.

    The first state is drawn from the stationary law P(on) = a/(a+b); one
    independent chain per expert, not reset at chunk borders.
    """
    rng = _rng(seed, stream)
    u = rng.random(size=(T, E))
    m = np.empty((T, E), dtype=bool)
    m[0] = u[0] < a / (a + b)
    for t in range(1, T):
        prev = m[t - 1]
        m[t] = np.where(prev, u[t] >= b, u[t] < a)
    return m


def bernoulli_mask(seed: int, stream: int, T: int, E: int, p_on: float) -> np.ndarray:
    return _rng(seed, stream).random(size=(T, E)) < p_on


def gate_values(seed: int, stream: int, mask: np.ndarray) -> np.ndarray:
    """|N(0,1)| on active entries, exactly 0 elsewhere (fp32)."""
    v = np.abs(normal(seed, stream, mask.shape))
    v[v == 0] = 1.0  # an active gate must be non-zero
    return np.where(mask, v, np.float32(0)).astype(np.float32)


def ar1_tokens(seed: int, stream: int, T: int, d_h: int, rho: float) -> np.ndarray:
    """x_t = rho x_{t-1} + sqrt(1-rho^2) eps_t, x_0 = eps_0 (stationary, unit variance)."""
    eps = normal(seed, stream, (T, d_h))
    x = np.empty_like(eps)
    x[0] = eps[0]
    c = np.float32(np.sqrt(1.0 - rho * rho))
    r = np.float32(rho)
    for t in range(1, T):
        x[t] = r * x[t - 1] + c * eps[t]
    return x


@dataclasses.dataclass
class Workload:
    """One layer call's inputs (numpy float32, bf16-representable for bf16)."""
    name: str
    T: int
    n: int
    d_h: int
    E: int
    d_e: int
    dtype: str                      # "f32" or "bf16"
    x: np.ndarray                   # [T, d_h]
    W_in: np.ndarray                # [E, d_e, d_h]
    W_out: np.ndarray               # [E, d_h, d_e]
    gates: Optional[np.ndarray] = None   # [T, E] injected gates, or None -> router
    W_r: Optional[np.ndarray] = None     # [E, d_h]
    b_r: Optional[np.ndarray] = None     # [E] fp32
    gamma: Optional[np.ndarray] = None   # [E] fp32
    eps: float = RMS_EPS
    meta: dict = dataclasses.field(default_factory=dict)

    @property
    def C(self) -> int:
        return (self.T + self.n - 1) // self.n

    @property
    def uses_router(self) -> bool:
        return self.gates is None


def _round(a: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_round(a) if dtype == "bf16" else np.ascontiguousarray(a, np.float32)


def expert_weights(seed: int, E: int, d_e: int, d_h: int, dtype: str):
    W_in = _round(normal(seed, 3, (E, d_e, d_h), 1.0 / np.sqrt(d_h)), dtype)
    W_out = _round(normal(seed, 4, (E, d_h, d_e), 1.0 / np.sqrt(d_e)), dtype)
    return W_in, W_out


def _uniform(seed: int, stream: int, shape, bound: float) -> np.ndarray:
    return _rng(seed, stream).uniform(-bound, bound, shape)


def expert_biases(seed: int, E: int, d_e: int, d_h: int, scale: float = 1.0):
    """fc1 biases [E, d_e] and fc2 biases [E, d_h], fp32: nn.Linear's initial
    distribution U(-1/sqrt(fan_in), 1/sqrt(fan_in)) times ``scale``."""
    b_in = _uniform(seed, 7, (E, d_e), scale / np.sqrt(d_h)).astype(np.float32)
    b_out = _uniform(seed, 8, (E, d_h), scale / np.sqrt(d_e)).astype(np.float32)
    return b_in, b_out


def layernorm_params(seed: int, d_h: int):
    """LayerNorm scale U(0.5, 1.5) and shift N(0, 0.1^2), fp32 [d_h] each."""
    w = _rng(seed, 9).uniform(0.5, 1.5, d_h).astype(np.float32)
    b = (0.1 * _rng(seed, 10).standard_normal(d_h)).astype(np.float32)
    return w, b


def router_weights(seed: int, E: int, d_h: int, dtype: str):
    return _round(normal(seed, 2, (E, d_h), 1.0 / np.sqrt(d_h)), dtype)


def make_injected(name: str, T: int, n: int, d_h: int, E: int, d_e: int, dtype: str,
                  regime: str = "markov80", seed: int = 0, weights=None,
                  x_seed: Optional[int] = None) -> Workload:
    """Injected-gate workload; ``regime`` in all_on / bern0.2 / markov80 / markov90."""
    xs = seed if x_seed is None else x_seed
    x = _round(normal(xs, 1, (T, d_h)), dtype)
    if regime == "all_on":
        mask = np.ones((T, E), bool)
    elif regime == "all_off":
        mask = np.zeros((T, E), bool)
    elif regime.startswith("bern"):
        mask = bernoulli_mask(xs, 5, T, E, float(regime[4:]))
    elif regime == "markov80":
        mask = markov_mask(xs, 5, T, E, *MARKOV80)
    elif regime == "markov90":
        mask = markov_mask(xs, 5, T, E, *MARKOV90)
    else:
        raise ValueError(f"unknown regime {regime!r}")
    gates = gate_values(xs, 6, mask)
    W_in, W_out = weights if weights is not None else expert_weights(seed, E, d_e, d_h, dtype)
    return Workload(name, T, n, d_h, E, d_e, dtype, x, W_in, W_out, gates=gates,
                    meta={"regime": regime, "seed": seed, "x_seed": xs})


def make_routed(name: str, T: int, n: int, d_h: int, E: int, d_e: int, dtype: str,
                seed: int = 0, bias_shift: Optional[float] = None, ar_rho: Optional[float] = None,
                gamma: Optional[np.ndarray] = None) -> Workload:
    """Router workload: gates come from g = RMSNorm(ReLU(W_r x + b_r))."""
    if ar_rho is None:
        x = _round(normal(seed, 1, (T, d_h)), dtype)
    else:
        x = _round(ar1_tokens(seed, 1, T, d_h, ar_rho), dtype)
    W_r = router_weights(seed, E, d_h, dtype)
    b_r = None
    if bias_shift is not None:
        sigma = np.sqrt(np.sum(W_r.astype(np.float64) ** 2, axis=1))
        b_r = (bias_shift * sigma).astype(np.float32)
    W_in, W_out = expert_weights(seed, E, d_e, d_h, dtype)
    g = np.ones(E, np.float32) if gamma is None else np.asarray(gamma, np.float32)
    return Workload(name, T, n, d_h, E, d_e, dtype, x, W_in, W_out, gates=None, W_r=W_r,
                    b_r=b_r, gamma=g, meta={"seed": seed, "bias_shift": bias_shift,
                                            "ar_rho": ar_rho})


def tiny_f32(seed: int = 0) -> Workload:
    return make_routed("tiny_f32", 32, 32, 256, 16, 64, "f32", seed=seed)


def chunk32(seed: int = 0, weights=None, x_seed: Optional[int] = None) -> Workload:
    return make_injected("chunk32", 32, 32, 2048, 64, 128, "bf16", "markov80", seed=seed,
                         weights=weights, x_seed=x_seed)


def batch16(seed: int = 0) -> Workload:
    """16 independent chunks: sequence b draws x and mask from seed 1000+b."""
    T, n, d_h, E, d_e = 32, 32, 2048, 64, 128
    weights = expert_weights(seed, E, d_e, d_h, "bf16")
    parts = [make_injected("batch16", T, n, d_h, E, d_e, "bf16", "markov80", seed=seed,
                           weights=weights, x_seed=1000 + b) for b in range(16)]
    x = np.concatenate([p.x for p in parts], axis=0)
    gates = np.concatenate([p.gates for p in parts], axis=0)
    return Workload("batch16", 16 * T, n, d_h, E, d_e, "bf16", x, weights[0], weights[1],
                    gates=gates, meta={"regime": "markov80", "seed": seed, "B": 16})


def seq4096(seed: int = 0) -> Workload:
    return make_routed("seq4096", 4096, 32, 2048, 64, 128, "bf16", seed=seed,
                       bias_shift=-0.8, ar_rho=0.95)


SWEEP_REGIMES = ("all_on", "bern0.2", "markov80", "markov90")
SWEEP_CHUNKS = (1, 8, 32)


def sweep(n: int, regime: str, seed: int = 0, T: int = 4096, weights=None) -> Workload:
    return make_injected(f"sweep_n{n}_{regime}", T, n, 4096, 128, 128, "bf16", regime,
                         seed=seed, weights=weights)


def markov_closed_forms(a: float, b: float, L: int) -> dict:
    """Closed forms of the stationary two-state chain used as a generator check.

    TLS = P(off) = b/(a+b); an expert stays off for a whole L-token window with
    probability P(off) * (1-a)^(L-1), which is CLS_L.
    """
    p_off = b / (a + b)
    return {"tls": p_off, "cls": p_off * (1.0 - a) ** (L - 1)}


def layer_stack(L: int, n: int, d_h: int, E: int, d_e: int, dtype: str, regime: str = "markov80",
                seed: int = 0) -> list:
    """L synthetic layers for the verification driver: expert weights, an injected
    gate matrix [n, E] (the regime's masks, as a router would give them for one
    draft chunk) and a LayerNorm scale and shift, each layer from its own seed."""
    layers = []
    for l in range(L):
        s = 10_000 * (seed + 1) + l
        w = make_injected(f"layer{l}", n, n, d_h, E, d_e, dtype, regime, seed=s)
        ln_gamma = (1.0 + 0.1 * normal(s, 7, (d_h,))).astype(np.float32)
        ln_beta = (0.1 * normal(s, 8, (d_h,))).astype(np.float32)
        layers.append({"W_in": w.W_in, "W_out": w.W_out, "gates": w.gates.astype(np.float32),
                       "ln_gamma": ln_gamma, "ln_beta": ln_beta})
    return layers


def accept_lengths(seed: int, steps: int, n: int, p_accept: float) -> np.ndarray:
    """Synthetic verification outcomes: each drafted token is accepted with
    probability p_accept until the first rejection; a step yields the accepted
    prefix plus the one token the verifier itself produces, so 1 .. n + 1 tokens."""
    u = _rng(seed, 9).random((steps, n))
    rejected = u >= p_accept
    first = np.where(rejected.any(axis=1), rejected.argmax(axis=1), n)
    return (first + 1).astype(np.int64)


def accept_mean(n: int, p_accept: float) -> float:
    """Closed form of accept_lengths' mean: 1 + sum_{k=1..n} p^k."""
    p = float(p_accept)
    return 1.0 + sum(p ** k for k in range(1, n + 1))
