"""Synthetic speculative-verification driver: draft chunks of n tokens through a
stack of BlockFFN layers.

Pages: "BlockFFN: Towards End-Side Acceleration-Friendly Mixture-of-Experts
with Chunk-Level Activation Sparsity", Abstract (chunk-level sparsity is what
lets speculative decoding verify several drafted tokens at the cost of one
union), and "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
Deployment", Full BlockFFN Layer with Combined Losses (a layer is the expert
sum, then the residual and LayerNorm).

A verification step takes the hidden states of n drafted tokens and runs every
layer on them: one ``forward`` per layer (the union of the chunk's experts,
gates either injected per layer or from the layer's router, optional expert
biases, and the closing LayerNorm(y + h), which the single-chunk kernel applies
in its last step), all issued on one stream with no host synchronisation (each
kernel is a programmatic dependent of the one before it).  There is no draft model and no
language-model head: how many tokens a step accepts is a synthetic input (see
``workloads.accept_lengths``), so the driver measures the verifier's cost per
drafted and per accepted token.  Only orchestration lives here; every step of
the arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

from .api import Workspace, forward


@dataclass
class Layer:
    W_in: torch.Tensor                       # [E, d_e, d_h]
    W_out: torch.Tensor                      # [E, d_h, d_e]
    ln_gamma: torch.Tensor                   # [d_h] fp32
    ln_beta: torch.Tensor                    # [d_h] fp32
    gates: Optional[torch.Tensor] = None     # [n, E] fp32 injected gates, or the router below
    W_r: Optional[torch.Tensor] = None       # [E, d_h]
    b_r: Optional[torch.Tensor] = None       # [E] fp32
    gamma: Optional[torch.Tensor] = None     # [E] fp32
    eps: float = 2.0 ** -23                  # router RMSNorm epsilon
    ln_eps: float = 1e-5                     # LayerNorm epsilon
    b_in: Optional[torch.Tensor] = None      # [E, d_e] fp32 expert fc1 biases
    b_out: Optional[torch.Tensor] = None     # [E, d_h] fp32 expert fc2 biases


class Verifier:
    """Runs n-token draft chunks through ``layers``; owns one workspace per layer
    and the activation buffers, so a step allocates nothing (it can be captured
    in a CUDA graph)."""

    def __init__(self, layers: Sequence[Layer], n: int, dtype: torch.dtype = torch.bfloat16,
                 device=None):
        if not layers:
            raise ValueError("at least one layer")
        self.layers: List[Layer] = list(layers)
        self.n = n
        E, d_e, d_h = self.layers[0].W_in.shape
        self.d_h = d_h
        device = device or self.layers[0].W_in.device
        self.ws = [Workspace.for_shapes(n, L.W_in.shape[2], L.W_in.shape[0], L.W_in.shape[1], n, dtype,
                                        L.gates is None, device, with_bias=L.b_out is not None)
                   for L in self.layers]
        self.h = [torch.empty((n, d_h), dtype=dtype, device=device) for _ in range(2)]

    def step(self, x: torch.Tensor) -> torch.Tensor:
        """Hidden states [n, d_h] of the chunk after every layer (a buffer of the
        verifier's, overwritten by the next step)."""
        h = x
        for i, L in enumerate(self.layers):
            # the layer's output goes to the buffer its input is not in
            kw = dict(y=self.h[i % 2], workspace=self.ws[i], b_in=L.b_in, b_out=L.b_out,
                      ln_weight=L.ln_gamma, ln_bias=L.ln_beta, ln_eps=L.ln_eps)
            if L.gates is not None:
                h = forward(h, L.W_in, L.W_out, self.n, gates=L.gates, **kw)
            else:
                h = forward(h, L.W_in, L.W_out, self.n, W_r=L.W_r, b_r=L.b_r, gamma=L.gamma, eps=L.eps, **kw)
        return h


def run(verifier: Verifier, drafts: Sequence[torch.Tensor], accepted: Sequence[int],
        graph: bool = True) -> dict:
    """Verify len(accepted) steps, step k on drafts[k % len(drafts)], timed on the
    device.  ``accepted[k]`` is the synthetic number of tokens step k yields.
    Returns the time per step and the drafted / accepted tokens per second."""
    steps = len(accepted)
    stream = torch.cuda.current_stream()
    for k in range(min(3, steps)):
        verifier.step(drafts[k % len(drafts)])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph:
        # one graph over one pass of the drafts, replayed
        per = len(drafts)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for d in drafts:
                    verifier.step(d)
        torch.cuda.synchronize()
        reps = max(1, steps // per)
        steps = reps * per
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    else:
        e0.record(stream)
        for k in range(steps):
            verifier.step(drafts[k % len(drafts)])
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    acc = int(sum(int(a) for a in list(accepted)[:steps]))
    return {"steps": steps, "us_per_step": ms * 1e3 / steps,
            "drafted_tokens_per_s": steps * verifier.n / (ms * 1e-3),
            "accepted_tokens_per_s": acc / (ms * 1e-3), "mean_accepted": acc / steps,
            "layers": len(verifier.layers)}
