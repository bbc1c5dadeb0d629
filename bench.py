"""Benchmark of the BlockFFN chunk-union layer forward at one n=32 verification chunk.

Workload (one step = one layer call on one chunk): n = 32 tokens, d_h = 2048,
E = 64 experts, d_e = 128, bf16, injected gates from a per-expert Markov chain
(off->on 0.019, on->off 0.076: about 80 % token-level and 70 % 8-token
chunk-level sparsity), active gate values |N(0,1)|, x ~ N(0,1), weights
~ N(0, 1/fan_in).  Synthetic data (no trained model exists here).

Device timing: R = 8 copies of (W_in, W_out, x, gates) rotate step by step, so
the 512 MiB of weights exceed the 126 MB L2 and every step streams its union
experts from HBM.  The K timed steps run as CUDA-graph replays on one stream,
bracketed by a barrier and a device synchronize, with CUDA events; per-step
events around each launch give the kernel's own time for the roofline.

The JSON line also carries: the end-to-end number through the public API with
host buffers (x and gates copied in from pinned memory, y copied out, every
step), the same-size dense FFN on the GPU (torch bf16 matmuls), the routed
decode step (router + forward) and the step with the layer's optional expert
biases and LayerNorm for context, the HBM roofline fraction on union-expert
bytes, the fp64 CPU oracle timed on a bounded sample (rank 0, one GPU), the SM
clocks sampled during the run, and the other workloads (batch16, seq4096 and
the d_h 4096 sweep, each beside its dense FFN; ``--workloads`` /
``--no-workloads``).

``--impl reference`` times the fp64 CPU oracle alone on the same workload and
metric: the pages ship no runnable implementation of the layer, so the oracle
(the dense definition in fp64 on the host cores) is the reference arm.
Multi-GPU (torchrun): independent replicas, one per GPU, no collective on the
data path (the layer does not shard); weak scaling, max time over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "tokens/s per BlockFFN layer at n=32 chunk"
UNIT = "tokens/s"
R_COPIES = 8
L2_BYTES = 126 * 1024 * 1024

# DRAM traffic of the single-chunk forward kernel from an ncu capture of this
# benchmark's own command (dram__bytes_read.sum + dram__bytes_write.sum of two
# launches, each on one of the rotating input copies): pairs of (algorithmic
# bytes, measured bytes) per captured launch.  The reported per-launch traffic is
# their measured / algorithmic ratio times this run's mean algorithmic bytes.
# Empty (traffic reported as null) when the kernel has changed since the capture.
TRAFFIC_CAPTURE = [(30679040, 30645760 + 0), (36970496, 36937984 + 5632)]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def union_bytes(w: wl.Workload) -> int:
    """Algorithmic bytes of one call: every union expert's W_in_e and W_out_e once,
    plus x, y (bf16) and the gates (fp32)."""
    active = np.any(w.gates != 0, axis=0)
    U = int(np.sum(active))
    return U * 2 * w.d_h * w.d_e * 2 + 2 * w.T * w.d_h * 2 + w.T * w.E * 4


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    """One process per GPU (torchrun env); NCCL on GPUs, gloo on CPU-only hosts."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_baseline(budget_s: float = 12.0) -> dict:
    """The fp64 oracle (dense definition) on whole chunks of the workload, timed on
    this host's cores for about ``budget_s`` seconds."""
    import oracle
    w = wl.chunk32()
    x, g, Wi, Wo = (np.asarray(a, np.float64) for a in (w.x, w.gates, w.W_in, w.W_out))
    oracle.forward_dense(x[:1], g[:1], Wi, Wo)  # build + warm
    t0 = time.perf_counter()
    tokens = 0
    calls = 0
    while True:
        oracle.forward_dense(x, g, Wi, Wo)
        tokens += w.T
        calls += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{calls} dense fp64 oracle calls on the 32-token chunk "
                      f"({w.T * calls} tokens, {dt:.1f} s)"}


def tensor_peak():
    """Sustained dense bf16 tensor throughput (TFLOP/s) for kernels timed inside a
    long run, from the measured peaks, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1400.0, "fallback"


def roofline_of(bytes_alg: float, flops: float, us: float) -> dict:
    """The binding roofline of a call that moves bytes_alg bytes and does flops
    union flops in us microseconds: whichever of HBM time and tensor time is
    longer bounds it; frac = that bound's time / the measured time."""
    hbm, hbm_kind = peaks()
    tc, tc_kind = tensor_peak()
    t_hbm = bytes_alg / (hbm * 1e9)
    t_tc = flops / (tc * 1e12)
    sec = us * 1e-6
    if t_hbm >= t_tc:
        ach = bytes_alg / sec / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "peak_kind": hbm_kind, "tensor_frac": flops / sec / 1e12 / tc}
    ach = flops / sec / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": tc, "unit": "TFLOP/s", "frac": ach / tc,
            "peak_kind": tc_kind + " sustained", "hbm_frac": bytes_alg / sec / 1e9 / hbm}


def graph_us(calls, stream, reps=3):
    """Mean device time per call of ``calls`` (thunks), captured once in a CUDA
    graph on ``stream`` and replayed ``reps`` times after one untimed replay."""
    import torch
    with torch.cuda.stream(stream):
        for c in calls:
            c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    with torch.cuda.stream(stream):
        g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
    b.synchronize()
    us = a.elapsed_time(b) * 1e3 / (reps * len(calls))
    del g
    return us


def oracle_sample(w: wl.Workload, tokens: int, routed: bool) -> dict:
    """The fp64 oracle (router when routed, then the dense definition) on the
    workload's first ``tokens`` tokens, timed on this host's cores."""
    import oracle
    x = np.asarray(w.x[:tokens], np.float64)
    t0 = time.perf_counter()
    if routed:
        _, g = oracle.route(x, w.W_r, w.gamma, w.eps, b_r=w.b_r)
    else:
        g = w.gates[:tokens]
    oracle.forward_dense(x, g, w.W_in, w.W_out)
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {tokens} tokens, {'router + ' if routed else ''}dense fp64 definition "
                      f"({dt:.1f} s)"}


def union_stats(gates: np.ndarray, n: int):
    """Per-chunk union sizes and the number of distinct experts over all chunks."""
    T, E = gates.shape
    C = (T + n - 1) // n
    act = gates != 0
    sizes = [int(np.sum(np.any(act[c * n:(c + 1) * n], axis=0))) for c in range(C)]
    distinct = int(np.sum(np.any(act, axis=0)))
    return sizes, distinct


def measure_workloads(dev, stream, with_oracle: bool, which=("batch16", "seq4096", "sweep")) -> dict:
    """The other configurations, each timed on the device as CUDA-graph replays of
    the call a user makes, beside the same-size dense FFN (torch bf16 matmuls):

    * batch16 -- 16 independent 32-token chunks in one call (group kernel);
    * seq4096 -- 4096 tokens, router + union + forward in one call;
    * sweep   -- d_h 4096, E 128: the whole 4096-token sequence as consecutive
                 one-chunk decode calls, n in {1, 8, 32}, four gate regimes.
    Inputs larger than L2 between replays: rotating copies (batch16, seq4096) or
    weights of 256 MiB (sweep)."""
    import torch
    dt = torch.bfloat16
    d = lambda a, t=dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, t)
    out = {}

    def dense_us(x_list, W_in, W_out):
        E, d_e, d_h = W_in.shape
        Wi = W_in.reshape(E * d_e, d_h)
        Wo = W_out.permute(1, 0, 2).reshape(d_h, E * d_e).contiguous()
        return graph_us([lambda x=x: torch.nn.functional.silu(x @ Wi.t()) @ Wo.t() for x in x_list], stream)

    if "batch16" in which:
        out["batch16"] = _batch16(dev, stream, d, dense_us, with_oracle)
    if "seq4096" in which:
        out["seq4096"] = _seq4096(dev, stream, d, dense_us, with_oracle)
    if "sweep" in which:
        out["sweep"] = _sweep(dev, stream, d, dense_us, with_oracle)
    return out


def _batch16(dev, stream, d, dense_us, with_oracle):
    """16 independent 32-token chunks in one call (the group kernel); 4 rotating
    copies of the weights and x (256 MiB of weights > L2)."""
    import torch
    import chunk_sparse_moe_b200 as bffn
    dt = torch.bfloat16
    w = wl.batch16()
    R = 4
    W_in = [d(w.W_in) for _ in range(R)]
    W_out = [d(w.W_out) for _ in range(R)]
    x, g = d(w.x), d(w.gates, torch.float32)
    xs = [x.clone() for _ in range(R)]
    y = torch.empty_like(x)
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, dt, False, dev)
    us = graph_us([lambda k=k: bffn.forward(xs[k], W_in[k], W_out[k], w.n, gates=g, y=y, workspace=ws)
                   for k in range(R)], stream)
    assert bffn.device_status(ws) == (0, 0)
    sizes, distinct = union_stats(w.gates, w.n)
    gsizes, _ = union_stats(w.gates, 256)
    flops = sum(sizes) * w.n * 4 * w.d_h * w.d_e
    nbytes = distinct * 2 * w.d_h * w.d_e * 2 + 2 * w.T * w.d_h * 2 + w.T * w.E * 4
    out = {
        "what": "16 chunks x 32 tokens, d_h 2048, E 64, d_e 128, bf16, Markov80 gates per sequence",
        "us_per_call": us, "tokens_per_s": w.T / (us * 1e-6),
        "union_experts_sum": sum(sizes), "distinct_experts": distinct,
        "algorithmic_bytes": nbytes, "union_flops": flops,
        "executed_flops": sum(gsizes) * 256 * 4 * w.d_h * w.d_e,
        "roofline": roofline_of(nbytes, flops, us),
        "dense_ffn_us": dense_us(xs, W_in[0], W_out[0]),
    }
    if with_oracle:
        out["cpu_baseline"] = oracle_sample(w, 32, False)
    del W_in, W_out, xs, ws
    torch.cuda.empty_cache()
    return out


def _seq4096(dev, stream, d, dense_us, with_oracle):
    """4096 tokens, router + union + forward in one call; 2 rotating copies of
    the weights, router and x (160 MiB > L2)."""
    import torch
    import chunk_sparse_moe_b200 as bffn
    dt = torch.bfloat16
    w = wl.seq4096()
    R = 2
    W_in = [d(w.W_in) for _ in range(R)]
    W_out = [d(w.W_out) for _ in range(R)]
    W_r = [d(w.W_r) for _ in range(R)]
    xs = [d(w.x) for _ in range(R)]
    b_r, gam = d(w.b_r, torch.float32), d(w.gamma, torch.float32)
    y = torch.empty_like(xs[0])
    ws = bffn.Workspace.for_shapes(w.T, w.d_h, w.E, w.d_e, w.n, dt, True, dev)
    us = graph_us([lambda k=k: bffn.forward(xs[k], W_in[k], W_out[k], w.n, W_r=W_r[k], b_r=b_r, gamma=gam,
                                            eps=w.eps, y=y, workspace=ws) for k in range(R)], stream)
    assert bffn.device_status(ws) == (0, 0)
    gates = bffn.route(xs[0], W_r[0], gam, w.eps, b_r=b_r).cpu().numpy()
    sizes, distinct = union_stats(gates, w.n)
    gsizes, _ = union_stats(gates, 256)
    flops = sum(sizes) * w.n * 4 * w.d_h * w.d_e + 2 * w.T * w.d_h * w.E
    nbytes = (distinct * 2 * w.d_h * w.d_e * 2 + 2 * w.T * w.d_h * 2 + w.E * w.d_h * 2 + w.T * w.E * 4)
    out = {
        "what": "4096 tokens (128 chunks of 32), router with bias -0.8 sigma, AR(1) x, d_h 2048, E 64, "
                "d_e 128, bf16; route + union + forward in the call",
        "us_per_call": us, "tokens_per_s": w.T / (us * 1e-6),
        "mean_union_experts": float(np.mean(sizes)), "distinct_experts": distinct,
        "mean_group_union_experts": float(np.mean(gsizes)),
        "algorithmic_bytes": nbytes, "union_flops": flops,
        "executed_flops": sum(gsizes) * 256 * 4 * w.d_h * w.d_e,
        "roofline": roofline_of(nbytes, flops, us),
        "dense_ffn_us": dense_us(xs, W_in[0], W_out[0]),
    }
    if with_oracle:
        out["cpu_baseline"] = oracle_sample(w, 16, True)
    del W_in, W_out, W_r, xs, ws
    torch.cuda.empty_cache()
    return out


def _sweep(dev, stream, d, dense_us, with_oracle=False):
    """d_h 4096, E 128: every chunk of the 4096-token sequence as its own decode
    call, n in {1, 8, 32}, four gate regimes (256 MiB of weights > L2)."""
    import torch
    import chunk_sparse_moe_b200 as bffn
    dt = torch.bfloat16
    base = wl.sweep(32, "all_on", T=32)
    W_in, W_out = d(base.W_in), d(base.W_out)
    rows = []
    dense_cache = {}
    for n in wl.SWEEP_CHUNKS:
        ws = bffn.Workspace.for_shapes(n, base.d_h, base.E, base.d_e, n, dt, False, dev)
        for regime in wl.SWEEP_REGIMES:
            w = wl.sweep(n, regime, weights=(base.W_in, base.W_out))
            x, g = d(w.x), d(w.gates, torch.float32)
            y = torch.empty_like(x)
            C = w.T // n
            calls = [lambda c=c: bffn.forward(x[c * n:(c + 1) * n], W_in, W_out, n, gates=g[c * n:(c + 1) * n],
                                              y=y[c * n:(c + 1) * n], workspace=ws) for c in range(C)]
            us = graph_us(calls, stream, reps=2)
            assert bffn.device_status(ws) == (0, 0)
            sizes, _ = union_stats(w.gates, n)
            mean_bytes = float(np.mean(sizes)) * 2 * w.d_h * w.d_e * 2 + 2 * n * w.d_h * 2 + n * w.E * 4
            flops = float(np.mean(sizes)) * n * 4 * w.d_h * w.d_e
            if n not in dense_cache:
                xd = [x[c * n:(c + 1) * n] for c in range(min(C, 64))]
                dense_cache[n] = dense_us(xd, W_in, W_out)
            rows.append({"n": n, "regime": regime, "us_per_call": us, "tokens_per_s": n / (us * 1e-6),
                         "mean_union_experts": float(np.mean(sizes)),
                         "algorithmic_bytes_per_call": mean_bytes,
                         "roofline": roofline_of(mean_bytes, flops, us),
                         "dense_ffn_us": dense_cache[n],
                         "speedup_vs_dense": dense_cache[n] / us})
        del ws
    out = {"what": "d_h 4096, E 128, d_e 128, bf16, T 4096: every chunk of the sequence as its own decode "
                   "call (a graph of the consecutive calls), mean per call; dense = the same-size dense FFN "
                   "on n tokens (torch bf16)",
           "rows": rows}
    if with_oracle:
        # the dense fp64 definition costs the same in every regime: one 32-token chunk
        out["cpu_baseline"] = oracle_sample(wl.sweep(32, "markov80"), 32, False)
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return
    cb = cpu_baseline(budget_s=max(2.0, min(60.0, 1.0 * (args.steps + args.warmup) / 100)))
    line = {"metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * 32 / cb["value"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "chunk32: n=32, d_h=2048, E=64, d_e=128, Markov(0.019, 0.076)"
                                   " gates; fp64 dense CPU oracle"},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the batch16 / seq4096 / sweep measurements")
    ap.add_argument("--workloads", default="batch16,seq4096,sweep",
                    help="comma list of the other workloads to measure (batch16, seq4096, sweep)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import torch
    torch.cuda.set_device(local)
    import chunk_sparse_moe_b200 as bffn

    dev = torch.device("cuda", local)
    dt = torch.bfloat16
    base = wl.chunk32(seed=0)
    copies = [base] + [wl.chunk32(seed=0, weights=(base.W_in, base.W_out), x_seed=k)
                       for k in range(1, R_COPIES)]
    W_in0 = torch.from_numpy(base.W_in).to(dev, dt)
    W_out0 = torch.from_numpy(base.W_out).to(dev, dt)
    bufs = []
    for k, w in enumerate(copies):
        bufs.append({
            "x": torch.from_numpy(w.x).to(dev, dt),
            "g": torch.from_numpy(w.gates).to(dev, torch.float32),
            "W_in": W_in0 if k == 0 else W_in0.clone(),
            "W_out": W_out0 if k == 0 else W_out0.clone(),
            "y": torch.empty((w.T, w.d_h), dtype=dt, device=dev),
        })
    T, n, d_h, E, d_e = base.T, base.n, base.d_h, base.E, base.d_e
    ws = bffn.Workspace.for_shapes(T, d_h, E, d_e, n, dt, False, dev)
    alg_bytes = [union_bytes(w) for w in copies]
    resident = sum(b["W_in"].numel() * 2 + b["W_out"].numel() * 2 for b in bufs)
    assert resident > 2 * L2_BYTES

    stream = torch.cuda.Stream(device=dev)

    def step(k):
        b = bufs[k % R_COPIES]
        bffn.forward(b["x"], b["W_in"], b["W_out"], n, gates=b["g"], y=b["y"], workspace=ws)

    # correctness gate before timing: one call of every copy, finite output
    with torch.cuda.stream(stream):
        for k in range(R_COPIES):
            step(k)
    stream.synchronize()
    st = bffn.device_status(ws)
    if st[0] != 0:
        raise SystemExit(f"device status {st} after warm-up")

    # CUDA graphs of R steps (one per copy) and of the remainder
    def capture(count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for k in range(count):
                step(k)
        return g

    use_graph = not args.no_graph
    graph_err = None
    if use_graph:
        try:
            g_full = capture(R_COPIES)
            rem = args.steps % R_COPIES
            g_rem = capture(rem) if rem else None
        except Exception as e:  # report and time eagerly
            use_graph, graph_err = False, repr(e)
            torch.cuda.synchronize()

    def run_steps(count):
        if use_graph:
            for _ in range(count // R_COPIES):
                g_full.replay()
            if count % R_COPIES:
                if count % R_COPIES == args.steps % R_COPIES and g_rem is not None:
                    g_rem.replay()
                else:
                    for k in range(count % R_COPIES):
                        step(k)
        else:
            for k in range(count):
                step(k)

    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    stream.synchronize()

    # The timed region (K steps between a barrier + synchronize on both sides) is
    # repeated, and the median repeat reported, so that a short K gives the same
    # steady number as a long one; every repeat times exactly K steps.
    repeats = max(3, min(50, 20000 // max(1, args.steps)))
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    region_ms = []
    for _ in range(repeats):
        barrier(world)
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            run_steps(args.steps)
            ev1.record(stream)
        ev1.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        region_ms.append(max_over_ranks(ev0.elapsed_time(ev1), world))
    clock_info = clocks.stop()
    elapsed_ms = statistics.median(region_ms)
    st = bffn.device_status(ws)
    if st[0] != 0:
        raise SystemExit(f"device status {st} after the timed run")

    # kernel-only time for the roofline: per-step events around single launches
    # (a GPU-side sleep first, so every launch is queued before the GPU reaches it
    # and the events see device time, not host launch gaps)
    with torch.cuda.stream(stream):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(4 * R_COPIES)]
        torch.cuda._sleep(100_000_000)
        for k, (a, b) in enumerate(evs):
            a.record(stream)
            step(k)
            b.record(stream)
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in evs]
    kernel_ms = statistics.median(per)
    mean_bytes = sum(alg_bytes) / len(alg_bytes)
    hbm_peak, peak_kind = peaks()
    # every step of the timed region is one launch of the single-chunk kernel, so
    # the region's mean step time is that kernel's mean launch duration there
    # (consecutive launches overlap one's set-up with the previous one's tail);
    # a launch timed alone behind a GPU sleep also pays its own launch and set-up
    step_ms = elapsed_ms / args.steps
    achieved_gbs = mean_bytes / (step_ms * 1e-3) / 1e9
    isolated_gbs = mean_bytes / (kernel_ms * 1e-3) / 1e9

    # end to end through the public API with host buffers
    x_h = [torch.from_numpy(w.x).to(dt).pin_memory() for w in copies]
    g_h = [torch.from_numpy(w.gates).pin_memory() for w in copies]
    y_h = [torch.empty((T, d_h), dtype=dt).pin_memory() for _ in copies]
    e2e_steps = min(args.e2e_steps, args.steps)

    # One CUDA graph of R_COPIES steps, replayed: step i copies its inputs in on
    # s_in, runs the forward on the compute stream and reads y back on s_out, so
    # a step's copies overlap its neighbours' kernels (each rotating buffer is
    # used once per replay; replays are ordered on the compute stream).  Every
    # step's host->device copies and read-back are inside the timed region.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(R_COPIES)]
    ev_done = [torch.cuda.Event() for _ in range(R_COPIES)]
    ev_out = [torch.cuda.Event() for _ in range(R_COPIES)]

    def e2e_steps_body():
        fork = torch.cuda.Event()
        fork.record(stream)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        for i in range(R_COPIES):
            b = bufs[i]
            with torch.cuda.stream(s_in):
                b["x"].copy_(x_h[i], non_blocking=True)
                b["g"].copy_(g_h[i], non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            with torch.cuda.stream(stream):
                bffn.forward(b["x"], b["W_in"], b["W_out"], n, gates=b["g"], y=b["y"], workspace=ws)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                y_h[i].copy_(b["y"], non_blocking=True)
                ev_out[i].record(s_out)
        for i in range(R_COPIES):
            stream.wait_event(ev_out[i])

    e2e_steps = max(R_COPIES, (e2e_steps // R_COPIES) * R_COPIES)
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=stream):
        e2e_steps_body()
    torch.cuda.synchronize()
    for _ in range(max(1, args.warmup // (10 * R_COPIES))):
        e2e_graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(e2e_steps // R_COPIES):
            e2e_graph.replay()
    e1.record(stream)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = T * d_h * 2 + T * E * 4
    d2h = T * d_h * 2

    # same-size dense FFN on the GPU (torch bf16 matmuls), context only
    W_in_cat = [b["W_in"].reshape(E * d_e, d_h) for b in bufs]
    W_out_cat = [b["W_out"].permute(1, 0, 2).reshape(d_h, E * d_e) for b in bufs]
    W_out_cat = [w.contiguous() for w in W_out_cat]

    def dense(k):
        b = bufs[k % R_COPIES]
        h = torch.nn.functional.silu(b["x"] @ W_in_cat[k % R_COPIES].t())
        return h @ W_out_cat[k % R_COPIES].t()

    with torch.cuda.stream(stream):
        for k in range(2 * R_COPIES):
            dense(k)
        dd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(4 * R_COPIES)]
        torch.cuda._sleep(100_000_000)
        for k, (a, b) in enumerate(dd):
            a.record(stream)
            dense(k)
            b.record(stream)
    torch.cuda.synchronize()
    dense_ms = statistics.median([a.elapsed_time(b) for a, b in dd])

    # the routed decode step, context only: a seeded N(0, 1/d_h) router
    # (gamma = 1, eps = 2^-23) on the same rotating inputs; the router alone and
    # router + forward, each as replays of one CUDA graph over the R_COPIES copies
    W_r = [torch.from_numpy(wl.router_weights(100 + i, E, d_h, "bf16")).to(device=dev, dtype=dt)
           for i in range(R_COPIES)]
    gam = torch.ones(E, dtype=torch.float32, device=dev)
    g_out = torch.empty((T, E), dtype=torch.float32, device=dev)
    ws_r = bffn.Workspace.for_shapes(T, d_h, E, d_e, n, dt, True, dev)

    def graph_us(fn, reps=8):
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(R_COPIES):
                fn(i)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(gr, stream=side):
                for i in range(R_COPIES):
                    fn(i)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            gr.replay()
            a.record(stream)
            for _ in range(reps):
                gr.replay()
            b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) * 1e3 / (reps * R_COPIES)

    router_us = graph_us(lambda i: bffn.route(bufs[i]["x"], W_r[i], gam, 2.0 ** -23, out=g_out))
    routed_us = graph_us(lambda i: bffn.forward(bufs[i]["x"], bufs[i]["W_in"], bufs[i]["W_out"], n, W_r=W_r[i],
                                                gamma=gam, eps=2.0 ** -23, y=bufs[i]["y"], workspace=ws_r))

    # the layer's optional parts, context only: the same decode step with the
    # experts' fc1/fc2 biases and with LayerNorm(y + x)
    bi_np, bo_np = wl.expert_biases(7, E, d_e, d_h)
    lw_np, lb_np = wl.layernorm_params(7, d_h)
    f32d = lambda a: torch.from_numpy(a).to(device=dev, dtype=torch.float32)
    b_in_t, b_out_t, lw_t, lb_t = f32d(bi_np), f32d(bo_np), f32d(lw_np), f32d(lb_np)
    ws_o = bffn.Workspace.for_shapes(T, d_h, E, d_e, n, dt, False, dev, with_bias=True)

    def opt_step(i, biases=False, ln=False):
        b = bufs[i]
        bffn.forward(b["x"], b["W_in"], b["W_out"], n, gates=b["g"], y=b["y"], workspace=ws_o,
                     b_in=b_in_t if biases else None, b_out=b_out_t if biases else None,
                     ln_weight=lw_t if ln else None, ln_bias=lb_t if ln else None)

    def plain_then_ln(i):
        b = bufs[i]
        bffn.forward(b["x"], b["W_in"], b["W_out"], n, gates=b["g"], y=b["y"], workspace=ws)
        bffn.residual_layernorm(b["y"], b["x"], lw_t, lb_t, 1e-5, out=b["y"])

    layer_opts = {
        "plain_step_us": graph_us(lambda i: opt_step(i)),
        "biases_step_us": graph_us(lambda i: opt_step(i, biases=True)),
        "layernorm_step_us": graph_us(lambda i: opt_step(i, ln=True)),
        "biases_and_layernorm_step_us": graph_us(lambda i: opt_step(i, biases=True, ln=True)),
        "step_then_layernorm_call_us": graph_us(plain_then_ln),
        "what": "chunk32 decode step through blockffn_forward with fc1/fc2 biases (nn.Linear init) and/or "
                "LayerNorm(y + x) (the LayerNorm kernel follows the forward as its programmatic "
                "dependent); beside it the plain step and a separate blockffn_residual_layernorm call; "
                "CUDA-graph replays over the rotating copies",
    }
    st_o = bffn.device_status(ws_o)
    if st_o[0] != 0:
        raise SystemExit(f"device status {st_o} after the layer-option steps")

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline()
    other = None
    if not args.no_workloads:
        other = measure_workloads(dev, stream, with_oracle=rank == 0 and world == 1 and not args.no_cpu_baseline,
                                  which=set(args.workloads.split(",")))

    if rank == 0:
        value = world * T * args.steps / (elapsed_ms * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "timed_repeats": {"count": repeats, "ms_per_step_each": [r / args.steps for r in region_ms],
                              "reported": "median"},
            "data": "synthetic (seeded; random-init weights, Markov gate masks)",
            "config": {
                "workload": "chunk32: one n=32 verification chunk, d_h=2048, E=64, d_e=128, "
                            "bf16, injected gates Markov(0.019, 0.076), |N(0,1)| values",
                "parallelism": f"replicas x{world} (no collective)",
                "l2": f"{R_COPIES} rotating copies of weights/x/gates "
                      f"({resident / 2**20:.0f} MiB > 126 MB L2)",
                "launch": "CUDA graph replays" if use_graph else "eager",
                "mean_union_experts": float(np.mean([np.sum(np.any(w.gates != 0, axis=0))
                                                     for w in copies])),
            },
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak,
                         "unit": "GB/s", "frac": achieved_gbs / hbm_peak,
                         "traffic": (mean_bytes * sum(t for _, t in TRAFFIC_CAPTURE)
                                     / sum(b for b, _ in TRAFFIC_CAPTURE)) if TRAFFIC_CAPTURE else None,
                         "peak_kind": peak_kind,
                         "kernel": "union_expert_decode",
                         "launch_us": step_ms * 1e3,
                         "launch_us_how": "mean launch duration over the timed region (one launch per "
                                          "step, CUDA-graph replays)",
                         "algorithmic_bytes_per_launch": mean_bytes,
                         "isolated_launch_us": kernel_ms * 1e3,
                         "isolated_frac": isolated_gbs / hbm_peak,
                         "isolated_how": "one launch between CUDA events, queued behind a GPU sleep: "
                                         "pays its own launch and set-up, which graph replays overlap "
                                         "with the previous launch",
                         "frac_of_8tbs": achieved_gbs / 8000.0},
            "e2e": {"value": world * T * e2e_steps / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "how": "blockffn_forward with pinned host x/gates copied in and y read back every "
                           "step; a CUDA graph of 8 steps (copies on two side streams, overlapping the "
                           "neighbouring steps' kernels), replayed"},
            "gpu_launches": args.steps,
            "layer_options": layer_opts,
            "routed_decode": {"router_us": router_us, "step_us": routed_us,
                              "what": "router (tensor cores) + single-chunk forward, gates from a seeded "
                                      "router instead of injected; graph replay"},
            "dense_ffn": {"us": dense_ms * 1e3, "tokens_per_s": T / (dense_ms * 1e-3),
                          "what": "torch bf16: silu(x W_in_cat^T) W_out_cat^T, d_ff = E*d_e"},
            "clocks": clock_info,
        }
        if other is not None:
            line["workloads"] = other
        if graph_err:
            line["graph_error"] = graph_err
        if cb is not None:
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
