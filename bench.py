#!/usr/bin/env python
"""Throughput of one GPT transformer layer's training step on B200.

One step = gpt_layer_fwd + gpt_layer_bwd_checked +
adam_step_fp32_master_prechecked + loss_scale_update through the C ABI of
libgptlayer.so, on one CUDA stream (the overflow check of the dynamic loss
scaling made by the kernels that write the gradients; --scan-overflow uses
gpt_layer_bwd + adam_step_fp32_master, whose check re-reads the arena),
by default for the hidden-10240 layer of the Megatron-LM 3D-parallelism
example (hidden 10240, 80 heads of 128, ffn 40960, seq 2048, micro-batch 1,
tp 4 sharded on one GPU, bf16 compute with fp32 master weights, weights
N(0, 0.006), initial loss scale 2^16), the largest of the pages' GPT layer
shapes, on synthetic seeded inputs.  --workload picks another shape (the
GPT-2 117M / 345M layers, the 2.4B model's layer, the tiny layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is tokens/s over all ranks with the
inputs resident in HBM: per-step device time from CUDA events on the
launching stream, the L2 flushed (256 MiB write) between steps outside the
per-step events, max over ranks.  Several GPUs run independent replicas
(the step has no cross-GPU exchange), so scaling is weak.

Also reported: `e2e` (the same step with the inputs copied from pinned host
memory and the output read back inside the timed region), the roofline of
the dominant kernel (the one with the largest share of the step's device
time, from per-launch events recorded by the library in a second timed
pass: the tcgen05 GEMM at the default shape, its algorithmic FLOPs over its
launches' summed time), the same figures for every kernel family
(`roofline_by_kernel`), a per-kernel breakdown, SM clocks sampled during the
timed region, and `cpu_baseline`, the float64 CPU oracle timed on a bounded
sample of the same workload on this host's cores.

`--impl reference` times that oracle alone, as the comparison arm.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from transformer_layer_step_b200 import synth  # noqa: E402

METRIC = "GPT layer fwd+bwd+Adam tokens/sec at 1 B200"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "large-h10240"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20
# the sources each recorded DRAM traffic depends on: the family's kernels,
# the shared device helpers, and the host code that picks its launch shape
# and lays out its operands
FAMILY_SOURCES = {
    "gemm": ("transformer_layer_step_b200/csrc/gemm_tc.cuh",
             "transformer_layer_step_b200/csrc/common.cuh",
             "transformer_layer_step_b200/csrc/gptlayer.cu"),
}


# ----------------------------------------------------------------- workload
def step_flops(cfg) -> dict:
    """Algorithmic FLOPs of one step.  Causal: the attention products count
    only the lower triangle q <= p that the method computes; dense: the
    usual full-square convention."""
    b, s, h, f = cfg.batch, cfg.seq, cfg.hidden, cfg.ffn
    T = b * s
    linear = 2 * T * (4 * h * h + 2 * h * f)            # QKV, out-proj, FFN1, FFN2
    attn_causal = 2 * 2 * b * h * (s * (s + 1) // 2)     # QK^T and PV over the triangle
    attn_dense = 2 * 2 * b * h * s * s
    return {"causal": 3 * (linear + attn_causal), "dense": 3 * (linear + attn_dense),
            "linear": 3 * linear, "attn_fwd": attn_causal, "attn_bwd": 2 * attn_causal}


def kernel_bytes(cfg, n_params: int, layers: int = 1, weight_copies: bool = False) -> dict:
    """Algorithmic HBM bytes of each bandwidth kernel of the step, summed over
    its launches in one step (2-byte activations, 4-byte fp32 state; a stack
    of `layers` layers launches each per-layer kernel once per layer; the
    optimizer's n_params covers every layer).  With weight_copies the
    optimizer step also writes the transposed 16-bit weight matrices (2 B per
    matrix element) and the backward does not transpose them."""
    b, s, h, a, f = cfg.batch, cfg.seq, cfg.hidden, cfg.heads, cfg.ffn
    T = b * s
    # the residual stream H and its gradient dH are fp32 (4 B), the rest 2 B
    per_layer = {
        "F1 ln1": 4 * T * h,                                  # read x, write L1
        "F7 ln2": 6 * T * h,                                  # read H (fp32), write L2
        "B6 ln2 bwd": 14 * T * h,   # read dL2, H (fp32), dOut; write dH (16-bit and fp32)
        "B12 ln1 bwd": 10 * T * h,  # read dL1, X, dH (fp32); write dX
        "B9 rowdot": 4 * T * h,                               # read dO and O
        "B0 weights^T": 4 * (4 * h * h + 2 * h * f),          # the four weight matrices
        "B2 dOut^T": 4 * T * h, "B5 L2^T": 4 * T * h,         # transposes: read + write
        "B7 dH^T": 4 * T * h, "B11 L1^T": 4 * T * h,
        # bias gradients: db_1 a column-sum pass over dZ; db_qkv summed every
        # 32 rows by the attention kernels that write dC, then this pass reads
        # those partials and writes the sum
        "B3 db1": 2 * T * f,
        "B11 dbqkv": 4 * 3 * h * (b * ((s + 31) // 32) + 1),
    }
    out = {k: v * layers for k, v in per_layer.items()}
    adam = 30 * n_params
    if weight_copies:
        adam += 2 * (4 * h * h + 2 * h * f) * layers
    out.update({"O1 overflow": 4 * n_params, "O2 adam": adam})
    return out


def kernel_rooflines(kinds: dict, rows: list, cfg, n_params: int, flops: dict, peaks: dict,
                     peak_src: str, layers: int = 1, weight_copies: bool = False) -> dict:
    """Achieved rate against the roofline of every kernel family of the
    step, per step: the tensor-core families (the GEMM with its split-K sums,
    the attention forward and backward) as algorithmic FLOPs over their
    summed launch time against the measured bf16 GEMM rate (sustained: they
    are timed inside a long step), the bandwidth families as algorithmic
    bytes (kernel_bytes, summed over the step's launches of the family) over
    their time against the measured copy bandwidth."""
    def ms(*names):
        return sum(kinds.get(k, {}).get("ms_per_step", 0.0) for k in names)

    peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    hbm = peaks["hbm_gbs"]
    out = {}
    for fam, names, work in (("gemm", ("gemm", "splitk"), flops["linear"]),
                             ("attn_fwd", ("attn_fwd",), flops["attn_fwd"]),
                             ("attn_bwd", ("attn_bwd", "rowdot"), flops["attn_bwd"])):
        t = ms(*names)
        if t > 0:
            a = work / (t * 1e-3) / 1e12
            out[fam] = {"bound": "tensor", "ms_per_step": round(t, 5), "achieved": round(a, 1),
                        "peak": peak_tf, "unit": "TFLOP/s", "frac": round(a / peak_tf, 4),
                        "peak_source": f"{peak_src} bf16_tflops_sustained"}
    nbytes = kernel_bytes(cfg, n_params, layers, weight_copies)
    for row in rows:
        if row["step"] not in nbytes or row["kind"] in ("gemm", "splitk", "attn_fwd", "attn_bwd"):
            continue
        fam = out.setdefault(row["kind"], {"bound": "hbm", "ms_per_step": 0.0, "bytes": 0})
        fam["ms_per_step"] += row["ms_per_step"]
        fam["bytes"] += nbytes[row["step"]]
    for fam in out.values():
        if fam["bound"] == "hbm" and fam["ms_per_step"] > 0:
            a = fam["bytes"] / (fam["ms_per_step"] * 1e-3) / 1e9
            fam.update(ms_per_step=round(fam["ms_per_step"], 5), achieved=round(a, 1), peak=hbm,
                       unit="GB/s", frac=round(a / hbm, 4), peak_source=f"{peak_src} hbm_gbs")
    return out


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return json.load(fh), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def code_without_comments(text: str) -> str:
    """C/CUDA source with comments and blank lines removed, so that a
    change of wording alone keeps the recorded DRAM traffic valid."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash(family: str = "gemm") -> str:
    h = hashlib.sha256()
    for rel in FAMILY_SOURCES[family]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as fh:
            h.update(code_without_comments(fh.read()).encode())
    return h.hexdigest()[:16]


# the kernels behind each family name of kernel_rooflines
DOMINANT_KERNELS = {
    "gemm": "gemm_tc_kernel (the tcgen05 GEMM; its split-K sums included)",
    "attn_fwd": "attn_fwd_kernel", "attn_bwd": "attn_bwd_dq_kernel + attn_bwd_kv_kernel (+ row term)",
    "adam": "adam_kernel", "overflow": "overflow_kernel",
}


def recorded_traffic(workload: str, family: str):
    """DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
    step's launches of a kernel family, from the committed ncu summary
    (profiles/traffic.json), or None when it is absent or the kernels
    changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except (OSError, ValueError):
        return None
    ent = rec.get(workload, {}).get(family)
    if not ent or family not in FAMILY_SOURCES or ent.get("kernel_sources") != kernel_source_hash(family):
        return None
    return ent.get("dram_bytes_per_step")


# ------------------------------------------------------------ clock sampler
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = max((num(r[2]) for r in rows if num(r[2]) is not None), default=None)
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        loaded = [v for v, p in zip(sm, power) if p is not None and p > 250] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


# --------------------------------------------------------------- CPU oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def sample_plan(cfg, seconds: float) -> tuple[int, int | None]:
    """Size of a bounded oracle sample: (sequences, position prefix or None)
    whose fwd + bwd + Adam takes about `seconds` on a 16-core host, from a
    rough cost model of the float64 oracle measured on the GPT-2 117M and
    2.4B shapes: ~2 us per token and hidden unit of element-wise work and
    16-bit rounding, ~2e11 FLOP/s in the BLAS products, ~20 ns per parameter
    in the optimizer step over the same fraction of the arena.  At least 64
    positions of one sequence."""
    h, f, s = cfg.hidden, cfg.ffn, cfg.seq
    n_params = 12 * h * h + 13 * h
    per_token = (2e-6 * h + 3 * 2 * (4 * h * h + 2 * h * f) / 2e11
                 + n_params / cfg.tokens * 2e-8)
    tokens = int(seconds / per_token)
    if tokens >= s:
        return max(1, min(cfg.batch, tokens // s)), None
    return 1, max(64, tokens // 64 * 64)


def oracle_sample(cfg, n_seq: int, seq_prefix: int | None = None, repeats: int = 1) -> dict:
    """Times the oracle (test infrastructure, float64 numpy) on a bounded
    sample of the workload: fwd + bwd of `n_seq` of the step's sequences
    (optionally only their first `seq_prefix` positions, a causal problem of
    its own) at the method's precision, plus the Adam step and overflow check
    over the same fraction of the parameter arena.  Returns tokens/s."""
    import oracle
    s = seq_prefix or cfg.seq
    sub = dataclasses.replace(cfg, batch=n_seq, seq=s)
    inp = synth.make_inputs(sub, seed=0, variant="biased", with_r=True)
    x = synth.from_bits(inp["x"], cfg.dtype).reshape(sub.tokens, cfg.hidden)
    p = {k: synth.from_bits(v, cfg.dtype).reshape(v.shape) for k, v in inp["params"].items()}
    dout = synth.from_bits(synth.loss_grad_bits(sub, 65536.0, inp["r"]),
                           cfg.dtype).reshape(x.shape)
    n_params = sum(int(v.size) for v in inp["params"].values())
    frac = sub.tokens / cfg.tokens
    n_adam = max(1024, int(n_params * frac))
    rng = np.random.default_rng(1)
    master = rng.standard_normal(n_adam).astype(np.float32) * 0.02
    m = np.zeros(n_adam, np.float32)
    v = np.zeros(n_adam, np.float32)
    g = rng.standard_normal(n_adam).astype(np.float32)
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        _, cache = oracle.layer_fwd(x, p, sub.dims(), precision=cfg.dtype)
        oracle.layer_bwd(cache, p, sub.dims(), dout)
        del cache
        inf = oracle.found_inf(g)
        oracle.adam_step(master, m, v, g, 65536.0, 0, 6e-5, 0.9, 0.95, 1e-8, 0.0, cfg.dtype, inf)
        times.append(time.perf_counter() - t0)
    desc = (f"{n_seq} of {cfg.batch} sequences" +
            (f" (first {s} of {cfg.seq} positions)" if seq_prefix else "") +
            f" fwd+bwd at {cfg.dtype} storage precision, plus overflow check and Adam over "
            f"{n_adam} of {n_params} parameters; float64 numpy oracle")
    return {"tokens": sub.tokens, "seconds": times, "sample": desc,
            "value": sub.tokens * len(times) / sum(times)}


# ------------------------------------------------------- replica bookkeeping
def reduce_max_over_ranks(v: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its own device-timed
    value and all ranks get the maximum (the job ends when the last replica
    does).  One collective, taken by every rank in the same order."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens_per_replica_step: int, ms_per_step: float) -> float:
    """Weak scaling: every replica processes its own batch each step, so the
    job's throughput is all replicas' tokens over the slowest rank's step time."""
    return world * tokens_per_replica_step / (ms_per_step * 1e-3)


# ---------------------------------------------------------------- GPU arm
def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from transformer_layer_step_b200 import gptlayer as G
    from transformer_layer_step_b200.harness import LayerStack, LayerStep

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    inp = synth.make_inputs(cfg, seed=rank, variant="biased", with_r=True)
    stack = args.layers > 1
    if stack:
        # L layers of the shape, each starting from the same seeded weights,
        # with parameters of their own in one arena, and one Adam over all
        ls = LayerStack(cfg, [inp["params"]] * args.layers, inp["x"], device=dev,
                        recompute_gelu=args.recompute_gelu,
                        weight_copies=not args.transpose_in_backward)
    else:
        ls = LayerStep(cfg, inp, device=dev, recompute_gelu=args.recompute_gelu,
                       weight_copies=not args.transpose_in_backward)
    dy_bits = synth.loss_grad_bits(cfg, ls.hyper["init_scale"], inp["r"])
    ls.set_dy_bits(dy_bits)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    K, W = args.steps, args.warmup

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max_over_ranks(v, world, dev)

    def timed_steps(n, body):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for i in range(n):
            ev[i][0].record(stream)
            body()
            ev[i][1].record(stream)
            flush.zero_()
        return ev

    fused = not args.scan_overflow and not stack

    def step(**kw):
        ls.step(fused_check=fused, **kw)

    for _ in range(W):
        step()
        flush.zero_()
    torch.cuda.synchronize()
    if G.read_device_error(clear=True):
        raise RuntimeError("device error word set during warm-up")

    # ---- the step as a CUDA graph (captured after the warm-up, which set the
    # kernels' shared-memory opt-ins): one launch of the graph per step, so no
    # host launch latency between the step's kernels
    step_fn = step
    graph = None
    graph_launches = 0
    if not args.no_graph:
        n0 = G.launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph_launches = G.launch_count() - n0
        for _ in range(2):
            graph.replay()
            flush.zero_()
        torch.cuda.synchronize()
        step_fn = graph.replay

    # ---- value: inputs resident in HBM
    sampler = ClockSampler(local_rank)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    launches0 = G.launch_count()
    ev = timed_steps(K, step_fn)
    torch.cuda.synchronize()
    barrier()
    launches = G.launch_count() - launches0 + graph_launches * K
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms))
    ms_per_step = total_ms / K

    # ---- per-launch device times (second pass, library events between launches)
    per_step = launches // K
    G.profile_begin(per_step * K + 16)
    timed_steps(K, step)
    recs, dropped = G.profile_end(per_step * K + 16)
    if dropped:
        raise RuntimeError(f"{dropped} launches were not timed")

    # ---- e2e: every step's inputs (x, dOut) copied in from pinned host memory
    # and its output y plus the scaler state read back, inside the timed
    # region.  Double-buffered device buffers; one copy stream per direction,
    # so that step i+1's input copy, step i-1's read-back and step i's compute
    # run at the same time (host-to-device and device-to-host use separate
    # copy engines and separate PCIe directions).
    x_host = torch.empty(ls.x.shape, dtype=ls.x.dtype).pin_memory()
    dy_host = torch.empty(ls.dy.shape, dtype=ls.dy.dtype).pin_memory()
    y_host = torch.empty(ls.y.shape, dtype=ls.y.dtype).pin_memory()
    st_host = torch.empty(ls.state.shape, dtype=ls.state.dtype).pin_memory()
    x_host.copy_(ls.x.cpu())
    dy_host.copy_(ls.dy.cpu())
    xb = [torch.empty_like(ls.x) for _ in range(2)]
    dyb = [torch.empty_like(ls.dy) for _ in range(2)]
    yb = [torch.empty_like(ls.y) for _ in range(2)]
    stb = [torch.empty_like(ls.state) for _ in range(2)]   # per-step snapshot of the scaler
    h2d_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    read_back = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def copy_in(i):
        b = i % 2
        with torch.cuda.stream(h2d_stream):
            if i >= 2:
                h2d_stream.wait_event(computed[b])       # step i-2 done with these buffers
            xb[b].copy_(x_host, non_blocking=True)
            dyb[b].copy_(dy_host, non_blocking=True)
            copied[b].record(h2d_stream)

    def compute(b):
        if stack:                 # the stack writes its output into its last activation
            step(x=xb[b], dy=dyb[b])
            yb[b].copy_(ls.y, non_blocking=True)
        else:
            step(x=xb[b], dy=dyb[b], y=yb[b])
        stb[b].copy_(ls.state, non_blocking=True)

    # one CUDA graph per buffer set replays the step (--e2e-eager: kernel by kernel)
    e2e_step = [lambda b=b: compute(b) for b in range(2)]
    e2e_graphs = []
    if not args.e2e_eager:
        for b in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                compute(b)
            e2e_graphs.append(g)
            e2e_step[b] = g.replay
        for b in range(2):
            e2e_step[b]()
        torch.cuda.synchronize()

    def e2e_steps(n):
        copy_in(0)
        for i in range(n):
            b = i % 2
            stream.wait_event(copied[b])
            if i >= 2:
                stream.wait_event(read_back[b])          # y buffer b read back (step i-2)
            e2e_step[b]()
            computed[b].record(stream)
            if i + 1 < n:
                copy_in(i + 1)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(computed[b])
                y_host.copy_(yb[b], non_blocking=True)
                st_host.copy_(stb[b], non_blocking=True)
                read_back[b].record(d2h_stream)
        stream.wait_event(read_back[(n - 1) % 2])

    e2e_steps(W)                                         # untimed: warms the copy path
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    h2d_stream.wait_event(t0)
    d2h_stream.wait_event(t0)
    e2e_steps(K)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1)) / K
    if G.read_device_error(clear=True):
        raise RuntimeError("device error word set during the timed steps")
    sc = ls.scaler()
    # (a stack's arena is too large for the extensions' copies of the state)
    ext = None if stack else measure_extensions(G, ls, cfg, dev, flush, peaks=load_peaks()[0])
    h2d = x_host.numel() * x_host.element_size() + dy_host.numel() * dy_host.element_size()
    d2h = y_host.numel() * y_host.element_size() + st_host.numel() * st_host.element_size()
    return dict(ms_per_step=ms_per_step, step_ms=step_ms, launches=launches, recs=recs,
                e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, clocks=clocks, n_params=ls.n_params,
                scaler=sc, ext=ext)


def measure_extensions(G, ls, cfg, dev, flush, peaks, reps=5):
    """Per-launch device times of the optimizer extensions on this workload's
    parameter arena: the clipped optimizer step (norm + overflow pass, clip
    coefficient, Adam) with max_norm 1.0, and one gradient accumulation.
    They run on copies of the optimizer state, after the timed regions, with
    the L2 flushed before each call.  Algorithmic bytes per parameter: norm
    pass 4 (read grad), Adam 30, accumulation 12 (read acc and grad, write
    acc)."""
    import torch
    n = ls.n_params
    hp = ls.hyper
    st = ls.stream()
    master, m, v, w16, state = (ls.master.clone(), ls.m.clone(), ls.v.clone(), ls.w16.clone(),
                                ls.state.clone())
    acc = ls.grad.clone()
    ws = torch.zeros(G.CLIP_WORKSPACE_BYTES // 4, dtype=torch.float32, device=dev)
    cap = 4 * reps + 4
    G.profile_begin(cap)
    for _ in range(reps):
        flush.zero_()
        G.adam_step_clip(n, master, m, v, ls.grad, w16, cfg.dtype, hp["lr"], hp["beta1"],
                         hp["beta2"], hp["eps"], hp["weight_decay"], 1.0, ws, state, st)
        flush.zero_()
        G.grad_accumulate(n, acc, ls.grad, st)
    recs, dropped = G.profile_end(cap)
    if dropped:
        raise RuntimeError(f"{dropped} extension launches were not timed")
    ms = {}
    for kind, _tag, t in recs:
        ms.setdefault(kind, []).append(t)
    mean = {k: sum(v) / len(v) for k, v in ms.items()}
    hbm = peaks["hbm_gbs"]

    def rate(kind, bpp):
        gbs = bpp * n / (mean[kind] * 1e-3) / 1e9
        return {"ms": round(mean[kind], 5), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)}

    return {
        "params": n,
        "clip_step_ms": round(mean["overflow"] + mean["clip"] + mean["adam"], 5),
        "norm_overflow_pass": rate("overflow", 4),
        "clip_coefficient_ms": round(mean["clip"], 5),
        "adam": rate("adam", 30),
        "accumulate": rate("accumulate", 12),
        "norm_of_unscaled_grad": round(float(ws[0]), 6),
        "clip_coef": round(float(ws[1]), 6),
    }


def summarize_kernels(recs, K, cfg, n_params, peaks, flops, layers=1, weight_copies=False):
    """Per-kernel device time per step, share, and achieved rate."""
    by_tag, by_kind = {}, {}
    for kind, tag, ms in recs:
        e = by_tag.setdefault(tag, {"kind": kind, "launches": 0, "ms": 0.0})
        e["launches"] += 1
        e["ms"] += ms
        k = by_kind.setdefault(kind, {"launches": 0, "ms": 0.0})
        k["launches"] += 1
        k["ms"] += ms
    total = sum(e["ms"] for e in by_kind.values())
    nbytes = kernel_bytes(cfg, n_params, layers, weight_copies)
    rows = []
    for tag, e in by_tag.items():
        ms = e["ms"] / K
        row = {"step": tag, "kind": e["kind"], "launches_per_step": e["launches"] // K,
               "ms_per_step": round(ms, 5), "share": round(e["ms"] / total, 4)}
        if tag in nbytes and ms > 0:
            row["GB/s"] = round(nbytes[tag] / (ms * 1e-3) / 1e9, 1)
            row["frac_hbm"] = round(row["GB/s"] / peaks["hbm_gbs"], 3)
        rows.append(row)
    kinds = {k: {"launches_per_step": v["launches"] // K, "ms_per_step": round(v["ms"] / K, 5),
                 "share": round(v["ms"] / total, 4)} for k, v in by_kind.items()}
    return rows, kinds, total / K


# ------------------------------------------------------- single-kernel cases
CASES = ("gemm-ffn2", "gemm-dw1", "attention", "layernorm", "adam", "adam-wt")


def run_case(args, cfg):
    """One launch (or launch pair) of one kernel family at this workload's
    shapes, holding at most a few GB on the device, for a profiler capture of
    that kernel alone: the tcgen05 GEMM as the FFN2 product (row split, shard
    sum in the K loop, bias + fp32 residual epilogue) or as the FFN1 weight
    gradient (fp32 output, token reduction), the fused attention forward and
    backward, the LayerNorm forward and backward, or the optimizer step (the
    overflow check and Adam) over 64 M parameters.  Runs the case `warmup`
    times, then once more between CUDA events, and prints the time."""
    import torch
    from transformer_layer_step_b200 import gptlayer as G
    torch.cuda.set_device(0)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float16
    T, h, f, t = cfg.tokens, cfg.hidden, cfg.ffn, cfg.tp
    fs, hs = f // t, h // t
    st = torch.cuda.current_stream().cuda_stream
    rnd = lambda *shape, std=1.0: (torch.randn(*shape, device="cuda") * std).to(tdt)
    if args.case == "gemm-ffn2":          # Out = H + sum_i A_i W2_i^T + b2
        a, w = rnd(t, T, fs), rnd(t, h, fs, std=0.02)
        hid = torch.randn(T, h, device="cuda")
        b2, out = rnd(h), torch.empty(T, h, dtype=tdt, device="cuda")
        d = G.GemmDesc()
        d.M, d.N, d.K, d.groups, d.k_shards = T, h, fs, 1, t
        d.a = G.operand(a, fs, T, t, fs, T * fs, g_div=1 << 30, k_shard=1)
        d.b = G.operand(w, fs, h, t, fs, h * fs, g_div=1 << 30, k_shard=1)
        d.out, d.ldo, d.o_mod = out.data_ptr(), h, 1
        d.bias, d.resid, d.ld_resid, d.resid_f32 = b2.data_ptr(), hid.data_ptr(), h, 1
        work = lambda: G.gemm(d, cfg.dtype, st)
        flops = 2.0 * T * h * f
    elif args.case == "gemm-dw1":         # dW1_i = dZ_i^T L2   [t][f/t][h] fp32
        dz, l2t = rnd(t, T, fs), rnd(h, T)
        out = torch.empty(t, fs, h, dtype=torch.float32, device="cuda")
        ws = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
        d = G.GemmDesc()
        d.M, d.N, d.K, d.groups, d.k_shards = fs, h, T, t, 1
        d.a = G.operand(dz, fs, T, t, fs, T * fs, mn_major=1)
        d.b = G.operand(l2t, T, h, 1, T)
        d.out, d.out_f32, d.ldo, d.o_mod, d.o_str_div = out.data_ptr(), 1, h, 1, fs * h
        d.ws, d.ws_bytes = ws.data_ptr(), 64 << 20
        work = lambda: G.gemm(d, cfg.dtype, st)
        flops = 2.0 * T * h * f
    elif args.case == "attention":
        as_ = cfg.heads // t
        c = rnd(t, T, 3 * hs)
        o, do = torch.empty(t, T, hs, dtype=tdt, device="cuda"), rnd(t, T, hs)
        lse = torch.empty(t * cfg.batch * as_, cfg.seq, device="cuda")
        dvec, dc = torch.empty_like(lse), torch.empty_like(c)
        # the QKV bias gradient, summed by the kernels that write dC
        dpart = torch.empty(cfg.batch * ((cfg.seq + 31) // 32) * 3 * h, device="cuda")
        db = torch.empty(3 * h, device="cuda")

        def work():
            G.attention_fwd(cfg.batch, cfg.seq, h, cfg.heads, t, cfg.dtype, c, o, lse, st)
            G.attention_bwd(cfg.batch, cfg.seq, h, cfg.heads, t, cfg.dtype, c, o, do, lse, dvec,
                            dc, dpart, db, stream=st)
        flops = 3 * 2 * 2 * cfg.batch * h * (cfg.seq * (cfg.seq + 1) // 2)
    elif args.case == "layernorm":
        x, gy, res = rnd(T, h), rnd(T, h), rnd(T, h)
        g, b = rnd(h), rnd(h)
        y, dx = torch.empty_like(x), torch.empty_like(x)
        mu, rs = torch.empty(T, device="cuda"), torch.empty(T, device="cuda")
        dg, db, dsum = (torch.empty(h, device="cuda") for _ in range(3))
        scr = torch.empty(G.layernorm_bwd_scratch_bytes(T, h), dtype=torch.uint8, device="cuda")

        def work():
            G.layernorm_fwd(T, h, cfg.dtype, x, g, b, 1e-5, y, mu, rs, st)
            G.layernorm_bwd(T, h, cfg.dtype, gy, x, mu, rs, g, res, dx, dg, db, dsum, scr, st)
        flops = 0.0
    elif args.case == "adam-wt":          # the step's optimizer: Adam + the transposed weights
        # of one layer of the 2.4B recipe's shape (78.7 M parameters, 1.4 GB of arrays)
        c2 = synth.CONFIGS["gpt-2.4b"]
        sh = G.make_shape(c2.batch, c2.seq, c2.hidden, c2.heads, c2.ffn, c2.tp, cfg.dtype)
        _, n = G.param_layout(sh)
        p32, m, v, g = (torch.randn(n, device="cuda") * 0.02 for _ in range(4))
        w16 = torch.empty(n, dtype=tdt, device="cuda")
        w16t = torch.zeros_like(w16)
        state = torch.zeros(8, dtype=torch.int32, device="cuda")
        state[0] = int(np.array([65536.0], np.float32).view(np.int32)[0])
        work = lambda: G.layer_adam_step(sh, 1, p32, m, v, g, w16, w16t, 6e-5, 0.9, 0.95, 1e-8, 0.0,
                                         True, state, st)
        flops = 0.0
    else:                                 # adam: overflow check + Adam over 64 M parameters
        n = 64 << 20
        p32, m, v, g = (torch.randn(n, device="cuda") * 0.02 for _ in range(4))
        w16 = torch.empty(n, dtype=tdt, device="cuda")
        state = torch.zeros(8, dtype=torch.int32, device="cuda")
        state[0] = int(np.array([65536.0], np.float32).view(np.int32)[0])
        work = lambda: G.adam_step(n, p32, m, v, g, w16, cfg.dtype, 6e-5, 0.9, 0.95, 1e-8, 0.0,
                                   state, st)
        flops = 0.0
    for _ in range(args.warmup):
        work()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    work()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if G.read_device_error(clear=True):
        raise RuntimeError("device error word set")
    line = {"case": args.case, "workload": cfg.name, "ms": round(ms, 4)}
    if flops:
        line["TFLOP/s"] = round(flops / (ms * 1e-3) / 1e12, 1)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(synth.CONFIGS))
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step's kernels one by one instead of as a CUDA graph")
    ap.add_argument("--e2e-eager", action="store_true",
                    help="launch the end-to-end steps kernel by kernel instead of as CUDA graphs")
    ap.add_argument("--scan-overflow", action="store_true",
                    help="check the gradients for inf/NaN in a separate pass over the arena "
                         "(gpt_layer_bwd + adam_step_fp32_master) instead of in the kernels "
                         "that write them (gpt_layer_bwd_checked + adam_step_fp32_master_prechecked)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the CPU oracle timing (it runs on rank 0 at N=1 only)")
    ap.add_argument("--layers", type=int, default=1,
                    help="a stack of this many layers of the workload's shape per step "
                         "(gpt_stack_fwd / gpt_stack_bwd and one Adam over every layer)")
    ap.add_argument("--transpose-in-backward", action="store_true",
                    help="the backward transposes the weight matrices itself every step, instead "
                         "of reading the copies that the optimizer step writes "
                         "(gpt_layer_adam_step)")
    ap.add_argument("--recompute-gelu", action="store_true",
                    help="selective recompute: the FFN activation is written again in the "
                         "backward (by the FFN2 input-gradient GEMM) instead of saved")
    ap.add_argument("--case", choices=CASES,
                    help="run one kernel family once at this workload's shapes (a small "
                         "device footprint for a profiler capture) instead of the benchmark")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    cfg = synth.CONFIGS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    config = {"workload": cfg.name, "batch": cfg.batch, "seq_len": cfg.seq,
              "hidden": cfg.hidden, "heads": cfg.heads, "ffn": cfg.ffn, "tp": cfg.tp,
              "tokens_per_step": cfg.tokens, "parallelism": f"replicas{world}",
              "step_launch": "kernel by kernel" if args.no_graph else "one CUDA graph per step",
              "overflow_check": ("a separate pass over the gradient arena" if args.scan_overflow
                                 else "in the kernels that write the gradients"),
              "e2e_step_launch": "kernel by kernel" if args.e2e_eager else "one CUDA graph per step",
              "e2e_copies": "one stream per direction, overlapped with the neighbouring steps",
              "l2": "flushed between steps (256 MiB write, outside the per-step events)"}
    config["weight_transposes"] = ("in the backward" if args.transpose_in_backward else
                                   "written by the optimizer step (gpt_layer_adam_step)")
    if args.recompute_gelu:
        config["recompute_gelu"] = True
    L = args.layers
    if L < 1:
        ap.error("--layers must be at least 1")
    if L > 1:
        config.update(layers=L, workload=f"{cfg.name} x{L} layers",
                      overflow_check="a separate pass over the gradient arena")
    flops = {k: L * v for k, v in step_flops(cfg).items()}

    if args.case:
        run_case(args, cfg)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        # every step a bounded sample: the whole run about two minutes of CPU work
        n_seq, prefix = sample_plan(cfg, 120.0 / (args.steps + args.warmup))
        oracle_sample(cfg, n_seq, prefix, repeats=args.warmup)
        r = oracle_sample(cfg, n_seq, prefix, repeats=args.steps)
        cores = blas_threads()
        line = {"impl": "reference", "metric": METRIC, "value": round(r["value"], 3),
                "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * sum(r["seconds"]) / len(r["seconds"]), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": round(r["value"], 3), "unit": UNIT, "cores": cores,
                                 "kind": "oracle", "sample": "per step: " + r["sample"]},
                "e2e": {"value": round(r["value"], 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import torch
    res = run_ours(args, cfg, rank, world, local_rank)
    peaks, peak_src = load_peaks()
    wcp = not args.transpose_in_backward
    rows, kinds, prof_ms = summarize_kernels(res["recs"], args.steps, cfg, res["n_params"],
                                             peaks, flops, L, wcp)
    by_kernel = kernel_rooflines(kinds, rows, cfg, res["n_params"], flops, peaks, peak_src, L, wcp)
    dom_name = max(by_kernel, key=lambda k: by_kernel[k]["ms_per_step"])
    dom = by_kernel[dom_name]
    peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    traffic = recorded_traffic(cfg.name, dom_name) if L == 1 else None
    roofline = {"kernel": DOMINANT_KERNELS.get(dom_name, dom_name), "bound": dom["bound"],
                "achieved": dom["achieved"], "peak": dom["peak"], "unit": dom["unit"],
                "frac": dom["frac"], "peak_source": dom["peak_source"],
                "unit_of_work": "one layer step's launches of the kernel",
                "work": ("algorithmic FLOPs of the step's twelve linear-layer products (causal "
                         "attention excluded)" if dom_name == "gemm" else
                         "algorithmic work of the step's launches of the kernel"),
                "share_of_step": round(dom["ms_per_step"] / prof_ms, 4) if prof_ms else None,
                "traffic": traffic}
    ms = res["ms_per_step"]
    value = whole_job_tokens_per_s(world, cfg.tokens, ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic", "config": config,
        "tflops_causal": round(flops["causal"] / (ms * 1e-3) / 1e12, 1),
        "tflops_dense_convention": round(flops["dense"] / (ms * 1e-3) / 1e12, 1),
        "frac_of_bf16_peak": round(flops["causal"] / (ms * 1e-3) / 1e12 / peak_tf, 4),
        "roofline": roofline,
        "roofline_by_kernel": by_kernel,
        "kernels": kinds,
        "steps_detail": sorted(rows, key=lambda r: -r["ms_per_step"]),
        "profiled_ms_per_step": round(prof_ms, 4),
        "e2e": {"value": round(world * cfg.tokens / (res["e2e_ms"] * 1e-3), 1), "unit": UNIT,
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
        "scaler_after": res["scaler"],
        "optimizer_extensions": res["ext"],
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        r = oracle_sample(cfg, *sample_plan(cfg, 10.0))   # about 10 s of float64 CPU work
        # a stack runs its layers one after another: one layer's oracle time, L times
        line["cpu_baseline"] = {"value": round(r["value"] / L, 3), "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": r["sample"] + (f"; one layer timed, the stack taken as "
                                                         f"{L} such layers" if L > 1 else ""),
                                "seconds": round(sum(r["seconds"]), 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
