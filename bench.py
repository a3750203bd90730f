"""Benchmark of the fused top-k MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole layer (route -> align -> gather -> GEMM1
(+SiLU*up) -> GEMM2 (+routed weight) -> combine) over one batch of seeded
synthetic input resident in HBM, replayed from a CUDA graph of one
moe_fused_forward call (the way a serving loop runs it).  Per-kernel times
come from a second graph of the same stages with event nodes between them.

The default run's headline is the largest single-GPU configuration: the
skewed-routing FP8 layer (H=7168, E=256, top-8, I=2048, 128x128 block
scales, Zipf(1.2) expert choice), headline batch T=8192, every sweep point
(T = 1, 32, 512, 8192) reported.  Two sub-records ride along, each with its
own roofline and CPU baseline: the compute-bound FP8 prefill layer
(H=4096, E=128, top-8, I=1536, T=16384) and the bf16 decode layer of the
same shape (T = 1 ... 64).  ``--workload NAME`` times one workload alone.

L2 is flushed before every timed step, outside the CUDA-event brackets: a
256 MiB write, then a read of the same buffer, so that the flush's own dirty
lines are written back before the step instead of inside it.  Multi-GPU runs
are independent replicas by default (each rank runs the same workload; the
time is the max over ranks).  With
``--ep N`` the layer is expert-parallel instead: each of N ranks holds E/N
experts, runs its share of the replicated batch and the output is all-reduced
over NCCL; on one GPU ``--ep N`` times one rank's share alone.

The ``--impl reference`` arm times the CPU oracle (the plain C++
double-precision restatement of the layer, OpenMP over rows) on the host
cores, on bounded token samples of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from moe_layer_top_b200 import inputs  # noqa: E402

L2_FLUSH_BYTES = 256 << 20


def flush_l2(buf: torch.Tensor) -> None:
    """Evict the layer's data from L2: write a buffer twice L2's size, then read
    it back (the read pass writes the written lines back to HBM, so the step
    starts with clean lines of an unrelated buffer rather than paying for the
    flush's write-backs)."""
    buf.zero_()
    buf.sum()


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=sorted(inputs.CONFIGS),
                    help="one workload only (default: the largest single-GPU configuration, skewed_fp8, with the "
                         "prefill_fp8 and decode_bf16 layers as sub-records)")
    ap.add_argument("--no-sub-records", action="store_true", help="default workload without the sub-records")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run only this batch size (default: the workload's sweep, headline = its largest)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the expert count (small profiling cases of the same kernels)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ep", type=int, default=0,
                    help="expert parallelism over N ranks: each rank holds E/N experts, x is replicated and an "
                         "all-reduce of the output completes the layer; on one GPU, time one rank's share")
    ap.add_argument("--ep-rank", type=int, default=0, help="with --ep on one GPU: which rank's share to time")
    ap.add_argument("--persistent-decode", action="store_true",
                    help="small bf16 batches: the whole layer in one persistent cooperative launch (opt-in)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- distributed plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if (torch.cuda.is_available() and args.impl == "ours") else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available() and args.impl == "ours":
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        smax = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


KERNEL_SOURCES = {
    "gemm1": ("common.cuh", "gemm.cu", "kernels.h"),
    "gemm2": ("common.cuh", "gemm.cu", "kernels.h"),
}


def kernel_source_sha(kernel: str) -> str:
    """Hash of the sources that define a kernel (a stored ncu figure is only
    valid while it matches)."""
    src = os.path.join(ROOT, "moe_layer_top_b200", "csrc")
    h = hashlib.sha256()
    for name in KERNEL_SOURCES.get(kernel, tuple(sorted(os.listdir(src)))):
        with open(os.path.join(src, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, workload: str, T: int):
    """DRAM bytes per launch from a committed ncu summary, if the kernel
    source is unchanged since it was captured."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            recs = json.load(f)
    except (OSError, ValueError):
        return None
    digest = kernel_source_sha(kernel)
    for r in recs:
        if r.get("kernel") == kernel and r.get("workload") == workload and int(r.get("T", -1)) == T \
                and r.get("source_sha") == digest:
            return float(r["dram_bytes_per_launch"])
    return None


# ----------------------------------------------------------------------------- our arm
def workload_config(args):
    import dataclasses
    cfg = inputs.CONFIGS[args.workload or DEFAULT_WORKLOAD]
    if args.experts:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}[E={args.experts}]", E=args.experts)
    return cfg


class Workload:
    """One batch of the layer on this GPU.  ``ep = (first, count, reduce)``: this
    rank's share of an expert-parallel layer (experts [first, first + count) of
    cfg.E; ``reduce``: all-reduce the output over the process group after the
    share, which completes the layer on every rank)."""

    def __init__(self, cfg, T, seed, weights, persistent_decode=False, ep=None):
        from moe_layer_top_b200 import ops
        self.ops = ops
        self.cfg, self.T = cfg, T
        dev = torch.device("cuda")
        self.w13, self.w2, self.s13, self.s2 = weights
        self.x = inputs.make_tokens(cfg, T, seed, device=dev)
        self.routing = inputs.make_routing(cfg, T, seed, device=dev)
        self.ep = ep
        first, count = (0, cfg.E) if ep is None else ep[:2]
        self.p = ops.problem(T, count, cfg.topk, cfg.H, cfg.I, fp8=cfg.fp8, mx=cfg.mx,
                             persistent_decode=persistent_decode, num_global_experts=cfg.E, first_expert=first)
        self.q = ops.resolve_problem(self.p)
        self.ws = ops.alloc_workspace(self.p)
        self.out = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)

    def kw(self):
        return dict(logits=self.routing.get("logits"), topk_ids=self.routing.get("topk_ids"),
                    topk_weights=self.routing.get("topk_weights"), w13_scale=self.s13, w2_scale=self.s2,
                    out=self.out, ws=self.ws)

    def stage(self, s):
        self.ops.forward_stages(self.p, self.x, self.w13, self.w2, s, s + 1, **self.kw())

    def forward(self):
        self.ops.fused_forward(self.p, self.x, self.w13, self.w2, **self.kw())

    def collective(self):
        """The step's exchange: the all-reduce of an expert-parallel share (nothing otherwise)."""
        if self.ep is not None and self.ep[2]:
            import torch.distributed as dist
            dist.all_reduce(self.out, op=dist.ReduceOp.SUM)

    def algorithmic(self):
        """Algorithmic bytes / FLOPs of the layer and of each GEMM for this routing."""
        v = self.ops.workspace_views(self.p, self.ws)
        return algorithmic_counts(self.cfg, self.T, v["expert_counts"].cpu().numpy(),
                                  int(v["num_tokens_post_padded"].item()), "logits" in self.routing)


def algorithmic_counts(cfg, T, counts, ntpp, has_logits):
    """Algorithmic bytes and FLOPs of one layer step: every hit expert's weights read once (with
    their scales), x read and out written once, the routing input read; per GEMM also the padded
    token rows it reads and the rows it writes.  FLOPs count real assignments only (2 * 3 * H * I
    each).  counts: assignments per expert run here; ntpp: padded rows of the alignment."""
    hit = int((counts > 0).sum())
    elem = 1 if cfg.fp8 else 2
    if cfg.mx:   # one E8M0 byte per 32 weights
        w13_e = 2 * cfg.I * cfg.H * (1 + 1 / 32)
        w2_e = cfg.H * cfg.I * (1 + 1 / 32)
    else:
        w13_e = 2 * cfg.I * cfg.H * elem + (2 * cfg.I // 128) * (cfg.H // 128) * 4 * cfg.fp8
        w2_e = cfg.H * cfg.I * elem + (cfg.H // 128) * (cfg.I // 128) * 4 * cfg.fp8
    nflat = T * cfg.topk
    nlocal = int(counts.sum())       # assignments run here (all of them without expert parallelism)
    route_io = T * cfg.E * 4 if has_logits else nflat * 8
    rows = ntpp
    gemm1 = hit * w13_e + rows * cfg.H * elem + rows * cfg.I * elem
    gemm2 = hit * w2_e + rows * cfg.I * elem + nlocal * cfg.H * 2
    layer = hit * (w13_e + w2_e) + T * cfg.H * 2 * 2 + route_io
    flops = 2.0 * nlocal * 3 * cfg.H * cfg.I
    return {"hit_experts": hit, "padded_rows": ntpp, "layer_bytes": layer, "gemm1_bytes": gemm1,
            "gemm2_bytes": gemm2, "flops": flops, "w13_bytes_per_expert": w13_e, "w2_bytes_per_expert": w2_e}


def kernels_per_forward(cfg, T, has_logits):
    """Kernels of this library one moe_fused_forward launches: a single-CTA
    route+align for T*topk <= 8192 and E <= 256, else route + 3 align passes;
    then gather, GEMM1, GEMM2, combine (not counting a split-K reduce, which
    only small swap-AB problems launch).  Used only when the captured graph
    cannot be inspected."""
    small = T * cfg.topk <= 8192 and cfg.E <= 256
    head = 1 if small else (1 if has_logits else 0) + 3
    return head + 4


def graph_kernel_count(g):
    """Kernel nodes of a captured CUDA graph (None if it cannot be read).  The
    forward graph captures nothing but this library's launches."""
    try:
        import cuda.bindings.runtime as rt
        graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
        return sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)
    except Exception:
        return None


def make_weights(cfg, seed, ep=None):
    """The layer's weights on the GPU (with ``ep = (first, count, ...)`` only
    experts [first, first + count), drawn exactly as in the full layer)."""
    from moe_layer_top_b200 import ops
    if ep is None:
        w13, w2 = inputs.make_weights(cfg, seed, device="cuda")
    else:
        first, count = ep[:2]
        w13 = torch.empty((count, 2 * cfg.I, cfg.H), dtype=torch.bfloat16, device="cuda")
        w2 = torch.empty((count, cfg.H, cfg.I), dtype=torch.bfloat16, device="cuda")
        for i in range(count):
            a, b = inputs.make_expert_weights(cfg, first + i, seed, device="cuda")
            w13[i].copy_(a)
            w2[i].copy_(b)
    if cfg.fp8:
        quant = ops.quantize_weights_mxfp8 if cfg.mx else ops.quantize_weights_fp8
        q13, s13 = quant(w13)
        q2, s2 = quant(w2)
        del w13, w2
        torch.cuda.empty_cache()
        return q13, q2, s13, s2
    return w13, w2, None, None


class StageEvents:
    """CUDA events recorded as nodes of a captured graph.

    Inside stream capture a plain event record only expresses a dependency;
    cudaEventRecordWithFlags(..., cudaEventRecordExternal) makes it a timing
    node of the graph, so every replay stamps the events again."""

    def __init__(self, n):
        import ctypes
        import glob
        self.ctypes = ctypes
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in self.ev:
            e.record()
        torch.cuda.synchronize()
        libs = glob.glob(os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib",
                                      "libcudart.so*")) + ["libcudart.so.12", "libcudart.so"]
        self.rt = None
        for lib in libs:
            try:
                self.rt = ctypes.CDLL(lib)
                break
            except OSError:
                continue
        if self.rt is None:
            raise RuntimeError("libcudart not found")
        self.rt.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
        self.rt.cudaEventRecordWithFlags.restype = ctypes.c_int

    def record(self, i):
        if not torch.cuda.is_current_stream_capturing():
            self.ev[i].record()
            return
        stream = torch.cuda.current_stream().cuda_stream
        rc = self.rt.cudaEventRecordWithFlags(self.ctypes.c_void_p(self.ev[i].cuda_event),
                                              self.ctypes.c_void_p(stream), 1)
        if rc != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")

    def elapsed(self):
        return [self.ev[i].elapsed_time(self.ev[i + 1]) for i in range(len(self.ev) - 1)]


def capture(fn):
    """Capture fn() into a CUDA graph (after it has run once eagerly)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def count_kernels(fn):
    """Kernel launches of one fn() call, read from a separate capture that is
    never replayed (the timed graph is captured the ordinary way)."""
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    n = graph_kernel_count(g)
    del g
    return n


def time_steps(wl: Workload, steps: int, warmup: int, flush: torch.Tensor, world: int):
    """Two timed passes, L2 flushed before every step (outside the events):
    A) a CUDA graph of moe_fused_forward, one event pair per replay -> step times;
    B) a CUDA graph of the same stages with event nodes between them -> per-stage times."""
    ops = wl.ops
    stream = torch.cuda.current_stream()
    n_kernels = count_kernels(wl.forward)
    g_fwd = capture(wl.forward)
    se = StageEvents(ops.NUM_STAGES + 1)

    def staged():
        se.record(0)
        for s in range(ops.NUM_STAGES):
            wl.stage(s)
            se.record(s + 1)

    g_stg = capture(staged)
    for _ in range(warmup):
        flush_l2(flush)
        g_fwd.replay()
        wl.collective()
        flush_l2(flush)
        g_stg.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(steps):
        flush_l2(flush)
        ev[i][0].record(stream)
        g_fwd.replay()
        wl.collective()     # outside the graph: no NCCL call is ever captured
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    step_ms = np.array([a.elapsed_time(b) for a, b in ev])
    per_stage = []
    for i in range(steps):
        flush_l2(flush)
        g_stg.replay()
        torch.cuda.synchronize()
        per_stage.append(se.elapsed())
    return step_ms, np.array(per_stage), wall, n_kernels


def e2e_steps(wl: Workload, steps: int, warmup: int, flush: torch.Tensor):
    """Same metric with host buffers: pinned H2D of x (+ routing input), the
    layer, D2H of the output, all inside the CUDA-event brackets."""
    x_h = wl.x.cpu().pin_memory()
    r_h = {k: v.cpu().pin_memory() for k, v in wl.routing.items()}
    out_h = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
    x_d = torch.empty_like(wl.x)
    r_d = {k: torch.empty_like(v) for k, v in wl.routing.items()}
    stream = torch.cuda.current_stream()
    ops = wl.ops

    def one():
        x_d.copy_(x_h, non_blocking=True)
        for k in r_d:
            r_d[k].copy_(r_h[k], non_blocking=True)
        ops.fused_forward(wl.p, x_d, wl.w13, wl.w2, logits=r_d.get("logits"), topk_ids=r_d.get("topk_ids"),
                          topk_weights=r_d.get("topk_weights"), w13_scale=wl.s13, w2_scale=wl.s2, out=wl.out,
                          ws=wl.ws)
        wl.collective()
        out_h.copy_(wl.out, non_blocking=True)

    for _ in range(warmup):
        flush_l2(flush)
        one()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush_l2(flush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        one()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    h2d = x_h.numel() * x_h.element_size() + sum(v.numel() * v.element_size() for v in r_h.values())
    d2h = out_h.numel() * out_h.element_size()
    return float(np.sum(times)), h2d, d2h


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(cfg, T, seed, budget_s, single_thread=True):
    """The oracle, as it stands (C++, double precision), timed on bounded token
    samples of the workload: with OpenMP over the rows on every host core
    (``value``), and on one thread (``single_thread``).

    The generator's inputs for the sampled tokens (and the oracle's own FP8
    quantisation of the weights they touch) are prepared untimed; the timed
    region is the oracle's forward on those tokens."""
    from oracle import moe_oracle as O
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = inputs.make_tokens(cfg, T, seed, device=dev).float().cpu().double().numpy()
    routing = {k: v.cpu().numpy() for k, v in inputs.make_routing(cfg, T, seed, device=dev).items()}
    if "logits" in routing:
        ids_all, _ = O.route(routing["logits"], cfg.topk)
        rkw = {"logits": routing["logits"]}
    else:
        ids_all = routing["topk_ids"]
        rkw = {"topk_ids": routing["topk_ids"], "topk_weights": routing["topk_weights"]}
    host = {}

    def bits(w):
        return w.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def prepare(tokens):
        for e in np.unique(ids_all[tokens]):
            e = int(e)
            if e not in host:
                a, b = inputs.make_expert_weights(cfg, e, seed, device=dev)
                a, b = bits(a), bits(b)
                if cfg.mx:
                    host[e] = (*O.quantize_mx_group32(a), *O.quantize_mx_group32(b))
                elif cfg.fp8:
                    host[e] = (*O.quantize_weight_block128(a), *O.quantize_weight_block128(b))
                else:
                    host[e] = (a, None, b, None)

    class View:
        def __init__(self, i):
            self.i = i

        def __getitem__(self, e):
            return host[int(e)][self.i]

    def timed(threads, budget):
        order = np.random.default_rng(seed).permutation(T)
        done, t_spent, n = 0, 0.0, 1
        while done < T and (done == 0 or t_spent < budget):
            tok = order[done:done + n]
            prepare(tok)
            t0 = time.perf_counter()
            if cfg.fp8:
                O.moe_forward(x, View(0), View(2), cfg.topk, w13_scale=View(1), w2_scale=View(3), tokens=tok,
                              mx=cfg.mx, threads=threads, **rkw)
            else:
                O.moe_forward(x, View(0), View(2), cfg.topk, tokens=tok, threads=threads, **rkw)
            t_spent += time.perf_counter() - t0
            done += len(tok)
            n = min(2 * n, T - done) if done < T else n
        return done, t_spent

    cores = O.max_threads()
    done, t_spent = timed(0, budget_s)
    rec = {"value": round(done / t_spent, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"{done} of {T} tokens of {cfg.name} (T={T}); C++ double-precision oracle forward, OpenMP "
                     f"over rows on {cores} threads, inputs prepared untimed; {t_spent:.2f} s timed",
           "cpu": _cpu_model()}
    if single_thread:
        d1, t1 = timed(1, budget_s / 2)
        rec["single_thread"] = {"value": round(d1 / t1, 3), "unit": "tokens/s", "cores": 1,
                                "sample": f"{d1} of {T} tokens, one thread; {t1:.2f} s timed"}
    return rec


def measure(cfg, args, world, flush, peaks, ep=None, T_only=0):
    """Time one workload (its sweep, headline = the largest batch) and return its record."""
    from moe_layer_top_b200 import ops
    T_head = T_only or max(cfg.tokens)
    sweep_T = [T_head] if T_only else sorted(cfg.tokens)
    weights = make_weights(cfg, args.seed, ep)
    results = {}
    for T in sweep_T:
        wl = Workload(cfg, T, args.seed, weights, args.persistent_decode, ep)
        steps = args.steps if T == T_head else max(3, args.steps // 2)
        step_ms, per_stage, wall, n_kernels = time_steps(wl, steps, args.warmup, flush, world)
        total_ms = max_over_ranks(float(step_ms.sum()), world)
        results[T] = {"wl": wl, "per_stage": per_stage, "total_ms": total_ms, "steps": steps, "wall_s": wall,
                      "kernels": n_kernels}
    head = results[T_head]
    wl = head["wl"]
    alg = wl.algorithmic()
    K = head["steps"]
    # replicas: every rank runs its own batch; expert parallelism: the ranks share one batch
    layer_copies = 1 if ep is not None else world
    value = layer_copies * T_head * K / (head["total_ms"] / 1e3)
    ms_per_step = head["total_ms"] / K
    stage_ms = head["per_stage"].mean(axis=0)
    fp8_ratio = 2.0 if cfg.fp8 else 1.0
    tc_peak = peaks["bf16_tflops"] * fp8_ratio
    # dominant kernel: the stage with the largest share of the step
    dom = int(np.argmax(stage_ms))
    dom_name = ops.STAGE_NAMES[dom]
    dom_bytes = {"gemm1": alg["gemm1_bytes"], "gemm2": alg["gemm2_bytes"]}.get(dom_name)
    if dom_bytes is None:
        dom_bytes = alg["layer_bytes"]
    traffic = traffic_record(dom_name, cfg.name, T_head) if ep is None else None
    # FLOPs of the dominant GEMM (GEMM1 = 2/3 of the layer, GEMM2 = 1/3)
    dom_flops = alg["flops"] * {"gemm1": 2.0 / 3.0, "gemm2": 1.0 / 3.0}.get(dom_name, 1.0)
    # tensor-core peak for the arithmetic dtype: measured bf16 (burst: the kernel
    # is timed on its own inside a short step); FP8 = 2x that, the nominal ratio
    tc_source = f"{peaks['source']} bf16 burst" + (" x 2 (nominal FP8/bf16 ratio)" if cfg.fp8 else "")
    if dom_flops / (tc_peak * 1e12) > dom_bytes / (peaks["hbm_gbs"] * 1e9):
        achieved = dom_flops / (stage_ms[dom] / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": dom_name, "achieved": round(achieved, 1), "peak": round(tc_peak, 1),
                    "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4), "traffic": traffic,
                    "peak_source": tc_source, "algorithmic_flops": dom_flops, "algorithmic_bytes": dom_bytes}
    else:
        achieved = dom_bytes / (stage_ms[dom] / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": dom_name, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                    "peak_source": peaks["source"], "algorithmic_bytes": dom_bytes}
    sweep = []
    for T in sweep_T:
        r = results[T]
        a = r["wl"].algorithmic()
        ms = r["total_ms"] / r["steps"]
        sm = r["per_stage"].mean(axis=0)
        sweep.append({"T": T, "tokens_per_s": round(layer_copies * T / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
                      "layer_hbm_frac": round(a["layer_bytes"] / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                      "tflops": round(a["flops"] / (ms / 1e3) / 1e12, 2),
                      "layer_tc_frac": round(a["flops"] / (ms / 1e3) / 1e12 / tc_peak, 4),
                      "hit_experts": a["hit_experts"],
                      "stage_us": {ops.STAGE_NAMES[s]: round(float(sm[s]) * 1e3, 1) for s in range(ops.NUM_STAGES)},
                      "mode": "swap_ab" if r["wl"].q.mode == ops.MODE_SWAP_AB else "normal",
                      "kernels_per_step": r["kernels"],
                      "block_m": r["wl"].q.block_m})
    e2e_ms, h2d, d2h = e2e_steps(wl, K, args.warmup, flush)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e = {"value": round(layer_copies * T_head * K / (e2e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if ep is None:
        parallelism, scaling, wl_name = f"replicas{world}", "weak", cfg.name
    elif world > 1:
        parallelism, scaling = f"ep{world} (experts [{ep[0]}, {ep[0] + ep[1]}) on rank 0; NCCL all-reduce)", "strong"
        wl_name = cfg.name
    else:
        parallelism, scaling = (f"ep{args.ep} share of rank {args.ep_rank} (experts [{ep[0]}, {ep[0] + ep[1]})) "
                                f"alone on one GPU: no all-reduce", "strong")
        wl_name = f"{cfg.name} (one EP={args.ep} share)"
    rec = {
        "value": round(value, 1), "unit": "tokens/s", "steps": K, "ms_per_step": round(ms_per_step, 4),
        "scaling": scaling,
        "dtype": ("mxfp8_e4m3" if cfg.mx else "fp8_e4m3") if cfg.fp8 else "bf16",
        "config": {"workload": f"{wl_name}: H={cfg.H} E={cfg.E} topk={cfg.topk} I={cfg.I} T={T_head}",
                   "global_batch": layer_copies * T_head, "tokens_per_gpu": T_head, "parallelism": parallelism,
                   "weights": ("mxfp8 e4m3 + per-32 e8m0 scales" if cfg.mx else "fp8 e4m3 + 128x128 fp32 scales")
                   if cfg.fp8 else "bf16",
                   "routing": cfg.routing, "l2": "flushed (256 MiB write, then read back) before every step, outside the timing",
                   "launch": ("CUDA graph of moe_fused_forward (persistent decode kernel where eligible)"
                              if args.persistent_decode else "CUDA graph of moe_fused_forward (PDL between kernels)"),
                   "layer_bytes_per_step": alg["layer_bytes"], "layer_flops_per_step": alg["flops"],
                   "hit_experts": alg["hit_experts"]},
        "roofline": roofline,
        "layer_hbm_frac": round(alg["layer_bytes"] / (ms_per_step / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "layer_tc_frac": round(alg["flops"] / (ms_per_step / 1e3) / 1e12 / tc_peak, 4),
        "stage_us": {ops.STAGE_NAMES[s]: round(float(stage_ms[s]) * 1e3, 1) for s in range(ops.NUM_STAGES)},
        "sweep": sweep,
        "e2e": e2e,
        "gpu_launches": K * (head["kernels"] or kernels_per_forward(cfg, T_head, "logits" in wl.routing)),
        "gpu_launches_source": "kernel nodes of the captured forward graph" if head["kernels"] else "formula",
    }
    del results, wl, weights
    torch.cuda.empty_cache()
    return rec, T_head


# the default run: the largest single-GPU configuration is the headline; the
# compute-bound prefill layer and the bf16 decode layer ride along as sub-records
DEFAULT_WORKLOAD = "skewed_fp8"
DEFAULT_SUB_RECORDS = ("prefill_fp8", "decode_bf16")


def run_ours(args, rank, world, local):
    from moe_layer_top_b200 import build, ops
    build.build()
    ops.lib()
    cfg = workload_config(args)
    peaks = measured_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    ep = None
    if args.ep:
        # expert parallelism: on N ranks each runs its share and the output is
        # all-reduced; on one GPU the step is one rank's share alone
        from moe_layer_top_b200.expert_parallel import expert_shard
        if world not in (1, args.ep):
            raise SystemExit(f"--ep {args.ep} runs on {args.ep} ranks, or on one GPU (one share)")
        ep_rank = rank if world > 1 else args.ep_rank
        ep = (*expert_shard(cfg.E, args.ep, ep_rank), world > 1)
    subs = []
    if args.workload is None and not (args.tokens or args.experts or args.ep or args.no_sub_records):
        subs = list(DEFAULT_SUB_RECORDS)
    with ClockSampler(local) as clocks:
        head, T_head = measure(cfg, args, world, flush, peaks, ep, args.tokens)
        sub_recs = {name: measure(inputs.CONFIGS[name], args, world, flush, peaks) for name in subs}
    clk = clocks.summary()
    line = {"metric": "fused-MoE tokens/s; % HBM roofline (decode), % FP8/BF16 TC peak (prefill)",
            "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": head["steps"],
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": head["scaling"], "vs_baseline": None, "dtype": head["dtype"], "data": "synthetic"}
    line.update({k: v for k, v in head.items() if k not in line})
    line["clocks"] = clk
    cpu = rank == 0 and world == 1 and not args.no_cpu_baseline and ep is None
    if cpu:
        line["cpu_baseline"] = cpu_baseline(cfg, T_head, args.seed, args.cpu_budget)
    if sub_recs:
        line["sub_records"] = {}
        for name, (rec, T) in sub_recs.items():
            if cpu:
                rec["cpu_baseline"] = cpu_baseline(inputs.CONFIGS[name], T, args.seed, args.cpu_budget / 2,
                                                   single_thread=False)
            line["sub_records"][name] = rec
    return line


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, rank, world):
    cfg = workload_config(args)
    T = args.tokens or max(cfg.tokens)
    if rank != 0:
        return None
    for _ in range(args.warmup):
        cpu_baseline(cfg, T, args.seed, budget_s=0.0, single_thread=False)
    vals = []
    base = None
    per_step_budget = max(1.0, args.cpu_budget / max(1, args.steps))
    for _ in range(args.steps):
        base = cpu_baseline(cfg, T, args.seed, budget_s=per_step_budget, single_thread=False)
        vals.append(base["value"])
    value = float(np.mean(vals))
    base["value"] = round(value, 3)
    return {
        "impl": "reference",
        "metric": "fused-MoE tokens/s; % HBM roofline (decode), % FP8/BF16 TC peak (prefill)",
        "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * T / value, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: H={cfg.H} E={cfg.E} topk={cfg.topk} I={cfg.I} T={T}",
                   "global_batch": T, "parallelism": "cpu"},
        "cpu_baseline": base,
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
