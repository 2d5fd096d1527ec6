#!/usr/bin/env python
"""MoE feed-forward layer, forward + backward, on B200s: throughput bench.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config olmo128]
    python bench.py --impl reference ...     (the CPU oracle on the host cores)

One step = moe_layer_fwd + moe_layer_bwd on one batch of seeded synthetic
inputs already resident in HBM (router, routing metadata, dispatch, the two
SwiGLU grouped GEMMs, combine, and the whole backward including all weight
gradients).  The N GPUs run independent replicas (the single-GPU layer has
no exchange step); `value` counts the tokens of all ranks over the slowest
rank's device time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import moe_inputs  # noqa: E402

METRIC = "MoE layer fwd+bwd tokens/sec and grouped-GEMM TFLOP/s (% of peak) on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="olmo128", choices=sorted(moe_inputs.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (a smaller case of the same layer, e.g. for ncu captures)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E at fixed T, d, k, F (expert-count sweep: same active "
                         "FLOPs per token, E times the expert weights)")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = str(index)
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", self.index], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                "sw_power_cap"), f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------ CPU baseline
def _oracle_step(oracle, cfg, x, dout, W, Wr, b, topk=None, gates=None):
    if topk is None:
        ctx = oracle.layer_forward(x, *W, cfg.k, Wr=Wr, bias=b, mx=cfg.mx)
    else:
        ctx = oracle.layer_forward(x, *W, cfg.k, topk_idx=topk, gates=gates, mx=cfg.mx)
    oracle.layer_backward(ctx, dout)


class OracleRunner:
    """The CPU oracle, as it stands, on a token sample of the workload.

    Router workloads: the first n tokens with all experts.  Given-routing
    workloads (the trillion shape): the first n tokens with only the experts
    they are routed to (expert ids renumbered in order), which gives the same
    per-token results, so that the fp64 weights stay within `mem_limit`
    bytes of host memory (all 384 experts would need 116 GB)."""

    def __init__(self, cfg, inp, target_s, mem_limit=8e9):
        import oracle
        from threadpoolctl import threadpool_limits
        self.oracle = oracle
        self.cfg = cfg
        self.cores = len(os.sched_getaffinity(0))
        self._limit = threadpool_limits(self.cores)
        f64 = moe_inputs.to_f64
        self.given = cfg.routing != "router"
        self.Wsrc = [inp[n] for n in ("W1", "W3", "W2")]
        self.W = None if self.given else [
            w.to(torch.float64).cpu().numpy() if w.is_cuda else f64(w) for w in self.Wsrc]
        self.x = f64(inp["x"]); self.dout = f64(inp["dout"])
        self.Wr = f64(inp["Wr"]); self.b = f64(inp["bias"])
        self.topk = inp["topk_idx"].cpu().numpy() if self.given else None
        self.gates = f64(inp["gates"]) if self.given else None
        self.e_used = cfg.E
        per_expert = 3 * cfg.d * cfg.F * 8
        # grow the sample (doubling) until one step takes about target_s / 2
        # or more; the groups are padded to 128 rows, so the cost is far from
        # linear in the sample at small sizes
        n = 1 if self.given else min(cfg.T, 256)
        while True:
            self._prepare(n)
            t = self._time(n)
            nxt = min(cfg.T, 2 * n)
            if t >= target_s / 2 or n >= cfg.T:
                break
            if self.given and len(np.unique(self.topk[:nxt])) * per_expert > mem_limit:
                break
            n = nxt
        self.n, self.last_t = n, t

    def _prepare(self, n):
        """fp64 weights of the experts the first n tokens use (given routing)."""
        if not self.given:
            self._Wn, self._topk_n = self.W, None
            return
        used = np.unique(self.topk[:n])
        remap = np.full(self.cfg.E, -1, np.int64)
        remap[used] = np.arange(len(used))
        sel = torch.from_numpy(used).to(self.Wsrc[0].device)
        self._Wn = [w.index_select(0, sel).to(torch.float64).cpu().numpy() for w in self.Wsrc]
        self._topk_n = remap[self.topk[:n]].astype(np.int32)
        self.e_used = len(used)

    def _time(self, n):
        sl = slice(0, n)
        t0 = time.perf_counter()
        _oracle_step(self.oracle, self.cfg, self.x[sl], self.dout[sl], self._Wn, self.Wr, self.b,
                     self._topk_n, None if self.gates is None else self.gates[sl])
        return time.perf_counter() - t0

    def step(self):
        return self._time(self.n)

    def describe(self):
        experts = (f"the {self.e_used} of {self.cfg.E} experts they are routed to"
                   if self.given else f"all {self.cfg.E} experts")
        return (f"first {self.n} of {self.cfg.T} tokens of the workload, full fwd+bwd of the fp64 "
                f"NumPy oracle ({experts}, groups padded to 128 rows"
                f"{', MXFP8 operands' if self.cfg.mx else ''})")


# ----------------------------------------------------------------- helpers
def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _maxreduce(v, world):
    """The largest v over the ranks (device time of the slowest replica)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _job_rate(world, tokens_per_rank, steps, max_ms):
    """Whole-job tokens/s: the tokens of all replicas over the slowest one's time."""
    return world * tokens_per_rank * steps / (max_ms * 1e-3)


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` from a committed ncu summary
    (profiles/traffic_<kernel>.md: lines `workload: <name>`,
    `source_sha256: <hex>` of the kernel's source file, `source: <file>` and
    `dram_bytes_per_launch: <int>`), or None unless that capture was taken
    on the current source and on the workload being timed."""
    p = os.path.join(ROOT, "profiles", f"traffic_{kernel}.md")
    if not os.path.exists(p):
        return None
    fields = {}
    for line in open(p):
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip().strip("`- ")] = v.strip().strip("`")
    src_file = fields.get("source", "")
    src_path = os.path.join(ROOT, "mixture_experts_layer_25_b200", "csrc", src_file)
    if not src_file or not os.path.exists(src_path):
        return None
    if fields.get("source_sha256") != hashlib.sha256(open(src_path, "rb").read()).hexdigest():
        return None
    if fields.get("workload") != workload:
        return None
    try:
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


NOMINAL_BF16_TFLOPS = 2250.0     # dense bf16 per B200; fp8 is twice that


def _tensor_peak(peaks, peak_kind, clk, timed_s, mx):
    """The roofline's tensor peak: the measured burst figure when the timed
    region is short (under 2 s) and no power-cap throttling was sampled in
    it, the measured sustained (power-capped) figure otherwise; x2 for fp8
    (the nominal fp8 : bf16 ratio).  Returns (chosen peak, its name, all
    candidate peaks)."""
    f = 2.0 if mx else 1.0
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * f
    sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])) * f
    capped = bool(clk and "sw_power_cap" in clk.get("reasons", []))
    use_burst = timed_s < 2.0 and not capped
    name = ("bf16_tflops" if use_burst else "bf16_tflops_sustained") + f" of {peak_kind}"
    if mx:
        name += " x2 for fp8"
    return (burst if use_burst else sus), name, {"burst": burst, "sustained": sus,
                                                 "nominal": NOMINAL_BF16_TFLOPS * f}


def schedule_efficiency(work, workers):
    """Busy fraction of `workers` persistent CTAs (or CTA pairs) that take
    tiles round-robin (tile i -> worker i mod workers, as the grouped GEMMs
    walk their schedules): mean worker load over the largest one."""
    work = np.asarray(work, np.float64)
    if work.size == 0 or work.sum() == 0:
        return 1.0
    loads = np.bincount(np.arange(work.size) % workers, weights=work, minlength=workers)
    return float(loads.mean() / loads.max())


def load_metrics(counts, poff, cfg, num_sms=148):
    """Expert load of one routing: imbalance, a histogram of the per-expert
    row counts, the rows the 128-row group padding adds, and how evenly the
    GEMM tile schedules spread that load over the SMs (value-dependent
    kernel timing: the same FLOPs take longer when a few experts are hot)."""
    E, A = cfg.E, cfg.T * cfg.k
    counts = np.asarray(counts, np.int64)
    edges = np.unique(np.concatenate([[0, 1], np.geomspace(1, max(2, counts.max() + 1), 10).astype(np.int64)]))
    hist, _ = np.histogram(counts, bins=np.append(edges, counts.max() + 1))
    # rows-mode GEMMs: 128-row tiles of every group times the N tiles, each
    # tile the same K work (fwd GEMM1 at F / 128 column tiles)
    rows_tiles = np.repeat(np.ones(int(poff[-1]) // 128), max(1, cfg.F // 128))
    # weight-gradient GEMMs (BF16, SM pairs): per expert (d / 256) x (2F / 256)
    # output tiles, each reducing over the group's real rows in 64-row
    # blocks, experts taken longest first
    kb = -(-counts // 64)[np.argsort(-counts, kind="stable")]
    wg_tiles = np.repeat(kb, max(1, (cfg.d // 256) * (2 * cfg.F // 256)))
    return {"max_over_mean": round(float(counts.max() / max(counts.mean(), 1e-9)), 3),
            "hottest_share": round(float(counts.max() / A), 4),
            "empty_experts": int((counts == 0).sum()),
            "count_quantiles": {q: int(np.percentile(counts, q)) for q in (0, 10, 50, 90, 100)},
            "count_histogram": {"edges": [int(v) for v in edges], "experts": [int(v) for v in hist]},
            "padded_rows": int(poff[-1]), "pad_overhead": round(float(poff[-1] / A - 1.0), 4),
            "schedule_efficiency": {
                "rows_gemm_1sm": round(schedule_efficiency(rows_tiles, num_sms), 4),
                "wgrad_gemm_pairs": round(schedule_efficiency(wg_tiles, num_sms // 2), 4)}}


def _cfg_dict(cfg, extra):
    d = {"workload": f"{cfg.name}: one MoE SwiGLU FFN layer fwd+bwd, T={cfg.T} tokens, d_model={cfg.d}, "
                     f"E={cfg.E} experts, top-{cfg.k}, d_ff={cfg.F}, "
                     f"{'router softmax/top-k' if cfg.routing == 'router' else 'random routing'}"
                     f"{' + Zipf bias' if cfg.bias else ''}, {'MXFP8' if cfg.mx else 'BF16'} grouped GEMMs",
         "T": cfg.T, "d_model": cfg.d, "experts": cfg.E, "top_k": cfg.k, "d_ff": cfg.F,
         "routing": cfg.routing, "grouped_gemm_dtype": "mxfp8" if cfg.mx else "bf16",
         "l2": "inputs larger than L2 (expert weights %.2f GB per step)" % (3 * cfg.E * cfg.d * cfg.F * 2 / 1e9),
         "parallelism": "replicas (no exchange step in the single-GPU layer)"}
    d.update(extra)
    return d


def _config(args):
    cfg = moe_inputs.CONFIGS[args.config]
    if args.tokens:
        cfg = cfg.with_(T=args.tokens)
    if args.experts:
        cfg = cfg.with_(E=args.experts)
    return cfg


# ------------------------------------------------------------ reference arm
def run_reference(args):
    world, rank, local = _dist()
    if rank != 0:
        return
    cfg = _config(args)
    inp = moe_inputs.make_layer_inputs(cfg, "cpu")
    # each step is a token sample sized so that the whole run takes about
    # four minutes (at most ~15 s per step, the sample of the cpu_baseline).
    # Small samples run slower per token: every expert group is padded to 128
    # rows, a fixed cost of E * 128 rows whatever the sample.
    r = OracleRunner(cfg, inp, target_s=min(15.0, 240.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        r.step()
    t = 0.0
    for _ in range(args.steps):
        t += r.step()
    value = r.n * args.steps / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _cfg_dict(cfg, {"sample_tokens_per_step": r.n}),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r.cores, "kind": "oracle",
                             "sample": r.describe()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- our arm
def run_ours(args):
    import mixture_experts_layer_25_b200 as moe
    from mixture_experts_layer_25_b200 import _lib
    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    cfg = _config(args)
    peaks, peak_kind = _peaks()
    inp = moe_inputs.make_layer_inputs(cfg, "cuda")
    layer = moe.MoELayer(T=cfg.T, d=cfg.d, E=cfg.E, k=cfg.k, F=cfg.F, W1=inp["W1"], W3=inp["W3"],
                         W2=inp["W2"], Wr=inp["Wr"] if cfg.routing == "router" else None,
                         bias=inp["bias"], topk_idx=inp.get("topk_idx"), gates=inp.get("gates"),
                         mx=cfg.mx)
    x, dout = inp["x"], inp["dout"]
    out = torch.empty_like(x)
    dx = torch.empty_like(dout)
    stream = torch.cuda.current_stream()

    def step():
        layer.forward(x, out)
        layer.backward(x, dout, dx)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if layer.status.item() != 0:
        raise RuntimeError(f"device status {layer.status.item()} after warm-up")

    nst = len(_lib.STAGES)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nst)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record(stream)     # torch creates the event handles on first record
    torch.cuda.synchronize()
    arrs = [(ctypes.c_void_p * (2 * nst))(*[e.cuda_event for e in row]) for row in evs]
    assert all(a[i] for a in arrs for i in range(2 * nst))
    lib = _lib.lib()
    launches0 = lib.moe_launch_count()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_index = vis.split(",")[local] if vis else str(local)
    clocks = ClockSampler(smi_index)
    clocks.start()
    time.sleep(0.5)          # let the sampler take its first readings before the timed region
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        lib.moe_set_stage_events(arrs[i], 2 * nst)
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    lib.moe_set_stage_events(None, 0)
    launches = lib.moe_launch_count() - launches0
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    ms = _maxreduce(ms, world)
    if layer.status.item() != 0:
        raise RuntimeError(f"device status {layer.status.item()} after timing")

    # per-stage device time, from the stage events recorded inside the steps
    stage_ms = {}
    for s in range(nst):
        # a stage this mode does not run keeps the timestamp of its set-up
        # record, which precedes the timed region
        if t_start.elapsed_time(evs[0][2 * s]) <= 0.0:
            continue
        v = [evs[i][2 * s].elapsed_time(evs[i][2 * s + 1]) for i in range(args.steps)]
        stage_ms[_lib.STAGES[s]] = statistics.mean(v)

    T, d, E, k, F = cfg.T, cfg.d, cfg.E, cfg.k, cfg.F
    A = T * k
    gemm_flops = {"gemm1_swiglu": 4.0 * A * d * F, "gemm2": 2.0 * A * F * d,
                  "gemm2_dgrad_swiglu_bwd": 2.0 * A * d * F, "gemm2_wgrad": 2.0 * A * F * d,
                  "gemm1_dgrad": 4.0 * A * F * d, "gemm1_wgrad": 4.0 * A * d * F}
    gemm_ms = sum(stage_ms[n] for n in gemm_flops)
    flops = sum(gemm_flops.values())
    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12
    per_gemm = {n: round(gemm_flops[n] / (stage_ms[n] * 1e-3) / 1e12, 1) for n in gemm_flops}
    bpe = 2
    mem_bytes = {
        "route": T * d * bpe + d * E * 4 + T * E * 4 + T * k * 16,
        "permute": T * d * bpe + A * d * bpe,
        "combine": A * d * bpe + T * d * bpe,
        # the MXFP8 layer writes no bf16 dY here (its dY leaves as MX codes)
        "combine_bwd": T * d * bpe + (1 if cfg.mx else 2) * A * d * bpe,
        "unpermute_sum": A * d * bpe + T * d * bpe,
    }
    if cfg.mx:
        # codes along both K axes (1 byte each) plus one scale byte per 32
        wq = 3 * E * d * F
        mem_bytes["quant_w_fwd"] = wq * bpe + 2 * wq + 2 * wq // 32
        mem_bytes["quant_dgrad2"] = T * d * bpe + 2 * A * d + 2 * A * d // 32
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    mem = {n: {"GB_s": round(b / (stage_ms[n] * 1e-3) / 1e9, 1),
               "frac_of_hbm": round(b / (stage_ms[n] * 1e-3) / 1e9 / hbm, 3),
               "ms": round(stage_ms[n], 4)} for n, b in mem_bytes.items() if n in stage_ms}

    # expert load of this input (read after the timed region): the skewed
    # workload's imbalance, empty experts and the rows the 128-row group
    # padding adds to the GEMMs
    counts = layer.ctx_tensor("counts", (E,), torch.int32).cpu().numpy().astype(np.int64)
    poff = layer.ctx_tensor("poff", (E + 1,), torch.int32).cpu().numpy().astype(np.int64)
    load = load_metrics(counts, poff, cfg, num_sms=torch.cuda.get_device_properties(local).multi_processor_count)

    # end to end through the C ABI with host buffers (copies inside)
    e2e = None
    if not args.no_e2e:
        xh = x.cpu().pin_memory(); dh = dout.cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory(); dxh = torch.empty_like(xh).pin_memory()
        # two alternating sets of device buffers: a step's uploads run under
        # the previous step's backward
        bufs = [[torch.empty_like(x) for _ in range(4)] for _ in range(2)]
        for i in range(2):
            layer.step_host(xh, dh, oh, dxh, *bufs[i % 2])
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
        _barrier(world)
        a.record(stream)
        for i in range(args.steps):
            layer.step_host(xh, dh, oh, dxh, *bufs[i % 2])
        layer.step_host_sync()     # the last steps' downloads inside the timed region
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = _maxreduce(a.elapsed_time(b), world)
        nb = T * d * 2
        e2e = {"value": _job_rate(world, T, args.steps, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": 2 * nb, "d2h_bytes_per_step": 2 * nb,
               "ms_per_step": e_ms / args.steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            r = OracleRunner(cfg, inp, target_s=15.0)
            t = r.last_t
            cpu = {"value": r.n / t, "unit": "tokens/s", "cores": r.cores, "kind": "oracle",
                   "sample": r.describe(), "seconds": round(t, 2)}
        except MemoryError:
            cpu = None

    traffic = _traffic("grouped_gemm", cfg.name)
    peak, peak_name, cand = _tensor_peak(peaks, peak_kind, clk, ms * 1e-3, cfg.mx)
    line = {
        "metric": METRIC,
        "value": _job_rate(world, T, args.steps, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "mxfp8" if cfg.mx else "bf16",
        "data": "synthetic: seeded N(0,1) bf16 activations and upstream grads, N(0,0.02) random-init weights",
        "config": _cfg_dict(cfg, {}),
        "roofline": {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(gemm_tflops / peak, 4),
                     "traffic": traffic,
                     "kernel": "grouped GEMMs (all 6 launches of a step; algorithmic FLOPs "
                               "18*T*k*d*F over their summed event time)",
                     "peak_source": peak_name,
                     "frac_vs": {k_: round(gemm_tflops / v, 4) for k_, v in cand.items()},
                     "peaks_vs": cand},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk,
        "detail": {"stage_ms": {n: round(v, 4) for n, v in stage_ms.items()},
                   "grouped_gemm_tflops": per_gemm, "memory_bound": mem, "load": load,
                   "gemm_ms_per_step": round(gemm_ms, 4)},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
