"""Benchmark of the sparse-MoE block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qwen]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed

One step = one moe_forward (router GEMM + softmax + top-k, permutation,
grouped gate/up + SwiGLU GEMM, grouped down GEMM + routing weight, combine)
over one batch of T tokens of the named workload, with every input already
resident in HBM.  L2 is flushed (a 256 MiB write) between timed steps, and
each step is timed with CUDA events on the launching stream; inside a step
the library records events only around the gate/up GEMM (the roofline
kernel), because a recorded event stops the next kernel from launching
early.  A second pass of the same steps records every stage boundary for
the stage breakdown.  `e2e` repeats the measurement through the public API
with each step's token batch copied host->device from pinned memory and its
output copied back inside the timed region; consecutive steps overlap their
copies with the neighbouring step's compute on separate streams, as a
serving loop would, with no L2 flush (inputs larger than L2: the expert
weights alone exceed it).  `e2e_f16out` is the same loop with the block's fp16
output option (MOE_FLAG_OUT_F16: the fp32 result rounded once, half the
bytes read back); `value` and `e2e` keep the fp32 output.  SM clocks and
throttle reasons are sampled through NVML during the timed region.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica
on its own batch (the block is independent per token, so the path shards by
tokens with no data-path collective: weak scaling).  Ranks meet at a barrier
before and after the timed region and the slowest rank's time is used.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s & grouped-GEMM TFLOP/s vs roofline, 1×B200"
# The end-to-end legs do not flush L2 between steps: inputs larger than L2.
E2E_L2 = ("not flushed between steps: each step copies a fresh token batch in, and the block's working set "
          "(its expert weights alone, plus the grouped rows it writes) is larger than the 126 MB L2")
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
STAGES = ("route", "permute", "gateup_gemm", "down_gemm", "combine")
# router (GEMM + softmax + top-k), chunk scan, rank, row gather, gate/up GEMM, down GEMM, combine
KERNELS_PER_FORWARD = 7


# ------------------------------------------------------------- host logic
def dist_env():
    """(rank, local_rank, world) from the torchrun environment (1 process if unset)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, local, world


def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own token batch (weights use the same recipe)."""
    return base_seed + 1000 * rank


def whole_job_rate(units_per_rank: float, world: int, seconds_per_rank) -> float:
    """Aggregate throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / max(seconds_per_rank)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def algorithmic(cfg, active_experts=None, n_shared=0):
    """FLOPs and compulsory HBM bytes of one forward, and of its gate/up GEMM
    (n_shared shared experts of size f add 2*T*3*d*f FLOPs and their weights
    each)."""
    T, d, E, k, f = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f
    flops = 2 * T * (d * E + 3 * k * d * f) + n_shared * 2 * T * 3 * d * f
    gateup_flops = 2 * T * k * d * 2 * f
    down_flops = 2 * T * k * f * d
    nact = E if active_experts is None else active_experts
    # x read + out write (fp32) + router weights + weights of the experts in use
    compulsory = T * d * 2 + T * d * 4 + d * E * 2 + (nact + n_shared) * 3 * d * f * 2
    # per-stage algorithmic HBM bytes: route reads x and W_router and writes
    # ids + weights; permute reads x and writes x_perm (+ 12 B per
    # assignment of indices and weights); combine reads y (fp16), writes out
    stage_bytes = {
        "route": T * d * 2 + d * E * 2 + T * k * 8,
        "permute": T * d * 2 + T * k * d * 2 + T * k * 12,
        "combine": T * k * d * 2 + T * d * 4,
    }
    return {"flops": flops, "gateup_flops": gateup_flops, "down_flops": down_flops, "bytes": compulsory,
            "stage_bytes": stage_bytes}


# Datasheet figures for a B200 (dense bf16, HBM3e), for the second fraction
# of the forward roofline; the primary fraction uses the measured peaks
# (the fallback figures when the peaks file is absent).
DATASHEET = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}


class ClockSampler:
    """SM clock / throttle-reason sampling while the timed region runs.

    Reads NVML every few milliseconds from a background thread (read-only
    queries; no clock or power setting is touched); without NVML the summary
    says "unsampled".  The device is matched by its PCI bus id, so
    CUDA_VISIBLE_DEVICES does not matter.
    """

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    PERIOD_S = 0.004

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []   # (sm_mhz, max_mhz, power_w, reasons_bitmask)
        self.stop = None
        self.thread = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        prop = torch.cuda.get_device_properties(self.dev)
        bus = f"{prop.pci_domain_id:08x}:{prop.pci_bus_id:02x}:{prop.pci_device_id:02x}.0"
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except pynvml.NVMLError:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def _run(self, nv, h):
        while not self.stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def __enter__(self):
        import threading
        try:
            nv, h = self._handle()
        except Exception:
            return self
        self.stop = threading.Event()
        self.thread = threading.Thread(target=self._run, args=(nv, h), daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)

    def summary(self):
        rows = self.samples
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        reasons = sorted({name for r in rows for name, bit in self.REASONS if r[3] & bit})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_mhz_min": min(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "power_w_max": max(r[2] for r in rows),
                "samples": len(rows), "source": "NVML, every 4 ms during the timed region", "reasons": reasons}


# ------------------------------------------------------------ CPU oracle
def time_oracle(cfg, n_tokens: int, seed: int, inp=None):
    """Run the fp64 oracle (single thread) on the first n_tokens of the workload.

    Returns (seconds, n_tokens).  Same recipe, same shapes; only the token
    count is bounded so the CPU leg takes seconds, not hours.
    """
    import numpy as np
    from oracle.oracle import default_oracle
    from top_routing_grouped_softmax_b200.synth import make_inputs

    if inp is None:
        inp = make_inputs(cfg.with_(seed=seed))
    o = default_oracle()
    x = inp.bits("x")[:n_tokens]
    t0 = time.perf_counter()
    r = o.route(x, inp.bits("W_router"), inp.bias_np(), cfg.k)
    o.permute(r.ids, cfg.E)
    o.expert_rows(x, inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"), r.ids, r.weights,
                  np.arange(n_tokens, dtype=np.int64))
    return time.perf_counter() - t0, n_tokens


def host_cpu():
    """CPU model and logical core count of the host the oracle runs on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "host_logical_cpus": os.cpu_count()}


def cpu_baseline(cfg, n_tokens: int, seed: int, inp=None):
    secs, n = time_oracle(cfg, n_tokens, seed, inp)
    return {"value": n / secs, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"first {n} of {cfg.T} tokens of the {cfg.name} workload, full block "
                      f"(route, permute, expert MLPs, combine), fp64, one thread", **host_cpu()}


def route_parity(cfg, ids_gpu, seed):
    """Expert ids of the timed batch against the oracle's routing of every
    token (part of the CPU-oracle leg): tokens whose k-th and (k+1)-th
    probabilities differ by less than 1e-6 are counted and left out; tokens
    with a near tie between two selected slots are compared as sets."""
    import numpy as np
    from oracle.oracle import default_oracle, inner_gap, topk_gap
    from top_routing_grouped_softmax_b200.synth import make_inputs

    inp = make_inputs(cfg.with_(seed=seed))
    r = default_oracle().route(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), cfg.k)
    excluded = topk_gap(r.probs, cfg.k) < 1e-6
    inner = (inner_gap(r.probs, cfg.k) < 1e-6) & ~excluded
    exact = ~excluded & ~inner
    mism_exact = int(np.any(ids_gpu[exact] != r.ids[exact], axis=1).sum())
    mism_inner = int(np.any(np.sort(ids_gpu[inner], 1) != np.sort(r.ids[inner], 1), axis=1).sum())
    return {"tokens": int(cfg.T), "ids_mismatch": mism_exact + mism_inner, "excluded_near_tie": int(excluded.sum()),
            "inner_near_tie": int(inner.sum()),
            "rule": "ids bit-exact per slot; tokens with p_(k) - p_(k+1) < 1e-6 excluded; tokens with a "
                    "gap < 1e-6 between two selected slots compared as sets"}


# ------------------------------------------------------------- reference
def run_reference(args, cfg):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from top_routing_grouped_softmax_b200.synth import make_inputs
    inp = make_inputs(cfg.with_(seed=replica_seed(cfg.seed, 0)))
    n = args.ref_tokens
    for _ in range(args.warmup):
        time_oracle(cfg, n, cfg.seed, inp)
    secs = [time_oracle(cfg, n, cfg.seed, inp)[0] for _ in range(args.steps)]
    total = sum(secs)
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(cfg, extra={"tokens_per_step": n}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"first {n} of {cfg.T} tokens per step, full block, fp64, one thread",
                         **host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(cfg, extra=None):
    c = {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "f": cfg.f,
         "router_bias": "zipf" if cfg.skew else None, "weights_sigma": cfg.sigma,
         "inputs": "seeded synthetic (x ~ N(0,1), weights ~ N(0, sigma^2), bf16)",
         "l2": "flushed between timed steps (256 MiB write)", "parallelism": "replicas"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------- GPU
def run_gpu(args, cfg):
    import torch
    import torch.distributed as dist

    import top_routing_grouped_softmax_b200 as moe
    from top_routing_grouped_softmax_b200.synth import make_inputs

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    inp = make_inputs(cfg.with_(seed=replica_seed(cfg.seed, rank)))
    x = inp.x.to(dev)
    w = {n: getattr(inp, n).to(dev) for n in ("W_router", "W_gate", "W_up", "W_down")}
    bias = None if inp.bias is None else inp.bias.to(dev)
    blk = moe.MoEBlock(w["W_router"], w["W_gate"], w["W_up"], w["W_down"], cfg.k, bias=bias)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    if args.path == "stages":
        # the four ABI stages called one by one (x_perm materialised)
        st_ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
        st_w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
        st_h = torch.empty(cfg.T * cfg.k, cfg.f, dtype=torch.bfloat16, device=dev)
        st_y = torch.empty(cfg.T * cfg.k, cfg.d, dtype=torch.float16, device=dev)

        def step(events=None):
            def rec(i):
                if events and events[i] is not None:
                    events[i].record()
            rec(0)
            moe.route(x, w["W_router"], cfg.k, bias=bias, topk_ids=st_ids, topk_w=st_w)
            rec(1)
            pm = moe.permute(x, st_ids, st_w, cfg.E)
            rec(2)
            h_, y_ = moe.expert_ffn(pm["x_perm"], pm["w_perm"], pm["offsets"], w["W_gate"], w["W_up"],
                                    w["W_down"], h=st_h, y=st_y)
            rec(3)  # gate/up and down are not split on this path
            rec(4)
            moe.combine(y_, pm["inv"], cfg.T, cfg.k, out=out)
            rec(5)
            ids.copy_(st_ids)

        def fwd(xin, events=None, topk_ids=None):  # e2e leg: the public fused call
            blk(xin, out=out, topk_ids=topk_ids, events=events)
    else:
        flags = moe.MOE_FLAG_FUSED_GATHER if args.gather else 0
        if args.round > 0:
            ws_rd = None
            counts_rd = torch.empty(cfg.E, dtype=torch.int32, device=dev)

            def fwd(xin, events=None, topk_ids=None):
                nonlocal ws_rd
                if ws_rd is None:
                    nb = moe.lib().moe_workspace_size_rounded(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, args.round)
                    ws_rd = torch.empty(int(nb), dtype=torch.uint8, device=dev)
                moe.forward_rounded(xin, w["W_router"], w["W_gate"], w["W_up"], w["W_down"], cfg.k, tile=args.round,
                                    bias=bias, out=out, workspace=ws_rd, counts=counts_rd, events=events)
        elif args.shared > 0:
            from top_routing_grouped_softmax_b200.synth import make_shared_weights
            sw = {n: t.to(dev) for n, t in make_shared_weights(cfg, args.shared).items()}
            ws_sh = None

            def fwd(xin, events=None, topk_ids=None):
                nonlocal ws_sh
                if ws_sh is None:
                    nb = moe.lib().moe_workspace_size_shared(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, args.shared, cfg.f)
                    ws_sh = torch.empty(int(nb), dtype=torch.uint8, device=dev)
                moe.forward_shared(xin, w["W_router"], w["W_gate"], w["W_up"], w["W_down"], sw["W_gate_s"],
                                   sw["W_up_s"], sw["W_down_s"], cfg.k, bias=bias, out=out, workspace=ws_sh,
                                   topk_ids=topk_ids, events=events, flags=flags)
        else:
            def fwd(xin, events=None, topk_ids=None):
                blk(xin, out=out, topk_ids=topk_ids, events=events, flags=flags)

        def step(events=None):
            fwd(x, events, ids)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK

    # Timed region: per step, events at the step boundaries and around the
    # gate/up GEMM only (every recorded event stops the next kernel from
    # launching early, so the other stage boundaries are left open).
    n_ev = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    timed = [[e[0], None, e[2], e[3], None, e[5]] for e in evs]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            step(timed[i])
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    # Stage breakdown (diagnostic): the same steps again with every stage
    # boundary recorded.
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        step(sev[i])
    torch.cuda.synchronize()
    status = moe.get_status()
    assert status == moe.MOE_OK, moe.strerror(status)
    clocks = clk.summary()

    step_ms = [e[0].elapsed_time(e[n_ev - 1]) for e in evs]
    gateup_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    stage_ms = {s: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in sev) for i, s in enumerate(STAGES)}
    total_s = sum(step_ms) / 1e3

    # expert load statistics of the batch
    rounded_rows = None
    if args.round > 0:
        moe.route(x, w["W_router"], cfg.k, bias=bias, topk_ids=ids)   # top-k ids for the report (untimed)
        rounded_rows = int(counts_rd.sum().item())
    counts = torch.bincount(ids.flatten().long(), minlength=cfg.E).cpu()
    active = int((counts > 0).sum())
    # the grouped GEMMs run 256-row CTA-pair tiles: rows past a group's end
    # are computed and not stored
    gemm_counts = counts_rd.cpu() if args.round > 0 else counts
    tiles = int(((gemm_counts + 255) // 256).sum())
    padding = 1.0 - int(gemm_counts.sum()) / max(1, tiles * 256)

    # ---- end to end through the public API, host buffers, copies timed.
    # Consecutive batches are pipelined the way a serving loop runs them: the
    # host->device copy of batch i+1 and the device->host copy of batch i-1
    # run on their own streams while batch i computes (two device buffers of
    # each).  Every step still copies its whole token batch in and its whole
    # output back inside the timed region.
    x_host = inp.x.pin_memory()
    pipelined = args.path == "fused" and not (args.round or args.shared or args.gather)
    nbuf = 2 if pipelined else 1
    out_host = [torch.empty(cfg.T, cfg.d, dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    x_dev = [torch.empty_like(x) for _ in range(nbuf)]
    out_dev = [out] + [torch.empty_like(out) for _ in range(nbuf - 1)]
    s_in = torch.cuda.Stream(dev) if pipelined else stream
    s_out = torch.cuda.Stream(dev) if pipelined else stream
    # the same loop with the block's fp16-output option (MOE_FLAG_OUT_F16):
    # half the bytes read back
    out_host16 = [torch.empty(cfg.T, cfg.d, dtype=torch.float16).pin_memory() for _ in range(nbuf)]
    out_dev16 = [torch.empty(cfg.T, cfg.d, dtype=torch.float16, device=dev) for _ in range(nbuf)]

    def e2e_run(n_steps, t0=None, t1=None, f16=False):
        o_dev, o_host = (out_dev16, out_host16) if f16 else (out_dev, out_host)
        in_done = [torch.cuda.Event() for _ in range(nbuf)]
        comp_done = [torch.cuda.Event() for _ in range(nbuf)]
        out_done = [torch.cuda.Event() for _ in range(nbuf)]
        if t0 is not None:
            t0.record(stream)
            s_in.wait_event(t0)
        for i in range(n_steps):
            b = i % nbuf
            if i >= nbuf:
                s_in.wait_event(comp_done[b])        # x_dev[b] no longer read
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= nbuf:
                stream.wait_event(out_done[b])       # out_dev[b] copied out
            # no L2 flush here: each step copies a fresh batch in, and the
            # block's working set (its weights alone) is larger than L2
            if pipelined:
                blk(x_dev[b], out=o_dev[b], flags=moe.MOE_FLAG_OUT_F16 if f16 else None)
            else:
                fwd(x_dev[b])
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                o_host[b].copy_(o_dev[b], non_blocking=True)
                out_done[b].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        if t1 is not None:
            t1.record(stream)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_t0, e2e_t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, e2e_t0, e2e_t1)
    torch.cuda.synchronize()
    e2e_s = e2e_t0.elapsed_time(e2e_t1) / 1e3
    if world > 1:
        dist.barrier()
    e2e16_s = 0.0
    if pipelined:
        e2e_run(2, f16=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e2e_t0, e2e_t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(args.steps, e2e_t0, e2e_t1, f16=True)
        torch.cuda.synchronize()
        e2e16_s = e2e_t0.elapsed_time(e2e_t1) / 1e3
        if world > 1:
            dist.barrier()

    # max over ranks
    if world > 1:
        t = torch.tensor([total_s, e2e_s, gateup_ms, e2e16_s], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_s, e2e_s, gateup_ms_max, e2e16_s = t.tolist()
    else:
        gateup_ms_max = gateup_ms

    result = None
    if rank == 0:
        peaks = load_peaks()
        alg = algorithmic(cfg, active, args.shared)
        if rounded_rows is not None:
            # token rounding changes the number of (token, expert) rows the GEMMs compute
            scale = rounded_rows / (cfg.T * cfg.k)
            alg["gateup_flops"] = int(alg["gateup_flops"] * scale)
            alg["down_flops"] = int(alg["down_flops"] * scale)
            alg["flops"] = 2 * cfg.T * cfg.d * cfg.E + alg["gateup_flops"] + alg["down_flops"]
        ms = 1e3 * total_s / args.steps
        tok_s = whole_job_rate(cfg.T * args.steps, world, [total_s])
        # --path stages times both GEMMs together (moe_expert_ffn is one call)
        roof_flops = alg["gateup_flops"] + (alg["down_flops"] if args.path == "stages" else 0)
        achieved = roof_flops / (gateup_ms_max * 1e-3) / 1e12
        roof_time = max(alg["flops"] / (peaks["bf16_tflops"] * 1e12), alg["bytes"] / (peaks["hbm_gbs"] * 1e9))
        roof_ds = max(alg["flops"] / (DATASHEET["bf16_tflops"] * 1e12), alg["bytes"] / (DATASHEET["hbm_gbs"] * 1e9))
        traffic = None
        tpath = os.path.join(ROOT, "profiles", "gateup_traffic.json")
        if os.path.exists(tpath):
            with open(tpath) as fh:
                tr = json.load(fh)
            from top_routing_grouped_softmax_b200 import _build
            if tr.get("source_hash") == _build.kernel_hash() and tr.get("workload") == cfg.name:
                traffic = tr.get("dram_bytes_per_launch")
        result = {
            "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(cfg, extra={"out_dtype": "fp32",
                                                  **({"routing": f"token rounding to {args.round}-row tiles "
                                                                 "(an approximation of the block)",
                                                      "rounded_rows": rounded_rows} if args.round else {}),
                                                  **({"shared_experts": args.shared,
                                                                             "f_shared": cfg.f}
                                                                          if args.shared else {})}),
            "tflops": alg["flops"] / (ms * 1e-3) / 1e12,
            "grouped_gemm_tflops": (alg["gateup_flops"] + alg["down_flops"]) /
                                   ((stage_ms["gateup_gemm"] + stage_ms["down_gemm"]) * 1e-3) / 1e12,
            "grouped_gemm_tflops_padded": (alg["gateup_flops"] + alg["down_flops"]) / (1.0 - padding) /
                                          ((stage_ms["gateup_gemm"] + stage_ms["down_gemm"]) * 1e-3) / 1e12,
            "roofline": {"bound": "tensor",
                         "scope": "kernel: the dominant kernel alone (achieved, frac, traffic); "
                                  "the whole forward is in `forward`",
                         "kernel": ("grouped_gemm_pair_kernel<SwiGLU> (gate/up + SwiGLU)" if args.path == "fused"
                                    else "moe_expert_ffn (gate/up + down GEMMs)"),
                         "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                         "peak_source": f"{peaks['source']} burst bf16",
                         "forward": {"frac": roof_time / (ms * 1e-3), "roofline_ms": roof_time * 1e3,
                                     "ms_per_step": ms, "frac_of_datasheet": roof_ds / (ms * 1e-3),
                                     "bound": "max(FLOPs / bf16 peak, compulsory bytes / HBM peak)"}},
            "forward_roofline": {"roofline_ms": roof_time * 1e3, "frac": roof_time / (ms * 1e-3),
                                 "flops": alg["flops"], "compulsory_bytes": alg["bytes"],
                                 "peaks": ("of measured (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
                                           else "of fallback (no MEASURED_PEAKS.json: "
                                                f"{peaks['bf16_tflops']:.0f} TFLOP/s, {peaks['hbm_gbs']:.0f} GB/s)"),
                                 "frac_of_datasheet": roof_ds / (ms * 1e-3),
                                 "datasheet_peaks": "2250 TFLOP/s dense bf16, 8000 GB/s"},
            "stage_gbs": {st: alg["stage_bytes"][st] / (stage_ms[st] * 1e-3) / 1e9
                          for st in ("route", "permute", "combine")},
            "stage_ms": stage_ms,
            "stage_ms_note": "second pass of the same steps with every stage boundary recorded",
            "experts": {"active": active, "max_count": int(counts.max()), "min_count": int(counts.min()),
                        "pair_tile_padding": padding},
            "e2e": {"value": whole_job_rate(cfg.T * args.steps, world, [e2e_s]), "unit": UNIT,
                    "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 4,
                    "copies": ("pinned host buffers; batch i+1 in and batch i-1 out on their own streams while "
                               "batch i computes" if pipelined else "pinned host buffers, in order on one stream"),
                    "l2": E2E_L2},
            "e2e_f16out": ({"value": whole_job_rate(cfg.T * args.steps, world, [e2e16_s]), "unit": UNIT,
                            "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 2,
                            "out": "fp16: the fp32 sum rounded once (MOE_FLAG_OUT_F16); out16 == fp16(out32) bit "
                                   "for bit, within the out criteria of the oracle",
                            "copies": "as e2e", "l2": E2E_L2} if pipelined else None),
            "gpu_launches": (KERNELS_PER_FORWARD + 2 * args.shared + (3 if args.round else 0)) * args.steps,
            "clocks": clocks,
            "wall_s_timed_region": wall,
            "_topk_ids": ids.cpu().numpy(),
        }
    if world > 1:
        dist.destroy_process_group()
    return result


def time_workload(name, args, dev):
    """Time moe_forward on another of the workloads (fused path, N = 1) with
    the headline's rules -- inputs resident in HBM, L2 flushed between timed
    steps, CUDA events on the launching stream, NVML clocks sampled during
    the timed region -- and return its figures for the `workloads` object."""
    import torch

    import top_routing_grouped_softmax_b200 as moe
    from top_routing_grouped_softmax_b200.synth import CONFIGS, make_inputs

    cfg = CONFIGS[name]
    inp = make_inputs(cfg)
    x = inp.x.to(dev)
    w = {n: getattr(inp, n).to(dev) for n in ("W_router", "W_gate", "W_up", "W_down")}
    bias = None if inp.bias is None else inp.bias.to(dev)
    del inp
    blk = moe.MoEBlock(w["W_router"], w["W_gate"], w["W_up"], w["W_down"], cfg.k, bias=bias)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        blk(x, out=out, topk_ids=ids)
    torch.cuda.synchronize()
    n_ev = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            flush.zero_()
            e = evs[i]
            blk(x, out=out, topk_ids=ids, events=[e[0], None, e[2], e[3], None, e[5]])
        torch.cuda.synchronize()
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        blk(x, out=out, topk_ids=ids, events=sev[i])
    torch.cuda.synchronize()
    status = moe.get_status()
    assert status == moe.MOE_OK, moe.strerror(status)
    ms = statistics.mean(e[0].elapsed_time(e[n_ev - 1]) for e in evs)
    gateup_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    stage_ms = {s: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in sev) for i, s in enumerate(STAGES)}
    counts = torch.bincount(ids.flatten().long(), minlength=cfg.E).cpu()
    active = int((counts > 0).sum())
    tiles = int(((counts + 255) // 256).sum())
    peaks = load_peaks()
    alg = algorithmic(cfg, active)
    roof = max(alg["flops"] / (peaks["bf16_tflops"] * 1e12), alg["bytes"] / (peaks["hbm_gbs"] * 1e9))
    roof_ds = max(alg["flops"] / (DATASHEET["bf16_tflops"] * 1e12), alg["bytes"] / (DATASHEET["hbm_gbs"] * 1e9))
    gateup = alg["gateup_flops"] / (gateup_ms * 1e-3) / 1e12
    res = {
        "config": workload_config(cfg, extra={"out_dtype": "fp32"}),
        "ms_per_step": ms, "tokens_per_s": cfg.T / (ms * 1e-3), "steps": args.steps,
        "tflops": alg["flops"] / (ms * 1e-3) / 1e12,
        "forward_roofline": {"frac": roof / (ms * 1e-3), "roofline_ms": roof * 1e3,
                             "frac_of_datasheet": roof_ds / (ms * 1e-3)},
        "gateup": {"achieved_tflops": gateup, "frac": gateup / peaks["bf16_tflops"],
                   "peak_source": f"{peaks['source']} burst bf16"},
        "stage_ms": stage_ms,
        "experts": {"active": active, "max_count": int(counts.max()), "min_count": int(counts.min()),
                    "pair_tile_padding": 1.0 - int(counts.sum()) / max(1, tiles * 256)},
        "clocks": clk.summary(),
    }
    del blk, x, w, out, ids, flush
    torch.cuda.empty_cache()
    return res


def backward_flops(cfg):
    """FLOPs of one moe_backward: the recomputed gate/up GEMM, dh, dx_perm,
    the three expert weight gradients and the router's three T x d x E
    products (logits again, dW_router, dx_router)."""
    T, d, E, k, f = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f
    expert = 2 * T * k * d * f
    return 2 * expert + expert + 2 * expert + 2 * expert + expert + 3 * 2 * T * d * E


def run_backward(args, cfg):
    """Time moe_backward on one GPU (inputs resident, L2 flushed between
    steps, CUDA events on the launching stream) and print its JSON line."""
    import torch

    import top_routing_grouped_softmax_b200 as moe
    from top_routing_grouped_softmax_b200.synth import make_dout, make_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = make_inputs(cfg)
    x = inp.x.to(dev)
    w = {n: getattr(inp, n).to(dev) for n in ("W_router", "W_gate", "W_up", "W_down")}
    bias = None if inp.bias is None else inp.bias.to(dev)
    dout = make_dout(cfg.T, cfg.d, cfg.seed).to(dev)
    ws = torch.empty(moe.backward_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(grad_dtype=torch.float32):
        return moe.backward(x, w["W_router"], w["W_gate"], w["W_up"], w["W_down"], cfg.k, dout, bias=bias,
                            workspace=ws, grad_dtype=grad_dtype)

    def timed(grad_dtype):
        for _ in range(max(args.warmup, 3)):
            step(grad_dtype)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        with ClockSampler(0) as clk:
            for a, b in evs:
                flush.zero_()
                a.record()
                step(grad_dtype)
                b.record()
            torch.cuda.synchronize()
        status = moe.get_status()
        assert status == moe.MOE_OK, moe.strerror(status)
        return statistics.mean(a.elapsed_time(b) for a, b in evs), clk

    ms, clk = timed(torch.float32)
    ms16, clk16 = timed(torch.bfloat16)
    peaks = load_peaks()
    flops = backward_flops(cfg)
    tflops = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": "MoE-layer bwd tokens/s & TFLOP/s vs roofline, 1xB200", "value": cfg.T / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(cfg, extra={"pass": "backward (activations recomputed)", "grads_dtype": "fp32"}),
        "roofline": {"bound": "tensor", "scope": "the whole backward", "achieved": tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
                     "traffic": None, "flops": flops, "peak_source": f"{peaks['source']} burst bf16"},
        "gpu_launches": 17 * args.steps,  # 6 routing and grouping, 7 GEMMs, router step, bias sum, router-gradient sum, combine
        "clocks": clk.summary(),
        "bf16_weight_grads": {"ms_per_step": ms16, "value": cfg.T / (ms16 * 1e-3), "unit": "tokens/s",
                              "grads": "MOE_FLAG_GRAD_BF16: the four weight gradients bf16 (the fp32 results "
                                       "rounded once), dx and dbias fp32; timed by the same rules",
                              "clocks": clk16.summary()},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="qwen")
    ap.add_argument("--path", choices=("fused", "stages"), default="fused",
                    help="fused: moe_forward; stages: moe_route/permute/expert_ffn/combine one by one")
    ap.add_argument("--round", type=int, default=0,
                    help="token rounding to this tile (e.g. 256): an approximation of the block, reported apart")
    ap.add_argument("--shared", type=int, default=0,
                    help="add this many shared experts (weight one, every token, intermediate size f)")
    ap.add_argument("--gather", action="store_true",
                    help="fused path: the gate/up GEMM gathers x rows itself (MOE_FLAG_FUSED_GATHER)")
    ap.add_argument("--cpu-tokens", type=int, default=384,
                    help="tokens of the workload the CPU-oracle baseline leg evaluates")
    ap.add_argument("--ref-tokens", type=int, default=32, help="tokens per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time moe_backward (gradients of the block, activations recomputed) on one GPU instead")
    ap.add_argument("--workloads", default="coarse,fine,skew",
                    help="other workloads to time at N=1 (fused path) into the line's `workloads` object; "
                         "empty to skip")
    args = ap.parse_args(argv)

    from top_routing_grouped_softmax_b200.synth import CONFIGS
    cfg = CONFIGS[args.workload]
    if args.impl == "reference":
        return run_reference(args, cfg)

    from top_routing_grouped_softmax_b200 import _build
    _build.build_library()
    if args.backward:
        return run_backward(args, cfg)
    res = run_gpu(args, cfg)
    rank, _, world = dist_env()
    if rank == 0 and res is not None:
        ids_gpu = res.pop("_topk_ids", None)
        extra = [n for n in args.workloads.split(",") if n and n != cfg.name]
        if world == 1 and extra and args.path == "fused" and not (args.round or args.shared or args.gather):
            import torch
            dev = torch.device("cuda", torch.cuda.current_device())
            wl = {n: time_workload(n, args, dev) for n in extra}
            res["workloads"] = wl
            res["roofline"]["forward_by_workload"] = {
                cfg.name: res["roofline"]["forward"]["frac"], **{n: v["forward_roofline"]["frac"] for n, v in wl.items()}}
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(cfg, args.cpu_tokens, replica_seed(cfg.seed, 0))
            if ids_gpu is not None and not args.round:
                res["cpu_baseline"]["route_parity"] = route_parity(cfg, ids_gpu, replica_seed(cfg.seed, 0))
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
