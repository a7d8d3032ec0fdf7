"""GPTQ layer quantization throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--config q_proj] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the whole hot path over one layer: Hessian
accumulation over all calibration tokens, inverse factor (dead columns,
damping, act-order if set), lazy-blocked sweep with the layer loss, pack and
dequant.  The default workload is the Llama-7B-shaped q_proj layer: W 4096 x
4096 fp16, X 262144 x 4096 fp16 (2.15 GB, larger than L2, so no flush is
needed between steps), int4 asymmetric, group 128, block 128, damp 0.01.

value  = weights quantized per second over all ranks (Mweights/s), inputs
         resident in HBM, device time (CUDA events), max over ranks.
e2e    = the same metric through the host-buffer API (pinned X and W copied in,
         packed result and loss copied out, inside the timed region).
N > 1  = weak scaling: every rank quantizes its own independent layer (a
         different seed); no collective is on the data path.  --mode sharded
         instead splits ONE layer over the ranks (tokens for H + all-reduce,
         rows for the sweep + all-gather): strong scaling.
other_configs = the other layer shapes (down_proj 4096 x 11008 act-order, the
         OPT-175B-width 12288 x 12288 3-bit layer, one decoder layer of the 7B
         stack), per phase, inputs drawn on the device (N = 1 only).
--impl reference runs the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only) and prints the same line with "impl": "reference".
"""

from __future__ import annotations

import argparse
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

import synth  # noqa: E402

METRIC = "GPTQ layer quantize Mweights/s end-to-end"
UNIT = "Mweights/s"


# DRAM traffic of hessian_tc_kernel per calibration token, by k, from ncu
# captures (dram__bytes_read.sum + dram__bytes_write.sum of one launch on a
# smaller token count, scaled by tokens to a full launch: an estimate).  Only
# the widths a capture exists for; the line reports null elsewhere.
HESS_TRAFFIC = {
    # per token: ncu dram__bytes_read.sum + dram__bytes_write.sum of one hessian_tc_kernel
    # launch on 32768 tokens of the config's width, divided by 32768
    4096: ((602.87e6 + 72.25e6) / 32768,
           "estimate: ncu dram bytes of hessian_tc_kernel on a 32768 x 4096 capture, scaled by "
           "tokens (profiles/hessian_tc_kernel_dram_by_width.md)"),
    11008: ((6971.02e6 + 249.56e6) / 32768,
            "estimate: ncu dram bytes of hessian_tc_kernel on a 32768 x 11008 capture, scaled by "
            "tokens (profiles/hessian_tc_kernel_dram_by_width.md)"),
    12288: ((8592.74e6 + 311.70e6) / 32768,
            "estimate: ncu dram bytes of hessian_tc_kernel on a 32768 x 12288 capture, scaled by "
            "tokens (profiles/hessian_tc_kernel_dram_by_width.md)"),
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi every 25 ms while
    the timed region runs (all GPUs are queried; the one on this process's
    PCI bus is kept, or the only one)."""
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.first = ""
        self.bus = None
        try:
            self.bus = str(torch.cuda.get_device_properties(device_index).pci_bus_id).lower()
        except Exception:
            pass

    def start(self):
        """Start sampling; returns once the first sample is in."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "25"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.first = self.proc.stdout.readline()
        except Exception:
            self.proc = None

    def _mine(self, bus_field, n_lines_seen):
        if self.bus is None:
            return True
        a = bus_field.lower().split(":", 1)[-1]
        b = self.bus.split(":", 1)[-1]
        return a == b

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        out = (self.first or "") + (out or "")
        rows = [[x.strip() for x in line.split(",")] for line in out.strip().splitlines()]
        rows = [f for f in rows if len(f) >= 9]
        buses = {f[0] for f in rows}
        if len(buses) > 1:
            rows = [f for f in rows if self._mine(f[0], 0)]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for f in rows:
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- oracle timing

def oracle_sample(spec, seed, n_tokens, n_rows):
    """Time the fp64 oracle on a bounded sample of the workload and
    extrapolate to the whole layer: Hessian over ``n_tokens`` tokens (scaled by
    n / n_tokens), the inverse factor at full k, the sweep, pack and dequant
    over ``n_rows`` rows (scaled by r / n_rows)."""
    import oracle as O
    X = synth.make_x(spec, seed, t0=0, t1=n_tokens)
    W = synth.make_w(spec, seed)[:n_rows]
    Xn = X.float().numpy() if X.dtype == torch.bfloat16 else X.numpy()
    Wn = W.float().numpy() if W.dtype == torch.bfloat16 else W.numpy()
    t0 = time.perf_counter()
    H = O.hessian(Xn, n_total=n_tokens)
    t1 = time.perf_counter()
    Hf, Wf, dead = O.fix_dead_columns(H, Wn)
    perm = O.act_order_perm(Hf) if spec.act_order else np.arange(spec.k)
    Hd = O.damp(Hf[np.ix_(perm, perm)], spec.percdamp)
    U = O.hinv_upper_factor(Hd)
    t2 = time.perf_counter()
    G = spec.k if spec.group_size == -1 else spec.group_size
    static = None
    if spec.static_groups:
        ss, zz = O.static_grids(Wf, spec.bits, spec.group_size, sym=spec.sym)
        static = (ss, zz, perm // G)
    res = O.sweep_blocked(Wf[:, perm], U, spec.bits, spec.group_size, spec.block_size,
                          sym=spec.sym, static=static)
    codes = np.zeros_like(res["codes"], dtype=np.int64)
    codes[:, perm] = res["codes"]
    qhat = np.zeros_like(res["qhat"])
    qhat[:, perm] = res["qhat"]
    O.layer_loss(Wn, qhat, H)
    t3 = time.perf_counter()
    if spec.static_groups:
        g_idx = np.arange(spec.k, dtype=np.int64) // G
    else:
        g_idx = np.zeros(spec.k, dtype=np.int64)
        g_idx[perm] = np.arange(spec.k) // G
    qw = O.pack(codes, spec.bits)
    O.dequant(O.unpack(qw, spec.k, spec.bits), res["scales"], res["zeros"], g_idx, np.float16)
    t4 = time.perf_counter()
    t_full = ((t1 - t0) * spec.n / n_tokens + (t2 - t1) + (t3 - t2) * spec.r / n_rows
              + (t4 - t3) * spec.r / n_rows)
    sample = (f"Hessian over {n_tokens} of {spec.n} tokens (x{spec.n / n_tokens:g}); inverse "
              f"factor at full k={spec.k}; sweep+loss, pack, dequant over {n_rows} of {spec.r} rows "
              f"(x{spec.r / n_rows:g}); phases {t1 - t0:.2f}/{t2 - t1:.2f}/{t3 - t2:.2f}/"
              f"{t4 - t3:.2f} s")
    return t_full, t4 - t0, sample


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def reference_arm(args, spec, world, rank):
    if rank != 0:
        return 0
    n_tok, n_rows = args.ref_tokens, args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(spec, args.seed, n_tok, n_rows)
    ts, wall, sample = [], 0.0, ""
    for _ in range(args.steps):
        t_full, w, sample = oracle_sample(spec, args.seed, n_tok, n_rows)
        ts.append(t_full)
        wall += w
    t = statistics.median(ts)
    value = spec.r * spec.k / t / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(spec),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(spec):
    G = "per-row" if spec.group_size == -1 else f"g{spec.group_size}"
    return {
        "workload": (f"{spec.name}: W {spec.r}x{spec.k} {spec.w_dtype}, X {spec.n}x{spec.k} "
                     f"{spec.x_dtype} ({spec.x_kind}), int{spec.bits} "
                     f"{'sym' if spec.sym else 'asym'} {G} B{spec.block_size} "
                     f"damp {spec.percdamp}{' act-order' if spec.act_order else ''}"
                     f"{' static-groups' if spec.static_groups else ''}"),
        "l2": f"inputs larger than L2 (X {spec.n * spec.k * 2 / 1e9:.2f} GB), no flush",
    }


# --------------------------------------------------------------------------- native arm

def _cfg_of(spec):
    from post_weight_quantization_23_b200 import QuantConfig
    return QuantConfig(spec.bits, spec.group_size, spec.block_size, spec.percdamp, spec.act_order,
                       spec.sym, spec.static_groups)


class LayerRun:
    """One layer's plan and its device-resident inputs; ``step`` issues the
    whole hot path (H reset, Hessian over all tokens, factor, sweep with the
    loss, pack, dequant)."""

    PHASES = ("hessian", "prepare", "quantize", "pack", "dequant")

    def __init__(self, spec, Xd, Wd, dev):
        from post_weight_quantization_23_b200 import GptqPlan
        self.spec, self.Xd, self.Wd, self.dev = spec, Xd, Wd, dev
        self.plan = GptqPlan(spec.r, spec.k, _cfg_of(spec), dev, want_loss=True,
                             deq_dtype=torch.float16, hessian_tokens_hint=spec.n)

    def lib_calls(self):
        p = self.plan
        p.hessian_add(self.Xd, self.spec.n)
        p.prepare()
        p.quantize(self.Wd)
        p.pack()
        p.dequant()

    def step(self):
        p = self.plan
        p.hessian_reset()
        p.hessian_add(self.Xd, self.spec.n)
        p.prepare()
        p.quantize(self.Wd)
        p.pack()
        p.dequant()

    def phase_ms(self, reps):
        """Per-phase device times inside the step: the whole step captured as
        one CUDA graph with timing events between the phases (external event
        nodes), replayed reps times; mean of the replays.  Host launch cost
        stays out (the eager form is host-bound for the factor's ~3 launches
        per 64 columns at the wide layers), and every phase runs in the step's
        own order and clocks."""
        p = self.plan
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]

        def body():
            ev[0].record()
            p.hessian_reset()
            p.hessian_add(self.Xd, self.spec.n)
            for i, fn in enumerate((p.prepare, lambda: p.quantize(self.Wd), p.pack, p.dequant)):
                ev[i + 1].record()
                fn()
            ev[5].record()

        g = p.capture(body)
        acc = np.zeros(5)
        for _ in range(reps):
            g.replay()
            torch.cuda.synchronize(self.dev)
            acc += [ev[i].elapsed_time(ev[i + 1]) for i in range(5)]
        del g
        return acc / reps

def timed_replays(graph, steps, dev, stream):
    """Device ms per replay of ``graph`` over ``steps`` back-to-back replays."""
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for _ in range(steps):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1) / steps


def measured_rates():
    """fp32-FMA and kind::tf32 peak rates of this device (gptq_measure_peaks),
    the denominators of the inverse factor's and the updates' fractions."""
    from post_weight_quantization_23_b200 import _lib
    try:
        r = _lib.measure_peaks()
    except Exception as e:  # report, do not fail the bench over a calibration
        return {"error": repr(e)}
    r["how"] = ("gptq_measure_peaks: packed fp32x2 FMA chains on every SM; kind::tf32 "
                "128x256x8 MMAs back to back, one issuing thread per SM; one timed launch each")
    return r


def phase_figures(spec, phase, peaks, rates=None):
    """Absolute and roofline figures of one layer's per-phase times (ms)."""
    flops = float(spec.n) * spec.k * (spec.k + 1)  # symmetric triangle, algorithmic
    t_h = phase[0] / 1e3
    sweep_bytes = sweep_model_bytes(spec)
    hess = flops / t_h / 1e12
    out = {
        "hessian_ms": phase[0], "prepare_ms": phase[1], "quantize_ms": phase[2],
        "pack_ms": phase[3], "dequant_ms": phase[4],
        "hessian_tflops": hess,
        "hessian_frac_bf16_burst": hess / peaks["bf16"],
        "hessian_frac_bf16_sustained": hess / peaks["bf16_sustained"],
        "hessian_issued_tflops": hessian_issued_flop(spec) / t_h / 1e12,
        "prepare_tflops_algorithmic": (2.0 / 3.0) * float(spec.k) ** 3 / (phase[1] / 1e3) / 1e12,
        "hessian_x_gbs": spec.n * spec.k * 2 / t_h / 1e9,
        "sweep_model_bytes": sweep_bytes,
        "sweep_model_gbs": sweep_bytes / (phase[2] / 1e3) / 1e9,
        "sweep_frac_hbm": sweep_bytes / (phase[2] / 1e3) / 1e9 / peaks["hbm"],
    }
    if spec.k in HESS_TRAFFIC:
        per_tok, src = HESS_TRAFFIC[spec.k]
        out["hessian_traffic_bytes"] = per_tok * spec.n
        out["hessian_traffic_source"] = src
        out["hessian_traffic_over_x"] = per_tok * spec.n / (spec.n * spec.k * 2.0)
    if rates and "tf32_tflops" in rates:
        # the factor's rank updates issue 3 kind::tf32 MMAs per useful product
        out["prepare_frac_tf32_issued"] = (3.0 * out["prepare_tflops_algorithmic"]
                                           / rates["tf32_tflops"])
    return out


def other_configs(dev, stream, peaks, seed, steps, names, rates=None):
    """The other layer shapes of the pages (down_proj, the OPT-175B-width
    layer, one decoder layer of the 7B stack), each measured alone with inputs
    drawn on the device (same distributions as the CPU generator; timing
    only): per-phase device times, Mweights/s over one CUDA graph per step."""
    out = {}
    for name in names:
        subs = ([n for n in synth.CONFIGS if n.startswith("stack_")] if name == "stack_layer"
                else [name])
        runs = []
        for sub in subs:
            spec = synth.CONFIGS[sub]
            runs.append(LayerRun(spec, synth.make_x_device(spec, seed, dev),
                                 synth.make_w_device(spec, seed, dev), dev))
        for run in runs:
            for _ in range(2):
                run.step()
            run.plan.check()
        entry = {}
        for run in runs:
            ph = run.phase_ms(3)
            entry[run.spec.name] = {"workload": workload_config(run.spec)["workload"],
                                    **phase_figures(run.spec, ph, peaks, rates)}
        graph = runs[0].plan.capture(lambda: [r.step() for r in runs])
        ms = timed_replays(graph, steps, dev, stream)
        for run in runs:
            run.plan.check()
        weights = sum(r.spec.r * r.spec.k for r in runs)
        out[name] = {"value": weights / (ms / 1e3) / 1e6, "unit": UNIT, "ms_per_step": ms,
                     "steps": steps, "layers": entry,
                     "data": "synthetic, drawn on the device (same distributions)"}
        if name == "stack_layer":
            out[name]["note"] = ("one decoder layer of the 32-layer 7B-shaped stack (qkv and "
                                 "gate/up stacked on their shared Hessians); the 32 layers are "
                                 "identical in shape and independent")
        del graph, runs
        torch.cuda.empty_cache()
    return out


def native_arm(args, spec, world, rank, local):
    from post_weight_quantization_23_b200.api import HostPipeline

    dev = torch.device("cuda", local if world > 1 else 0)
    seed = args.seed + rank  # independent layer per rank (weak scaling)
    xdt = synth.dtype_of(spec.x_dtype)
    X_host = torch.empty(spec.n, spec.k, dtype=xdt, pin_memory=True)
    synth.make_x(spec, seed, out=X_host)
    W_host = synth.make_w(spec, seed).pin_memory()
    run = LayerRun(spec, X_host.to(dev), W_host.to(dev), dev)
    plan = run.plan
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        run.step()
    plan.check()
    phase = run.phase_ms(max(2, min(args.steps, 5)))

    launches = count_launches(run.lib_calls, dev)  # the H reset is a torch fill, not ours
    plan.check()
    graph = plan.capture(run.step)  # the timed steps replay one CUDA graph per step

    clocks = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    ms = timed_replays(graph, args.steps, dev, stream)
    barrier(world)
    clk = clocks.stop()
    plan.check()
    ms = max_over_ranks(ms, world)
    value = world * spec.r * spec.k / (ms / 1e3) / 1e6

    e2e = None
    if not args.no_e2e:
        pipe = HostPipeline(plan, args.e2e_chunk, xdt, W_host.dtype)
        for _ in range(2):
            pipe.run(X_host, W_host)
            pipe.wait()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        k_e2e = max(1, min(args.steps, args.e2e_steps))
        barrier(world)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(k_e2e):
            pipe.run(X_host, W_host)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        pipe.wait()
        barrier(world)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / k_e2e, world)
        e2e = {"value": world * spec.r * spec.k / (ms_e2e / 1e3) / 1e6, "unit": UNIT,
               "ms_per_step": ms_e2e, "steps": k_e2e,
               "h2d_bytes_per_step": pipe.h2d_bytes(X_host, W_host),
               "d2h_bytes_per_step": pipe.d2h_bytes()}

    peaks = _peaks()
    rates = measured_rates()
    phases = phase_figures(spec, phase, peaks, rates)
    flops = float(spec.n) * spec.k * (spec.k + 1)
    traffic, tsrc = None, None
    if args.traffic is not None:
        traffic, tsrc = args.traffic, "given on the command line (ncu capture of this workload)"
    elif spec.k in HESS_TRAFFIC:
        per_tok, src = HESS_TRAFFIC[spec.k]
        traffic, tsrc = per_tok * spec.n, src
    roofline = {"bound": "tensor", "kernel": "gptq_hessian_accumulate (X^T X)",
                "achieved": phases["hessian_tflops"], "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": phases["hessian_tflops"] / peaks["bf16"], "traffic": traffic,
                "traffic_source": tsrc,
                "peak_kind": (f"bf16 dense burst ({peaks['source']}); f16 has the same nominal "
                              f"rate"),
                "frac_of_sustained": phases["hessian_tflops"] / peaks["bf16_sustained"],
                "algorithmic": f"n*k*(k+1) = {flops:.4g} flop per launch"}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": dict(workload_config(spec), parallelism=f"{world} independent layers",
                       launch="one CUDA graph per step (library calls captured once)"),
        "roofline": roofline, "phases": phases,
        "gpu_launches": launches * args.steps if launches is not None else None,
        "gpu_launches_per_step": launches, "clocks": clk, "e2e": e2e, "measured_rates": rates,
    }
    del graph
    if not args.no_other_configs and world == 1:
        names = [n for n in ("down_proj", "opt175_width", "stack_layer") if n != spec.name]
        line["other_configs"] = other_configs(dev, stream, peaks, seed, args.other_steps, names,
                                              rates)
    if not args.no_qgemm:
        line["inference_matmul"] = qgemm_measure(dev, stream, peaks, args.seed + rank)
    if not args.no_rotation:
        line["rotation"] = rotation_measure(run.Xd, dev, stream, peaks, args.seed + rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_full, wall, sample = oracle_sample(spec, args.seed, args.ref_tokens, args.ref_rows)
        line["cpu_baseline"] = {"value": spec.r * spec.k / t_full / 1e6, "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": sample + f"; wall {wall:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def sharded_arm(args, spec, world, rank, local):
    """One layer split over the ranks (strong scaling): each rank accumulates
    the Hessian of its share of the tokens, one all-reduce sums H, every rank
    computes the factor, each sweeps its block of rows, and the codes,
    scales, zeros and per-row losses are all-gathered.  Eager launches (the
    collectives are not captured); device time, max over ranks."""
    from post_weight_quantization_23_b200.sharded import ShardedLayer

    dev = torch.device("cuda", local if world > 1 else 0)
    own_group = False
    if not torch.distributed.is_initialized():  # N = 1: a one-rank group
        import datetime
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        torch.distributed.init_process_group(
            "nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
            timeout=datetime.timedelta(seconds=300), device_id=dev)
        own_group = True
    group = torch.distributed.group.WORLD
    layer = ShardedLayer(spec.r, spec.k, _cfg_of(spec), dev, group=group, want_loss=True,
                         deq_dtype=None, hessian_tokens_hint=spec.n)
    t0, t1 = layer.token_range(spec.n)
    X_all = synth.make_x_device(spec, args.seed, dev)
    X_local = X_all[t0:t1].contiguous()
    del X_all
    W = synth.make_w_device(spec, args.seed, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.plan.hessian_reset()
        return layer.run(X_local, spec.n, W)

    for _ in range(args.warmup):
        step()
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    line = {
        "metric": METRIC, "value": spec.r * spec.k / (ms / 1e3) / 1e6, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic, drawn on the device",
        "config": dict(workload_config(spec), parallelism=(
            f"one layer over {world} ranks: tokens sharded for H + all-reduce, factor "
            f"replicated, rows sharded for the sweep + all-gather"),
            launch="eager (collectives between the library calls)"),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if own_group:
        torch.distributed.destroy_process_group()
    return 0


# Linear layers of one Llama-2-7B-shaped block, (out-features n, in-features k)
QG_BLOCK = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
QG_BLOCKS = 4  # 4 blocks: 405 MB of int4 weights, more than L2


def qgemm_measure(dev, stream, peaks, seed, bits=4, G=128, reps=20):
    """The inference product (gptq_gemm) on one decode token (m = 1) through
    the linear layers of QG_BLOCKS blocks of a 7B-shaped model, int4 g128,
    synthetic packed weights resident in HBM; the 28 calls are one CUDA
    graph, timed with events.  Algorithmic bytes: packed weights + fp32 scales
    + int32 zeros + X + Y of every layer.  Also m = 16 (a small batch) and
    m = 2048 (prefill, the tensor-core kernel, against the dense bf16 peak;
    f16 has the same nominal rate)."""
    from post_weight_quantization_23_b200 import quant_matmul
    g = torch.Generator(device=dev).manual_seed(seed)
    layers = []
    for _ in range(QG_BLOCKS):
        for n, k in QG_BLOCK:
            ng = k // G
            qw = torch.randint(-2 ** 31, 2 ** 31 - 1, (n, k * bits // 32), generator=g,
                               dtype=torch.int32, device=dev)
            sc = torch.rand(n, ng, generator=g, device=dev) * 0.01 + 1e-3
            z = torch.randint(0, 2 ** bits, (n, ng), generator=g, dtype=torch.int32, device=dev)
            layers.append((n, k, qw, sc, z))
    out = {"workload": (f"one token through the linear layers of {QG_BLOCKS} Llama-2-7B-shaped "
                        f"blocks ({len(layers)} layers: 4x 4096x4096, 2x 11008x4096, "
                        f"1x 4096x11008 per block), int{bits} g{G}, f16 activations"),
           "l2": "weights larger than L2, each layer read once per pass", "bound": "hbm",
           "peak": peaks["hbm"], "unit": "GB/s", "kernel": "qgemv_kernel (gptq_gemm)",
           "m16_kernel": "qgemm_mma_kernel (mma.sync m16n8k16, weights formed in f16)",
           "m2048_kernel": "qgemm_tc_kernel (tcgen05)"}
    for m in (1, 16, 2048):
        xs = [torch.randn(m, k, generator=g, device=dev).half() for (_, k, *_r) in layers]
        ys = [torch.empty(m, n, dtype=torch.float16, device=dev) for (n, *_r) in layers]

        def run():
            for (n, k, qw, sc, z), x, y in zip(layers, xs, ys):
                quant_matmul(x, qw, sc, z, bits, G, None, y)

        for _ in range(3):
            run()
        torch.cuda.synchronize(dev)
        s2 = torch.cuda.Stream(dev)
        s2.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s2):
            run()
        torch.cuda.synchronize(dev)
        for _ in range(3):
            graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / reps
        nbytes = sum(n * k * bits // 8 + n * (k // G) * 8 + m * k * 2 + m * n * 2
                     for (n, k, *_r) in layers)
        gbs = nbytes / (us / 1e6) / 1e9
        tag = f"m{m}"
        out[f"{tag}_us_per_pass"] = us
        if m >= 17:  # the tensor-core kernel: bound by the multiply
            flop = 2.0 * m * sum(n * k for (n, k, *_r) in layers)
            out[f"{tag}_tflops"] = flop / (us / 1e6) / 1e12
            out[f"{tag}_frac_of_bf16_dense"] = out[f"{tag}_tflops"] / peaks["bf16"]
        else:
            out[f"{tag}_bytes_per_pass"] = nbytes
            out[f"{tag}_achieved_gbs"] = gbs
            out[f"{tag}_frac"] = gbs / peaks["hbm"]
        del graph, xs, ys
    out["achieved"] = out["m1_achieved_gbs"]
    out["frac"] = out["m1_frac"]
    out["launches_per_pass"] = len(layers)
    return out


def rotation_measure(Xd, dev, stream, peaks, seed, reps=10):
    """Rotation preprocessing (gptq_rotate) of the whole calibration matrix X
    (n x k, resident in HBM) into a second buffer: algorithmic bytes = X read
    + X written + the signs, per launch; events around `reps` launches (each
    launch streams 2 x |X|, more than L2)."""
    from post_weight_quantization_23_b200 import hadamard_block, rotate, rotation_signs
    n, k = Xd.shape
    block = hadamard_block(k)
    if block == 0:
        return None
    signs = rotation_signs(k, seed, dev)
    out = torch.empty_like(Xd)
    for _ in range(3):
        rotate(Xd, signs, block, out=out)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(reps):
        rotate(Xd, signs, block, out=out)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / reps
    nbytes = 2 * Xd.numel() * Xd.element_size() + k
    gbs = nbytes / (us / 1e6) / 1e9
    del out
    return {"workload": f"X {n}x{k} {str(Xd.dtype)[6:]} rotated by diag(s) H_{block} / sqrt({block})",
            "kernel": "rotate_kernel (gptq_rotate)", "bound": "hbm", "us_per_launch": us,
            "bytes_per_launch": nbytes, "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
            "frac": gbs / peaks["hbm"]}


def hessian_issued_flop(spec, tm=128, tn=256):
    """Flops the Hessian kernel issues: 2 n tm tn per tile of tm x tn that
    reaches the upper triangle (f16/bf16 path; the algorithmic count is
    n k (k + 1))."""
    ntm, ntn = -(-spec.k // tm), -(-spec.k // tn)
    tiles = sum(1 for i in range(ntm) for j in range(ntn) if (j + 1) * tn > i * tm)
    return 2.0 * spec.n * tiles * tm * tn


def sweep_model_bytes(spec):
    """Algorithmic bytes of the lazy-blocked sweep: per block the trailing fp32
    slice of W in and out (8 r (k-e)), the U panel (4 B (k-e)), plus the W
    read (input dtype), the fp32 working copy in and out, the error block, and
    the codes written."""
    r, k, B = spec.r, spec.k, spec.block_size
    nb = -(-k // B)
    sigma = sum(k - min((b + 1) * B, k) for b in range(nb))
    wbytes = 2 if spec.w_dtype in ("f16", "bf16") else 4
    return 8 * r * sigma + 4 * B * sigma + 16 * r * k + r * k + wbytes * r * k


def count_launches(step, dev):
    """Kernel launches of one step, counted from a CUDA-graph capture of it."""
    try:
        from cuda.bindings import runtime as cudart
    except Exception:
        try:
            from cuda import cudart  # type: ignore
        except Exception:
            return None
    try:
        g = torch.cuda.CUDAGraph(keep_graph=True)
    except TypeError:
        g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        g.capture_begin()
        step()
        g.capture_end()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    try:
        raw = g.raw_cuda_graph()
        handle = raw if isinstance(raw, cudart.cudaGraph_t) else cudart.cudaGraph_t(int(raw))
        err, nodes, num = cudart.cudaGraphGetNodes(handle, 0)
        err, nodes, num = cudart.cudaGraphGetNodes(handle, num)
        n = 0
        for nd in nodes:
            err, ty = cudart.cudaGraphNodeGetType(nd)
            if ty == cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                n += 1
        return n
    except Exception as e:  # report, but do not fail the bench over the count
        print(f"launch count unavailable: {e!r}", file=sys.stderr)
        return None
    finally:
        del g


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", default="q_proj", choices=sorted(synth.CONFIGS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-chunk", type=int, default=32768)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-tokens", type=int, default=8192)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the calibration token count (smaller cases for profiling)")
    ap.add_argument("--rows", type=int, default=None, help="override the row count of W")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per Hessian launch from an ncu capture of this kernel")
    ap.add_argument("--no-qgemm", action="store_true",
                    help="skip the inference-product measurement")
    ap.add_argument("--no-rotation", action="store_true",
                    help="skip the rotation-preprocessing measurement")
    ap.add_argument("--only", choices=["inference", "rotation", "peaks"], default=None,
                    help="run one side measurement alone (a short command for profiling)")
    ap.add_argument("--act-order", action="store_true", help="variant: act-order")
    ap.add_argument("--sym", action="store_true", help="variant: symmetric grid")
    ap.add_argument("--static-groups", action="store_true", help="variant: static groups")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the down_proj / OPT-175B-width / stack-layer measurements")
    ap.add_argument("--other-steps", type=int, default=5,
                    help="timed steps of each other config")
    ap.add_argument("--mode", choices=["layers", "sharded"], default="layers",
                    help="layers: every rank its own layer (weak scaling); sharded: one layer "
                         "split over the ranks (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    spec = synth.CONFIGS[args.config]
    if args.tokens or args.rows:
        spec = spec.scaled(r=args.rows, n=args.tokens)
    if args.act_order or args.sym or args.static_groups:
        spec = spec.scaled(act_order=spec.act_order or args.act_order, sym=args.sym,
                           static_groups=args.static_groups)
    if args.impl == "reference":
        # CPU only: rank 0 runs the oracle, other ranks exit without work
        return reference_arm(args, spec, int(os.environ.get("WORLD_SIZE", "1")),
                             int(os.environ.get("RANK", "0")))
    if args.only is not None:
        dev = torch.device("cuda", 0)
        stream = torch.cuda.current_stream(dev)
        if args.only == "inference":
            out = qgemm_measure(dev, stream, _peaks(), args.seed, reps=args.steps)
        elif args.only == "peaks":
            out = measured_rates()
        else:
            X = synth.make_x(spec, args.seed).to(dev)
            out = rotation_measure(X, dev, stream, _peaks(), args.seed)
        print(json.dumps({"only": args.only, **out}), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    try:
        if args.mode == "sharded":
            return sharded_arm(args, spec, world, rank, local)
        return native_arm(args, spec, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
