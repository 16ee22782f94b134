"""Benchmark of the VQ-MoE hot path on B200 (one JSON line on rank 0).

Default workload (the headline): the MoE decode layer with d=4/K=512 (9-bit
codes) in all three projections, 256 experts top-8, hidden 6144, inter 2048, 16
tokens per step. A step is one vq_moe_decode call: routing and bucketing, the
gate/up grouped VQ GEMV, SwiGLU, the down grouped VQ GEMV and the weighted
combine, over one batch of seeded synthetic inputs rotated among 16 routing
draws (3.0 GB of expert weights, far beyond L2, so a step's experts are not
L2-resident from the previous step).

metric: decode HBM GB/s = algorithmic bytes of a step (live codes and group
scales of the experts the step touches, codebooks, activations, logits and
outputs) / step time. The roofline object reports the gate/up grouped GEMV
(the dominant kernel) against the measured HBM copy bandwidth. The other
workloads of the configuration list (the single GEMV, the d=2/K=256 decode
layer at 1 and 8 tokens, the d=4/K=2048 layer, the skipzero layer, the
prefill layers) are reported under "extra", and a compact per-workload summary
closes the line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: the path does not shard (one GPU per layer); N ranks run N
independent replicas and value sums their bytes over the slowest rank's time.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import workloads as wl  # noqa: E402

METRIC = "VQ expert decode HBM GB/s (% of B200 peak); prefill TFLOP/s; MoE-layer tokens/s"
UNIT = "GB/s"
N_DRAWS = 16
MAIN_SPEC, MAIN_T = wl.DECODE_D4K512, 16
# the other decode workloads, reported under "extra": (layer, tokens)
OTHER_DECODE = {"decode_d2k256_T8": (wl.DECODE_D2K256, 8), "decode_d2k256_T1": (wl.DECODE_D2K256, 1),
                "decode_d4k2048_T16": (wl.DECODE_D4K2048, 16), "decode_skipzero_T1": (wl.SKIPZERO_MIXED, 1)}


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _row_words(cols, geo):
    """uint32 words of one packed row (the format's closed form, computed without either library)."""
    return (cols // geo.d // 32) * geo.bits


def _module_bytes(md):
    """Bytes of one expert's live codes + scales, per expert, for a module."""
    per_row = _row_words(md.cols, wl.Geometry(md.d, md.bits)) * 4 + (md.cols // 64) * 2
    if md.bitmap is None:
        live = np.full(md.E, md.rows)
    else:
        live = np.array([sum(bin(int(w)).count("1") for w in md.bitmap[e]) for e in range(md.E)])
    return live * per_row


KERNEL_SOURCES = {
    "grouped_gemv_gate_up_d4k512": ("vq_decode.cu", "vq_device.cuh", "vq_sm100.cuh"),
    "grouped_gemv_gate_up_d2k256": ("vq_decode.cu", "vq_device.cuh", "vq_sm100.cuh"),
    "grouped_gemv_gate_up_d4k2048": ("vq_decode.cu", "vq_device.cuh", "vq_sm100.cuh"),
    "prefill_gemm_gate_up": ("vq_prefill.cu", "vq_device.cuh", "vq_sm100.cuh"),
}


def _kernel_source_hash(tag):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[tag]:
        with open(os.path.join(ROOT, "vector_quantized_moe_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic_per_launch(kernel_tag):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None when the summary is missing or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f).get(kernel_tag)
        if t and t.get("source_hash") == _kernel_source_hash(kernel_tag):
            return float(t["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples every 200 ms while a window of GPU work runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def dist_max(v, device, ws):
    """Max of a float over the ranks (the slowest rank's time)."""
    if ws == 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def dist_sum(v, device, ws):
    """Sum of a float over the ranks (bytes processed by all replicas)."""
    if ws == 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t)
    return float(t.item())


def _main_config(spec, T, per_expert, n_gpus):
    """The workload's config, the same in both arms."""
    return {"workload": spec.name, "T": T, "top_k": spec.top_k, "E": spec.E, "hidden": spec.hidden,
            "inter": spec.inter, "geometry": f"d{spec.gate.d}K{1 << spec.gate.bits} ({spec.gate.bits}-bit codes) x3",
            "l2": f"inputs larger than L2: {N_DRAWS} rotating routing draws over "
                  f"{sum(float(p.sum()) for p in per_expert) / 1e9:.2f} GB of expert weights",
            "parallelism": "replicas" if n_gpus > 1 else "single-gpu"}


def _token_bytes(spec, per_expert, cb_bytes, ids):
    """Algorithmic bytes of a set of routed tokens: the live codes and scales of the experts they
    touch, the codebooks, and each token's activations (bf16), logits (fp32) and output (fp32)."""
    n = ids.shape[0]
    return float(sum(p[np.unique(ids)].sum() for p in per_expert) + cb_bytes
                 + n * (spec.hidden * 2 + spec.E * 4 + spec.hidden * 4))


def run_reference(args):
    """The reference arm: the oracle (CPU, float64) on bounded samples of the headline workload,
    timed on the host's cores; rank 0 only. It loads nothing but the oracle."""
    ws, rank, _ = _dist()
    if rank != 0:
        return
    import oracle
    from tests.helpers import oracle_module
    oracle.build()
    spec, T = MAIN_SPEC, MAIN_T
    mds = wl.layer_modules(spec, raw=False, row_words=_row_words)
    oms = [oracle_module(m) for m in mds]
    per_expert = [_module_bytes(m) for m in mds]
    cb_bytes = sum(m.codebook.nbytes for m in mds)
    draws = [wl.layer_inputs(spec, T, i) for i in range(N_DRAWS)]
    total_b, total_t = 0.0, 0.0
    for step in range(args.warmup + args.steps):
        x, lg = draws[step % N_DRAWS]
        tok = np.array([step % T])
        ids, *_ = oracle.route(lg[tok], spec.top_k)
        t0 = time.perf_counter()
        oracle.moe(*oms, x, lg, spec.top_k, tokens=tok)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            total_b += _token_bytes(spec, per_expert, cb_bytes, ids)
            total_t += dt
    value = total_b / total_t / 1e9
    sample = f"one token of the {T}-token batch per step (its {spec.top_k} experts, all three projections), float64"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_t / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": _main_config(spec, T, per_expert, args.gpus),
           "tokens_per_s": args.steps / total_t,
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_ours(args):
    import torch
    import vector_quantized_moe_b200 as vq
    from tests.helpers import lib_module

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    if args.only == "prefill":
        layer_p, fn = measure_prefill(torch, vq, dev, args.steps, args.warmup, small=args.small, ncu_mode=True)
        for i in range(args.steps):
            fn(i)
        torch.cuda.synchronize()
        return
    if args.only == "fit":
        # profiler runs of the data-free fit of one d4K512 expert tensor: warm-up, then the steps
        g = synth.rng(900)
        w = torch.from_numpy(synth.weights(2048, 6144, g).view(np.int16)).to(dev)
        sample, init = synth.fit_draw(2048 * 6144 // 4, 65536, 512, g)
        st, itx = torch.from_numpy(sample).to(dev), torch.from_numpy(init).to(dev)
        for i in range(args.warmup + args.steps):
            vq.fit(w, 4, 512, st, itx, 10)
        torch.cuda.synchronize()
        return

    spec, T = MAIN_SPEC, MAIN_T
    if args.only in OTHER_DECODE:
        spec, T = OTHER_DECODE[args.only]
    if args.small:
        # same per-expert shapes with 64 experts: the case for full ncu captures
        import dataclasses
        spec = dataclasses.replace(spec, E=64, name=spec.name.replace(f"e{spec.E}", "e64"))
    k = spec.top_k
    mds = wl.layer_modules(spec, raw=False, row_words=_row_words)
    mods = [lib_module(m, device=dev) for m in mds]
    layer = vq.MoELayer(*mods)
    per_expert = [_module_bytes(m) for m in mds]
    cb_bytes = sum(m.codebook.nbytes for m in mds)

    draws = [wl.layer_inputs(spec, T, i) for i in range(N_DRAWS)]
    xs = [torch.from_numpy(x.view(np.int16)).to(dev) for x, _ in draws]
    lgs = [torch.from_numpy(lg).to(dev) for _, lg in draws]
    y = torch.empty((T, spec.hidden), dtype=torch.float32, device=dev)
    wsp = layer.workspace(T, k, vq.VQ_MODE_DECODE, dev)

    # algorithmic bytes of each draw from its routing (untimed)
    step_bytes, gu_bytes = [], []
    io = T * spec.hidden * 2 + T * spec.E * 4 + T * spec.hidden * 4
    for lg in lgs:
        _, _, off, _ = vq.route(lg, k)
        touched = np.nonzero(np.diff(off.cpu().numpy()) > 0)[0]
        g, u, d = (float(p[touched].sum()) for p in per_expert)
        step_bytes.append(g + u + d + cb_bytes + io)
        gu_bytes.append(g + u + mds[0].codebook.nbytes + mds[1].codebook.nbytes + T * spec.hidden * 2)

    def step(i):
        layer.decode(xs[i % N_DRAWS], lgs[i % N_DRAWS], k, out=y, workspace=wsp)

    def barrier():
        if ws > 1:
            torch.distributed.barrier()

    def max_over_ranks(v):
        return dist_max(v, dev, ws)

    def sum_over_ranks(v):
        return dist_sum(v, dev, ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    if args.ncu:
        # minimal launch sequence for profiler captures: 16 route calls above,
        # the warm-up steps, then the timed steps (5 launches per step)
        for i in range(args.steps):
            step(i)
        torch.cuda.synchronize()
        return

    # main timed region, with clocks sampled over a window that contains it
    clk = ClockSampler(local)
    clk.start()
    t_end = time.perf_counter() + 1.0
    i = 0
    while time.perf_counter() < t_end:       # pre-roll so the sampler sees the loaded clock
        for _ in range(50):
            step(i)
            i += 1
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    ms_step = ms_total / args.steps
    my_bytes = sum(step_bytes[i % N_DRAWS] for i in range(args.steps))
    value = sum_over_ranks(my_bytes) / (ms_total * 1e-3) / 1e9

    # trace pass: per-stage durations from events recorded at stage boundaries
    stage_ms = _traced(torch, vq, step, args.steps).mean(axis=0)
    gu_ms = float(stage_ms[1])
    gu_avg_bytes = float(np.mean([gu_bytes[i % N_DRAWS] for i in range(args.steps)]))
    hbm, tf_burst, tf_sust, src = _peaks()
    achieved = gu_avg_bytes / (gu_ms * 1e-3) / 1e9

    # end-to-end: host buffers in pinned memory, every step's copies inside the timed region. A serving loop
    # overlaps them with compute: step i+1's inputs copy in (copy stream, double-buffered) while step i runs,
    # and step i's output copies out while step i+1 runs.
    hx = [torch.from_numpy(x.view(np.int16)).pin_memory() for x, _ in draws]
    hl = [torch.from_numpy(lg).pin_memory() for _, lg in draws]
    hy = [torch.empty((T, spec.hidden), dtype=torch.float32).pin_memory() for _ in range(2)]
    dx = [torch.empty_like(xs[0]) for _ in range(2)]
    dl = [torch.empty_like(lgs[0]) for _ in range(2)]
    dy = [torch.empty_like(y) for _ in range(2)]
    comp = torch.cuda.current_stream()
    cin = torch.cuda.Stream()
    cout = torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_ready = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):
        in_free[b].record(comp)
        out_free[b].record(comp)
    torch.cuda.synchronize()
    barrier()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(comp)
    cin.wait_stream(comp)                       # every copy falls inside the timed region
    cout.wait_stream(comp)
    for i in range(args.steps):
        b = i % 2
        with torch.cuda.stream(cin):
            cin.wait_event(in_free[b])          # the step that last read buffer b has run
            dx[b].copy_(hx[i % N_DRAWS], non_blocking=True)
            dl[b].copy_(hl[i % N_DRAWS], non_blocking=True)
            in_ready[b].record(cin)
        comp.wait_event(in_ready[b])
        comp.wait_event(out_free[b])            # output buffer b has been copied out
        layer.decode(dx[b], dl[b], k, out=dy[b], workspace=wsp, stream=comp)
        in_free[b].record(comp)
        out_ready[b].record(comp)
        with torch.cuda.stream(cout):
            cout.wait_event(out_ready[b])
            hy[b].copy_(dy[b], non_blocking=True)
            out_free[b].record(cout)
    comp.wait_stream(cin)
    comp.wait_stream(cout)
    f1.record(comp)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1))
    e2e_value = sum_over_ranks(my_bytes) / (e2e_ms * 1e-3) / 1e9

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(mds, draws, spec, T, per_expert, cb_bytes)
    del layer, mods, xs, lgs, y, wsp, hx, hl, hy, dx, dl, dy
    torch.cuda.empty_cache()

    extra = {}
    if not args.no_extra:
        for key, (spec_x, T_x) in OTHER_DECODE.items():
            extra[key] = measure_decode_layer(torch, vq, spec_x, T_x, dev, min(args.steps, 100), args.warmup,
                                              traffic_tag={"decode_d2k256_T8": "grouped_gemv_gate_up_d2k256",
                                                           "decode_d4k2048_T16": "grouped_gemv_gate_up_d4k2048"}.get(key))
        extra["gemv_d2k256_512x1024"] = measure_gemv_single(torch, vq, dev, min(args.steps, 20), args.warmup)
        extra["prefill"] = measure_prefill(torch, vq, dev, min(args.steps, 20), args.warmup)
        extra["prefill_skipzero_T2048"] = measure_prefill(torch, vq, dev, min(args.steps, 20), args.warmup,
                                                          spec=wl.SKIPZERO_MIXED, T=2048)
        extra["prefill_chunked_T8192"] = measure_prefill_chunked(torch, vq, dev, min(args.steps, 5), args.warmup)
        extra["fit_d4k512"] = measure_fit(torch, vq, dev, min(args.steps, 5), args.warmup)

    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": _traffic_per_launch("grouped_gemv_gate_up_d4k512") if not args.small else None,
                "kernel": f"vq_gemv_tma_kernel<{spec.gate.d},{spec.gate.bits},fp16,dense> (gate+up)",
                "peak_source": f"{src} hbm_gbs", "bytes_per_launch": gu_avg_bytes, "ms_per_launch": gu_ms}
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16xf16->f32", "data": "synthetic",
        "config": _main_config(spec, T, per_expert, ws),
        "tokens_per_s": T * args.steps * ws / (ms_total * 1e-3),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(draws[0][0].nbytes + draws[0][1].nbytes),
                "d2h_bytes_per_step": int(T * spec.hidden * 4),
                "pipeline": "pinned host buffers; inputs copied in on a copy stream one step ahead "
                            "(double-buffered), outputs copied out on another while the next step runs"},
        "gpu_launches": 5 * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "stage_ms": {"route": float(stage_ms[0]), "gate_up_gemv": gu_ms, "swiglu": float(stage_ms[2]),
                     "down_gemv": float(stage_ms[3]), "combine": float(stage_ms[4])},
        "extra": extra,
        "roofline": roofline,
    }
    out["summary"] = _summary(out)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def _summary(out):
    """A compact line per workload (value, unit, roofline fraction, ms per step), last in the JSON line so
    that a truncated tail still holds every workload."""
    def frac(d):
        r = d.get("roofline") or d.get("gate_up_stage") or {}
        return None if r.get("frac") is None else round(float(r["frac"]), 4)
    s = {out["config"]["workload"] + f"_T{out['config']['T']}": {
        "value": round(out["value"], 1), "unit": out["unit"], "gate_up_frac_of_hbm": frac(out),
        "ms_per_step": round(out["ms_per_step"], 4), "e2e": round(out["e2e"]["value"], 1)}}
    for k, d in out.get("extra", {}).items():
        e = {"value": round(float(d["value"]), 3 if d.get("unit") == "ms" else 1), "unit": d.get("unit")}
        f = frac(d)
        if f is not None:
            e["frac"] = f
            e["of"] = ((d.get("roofline") or {}).get("peak_source")
                       or (d.get("gate_up_stage") or {}).get("peak_source") or "")
        if "ms_per_step" in d:
            e["ms_per_step"] = round(float(d["ms_per_step"]), 4)
        if "gate_up_hbm" in d:
            e["gate_up_frac_of_hbm"] = round(float(d["gate_up_hbm"]["frac"]), 4)
        s[k] = e
    if out.get("cpu_baseline"):
        c = out["cpu_baseline"]
        s["cpu_oracle"] = {"value": round(c["value"], 3), "cores": c["cores"],
                           "single_thread": round(c.get("single_thread", {}).get("value", 0.0), 4)}
    return s


def _time_steps(torch, fn, steps):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for i in range(steps):
        fn(i)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def _traced(torch, vq, fn, steps, n_events=6):
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)] for _ in range(steps)]
    for i in range(steps):
        vq.set_trace_events(evs[i])
        fn(i)
    vq.set_trace_events(None)
    torch.cuda.synchronize()
    return np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(n_events - 1)] for i in range(steps)])


def measure_decode_layer(torch, vq, spec, T, dev, steps, warmup, traffic_tag=None):
    """Another decode workload (its own layer, 16 rotating routing draws): step GB/s and the gate+up
    launch's fraction of the measured HBM bandwidth."""
    from tests.helpers import lib_module
    mds = wl.layer_modules(spec, raw=False, row_words=_row_words)
    per_expert = [_module_bytes(m) for m in mds]
    cb_bytes = sum(m.codebook.nbytes for m in mds)
    gu_cb = mds[0].codebook.nbytes + mds[1].codebook.nbytes
    layer = vq.MoELayer(*[lib_module(m, device=dev) for m in mds])
    del mds
    draws = [wl.layer_inputs(spec, T, 200 + i) for i in range(N_DRAWS)]
    xs = [torch.from_numpy(x.view(np.int16)).to(dev) for x, _ in draws]
    lgs = [torch.from_numpy(lg).to(dev) for _, lg in draws]
    y = torch.empty((T, spec.hidden), dtype=torch.float32, device=dev)
    ws = layer.workspace(T, spec.top_k, vq.VQ_MODE_DECODE, dev)
    io = T * spec.hidden * 2 + T * spec.E * 4 + T * spec.hidden * 4
    step_bytes, gu_bytes = [], []
    for lg in lgs:
        _, _, off, _ = vq.route(lg, spec.top_k)
        touched = np.nonzero(np.diff(off.cpu().numpy()) > 0)[0]
        g, u, d = (float(p[touched].sum()) for p in per_expert)
        step_bytes.append(g + u + d + cb_bytes + io)
        gu_bytes.append(g + u + gu_cb + T * spec.hidden * 2)
    fn = lambda i: layer.decode(xs[i % N_DRAWS], lgs[i % N_DRAWS], spec.top_k, out=y, workspace=ws)
    for i in range(warmup):
        fn(i)
    ms = _time_steps(torch, fn, steps)
    stage = _traced(torch, vq, fn, steps).mean(axis=0)
    hbm, _, _, src = _peaks()
    gu_avg = float(np.mean([gu_bytes[i % N_DRAWS] for i in range(steps)]))
    gu_ach = gu_avg / (stage[1] * 1e-3) / 1e9
    out = {"workload": spec.name, "T": T, "value": sum(step_bytes[i % N_DRAWS] for i in range(steps)) / (ms * 1e-3) / 1e9,
           "unit": UNIT, "ms_per_step": ms / steps, "tokens_per_s": T * steps / (ms * 1e-3),
           "stage_ms": {"route": float(stage[0]), "gate_up_gemv": float(stage[1]), "swiglu": float(stage[2]),
                        "down_gemv": float(stage[3]), "combine": float(stage[4])},
           "gate_up_stage": {"achieved": gu_ach, "peak": hbm, "unit": "GB/s", "frac": gu_ach / hbm,
                             "peak_source": f"{src} hbm_gbs", "bytes_per_launch": gu_avg,
                             "traffic": _traffic_per_launch(traffic_tag) if traffic_tag else None},
           "geometry": f"gate {spec.gate.d}/{spec.gate.bits}b, up {spec.up.d}/{spec.up.bits}b, "
                       f"down {spec.down.d}/{spec.down.bits}b (d / code bits)", "launches_per_step": 5}
    del layer, xs, lgs, y, ws
    torch.cuda.empty_cache()
    return out


def measure_gemv_single(torch, vq, dev, steps, warmup, copies=512):
    """The single VQ GEMV (512 x 1024, d=2/K=256, one token). One call streams 276 KB, far less than the
    launch latency covers, so it is measured in throughput mode: `copies` seeded modules (141 MB, more
    than L2) called round-robin from one CUDA graph, bytes of the calls / device time."""
    from tests.helpers import lib_module
    s = wl.GEMV_D2K256
    mods = []
    for c in range(copies):
        md = wl.module_data(1, s.rows, s.cols, s.geo, 0, (s.seed, 5000 + c), raw=False,
                            row_words=_row_words(s.cols, s.geo))
        mods.append(lib_module(md, device=dev))
    x = torch.from_numpy(synth.activations(s.T, s.cols, synth.rng(s.seed, 1)).view(np.int16)).to(dev)
    ys = [torch.empty((s.T, s.rows), dtype=torch.float32, device=dev) for _ in range(copies)]
    nbytes = (s.rows * _row_words(s.cols, s.geo) * 4 + s.rows * (s.cols // 64) * 2 + (1 << s.geo.bits) * s.geo.d * 2
              + s.T * s.cols * 2 + s.T * s.rows * 4)
    stream = torch.cuda.Stream()
    for c in range(min(copies, warmup * 8)):
        vq.gemv(mods[c], 0, x, out=ys[c], stream=stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for c in range(copies):
            vq.gemv(mods[c], 0, x, out=ys[c], stream=stream)
    graph.replay()
    torch.cuda.synchronize()
    ms = _time_steps(torch, lambda i: graph.replay(), steps)
    per_call_ms = ms / steps / copies
    out = {"workload": s.name, "T": s.T, "value": nbytes / (per_call_ms * 1e-3) / 1e9, "unit": UNIT,
           "ms_per_call": per_call_ms, "bytes_per_call": nbytes,
           "mode": f"{copies} modules round-robin in one CUDA graph (141 MB > L2)",
           "note": "launch-latency bound: one call streams 276 KB", "launches_per_step": copies}
    del graph, mods, ys
    torch.cuda.empty_cache()
    return out


def measure_prefill(torch, vq, dev, steps, warmup, small=False, ncu_mode=False, spec=None, T=None):
    """MoE prefill layer (default: d=4/K=512, 4096 tokens, Zipf(1.1) routing): tcgen05 grouped GEMM path.
    FLOPs count live weights only; GB/s counts the touched experts' live codes and scales."""
    import dataclasses
    from tests.helpers import lib_module
    default = spec is None
    if default:
        spec = wl.PREFILL_D4K512
        T = spec.batches[0]
    if small:
        spec = dataclasses.replace(spec, E=64, name=spec.name.replace("e256", "e64"))
        T = 1024
    mds = wl.layer_modules(spec, raw=False, row_words=_row_words)
    layer = vq.MoELayer(*[lib_module(m, device=dev) for m in mds])
    per_expert = [_module_bytes(m) for m in mds]
    draws = [wl.layer_inputs(spec, T, i) for i in range(2)]
    xs = [torch.from_numpy(x.view(np.int16)).to(dev) for x, _ in draws]
    lgs = [torch.from_numpy(lg).to(dev) for _, lg in draws]
    y = torch.empty((T, spec.hidden), dtype=torch.float32, device=dev)
    ws = layer.workspace(T, spec.top_k, vq.VQ_MODE_PREFILL, dev)
    fn = lambda i: layer.prefill(xs[i % 2], lgs[i % 2], spec.top_k, out=y, workspace=ws)
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    pairs = T * spec.top_k
    # live weights only (skipzero rows are never multiplied)
    flops_gu = 2.0 * pairs * (2 * spec.inter - spec.dead_gate - spec.dead_up) * spec.hidden
    flops_dn = 2.0 * pairs * (spec.hidden - spec.dead_down) * spec.inter
    if ncu_mode:
        return layer, fn
    # weight bytes streamed per step: live codes + scales of the experts the two draws touch
    wbytes = []
    for lg in lgs:
        _, _, off, _ = vq.route(lg, spec.top_k)
        touched = np.nonzero(np.diff(off.cpu().numpy()) > 0)[0]
        wbytes.append([float(p[touched].sum()) for p in per_expert])
    gu_w = float(np.mean([b[0] + b[1] for b in wbytes]))
    step_w = float(np.mean([sum(b) for b in wbytes]))
    ms = _time_steps(torch, fn, steps)
    stage = _traced(torch, vq, fn, steps).mean(axis=0)
    hbm, tf_burst, tf_sust, src = _peaks()
    gu_tflops = flops_gu / (stage[2] * 1e-3) / 1e12
    gu_gbs = gu_w / (stage[2] * 1e-3) / 1e9
    out = {"workload": spec.name, "T": T, "metric": "prefill TFLOP/s", "unit": "TFLOP/s",
           "value": (flops_gu + flops_dn) / (ms / steps * 1e-3) / 1e12, "ms_per_step": ms / steps,
           "tokens_per_s": T * steps / (ms * 1e-3), "flops_per_step": flops_gu + flops_dn,
           "weights_gbs": step_w / (ms / steps * 1e-3) / 1e9,
           "stage_ms": {"route": float(stage[0]), "gather": float(stage[1]), "gate_up_gemm": float(stage[2]),
                        "down_gemm": float(stage[3]), "combine": float(stage[4])},
           "roofline": {"bound": "tensor", "achieved": gu_tflops, "peak": tf_burst, "unit": "TFLOP/s",
                        "frac": gu_tflops / tf_burst,
                        "traffic": _traffic_per_launch("prefill_gemm_gate_up") if default else None,
                        "kernel": f"vq_prefill_gemm_kernel<{spec.gate.d},{spec.gate.bits},2> (gate+up, SwiGLU epilogue)",
                        "peak_source": f"{src} bf16_tflops (fp16 runs at the bf16 rate)",
                        "flops_per_launch": flops_gu, "ms_per_launch": float(stage[2])},
           "gate_up_hbm": {"achieved": gu_gbs, "peak": hbm, "unit": "GB/s", "frac": gu_gbs / hbm,
                           "bytes_per_launch": gu_w},
           "launches_per_step": 6}
    del layer
    torch.cuda.empty_cache()
    return out


def measure_prefill_chunked(torch, vq, dev, steps, warmup, T=8192, chunk=2048):
    """A long prompt of the Zipf prefill layer in `chunk`-token chunks through one chunk-sized
    workspace (vq_moe_prefill_chunked): TFLOP/s and the workspace it needs against one call's."""
    from tests.helpers import lib_module
    spec = wl.PREFILL_D4K512
    mds = wl.layer_modules(spec, raw=False, row_words=_row_words)
    layer = vq.MoELayer(*[lib_module(m, device=dev) for m in mds])
    del mds
    x, lg = wl.layer_inputs(spec, T, 300)
    xt, lt = torch.from_numpy(x.view(np.int16)).to(dev), torch.from_numpy(lg).to(dev)
    y = torch.empty((T, spec.hidden), dtype=torch.float32, device=dev)
    ws = layer.workspace(chunk, spec.top_k, vq.VQ_MODE_PREFILL, dev)
    fn = lambda i: layer.prefill_chunked(xt, lt, spec.top_k, chunk=chunk, out=y, workspace=ws)
    for i in range(warmup):
        fn(i)
    ms = _time_steps(torch, fn, steps)
    flops = 2.0 * T * spec.top_k * 3 * spec.inter * spec.hidden
    out = {"workload": spec.name, "T": T, "chunk": chunk, "metric": "prefill TFLOP/s", "unit": "TFLOP/s",
           "value": flops / (ms / steps * 1e-3) / 1e12, "ms_per_step": ms / steps,
           "tokens_per_s": T * steps / (ms * 1e-3),
           "workspace_bytes": layer.workspace_size(chunk, spec.top_k, vq.VQ_MODE_PREFILL),
           "workspace_bytes_one_call": layer.workspace_size(T, spec.top_k, vq.VQ_MODE_PREFILL),
           "launches_per_step": 6 * ((T + chunk - 1) // chunk)}
    del layer, xt, lt, y, ws
    torch.cuda.empty_cache()
    return out


def measure_fit(torch, vq, dev, steps, warmup, rows=2048, cols=6144, d=4, K=512, n_sample=65536, iters=10):
    """Data-free VQ fit of one expert tensor (vq_fit): Lloyd steps on a subsample, then the codes
    of every subvector. Work = squared-distance evaluations (point x centroid); each takes 3d
    fp32 operations on the CUDA cores, so the roofline is the fp32 issue rate (148 SMs x 128
    lanes x the SM clock) / 3d."""
    g = synth.rng(900)
    w = torch.from_numpy(synth.weights(rows, cols, g).view(np.int16)).to(dev)
    sample, init = synth.fit_draw(rows * cols // d, n_sample, K, g)
    st, it = torch.from_numpy(sample).to(dev), torch.from_numpy(init).to(dev)
    _, _, _, ws = vq.fit(w, d, K, st, it, iters)
    fn = lambda i: vq.fit(w, d, K, st, it, iters, workspace=ws)
    for i in range(warmup):
        fn(i)
    ms = _time_steps(torch, fn, steps) / steps
    n_sub = rows * cols // d
    evals = float(n_sample * iters + n_sub) * K
    clocks = 1965e6
    peak = 148 * 128 * clocks / (3 * d)
    ach = evals / (ms * 1e-3)
    return {"workload": f"vq_fit d{d}K{K} {rows}x{cols} (one expert tensor), {n_sample} sample points, {iters} Lloyd steps",
            "value": ms, "unit": "ms", "subvectors_per_s": n_sub / (ms * 1e-3),
            "roofline": {"bound": "alu", "achieved": ach, "peak": peak, "unit": "distance evaluations/s",
                         "frac": ach / peak, "peak_source": "148 SMs x 128 fp32 lanes x 1965 MHz / (3 d)"},
            "launches_per_step": 4 + 2 * iters}


def cpu_baseline(mds, draws, spec, T, per_expert, cb_bytes, budget_s=10.0):
    """The oracle as it stands on a bounded sample of the headline workload: tokens of the first draw
    until about budget_s seconds of CPU work on all the host's cores, then one token on one core."""
    import oracle
    from tests.helpers import oracle_module
    oracle.build()
    oms = [oracle_module(m) for m in mds]
    x, lg = draws[0]
    cores = oracle.num_threads()

    def run(n_max, budget):
        done, nbytes, t_used = 0, 0.0, 0.0
        while done < n_max and t_used < budget:
            tok = np.array([done % T])
            ids, *_ = oracle.route(lg[tok], spec.top_k)
            t0 = time.perf_counter()
            oracle.moe(*oms, x, lg, spec.top_k, tokens=tok)
            t_used += time.perf_counter() - t0
            nbytes += _token_bytes(spec, per_expert, cb_bytes, ids)
            done += 1
        return done, nbytes, t_used

    done, nbytes, t_used = run(T, budget_s)
    oracle.set_num_threads(1)
    try:
        d1, b1, t1 = run(1, float("inf"))
    finally:
        oracle.set_num_threads(cores)
    return {"value": nbytes / t_used / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} token(s) of the {T}-token batch ({done * spec.top_k} expert passes of all three "
                      f"projections), float64, OpenMP over {cores} threads",
            "seconds": t_used,
            "single_thread": {"value": b1 / t1 / 1e9, "unit": UNIT, "cores": 1, "seconds": t1,
                              "sample": "1 token (its experts, all three projections), float64, one thread"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu", action="store_true", help="only warmup + timed steps, for profiler captures")
    ap.add_argument("--small", action="store_true", help="64-expert variant of the workload (profiling)")
    ap.add_argument("--only", choices=("decode", "prefill", "fit", *OTHER_DECODE), default="decode",
                    help="with --ncu: which path the profiler run exercises")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' lines")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
