"""Benchmark: one decode step of the Llama-3.2-1B-shaped decoder at batch 1 with
128 cached positions, run as one persistent megakernel launch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mk|reference]

Prints ONE JSON line (rank 0). For N > 1 (torchrun, one process per GPU) every
rank runs an independent replica of the step (the path has no exchange step):
``value`` is the sum of all replicas' tokens/s, timed as the max over ranks.

Timing: CUDA events on the launching stream, W untimed warm-up steps, K timed
steps, a device synchronisation and a barrier on both sides. The weights
(2.47 GB) are far larger than the 126 MB L2, so every step streams them from
HBM; no separate L2 flush is needed.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/decode step & tokens/s, Llama-1B-style bf16 bs1; HBM GB/s vs peak"
PAST = 128            # cached positions before the step
BATCH = 1
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
PROFILE_FILE = os.path.join(ROOT, "profiles", "megakernel_llama1b_bs1_ctx128.md")
KERNEL_SOURCES = ["mk_device.cuh", "megakernel.cu", "mk_internal.h"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "persistent_megakernel_interpreter_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(default_workload=True):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source and this run times its workload, the default one
    (else None)."""
    if not default_workload:
        return None
    try:
        text = open(PROFILE_FILE).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not (m_hash and m_bytes) or m_hash.group(1) != kernel_source_hash():
        return None
    return int(m_bytes.group(1))


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class NvmlClocks:
    """Read-only NVML queries in this process: the SM clock and the clock-event
    (throttle) reasons, sampled at the start and the end of the timed region and
    every few milliseconds in between, so a short timed region still has a record.
    Changes nothing on the GPU."""
    # NVML clock-event reason bits (nvmlClocksEventReason*)
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.dev, self.period = device_index, period_s
        self.samples, self.max_mhz, self.handle = [], None, None
        self._stop = threading.Event()
        self.thread = None

    def __enter__(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            prop = torch.cuda.get_device_properties(self.dev)
            bus = f"{prop.pci_domain_id:08x}:{prop.pci_bus_id:02x}:{prop.pci_device_id:02x}.0"
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.sample()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception:  # no NVML on this machine: the nvidia-smi record stands alone
            self.handle = None
        return self

    def sample(self):
        if self.handle is None:
            return
        try:
            mhz = float(self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM))
            bits = int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
            self.samples.append((mhz, bits))
        except Exception:
            pass

    def _run(self):
        while not self._stop.wait(self.period):
            self.sample()

    def __exit__(self, *exc):
        if self.handle is None:
            return
        self._stop.set()
        self.thread.join(timeout=2)
        self.sample()
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass

    def summary(self):
        reasons = sorted({n for _, b in self.samples for n, m in self.REASONS.items() if b & m})
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


class ClockSampler:
    """SM clock and throttle reasons during the timed region: nvidia-smi samples
    every 100 ms and in-process NVML samples (NvmlClocks), merged."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.nvml = NvmlClocks(gpu_index)

    def __enter__(self):
        self.nvml.__enter__()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        self.nvml.__exit__(*exc)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        mhz, max_mhz, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                max_mhz = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        nv = self.nvml.summary()
        reasons |= set(nv["reasons"])
        nv_mhz = [m for m, _ in self.nvml.samples]
        allm = mhz + nv_mhz
        return {"sm_mhz": statistics.median(allm) if allm else None,
                "sm_max_mhz": max_mhz if max_mhz is not None else nv["sm_max_mhz"],
                "reasons": sorted(reasons), "samples": len(allm),
                "samples_nvidia_smi": len(mhz), "samples_nvml": len(nv_mhz)}


def dist_setup(n_gpus: int):
    """(rank, world, local_rank, group-or-None). torchrun sets the env."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world <= 1:
        return 0, 1, 0, None
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    import datetime
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local, dist


def aggregate(elapsed_ms: float, units: float, dist, device=None):
    """Max of the elapsed time and sum of the units over ranks (all ranks call it)."""
    if dist is None:
        return elapsed_ms, units
    import torch
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def workload_config(n_gpus: int, layers: int = 16, past: int = PAST, model: str = "1b", batch: int = BATCH):
    if model == "3b":
        name = "Llama-3.2-3B-style" if layers == 28 else f"Llama-3.2-3B-style ({layers} of 28 layers)"
        dims = {"layers": layers, "hidden": 3072, "heads": "24q/8kv x 128", "ffn": 8192, "vocab": 128256}
        size = "the 6.4 GB of weights"
    else:
        name = "Llama-3.2-1B" if layers == 16 else f"Llama-3.2-1B-shaped ({layers} of 16 layers)"
        dims = {"layers": layers, "hidden": 2048, "heads": "32q/8kv x 64", "ffn": 8192, "vocab": 128256}
        size = "the 2.47 GB of weights"
    return {"workload": f"{name} decoder, one decode step, batch {batch}, {past} cached positions "
                        f"({past + 1} keys) per sequence, random bf16 weights N(0,0.02), KV N(0,1)",
            **dims, "global_batch": batch * n_gpus, "seq_len": past + 1,
            "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU",
            "l2": f"no flush: {size} streamed per step exceed the 126 MB L2"}


def time_oracle(cfg, w, k, v, budget_s: float, past: int, batch: int = BATCH):
    """The CPU oracle on this host's cores: full decode steps of the same workload until
    ``budget_s`` has passed (at least one). Returns (tokens/s, steps, threads, s/step)."""
    import numpy as np
    import oracle
    from persistent_megakernel_interpreter_b200.inputs import make_tokens
    om = oracle.Model(cfg, w)
    kc, vc = oracle.bits(k).copy(), oracle.bits(v).copy()
    toks = make_tokens(cfg, batch, seed=2).numpy()
    threads = oracle.max_threads()
    n = 0
    t0 = time.perf_counter()
    while True:
        om.decode_step(toks, np.array([past] * batch), kc, vc, threads=threads)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return batch * n / el, n, threads, el / n


def run_reference(args):
    rank, world, local, dist = dist_setup(args.gpus)
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    from persistent_megakernel_interpreter_b200.config import LLAMA_1B
    from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_weights
    cfg = LLAMA_1B
    w = make_weights(cfg, seed=0)
    k, v = make_kv_cache(cfg, BATCH, PAST + 1, PAST, seed=1)
    # each timed step is one full oracle decode step; warm-up steps are untimed
    import numpy as np
    import oracle
    from persistent_megakernel_interpreter_b200.inputs import make_tokens
    om = oracle.Model(cfg, w)
    kc, vc = oracle.bits(k).copy(), oracle.bits(v).copy()
    toks = make_tokens(cfg, 1, seed=2).numpy()
    threads = oracle.max_threads()
    tw = time.perf_counter()
    for _ in range(args.warmup):
        om.decode_step(toks, np.array([PAST]), kc, vc, threads=threads)
    t_step = (time.perf_counter() - tw) / max(1, args.warmup)
    # exactly K timed steps while they fit in about two and a half minutes of host
    # time; beyond that as many as fit (the sample below says how many ran)
    steps = max(1, min(args.steps, int(150.0 / max(t_step, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(steps):
        om.decode_step(toks, np.array([PAST]), kc, vc, threads=threads)
    el = time.perf_counter() - t0
    value = BATCH * steps / el
    sample = (f"{steps} full decode steps of the workload (oracle, fp32 C, {threads} threads)"
              + ("" if steps == args.steps else f"; {args.steps} requested, capped to fit the time budget"))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / steps, "us_per_step": 1e6 * el / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "arithmetic": "fp32 over bf16 weights and KV cache, fp32 activations (the oracle)",
            "data": "synthetic", "config": workload_config(args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_mk(args):
    import numpy as np
    import torch
    rank, world, local, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from persistent_megakernel_interpreter_b200.config import LLAMA_1B, LLAMA_3B
    from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights
    from persistent_megakernel_interpreter_b200.model import Megakernel
    import dataclasses
    base_cfg = LLAMA_3B if args.model == "3b" else LLAMA_1B
    layers = args.layers or base_cfg.n_layers
    cfg = dataclasses.replace(base_cfg, n_layers=layers) if layers != base_cfg.n_layers else base_cfg
    past = args.past
    BATCH = args.batch
    w = make_weights(cfg, seed=0)
    k, v = make_kv_cache(cfg, BATCH, past + 1, past, seed=1)
    mk = Megakernel(cfg, w.to(dev), max_batch=BATCH, max_seq=past + 1)
    torch.cuda.empty_cache()
    sched_opts = {"proj": {"auto": 0, "cuda": 1, "tensor": 2}[args.proj]}
    if args.part_keys:
        sched_opts["part_keys"] = args.part_keys
    info = mk.build_schedule(BATCH, past + 1, **sched_opts)
    kd, vd = k.to(dev), v.to(dev)
    tokens = make_tokens(cfg, BATCH, seed=2).to(dev)
    positions = torch.full((BATCH,), past, dtype=torch.int32, device=dev)
    logits = torch.empty(BATCH, cfg.vocab, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    bytes_step = cfg.step_bytes(BATCH, past)

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()

    # ---------------- device-timed megakernel steps
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            mk.decode_step(tokens, positions, kd, vd, logits, stream)
    code, msg = mk.status()
    if code != 0:
        raise RuntimeError(f"warm-up step failed: {msg}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    with ClockSampler(local) as clocks:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            mk.decode_step(tokens, positions, kd, vd, logits, stream)
            ev[i][1].record(stream)
        end.record(stream)
        barrier()
    elapsed = start.elapsed_time(end)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    code, msg = mk.status()
    if code != 0:
        raise RuntimeError(f"timed step failed: {msg}")
    t_max, units = aggregate(elapsed, BATCH * args.steps, dist, dev if dist is not None and
                             torch.distributed.get_backend() == "nccl" else None)

    # ---------------- end to end through the host-buffer entry point
    th = torch.zeros(BATCH, dtype=torch.int32).pin_memory()
    th.copy_(tokens.cpu())
    ph = torch.full((BATCH,), past, dtype=torch.int32).pin_memory()
    lh = torch.empty(BATCH, cfg.vocab, dtype=torch.float32).pin_memory()
    for _ in range(min(args.warmup, 10)):
        mk.decode_step_host(th, ph, kd, vd, lh, stream)
    e2e_steps = max(1, args.steps // 4)
    barrier()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        mk.decode_step_host(th, ph, kd, vd, lh, stream)
    s1.record(stream)
    barrier()
    e2e_max, e2e_units = aggregate(s0.elapsed_time(s1), BATCH * e2e_steps, dist,
                                   dev if dist is not None and torch.distributed.get_backend() == "nccl" else None)

    # ---------------- the multi-kernel bubble baseline, replayed from a CUDA graph
    base = None
    if not args.skip_baseline:
        with torch.cuda.stream(stream):
            mk.baseline_decode_step(tokens, positions, kd, vd, logits, stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                mk.baseline_decode_step(tokens, positions, kd, vd, logits, stream)
            for _ in range(args.warmup):
                g.replay()
        nb = max(1, args.steps // 4)
        barrier()
        b0 = torch.cuda.Event(enable_timing=True)
        b1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            b0.record(stream)
            for _ in range(nb):
                g.replay()
            b1.record(stream)
        barrier()
        bt, _ = aggregate(b0.elapsed_time(b1), nb, dist,
                          dev if dist is not None and torch.distributed.get_backend() == "nccl" else None)
        base = {"us_per_step": 1e3 * bt / nb, "launches_per_step": 2 + 6 * cfg.n_layers,
                "replay": "CUDA graph"}
        del g
        code, msg = mk.status()
        if code != 0:
            raise RuntimeError(f"baseline step failed: {msg}")

    # ---------------- optional per-job trace of one step (outside the timed region)
    if args.trace and rank == 0:
        import numpy as np
        from persistent_megakernel_interpreter_b200.trace import format_summary, summarize
        mk.build_schedule(BATCH, past + 1, trace=1, **sched_opts)
        for _ in range(3):
            mk.decode_step(tokens, positions, kd, vd, logits, stream)
        stream.synchronize()
        tr = mk.trace()
        np.save(args.trace, tr)
        with open(os.path.splitext(args.trace)[0] + ".txt", "w") as f:
            f.write(format_summary(summarize(tr)) + "\n")
        mk.build_schedule(BATCH, past + 1, **sched_opts)

    # ---------------- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        val, n, threads, sps = time_oracle(cfg, w, k, v, args.cpu_budget, past, BATCH)
        cpu = {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} full decode step(s) of this workload, {sps:.2f} s each"}

    if rank == 0:
        peak, peak_kind = hbm_peak()
        per_launch_ms = statistics.mean(launch_ms)
        achieved = bytes_step / (per_launch_ms * 1e-3) / 1e9
        traffic = profiled_traffic(args.model == "1b" and BATCH == 1 and past == PAST and
                                   cfg.n_layers == LLAMA_1B.n_layers)
        ms_per_step = t_max / args.steps
        metric = METRIC if (args.model == "1b" and BATCH == 1) else (
            f"µs/decode step & tokens/s, {'Llama-3B' if args.model == '3b' else 'Llama-1B'}-style bf16 "
            f"bs{BATCH}; HBM GB/s vs peak")
        line = {
            "metric": metric, "value": units / (t_max * 1e-3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "us_per_step": 1e3 * ms_per_step,
            "us_per_launch_median": 1e3 * statistics.median(launch_ms),
            "us_per_launch_p10_p90": [1e3 * q for q in (statistics.quantiles(launch_ms, n=10)[0],
                                                         statistics.quantiles(launch_ms, n=10)[8])]
            if len(launch_ms) >= 2 else None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            # the type the products are computed in; weights and KV cache are bf16 either way
            "dtype": "bf16" if info.proj == 2 else "f32",
            "arithmetic": ("bf16 tcgen05 MMA (activations as bf16 high + low parts), fp32 accumulation"
                           if info.proj == 2 else
                           "fp32 FMA over bf16 weights and KV cache, fp32 activations"),
            "data": "synthetic", "config": workload_config(world, cfg.n_layers, past, args.model, BATCH),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind,
                         "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                         "traffic": traffic, "algorithmic_bytes": bytes_step,
                         "kernel": "megakernel"},
            "e2e": {"value": e2e_units / (e2e_max * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": 2 * 4 * BATCH,
                    "d2h_bytes_per_step": 4 * BATCH * cfg.vocab,
                    "us_per_step": 1e3 * e2e_max / e2e_steps},
            "gpu_launches": args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
            "multikernel_baseline": base,
            "schedule": {"n_sm": info.n_sm, "instructions": info.n_instr,
                         "ring_stages": info.n_stages, "stage_bytes": info.stage_bytes,
                         "attn_partitions": info.n_parts,
                         "projections": "tensor cores (tcgen05)" if info.proj == 2 else "CUDA cores"},
        }
        print(json.dumps(line), flush=True)
    mk.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_greedy(args):
    """Greedy decoding at batch 1: a 32-token random prompt fed as decode steps into
    an empty cache, then ``--greedy`` generated tokens, each the argmax of the
    previous step's logits (chosen on the device by mk_greedy_select, outside the
    timed region). Every
    step is timed alone with CUDA events around its launch; prints one JSON line
    with the per-step latency distribution."""
    import numpy as np
    import torch
    from persistent_megakernel_interpreter_b200.config import LLAMA_1B, LLAMA_3B
    from persistent_megakernel_interpreter_b200.inputs import make_kv_cache, make_tokens, make_weights
    from persistent_megakernel_interpreter_b200.model import Megakernel, greedy_select
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = LLAMA_3B if args.model == "3b" else LLAMA_1B
    n_prompt, n_gen = 32, args.greedy
    steps = n_prompt + n_gen
    w = make_weights(cfg, seed=0)
    k, v = make_kv_cache(cfg, 1, steps, 0, seed=1)
    mk = Megakernel(cfg, w.to(dev), max_batch=1, max_seq=steps)
    mk.build_schedule(1, steps, **({"part_keys": args.part_keys} if args.part_keys else {}))
    kd, vd = k.to(dev), v.to(dev)
    prompt = make_tokens(cfg, n_prompt, seed=50).to(dev)
    tok = torch.zeros(1, dtype=torch.int32, device=dev)
    pos = torch.zeros(1, dtype=torch.int32, device=dev)
    logits = torch.empty(1, cfg.vocab, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        tok.copy_(prompt[:1])
        for _ in range(args.warmup):
            mk.decode_step(tok, pos, kd, vd, logits, stream)
        kd.zero_()
        vd.zero_()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        with ClockSampler(0) as clocks:
            for p in range(steps):
                pos.fill_(p)
                if p < n_prompt:
                    tok.copy_(prompt[p:p + 1])
                else:
                    greedy_select(logits, tok)
                ev[p][0].record(stream)
                mk.decode_step(tok, pos, kd, vd, logits, stream)
                ev[p][1].record(stream)
            stream.synchronize()
    code, msg = mk.status()
    if code != 0:
        raise RuntimeError(f"greedy decode failed: {msg}")
    us = np.array([1e3 * a.elapsed_time(b) for a, b in ev])
    gen = us[n_prompt:]

    # The generated tokens again, each variant timed as a whole from the same state
    # (the prompt decoded into an empty cache): (a) mk_decode_step + mk_greedy_select
    # launches, selection inside the timed region; (b) mk_decode_steps_greedy, the
    # choice fused into each step's LM head, one call for all tokens.
    def after_prompt():
        kd.zero_()
        vd.zero_()
        for p in range(n_prompt):
            pos.fill_(p)
            tok.copy_(prompt[p:p + 1])
            mk.decode_step(tok, pos, kd, vd, logits, stream)
        greedy_select(logits, tok, pos)  # the first generated token, position n_prompt

    timed = {}
    seqs = {}
    with torch.cuda.stream(stream):
        for variant in ("select_launch", "fused"):
            after_prompt()
            out = torch.empty(n_gen, 1, dtype=torch.int32, device=dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if variant == "fused":
                mk.decode_steps_greedy(tok, pos, kd, vd, logits, n_gen, generated=out, stream=stream)
            else:
                for i in range(n_gen):
                    mk.decode_step(tok, pos, kd, vd, logits, stream)
                    greedy_select(logits, tok, pos, stream=stream)
                    out[i].copy_(tok)
            e1.record(stream)
            stream.synchronize()
            timed[variant] = 1e3 * e0.elapsed_time(e1) / n_gen
            seqs[variant] = out.cpu().numpy().ravel()
    code, msg = mk.status()
    if code != 0:
        raise RuntimeError(f"greedy decode failed: {msg}")
    peak, peak_kind = hbm_peak()
    line = {
        "metric": "µs per decode step, greedy decode at batch 1 (each step timed alone)",
        "value": 1e6 / float(gen.mean()), "unit": "tokens/s", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{'Llama-3.2-3B-style' if args.model == '3b' else 'Llama-3.2-1B'} decoder, "
                               f"greedy decode of {n_gen} tokens after a {n_prompt}-token random prompt "
                               f"fed as decode steps into an empty cache, batch 1"},
        "per_step_us": {"generated_mean": float(gen.mean()), "generated_median": float(np.median(gen)),
                        "generated_p10": float(np.percentile(gen, 10)),
                        "generated_p90": float(np.percentile(gen, 90)),
                        "first_prompt_step": float(us[0]), "last_step": float(us[-1]),
                        "prompt_mean": float(us[:n_prompt].mean())},
        "roofline_last_step": {"bound": "hbm", "achieved": cfg.step_bytes(1, steps - 1) / (us[-1] * 1e-6) / 1e9,
                               "peak": peak, "unit": "GB/s",
                               "frac": cfg.step_bytes(1, steps - 1) / (us[-1] * 1e-6) / 1e9 / peak,
                               "peak_source": peak_kind},
        "gpu_launches": steps,
        "per_token_us_selection_inside": {
            "decode_step_then_greedy_select_launch": timed["select_launch"],
            "fused_into_lm_head_one_call": timed["fused"],
            "same_tokens": bool(np.array_equal(seqs["select_launch"], seqs["fused"]))},
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    mk.close()


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["mk", "reference"], default="mk")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle time")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-baseline", action="store_true")
    ap.add_argument("--model", choices=["1b", "3b"], default="1b",
                    help="1b: the Llama-3.2-1B shape (default); 3b: the 3B-style shape")
    ap.add_argument("--batch", type=int, default=BATCH, help="sequences per step")
    ap.add_argument("--layers", type=int, default=0,
                    help="decoder layers (16 = the Llama-3.2-1B workload; fewer only for "
                         "small profiling captures of the same kernels)")
    ap.add_argument("--past", type=int, default=PAST, help="cached positions before the step")
    ap.add_argument("--proj", choices=["auto", "cuda", "tensor"], default="auto",
                    help="projections at batch > 1: tensor cores (auto) or CUDA cores")
    ap.add_argument("--part-keys", type=int, default=0,
                    help="keys per attention partition (0 = the schedule builder's choice)")
    ap.add_argument("--greedy", type=int, default=0, metavar="N",
                    help="instead of the step benchmark: greedy-decode N tokens after a 32-token "
                         "prompt at batch 1 and report the per-step latency")
    ap.add_argument("--trace", default=None, metavar="FILE",
                    help="after the timed run, trace one step's per-job timestamps and save "
                         "them (.npy) with a text summary beside them")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return args


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    elif args.greedy:
        run_greedy(args)
    else:
        run_mk(args)


if __name__ == "__main__":
    main()
