#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one decode step of a batch: for every layer, pa_copy_blocks of
the copy-on-write pairs (parallel-sampling workload only), then
pa_decode_append, which writes each sequence's new token into its cache slot
and attends over the whole paged context in one launch (`--step separate`:
pa_reshape_and_cache, then pa_decode, as two launches; the default run
measures that form too, under `also_measured`).
Inputs are resident in HBM before the timed region; each layer has its own
KV cache (all larger than the 126 MB L2, so no flush is needed).  Prints one
JSON line: tokens/s (`value`), the decode call's achieved HBM GB/s against
the measured copy bandwidth (`roofline`), the same metric through host
buffers (`e2e`), and the fp64 CPU oracle timed on a bounded sample
(`cpu_baseline`).

N > 1 (torchrun): every rank runs its own replica of the workload on its
GPU (sequences are independent, so there is no data-path exchange; weak
scaling); the time is the max over ranks.

`--impl reference` times the CPU oracle itself on the same workload (rank 0
only), each step a bounded sample of it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "paged decode attention tokens/s and achieved KV GB/s as % of B200 HBM peak"
FALLBACK_HBM_GBS = 6650.0
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b",
                    choices=["llama7b", "llama13b", "gqa_long", "cow", "cow_run", "tiny", "swap",
                             "prefill"])
    ap.add_argument("--layers", type=int, default=0,
                    help="layer caches to allocate (0: the workload's layer count; fewer "
                         "caches are cycled so every step still runs every layer)")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="run the workload with fewer sequences (small profiling case; "
                         "the bench line then names the reduced size)")
    ap.add_argument("--prefill-kernel", choices=["auto", "mma_sync", "tcgen05"], default="auto",
                    help="prefill workload: which pa_prefill kernel runs (auto = tcgen05)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--step", choices=["fused", "separate"], default="fused",
                    help="fused: pa_decode_append per layer; separate: pa_reshape_and_cache "
                         "then pa_decode")
    ap.add_argument("--extra", default=None,
                    help="comma-separated workloads measured after the main one in the same run "
                         "(default for llama7b: gqa_long,llama13b; 'none' for none); each is "
                         "reported as a sub-record with its own roofline and clocks")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the CPU-oracle sample")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- distributed helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the process group (identity when alone)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- workload description
def algorithmic_bytes(lens, num_q_heads, num_kv_heads, head_dim, elem=2, block=16,
                      append: bool = False) -> int:
    """Bytes one pa_decode call must move: K and V of every cached token, q and
    out, the block-table entries it reads and the context lengths.  With
    `append` (pa_decode_append): also each sequence's new K and V rows, read
    once and written once into the cache."""
    lens = np.asarray(lens, dtype=np.int64)
    S = len(lens)
    kv = int(2 * lens.sum() * num_kv_heads * head_dim * elem)
    qo = 2 * S * num_q_heads * head_dim * elem
    tables = int(4 * ((lens + block - 1) // block).sum())
    new_rows = 2 * 2 * int((lens > 0).sum()) * num_kv_heads * head_dim * elem if append else 0
    return kv + qo + tables + 4 * S + new_rows


# Layer caches allocated per workload when the bench measures it after the
# main workload: fewer caches than layers are cycled (each still far larger
# than L2), so 13B's 40 x 5.6 GB fit in HBM.
EXTRA_LAYER_CACHES = {"gqa_long": 8, "llama13b": 16, "llama7b": 32, "cow": 32, "tiny": 1}


def decode_partitions(max_blocks: int) -> int:
    """Partitions per sequence of a decode call whose tables are `max_blocks`
    wide: 512-token partitions, 1024 when the tables span >= 16384 tokens
    (the rule the library applies; reported in the config only)."""
    pb = 64 if max_blocks * 16 >= 16384 else 32
    return (max_blocks + pb - 1) // pb


def cow_pairs(w: wl.Workload) -> int:
    """Copy-on-write copies at the divergence step: every branch but the last
    holder of a prompt's partly filled last block copies it."""
    if w.name != "cow" or w.prompt_len % w.block_size == 0:
        return 0
    return w.prompts * (w.branches - 1)


def describe(w: wl.Workload, lens, num_blocks: int, max_blocks: int, world: int = 1) -> dict:
    """The workload as both arms run it (no measured or arm-specific fields)."""
    return {
        "workload": w.name,
        "num_seqs": int(len(lens)),
        "num_q_heads": w.num_q_heads,
        "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim,
        "block_size": w.block_size,
        "layers_per_step": w.layers,
        "context_lens": f"{w.lens}; mean {float(np.mean(lens)):.1f}, max {int(np.max(lens))}",
        "l2": "inputs larger than L2: every layer call streams its own KV cache (> 126 MB)",
        "seed": 0,
        "parallelism": f"replicas x{world}",
        "num_blocks": int(num_blocks),
        "decode_partitions": decode_partitions(max_blocks),
        "cow_pairs_per_layer": cow_pairs(w),
    }


def load_peak():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCE_END = b"// ------------------------------------------------------------------ chunked prefill"


def decode_source_digest(read=None) -> str:
    """Hash of the source the decode, scatter, copy and merge kernels are built
    from: the device helpers, the kernel header up to its chunked-prefill
    section, and the host's choice of decode kernel for one query head per kv
    head.  `read(name) -> bytes` reads a source file (default: this tree)."""
    import hashlib
    if read is None:
        def read(name):
            with open(os.path.join(ROOT, "paged_kv_cache_425_b200", "csrc", name), "rb") as fh:
                return fh.read()
    kernels = read("pa_kernels.cuh")
    cut = kernels.find(DECODE_SOURCE_END)
    h = hashlib.sha256()
    h.update(kernels[:cut] if cut >= 0 else kernels)
    h.update(read("pa_device.cuh"))
    # which kernel the host picks for one query head per kv head
    for line in read("pa_api.cu").splitlines():
        if line.startswith(b"#define PA_MHA_ON_MMA"):
            h.update(line)
    return h.hexdigest()[:16]


def traffic_per_call(workload: str, calls_bytes: int):
    """ncu DRAM bytes of one decode call, scaled to this call, if the record
    matches the current kernel sources; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_digest") != decode_source_digest():
        return None
    r = rec.get("workloads", {}).get(workload)
    if not r:
        return None
    return int(r["dram_bytes_per_call"] * calls_bytes / r["algorithmic_bytes_per_call"])


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons, read through NVML every
    few milliseconds on a background thread during the timed region."""

    REASONS = {  # NVML clocks-event-reason bits that matter for a timing
        0x8: "hw_slowdown",
        0x40: "hw_thermal_slowdown",
        0x20: "sw_thermal_slowdown",
        0x4: "sw_power_cap",
    }

    def __init__(self, device, period_s: float = 0.005):
        self.device = device
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.thread = None
        self.error = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: report that instead of clocks
            self.error = f"nvml unavailable: {e}"
            return
        self.stop_flag = threading.Event()

        def loop():
            while not self.stop_flag.is_set():
                try:
                    self.samples.append(float(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)))
                    bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.reasons |= {n for b, n in self.REASONS.items() if bits & b}
                except Exception as e:
                    self.error = str(e)
                    return
                self.stop_flag.wait(self.period)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self) -> dict:
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "not sampled"]}
        self.stop_flag.set()
        self.thread.join(5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "sm_mhz_min": min(self.samples)}


# ---------------------------------------------------------------- our arm
class Setup:
    """Device-resident inputs of one workload (one replica)."""

    def __init__(self, args, device, rank, workload=None, layer_caches=None):
        import torch
        import paged_kv_cache_425_b200 as pk
        from paged_kv_cache_425_b200 import batch
        self.pk = pk
        name = workload or args.workload
        w = wl.WORKLOADS[name]
        if args.num_seqs and workload is None:
            w = wl.scaled(w, num_seqs=args.num_seqs)
        self.w = w
        rng = wl.rng_for(args.seed + rank)
        tdt = torch.float16 if w.dtype == wl.F16 else torch.bfloat16
        self.tdt = tdt
        t0 = time.time()
        if name == "cow":
            own = wl.draw_branch_tokens(w, rng)
            nb = batch.cow_pool_blocks(w)
            fb = batch.ForkedBatch(w, own, wl.draw_block_order(nb, rng), nb)
            b = fb.step()  # the divergence step: every branch copies or writes in place
        else:
            lens = wl.draw_context_lens(w, rng)
            nb = wl.pool_size(w, lens)
            b = batch.decode_batch(w, lens, wl.draw_block_order(nb, rng), nb,
                                   batch.max_blocks_for(w))
        self.alloc_seconds = time.time() - t0
        self.batch = b
        self.S = len(b.seq_ids)
        self.nb = nb
        self.layers = w.layers
        if layer_caches is None:
            layer_caches = args.layers if args.layers > 0 else w.layers
        self.ncache = min(layer_caches, w.layers)
        H, Hq, d = w.num_kv_heads, w.num_q_heads, w.head_dim
        gen = torch.Generator(device=device)
        gen.manual_seed(1000 + args.seed + rank)
        shape = (nb, H, 16, d)
        self.kc = [torch.randn(shape, generator=gen, device=device, dtype=tdt)
                   for _ in range(self.ncache)]
        self.vc = [torch.randn(shape, generator=gen, device=device, dtype=tdt)
                   for _ in range(self.ncache)]
        L = self.layers
        self.q = torch.randn((L, self.S, Hq, d), generator=gen, device=device, dtype=tdt)
        self.k_new = torch.randn((L, self.S, H, d), generator=gen, device=device, dtype=tdt)
        self.v_new = torch.randn((L, self.S, H, d), generator=gen, device=device, dtype=tdt)
        self.out = torch.empty((L, self.S, Hq, d), device=device, dtype=tdt)
        self.tables = torch.from_numpy(b.tables).to(device)
        self.lens = torch.from_numpy(b.context_lens).to(device)
        self.slots = torch.from_numpy(b.slots).to(device)
        self.pairs = torch.from_numpy(b.pairs).to(device) if len(b.pairs) else None
        nws = pk.decode_workspace_size(self.S, Hq, d, b.max_blocks)
        self.ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=device) if nws else None
        self.parts = decode_partitions(b.max_blocks)
        torch.cuda.synchronize(device)
        self.stream = torch.cuda.Stream(device)  # a dedicated stream for every timed call
        self.set_mode(getattr(args, "step", "fused"))
        # K/V bytes of distinct physical blocks (shared prompt blocks once)
        self.unique_kv_bytes = int(b.alloc.stats()["filled_slots"]) * H * d * 2 * 2

    def set_mode(self, mode: str):
        """fused: pa_decode_append per layer; separate: pa_reshape_and_cache
        then pa_decode."""
        b, w = self.batch, self.w
        self.fused = mode == "fused"
        self.bytes_per_call = algorithmic_bytes(b.context_lens, w.num_q_heads, w.num_kv_heads,
                                                w.head_dim, append=self.fused)
        self.launches_per_step = self.layers * ((1 if self.fused else 2)
                                                + (1 if self.parts > 1 else 0)
                                                + (1 if self.pairs is not None else 0))

    def step(self):
        self.step_layers(0, self.layers)

    def step_layers(self, first: int, last: int, bufs=None):
        """Layers [first, last) of a step; `bufs` (an InputSet) replaces the
        step's inputs and outputs (q, k_new, v_new, out and the metadata)."""
        pk, w = self.pk, self.w
        b = bufs or self
        for l in range(first, last):
            c = l % self.ncache
            if b.pairs is not None:
                pk.copy_blocks(self.kc[c], self.vc[c], b.pairs, stream=self.stream)
            if self.fused:
                pk.decode_append(b.out[l], b.q[l], b.k_new[l], b.v_new[l], self.kc[c],
                                 self.vc[c], b.tables, b.lens, w.num_kv_heads, w.scale,
                                 workspace=self.ws, stream=self.stream)
            else:
                pk.reshape_and_cache(b.k_new[l], b.v_new[l], self.kc[c], self.vc[c], b.slots,
                                     stream=self.stream)
                pk.decode(b.out[l], b.q[l], self.kc[c], self.vc[c], b.tables, b.lens,
                          w.num_kv_heads, w.scale, workspace=self.ws, stream=self.stream)

    def decode_all(self):
        """Only the attention calls of one step (every layer's own cache):
        pa_decode_append in the fused mode (writing the same rows again),
        pa_decode otherwise."""
        pk, w = self.pk, self.w
        for l in range(self.layers):
            c = l % self.ncache
            if self.fused:
                pk.decode_append(self.out[l], self.q[l], self.k_new[l], self.v_new[l],
                                 self.kc[c], self.vc[c], self.tables, self.lens, w.num_kv_heads,
                                 w.scale, workspace=self.ws, stream=self.stream)
            else:
                pk.decode(self.out[l], self.q[l], self.kc[c], self.vc[c], self.tables,
                          self.lens, w.num_kv_heads, w.scale, workspace=self.ws,
                          stream=self.stream)


def measure(st, args, device, world) -> dict:
    """Warm-up, then the timed region (whole steps, events only at its two
    ends, clocks sampled throughout), then the decode calls alone; returns
    the timings (max over ranks) and the clock record."""
    import torch
    for _ in range(args.warmup):
        st.step()
    rc, bits = st.pk.get_error(st.stream)
    if rc != 0:
        raise RuntimeError(f"device error word {bits:#x} during warm-up ({st.w.name})")
    # (an event recorded between two kernels would break their programmatic
    # dependent launch and slow the step down)
    L = st.layers
    sampler = ClockSampler(device)
    barrier(device)
    torch.cuda.synchronize()
    sampler.start()
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    marks[0].record(st.stream)
    for i in range(args.steps):
        st.step()
        marks[i + 1].record(st.stream)  # at step boundaries only
    torch.cuda.synchronize()
    barrier(device)
    clocks = sampler.stop()
    local_ms = marks[0].elapsed_time(marks[-1])
    step_ms = [marks[i].elapsed_time(marks[i + 1]) for i in range(args.steps)]
    rc, bits = st.pk.get_error(st.stream)
    if rc != 0:
        raise RuntimeError(f"device error word {bits:#x} in the timed region ({st.w.name})")
    total_ms = max_over_ranks(local_ms, device)
    # ---- the decode call alone: the same layer calls back to back
    barrier(device)
    torch.cuda.synchronize()
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    d0.record(st.stream)
    for _ in range(args.steps):
        st.decode_all()
    d1.record(st.stream)
    torch.cuda.synchronize()
    barrier(device)
    dec_avg_ms = max_over_ranks(d0.elapsed_time(d1) / (args.steps * L), device)
    return {"total_ms": total_ms, "step_ms": step_ms, "dec_avg_ms": dec_avg_ms, "clocks": clocks}


def roofline_record(st, workload: str, dec_avg_ms: float) -> dict:
    peak, peak_src = load_peak()
    achieved = st.bytes_per_call / (dec_avg_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic_per_call(workload, st.bytes_per_call),
            "kernel": ("pa_decode_append call (new-row write + partition kernel + merge kernel)"
                       if st.fused else "pa_decode call (partition kernel + merge kernel)")
                      + ", timed over the step's layer calls run back to back",
            "algorithmic_bytes_per_call": st.bytes_per_call,
            "avg_call_us": round(dec_avg_ms * 1e3, 2), "peak_source": peak_src}


def step_calls(st) -> str:
    """The library calls one layer of the step makes."""
    calls = "pa_decode_append" if st.fused else "pa_reshape_and_cache, pa_decode"
    return ("pa_copy_blocks, " if st.pairs is not None else "") + calls + " per layer"


def extra_workloads(args) -> list:
    if args.extra is None:
        return ["gqa_long", "llama13b"] if args.workload == "llama7b" and not args.num_seqs else []
    return [x for x in args.extra.split(",") if x and x != "none"]


def run_ours(args, world, rank, local):
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    st = Setup(args, device, rank)
    torch.cuda.synchronize()
    m = measure(st, args, device, world)
    total_ms, step_ms, dec_avg_ms, clocks = m["total_ms"], m["step_ms"], m["dec_avg_ms"], m["clocks"]

    # ---- end to end through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(st, args, device, world)
    main = {"w": st.w, "lens": st.batch.context_lens, "nb": st.nb, "max_blocks": st.batch.max_blocks,
            "S": st.S, "ncache": st.ncache, "alloc_seconds": st.alloc_seconds,
            "unique_kv_bytes": st.unique_kv_bytes, "launches": st.launches_per_step,
            "roofline": roofline_record(st, args.workload, dec_avg_ms),
            "step": step_calls(st)}
    # ---- the default run also times the two-launch step on the same inputs
    separate = None
    if st.fused and extra_workloads(args):
        st.set_mode("separate")
        ms = measure(st, args, device, world)
        separate = {
            "value": round(world * st.S * args.steps / (ms["total_ms"] * 1e-3), 1),
            "unit": "tokens/s",
            "ms_per_step": round(ms["total_ms"] / args.steps, 4),
            "ms_per_step_p10_p50_p90": [round(float(np.percentile(ms["step_ms"], q)), 4)
                                        for q in (10, 50, 90)],
            "step": step_calls(st),
            "config": describe(st.w, st.batch.context_lens, st.nb, st.batch.max_blocks, world),
            "roofline": roofline_record(st, args.workload, ms["dec_avg_ms"]),
            "gpu_launches": st.launches_per_step * args.steps,
            "clocks": ms["clocks"],
        }
    del st
    torch.cuda.empty_cache()

    # ---- the other target shapes, one at a time, in the same run
    subs = {}
    for name in extra_workloads(args):
        sx = Setup(args, device, rank, workload=name,
                   layer_caches=EXTRA_LAYER_CACHES.get(name, wl.WORKLOADS[name].layers))
        torch.cuda.synchronize()
        mx = measure(sx, args, device, world)
        subs[name] = {
            "value": round(world * sx.S * args.steps / (mx["total_ms"] * 1e-3), 1),
            "unit": "tokens/s",
            "ms_per_step": round(mx["total_ms"] / args.steps, 4),
            "step": step_calls(sx),
            "ms_per_step_p10_p50_p90": [round(float(np.percentile(mx["step_ms"], q)), 4)
                                        for q in (10, 50, 90)],
            "dtype": "f16" if sx.w.dtype == wl.F16 else "bf16",
            "config": describe(sx.w, sx.batch.context_lens, sx.nb, sx.batch.max_blocks, world),
            "layer_caches": sx.ncache,
            "roofline": roofline_record(sx, name, mx["dec_avg_ms"]),
            "gpu_launches": sx.launches_per_step * args.steps,
            "clocks": mx["clocks"],
        }
        del sx
        torch.cuda.empty_cache()
    if separate is not None:
        subs[f"{args.workload}_separate_calls"] = separate

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, main["w"])

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    w = main["w"]
    roof = main["roofline"]
    value = world * main["S"] * args.steps / (total_ms * 1e-3)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "ms_per_step_p10_p50_p90": [round(float(np.percentile(step_ms, q)), 4) for q in (10, 50, 90)],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16" if w.dtype == wl.F16 else "bf16",
        "data": "synthetic: seeded N(0,1) q/k/v/cache, seeded context lengths, allocator-built scattered tables",
        "config": describe(w, main["lens"], main["nb"], main["max_blocks"], world),
        "step": main["step"],
        "layer_caches": main["ncache"],
        "unique_kv_bytes_per_call": main["unique_kv_bytes"],
        "host_alloc_seconds": round(main["alloc_seconds"], 3),
        "kv_gbs": roof["achieved"],
        "hbm_frac": roof["frac"],
        "roofline": roof,
        "gpu_launches": main["launches"] * args.steps,
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if subs:
        line["also_measured"] = subs
    print(json.dumps(line), flush=True)


class InputSet:
    """One device copy of a step's inputs (q, new k / v, tables, lengths,
    slots, copy pairs) and outputs."""

    def __init__(self, st, clone: bool):
        f = (lambda t: t.clone()) if clone else (lambda t: t)
        self.q, self.k_new, self.v_new, self.out = f(st.q), f(st.k_new), f(st.v_new), f(st.out)
        self.tables, self.lens, self.slots = f(st.tables), f(st.lens), f(st.slots)
        self.pairs = f(st.pairs) if st.pairs is not None else None

    def meta(self):
        return [t for t in (self.tables, self.lens, self.slots, self.pairs) if t is not None]


def run_e2e(st, args, device, world, first_groups: int = 4):
    """Same steps, with every step's inputs copied from pinned host memory and
    its outputs read back, inside the timed region.

    Steps are double-buffered: two device copies of the inputs and outputs
    alternate, so step i + 1's upload (its own stream) runs while step i
    computes, and step i's read-back (a third stream) runs while step i + 1
    computes.  The compute stream waits on one event per step, so the step's
    32 layers stay chained by programmatic dependent launch.  An upload into
    a buffer set waits until the step two back has finished reading it, and a
    step waits until the read-back two back has finished with its output set.
    The first timed step has nothing to hide its upload behind, so it is
    uploaded in layer groups that its compute follows group by group.  A
    one-layer step has nothing to overlap, and there copies and kernels
    share one stream.  The region starts before the first upload and ends
    when the last step's outputs are on the host."""
    import torch
    L = st.layers
    sets = [InputSet(st, clone=False), InputSet(st, clone=True)]
    hq = st.q.cpu().pin_memory()
    hk = st.k_new.cpu().pin_memory()
    hv = st.v_new.cpu().pin_memory()
    hmeta = [t.cpu().pin_memory() for t in sets[0].meta()]
    hout = [torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(h.numel() * h.element_size() for h in (hq, hk, hv)) + \
        sum(h.numel() * h.element_size() for h in hmeta)
    d2h = hout[0].numel() * hout[0].element_size()
    up = torch.cuda.Stream(device)      # a step's inputs, host -> device
    down = torch.cuda.Stream(device)    # a step's outputs, device -> host
    comp = st.stream
    ev_up = [torch.cuda.Event() for _ in range(2)]     # set b's inputs are on the device
    ev_comp = [torch.cuda.Event() for _ in range(2)]   # the step on set b has computed
    ev_down = [torch.cuda.Event() for _ in range(2)]   # set b's outputs are on the host
    used = [False, False]
    per = (L + first_groups - 1) // first_groups
    groups = [(c * per, min(L, (c + 1) * per)) for c in range(first_groups) if c * per < L]
    ev_grp = [torch.cuda.Event() for _ in groups]

    def upload(b, grouped):
        s = sets[b]
        with torch.cuda.stream(up):
            if used[b]:
                up.wait_event(ev_comp[b])           # the step two back has read set b
            for dev, host in zip(s.meta(), hmeta):
                dev.copy_(host, non_blocking=True)
            for g, (a, e) in enumerate(groups if grouped else [(0, L)]):
                s.q[a:e].copy_(hq[a:e], non_blocking=True)
                s.k_new[a:e].copy_(hk[a:e], non_blocking=True)
                s.v_new[a:e].copy_(hv[a:e], non_blocking=True)
                if grouped:
                    ev_grp[g].record(up)
            ev_up[b].record(up)

    def compute(b, grouped):
        s = sets[b]
        if used[b]:
            comp.wait_event(ev_down[b])             # the read-back two back has its outputs
        if grouped:
            for g, (a, e) in enumerate(groups):
                comp.wait_event(ev_grp[g])
                st.step_layers(a, e, s)
        else:
            comp.wait_event(ev_up[b])
            st.step_layers(0, L, s)
        ev_comp[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(ev_comp[b])
            hout[b].copy_(s.out, non_blocking=True)
            ev_down[b].record(down)
        used[b] = True

    def run(n):
        # step i computes on set i % 2 while step i + 1 uploads into the other
        upload(0, grouped=True)
        for i in range(n):
            if i + 1 < n:
                upload((i + 1) % 2, grouped=False)
            compute(i % 2, grouped=(i == 0))
        comp.wait_event(ev_down[(n - 1) % 2])  # the region ends with the last read-back

    def run_serial(n):
        # one layer leaves nothing to overlap: cross-stream handshakes would
        # cost more than they hide, so copies and kernels share one stream
        s = sets[0]
        with torch.cuda.stream(comp):
            for _ in range(n):
                for dev, host in zip(s.meta(), hmeta):
                    dev.copy_(host, non_blocking=True)
                s.q.copy_(hq, non_blocking=True)
                s.k_new.copy_(hk, non_blocking=True)
                s.v_new.copy_(hv, non_blocking=True)
                st.step_layers(0, L, s)
                hout[0].copy_(s.out, non_blocking=True)

    serial = L == 1
    step_loop = run_serial if serial else run
    step_loop(max(1, args.warmup))
    barrier(device)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp if serial else up)  # before the first upload
    step_loop(args.steps)
    b.record(comp)
    torch.cuda.synchronize()
    barrier(device)
    ms = max_over_ranks(a.elapsed_time(b), device)
    last = 0 if serial else (args.steps - 1) % 2
    if not torch.equal(hout[last].to(device), sets[last].out):
        raise RuntimeError("end-to-end outputs read back differ from the device outputs")
    return {"value": round(world * st.S * args.steps / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms / args.steps, 4),
            "overlap": ("none (one layer): copies and kernels on one stream" if serial else
                        "double-buffered steps: step i + 1 uploads and step i - 1 reads back "
                        "while step i computes; the first timed step uploads in "
                        f"{len(groups)} layer groups")}


# ---------------------------------------------------------------- CPU oracle
def host_tables(w: wl.Workload, seed: int):
    """Context lengths, pool size and block tables of the workload, built
    with numpy from the same seeded draws (lengths, then the block order).
    Each sequence takes the next ceil(L / 16) ids of the order; in the
    parallel-sampling workload the branches of a prompt share its blocks,
    and every branch but the last owns a copy of the partly filled last
    block (the divergence step).  The oracle's cost depends only on the
    lengths; this keeps the CPU side free of the library."""
    rng = wl.rng_for(seed)
    bs = w.block_size
    if w.name == "cow":
        wl.draw_branch_tokens(w, rng)  # same draw order as the GPU arm
        pb = (w.prompt_len + bs - 1) // bs
        n = w.prompts * w.branches
        per_branch = (w.own_max + bs - 1) // bs + 2
        nb = int(np.ceil(w.pool_factor * (w.prompts * pb + n * per_branch)))
        order = wl.draw_block_order(nb, rng)
        lens = np.full(n, w.prompt_len + 1, np.int32)
        need = (w.prompt_len + 1 + bs - 1) // bs
        width = (w.prompt_len + w.own_max + 1 + bs - 1) // bs  # as wide as the GPU arm's tables
        tables = np.full((n, width), -1, np.int32)
        pos = 0
        for p in range(w.prompts):
            shared = order[pos:pos + pb]
            pos += pb
            for b in range(w.branches):
                t = tables[p * w.branches + b]
                t[:pb] = shared
                if w.prompt_len % bs and b < w.branches - 1:
                    t[pb - 1] = order[pos]  # the branch's own copy of the last block
                    pos += 1
                if need > pb:
                    t[pb] = order[pos]
                    pos += 1
        return lens, nb, tables
    lens = wl.draw_context_lens(w, rng)
    nb = wl.pool_size(w, lens)
    order = wl.draw_block_order(nb, rng)
    hi = w.lens[-1]
    maxb = (int(hi) + bs - 1) // bs
    tables = np.full((len(lens), maxb), -1, np.int32)
    pos = 0
    for s_, L in enumerate(lens):
        k = (int(L) + bs - 1) // bs
        tables[s_, :k] = order[pos:pos + k]
        pos += k
    return lens, nb, tables


class OracleSample:
    """The fp64 oracle on one layer of the workload, host-generated inputs,
    over the first sequences of the batch that fit `budget_tokens` cached
    tokens (all of them when they fit)."""

    def __init__(self, w: wl.Workload, seed: int, budget_tokens: int):
        import oracle
        self.oracle = oracle
        lens, nb, tables = host_tables(w, seed)
        rng = wl.rng_for(seed + 7919)
        n = int(np.searchsorted(np.cumsum(lens), budget_tokens, side="right"))
        self.seqs = np.arange(max(1, min(n, len(lens))), dtype=np.int32)
        self.sample_tokens = int(lens[self.seqs].sum())
        self.w, self.lens, self.nb, self.tables = w, lens, nb, tables
        self.q = wl.draw_values(rng, (len(lens), w.num_q_heads, w.head_dim), w.dtype)
        # only the blocks the sampled sequences use are generated; others stay zero
        sel = tables[self.seqs]
        used = np.unique(sel[sel >= 0])
        self.kc = np.zeros((nb, w.num_kv_heads, 16, w.head_dim), np.uint16)
        self.vc = np.zeros_like(self.kc)
        self.kc[used] = wl.draw_values(rng, (len(used), w.num_kv_heads, 16, w.head_dim), w.dtype)
        self.vc[used] = wl.draw_values(rng, (len(used), w.num_kv_heads, 16, w.head_dim), w.dtype)

    @property
    def whole(self) -> bool:
        return len(self.seqs) == len(self.lens)

    def run_layer(self):
        self.oracle.decode(self.q, self.kc, self.vc, self.tables, self.lens,
                           self.w.num_kv_heads, self.w.scale, self.w.dtype, seqs=self.seqs)

    def describe(self, calls):
        who = (f"all {len(self.lens)} sequences" if self.whole else
               f"the first {len(self.seqs)} of {len(self.lens)} sequences")
        return (f"{calls} oracle calls of one whole layer over {who} ({self.sample_tokens} cached "
                f"tokens x {self.w.num_q_heads} q heads); a decode step = {self.w.layers} such "
                f"layer calls; tables built with numpy from the seeded draws")


def cpu_baseline(args, w: wl.Workload):
    import oracle
    s = OracleSample(w, args.seed, budget_tokens=40000)
    s.run_layer()  # warm
    calls, t0 = 0, time.perf_counter()
    while True:
        s.run_layer()
        calls += 1
        el = time.perf_counter() - t0
        if el >= args.cpu_seconds:
            break
    per_layer = el / calls
    tok_s = len(s.seqs) / (per_layer * w.layers)
    return {"value": round(tok_s, 3), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": s.describe(calls)}


def run_reference(args, world, rank):
    """Reference arm: the fp64 CPU oracle as it stands, on the host cores.

    A timed step is one whole layer call of the decode step over all the
    batch's sequences (over the first sequences that fit 40k cached tokens
    for the larger workloads, which the record then says); the value is
    tokens per second of the full decode step, i.e. the sequences divided
    by `layers` x the measured time of one layer call."""
    if rank != 0:
        return
    import oracle
    w = wl.WORKLOADS[args.workload]
    s = OracleSample(w, args.seed, budget_tokens=40000)
    for _ in range(args.warmup):
        s.run_layer()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.run_layer()
    el = time.perf_counter() - t0
    per_layer = el / args.steps
    tok_s = len(s.seqs) / (per_layer * w.layers)
    cores = oracle.num_threads()
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(tok_s, 3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(per_layer * 1e3, 3),
        "step": "one whole layer call of the decode step (the bounded sample)",
        "extrapolated": {
            "what": "value = sequences / (layers x measured ms of one layer call)",
            "layers": w.layers,
            "ms_per_decode_step": round(per_layer * w.layers * 1e3, 3),
            "sequences_timed": int(len(s.seqs)),
        },
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: seeded N(0,1) values, seeded context lengths, numpy-built tables",
        "config": describe(w, s.lens, s.nb, s.tables.shape[1], 1),
        "cpu_baseline": {"value": round(tok_s, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": s.describe(args.steps)},
        "e2e": {"value": round(tok_s, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_cow_run(args, world, rank, local):
    """The whole parallel-sampling run: every generation step of the 32 x 4
    branches (step 0 copies the diverging shared last prompt block; later
    steps decode a shrinking set of live branches), 32 layers per step.  All
    steps' tables, lengths, slots and copy pairs come from the allocator
    before timing; the run is captured once in a CUDA graph and replayed, so
    host launch overhead stays out of the timing.  value = mean tokens/s."""
    import torch
    import paged_kv_cache_425_b200 as pk
    from paged_kv_cache_425_b200 import batch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    w = wl.WORKLOADS["cow"]
    rng = wl.rng_for(args.seed + rank)
    own = wl.draw_branch_tokens(w, rng)
    nb = batch.cow_pool_blocks(w)
    fb = batch.ForkedBatch(w, own, wl.draw_block_order(nb, rng), nb)
    plan = []
    while fb.step_index < fb.num_steps:
        b = fb.step()
        plan.append((torch.from_numpy(b.tables).to(device), torch.from_numpy(b.context_lens).to(device),
                     torch.from_numpy(b.slots).to(device),
                     torch.from_numpy(b.pairs).to(device) if len(b.pairs) else None,
                     len(b.seq_ids), algorithmic_bytes(b.context_lens, w.num_q_heads, w.num_kv_heads,
                                                       w.head_dim)))
    tokens_per_run = sum(p[4] for p in plan)
    bytes_per_run = sum(p[5] for p in plan) * w.layers
    S, H, Hq, d, L = w.num_seqs, w.num_kv_heads, w.num_q_heads, w.head_dim, w.layers
    ncache = min(args.layers if args.layers > 0 else L, L)
    gen = torch.Generator(device=device)
    gen.manual_seed(3000 + args.seed + rank)
    kc = [torch.randn((nb, H, 16, d), generator=gen, device=device, dtype=torch.bfloat16)
          for _ in range(ncache)]
    vc = [torch.randn((nb, H, 16, d), generator=gen, device=device, dtype=torch.bfloat16)
          for _ in range(ncache)]
    q = torch.randn((L, S, Hq, d), generator=gen, device=device, dtype=torch.bfloat16)
    kn = torch.randn((L, S, H, d), generator=gen, device=device, dtype=torch.bfloat16)
    vn = torch.randn((L, S, H, d), generator=gen, device=device, dtype=torch.bfloat16)
    out = torch.empty_like(q)
    nws = pk.decode_workspace_size(S, Hq, d, fb.max_blocks)
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=device)
    torch.cuda.synchronize(device)
    stream = torch.cuda.Stream(device)
    fused = args.step == "fused"

    def run():
        for tables, lens, slots, pairs, n, _ in plan:
            for l in range(L):
                c = l % ncache
                if pairs is not None:
                    pk.copy_blocks(kc[c], vc[c], pairs, stream=stream)
                if fused:
                    pk.decode_append(out[l][:n], q[l][:n], kn[l][:n], vn[l][:n], kc[c], vc[c],
                                     tables, lens, H, w.scale, workspace=ws, stream=stream)
                else:
                    pk.reshape_and_cache(kn[l][:n], vn[l][:n], kc[c], vc[c], slots, stream=stream)
                    pk.decode(out[l][:n], q[l][:n], kc[c], vc[c], tables, lens, H, w.scale,
                              workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    for _ in range(args.warmup):
        graph.replay()
    rc, bits = pk.get_error()
    if rc != 0:
        raise RuntimeError(f"device error word {bits:#x}")
    sampler = ClockSampler(device)
    barrier(device)
    torch.cuda.synchronize()
    sampler.start()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(device)
    a.record(cur)
    for _ in range(args.steps):
        graph.replay()
    b.record(cur)
    torch.cuda.synchronize()
    barrier(device)
    clocks = sampler.stop()
    ms = max_over_ranks(a.elapsed_time(b), device)
    del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    per_run_s = ms * 1e-3 / args.steps
    peak, src = load_peak()
    gbs = bytes_per_run / per_run_s / 1e9
    print(json.dumps({
        "metric": "parallel-sampling run: mean decode tokens/s over the whole generation",
        "value": round(world * tokens_per_run / per_run_s, 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_run": round(per_run_s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "cow_run: 32 prompts x 4 branches, 1000-token prompt, branch b "
                               "generates 1 + U{0..256} tokens, 32 layers per step",
                   "generation_steps": len(plan), "tokens_per_run": tokens_per_run,
                   "layer_caches": ncache, "timing": "whole run captured in one CUDA graph"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": None,
                     "kernel": "whole run (copy + " + ("pa_decode_append" if fused else "scatter + decode")
                               + "), logical bytes",
                     "peak_source": src},
        "step": ("pa_copy_blocks (divergence step), " if any(p[3] is not None for p in plan) else "")
                + ("pa_decode_append per layer" if fused else "pa_reshape_and_cache, pa_decode per layer"),
        "gpu_launches": args.steps * sum(L * ((1 if fused else 2) + (1 if p[3] is not None else 0) + 1)
                                         for p in plan),
        "clocks": clocks}), flush=True)


def prefill_flops(lens, chunk, num_q_heads, head_dim):
    """Multiply-adds x 2 of chunked prefill: query token i of a sequence with
    context L attends to L - chunk + i + 1 keys, for q.K and for P.V."""
    total = 0
    for L in np.asarray(lens, dtype=np.int64):
        n = min(chunk, int(L))
        keys = (L - n + 1) * n + n * (n - 1) // 2
        total += 4 * int(keys) * head_dim * num_q_heads
    return total


def run_prefill(args, world, rank, local):
    """Chunked-prefill step: for each of 32 layers, pa_reshape_and_cache of
    the step's 16 x 512 chunk tokens, then pa_prefill over the paged cache."""
    import torch
    import paged_kv_cache_425_b200 as pk
    from paged_kv_cache_425_b200 import batch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    w = wl.WORKLOADS["prefill"]
    if args.num_seqs:
        w = wl.scaled(w, num_seqs=args.num_seqs)
    rng = wl.rng_for(args.seed + rank)
    lens = wl.draw_context_lens(w, rng)
    nb = wl.pool_size(w, lens)
    a = batch.scattered_allocator(nb, wl.draw_block_order(nb, rng))
    chunk = w.chunk
    slots = []
    for s_, L in enumerate(lens):
        a.add_seq(s_, int(L) - chunk)            # context cached before this step
        sl, _ = a.append_slots(np.full(chunk, s_, np.int64))
        slots.append(sl)                         # the chunk's own slots
    maxb = batch.max_blocks_for(w)
    tables, ctx = a.build_tables(np.arange(len(lens)), maxb)
    T = chunk * len(lens)
    H, Hq, d = w.num_kv_heads, w.num_q_heads, w.head_dim
    layers = w.layers
    ncache = min(args.layers if args.layers > 0 else layers, layers)
    gen = torch.Generator(device=device)
    gen.manual_seed(2000 + args.seed + rank)
    tdt = torch.bfloat16 if w.dtype == wl.BF16 else torch.float16
    kc = [torch.randn((nb, H, 16, d), generator=gen, device=device, dtype=tdt) for _ in range(ncache)]
    vc = [torch.randn((nb, H, 16, d), generator=gen, device=device, dtype=tdt) for _ in range(ncache)]
    q = torch.randn((layers, T, Hq, d), generator=gen, device=device, dtype=tdt)
    kn = torch.randn((layers, T, H, d), generator=gen, device=device, dtype=tdt)
    vn = torch.randn((layers, T, H, d), generator=gen, device=device, dtype=tdt)
    out = torch.empty_like(q)
    d_tables = torch.from_numpy(tables).to(device)
    d_lens = torch.from_numpy(ctx).to(device)
    d_qs = torch.from_numpy(np.arange(0, T + 1, chunk, dtype=np.int32)).to(device)
    d_slots = torch.from_numpy(np.concatenate(slots)).to(device)
    torch.cuda.synchronize(device)
    stream = torch.cuda.Stream(device)
    pk.prefill_select(args.prefill_kernel)
    kernel_name = ("prefill_mma_kernel (mma.sync m16n8k16)" if args.prefill_kernel == "mma_sync"
                   else "prefill_umma_kernel (tcgen05.mma, TMEM accumulators)")

    def step():
        for l in range(layers):
            c = l % ncache
            pk.reshape_and_cache(kn[l], vn[l], kc[c], vc[c], d_slots, stream=stream)
            pk.prefill(out[l], q[l], kc[c], vc[c], d_tables, d_lens, d_qs, chunk, H, w.scale,
                       stream=stream)

    for _ in range(args.warmup):
        step()
    rc, bits = pk.get_error(stream)
    if rc != 0:
        raise RuntimeError(f"device error word {bits:#x}")
    sampler = ClockSampler(device)
    barrier(device)
    torch.cuda.synchronize()
    sampler.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(device)
    clocks = sampler.stop()
    total_ms = max_over_ranks(t0.elapsed_time(t1), device)
    # the prefill calls alone, back to back
    barrier(device)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(args.steps):
        for l in range(layers):
            c = l % ncache
            pk.prefill(out[l], q[l], kc[c], vc[c], d_tables, d_lens, d_qs, chunk, H, w.scale,
                       stream=stream)
    d1.record(stream)
    torch.cuda.synchronize()
    barrier(device)
    call_ms = max_over_ranks(d0.elapsed_time(d1) / (args.steps * layers), device)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    flops = prefill_flops(ctx, chunk, Hq, d)
    tflops = flops / (call_ms * 1e-3) / 1e12
    try:
        with open(PEAKS_FILE) as f:
            peak = float(json.load(f)["bf16_tflops"])
        src = "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"
    except Exception:
        peak, src = 1590.0, "fallback"
    line = {
        "metric": "chunked-prefill attention query tokens/s and achieved TFLOP/s",
        "value": round(world * T * args.steps / (total_ms * 1e-3), 1), "unit": "query tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**describe(w, ctx, nb, maxb, world), "chunk": chunk,
                   "query_tokens_per_step_layer": T},
        "layer_caches": ncache,
        "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "traffic": None,
                     "kernel": kernel_name, "flops_per_call": flops,
                     "avg_call_us": round(call_ms * 1e3, 2), "peak_source": src},
        "gpu_launches": args.steps * layers * 2,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_swap(args):
    """Swap bandwidth: scattered blocks of the Llama-7B layer shape (32 kv
    heads x 16 x 128, fp16; 128 KiB per K or V block) between the device
    pool and a pinned host pool, through pa_swap_blocks."""
    import torch
    import paged_kv_cache_425_b200 as pk
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nb_dev, nb_host, n = 8192, 4096, 2048
    shape = (32, 16, 128)
    kc = torch.randn((nb_dev, *shape), device=dev, dtype=torch.float16)
    vc = torch.randn_like(kc)
    hk = torch.empty((nb_host, *shape), dtype=torch.float16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    rng = wl.rng_for(args.seed)
    src = rng.choice(nb_dev, n, replace=False).astype(np.int32)
    dst = rng.choice(nb_host, n, replace=False).astype(np.int32)
    out_pairs = np.stack([src, dst], axis=1)
    in_pairs = np.stack([dst, rng.choice(nb_dev, n, replace=False).astype(np.int32)], axis=1)
    bytes_each = 2 * n * 32 * 16 * 128 * 2
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    ms_out = timed(lambda: pk.swap_blocks(kc, vc, hk, hv, out_pairs))
    ms_in = timed(lambda: pk.swap_blocks(hk, hv, kc, vc, in_pairs))
    print(json.dumps({
        "metric": "block swap bandwidth (device <-> pinned host)", "value": round(bytes_each / (ms_in * 1e-3) / 1e9, 2),
        "unit": "GB/s (swap in)", "swap_out_gbs": round(bytes_each / (ms_out * 1e-3) / 1e9, 2),
        "bytes_per_direction": bytes_each, "blocks": n, "block_bytes_k_or_v": 32 * 16 * 128 * 2,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "dtype": "f16",
        "config": {"workload": "swap: 2048 scattered Llama-7B-shaped blocks, K and V"}}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_env()
    if args.workload == "swap":
        if rank == 0:
            run_swap(args)
        return 0
    if args.workload == "prefill" and args.impl == "ours":
        run_prefill(args, world, rank, local)
        return 0
    if args.workload == "cow_run" and args.impl == "ours":
        run_cow_run(args, world, rank, local)
        return 0
    if world > 1 and args.gpus != world:
        args.gpus = world
    if args.impl == "reference":
        if args.workload in ("swap", "prefill", "cow_run"):
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable":
                                  "the CPU reference arm times decode workloads only"}))
            return 0
        run_reference(args, world, rank)
        return 0
    run_ours(args, world, rank, local)
    return 0


if __name__ == "__main__":
    sys.exit(main())
