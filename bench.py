#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one decode step of a batch: for every layer, pa_copy_blocks of
the copy-on-write pairs (parallel-sampling workload only), pa_reshape_and_cache
of one new token per sequence, then pa_decode over the whole paged context.
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
def algorithmic_bytes(lens, num_q_heads, num_kv_heads, head_dim, elem=2, block=16) -> int:
    """Bytes one pa_decode call must move: K and V of every cached token, q and
    out, the block-table entries it reads and the context lengths."""
    lens = np.asarray(lens, dtype=np.int64)
    S = len(lens)
    kv = int(2 * lens.sum() * num_kv_heads * head_dim * elem)
    qo = 2 * S * num_q_heads * head_dim * elem
    tables = int(4 * ((lens + block - 1) // block).sum())
    return kv + qo + tables + 4 * S


def describe(w: wl.Workload, lens, layers_alloc: int) -> dict:
    return {
        "workload": w.name,
        "num_seqs": int(len(lens)),
        "num_q_heads": w.num_q_heads,
        "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim,
        "block_size": w.block_size,
        "layers_per_step": w.layers,
        "layer_caches": layers_alloc,
        "context_lens": f"{w.lens}; mean {float(np.mean(lens)):.1f}, max {int(np.max(lens))}",
        "l2": "inputs larger than L2: every layer call streams its own KV cache (> 126 MB)",
        "seed": 0,
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

    def __init__(self, args, device, rank):
        import torch
        import paged_kv_cache_425_b200 as pk
        from paged_kv_cache_425_b200 import batch
        self.pk = pk
        w = wl.WORKLOADS[args.workload]
        if args.num_seqs:
            w = wl.scaled(w, num_seqs=args.num_seqs)
        self.w = w
        rng = wl.rng_for(args.seed + rank)
        tdt = torch.float16 if w.dtype == wl.F16 else torch.bfloat16
        self.tdt = tdt
        t0 = time.time()
        if args.workload == "cow":
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
        self.ncache = args.layers if args.layers > 0 else w.layers
        self.ncache = min(self.ncache, w.layers)
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
        self.parts = (b.max_blocks + 31) // 32
        torch.cuda.synchronize(device)
        self.stream = torch.cuda.Stream(device)  # a dedicated stream for every timed call
        self.bytes_per_call = algorithmic_bytes(b.context_lens, Hq, H, d)
        # K/V bytes of distinct physical blocks (shared prompt blocks once)
        self.unique_kv_bytes = int(b.alloc.stats()["filled_slots"]) * H * d * 2 * 2
        self.launches_per_step = L * (1 + 1 + (1 if self.parts > 1 else 0)
                                      + (1 if self.pairs is not None else 0))

    def step(self):
        self.step_layers(0, self.layers)

    def step_layers(self, first: int, last: int):
        pk, w = self.pk, self.w
        for l in range(first, last):
            c = l % self.ncache
            if self.pairs is not None:
                pk.copy_blocks(self.kc[c], self.vc[c], self.pairs, stream=self.stream)
            pk.reshape_and_cache(self.k_new[l], self.v_new[l], self.kc[c], self.vc[c], self.slots,
                                 stream=self.stream)
            pk.decode(self.out[l], self.q[l], self.kc[c], self.vc[c], self.tables, self.lens,
                      w.num_kv_heads, w.scale, workspace=self.ws, stream=self.stream)

    def decode_all(self):
        """Only the decode calls of one step (every layer's own cache)."""
        pk, w = self.pk, self.w
        for l in range(self.layers):
            c = l % self.ncache
            pk.decode(self.out[l], self.q[l], self.kc[c], self.vc[c], self.tables, self.lens,
                      w.num_kv_heads, w.scale, workspace=self.ws, stream=self.stream)


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
    for _ in range(args.warmup):
        st.step()
    rc, bits = st.pk.get_error(st.stream)
    if rc != 0:
        raise RuntimeError(f"device error word {bits:#x} during warm-up")

    # ---- device-resident timing: whole steps, events only at the two ends
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
        raise RuntimeError(f"device error word {bits:#x} in the timed region")
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

    # ---- end to end through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(st, args, device, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, st)

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    peak, peak_src = load_peak()
    achieved = st.bytes_per_call / (dec_avg_ms * 1e-3) / 1e9
    value = world * st.S * args.steps / (total_ms * 1e-3)
    traffic = traffic_per_call(args.workload, st.bytes_per_call)
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
        "dtype": "f16" if st.w.dtype == wl.F16 else "bf16",
        "data": "synthetic: seeded N(0,1) q/k/v/cache, seeded context lengths, allocator-built scattered tables",
        "config": {**describe(st.w, st.batch.context_lens, st.ncache), "parallelism": f"replicas x{world}",
                   "num_blocks": st.nb, "decode_partitions": st.parts,
                   "cow_pairs_per_layer": 0 if st.pairs is None else int(st.pairs.shape[0]),
                   "unique_kv_bytes_per_call": st.unique_kv_bytes,
                   "host_alloc_seconds": round(st.alloc_seconds, 3)},
        "kv_gbs": round(achieved, 1),
        "hbm_frac": round(achieved / peak, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "pa_decode call (partition kernel + merge kernel), timed over "
                               "the step's layer calls run back to back",
                     "algorithmic_bytes_per_call": st.bytes_per_call,
                     "avg_call_us": round(dec_avg_ms * 1e3, 2), "peak_source": peak_src},
        "gpu_launches": st.launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def run_e2e(st, args, device, world, chunks: int = 4):
    """Same steps, with every step's inputs copied from pinned host memory and
    its outputs read back, inside the timed region.  Upload and read-back
    streams move the inputs of the next group of layers while the current
    group computes and read each group's outputs back as soon as they are
    done; per-group events keep a step's copies from overwriting buffers the
    previous step still uses, so copies of one step overlap the compute of
    its neighbours.  The region ends once the last step's outputs are on the
    host."""
    import torch
    L = st.layers
    per = (L + chunks - 1) // chunks
    groups = [(c * per, min(L, (c + 1) * per)) for c in range(chunks) if c * per < L]
    hq = st.q.cpu().pin_memory()
    hk = st.k_new.cpu().pin_memory()
    hv = st.v_new.cpu().pin_memory()
    meta = [(st.tables, st.tables.cpu().pin_memory()), (st.lens, st.lens.cpu().pin_memory()),
            (st.slots, st.slots.cpu().pin_memory())]
    if st.pairs is not None:
        meta.append((st.pairs, st.pairs.cpu().pin_memory()))
    hout = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    h2d = sum(h.numel() * h.element_size() for h in (hq, hk, hv)) + \
        sum(h.numel() * h.element_size() for _, h in meta)
    d2h = hout.numel() * hout.element_size()
    up = torch.cuda.Stream(device)      # inputs of each layer group, host -> device
    meta_s = torch.cuda.Stream(device)  # the step's tables, lengths and slots
    down = torch.cuda.Stream(device)    # each group's outputs, device -> host
    comp = st.stream
    ev_in = [torch.cuda.Event() for _ in groups]      # inputs of a group are on the device
    ev_done = [torch.cuda.Event() for _ in groups]    # a group's compute finished
    ev_read = [torch.cuda.Event() for _ in groups]    # a group's outputs are back on the host
    ev_meta = torch.cuda.Event()
    ev_meta_free = torch.cuda.Event()
    first = [True]

    def one_serial():
        with torch.cuda.stream(comp):
            for dev, host in meta:
                dev.copy_(host, non_blocking=True)
            st.q.copy_(hq, non_blocking=True)
            st.k_new.copy_(hk, non_blocking=True)
            st.v_new.copy_(hv, non_blocking=True)
            st.step()
            hout.copy_(st.out, non_blocking=True)

    def one_overlapped():
        # Uploads, metadata and read-backs each have their own stream, so a
        # group's upload waits only for the previous step's use of the same
        # group, and nothing but the small metadata copy sits between the
        # previous step's last layer and this step's first.
        with torch.cuda.stream(meta_s):
            if not first[0]:
                meta_s.wait_event(ev_meta_free)   # previous step no longer reads them
            for dev, host in meta:
                dev.copy_(host, non_blocking=True)
            ev_meta.record(meta_s)
        with torch.cuda.stream(up):
            for c, (a, b) in enumerate(groups):
                if not first[0]:
                    up.wait_event(ev_done[c])     # previous step no longer reads them
                st.q[a:b].copy_(hq[a:b], non_blocking=True)
                st.k_new[a:b].copy_(hk[a:b], non_blocking=True)
                st.v_new[a:b].copy_(hv[a:b], non_blocking=True)
                ev_in[c].record(up)
        comp.wait_event(ev_meta)
        for c, (a, b) in enumerate(groups):
            comp.wait_event(ev_in[c])
            if not first[0]:
                comp.wait_event(ev_read[c])       # previous outputs are read back
            st.step_layers(a, b)
            ev_done[c].record(comp)
        ev_meta_free.record(comp)
        with torch.cuda.stream(down):
            for c, (a, b) in enumerate(groups):
                down.wait_event(ev_done[c])
                hout[a:b].copy_(st.out[a:b], non_blocking=True)
                ev_read[c].record(down)
        first[0] = False

    # with one layer group there is nothing to overlap: one stream, no syncs
    one = one_overlapped if len(groups) > 1 else one_serial

    def drain():
        # the timed region ends when the last outputs are back on the host
        if one is one_overlapped:
            comp.wait_event(ev_read[-1])

    for _ in range(max(1, args.warmup)):
        one()
    drain()
    barrier(device)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp)
    for _ in range(args.steps):
        one()
    drain()
    b.record(comp)
    torch.cuda.synchronize()
    barrier(device)
    ms = max_over_ranks(a.elapsed_time(b), device)
    if not torch.equal(hout[-1].to(device), st.out[-1]):
        raise RuntimeError("end-to-end outputs read back differ from the device outputs")
    return {"value": round(world * st.S * args.steps / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms / args.steps, 4),
            "overlap": (f"upload, metadata and read-back streams, {len(groups)} layer groups" if len(groups) > 1
                        else "none (one layer): copies and kernels on one stream")}


# ---------------------------------------------------------------- CPU oracle
class OracleSample:
    """The fp64 oracle on one layer of the workload, host-generated inputs,
    over the first sequences of the batch (a bounded sample)."""

    def __init__(self, w: wl.Workload, seed: int, budget_tokens: int):
        import oracle
        from paged_kv_cache_425_b200 import batch as pbatch
        self.oracle = oracle
        rng = wl.rng_for(seed)
        if w.name == "cow":
            own = wl.draw_branch_tokens(w, rng)
            nb = pbatch.cow_pool_blocks(w)
            b = pbatch.ForkedBatch(w, own, wl.draw_block_order(nb, rng), nb).step()
        else:
            lens = wl.draw_context_lens(w, rng)
            nb = wl.pool_size(w, lens)
            b = pbatch.decode_batch(w, lens, wl.draw_block_order(nb, rng), nb,
                                    pbatch.max_blocks_for(w))
        lens = b.context_lens
        n = int(np.searchsorted(np.cumsum(lens), budget_tokens)) + 1
        self.seqs = np.arange(min(n, len(lens)), dtype=np.int32)
        self.sample_tokens = int(lens[self.seqs].sum())
        # only the blocks the sampled sequences use are generated; others stay zero
        self.w = w
        self.b = b
        self.q = wl.draw_values(rng, (len(lens), w.num_q_heads, w.head_dim), w.dtype)
        used = np.unique(b.tables[self.seqs][b.tables[self.seqs] >= 0])
        self.kc = np.zeros((nb, w.num_kv_heads, 16, w.head_dim), np.uint16)
        self.vc = np.zeros_like(self.kc)
        self.kc[used] = wl.draw_values(rng, (len(used), w.num_kv_heads, 16, w.head_dim), w.dtype)
        self.vc[used] = wl.draw_values(rng, (len(used), w.num_kv_heads, 16, w.head_dim), w.dtype)

    def run_layer(self):
        self.oracle.decode(self.q, self.kc, self.vc, self.b.tables, self.b.context_lens,
                           self.w.num_kv_heads, self.w.scale, self.w.dtype, seqs=self.seqs)

    def describe(self, calls):
        return (f"{calls} oracle calls of one layer over the first {len(self.seqs)} of "
                f"{len(self.b.context_lens)} sequences ({self.sample_tokens} cached tokens x "
                f"{self.w.num_q_heads} q heads); a step = {self.w.layers} such layer calls")


def cpu_baseline(args, st):
    import oracle
    s = OracleSample(st.w, args.seed, budget_tokens=20000)
    s.run_layer()  # warm
    calls, t0 = 0, time.perf_counter()
    while True:
        s.run_layer()
        calls += 1
        el = time.perf_counter() - t0
        if el >= args.cpu_seconds:
            break
    per_layer = el / calls
    tok_s = len(s.seqs) / (per_layer * st.w.layers)
    return {"value": round(tok_s, 3), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": s.describe(calls)}


def run_reference(args, world, rank):
    """Reference arm: the fp64 CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return
    import oracle
    w = wl.WORKLOADS[args.workload]
    s = OracleSample(w, args.seed, budget_tokens=4000)
    for _ in range(args.warmup):
        s.run_layer()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.run_layer()
    el = time.perf_counter() - t0
    per_layer = el / args.steps
    tok_s = len(s.seqs) / (per_layer * w.layers)
    ms_step = per_layer * w.layers * 1e3
    cores = oracle.num_threads()
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(tok_s, 3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: seeded N(0,1) values, seeded context lengths, allocator-built tables",
        "config": describe(w, s.b.context_lens, 1),
        "cpu_baseline": {"value": round(tok_s, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": s.describe(args.steps) + "; per-step time = layers x per-call"},
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

    def run():
        for tables, lens, slots, pairs, n, _ in plan:
            for l in range(L):
                c = l % ncache
                if pairs is not None:
                    pk.copy_blocks(kc[c], vc[c], pairs, stream=stream)
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
                     "kernel": "whole run (copy + scatter + decode), logical bytes",
                     "peak_source": src},
        "gpu_launches": args.steps * sum(L * (2 + (1 if p[3] is not None else 0) + 1)
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
        "config": {**describe(w, ctx, ncache), "chunk": chunk, "query_tokens_per_step_layer": T},
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
