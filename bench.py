#!/usr/bin/env python3
"""Decode-attention throughput of libgdattn on B200.

One step = one decode step of the Gemma-4-12B-shaped 48-layer attention stack
(40 sliding layers: 16 q / 8 KV heads, head_dim 256, ring of 1024; 8 global K=V
layers at 0-based 5, 11, ..., 47: 16 q / 1 KV head, head_dim 512), batch 8,
context 8192, bf16 N(0,1) synthetic inputs, all KV caches resident in HBM.  The
48 gdattn_decode calls of a step are captured in one CUDA graph and replayed.

Metric: algorithmic KV bytes per step / device time per step (GB/s), its share
of the 8 TB/s HBM roofline, and microseconds per 48-layer step.  A step reads
3.2 GB of KV, far more than the 126 MB L2, so no flush is needed between steps.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload instead (the reference arm).  With torchrun (N > 1) every rank
runs its own batch of 8 sequences (sequences are independent: weak scaling,
no collective on the data path); timings are reduced as the max over ranks.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402
from decode_attention_09_b200 import accounting, binding  # noqa: E402

METRIC = "decode-attention KV GB/s & % of 8 TB/s HBM roofline; µs per 48-layer step"
HBM_SPEC_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "decode_attention_09_b200", "csrc")
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "traffic.json")


# ------------------------------------------------------------------ helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def measured_peak_gbs():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0  # an earlier burst measurement on this machine


def measured_peak_tflops():
    """Dense bf16 tensor peak: the measured cuBLAS burst figure, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


_COMMENT_OR_LITERAL = re.compile(r'("(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\')|//[^\n]*|/\*.*?\*/',
                                 re.S)


def code_only(text):
    """C++ source without its comments and without whitespace, adjacent string
    literals joined: what a comment edit, re-indentation or re-wrapping leaves
    unchanged.  Comment markers inside string and character literals are kept."""
    text = _COMMENT_OR_LITERAL.sub(lambda m: m.group(1) or "", text)
    return re.sub(r"\s+", "", text).replace('""', "")


def kernel_source_hash(csrc=None):
    """Hash of the device code of the profiled kernels: every kernel lives in a
    csrc/*.cuh header (api.cu holds the host-side launches).  Comments and
    whitespace are left out, so a record taken on a kernel stays valid across
    comment and layout edits."""
    csrc = CSRC if csrc is None else csrc
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        if name.endswith(".cuh"):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode())
                h.update(code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel_key):
    """DRAM bytes per launch from the committed ncu record, if the kernels are unchanged."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_sha") != kernel_source_hash():
        return None
    ent = rec.get("kernels", {}).get(kernel_key)
    return None if ent is None else ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None

    def _ids(self):
        """nvidia-smi ids for this process's device: its UUID first (a CUDA index
        and nvidia-smi's index differ when CUDA_VISIBLE_DEVICES remaps devices),
        then the CUDA index."""
        ids = []
        try:
            u = str(torch.cuda.get_device_properties(self.idx).uuid)
            if u:
                ids.append(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:  # noqa: BLE001 - a device without a UUID: use the index
            pass
        ids.append(str(self.idx))
        return ids

    def _pick_id(self):
        """The first id that a one-shot nvidia-smi query accepts, or None."""
        for gid in self._ids():
            try:
                r = subprocess.run(["nvidia-smi", f"--id={gid}", "--query-gpu=index",
                                    "--format=csv,noheader"], capture_output=True, timeout=20)
            except (OSError, subprocess.TimeoutExpired):
                continue
            if r.returncode == 0 and r.stdout.strip():
                return gid
        return None

    def start(self):
        gid = self._pick_id()
        if gid is None:
            return
        self.path = os.path.join(tempfile.gettempdir(), f"gdattn_clocks_{os.getpid()}.csv")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gid}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            lines = f.readlines()
        os.remove(self.path)
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        top = max(sm)
        loaded = [s for s in sm if s >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ the GPU stack
def l2_bytes(device) -> int:
    """L2 size of the device (cudaDevAttrL2CacheSize through torch)."""
    return int(torch.cuda.get_device_properties(device).L2_cache_size)


def rotation_copies(kv_bytes_per_step: int, l2: int) -> int:
    """Independent copies of a workload's caches to cycle through so that the
    bytes streamed between two uses of one copy exceed 4x the L2 size (1 when
    one step already does)."""
    if kv_bytes_per_step >= 4 * l2:
        return 1
    return -(-4 * l2 // kv_bytes_per_step) + 1


class Stack:
    """Device-resident inputs, outputs and workspaces for every layer of a workload.

    With ``copies`` > 1 the layers are instantiated that many times over
    independent caches (copy c draws from seed offset c * 100003), laid out
    copy after copy; a step then is one pass over one copy, and a replay of all
    copies is ``copies`` steps whose caches are never L2-resident when reused."""

    def __init__(self, w: workloads.Workload, device, seed_offset=0, copies=1):
        self.w = w
        self.layers = []
        self.copies = copies
        self.kv_bytes = 0  # per step (one copy)
        seqlens = w.seqlens()
        self.max_seqlen = int(seqlens.max())
        for c in range(copies):
            for i, spec in enumerate(w.layers):
                self._add_layer(i, spec, seqlens, seed_offset + 100003 * c, device)
                if c == 0:
                    self.kv_bytes += accounting.layer_kv_bytes(spec, seqlens.tolist())

    def _add_layer(self, i, spec, seqlens, seed_offset, device):
        w = self.w
        inp = workloads.layer_inputs(spec, w.batch, seqlens, w.seed * 1000 + i + seed_offset,
                                     device=device, heavy_row_frac=w.heavy_row_frac,
                                     heavy_row_scale=w.heavy_row_scale)
        # all sequences of an even workload attend the same number of positions:
        # tell the planner, so it splits each unit into equal whole-tile parts
        desc = binding.desc_from_spec(
            spec, flags=binding.GDATTN_FLAG_EVEN_UNITS if w.ragged is None else 0)
        ws = binding.alloc_workspace(w.batch, self.max_seqlen, desc, device)
        out = torch.empty_like(inp.q)
        lse = torch.empty(inp.q.shape[:2], dtype=torch.float32, device=device)
        self.layers.append(dict(spec=spec, inp=inp, desc=desc, ws=ws, out=out, lse=lse))

    def launch(self, idx, stream):
        ly = self.layers[idx]
        inp = ly["inp"]
        st = binding.decode_raw(inp.q.data_ptr(), inp.k.data_ptr(),
                                inp.v.data_ptr() if inp.v is not None else None,
                                inp.seqlens.data_ptr(), self.w.batch, self.max_seqlen, ly["desc"],
                                ly["out"].data_ptr(), ly["lse"].data_ptr(), ly["ws"].data_ptr(),
                                ly["ws"].numel(), stream.cuda_stream)
        if st != binding.GDATTN_OK:
            raise binding.GdattnError(st, f"gdattn_decode layer {idx}")

    def graph(self, indices, stream):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for i in indices:  # warm the planner / attributes outside capture
                self.launch(i, stream)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in indices:
                    self.launch(i, stream)
        return g

    def launches_per_step(self, indices):
        return sum(binding.launches_per_call(self.w.batch, self.max_seqlen, self.layers[i]["desc"])
                   for i in indices)


def time_graph(g, stream, steps, warmup):
    """Device time per replay (ms): CUDA events on the stream the graph replays on."""
    return time_graph_replays(g, stream, steps, warmup)[0]


def time_graph_replays(g, stream, steps, warmup):
    """(mean ms per replay, [ms of each replay]): one CUDA event on the replay
    stream before the first replay and after each one, so the mean is the
    elapsed time of the whole run over `steps` and the list gives its spread."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        stream.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record(stream)
        for i in range(steps):
            g.replay()
            ev[i + 1].record(stream)
    ev[-1].synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return ev[0].elapsed_time(ev[-1]) / steps, per


def spread(samples_ms, scale=1.0):
    """Median, p10 and p90 (microseconds) of per-replay times, divided by `scale`
    (the steps one replay holds)."""
    xs = sorted(x * 1e3 / scale for x in samples_ms)
    def pct(q):
        if len(xs) == 1:
            return xs[0]
        pos = q * (len(xs) - 1)
        lo = int(pos)
        hi = min(lo + 1, len(xs) - 1)
        return xs[lo] + (xs[hi] - xs[lo]) * (pos - lo)
    return {"median_us": pct(0.5), "p10_us": pct(0.1), "p90_us": pct(0.9), "samples": len(xs)}


def read_ceiling(device, stream, gib=4, reps=10):
    """Read-only HBM ceiling (GB/s) of gdattn_read_probe over a `gib` GiB buffer:
    16-byte vector loads (mode 0) and bulk copies into shared memory (mode 1)."""
    buf = torch.empty(gib << 30, dtype=torch.uint8, device=device)
    buf.fill_(0x5A)
    sink = torch.zeros(2, dtype=torch.int32, device=device)
    res = {}
    for mode, name in ((0, "ldg16_gbs"), (1, "bulk_gbs")):
        with torch.cuda.stream(stream):
            for _ in range(3):
                binding.read_probe(buf, mode, sink, stream)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                binding.read_probe(buf, mode, sink, stream)
            e1.record(stream)
        e1.synchronize()
        res[name] = buf.numel() / (e0.elapsed_time(e1) / reps * 1e-3) / 1e9
    if int(sink[1].item()) != 0:
        raise RuntimeError("read probe: a bounded wait expired")
    del buf
    res["bytes"] = gib << 30
    res["how"] = ("gdattn_read_probe over a %d GiB buffer, %d launches each: 16-byte "
                  "non-coherent vector loads on every thread (ldg16), or 32 KiB bulk copies "
                  "into a 6-stage shared-memory ring, one CTA per SM (bulk)" % (gib, reps))
    return res


def max_over_ranks(x, world):
    """Largest value over all ranks (a step time: the job is as slow as its
    slowest GPU).  The tensor lives where the process group's backend wants it."""
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed_offset(rank):
    """Each rank decodes its own sequences: a distinct seed stream per rank."""
    return 1000003 * rank


def job_gbs(kv_bytes_per_rank, ms_step_max, world):
    """Whole-job throughput: the KV bytes all ranks processed over the slowest
    rank's device time per step (weak scaling: fixed work per GPU)."""
    return kv_bytes_per_rank * world / (ms_step_max * 1e-3) / 1e9


# --------------------------------------------------------- oracle baseline
def oracle_time(w: workloads.Workload, host_layers):
    """Time the float64 oracle over host copies of some layers' inputs.
    host_layers: list of (layer index, LayerInputs on the CPU).  Returns (kv_bytes, s)."""
    import oracle  # the CPU baseline leg is the one bench path that runs the oracle

    orc = oracle.get()
    total_bytes, total_s = 0, 0.0
    for i, inp in host_layers:
        spec = w.layers[i]
        t = time.perf_counter()
        orc.decode(inp.q, inp.k, inp.v, inp.seqlens, spec.window, spec.softcap, spec.scale)
        total_s += time.perf_counter() - t
        total_bytes += accounting.layer_kv_bytes(spec, inp.seqlens.tolist())
    return total_bytes, total_s


def host_sample(w: workloads.Workload, layers, seqs):
    """CPU-generated inputs of `layers`, restricted to sequences `seqs`."""
    seqlens = w.seqlens()
    idx = torch.as_tensor(seqs)
    out = []
    for i in layers:
        spec = w.layers[i]
        inp = workloads.layer_inputs(spec, w.batch, seqlens, w.seed * 1000 + i, device="cpu",
                                     heavy_row_frac=w.heavy_row_frac,
                                     heavy_row_scale=w.heavy_row_scale)
        out.append((i, workloads.LayerInputs(
            inp.q[idx].contiguous(), inp.k[idx].contiguous(),
            inp.v[idx].contiguous() if inp.v is not None else None, seqlens[idx], spec)))
    return out


REF_STEP_LAYERS = [0, 5]
REF_STEP_SEQS = [0, 1]
REF_STEP_TEXT = ("float64 oracle, 1 thread; one step = layers 0 (sliding) and 5 (global K=V) x "
                 "sequences 0-1 of the batch-8 / 8192-context stack")
CPU_BASELINE_TEXT = ("float64 oracle over the full step (every layer, every sequence) on host "
                     "copies of the exact inputs the GPU processed, one (layer, sequence) job "
                     "per task on %d threads")


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_time_threads(w: workloads.Workload, host_layers, threads):
    """The float64 oracle over every (layer, sequence) of host_layers on
    `threads` threads (the C oracle releases the GIL).  Returns (kv_bytes, s)
    with s the wall time of the whole batch of jobs."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    orc = oracle.get()
    jobs = []
    total_bytes = 0
    for i, inp in host_layers:
        spec = inp.spec
        for b in range(inp.q.shape[0]):
            jobs.append((inp.q[b:b + 1], inp.k[b:b + 1],
                         inp.v[b:b + 1] if inp.v is not None else None,
                         inp.seqlens[b:b + 1], spec))
        total_bytes += accounting.layer_kv_bytes(spec, inp.seqlens.tolist())
    t = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda j: orc.decode(j[0], j[1], j[2], j[3], j[4].window, j[4].softcap,
                                         j[4].scale), jobs))
    return total_bytes, time.perf_counter() - t


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = workloads.ALL_WORKLOADS[args.workload]()
    sample = host_sample(w, REF_STEP_LAYERS, REF_STEP_SEQS)
    for _ in range(args.warmup):
        oracle_time(w, sample[:1])
    tb, ts = 0, 0.0
    for _ in range(args.steps):
        b, s = oracle_time(w, sample)
        tb += b
        ts += s
    gbs = tb / ts / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * ts / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "layers": len(w.layers), "global_batch": w.batch,
                   "seq_len": w.seqlen, "parallelism": "none (host oracle)",
                   "step": "bounded sample: " + REF_STEP_TEXT},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": REF_STEP_TEXT},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (libgdattn has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    w = workloads.ALL_WORKLOADS[args.workload]()
    l2 = l2_bytes(device)
    step_bytes = sum(accounting.layer_kv_bytes(sp, w.seqlens().tolist()) for sp in w.layers)
    ncopy = rotation_copies(step_bytes, l2)
    stack = Stack(w, device, seed_offset=rank_seed_offset(rank), copies=ncopy)
    stream = torch.cuda.Stream(device)
    # Indices over every layer of every copy: one replay of a graph over them is
    # `ncopy` steps, and each copy's caches are cold in L2 when it comes round.
    all_idx = list(range(len(stack.layers)))
    sliding_idx = [i for i in all_idx if stack.layers[i]["spec"].kind == "sliding"]
    global_idx = [i for i in all_idx if stack.layers[i]["spec"].kind == "global"]
    g_all = stack.graph(all_idx, stream)
    g_sl = stack.graph(sliding_idx, stream) if sliding_idx else None
    g_gl = stack.graph(global_idx, stream) if global_idx else None
    torch.cuda.synchronize()
    replays = -(-args.steps // ncopy)  # at least `steps` steps in the timed region
    steps_timed = replays * ncopy

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    ms_replay, per_replay = time_graph_replays(g_all, stream, replays, args.warmup)
    barrier()
    clk = clocks.stop()
    ms_step = max_over_ranks(ms_replay / ncopy, world)
    step_spread = spread(per_replay, ncopy)
    ms_sl = time_graph(g_sl, stream, replays, 3) if g_sl else None
    ms_gl = time_graph(g_gl, stream, replays, 3) if g_gl else None
    want = lambda name: args.sections == "all" or name in args.sections.split(",")
    ceiling = read_ceiling(device, stream) if rank == 0 and want("ceiling") else None
    for ly in stack.layers:  # no device-side error latched during any of it
        st = binding.check_device_status(ly["ws"], stream)
        if st != binding.GDATTN_OK:
            raise binding.GdattnError(st, "device status after timing")

    # ---- end to end through the public API: pinned host q in, out + lse back.
    # The step's inputs (every layer's q, and seqlens) live in one pinned host
    # buffer and cross in one copy; the 48 calls read views of the device copy
    # and write views of one out and one lse buffer, which come back in one copy
    # each.  Fewer, larger copies, and nothing between the calls that would break
    # the dependent-launch chain.
    def views(total, shapes, dtype, device, pinned=False):
        flat = torch.empty(total, dtype=dtype, device=device, pin_memory=pinned)
        out, off = [], 0
        for shp in shapes:
            n = 1
            for d in shp:
                n *= d
            out.append(flat[off:off + n].view(shp))
            off += n
        return flat, out

    q_shapes = [tuple(ly["inp"].q.shape) for ly in stack.layers]
    o_shapes = [tuple(ly["out"].shape) for ly in stack.layers]
    l_shapes = [tuple(ly["lse"].shape) for ly in stack.layers]
    n_q = sum(a * b * c for a, b, c in q_shapes)
    n_o = sum(a * b * c for a, b, c in o_shapes)
    n_l = sum(a * b for a, b in l_shapes)
    q_host_all, q_host = views(n_q, q_shapes, torch.bfloat16, "cpu", pinned=True)
    for qh, ly in zip(q_host, stack.layers):
        qh.copy_(ly["inp"].q.cpu())
    q_dev_all, q_dev = views(n_q, q_shapes, torch.bfloat16, device)
    out_dev_all, out_dev = views(n_o, o_shapes, torch.bfloat16, device)
    lse_dev_all, lse_dev = views(n_l, l_shapes, torch.float32, device)
    out_host_all, out_host = views(n_o, o_shapes, torch.bfloat16, "cpu", pinned=True)
    lse_host_all = torch.empty(n_l, dtype=torch.float32, pin_memory=True)
    sl_host = stack.layers[0]["inp"].seqlens.cpu().pin_memory()
    sl_dev = torch.empty_like(stack.layers[0]["inp"].seqlens)
    # bytes per step: one e2e replay covers the `ncopy` steps of all copies
    h2d = (n_q * 2 + sl_host.numel() * 4) / ncopy
    d2h = (n_o * 2 + n_l * 4) / ncopy

    # Outputs go back in 4 chunks of layers on a side stream, each as soon as
    # its layers are done, overlapping the next chunk's compute.
    n_layers = len(stack.layers)
    chunk = max(1, (n_layers + 3) // 4)
    side = torch.cuda.Stream(device)
    bounds = []
    o_off = l_off = 0
    for c0 in range(0, n_layers, chunk):
        c1 = min(n_layers, c0 + chunk)
        no = sum(a * b * c for a, b, c in o_shapes[c0:c1])
        nl = sum(a * b for a, b in l_shapes[c0:c1])
        bounds.append((c1, o_off, o_off + no, l_off, l_off + nl))
        o_off += no
        l_off += nl

    q_bounds = []
    q_off = 0
    for c0 in range(0, n_layers, chunk):
        nq = sum(a * b * c for a, b, c in q_shapes[c0:min(n_layers, c0 + chunk)])
        q_bounds.append((q_off, q_off + nq))
        q_off += nq
    q_ready = [torch.cuda.Event() for _ in q_bounds]

    def e2e_step():
        # Inputs: the first chunk's q on the compute stream, the others on the
        # side stream meanwhile; each chunk's layers wait for their own q.
        sl_dev.copy_(sl_host, non_blocking=True)
        q0, q1 = q_bounds[0]
        q_dev_all[q0:q1].copy_(q_host_all[q0:q1], non_blocking=True)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for ci in range(1, len(q_bounds)):
                q0, q1 = q_bounds[ci]
                q_dev_all[q0:q1].copy_(q_host_all[q0:q1], non_blocking=True)
                q_ready[ci].record(side)
        i = 0
        for ci, (c1, o0, o1, l0, l1) in enumerate(bounds):
            if ci > 0:
                stream.wait_event(q_ready[ci])
            while i < c1:
                ly = stack.layers[i]
                binding.decode(q_dev[i], ly["inp"].k, ly["inp"].v, sl_dev, ly["desc"],
                               stack.max_seqlen, out=out_dev[i], lse=lse_dev[i],
                               workspace=ly["ws"], stream=stream)
                i += 1
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                out_host_all[o0:o1].copy_(out_dev_all[o0:o1], non_blocking=True)
                lse_host_all[l0:l1].copy_(lse_dev_all[l0:l1], non_blocking=True)
        stream.wait_stream(side)  # the step ends when its results are on the host

    def timed(fn, steps):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
            barrier()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
        e1.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / steps, world)

    # (a) each step issued call by call from Python;
    ms_e2e_eager = timed(e2e_step, min(replays, 200)) / ncopy
    # (b) the same step (copies + 48 calls) captured once in a CUDA graph, as a
    #     serving loop replays it.
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        e2e_step()
        stream.synchronize()
        with torch.cuda.graph(g_e2e, stream=stream):
            e2e_step()
    ms_e2e = timed(g_e2e.replay, replays) / ncopy
    # the graph's D2H landed in pinned memory: it must equal the device result
    torch.cuda.synchronize()
    assert torch.equal(out_host[-1], stack.layers[-1]["out"].cpu())  # same result both ways

    # ---- the same step with the current token's K/V append fused in
    # (gdattn_decode_append): each layer's new rows are written into their ring
    # slots by the decode kernels.  Last, since it writes into the caches.
    ms_app = None
    if want("append"):
        gen = torch.Generator(device="cpu").manual_seed(7 + rank)
        new_rows = []
        for ly in stack.layers:
            sp = ly["spec"]
            shape = (w.batch, sp.n_kv_heads, sp.head_dim)
            kn = torch.randn(shape, generator=gen).to(torch.bfloat16).to(device)
            vn = None if sp.kv_shared else torch.randn(shape, generator=gen).to(torch.bfloat16).to(device)
            new_rows.append((kn, vn))

        def append_step():
            for ly, (kn, vn) in zip(stack.layers, new_rows):
                binding.decode_append(ly["inp"].q, kn, vn, ly["inp"].k, ly["inp"].v, ly["inp"].seqlens,
                                      ly["desc"], stack.max_seqlen, out=ly["out"], lse=ly["lse"],
                                      workspace=ly["ws"], stream=stream)

        g_app = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            append_step()
            stream.synchronize()
            with torch.cuda.graph(g_app, stream=stream):
                append_step()
        barrier()
        ms_app = max_over_ranks(time_graph(g_app, stream, replays, args.warmup) / ncopy, world)
        for ly in stack.layers:
            st = binding.check_device_status(ly["ws"], stream)
            if st != binding.GDATTN_OK:
                raise binding.GdattnError(st, "device status after the append step")

    # ---- fp8 KV cache (gdattn_decode_fp8) on the sliding layers: the same
    # geometry and lengths with e4m3 codes and per-row scales; the global layers
    # (no fp8 kernel) stay bf16 in the mixed step.
    fp8_layers = {}
    for i in (sliding_idx if want("fp8") else []):
        sp = stack.layers[i]["spec"]
        inp8 = workloads.fp8_layer_inputs(sp, w.batch, w.seqlens(),
                                          w.seed * 1000 + 500 + i + rank_seed_offset(rank),
                                          device=device)
        fp8_layers[i] = dict(inp=inp8, desc=stack.layers[i]["desc"],
                             ws=binding.alloc_workspace(w.batch, stack.max_seqlen,
                                                        stack.layers[i]["desc"], device))

    def launch_fp8(i):
        f = fp8_layers[i]
        x, ly = f["inp"], stack.layers[i]
        binding.decode_fp8(x.q, x.k_codes, x.v_codes, x.k_scale, x.v_scale, x.seqlens, f["desc"],
                           stack.max_seqlen, out=ly["out"], lse=ly["lse"], workspace=f["ws"],
                           stream=stream)

    def fp8_graph(indices):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for i in indices:
                launch_fp8(i) if i in fp8_layers else stack.launch(i, stream)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in indices:
                    launch_fp8(i) if i in fp8_layers else stack.launch(i, stream)
        return g

    ms_fp8_sl = ms_fp8_step = None
    if fp8_layers:
        g_f8 = fp8_graph(sliding_idx)
        g_f8_step = fp8_graph(all_idx)
        barrier()
        ms_fp8_sl = max_over_ranks(time_graph(g_f8, stream, replays, 3), world)
        ms_fp8_step = max_over_ranks(time_graph(g_f8_step, stream, replays, 3) / ncopy, world)
        for f in fp8_layers.values():
            st = binding.check_device_status(f["ws"], stream)
            if st != binding.GDATTN_OK:
                raise binding.GdattnError(st, "device status after the fp8 step")
        del g_f8, g_f8_step

    # ---- multi-query decode (gdattn_decode_multi): a 4-token verify step over the
    # global layers (whole-context caches, so every token's range is resident)
    t_multi, ms_multi = 4, None
    if global_idx and want("multi"):
        gen_mq = torch.Generator(device="cpu").manual_seed(11 + rank)
        mq = {}
        for i in global_idx:
            ly = stack.layers[i]
            sp = ly["spec"]
            q4 = torch.randn((t_multi, w.batch, sp.n_q_heads, sp.head_dim),
                             generator=gen_mq).to(torch.bfloat16).to(device)
            ws4 = torch.empty(binding.multi_workspace_size(w.batch, t_multi, stack.max_seqlen,
                                                           ly["desc"]),
                              dtype=torch.uint8, device=device)
            binding.workspace_init(ws4, stream)
            mq[i] = (q4, ws4, torch.empty_like(q4),
                     torch.empty((t_multi, w.batch, sp.n_q_heads), device=device))

        def multi_step():
            for i in global_idx:
                q4, ws4, o4, l4 = mq[i]
                inp = stack.layers[i]["inp"]
                binding.decode_multi(q4, inp.k, inp.v, inp.seqlens, stack.layers[i]["desc"],
                                     stack.max_seqlen, out=o4, lse=l4, workspace=ws4,
                                     stream=stream)

        g_mq = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            multi_step()
            stream.synchronize()
            with torch.cuda.graph(g_mq, stream=stream):
                multi_step()
        barrier()
        ms_multi = max_over_ranks(time_graph(g_mq, stream, replays, 3), world)
        for q4, ws4, o4, l4 in mq.values():
            st = binding.check_device_status(ws4, stream)
            if st != binding.GDATTN_OK:
                raise binding.GdattnError(st, "device status after the multi-query step")
        del g_mq

    # ---- multi-query decode on the sliding layers: verify steps of speculative
    # decoding, 4 and 8 query tokens per sequence (8: 7 draft tokens and the last
    # accepted one), one pass over each ring.  Rings of w + 7 slots (the first
    # token's window must still be in the ring); 8 layers of their own, replayed
    # in turn (together over 4x the L2 size).
    multi_sl = {}
    n_multi_sl = 8
    if sliding_idx and want("multi"):
        sp0 = stack.layers[sliding_idx[0]]["spec"]
        spec_m = dataclasses.replace(sp0, capacity=sp0.window + 7)
        seqlens_m = w.seqlens()
        flags_m = binding.GDATTN_FLAG_EVEN_UNITS if w.ragged is None else 0
        desc_m = binding.desc_from_spec(spec_m, flags=flags_m)
        caches_m = [workloads.layer_inputs(spec_m, w.batch, seqlens_m,
                                           w.seed * 1000 + 900 + j + rank_seed_offset(rank),
                                           device=device)
                    for j in range(n_multi_sl)]
        gen_sq = torch.Generator(device="cpu").manual_seed(13 + rank)
        # one token through gdattn_decode on the same rings: the ratio's base
        ws1 = [binding.alloc_workspace(w.batch, stack.max_seqlen, desc_m, device)
               for _ in caches_m]
        q1 = [torch.randn((w.batch, spec_m.n_q_heads, spec_m.head_dim),
                          generator=gen_sq).to(torch.bfloat16).to(device) for _ in caches_m]

        def single_sl_step():
            for inp, qq, wsq in zip(caches_m, q1, ws1):
                binding.decode(qq, inp.k, inp.v, inp.seqlens, desc_m, stack.max_seqlen,
                               workspace=wsq, stream=stream)

        g_s1 = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            single_sl_step()
            stream.synchronize()
            with torch.cuda.graph(g_s1, stream=stream):
                single_sl_step()
        barrier()
        multi_sl[1] = (max_over_ranks(time_graph(g_s1, stream, replays, 3), world),
                       n_multi_sl * accounting.layer_multi_kv_bytes(spec_m, seqlens_m.tolist(), 1))
        del g_s1, ws1, q1
        for t_m in (4, 8):
            bufs = []
            for inp in caches_m:
                qm = torch.randn((t_m, w.batch, spec_m.n_q_heads, spec_m.head_dim),
                                 generator=gen_sq).to(torch.bfloat16).to(device)
                wsm = torch.empty(binding.multi_workspace_size(w.batch, t_m, stack.max_seqlen,
                                                               desc_m),
                                  dtype=torch.uint8, device=device)
                binding.workspace_init(wsm, stream)
                bufs.append((inp, qm, wsm, torch.empty_like(qm),
                             torch.empty((t_m, w.batch, spec_m.n_q_heads), device=device)))

            def multi_sl_step():
                for inp, qm, wsm, om, lm in bufs:
                    binding.decode_multi(qm, inp.k, inp.v, inp.seqlens, desc_m, stack.max_seqlen,
                                         out=om, lse=lm, workspace=wsm, stream=stream)

            g_msl = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                multi_sl_step()
                stream.synchronize()
                with torch.cuda.graph(g_msl, stream=stream):
                    multi_sl_step()
            barrier()
            ms_m = max_over_ranks(time_graph(g_msl, stream, replays, 3), world)
            for inp, qm, wsm, om, lm in bufs:
                st = binding.check_device_status(wsm, stream)
                if st != binding.GDATTN_OK:
                    raise binding.GdattnError(st, "device status after the sliding multi-query step")
            multi_sl[t_m] = (ms_m, n_multi_sl * accounting.layer_multi_kv_bytes(
                spec_m, seqlens_m.tolist(), t_m))
            del g_msl, bufs
        del caches_m

    # ---- flash prefill (gdattn_decode_multi with a prompt chunk): one 8192-token
    # prompt per layer (a cache of 8192 slots, L = T), on the stack's sliding and
    # global layer shapes, layers of their own replayed in turn (q, K, V and out
    # over 512 MiB per kind).
    prefill = None

    def time_prefill(sp0, n_pf, seed0, replays_pf):
        t_pf = 8192
        spec_p = dataclasses.replace(sp0, capacity=t_pf)
        seqlens_p = torch.full((1,), t_pf, dtype=torch.int32)
        desc_p = binding.desc_from_spec(spec_p)
        gen_p = torch.Generator(device="cpu").manual_seed(seed0 + rank)
        bufs_p = []
        for j in range(n_pf):
            inp = workloads.layer_inputs(spec_p, 1, seqlens_p,
                                         w.seed * 1000 + seed0 + j + rank_seed_offset(rank),
                                         device=device)
            qp = torch.randn((t_pf, 1, spec_p.n_q_heads, spec_p.head_dim),
                             generator=gen_p).to(torch.bfloat16).to(device)
            wsp = torch.empty(binding.multi_workspace_size(1, t_pf, t_pf, desc_p),
                              dtype=torch.uint8, device=device)
            binding.workspace_init(wsp, stream)
            bufs_p.append((inp, qp, wsp, torch.empty_like(qp),
                           torch.empty((t_pf, 1, spec_p.n_q_heads), device=device)))

        def prefill_step():
            for inp, qp, wsp, op, lp in bufs_p:
                binding.decode_multi(qp, inp.k, inp.v, inp.seqlens, desc_p, t_pf, out=op, lse=lp,
                                     workspace=wsp, stream=stream)

        g_pf = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            prefill_step()
            stream.synchronize()
            with torch.cuda.graph(g_pf, stream=stream):
                prefill_step()
        barrier()
        ms_pf = max_over_ranks(time_graph(g_pf, stream, replays_pf, 3), world)
        for inp, qp, wsp, op, lp in bufs_p:
            st = binding.check_device_status(wsp, stream)
            if st != binding.GDATTN_OK:
                raise binding.GdattnError(st, "device status after the prefill step")
        flops = n_pf * accounting.layer_prefill_flops(spec_p, seqlens_p.tolist(), t_pf)
        tf_peak, tf_kind = measured_peak_tflops()
        tflops = flops / (ms_pf * 1e-3) / 1e12
        del g_pf, bufs_p
        return {"tokens": t_pf, "us_per_layer": ms_pf / n_pf * 1e3, "tflops": tflops,
                "peak_tflops": tf_peak, "peak_kind": tf_kind, "frac": tflops / tf_peak,
                "bound": "tensor"}

    if want("prefill") and (sliding_idx or global_idx):
        prefill = {"how": "one 8192-token prompt per layer through gdattn_decode_multi, "
                          "layers replayed in turn in a CUDA graph; useful flops = 4 x "
                          "head_dim per (query head, token, attended position), so the weight "
                          "split's second P.V half (and, on the global layers, the scores "
                          "computed by both CTAs of a block) count as overhead"}
        if sliding_idx:
            prefill["sliding"] = time_prefill(stack.layers[sliding_idx[0]]["spec"], 4, 950,
                                              max(3, replays // 20))
            prefill["sliding"]["traffic"] = traffic_for("prefill_sliding")
            prefill["sliding"]["kernel"] = (
                "tc_pair_prefill_kernel (window 1024, 16 query / 8 KV heads, head_dim 256; "
                "M = 128 query rows, P in tensor memory)")
        if global_idx:
            prefill["global"] = time_prefill(stack.layers[global_idx[0]]["spec"], 2, 960,
                                             max(3, replays // 200))
            prefill["global"]["traffic"] = traffic_for("prefill_global")
            prefill["global"]["kernel"] = (
                "tc_global_prefill_kernel<16> (causal over the whole prompt, 16 query heads, "
                "one K = V head, head_dim 512; M = 64 query rows per CTA pair, each CTA half "
                "of the output dims)")

    # ---- CPU baseline: the oracle over the whole step (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        host = [(i, workloads.LayerInputs(ly["inp"].q.cpu(), ly["inp"].k.cpu(),
                                          ly["inp"].v.cpu() if ly["inp"].v is not None else None,
                                          ly["inp"].seqlens.cpu(), ly["spec"]))
                for i, ly in enumerate(stack.layers[:len(w.layers)])]
        cores = host_cores()
        b, s_all = oracle_time_threads(w, host, cores)
        b1, s1 = oracle_time(w, host[:max(1, len(host) // 8)])
        del host
        cpu = {"value": b / s_all / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": CPU_BASELINE_TEXT % cores, "seconds": s_all,
               "cpu_model": cpu_model(),
               "single_thread": {"value": b1 / s1 / 1e9, "unit": "GB/s", "seconds": s1,
                                 "sample": "the first eighth of the step's layers (at least "
                                           "one), all sequences, one thread"}}

    if world > 1:
        import torch.distributed as dist
        del g_all, g_sl, g_gl, g_e2e, g_app
        dist.destroy_process_group()
    if rank != 0:
        return 0

    kv_step = stack.kv_bytes
    gbs = job_gbs(kv_step, ms_step, world)
    peak, peak_kind = measured_peak_gbs()
    # bytes over every copy's layers of each kind (the sliding / global graphs
    # replay all of them)
    sl_bytes = sum(accounting.layer_kv_bytes(stack.layers[i]["spec"], w.seqlens().tolist())
                   for i in sliding_idx)
    gl_bytes = sum(accounting.layer_kv_bytes(stack.layers[i]["spec"], w.seqlens().tolist())
                   for i in global_idx)
    roof = None
    if ms_sl:
        per_launch_ms = ms_sl / len(sliding_idx)
        per_launch_bytes = sl_bytes / len(sliding_idx)
        ach = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak, "peak_kind": peak_kind,
                "kernel": "sliding layer: tc_pair_decode_kernel (tcgen05; split parts merged in the kernel)",
                "bytes_per_launch": per_launch_bytes, "us_per_launch": per_launch_ms * 1e3,
                "traffic": traffic_for("sliding")}
    if roof is None and ms_gl:  # a workload of global layers only
        per_launch_ms = ms_gl / len(global_idx)
        per_launch_bytes = gl_bytes / len(global_idx)
        ach = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak, "peak_kind": peak_kind,
                "kernel": "global layer: tc_decode_kernel (tcgen05) + LSE combine",
                "bytes_per_launch": per_launch_bytes, "us_per_launch": per_launch_ms * 1e3,
                "traffic": traffic_for("global")}
    per_type = {}
    if ms_gl:
        ach = gl_bytes / len(global_idx) / (ms_gl / len(global_idx) * 1e-3) / 1e9
        per_type["global"] = {"achieved_gbs": ach, "frac": ach / peak,
                              "us_per_layer": ms_gl / len(global_idx) * 1e3,
                              "kernel": "tc_decode_kernel (tcgen05) + LSE combine",
                              "traffic": traffic_for("global")}
    if ms_sl:
        per_type["sliding"] = {"achieved_gbs": roof["achieved"], "frac": roof["frac"],
                               "us_per_layer": roof["us_per_launch"]}
    fp8_summary = None
    if ms_fp8_sl:
        seq = w.seqlens().tolist()
        b8 = sum(accounting.layer_fp8_kv_bytes(stack.layers[i]["spec"], seq) for i in sliding_idx)
        step8 = (b8 + gl_bytes) / ncopy  # bytes of one step (one copy)
        ach8 = b8 / (ms_fp8_sl * 1e-3) / 1e9
        fp8_summary = {
            "kernel": "tc_pair_fp8_decode_kernel (tcgen05 kind::f8f6f4; e4m3 codes, per-row "
                      "fp32 scales)",
            "sliding_us_per_layer": ms_fp8_sl / len(sliding_idx) * 1e3,
            "sliding_achieved_gbs": ach8, "sliding_frac": ach8 / peak, "peak_kind": peak_kind,
            "sliding_bytes_per_launch": b8 / len(sliding_idx),
            "traffic": traffic_for("fp8_sliding"),
            "step_us": ms_fp8_step * 1e3, "step_kv_bytes": step8,
            "step_gbs": job_gbs(step8, ms_fp8_step, world),
            "how": "the sliding layers' caches as e4m3 codes + one fp32 scale per row "
                   "(gdattn_decode_fp8); the mixed step keeps the 8 global layers bf16; "
                   "bytes = codes + scales actually read; CUDA graphs, device time"}
    if ncopy == 1:
        l2_note = (f"no flush needed: {kv_step / 1e9:.2f} GB of KV per step vs "
                   f"{l2 / 2**20:.0f} MiB of L2")
    else:
        l2_note = (f"L2 rotation: {ncopy} independent copies of the step's caches replayed in "
                   f"turn ({ncopy * kv_step / 2**20:.0f} MiB streamed between two uses of one "
                   f"copy, over 4x the {l2 / 2**20:.0f} MiB L2)")
    if roof is not None and ceiling is not None:
        roof["ceiling"] = ceiling
        best = max(ceiling["ldg16_gbs"], ceiling["bulk_gbs"])
        roof["frac_of_ceiling"] = roof["achieved"] / best
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": steps_timed,
        "warmup": args.warmup, "ms_per_step": ms_step, "us_per_step": ms_step * 1e3,
        "step_spread": step_spread,
        "pct_of_8tbs": 100.0 * gbs / world / HBM_SPEC_GBS, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "layers": len(w.layers), "global_batch": w.batch * world,
                   "batch_per_gpu": w.batch, "seq_len": w.seqlen,
                   "parallelism": f"dp{world} (independent sequences per GPU)",
                   "kv_bytes_per_step_per_gpu": kv_step,
                   "l2": l2_note,
                   "graph": f"{len(w.layers)} gdattn_decode calls per step; one CUDA graph "
                            f"replay holds {ncopy} step(s)"},
        "roofline": roof, "per_layer_type": per_type, "cpu_baseline": cpu,
        "e2e": {"value": job_gbs(kv_step, ms_e2e, world), "unit": "GB/s",
                "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "pinned H2D of every layer's q (+ seqlens) and D2H of every output and "
                       "LSE, in 4 chunks of layers on a side stream overlapping the compute of "
                       "the others, around 48 gdattn_decode calls; the step captured once in a "
                       "CUDA graph and replayed",
                "eager_value": job_gbs(kv_step, ms_e2e_eager, world),
                "eager_ms_per_step": ms_e2e_eager},
        "append": None if ms_app is None else {"value": job_gbs(kv_step, ms_app, world),
                   "unit": "GB/s",
                   "us_per_step": ms_app * 1e3,
                   "how": "the same 48 layers through gdattn_decode_append: each layer's "
                          "current-token K/V rows written into their ring slots by the decode "
                          "kernels (CUDA graph, device time)"},
        "fp8_kv": fp8_summary,
        "multi_query": None if ms_multi is None else {
            "tokens": t_multi,
            "global_us_per_layer": ms_multi / len(global_idx) * 1e3,
            "single_token_global_us_per_layer": ms_gl / len(global_idx) * 1e3,
            "kv_gbs": t_multi * gl_bytes / (ms_multi * 1e-3) / 1e9,
            "how": "the 8 global layers through gdattn_decode_multi with 4 query tokens per "
                   "sequence (a speculative-decoding verify step): a lengths kernel, then one "
                   "decode launch over 4 x 8 query sequences that read the 8 caches (the "
                   "tokens of a sequence share its rows through L2); kv_gbs counts each "
                   "token's window; CUDA graph, device time"},
        "multi_query_sliding": None if not multi_sl else {
            "stack_sliding_us_per_layer": ms_sl / len(sliding_idx) * 1e3,
            **{f"t{t_m}": {"tokens": t_m, "us_per_layer": ms_m / n_multi_sl * 1e3,
                           "vs_single_token": ms_m / multi_sl[1][0],
                           "kv_gbs": b_m / (ms_m * 1e-3) / 1e9,
                           "kv_frac": b_m / (ms_m * 1e-3) / 1e9 / peak,
                           "traffic": traffic_for("multi_t4_sliding") if t_m == 4 else None}
               for t_m, (ms_m, b_m) in sorted(multi_sl.items())},
            "how": "8 sliding layers (rings of window + 7 slots, the stack's batch and "
                   "lengths) through gdattn_decode_multi with 4 and 8 query tokens per "
                   "sequence (8: 7 draft tokens and the last accepted one): one pass over the "
                   "union of the tokens' windows (tc_pair_multi_decode_kernel, split units "
                   "merged in the kernel); t1 is one token through gdattn_decode on the same "
                   "rings, the base of vs_single_token; kv_gbs counts the union once; CUDA "
                   "graph, device time, the 8 layers replayed in turn"},
        "prefill": prefill,
        "gpu_launches": stack.launches_per_step(all_idx) * replays,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gemma4_12b_stack_b8_l8192",
                    choices=sorted(workloads.ALL_WORKLOADS))
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--sections", default="all",
                    help="optional measurements to run beside the timed step, comma "
                         "separated: ceiling, append, fp8, multi, prefill; 'all' (default) "
                         "or 'none' (the step, its layer-type split and e2e only, as for "
                         "profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
