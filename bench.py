#!/usr/bin/env python
"""TPLA decode benchmark: one JSON line on rank 0.

A step is the whole decode hot path for one batch: tpla_append_kv of one new
token per sequence (Hadamard reparameterisation + sliced RMSNorm), then the
split-KV attention and the combine (split merge, W_UV, shard sum).  The
default workload is the DeepSeek-V3 attention shape at TP degree g = 2, one
rank's share (tpla_decode_shard, shard 0), batch 16, 32768 cached tokens per
sequence; every input is seeded synthetic data resident in HBM.  The
per-shard cache (335 MB) is more than twice the 126 MB L2, so consecutive
steps read it from HBM; a workload whose cache is smaller keeps several
replicas of it and each step reads the next one (replicas totalling more than
twice L2), so that its steps read HBM as well.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

Under torchrun (N > 1) every rank runs an independent replica by default; the
reported time is the max over ranks.  With --tp the N ranks are the N shards of
one tensor-parallel decode (N = the workload's g): each rank appends and decodes
its shard and the ranks all-reduce their outputs.
"""

import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "TPLA decode µs/step and latent-cache GB/s (% of B200 HBM peak) at 32K ctx"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024          # B200 L2
MIN_TIMED_S = 0.1                     # attention replays are repeated until they span this long


def cache_replicas(cache_bytes_per_step):
    """Cache copies a workload rotates through so that the bytes read between two reads of the same
    copy exceed twice the L2 (1 when one step already reads that much).  Even, so that the end-to-end
    leg's double-buffered inputs and the replicas cycle together."""
    if cache_bytes_per_step > 2 * L2_BYTES:
        return 1
    n = 2 * L2_BYTES // max(1, cache_bytes_per_step) + 1
    return n + (n & 1)


def l2_note(replicas, cache_bytes_per_step):
    if replicas == 1:
        return "no flush: one step reads %.0f MB of cache, more than twice the 126 MB L2" % (cache_bytes_per_step / 1e6)
    return "rotated: %d cache replicas, %.0f MB read between two reads of one replica (> 2 x L2)" % (
        replicas, replicas * cache_bytes_per_step / 1e6)


def percentile(xs, q):
    xs = sorted(xs)
    if not xs:
        return float("nan")
    k = (len(xs) - 1) * q
    i = int(math.floor(k))
    j = min(i + 1, len(xs) - 1)
    return xs[i] + (xs[j] - xs[i]) * (k - i)


# ---------------------------------------------------------------- workload description

def workload_spec(name):
    from latent_attention_decode_tpla_b200 import inputs as gen
    spec = dict(gen.WORKLOADS[name])
    spec["name"] = name
    spec.setdefault("mode", "shard" if spec["g"] > 1 else "full")
    return spec


def algorithmic_bytes(spec, seq_lens_sum, mode):
    """Bytes the attention stage must read: cache rows (+ queries).  Per shard call: latent slice
    plus RoPE key per token; all shards: the whole latent plus one RoPE key per token."""
    L, R, g, H, B = spec["L"], spec["R"], spec["g"], spec["H"], spec["B"]
    cols = (L // g + R) if mode == "shard" else (L + R)
    cache = seq_lens_sum * cols * 2
    queries = B * H * cols * 2
    return cache, cache + queries


# sources that decide what one launch of a kernel does (its code, the shared schedule, the host-side plan)
KERNEL_SOURCES = {
    "attn_sm100": ["attn_sm100.cu", "attn_sm100_common.cuh", "sm100_ptx.cuh", "tpla_internal.cuh", "api.cu"],
    "attn_sm100_wide": ["attn_sm100_wide.cu", "attn_sm100_common.cuh", "sm100_ptx.cuh", "tpla_internal.cuh",
                        "api.cu"],
}


def source_digest(kernel=None):
    """Digest of the kernel's sources (all of csrc/ when the kernel is not listed)."""
    csrc = os.path.join(ROOT, "latent_attention_decode_tpla_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(os.path.basename(f) for f in glob.glob(os.path.join(csrc, "*")))
    h = hashlib.sha256()
    for name in names:
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """dram bytes per launch from the committed ncu summary, if it was taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "%s_%s.txt" % (kernel, workload))
    if not os.path.exists(path):
        return None
    vals = {}
    for ln in open(path):
        if ":" in ln:
            k, v = ln.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_digest") != source_digest(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            return json.load(open(path)), "measured"
        except ValueError:
            pass
    return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


# ---------------------------------------------------------------- clocks sampling

class ClockSampler:
    """SM clock and throttle reasons while the timed region runs: NVML polled every 2 ms in a thread
    (read-only queries), else nvidia-smi at its shortest period."""
    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, index):
        self.index = index
        self.samples = []          # (sm_mhz, max_mhz, reason names)
        self.stop_flag = threading.Event()
        self.thread = None
        self.nv = None

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.handle = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM))
        except Exception:
            self.nv = None
            return
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def _poll(self):
        nv = self.nv
        masks = {name: getattr(nv, attr, 0) for name, attr in self.REASONS.items()}
        while not self.stop_flag.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((mhz, self.max_mhz, [n for n, m in masks.items() if m and bits & m]))
            except Exception:
                break
            time.sleep(0.002)

    def stop(self):
        if self.nv is None:
            return None
        self.stop_flag.set()
        if self.thread:
            self.thread.join(timeout=2)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        if not self.samples:
            return None
        reasons = sorted({r for _, _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _, _ in self.samples),
                "sm_max_mhz": max(x for _, x, _ in self.samples), "reasons": reasons,
                "samples": len(self.samples), "source": "nvml, 2 ms"}


# ---------------------------------------------------------------- distributed plumbing

def dist_init():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        backend = os.environ.get("BENCH_DIST_BACKEND", backend)     # gloo: several ranks on one GPU (tests)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    if torch.cuda.is_available():
        local = local % torch.cuda.device_count()
    return rank, world, local


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x):
    """Max of a float over ranks (a host-side timing reduction, not a data-path collective)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x):
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- GPU arm

def build_device_workload(spec, seed=0, replicas=1):
    """Seeded synthetic inputs created on the current GPU (bf16 cache N(0,1): unit RMS per shard row);
    ``replicas`` copies of the cache (w["ckvs"], w["kpes"]), the first one also as w["ckv"], w["kpe"]."""
    import torch
    from latent_attention_decode_tpla_b200 import inputs as gen
    from latent_attention_decode_tpla_b200 import tpla
    B, H, L, R, dv, g = spec["B"], spec["H"], spec["L"], spec["R"], spec["dv"], spec["g"]
    lens = gen.workload_seq_lens(spec, seed)
    maxp = gen.pages_for(int(lens.max()))
    num_pages = B * maxp
    gd = torch.Generator(device="cuda")
    gd.manual_seed(1000 * seed + 77)

    def rn(*shape, std=1.0):
        return (torch.randn(*shape, generator=gd, device="cuda", dtype=torch.float32) * std).to(torch.bfloat16)

    w = {}
    w["ckv"] = torch.empty((num_pages, g, 64, L // g), dtype=torch.bfloat16, device="cuda")
    step = max(1, (1 << 27) // (g * 64 * (L // g)))
    for i in range(0, num_pages, step):
        j = min(num_pages, i + step)
        w["ckv"][i:j] = rn(j - i, g, 64, L // g)
    w["kpe"] = rn(num_pages, 64, R)
    w["ckvs"], w["kpes"] = [w["ckv"]], [w["kpe"]]
    for _ in range(1, replicas):
        w["ckvs"].append(w["ckv"].clone())
        w["kpes"].append(w["kpe"].clone())
    w["q"] = rn(B, H, L)
    w["q_pe"] = rn(B, H, R)
    w["w_uv"] = rn(H, L, dv, std=1.0 / math.sqrt(L))
    w["x_new"] = rn(B, L)
    w["kpe_new"] = rn(B, R)
    w["block_table"] = gen.block_table(B, maxp, num_pages, seed).cuda()
    w["seq_lens"] = lens.cuda()
    w["positions"] = (lens - 1).clamp(min=0).cuda()      # the step's token is the newest cached one
    dims = tpla.make_dims(B=B, H=H, L=L, R=R, dv=dv, g=g, max_pages_per_seq=maxp, num_pages=num_pages,
                          softmax_scale=gen.softmax_scale(spec))
    w["dims"] = dims
    w["workspace"] = tpla.alloc_workspace(dims)
    w["out"] = torch.empty((B, H, dv), dtype=torch.float32, device="cuda")
    w["lens_sum"] = int(lens.sum())
    return w


def gpu_step(w, spec, r=0):
    """One step on cache replica r: append one token per sequence, attention, combine."""
    from latent_attention_decode_tpla_b200 import tpla
    shard = 0 if spec["mode"] == "shard" else -1
    d = w["dims"]
    ckv, kpe = w["ckvs"][r], w["kpes"][r]
    tpla.append_kv(d, w["x_new"], w["kpe_new"], spec["transform"], w.get("R_dense"), None, 1e-6,
                   w["positions"], w["block_table"], ckv, kpe)
    tpla.attention(d, shard, w["q"], w["q_pe"], ckv, kpe, w["block_table"], w["seq_lens"], w["workspace"])
    tpla.combine(d, shard, w["seq_lens"], w["w_uv"], w["out"], w["workspace"])


def run_gpu_arm(args, spec, rank, world, local):
    """Times K steps (CUDA events on the launching stream), the attention pass alone over repeated
    replays (median and p90 per launch), then K end-to-end steps."""
    import torch
    from latent_attention_decode_tpla_b200 import inputs as gen
    from latent_attention_decode_tpla_b200 import tpla
    torch.cuda.set_device(local)
    lens = gen.workload_seq_lens(spec, 0)
    cache_b, attn_b = algorithmic_bytes(spec, int(lens.sum()), spec["mode"])
    nrep = cache_replicas(cache_b)
    w = build_device_workload(spec, seed=0, replicas=nrep)
    if spec["transform"] == 2:
        w["R_dense"] = gen.random_orthogonal(spec["L"], 0).cuda()
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        gpu_step(w, spec, i % nrep)
    torch.cuda.synchronize()
    st = tpla.check_device_status()
    if st != tpla.TPLA_OK:
        raise RuntimeError("device status after warm-up: " + tpla.status_string(st))

    K = args.steps
    # The timed steps: K steps captured as one CUDA graph and replayed once, so the timed region holds
    # no host launches; step i reads cache replica i mod nrep.  The attention kernel's own duration
    # comes from a second graph of K attention launches, replayed several times.
    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(K):
                fn(i % nrep)
        g.replay()                                       # untimed: one more warm-up pass
        torch.cuda.synchronize()
        return g
    shard = 0 if spec["mode"] == "shard" else -1
    g_step = capture(lambda r: gpu_step(w, spec, r))
    g_attn = capture(lambda r: tpla.attention(w["dims"], shard, w["q"], w["q_pe"], w["ckvs"][r], w["kpes"][r],
                                              w["block_table"], w["seq_lens"], w["workspace"]))
    ev = lambda: torch.cuda.Event(enable_timing=True)
    start, end = ev(), ev()
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    start.record(stream)
    g_step.replay()
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    # attention alone: replays of the K-launch graph, each timed, until they span MIN_TIMED_S (at
    # least 5), so that the clock sampler sees the load and the spread between replays shows
    per_launch = []
    t_total = 0.0
    while len(per_launch) < 5 or t_total < args.attn_replay_s * 1e3:
        a0, a1 = ev(), ev()
        a0.record(stream)
        g_attn.replay()
        a1.record(stream)
        torch.cuda.synchronize()
        dt = a0.elapsed_time(a1)
        t_total += dt
        per_launch.append(dt / K)
        if len(per_launch) >= 1000:
            break
    clocks = sampler.stop()
    ms = start.elapsed_time(end) / K
    attn_med = statistics.median(per_launch)
    attn_p90 = percentile(per_launch, 0.9)
    ms_max = max_over_ranks(ms)
    attn_ms_max = max_over_ranks(attn_med)
    attn_p90_max = max_over_ranks(attn_p90)

    # End to end through the public API with host buffers: every step copies its inputs from pinned
    # host memory, runs, and its result is copied back and read on the host.  Consecutive steps are
    # pipelined (inputs and outputs double-buffered on the device, copies on their own streams), so
    # the copies of step i+1's inputs and of step i-1's result overlap step i; each step's kernels
    # are replayed from a CUDA graph (one per cache replica; the replica count is even, so replica
    # r always uses input buffer r mod 2).  The step's four bf16 inputs sit side by side in one pinned
    # host buffer and one device buffer, so each step uploads them with a single copy.
    keys = ("q", "q_pe", "x_new", "kpe_new")
    sizes = [w[k].numel() for k in keys]
    offs = [sum(sizes[:i]) for i in range(len(keys))]
    host_buf = torch.empty(sum(sizes), dtype=torch.bfloat16).pin_memory()
    for k, o, n in zip(keys, offs, sizes):
        host_buf[o:o + n].copy_(w[k].reshape(-1).cpu())
    dev_buf = [torch.empty(sum(sizes), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    for d in dev_buf:
        d.copy_(host_buf)
    dev_in = [{k: dev_buf[sb][o:o + n].view(w[k].shape) for k, o, n in zip(keys, offs, sizes)} for sb in range(2)]
    out_dev = [w["out"], torch.empty_like(w["out"])]
    out_host = [torch.empty(w["out"].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = host_buf.numel() * host_buf.element_size()
    d2h = out_host[0].numel() * out_host[0].element_size()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    graphs = []
    for r in range(max(2, nrep)):
        sb = r % 2
        wi = dict(w, out=out_dev[sb], **dev_in[sb])
        gpu_step(wi, spec, r % nrep)                        # outside capture: one-time setup
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            gpu_step(wi, spec, r % nrep)
        graphs.append(g)
    torch.cuda.synchronize()
    evs = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in", "done", "out")}
    e_start, e_end = ev(), ev()
    torch.cuda.synchronize()
    barrier()
    nsteps = 0 if args.no_e2e else K
    e_start.record(up)
    for i in range(nsteps):
        sb = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(evs["done"][sb])          # step i-2 has finished reading these buffers
            dev_buf[sb].copy_(host_buf, non_blocking=True)
            evs["in"][sb].record(up)
        stream.wait_event(evs["in"][sb])
        if i >= 2:
            stream.wait_event(evs["out"][sb])           # step i-2's result has left this buffer
        with torch.cuda.stream(stream):
            graphs[i % len(graphs)].replay()
        evs["done"][sb].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(evs["done"][sb])
            out_host[sb].copy_(out_dev[sb], non_blocking=True)
            evs["out"][sb].record(down)
        if i >= 1:                                      # read step i-1's result on the host
            evs["out"][(i - 1) % 2].synchronize()
            _ = float(out_host[(i - 1) % 2][0, 0, 0])
    if nsteps:
        evs["out"][(nsteps - 1) % 2].synchronize()
        _ = float(out_host[(nsteps - 1) % 2][0, 0, 0])
        e_end.record(down)
    else:
        e_end.record(up)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / K) if not args.no_e2e else float("nan")
    w["out"] = out_dev[0]
    st = tpla.check_device_status()
    if st != tpla.TPLA_OK:
        raise RuntimeError("device status after timing: " + tpla.status_string(st))

    kernel = tpla.get_option(tpla.OPT_LAST_ATTENTION_KERNEL)
    total_cache = sum_over_ranks(cache_b)
    return dict(ms=ms_max, attn_ms=attn_ms_max, attn_p90_ms=attn_p90_max, attn_replays=len(per_launch),
                e2e_ms=e2e_ms, cache_bytes=cache_b, attn_bytes=attn_b, total_cache=total_cache, clocks=clocks,
                h2d=h2d, d2h=d2h, launches=3 * K, kernel=kernel, lens_sum=w["lens_sum"], replicas=nrep)


# ---------------------------------------------------------------- tensor-parallel arm

def run_tp_arm(args, spec, rank, world, local):
    """One TP rank per process (TP degree g = world size, shard = rank): per step, the rank appends its
    slice of one new token per sequence, decodes its shard and all-reduces the [B, H, dv] output
    (latent_attention_decode_tpla_b200.tp).  K steps timed between CUDA events on every rank (a CUDA
    graph when the backend can be captured), the job's time the max over ranks."""
    import torch
    import torch.distributed as dist
    from latent_attention_decode_tpla_b200 import inputs as gen
    from latent_attention_decode_tpla_b200 import tp, tpla
    if spec["g"] != world:
        raise SystemExit("--tp needs the workload's g (%d) processes, got %d" % (spec["g"], world))
    torch.cuda.set_device(local)
    B, H, L, R, dv, g = spec["B"], spec["H"], spec["L"], spec["R"], spec["dv"], spec["g"]
    Ls = L // g
    lens = gen.workload_seq_lens(spec, 0)
    maxp = gen.pages_for(int(lens.max()))
    num_pages = B * maxp
    gd = torch.Generator(device="cuda")
    gd.manual_seed(1000 + 77 + rank)
    rn = lambda *shape, std=1.0: (torch.randn(*shape, generator=gd, device="cuda") * std).to(torch.bfloat16)
    ckv = torch.empty((num_pages, 64, Ls), dtype=torch.bfloat16, device="cuda")
    step_rows = max(1, (1 << 27) // (64 * Ls))
    for i in range(0, num_pages, step_rows):
        ckv[i:i + step_rows] = rn(min(step_rows, num_pages - i), 64, Ls)
    kpe = rn(num_pages, 64, R)
    q_local, q_pe = rn(B, H, Ls), rn(B, H, R)
    w_local = rn(H, Ls, dv, std=1.0 / math.sqrt(L))
    x_new, kpe_new = rn(B, L), rn(B, R)
    bt = gen.block_table(B, maxp, num_pages, 0).cuda()
    sl = lens.cuda()
    positions = (lens - 1).clamp(min=0).cuda()
    dims = tpla.make_dims(B=B, H=H, L=L, R=R, dv=dv, g=g, max_pages_per_seq=maxp, num_pages=num_pages,
                          softmax_scale=gen.softmax_scale(spec))
    r = tp.TensorParallelDecode(dims)
    ws = r.workspace()
    out = torch.empty((B, H, dv), dtype=torch.float32, device="cuda")
    R_dense = gen.random_orthogonal(L, 0).cuda() if spec["transform"] == 2 else None

    def step():
        r.append(x_new, kpe_new, spec["transform"], R_dense, None, 1e-6, positions, bt, ckv, kpe)
        r.decode(q_local, q_pe, ckv, kpe, bt, sl, w_local, out, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    graph = None
    if dist.get_backend() == "nccl":
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(K):
                    step()
            graph.replay()
            torch.cuda.synchronize()
        except Exception:
            graph = None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record()
    if graph is not None:
        graph.replay()
    else:
        for _ in range(K):
            step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / K)
    st = tpla.check_device_status()
    if st != tpla.TPLA_OK:
        raise RuntimeError("device status after timing: " + tpla.status_string(st))
    timed = "one CUDA graph of K steps" if graph is not None else "K eager steps"
    del graph                                  # release a graph holding collectives before the group goes
    cache_rank = int(lens.sum()) * (Ls + R) * 2
    total = sum_over_ranks(cache_rank)
    if rank != 0:
        return None
    cfg = config_of(spec, "no flush: %.0f MB of cache per rank per step" % (cache_rank / 1e6))
    cfg.update({"entry": "tensor parallel: per rank tpla_append_kv_shard + tpla_decode (L/g wide) + all_reduce",
                "parallelism": "tp%d" % world})
    return {"metric": METRIC, "value": total / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms, "us_per_step": ms * 1e3,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "backend": dist.get_backend(),
            "timed": timed,
            "gpu_launches": 3 * K}


# ---------------------------------------------------------------- oracle (CPU) arm

def oracle_sample(spec, seed=0, T=None):
    """One sequence of the workload (shard 0 for per-shard workloads) as CPU float64 arrays."""
    import numpy as np
    import torch
    from latent_attention_decode_tpla_b200 import inputs as gen
    lens = gen.workload_seq_lens(spec, seed)
    T = int(lens.max()) if T is None else T
    d = gen.make_workload(B=1, H=spec["H"], L=spec["L"], R=spec["R"], dv=spec["dv"], g=spec["g"], seq_lens=[T],
                          seed=seed, extra_pages=0)
    f = lambda t: t.to(torch.float64).numpy()
    s = dict(q=f(d["q"]), q_pe=f(d["q_pe"]), ckv=f(d["ckv"]), kpe=f(d["kpe"]), bt=d["block_table"].numpy(),
             w_uv=f(d["w_uv"]), x_new=f(d["x_new"]), kpe_new=f(d["kpe_new"]), T=T,
             maxp=d["max_pages_per_seq"])
    if spec["transform"] == 2:
        s["R_dense"] = gen.random_orthogonal(spec["L"], seed).numpy().astype(np.float64)
    return s


def oracle_step(spec, s):
    """The oracle's version of one step on the sample: append one token, then decode."""
    from latent_attention_decode_tpla_b200 import inputs as gen
    from oracle import tpla_ref as ref
    scale = gen.softmax_scale(spec)
    ref.append_kv(s["x_new"], s["kpe_new"], [s["T"] - 1], s["bt"], s["ckv"], s["kpe"], g=spec["g"],
                  max_pages_per_seq=s["maxp"], transform=spec["transform"], R_dense=s.get("R_dense"), eps=1e-6)
    if spec["mode"] == "shard":
        return ref.decode_shard(s["q"], s["q_pe"], s["ckv"], s["kpe"], s["bt"], [s["T"]], scale, 0,
                                max_pages_per_seq=s["maxp"], w_uv=s["w_uv"])
    return ref.decode(s["q"], s["q_pe"], s["ckv"], s["kpe"], s["bt"], [s["T"]], scale,
                      max_pages_per_seq=s["maxp"], w_uv=s["w_uv"])


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _time_oracle(spec, s, budget_s):
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(spec, s)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return n, time.perf_counter() - t0


def cpu_baseline(spec, budget_s=12.0, single_core_budget_s=6.0):
    """Time the oracle on a bounded sample: repeated single-sequence steps until ~budget_s with the
    BLAS threads of the host, then until ~single_core_budget_s on one thread."""
    s = oracle_sample(spec)
    cols = (spec["L"] // spec["g"] + spec["R"]) if spec["mode"] == "shard" else (spec["L"] + spec["R"])
    n, dt = _time_oracle(spec, s, budget_s)
    bytes_step = s["T"] * cols * 2
    out = {"value": n * bytes_step / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
           "sample": "%d oracle step(s) of 1 sequence x %d tokens (%s, all %d heads) in %.1f s; float64 numpy"
                     % (n, s["T"], "shard 0" if spec["mode"] == "shard" else "all shards", spec["H"], dt)}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            n1, dt1 = _time_oracle(spec, s, single_core_budget_s)
        out["single_core"] = {"value": n1 * bytes_step / dt1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": "%d oracle step(s) of the same sequence in %.1f s, BLAS limited to one "
                                        "thread" % (n1, dt1)}
    except Exception as e:          # threadpoolctl missing: report why, keep the multi-core figure
        out["single_core"] = {"unavailable": str(e)}
    return out


def run_reference(args, spec, rank):
    if rank != 0:
        return None
    s = oracle_sample(spec)
    cols = (spec["L"] // spec["g"] + spec["R"]) if spec["mode"] == "shard" else (spec["L"] + spec["R"])
    for _ in range(args.warmup):
        oracle_step(spec, s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(spec, s)
    dt = (time.perf_counter() - t0) / args.steps
    gbs = s["T"] * cols * 2 / dt / 1e9
    sample = "each step: oracle append + decode of 1 sequence x %d tokens (of the %d-sequence workload)" % (
        s["T"], spec["B"])
    return {"metric": METRIC, "value": gbs, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(spec),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def config_of(spec, l2=None):
    T = spec["T"]
    return {"workload": spec["name"], "entry": "tpla_decode_shard(shard 0)" if spec["mode"] == "shard"
            else ("mla_decode" if spec["g"] == 1 else "tpla_decode (all shards, on-chip sum)"),
            "batch": spec["B"], "heads": spec["H"], "kv_lora_rank": spec["L"], "rope_dim": spec["R"],
            "v_head_dim": spec["dv"], "shards_g": spec["g"],
            "context": T if not isinstance(T, tuple) else "uniform[%d,%d]" % T,
            "transform": {0: "none", 1: "hadamard", 2: "dense orthogonal (seeded QR)"}[spec["transform"]],
            "page_size": 64, "step": "append 1 token/seq + split-KV attention + combine",
            "l2": l2 if l2 is not None else "not applicable (oracle on the host)"}


# ---------------------------------------------------------------- main

def run_prefill(args, rank):
    """MLA-form prefill of one T-token prompt (DeepSeek-V3 shape, g = 2 cache for the decode that follows),
    timed with CUDA events over K prefills after W warm-ups.  The work is the absorbed form's causal
    attention: per query t and key i <= t, 2H(L+R) + 2HL FLOPs (scores and output over the whole latent),
    plus the W_UV projection of every output row; the line reports prompt tokens per second and the
    tensor-pipe roofline against the measured bf16 peak."""
    if rank != 0:
        return None
    import torch
    from latent_attention_decode_tpla_b200 import inputs as gen
    from latent_attention_decode_tpla_b200 import prefill, tpla
    T, H, L, R, dv, g = args.prefill, 128, 512, 64, 128, 2
    gcpu = torch.Generator().manual_seed(0)
    bf = lambda t: t.to(torch.bfloat16).cuda()
    x, kpe = bf(torch.randn(T, L, generator=gcpu)), bf(torch.randn(T, R, generator=gcpu))
    q, q_pe = bf(torch.randn(T, H, L, generator=gcpu)), bf(torch.randn(T, H, R, generator=gcpu))
    w_uv = bf(torch.randn(H, L, dv, generator=gcpu) / math.sqrt(L))
    maxp = (T + 63) // 64
    dims = tpla.make_dims(B=1, H=H, L=L, R=R, dv=dv, g=g, max_pages_per_seq=maxp, num_pages=maxp,
                          softmax_scale=1 / math.sqrt(192))
    ckv = torch.zeros((maxp, g, 64, L // g), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((maxp, 64, R), dtype=torch.bfloat16, device="cuda")
    row = torch.arange(maxp, dtype=torch.int32, device="cuda")
    out = torch.empty((T, H, dv), dtype=torch.float32, device="cuda")
    run = lambda: prefill.mla_prefill(dims, x, kpe, q, q_pe, w_uv, tpla.TRANSFORM_HADAMARD, None, None, 1e-6, row,
                                      ckv, kc, out, chunk=args.prefill_chunk)
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    if tpla.check_device_status() != tpla.TPLA_OK:
        raise RuntimeError("device status after the prefill warm-up")
    sampler = ClockSampler(0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.start()
    e0.record()
    for _ in range(args.steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    pairs = T * (T + 1) // 2
    flops = pairs * (2 * H * (L + R) + 2 * H * L) + T * 2 * H * L * dv
    peaks, kind = measured_peaks()
    peak = float(peaks.get("bf16_tflops", 1590.0))
    achieved = flops / (ms * 1e-3) / 1e12
    return {"metric": "MLA-form prefill prompt tokens/s", "value": T / (ms * 1e-3), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_prefill": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "mla_prefill_dsv3_%d" % T, "prompt": T, "heads": H, "kv_lora_rank": L,
                       "rope_dim": R, "v_head_dim": dv, "decode_shards_g": g, "transform": "hadamard",
                       "form": "absorbed MLA attention over the prompt (one-shard tcgen05 kernel), chunks of %d" % args.prefill_chunk},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None, "peak_kind": kind,
                         "flops_per_prefill": flops},
            "clocks": clocks}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="tpla_g2_dsv3_b16_32k")
    ap.add_argument("--mode", default=None, choices=[None, "shard", "full"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling)")
    ap.add_argument("--tp", action="store_true",
                    help="tensor parallel across the processes (TP degree = world size = the workload's g)")
    ap.add_argument("--tile", type=int, default=0, choices=[0, 64, 128],
                    help="tokens per tile of the tcgen05 kernel for L/g <= 256 (0: the library default)")
    ap.add_argument("--attn-replay-s", type=float, default=MIN_TIMED_S,
                    help="seconds the attention-only replays span at least (5 replays at least)")
    ap.add_argument("--prefill", type=int, default=0,
                    help="time the MLA-form prefill of a prompt of this many tokens instead of decode")
    ap.add_argument("--prefill-chunk", type=int, default=64, help="prompt tokens per attention call of the prefill")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    spec = workload_spec(args.workload)
    if args.mode:
        spec["mode"] = args.mode
    if args.batch:
        spec["B"] = args.batch
        spec["name"] = spec["name"] + "_batch%d" % args.batch

    rank, world, local = dist_init()
    if args.impl == "reference":
        line = run_reference(args, spec, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if args.tile:
        from latent_attention_decode_tpla_b200 import tpla
        tpla.set_option(tpla.OPT_TILE_TOKENS, args.tile)
    if args.prefill:
        line = run_prefill(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.tp:
        line = run_tp_arm(args, spec, rank, world, local)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    r = run_gpu_arm(args, spec, rank, world, local)
    if rank != 0:
        return
    peaks, peak_kind = measured_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    value = r["total_cache"] / (r["ms"] * 1e-3) / 1e9
    achieved = r["attn_bytes"] / (r["attn_ms"] * 1e-3) / 1e9
    kernel_name = {1: "attn_simt", 2: "attn_sm100", 3: "attn_sm100_wide"}.get(r["kernel"], "unknown")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"], "us_per_step": r["ms"] * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_of(spec, l2_note(r["replicas"], r["cache_bytes"])),
        "hbm_frac_step": value / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(kernel_name, spec["name"]),
                     "kernel": kernel_name + " (tpla_attention)", "peak_kind": peak_kind,
                     "bytes_per_launch": r["attn_bytes"], "us_per_launch": r["attn_ms"] * 1e3,
                     "us_per_launch_p90": r["attn_p90_ms"] * 1e3, "replays": r["attn_replays"],
                     "achieved_p90": r["attn_bytes"] / (r["attn_p90_ms"] * 1e-3) / 1e9},
        "e2e": None if args.no_e2e else {
            "value": r["total_cache"] / (r["e2e_ms"] * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"], "ms_per_step": r["e2e_ms"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(spec)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
    try:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass
