#!/usr/bin/env python
"""Benchmark of one Fathom decode step: allocation + bit-plane scan + top-k.

Default workload: the 1M-token decode step -- n = 1,048,576 keys, 8 KV heads x
d = 128 channels stored as 4-bit channel-major bit planes (512 MiB), 32 bf16
query heads (GQA 4), budget B = 92 bits per key, top-k = 2048 per query head.
Other workloads (--config): qwen3_8b_layer_131k, host_resident_1m (planes in
pinned host memory, read across the host link), ragged_32_sessions (one
batched launch set for 32 sessions), tiny_4k.  Inputs are seeded synthetic
(synthkv); the planes are packed once, before timing.

One step = fathom_allocate + fathom_scan_topk (plan, sample scan, threshold,
filtering scan, merge).  Device time per step comes from CUDA events on the
launching stream; L2 is flushed (256 MiB write) between steps, outside the
events.  The dominant kernel (the filtering scan) is timed alone with events
the library records around it, in K further steps: an event between two
kernels breaks their programmatic dependent launch, so the step time is
taken without them.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--config NAME] [--budget B]

Under torchrun each rank scores its own session (seed + rank): weak scaling,
no collective on the data path; the step time is the max over ranks.
--impl reference times the CPU oracle (the reference arm of this workload) on
a bounded sample of the same step.
"""

from __future__ import annotations

import argparse
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Gkeys/s scanned+top-k at 1M ctx, B=92 bits; achieved HBM GB/s vs B200 peak"
UNIT = "Gkeys/s"
FLUSH_BYTES = 256 << 20
def launches_per_step(n_max, k):
    """Our kernels per step: allocate, plan, filtering scan and merge, plus
    the sample scan and threshold when the longest session is sampled (the
    library samples a session of n >= 512 r keys, r = max(16, ceil(k / 32)))."""
    r = max(16, (k + 31) // 32)
    return 6 if n_max >= 512 * r else 4


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", default="decode_1m")
    ap.add_argument("--budget", type=int, default=92)
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--cuda-cores", action="store_true",
                    help="run the scan on the CUDA-core kernel instead of the tcgen05 kernel")
    ap.add_argument("--uniform", action="store_true",
                    help="allocate the budget query-independently (the same depth in every "
                         "channel, fathom_allocate_uniform) instead of by water-filling")
    ap.add_argument("--token-group", type=int, default=0,
                    help="quantiser statistics per run of this many keys (a multiple of 65536; "
                         "0 = per channel over the context)")
    ap.add_argument("--append", action="store_true",
                    help="also time fathom_append_planes: one decoded token into the store, "
                         "in place, and a 128-token append that lengthens the rows")
    ap.add_argument("--attention", action="store_true",
                    help="also time the sparse attention over each head's top-k (the step after "
                         "the scan; random bf16 K/V rows of the workload's shape), outside the step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args(argv)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ timing --

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "reasons": sorted(reasons), "samples": len(sm)}


_libcuda = None


def event_ms(a, b) -> float:
    """Elapsed ms between two torch CUDA events recorded by any runtime (the
    library records the scan-kernel events itself, which torch's own
    elapsed_time refuses), through the driver's cuEventElapsedTime."""
    import ctypes
    global _libcuda
    if _libcuda is None:
        _libcuda = ctypes.CDLL("libcuda.so.1")
        _libcuda.cuEventElapsedTime.restype = ctypes.c_int
        _libcuda.cuEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p,
                                                ctypes.c_void_p]
    ms = ctypes.c_float(0.0)
    rc = _libcuda.cuEventElapsedTime(ctypes.byref(ms), ctypes.c_void_p(a.cuda_event),
                                     ctypes.c_void_p(b.cuda_event))
    if rc != 0:
        raise RuntimeError("cuEventElapsedTime failed: %d" % rc)
    return float(ms.value)


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ------------------------------------------------------------ multi-rank --

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(x: float, world: int, device=None) -> float:
    """The max of x over all ranks (every rank calls it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_throughput(keys_this_rank: float, ms_this_rank: float, world: int, device=None):
    """Whole-job keys/s (in G): all ranks' keys over the slowest rank's time."""
    keys = reduce_sum(keys_this_rank, world, device)
    ms = reduce_max(ms_this_rank, world, device)
    return keys / (ms * 1e-3) / 1e9, ms


def get_cfg(name):
    import synthkv
    cfg = dict(synthkv.CONFIGS[name])
    cfg["name"] = name
    return cfg



def code_digest(path):
    """sha256 of a C++/CUDA source with its comments and blank lines removed,
    so that an edit to comments alone keeps a profile's counters valid."""
    import hashlib
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.split("\n")]
    code = "\n".join(ln for ln in lines if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()


def profiled_traffic(workload, kernel_source):
    """DRAM bytes (read + write) per launch of the filtering scan, from the ncu
    summaries under profiles/ -- only while the kernel source (comments aside)
    hashes to the one the counters were taken on and the workload matches;
    else None."""
    import glob
    src = os.path.join(ROOT, kernel_source)
    if not os.path.exists(src):
        return None
    digest = code_digest(src)
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        fields = {}
        with open(path) as f:
            for line in f:
                m = re.match(r"^(traffic_bytes_per_launch|kernel_source|kernel_code_sha256|workload): (\S+)$",
                             line.strip())
                if m:
                    fields[m.group(1)] = m.group(2)
        if (fields.get("kernel_source") == kernel_source and fields.get("workload") == workload
                and fields.get("kernel_code_sha256") == digest
                and "traffic_bytes_per_launch" in fields):
            return int(fields["traffic_bytes_per_launch"])
    return None

def workload_desc(cfg, budget, k, uniform=False, token_group=0):
    how = (", uniform allocation (the same depth in every channel for every query head)"
           if uniform else "")
    if token_group:
        how += ", quantiser statistics per %d-key token group" % token_group
    if cfg["name"] == "ragged_32_sessions":
        return ("ragged_32_sessions: 32 sessions, n ~ U[%d, %d] keys each, %d KV heads x d=%d, "
                "%d %s query heads (GQA %d), B=%d bits/key%s, top-k=%d, one batched launch set" % (
                    cfg["n_lo"], cfg["n_hi"], cfg["h_kv"], cfg["d"], cfg["h_q"], cfg["q_dtype"],
                    cfg["h_q"] // cfg["h_kv"], budget, how, k))
    where = " in pinned host memory" if cfg["name"] == "host_resident_1m" else ""
    return ("%s: n=%d keys, %d KV heads x d=%d (4-bit channel-major bit planes%s), %d %s query "
            "heads (GQA %d), B=%d bits/key%s, top-k=%d" % (
                cfg["name"], cfg["n"], cfg["h_kv"], cfg["d"], where, cfg["h_q"], cfg["q_dtype"],
                cfg["h_q"] // cfg["h_kv"], budget, how, k))


def union_plane_bytes(alloc, n, h_kv, words):
    """Bytes of the union prefixes one step reads: per KV head, for every
    channel, the longest prefix any of its query heads was allocated, each
    plane a row of `words` 32-bit words."""
    a = np.asarray(alloc)
    G = a.shape[0] // h_kv
    tstar = a.reshape(h_kv, G, -1).max(axis=1)
    return int(tstar.sum()) * words * 4


# ------------------------------------------------------------ CPU oracle --

def oracle_sample(case_np, budget, k, heads, uniform=False, token_group=0):
    """Oracle allocation + scores + top-k for the listed query heads; returns seconds."""
    import oracle
    codes, qmin, qscale, q, sigma = case_np
    G = q.shape[0] // codes.shape[0]
    d = q.shape[1]
    t0 = time.perf_counter()
    for h in heads:
        g = h // G
        if uniform:
            t = oracle.allocate_uniform(1, d, budget)[0]
        else:
            t = oracle.allocate(q[h], sigma[g], budget)
        if token_group:
            s = oracle.scores_from_codes_grouped(codes[g], qmin[g], qscale[g], q[h], t, token_group)
        else:
            s = oracle.scores_from_codes(codes[g], qmin[g], qscale[g], q[h], t)
        oracle.topk(s, k)
    return time.perf_counter() - t0


def case_numpy(case):
    return (case.codes.cpu().numpy(), case.qmin.cpu().numpy(), case.qscale.cpu().numpy(),
            case.q.cpu().numpy().astype(np.float64), case.sigma.cpu().numpy())


def run_reference(args):
    """The reference arm: the CPU oracle on a bounded sample of the same step."""
    import torch
    world, rank, local = dist_setup()
    if rank != 0:
        return
    cfg = get_cfg(args.config)
    k = args.k or cfg["k"]
    import oracle
    import synthkv
    oracle.build()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if cfg["name"] == "ragged_32_sessions":
        case = synthkv.make_ragged(cfg["seed"], 1, cfg["n_lo"], cfg["n_hi"], cfg["h_kv"],
                                   cfg["h_q"], cfg["d"], cfg["q_dtype"], device=dev)[0]
    else:
        case = synthkv.make_case(cfg["seed"], cfg["n"], cfg["h_kv"], cfg["h_q"], cfg["d"],
                                 cfg["q_dtype"], device=dev, keep_keys=False,
                                 token_group=args.token_group)
    cn = case_numpy(case)
    tg = args.token_group if cfg["name"] != "ragged_32_sessions" else 0
    for i in range(args.warmup):
        oracle_sample(cn, args.budget, k, [i % cfg["h_q"]], args.uniform, tg)
    secs = [oracle_sample(cn, args.budget, k, [(args.warmup + i) % cfg["h_q"]], args.uniform, tg)
            for i in range(args.steps)]
    t = float(np.mean(secs))
    value = case.n / t / 1e9
    sample = ("one query head per step (allocation, fp64 scores of all %d keys, brute-force "
              "top-%d), single thread" % (case.n, k))
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, synthkv)",
        "config": {"workload": workload_desc(cfg, args.budget, k, args.uniform, tg),
                   "budget_bits": args.budget,
                   "k": k, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


# ---------------------------------------------------------------- native --

def measure_h2d_gbs(device, nbytes=512 << 20):
    """Pinned host -> device copy bandwidth, the host link's measured peak."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    for _ in range(2):
        dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = 0.0
    for _ in range(5):
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del src, dst
    return best


def run_native(args):
    import torch
    world, rank, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl native needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    import bit_plane_kv_scan_b200 as F
    from bit_plane_kv_scan_b200 import build as fbuild
    import synthkv
    fbuild.build()

    cfg = get_cfg(args.config)
    k = args.k or cfg["k"]
    B = args.budget
    h_kv, h_q, d = cfg["h_kv"], cfg["h_q"], cfg["d"]
    flags = F.FLAG_CUDA_CORES if args.cuda_cores else 0
    ragged = cfg["name"] == "ragged_32_sessions"
    host = cfg["name"] == "host_resident_1m"
    tg = args.token_group
    if tg and ragged:
        raise SystemExit("--token-group applies to the single-session workloads")
    ws = F.Workspace(device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    if ragged:
        cases = synthkv.make_ragged(cfg["seed"] + 1000 * rank, cfg["sessions"], cfg["n_lo"],
                                    cfg["n_hi"], h_kv, h_q, d, cfg["q_dtype"], device=device)
    else:
        cases = [synthkv.make_case(cfg["seed"] + rank, cfg["n"], h_kv, h_q, d, cfg["q_dtype"],
                                   device=device, keep_keys=False, token_group=tg)]
    S = len(cases)
    q_all = torch.cat([c.q_storage() for c in cases]).contiguous()
    sigma_all = torch.cat([c.sigma for c in cases]).contiguous()
    alloc_all = torch.empty((S * h_q, d), dtype=torch.uint8, device=device)
    planes = []
    for c in cases:
        p = F.pack_planes(c.codes)
        if host:
            hp = torch.empty(p.shape, dtype=p.dtype, pin_memory=True)
            hp.copy_(p)
            p = hp
        planes.append(p)
        c.codes = None  # the scan reads only the planes
    torch.cuda.synchronize()
    outs = [(torch.empty((h_q, k), dtype=torch.int32, device=device),
             torch.empty((h_q, k), dtype=torch.float32, device=device)) for _ in range(S)]
    n_total = sum(c.n for c in cases)
    n_max_cfg = max(c.n for c in cases)

    def allocate(q_src):
        if args.uniform:
            F.allocate_uniform(S * h_q, d, B, out=alloc_all)
        else:
            F.allocate(q_src, sigma_all, B, out=alloc_all)

    def make_step(q_src):
        if ragged:
            descs = [dict(planes=planes[i], qmin=cases[i].qmin, qscale=cases[i].qscale,
                          q=q_src[i * h_q:(i + 1) * h_q], alloc=alloc_all[i * h_q:(i + 1) * h_q],
                          n=cases[i].n, out_idx=outs[i][0], out_score=outs[i][1])
                     for i in range(S)]
            scan = F.BatchedScan(descs, k, d, h_q, h_kv, q_src.dtype, flags=flags,
                                 device=device)

            def step():
                allocate(q_src)
                scan(ws)
        else:
            c = cases[0]

            def step():
                allocate(q_src)
                F.scan_topk(planes[0], c.qmin, c.qscale, q_src, alloc_all, k, c.n,
                            host_mapped=host, flags=flags, workspace=ws, out=outs[0],
                            token_group=tg)
        return step

    step = make_step(q_all)
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    K = args.steps
    sb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    se = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    kb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for ev in kb + ke:  # torch creates an event's handle at its first record
        ev.record(stream)
    sampler = ClockSampler(physical_gpu_index(local))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    for i in range(K):
        flush.zero_()
        sb[i].record(stream)
        step()
        se[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    # The filtering scan alone, timed with events the library records around
    # it in K more steps: events between two kernels break their dependent
    # launch, so the step time above is taken without them.
    for i in range(K):
        flush.zero_()
        F.profile_scan_kernel(kb[i], ke[i])
        step()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    F.profile_scan_kernel(None, None)
    step_ms = float(np.mean([a.elapsed_time(b) for a, b in zip(sb, se)]))
    kern_ms = float(np.mean([event_ms(a, b) for a, b in zip(kb, ke)]))
    rep = F.read_report(ws)
    keys_per_step = h_q * n_total
    value, t_step = job_throughput(keys_per_step, step_ms, world, device)
    t_kern = reduce_max(kern_ms, world, device)

    # algorithmic bytes of the filtering scan: the union plane prefixes of
    # every (session, KV head) plus the small per-head inputs (q, alloc, m, s)
    alloc_np = alloc_all.cpu().numpy()
    union_bytes = sum(union_plane_bytes(alloc_np[i * h_q:(i + 1) * h_q], c.n, h_kv,
                                        F.plane_words(c.n)) for i, c in enumerate(cases))
    small_bytes = S * (h_q * d * (q_all.element_size() + 1) + 2 * h_kv * d * 4)
    alg_bytes = union_bytes + small_bytes
    achieved = alg_bytes / (kern_ms * 1e-3) / 1e9
    if host:
        peak, peak_kind, bound = measure_h2d_gbs(device), "measured pinned host->device copy", \
            "host-link"
    else:
        peak, peak_kind = load_peaks()
        bound = "hbm"

    # end to end through the public API with host buffers: q uploaded from
    # pinned memory, top-k read back to pinned memory, inside the timed region
    q_host = q_all.cpu().pin_memory()
    q_dev = torch.empty_like(q_all)
    out_host = [(torch.empty((h_q, k), dtype=torch.int32, pin_memory=True),
                 torch.empty((h_q, k), dtype=torch.float32, pin_memory=True)) for _ in range(S)]
    inner = make_step(q_dev)

    def e2e_step():
        q_dev.copy_(q_host, non_blocking=True)
        inner()
        for (hi, hs), (di, ds) in zip(out_host, outs):
            hi.copy_(di, non_blocking=True)
            hs.copy_(ds, non_blocking=True)

    eb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for _ in range(3):
        flush.zero_()
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    for i in range(K):
        flush.zero_()
        eb[i].record(stream)
        e2e_step()
        ee[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms_local = float(np.mean([a.elapsed_time(b) for a, b in zip(eb, ee)]))
    e2e_value, e2e_ms = job_throughput(keys_per_step, e2e_ms_local, world, device)
    h2d = q_host.numel() * q_host.element_size()
    d2h = S * h_q * k * 8

    append = None
    if args.append and not ragged and not host:
        # a decode step's append: the store of the first n - 256 tokens takes the
        # next tokens one at a time (in place: the row length holds), then 128
        # at once across a row-length boundary (a copy into the longer layout)
        n1 = cases[0].n
        codes = synthkv.make_case(cfg["seed"] + rank, n1, h_kv, h_q, d, cfg["q_dtype"],
                                  device=device, keep_keys=False, token_group=tg).codes
        n0 = n1 - 256
        store = F.pack_planes(codes[:, :n0].contiguous())
        one = [codes[:, n0 + i:n0 + i + 1].contiguous() for i in range(64)]
        torch.cuda.synchronize()
        ab = [torch.cuda.Event(enable_timing=True) for _ in range(64)]
        ae = [torch.cuda.Event(enable_timing=True) for _ in range(64)]
        for i in range(64):
            ab[i].record(stream)
            store = F.append_planes(store, n0 + i, one[i])
            ae[i].record(stream)
        torch.cuda.synchronize()
        t_one = float(np.median([x.elapsed_time(y) for x, y in zip(ab[3:], ae[3:])]))
        n2 = n0 + 64
        n2r = ((n2 + 127) // 128) * 128  # fill to the row boundary, then cross it
        store = F.append_planes(store, n2, codes[:, n2:n2r].contiguous())
        blk = codes[:, n2r:n2r + 128].contiguous()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        grown = F.append_planes(store, n2r, blk)
        e1.record(stream)
        torch.cuda.synchronize()
        t_grow = e0.elapsed_time(e1)
        moved = 2 * F.lib().fathom_planes_bytes(n2r, d, h_kv)  # read and written once
        hbm_peak, hbm_kind = load_peaks()
        append = {"kernels": ["append_bits_kernel", "append_copy_kernel"],
                  "one_token_in_place_us": t_one * 1e3,
                  "grow_128_tokens_us": t_grow * 1e3,
                  "grow_bytes": moved, "grow_achieved_gbs": moved / (t_grow * 1e-3) / 1e9,
                  "grow_frac": moved / (t_grow * 1e-3) / 1e9 / hbm_peak, "peak_kind": hbm_kind}
        del store, grown, codes, one, blk

    attention = None
    if args.attention and not ragged:
        # the step after the scan, timed on its own: each head's attention over
        # the top-k rows this step selected, with random bf16 values and keys
        # either as bf16 rows or as 4-bit codes (dequantised in the gather),
        # in device memory or in pinned host memory (only the selected rows
        # cross the host link)
        gen = torch.Generator(device=device).manual_seed(1234 + rank)
        n1 = cases[0].n
        v_rows = torch.randn((h_kv, n1, d), generator=gen, device=device).to(torch.bfloat16)
        k_rows = torch.randn((h_kv, n1, d), generator=gen, device=device).to(torch.bfloat16)
        k_codes = torch.randint(0, 256, (h_kv, n1, d // 2), generator=gen, device=device,
                                dtype=torch.uint8)
        idx = outs[0][0]
        a_out = torch.empty((h_q, d), dtype=torch.float32, device=device)
        a_lse = torch.empty((h_q,), dtype=torch.float32, device=device)
        rows = int(((idx >= 0) & (idx < n1)).sum().item())
        small = idx.numel() * 4 + q_all.numel() * q_all.element_size() + a_out.numel() * 4 + \
            a_lse.numel() * 4
        hbm_peak, hbm_kind = load_peaks()

        def time_attn(call):
            for _ in range(3):
                call()
            ab = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
            ae = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
            for i in range(K):
                flush.zero_()
                ab[i].record(stream)
                call()
                ae[i].record(stream)
            torch.cuda.synchronize()
            return float(np.mean([x.elapsed_time(y) for x, y in zip(ab, ae)]))

        def entry(name, ms, row_bytes, peak, kind, link):
            b = rows * row_bytes + small
            gbs = b / (ms * 1e-3) / 1e9
            return {"variant": name, "ms": ms, "rows": rows, "algorithmic_bytes": b,
                    "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                    "peak_kind": kind, "bound": link}

        qs = dict(k_qmin=cases[0].qmin, k_qscale=cases[0].qscale)
        ents = []
        ms = time_attn(lambda: F.sparse_attention(q_all, k_rows, v_rows, idx, out=a_out, lse=a_lse))
        ents.append(entry("bf16 K, bf16 V, device", ms, 4 * d, hbm_peak, hbm_kind, "hbm"))
        ms = time_attn(lambda: F.sparse_attention(q_all, None, v_rows, idx, out=a_out, lse=a_lse,
                                                  k_codes=k_codes, **qs))
        ents.append(entry("4-bit K, bf16 V, device", ms, 2 * d + d // 2, hbm_peak, hbm_kind, "hbm"))
        del k_rows
        hv = v_rows.cpu().pin_memory()
        hc = k_codes.cpu().pin_memory()
        link = measure_h2d_gbs(device)
        ms = time_attn(lambda: F.sparse_attention(q_all, None, hv, idx, out=a_out, lse=a_lse,
                                                  k_codes=hc, host_mapped=True, **qs))
        ents.append(entry("4-bit K, bf16 V, pinned host memory", ms, 2 * d + d // 2, link,
                          "measured pinned host->device copy", "host-link"))
        attention = {"kernel": "attention_kernel", "k": k, "l2": "flushed before each launch",
                     "variants": ents}
        del v_rows, k_codes, hv, hc

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not ragged:
        import oracle
        oracle.build()
        c = cases[0]
        c.codes = synthkv.make_case(cfg["seed"], cfg["n"], h_kv, h_q, d, cfg["q_dtype"],
                                    device=device, keep_keys=False, token_group=tg).codes
        cn = case_numpy(c)
        heads = list(range(min(8, h_q)))
        secs = oracle_sample(cn, B, k, heads, args.uniform, tg)
        cpu = {"value": len(heads) * c.n / secs / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": "query heads 0-%d of this step: allocation, fp64 scores of all %d "
                         "keys, brute-force top-%d; single thread, %.1f s"
                         % (len(heads) - 1, c.n, k, secs)}

    if rank == 0:
        traffic = None
        if not ragged and not host:
            traffic = profiled_traffic("%s_b%d%s%s" % (cfg["name"], B, "_uniform" if args.uniform else "",
                                                        "_tg%d" % tg if tg else ""),
                                       "bit_plane_kv_scan_b200/csrc/scan.cu"
                                       if flags else "bit_plane_kv_scan_b200/csrc/scan_tc.cu")
        res = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": t_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded, synthkv: Qwen3-8B-shaped GQA keys with outlier "
                    "channels, 4-bit min-max codes)",
            "config": {"workload": workload_desc(cfg, B, k, args.uniform, tg), "sessions_per_rank": S,
                       "keys_per_rank": n_total, "h_kv": h_kv, "h_q": h_q, "d": d,
                       "budget_bits": B, "k": k, "scan_kernel": "cuda-core" if flags else "tcgen05",
                       "allocation": "uniform" if args.uniform else "water-filling",
                       "l2": "flushed between steps (256 MiB write, outside the events)"},
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_kind": peak_kind, "kernel": "filtering scan",
                         "kernel_ms": t_kern, "algorithmic_bytes": alg_bytes,
                         "union_planes": int(rep.union_planes)},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step(n_max_cfg, k) * K,
            "tokens_per_s": n_total * world / (t_step * 1e-3),
            "fallback_heads": int(rep.fallback_heads),
            "max_candidates": int(rep.max_candidates),
            "clocks": clocks,
        }
        if cpu is not None:
            res["cpu_baseline"] = cpu
        if attention is not None:
            res["attention"] = attention
        if append is not None:
            res["append"] = append
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_native(a)
