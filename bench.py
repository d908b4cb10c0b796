"""Benchmark of one decode step of the paged-KV hot path on B200.

A step is the whole path over one synthetic batch: the slot-mapped append
of each sequence's new K/V token, then paged decode attention (partials and
merge included).  Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama32]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores
    python bench.py --kv fp8 ...           # fp8 (E4M3) caches: the fused append_fp8 + decode_fp8

Metric: effective GB/s = algorithmic bytes / device time, where the
algorithmic bytes of a step are the distinct K/V rows the decode must read
plus q and out, plus the append's reads and writes.  Kernel times come from
CUDA events on the launching stream.  L2: each step reads one of several
copies of the paged cache, rotated so that a copy is untouched by at least
400 MB of other traffic before it is read again (inputs larger than the
126 MB L2); batches too small for that flush L2 with a 256 MB write between
steps, outside the timed events.  A batch whose sequences share prefix
blocks (the prefix-shared workload) runs the shared-prefix path: one prefix
attention launch per step before the fused append + decode; the same steps
on the plain path are timed beside it.  With N > 1 (torchrun) every rank runs an
independent replica of the batch (the path has no exchange step); value =
bytes of all ranks / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode effective KV GB/s and % of B200 HBM peak; µs per decode call"
E2E_COPIES = ("overlapped: step k's inputs copied up while step k-1 runs and its output read back while "
              "step k+1 runs (two copy streams, two input / output buffer pairs); 'serial' = copy up, "
              "step, read back on one stream")
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
ROTATE_BYTES = 400 << 20      # rotate cache copies totalling at least this much (L2 is 126 MB)
ROTATE_MIN_POOL = 8 << 20     # smaller caches are flushed with a write instead


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama32",
                    choices=["tiny", "qwen3", "llama32", "longskew", "prefix"])
    ap.add_argument("--impl", default="pa", choices=["pa", "reference"])
    ap.add_argument("--mode", default="decode", choices=["decode", "prefill"],
                    help="decode step (the default), or multi-query chunked prefill over the cache")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="cache format: bf16, or fp8 E4M3 codes with per-kv-head scales")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="with the default llama32 batch, skip timing the long/skewed batch beside it")
    return ap.parse_args()


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def _max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(ws: int) -> None:
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "paged_kv_attention_36_b200", "csrc", "*"))):
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode() + f.read())
    return h.hexdigest()[:16]


def _traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, or None
    when the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(workload)
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples every 100 ms, kept only inside the
    windows opened with begin() and closed with end() (end() also takes one
    synchronous sample, so every window has at least one).  The sampler is
    started before the warm-up; each window brackets a timed region and the
    untimed runs of the same step around it, so the samples see the step's
    load even when the timed region itself lasts a few milliseconds."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, enabled: bool):
        import threading
        self.proc = None
        self.idx = device_index
        self.samples = []      # (time, line)
        self.windows = []
        self.t_open = None
        self.enabled = enabled
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={device_index}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, FileNotFoundError):
                self.proc = None
        if self.proc is not None:
            threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line))

    def begin(self):
        self.t_open = time.time()

    def end(self):
        if not self.enabled or self.t_open is None:
            return
        try:
            r = subprocess.run(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
            now = time.time()
            self.samples += [(now, ln) for ln in r.stdout.splitlines()]
        except (OSError, subprocess.TimeoutExpired):
            now = time.time()
        self.windows.append((self.t_open, now + 0.01))
        self.t_open = None

    def stop(self):
        if not self.enabled:
            return None
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, line in list(self.samples):
            if not any(a <= t <= b for a, b in self.windows):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


HOLD = True  # untimed runs around the timed regions, for the clock samples (off with --no-clocks)


def hold_load(call, seconds: float, dev, between=None):
    """Runs `call` back to back, untimed, for about `seconds` of wall time
    (in bursts of 50, synchronised), so that the clock samples taken around
    a short timed region see the same load."""
    if not HOLD:
        return
    t0 = time.time()
    while time.time() - t0 < seconds:
        for _ in range(50):
            call()
            if between is not None:
                between()
        torch.cuda.synchronize(dev)


def _step_bytes(w):
    from paged_kv_attention_36_b200 import workloads
    dec = workloads.unique_kv_bytes(w) + workloads.qo_bytes(w)
    app = workloads.append_bytes(w)
    return dec, app


def cpu_baseline(w, dec_bytes: int, app_bytes: int, budget_s: float = 12.0):
    """The oracle, as it stands, on the host's cores: full append +
    decode steps of the same batch, repeated until about budget_s seconds."""
    import oracle
    from tests import paging  # bit-pattern views only
    nthreads = oracle.default_threads()
    kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
    qb = paging.bits(w.q)
    bt, cl = w.block_tables.numpy(), w.context_lens.numpy()
    kn, vn, sm = paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy()
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle.append(kn, vn, sm, kb, vb)
        oracle.decode(qb, kb, vb, bt, cl, w.scale, nthreads=nthreads)
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or steps >= 50:
            break
    per_step = el / steps
    return {"value": round((dec_bytes + app_bytes) / per_step / 1e9, 4), "unit": "GB/s",
            "cores": nthreads, "kind": "oracle",
            "sample": f"{steps} full steps (append + decode) of the '{w.spec.name}' batch, "
                      f"{per_step * 1e3:.1f} ms each, fp64, {nthreads} threads"}


def _fp8_scales(Hkv: int):
    """The benchmark's per-kv-head K and V scales of the fp8 caches (an input
    choice: they keep N(0,1) values and the x8 outliers inside E4M3's range)."""
    g = torch.arange(Hkv, dtype=torch.float32)
    return (g + 4) / 32, (g + 3) / 24


def _fp8_step_bytes(w):
    """Algorithmic bytes of one fp8 step: half the bf16 K/V bytes (one byte
    per value) + q/out; the append reads bf16 rows and writes fp8 ones."""
    from paged_kv_attention_36_b200 import workloads
    dec = workloads.unique_kv_bytes(w) // 2 + workloads.qo_bytes(w)
    n_valid = int((w.slot_mapping >= 0).sum().item())
    per_tok = w.k_new.shape[1] * w.k_new.shape[2]
    app = n_valid * per_tok * (2 * 2 + 2 * 1) + 4 * w.slot_mapping.numel()
    return dec, app


def _pool_rows(cache):
    """[NB][Hkv][16][D] bf16 pool -> [NB*16][Hkv][D] rows, one per slot."""
    NB, Hkv, bs, D = cache.shape
    return cache.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()


def run_reference_fp8(args, w):
    import numpy as np
    import oracle
    from tests import paging
    dec, app = _fp8_step_bytes(w)
    nthreads = oracle.default_threads()
    NB, Hkv, _, D = w.k_cache.shape
    ks, vs = (t.numpy() for t in _fp8_scales(Hkv))
    k8 = np.zeros((NB, Hkv, 16, D), np.uint8)
    v8 = np.zeros((NB, Hkv, D, 16), np.uint8)
    oracle.append_fp8(paging.bits(_pool_rows(w.k_cache)), paging.bits(_pool_rows(w.v_cache)),
                      np.arange(NB * 16, dtype=np.int32), k8, v8, ks, vs)
    qb = paging.bits(w.q)
    bt, cl = w.block_tables.numpy(), w.context_lens.numpy()
    kn, vn, sm = paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy()

    def step():
        oracle.append_fp8(kn, vn, sm, k8, v8, ks, vs)
        oracle.decode_fp8(qb, k8, v8, ks, vs, bt, cl, w.scale, nthreads=nthreads)
    return step, dec, app, nthreads


def run_reference(args, ws, rank):
    """--impl reference: the fp64 oracle on the host cores, rank 0 only."""
    if rank != 0:
        return
    from paged_kv_attention_36_b200 import workloads
    import oracle
    from tests import paging
    w = workloads.make(args.workload)
    if args.kv == "fp8":
        step, dec, app, nthreads = run_reference_fp8(args, w)
    else:
        dec, app = _step_bytes(w)
        nthreads = oracle.default_threads()
        kb, vb = paging.bits(w.k_cache).copy(), paging.bits(w.v_cache).copy()
        qb = paging.bits(w.q)
        bt, cl = w.block_tables.numpy(), w.context_lens.numpy()
        kn, vn, sm = paging.bits(w.k_new), paging.bits(w.v_new), w.slot_mapping.numpy()

        def step():
            oracle.append(kn, vn, sm, kb, vb)
            oracle.decode(qb, kb, vb, bt, cl, w.scale, nthreads=nthreads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    per = el / args.steps
    value = (dec + app) / per / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "description": w.spec.description, "kv": args.kv},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{args.steps} full steps of the '{args.workload}' batch"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class Packed:
    """A step's inputs as views into one device buffer (each at a 256-byte
    aligned offset) with a pinned host twin, so that a caller refreshes all of
    them with a single host-to-device copy."""

    def __init__(self, tensors, dev):
        offs, off = {}, 0
        for n, t in tensors.items():
            off = -(-off // 256) * 256
            offs[n] = (off, t.numel() * t.element_size())
            off += t.numel() * t.element_size()
        self.nbytes = off
        self.host = torch.empty(off, dtype=torch.uint8).pin_memory()
        self.dev = torch.empty(off, dtype=torch.uint8, device=dev)
        self.views = {}
        for n, t in tensors.items():
            o, nb = offs[n]
            self.host[o:o + nb].view(t.dtype).view(t.shape).copy_(t)
            self.views[n] = self.dev[o:o + nb].view(t.dtype).view(t.shape)
        self.dev.copy_(self.host)

    def h2d(self):
        self.dev.copy_(self.host, non_blocking=True)


def pipelined_e2e(launch, packs, outs, outs_h, K, W, dev, ws, between=lambda: None) -> float:
    """K end-to-end steps with their copies overlapped, as a serving loop
    runs them: step k's inputs go up from pinned host memory (one copy, on
    an input copy stream) while step k-1 runs, and step k's output comes
    back (on an output copy stream) while step k+1 runs.  Two input and two
    output buffers alternate; events keep an input buffer from being
    overwritten before the step that reads it has run, and an output buffer
    before its read-back has finished.  launch(i, k) launches step k on the
    current stream with input / output pair i.  Returns the time of the K
    steps in ms, from before the first copy up to the last read-back (max
    over ranks)."""
    s = torch.cuda.current_stream(dev)
    c_in, c_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run(n, start):
        in_free, out_free = [None, None], [None, None]
        c_in.wait_event(start)
        for k in range(n):
            i = k % 2
            with torch.cuda.stream(c_in):
                if in_free[i] is not None:
                    c_in.wait_event(in_free[i])
                packs[i].h2d()
                ready = torch.cuda.Event()
                ready.record(c_in)
            s.wait_event(ready)
            if out_free[i] is not None:
                s.wait_event(out_free[i])
            launch(i, k)
            done = torch.cuda.Event()
            done.record(s)
            in_free[i] = done
            between()
            with torch.cuda.stream(c_out):
                c_out.wait_event(done)
                outs_h[i].copy_(outs[i], non_blocking=True)
                back = torch.cuda.Event()
                back.record(c_out)
            out_free[i] = back
        for e in out_free:
            if e is not None:
                s.wait_event(e)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s)
    run(W, start)
    torch.cuda.synchronize(dev)
    _barrier(ws)
    torch.cuda.synchronize(dev)
    start.record(s)
    run(K, start)
    end.record(s)
    torch.cuda.synchronize(dev)
    _barrier(ws)
    return _max_over_ranks(start.elapsed_time(end), ws)


def time_fused_step(pa, name, args, dev, ws, clocks):
    """The fused append + decode step of batch `name` (larger than L2),
    timed like the headline step: the same --steps / --warmup, cache copies
    rotated, CUDA events on the launching stream, max over ranks.  Returns
    its own record (value, step time and roofline)."""
    from paged_kv_attention_36_b200 import workloads
    w = workloads.make(name)
    dec_bytes, app_bytes = _step_bytes(w)
    step_bytes = dec_bytes + app_bytes
    pool_bytes = 2 * w.k_cache.numel() * 2
    assert pool_bytes >= ROTATE_MIN_POOL
    ncopies = max(2, -(-ROTATE_BYTES // pool_bytes))
    q, bt, cl, kn, vn, sm = (t.to(dev) for t in (w.q, w.block_tables, w.context_lens, w.k_new, w.v_new,
                                                 w.slot_mapping))
    caches = [(w.k_cache.to(dev), w.v_cache.to(dev)) for _ in range(ncopies)]
    out = torch.empty_like(q)
    wsp = pa.alloc_workspace(pa.make_dims(q, caches[0][0], bt), device=dev)
    stream = torch.cuda.current_stream(dev)
    fused = [pa.prepare_append_decode(kn, vn, sm, q, kc, vc, bt, cl, w.scale, out, wsp, stream=stream)
             for kc, vc in caches]
    W_ = max(3, args.warmup)
    for k in range(W_):
        fused[k % ncopies]()
    torch.cuda.synchronize(dev)
    rot = iter(range(W_, 1 << 62))
    clocks.begin()
    hold_load(lambda: fused[next(rot) % ncopies](), 0.3, dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    _barrier(ws)
    torch.cuda.synchronize(dev)
    for k in range(K):
        ev[k][0].record(stream)
        fused[k % ncopies]()
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    _barrier(ws)
    hold_load(lambda: fused[next(rot) % ncopies](), 0.2, dev)
    clocks.end()
    errs = pa.pa_device_errors(clear=True)
    if errs:
        raise RuntimeError(f"device error bits {errs:#x} during the {name} benchmark")
    total_ms = _max_over_ranks(sum(ev[k][0].elapsed_time(ev[k][1]) for k in range(K)), ws)
    peak, peak_kind = _peaks()
    step_avg = total_ms / K
    achieved = step_bytes / (step_avg * 1e-3) / 1e9
    return {
        "workload": name, "description": w.spec.description,
        "value": round(ws * K * step_bytes / (total_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
        "steps": K, "warmup": W_, "step_us": round(step_avg * 1e3, 2),
        "l2": f"inputs larger than L2: {ncopies} copies of the {pool_bytes / 1e6:.0f} MB paged cache rotated, no flush",
        "step_pct_of_8tbs_nominal": round(100 * achieved / 8000.0, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "kernel": "pa::decode_kernel<..., APPEND> (pa_append_decode)",
                     "traffic": _traffic(name), "algorithmic_bytes_per_launch": step_bytes},
    }


def run_pa(args, ws, rank, local):
    from paged_kv_attention_36_b200 import binding as pa
    from paged_kv_attention_36_b200 import workloads

    dev = torch.device("cuda", local if ws > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    w = workloads.make(args.workload)
    dec_bytes, app_bytes = _step_bytes(w)
    step_bytes = dec_bytes + app_bytes

    # L2 hygiene: rotate enough copies of the paged cache that each step reads
    # a copy untouched by the last ~ROTATE_BYTES of traffic (inputs larger
    # than L2); a batch too small for that flushes L2 with a 256 MB write.
    pool_bytes = 2 * w.k_cache.numel() * 2
    rotate = pool_bytes >= ROTATE_MIN_POOL
    ncopies = max(2, -(-ROTATE_BYTES // pool_bytes)) if rotate else 1
    grouped = w.num_groups > 0
    step_in = {"q": w.q, "bt": w.block_tables, "cl": w.context_lens, "kn": w.k_new, "vn": w.v_new,
               "sm": w.slot_mapping}
    if grouped:
        step_in.update(go=w.group_offsets, gp=w.group_prefix_pages)
    packed = Packed(step_in, dev)  # the per-step inputs, one host-to-device copy in the e2e step
    q, bt, cl, kn, vn, sm = (packed.views[n] for n in ("q", "bt", "cl", "kn", "vn", "sm"))
    caches = [(w.k_cache.to(dev), w.v_cache.to(dev)) for _ in range(ncopies)]
    out = torch.empty_like(q)
    dims = pa.make_dims(q, caches[0][0], bt)
    if grouped:
        go, gp, mgs = packed.views["go"], packed.views["gp"], w.max_group_size
        wsp = torch.zeros(pa.pa_decode_shared_prefix_workspace_bytes(dims, w.num_groups, mgs),
                          dtype=torch.uint8, device=dev)
    else:
        wsp = pa.alloc_workspace(dims, device=dev)
    flush = None if rotate else torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    app = [pa.prepare_append(kn, vn, sm, kc, vc, stream=stream) for kc, vc in caches]
    plain = [pa.prepare_append_decode(kn, vn, sm, q, kc, vc, bt, cl, w.scale, out, wsp, stream=stream)
             for kc, vc in caches]
    if grouped:
        # one prefix-attention launch, then the fused append + decode of the members' own pages
        fused = [pa.prepare_decode_shared_prefix(q, kc, vc, bt, cl, w.scale, go, gp, mgs, out, wsp, k_new=kn,
                                                 v_new=vn, slot_mapping=sm, stream=stream) for kc, vc in caches]
        dec = [pa.prepare_decode_shared_prefix(q, kc, vc, bt, cl, w.scale, go, gp, mgs, out, wsp, stream=stream)
               for kc, vc in caches]
        launches = 2
    else:
        fused = plain
        dec = [pa.prepare_decode(q, kc, vc, bt, cl, w.scale, out, wsp, stream=stream) for kc, vc in caches]
        launches = 1

    def between():
        if flush is not None:
            flush.zero_()

    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    W_ = max(3, args.warmup)
    for k in range(W_):
        fused[k % ncopies]()
        between()
    torch.cuda.synchronize(dev)
    rot = iter(range(1 << 62))
    clocks.begin()
    hold_load(lambda: fused[next(rot) % ncopies](), 0.3, dev, between)  # untimed: the clock samples see the load

    # ---- timed region: K steps, each one launch of the fused append + decode ----
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    _barrier(ws)
    torch.cuda.synchronize(dev)
    for k in range(K):
        ev[k][0].record(stream)
        fused[k % ncopies]()
        ev[k][1].record(stream)
        between()
    torch.cuda.synchronize(dev)
    _barrier(ws)
    hold_load(lambda: fused[next(rot) % ncopies](), 0.2, dev, between)
    clocks.end()
    errs = pa.pa_device_errors(clear=True)
    if errs:
        raise RuntimeError(f"device error bits {errs:#x} during the benchmark")
    step_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    total_ms = _max_over_ranks(sum(step_ms), ws)

    # ---- the same steps as two launches (pa_cache_append, then pa_decode), for the split ----
    for k in range(W_):
        app[k % ncopies]()
        dec[k % ncopies]()
        between()
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    torch.cuda.synchronize(dev)
    for k in range(K):
        c = k % ncopies
        ev2[k][0].record(stream)
        app[c]()
        ev2[k][1].record(stream)
        dec[c]()
        ev2[k][2].record(stream)
        between()
    torch.cuda.synchronize(dev)
    app_avg = _max_over_ranks(sum(ev2[k][0].elapsed_time(ev2[k][1]) for k in range(K)) / K, ws)
    dec_avg = _max_over_ranks(sum(ev2[k][1].elapsed_time(ev2[k][2]) for k in range(K)) / K, ws)

    plain_avg = None
    if grouped:
        # ---- the same steps on the plain path (every member streams the shared pages) ----
        for k in range(W_):
            plain[k % ncopies]()
            between()
        ev3 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        torch.cuda.synchronize(dev)
        for k in range(K):
            ev3[k][0].record(stream)
            plain[k % ncopies]()
            ev3[k][1].record(stream)
            between()
        torch.cuda.synchronize(dev)
        plain_avg = _max_over_ranks(sum(ev3[k][0].elapsed_time(ev3[k][1]) for k in range(K)) / K, ws)

    # ---- end to end through the public API from pinned host memory: the
    # step's inputs in one pinned buffer (one copy), the output read back ----
    out_h = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = packed.nbytes
    d2h = out_h.numel() * out_h.element_size()

    def e2e_step(c):
        packed.h2d()
        fused[c]()
        out_h.copy_(out, non_blocking=True)

    for k in range(3):
        e2e_step(k % ncopies)
        between()
    torch.cuda.synchronize(dev)
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    _barrier(ws)
    torch.cuda.synchronize(dev)
    for k in range(K):
        ee[k][0].record(stream)
        e2e_step(k % ncopies)
        ee[k][1].record(stream)
        between()
    torch.cuda.synchronize(dev)
    _barrier(ws)
    e2e_total = _max_over_ranks(sum(ee[k][0].elapsed_time(ee[k][1]) for k in range(K)), ws)
    # the same steps with the copies overlapped (a second input / output pair)
    packed2 = Packed(step_in, dev)
    v2 = packed2.views
    out2 = torch.empty_like(q)
    out2_h = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    if grouped:
        fused2 = [pa.prepare_decode_shared_prefix(v2["q"], kc, vc, v2["bt"], v2["cl"], w.scale, v2["go"], v2["gp"],
                                                  mgs, out2, wsp, k_new=v2["kn"], v_new=v2["vn"],
                                                  slot_mapping=v2["sm"], stream=stream) for kc, vc in caches]
    else:
        fused2 = [pa.prepare_append_decode(v2["kn"], v2["vn"], v2["sm"], v2["q"], kc, vc, v2["bt"], v2["cl"],
                                           w.scale, out2, wsp, stream=stream) for kc, vc in caches]
    pairs = (fused, fused2)
    pipe_total = pipelined_e2e(lambda i, k: pairs[i][k % ncopies](), (packed, packed2), (out, out2),
                               (out_h, out2_h), K, 3, dev, ws, between)

    # the other batch the 70 %-of-HBM target names, timed the same way
    extra = None
    if args.workload == "llama32" and not args.no_extra:
        extra = time_fused_step(pa, "longskew", args, dev, ws, clocks)
    clk = clocks.stop()

    if rank != 0:
        return
    peak, peak_kind = _peaks()
    step_avg = total_ms / K
    achieved = step_bytes / (step_avg * 1e-3) / 1e9   # the fused kernel is the step (+ the prefix launch)
    value = ws * K * step_bytes / (total_ms * 1e-3) / 1e9
    l2 = (f"inputs larger than L2: {ncopies} copies of the {pool_bytes / 1e6:.0f} MB paged cache rotated, "
          f"no flush" if rotate else "flushed between steps (256 MB write, outside the timed events)")
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": K,
        "warmup": W_,
        "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "storage_dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "description": w.spec.description,
                   "num_seqs": w.spec.num_seqs, "q_heads": w.spec.num_q_heads,
                   "kv_heads": w.spec.num_kv_heads, "head_dim": w.spec.head_dim, "block_size": 16,
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU", "l2": l2,
                   "unique_kv_bytes": workloads.unique_kv_bytes(w),
                   "logical_kv_bytes": workloads.logical_kv_bytes(w)},
        "step_us": round(step_avg * 1e3, 2),
        "decode_us": round(dec_avg * 1e3, 2),
        "append_us": round(app_avg * 1e3, 2),
        "decode_only_gbs": round(dec_bytes / (dec_avg * 1e-3) / 1e9, 1),
        "step_pct_of_hbm_peak": round(100 * achieved / peak, 1),
        "step_pct_of_8tbs_nominal": round(100 * achieved / 8000.0, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "kernel": (("pa::prefix_kernel" if os.environ.get("PA_PREFILL_MMA") == "sync"
                                 else "pa::prefix_tc_kernel (tcgen05)")
                                + " + pa::decode_kernel<..., APPEND> (pa_decode_shared_prefix; the decode"
                                  " appends up to 256 new rows itself, the prefix launch any more)"
                                if grouped else "pa::decode_kernel<..., APPEND> (pa_append_decode)"),
                     "traffic": _traffic(args.workload),
                     "algorithmic_bytes_per_launch": step_bytes},
        "e2e": {"value": round(ws * K * step_bytes / (pipe_total * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(pipe_total / K, 5), "copies": E2E_COPIES,
                "serial": {"value": round(ws * K * step_bytes / (e2e_total * 1e-3) / 1e9, 2),
                           "ms_per_step": round(e2e_total / K, 5)}},
        "gpu_launches": launches * K,
        "clocks": clk,
    }
    if grouped:
        line["config"]["shared_prefix_groups"] = w.num_groups
        line["plain_path_step_us"] = round(plain_avg * 1e3, 2)
    if extra is not None:
        line["longskew_step"] = extra
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, dec_bytes, app_bytes)
    print(json.dumps(line), flush=True)


def run_pa_fp8(args, ws, rank, local):
    """The fp8 step: pa_append_decode_fp8 (the E4M3 append and the decode in
    one launch); the same steps as two launches (pa_cache_append_fp8, then
    pa_decode_fp8) are timed beside it for the split."""
    from paged_kv_attention_36_b200 import binding as pa
    from paged_kv_attention_36_b200 import workloads

    dev = torch.device("cuda", local if ws > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    w = workloads.make(args.workload)
    dec_bytes, app_bytes = _fp8_step_bytes(w)
    step_bytes = dec_bytes + app_bytes
    NB, Hkv, _, D = w.k_cache.shape
    ks, vs = (t.to(dev) for t in _fp8_scales(Hkv))
    # the fp8 pool: every slot of the bf16 pool encoded once (set-up, not timed)
    k8 = torch.empty((NB, Hkv, 16, D), dtype=torch.uint8, device=dev)
    v8 = torch.empty((NB, Hkv, D, 16), dtype=torch.uint8, device=dev)
    pa.pa_cache_append_fp8(_pool_rows(w.k_cache).to(dev), _pool_rows(w.v_cache).to(dev),
                           torch.arange(NB * 16, dtype=torch.int32, device=dev), k8, v8, ks, vs)
    torch.cuda.synchronize(dev)
    pool_bytes = 2 * k8.numel()
    rotate = pool_bytes >= ROTATE_MIN_POOL
    ncopies = max(2, -(-ROTATE_BYTES // pool_bytes)) if rotate else 1
    caches = [(k8.clone(), v8.clone()) for _ in range(ncopies)]
    del k8, v8
    packed = Packed({"q": w.q, "bt": w.block_tables, "cl": w.context_lens, "kn": w.k_new, "vn": w.v_new,
                     "sm": w.slot_mapping}, dev)  # one host-to-device copy in the e2e step
    q, bt, cl, kn, vn, sm = (packed.views[n] for n in ("q", "bt", "cl", "kn", "vn", "sm"))
    out = torch.empty_like(q)
    dims = pa.pa_dims(q.shape[0], q.shape[1], Hkv, D, 16, NB, bt.shape[1])
    wsp = pa.alloc_workspace(dims, device=dev)
    flush = None if rotate else torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    fused = [pa.prepare_append_decode_fp8(kn, vn, sm, q, kc, vc, ks, vs, bt, cl, w.scale, out, wsp, stream=stream)
             for kc, vc in caches]
    app = [pa.prepare_append_fp8(kn, vn, sm, kc, vc, ks, vs, stream=stream) for kc, vc in caches]
    dec = [pa.prepare_decode_fp8(q, kc, vc, ks, vs, bt, cl, w.scale, out, wsp, stream=stream) for kc, vc in caches]

    def between():
        if flush is not None:
            flush.zero_()

    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    W_ = max(3, args.warmup)
    for k in range(W_):
        fused[k % ncopies]()
        between()
    torch.cuda.synchronize(dev)
    rot = iter(range(1 << 62))
    clocks.begin()
    hold_load(lambda: fused[next(rot) % ncopies](), 0.3, dev, between)  # untimed: the clock samples see the load
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    _barrier(ws)
    torch.cuda.synchronize(dev)
    for k in range(K):
        ev[k][0].record(stream)
        fused[k % ncopies]()
        ev[k][1].record(stream)
        between()
    torch.cuda.synchronize(dev)
    _barrier(ws)
    hold_load(lambda: fused[next(rot) % ncopies](), 0.2, dev, between)
    clocks.end()
    errs = pa.pa_device_errors(clear=True)
    if errs:
        raise RuntimeError(f"device error bits {errs:#x} during the benchmark")
    total_ms = _max_over_ranks(sum(ev[k][0].elapsed_time(ev[k][1]) for k in range(K)), ws)

    # ---- the same steps as two launches, for the split ----
    for k in range(W_):
        app[k % ncopies]()
        dec[k % ncopies]()
        between()
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    torch.cuda.synchronize(dev)
    for k in range(K):
        c = k % ncopies
        ev2[k][0].record(stream)
        app[c]()
        ev2[k][1].record(stream)
        dec[c]()
        ev2[k][2].record(stream)
        between()
    torch.cuda.synchronize(dev)
    app_avg = _max_over_ranks(sum(ev2[k][0].elapsed_time(ev2[k][1]) for k in range(K)) / K, ws)
    dec_avg = _max_over_ranks(sum(ev2[k][1].elapsed_time(ev2[k][2]) for k in range(K)) / K, ws)

    out_h = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = packed.nbytes
    d2h = out_h.numel() * out_h.element_size()

    def e2e_step(c):
        packed.h2d()
        fused[c]()
        out_h.copy_(out, non_blocking=True)

    for k in range(3):
        e2e_step(k % ncopies)
        between()
    torch.cuda.synchronize(dev)
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    _barrier(ws)
    torch.cuda.synchronize(dev)
    for k in range(K):
        ee[k][0].record(stream)
        e2e_step(k % ncopies)
        ee[k][1].record(stream)
        between()
    torch.cuda.synchronize(dev)
    _barrier(ws)
    e2e_total = _max_over_ranks(sum(ee[k][0].elapsed_time(ee[k][1]) for k in range(K)), ws)
    packed2 = Packed({"q": w.q, "bt": w.block_tables, "cl": w.context_lens, "kn": w.k_new, "vn": w.v_new,
                      "sm": w.slot_mapping}, dev)
    v2 = packed2.views
    out2 = torch.empty_like(q)
    out2_h = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    fused2 = [pa.prepare_append_decode_fp8(v2["kn"], v2["vn"], v2["sm"], v2["q"], kc, vc, ks, vs, v2["bt"], v2["cl"],
                                           w.scale, out2, wsp, stream=stream) for kc, vc in caches]
    pairs = (fused, fused2)
    pipe_total = pipelined_e2e(lambda i, k: pairs[i][k % ncopies](), (packed, packed2), (out, out2),
                               (out_h, out2_h), K, 3, dev, ws, between)
    clk = clocks.stop()
    if rank != 0:
        return
    peak, peak_kind = _peaks()
    step_avg = total_ms / K
    achieved = step_bytes / (step_avg * 1e-3) / 1e9
    value = ws * K * step_bytes / (total_ms * 1e-3) / 1e9
    l2 = (f"inputs larger than L2: {ncopies} copies of the {pool_bytes / 1e6:.0f} MB fp8 cache rotated, "
          f"no flush" if rotate else "flushed between steps (256 MB write, outside the timed events)")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W_,
        "ms_per_step": round(step_avg, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "storage_dtype": "e4m3", "data": "synthetic",
        "config": {"workload": args.workload, "description": w.spec.description, "kv": "fp8-e4m3",
                   "num_seqs": w.spec.num_seqs, "q_heads": w.spec.num_q_heads, "kv_heads": w.spec.num_kv_heads,
                   "head_dim": w.spec.head_dim, "block_size": 16,
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU", "l2": l2,
                   "unique_kv_bytes": workloads.unique_kv_bytes(w) // 2},
        "step_us": round(step_avg * 1e3, 2),
        "two_launch_step_us": round((app_avg + dec_avg) * 1e3, 2),
        "decode_us": round(dec_avg * 1e3, 2),
        "append_us": round(app_avg * 1e3, 2),
        "decode_only_gbs": round(dec_bytes / (dec_avg * 1e-3) / 1e9, 1),
        "step_pct_of_hbm_peak": round(100 * achieved / peak, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "kernel": "pa::decode_kernel<..., APPEND, Fp8MmaMath> (pa_append_decode_fp8)",
                     "traffic": _traffic(args.workload + ":fp8"),
                     "algorithmic_bytes_per_launch": step_bytes},
        "e2e": {"value": round(ws * K * step_bytes / (pipe_total * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(pipe_total / K, 5),
                "copies": E2E_COPIES,
                "serial": {"value": round(ws * K * step_bytes / (e2e_total * 1e-3) / 1e9, 2),
                           "ms_per_step": round(e2e_total / K, 5)}},
        "gpu_launches": K,
        "clocks": clk,
    }
    if ws == 1 and not args.no_cpu_baseline:
        step, cdec, capp, nthreads = run_reference_fp8(args, w)
        n, t0 = 0, time.perf_counter()
        while True:
            step()
            n += 1
            el = time.perf_counter() - t0
            if el >= 12.0 or n >= 50:
                break
        line["cpu_baseline"] = {"value": round((cdec + capp) / (el / n) / 1e9, 4), "unit": "GB/s",
                                "cores": nthreads, "kind": "oracle",
                                "sample": f"{n} full fp8 steps (append + decode) of the '{w.spec.name}' batch, "
                                          f"{el / n * 1e3:.1f} ms each, fp64, {nthreads} threads"}
    print(json.dumps(line), flush=True)


PREFILL_METRIC = "paged chunked-prefill attention TFLOP/s (causal, over the cache)"


def run_prefill(args, ws, rank, local, reference: bool):
    """--mode prefill: pa_prefill on a chunked-prefill batch with the head
    shapes of --workload; value = algorithmic TFLOP/s (4*D per query row and
    visible key).  The reference arm times the oracle on a bounded sample."""
    from paged_kv_attention_36_b200 import workloads
    wl = args.workload if args.workload in ("llama32", "qwen3") else "llama32"
    pb = workloads.make_prefill(wl)
    flops = workloads.prefill_flops(pb)
    if reference:
        if rank != 0:
            return
        import numpy as np
        import oracle
        from tests import paging
        nthreads = oracle.default_threads()
        sub = 2  # a bounded sample: the first two sequences of the batch
        cu = pb.cu_q_lens[: sub + 1].numpy()
        sb = workloads.PrefillBatch(pb.q[: int(cu[-1])], pb.cu_q_lens[: sub + 1], pb.k_cache, pb.v_cache,
                                    pb.block_tables[:sub], pb.context_lens[:sub], pb.scale, pb.description)
        sflops = workloads.prefill_flops(sb)
        args_ = (paging.bits(sb.q), cu, paging.bits(pb.k_cache), paging.bits(pb.v_cache),
                 sb.block_tables.numpy(), sb.context_lens.numpy(), pb.scale)
        for _ in range(max(1, min(args.warmup, 1))):
            oracle.prefill(*args_, nthreads=nthreads)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle.prefill(*args_, nthreads=nthreads)
        per = (time.perf_counter() - t0) / args.steps
        value = sflops / per / 1e12
        print(json.dumps({
            "impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"prefill-{wl}", "description": pb.description},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
                             "sample": f"the first {sub} of {pb.cu_q_lens.shape[0] - 1} sequences per step"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return
    from paged_kv_attention_36_b200 import binding as pa
    dev = torch.device("cuda", local if ws > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    packed = Packed({k: getattr(pb, k) for k in ("q", "cu_q_lens", "block_tables", "context_lens")}, dev)
    t = dict(packed.views, k_cache=pb.k_cache.to(dev), v_cache=pb.v_cache.to(dev))
    out = torch.empty_like(t["q"])
    stream = torch.cuda.current_stream(dev)
    call = pa.prepare_prefill(t["q"], t["cu_q_lens"], pb.max_q_len, t["k_cache"], t["v_cache"], t["block_tables"],
                              t["context_lens"], pb.scale, out, stream=stream)
    clocks = ClockSampler(dev.index, enabled=not args.no_clocks)
    W_ = max(3, args.warmup)
    for _ in range(W_):
        call()
    torch.cuda.synchronize(dev)
    clocks.begin()
    hold_load(call, 0.3, dev)  # untimed: the clock samples see the load
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    _barrier(ws)
    torch.cuda.synchronize(dev)
    for k in range(K):
        ev[k][0].record(stream)
        call()
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    _barrier(ws)
    hold_load(call, 0.2, dev)
    clocks.end()
    clk = clocks.stop()
    errs = pa.pa_device_errors(clear=True)
    if errs:
        raise RuntimeError(f"device error bits {errs:#x} during the benchmark")
    total_ms = _max_over_ranks(sum(ev[k][0].elapsed_time(ev[k][1]) for k in range(K)), ws)
    # end to end: q and the batch metadata from pinned host memory (one
    # packed copy), out back
    out_h = torch.empty(pb.q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = packed.nbytes
    d2h = out_h.numel() * out_h.element_size()
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    torch.cuda.synchronize(dev)
    for k in range(K):
        ee[k][0].record(stream)
        packed.h2d()
        call()
        out_h.copy_(out, non_blocking=True)
        ee[k][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = _max_over_ranks(sum(ee[k][0].elapsed_time(ee[k][1]) for k in range(K)), ws)
    packed2 = Packed({k: getattr(pb, k) for k in ("q", "cu_q_lens", "block_tables", "context_lens")}, dev)
    v2 = packed2.views
    out2 = torch.empty_like(t["q"])
    out2_h = torch.empty(pb.q.shape, dtype=torch.bfloat16).pin_memory()
    call2 = pa.prepare_prefill(v2["q"], v2["cu_q_lens"], pb.max_q_len, t["k_cache"], t["v_cache"], v2["block_tables"],
                               v2["context_lens"], pb.scale, out2, stream=stream)
    pairs = (call, call2)
    pipe_ms = pipelined_e2e(lambda i, k: pairs[i](), (packed, packed2), (out, out2), (out_h, out2_h), K, 3, dev, ws)
    if rank != 0:
        return
    avg = total_ms / K
    achieved = flops / (avg * 1e-3) / 1e12
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peak, kind = 1590.0, "fallback"
    if os.path.exists(pk_path):
        with open(pk_path) as f:
            pk = json.load(f)
        if "bf16_tflops" in pk:
            peak, kind = float(pk["bf16_tflops"]), "measured"
    print(json.dumps({
        "metric": PREFILL_METRIC, "value": round(ws * achieved, 2), "unit": "TFLOP/s", "n_gpus": ws, "steps": K,
        "warmup": W_, "ms_per_step": round(avg, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "storage_dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"prefill-{wl}", "description": pb.description, "flops_per_step": flops,
                   "l2": (f"no flush: the {2 * pb.k_cache.numel() * 2 / 1e6:.0f} MB of K/V are re-read by every "
                          "row tile of a sequence, through L2 by design")},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_kind": kind,
                     "kernel": ("pa::prefill_kernel (mma.sync m16n8k16; P.V as two bf16 products)"
                                if os.environ.get("PA_PREFILL_MMA") == "sync" else
                                "pa::prefill_tc_kernel (tcgen05.mma, S/P and O in TMEM, TMA-fed K/V)"),
                     "traffic": (None if os.environ.get("PA_PREFILL_MMA") or os.environ.get("PA_PREFILL_BN")
                                 else _traffic(f"prefill-{wl}"))},
        "e2e": {"value": round(ws * flops / (pipe_ms / K * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(pipe_ms / K, 5),
                "copies": E2E_COPIES,
                "serial": {"value": round(ws * flops / (e2e_ms / K * 1e-3) / 1e12, 2),
                           "ms_per_step": round(e2e_ms / K, 5)}},
        "gpu_launches": K,
        "clocks": clk,
    }), flush=True)


def main():
    global HOLD
    args = _args()
    HOLD = not args.no_clocks
    ws, rank, local = _dist()
    try:
        if args.mode == "prefill":
            if args.impl != "reference" and not torch.cuda.is_available():
                raise SystemExit("bench.py needs a CUDA device for --impl pa")
            run_prefill(args, ws, rank, local, reference=args.impl == "reference")
        elif args.impl == "reference":
            run_reference(args, ws, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("bench.py needs a CUDA device for --impl pa")
            if args.kv == "fp8":
                run_pa_fp8(args, ws, rank, local)
            else:
                run_pa(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
