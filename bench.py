"""Benchmark of the BasisKV decode-attention block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--cache e4m3] [--router b16r16]
                    [--stack avg64|avg96] [--prefill] [--sweep all|POINTS]

Default workload (one step): the Llama-3.1-8B attention-layer shape at Value
width 64, B = 16 sequences, 32K-token context, page 16, top-k 128 pages: one
fused ``basiskv_decode`` that appends one token per sequence, routes over
the full context, attends over the selected pages and out-projects.  The
context grows by one token per step (32768 -> 32768 + W + K); the
algorithmic bytes are counted per step from the actual length.
``--workload llama8b_layer_b1_t4k_v96`` times the batch-1, 4K-context layer
(Value width 96, top-k 64, no append) instead.

Metric: achieved HBM TB/s = algorithmic bytes / device time (higher is
better), with microseconds per step beside it (mean, and the median, p10
and p90 of per-step event times).  Algorithmic bytes per step:
  route   B*Hkv*T*(r_v+r_k)*2          z and e of the whole context
  attend  B*Hkv*min(k,P)*S*(d+r_v)*2   exact K and z of the selected pages
  outproj Hq*r_v*H*2                   the folded out-projection W'
  small   q, y, appended token state, folded queries, scores, selection,
          latent outputs, and the factors read by the fold / append kernels.
A step whose inputs are larger than twice the L2 (the default workload:
about 1.9 GB of cache) runs back to back with no flush; smaller steps are
timed one by one with a 256 MB write between them that flushes the L2.

``--sweep`` times the 32-layer decode sweep (B x T x r_v, top-k = T/64
pages, one appended token per step): 32 layers with their own factors, K
model steps per point; points whose 32 caches exceed 150 GB cycle fewer
physical caches by layer (stated in each line).

With N > 1 (torchrun) every rank runs an independent replica ("replicas
only": sequences are independent and the single-GPU path has no exchange);
the value is the bytes of all ranks over the slowest rank's time.

``--impl reference`` times the CPU oracle (float64 numpy) on rank 0 on a
bounded sample of the same workload: one (sequence, KV head) group per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_decode_attention_basiskv_b200 import synth  # noqa: E402

METRIC = "BasisKV decode µs/step & achieved HBM TB/s vs peak (Llama-8B shape, 32K ctx)"
WL = synth.LLAMA8B_T32K_B16
N_QUERIES = 4  # distinct planted query sets cycled over the steps
N_TOKENS = 8   # distinct appended tokens per layer cycled over the steps (--stack)


def algorithmic_bytes(wl, T: int, append: bool = True) -> dict:
    """Bytes one decode step must move at context length T (after append)."""
    S = wl.sel_page  # tokens per selected (routing) page
    P = -(-T // S)
    sel = min(wl.top_k, P)
    r = wl.router  # the router reads z[:, :r_b] and e[:, :r_q]
    cb = 1 if wl.cache_fp8 else 2  # bytes per cached element (E4M3 or bf16)
    route = wl.B * wl.Hkv * T * (r["r_b"] + r["r_q"]) * cb
    attend = wl.B * wl.Hkv * sel * S * (wl.d + wl.r_v) * cb
    outproj = wl.Hq * wl.r_v * wl.hidden * 2
    small = (wl.B * wl.Hq * wl.d * 2                      # q (fold + attend)
             + wl.B * wl.hidden * 2                       # y
             + wl.B * wl.Hq * (wl.r_v + wl.r_k) * 4 * 2   # folded queries w + r
             + wl.B * wl.Hkv * P * 4 * 2                  # scores w + r
             + wl.B * wl.Hkv * wl.top_k * 4 * 2           # selection w + r
             + wl.B * wl.Hq * wl.r_v * 2 * 2              # latent a (bf16) w + r
             + wl.Hkv * (wl.r_v + wl.r_k) * wl.d * 2)     # P_K, U_K for the fold
    if append:
        small += (wl.B * wl.Hkv * (2 * wl.d * 2 + (wl.d + wl.r_v + wl.r_k) * cb)
                  + wl.Hkv * wl.d * wl.r_v * 2)           # k, v in; K, z, e out; A_V
    return {"route": route, "attend": attend, "outproj": outproj, "small": small,
            "total": route + attend + outproj + small}


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                mhz.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------------ shared
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024


def bench_config(wl, world: int, K: int, W: int) -> dict:
    """The ``config`` of a bench line: the same for both arms at the same
    arguments."""
    T0 = wl.T
    grows = wl.append_tokens > 0
    flush = needs_flush(wl)
    return {"workload": wl.name, "global_batch": wl.B * world, "seq_len": T0,
            "context": (f"{T0} -> {T0 + W + K} tokens (one appended per step)" if grows
                        else f"{T0} tokens"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": ("steps timed one by one, the L2 flushed (256 MB write) between them"
                   if flush else "inputs larger than L2 (no flush)"),
            **{k: v for k, v in wl.describe().items() if k not in ("name", "steps")}}


def needs_flush(wl) -> bool:
    return algorithmic_bytes(wl, wl.T, append=wl.append_tokens > 0)["total"] < 2 * L2_BYTES


def step_stats(ms: list) -> dict:
    """Median, p10 and p90 of per-step device times (microseconds)."""
    import numpy as np
    a = np.asarray(ms, dtype=np.float64) * 1e3
    return {"reps": len(ms), "median_us": float(np.median(a)),
            "p10_us": float(np.percentile(a, 10)), "p90_us": float(np.percentile(a, 90))}


class StepTimer:
    """CUDA events around each step on the launching stream.  Back to back:
    one event between consecutive steps (the per-step times add up to the
    span).  Flushed: the L2 is overwritten before each step, outside its
    start / end events; the span is the sum of the steps."""

    def __init__(self, stream, flush: bool):
        self.stream, self.flush = stream, flush
        self.buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda") if flush else None
        self.starts, self.ends = [], []

    def _ev(self):
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    def step(self, fn):
        if self.flush:
            self.buf.fill_(len(self.starts) & 0xff)
            self.starts.append(self._ev())
        elif not self.starts:
            self.starts.append(self._ev())
        fn()
        e = self._ev()
        self.ends.append(e)
        if not self.flush:
            self.starts.append(e)

    def per_step_ms(self) -> list:
        return [a.elapsed_time(b) for a, b in zip(self.starts, self.ends)]

    def total_ms(self) -> float:
        return sum(self.per_step_ms())


# ------------------------------------------------------------------ oracle
def oracle_sample(wl) -> dict:
    """The arrays of one (sequence 0, KV head 0) group on the CPU, float64,
    and the scalars of one decode step of it (oracle.sample_timing)."""
    factors = synth.make_factors(wl)
    cache = synth.make_cache(wl, factors, "cpu", seqs=[0])
    q, _ = synth.make_query(synth.with_sizes(wl, B=1), cache["K"], wl.T)
    k, v = synth.make_tokens(wl, factors, 1, "cpu")
    f = {n: t.double().numpy() for n, t in factors.items()}
    c = {n: t[0, 0].double().numpy() for n, t in cache.items()}
    from oracle import basiskv_oracle as O
    r = wl.router
    arrays = {"q": q[0, :wl.G].double().numpy(), "k": k[0, 0, 0].double().numpy(),
              "v": v[0, 0, 0].double().numpy(), "K": c["K"], "Z": c["Z"], "E": c["E"],
              "A_V": f["A_V"][0], "P_K": f["P_K"][0], "U_K": f["U_K"][0],
              "W": O.fold_outproj(f["B_V"][:1], f["W_O"][:wl.G * wl.d], wl.G)}
    scalars = {"T": wl.T, "S": wl.page_size, "top_k": wl.top_k, "fp8": wl.cache_fp8,
               "r_b": r["r_b"], "r_q": r["r_q"], "n_sink": r["n_sink"], "n_recent": r["n_recent"]}
    return {"arrays": arrays, "scalars": scalars}


def oracle_bytes_per_group(wl) -> int:
    one = synth.with_sizes(wl, B=1, Hkv=1, Hq=wl.G)
    return algorithmic_bytes(one, wl.T + 1)["total"]


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def _oracle_workers(path: str, n: int, seconds: float) -> list:
    """n worker processes (BLAS on one thread each) timing the sample over
    the same wall-clock window; returns their (steps, seconds)."""
    import subprocess as sp
    env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1",
               PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    start = time.time() + 4.0 + 0.02 * n
    procs = [sp.Popen([sys.executable, "-m", "oracle.sample_timing", path, str(start),
                       str(seconds)], cwd=ROOT, env=env, stdout=sp.PIPE, stderr=sp.PIPE,
                      text=True) for _ in range(n)]
    out = []
    for p in procs:
        o, e = p.communicate(timeout=seconds + 300)
        if p.returncode != 0:
            raise RuntimeError(f"oracle worker failed: {e[-500:]}")
        r = json.loads(o.strip().splitlines()[-1])
        out.append((r["n"], r["s"]))
    return out


def cpu_baseline(wl, seconds: float = 6.0) -> dict:
    """The oracle timed on this host's cores in two forms, one sample = one
    (sequence, KV head) group of a decode step: one worker with BLAS on one
    thread, then one such worker on every core at once (all time the same
    window).  value = the all-cores form, in bytes of the sample over time."""
    import tempfile
    from oracle.sample_timing import save_sample
    s = oracle_sample(wl)
    groups = wl.B * wl.Hkv
    nbytes = oracle_bytes_per_group(wl)
    cores = host_cores()
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "sample.npz")
        save_sample(path, s["arrays"], **s["scalars"])
        (n1, t1), = _oracle_workers(path, 1, seconds)
        many = _oracle_workers(path, cores, seconds)
    rate1 = n1 / t1
    rate_all = sum(n / t for n, t in many)
    return {"value": nbytes * rate_all / 1e12, "unit": "TB/s", "cores": cores, "kind": "oracle",
            "single_thread": {"value": nbytes * rate1 / 1e12, "unit": "TB/s", "cores": 1,
                              "ms_per_group_step": 1e3 / rate1,
                              "ms_per_step_equiv": groups * 1e3 / rate1},
            "all_cores": {"value": nbytes * rate_all / 1e12, "unit": "TB/s", "cores": cores,
                          "group_steps_per_s": rate_all,
                          "ms_per_step_equiv": groups * 1e3 / rate_all},
            "sample": (f"decode steps of one (sequence, KV head) group = 1/{groups} of a step "
                       f"(float64 numpy oracle): {n1} steps on one core, then "
                       f"{sum(n for n, _ in many)} on {cores} cores (one worker per core), "
                       f"{seconds:.0f} s each")}


def run_reference(args) -> None:
    """The reference arm: the oracle as it stands, in this process (numpy's
    own BLAS threads), on the GPU arm's workload; one step = the decode
    step of one (sequence, KV head) group, timed step by step."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from oracle.sample_timing import group_step
    K, W = args.steps, args.warmup
    wl = WL
    s = oracle_sample(wl)
    sample = {**s["arrays"], **s["scalars"]}
    for _ in range(W):
        group_step(sample)
    times = []
    for _ in range(K):
        t0 = time.perf_counter()
        group_step(sample)
        times.append((time.perf_counter() - t0) * 1e3)
    ms = sum(times) / K
    groups = wl.B * wl.Hkv
    value = oracle_bytes_per_group(wl) / (ms / 1e3) / 1e12
    threads = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TB/s",
            "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms,
            "step_times": step_stats(times),
            "sample_fraction": 1.0 / groups,
            "ms_per_full_step_extrapolated": ms * groups,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generators; planted-page queries)",
            "config": bench_config(wl, world, K, W),
            "cpu_baseline": {"kind": "oracle", "cores": threads, "value": value, "unit": "TB/s",
                             "sample": (f"each step: the decode step of one (sequence, KV head) "
                                        f"group, 1/{groups} of the workload's step; float64 "
                                        f"numpy, BLAS on {threads} threads")},
            "e2e": {"value": value, "unit": "TB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ replicas (N > 1)
def replica_throughput(local_ms: float, total_bytes: float, dist=None, device="cpu") -> tuple:
    """Whole-job timing of N independent replicas ("replicas only": the
    single-GPU step has no exchange): the slowest rank's span, and the bytes
    of all ranks over it in TB/s.  Returns (ms_max, TB/s)."""
    t = torch.tensor([float(local_ms)], device=device)
    world = 1
    if dist is not None and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        world = dist.get_world_size()
    ms_max = float(t.item())
    return ms_max, world * total_bytes / (ms_max / 1e3) / 1e12


# ---------------------------------------------------------------- GPU arm
def _init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return world, rank, local, dist


def run_gpu(args) -> None:
    import sparse_decode_attention_basiskv_b200 as bkv
    from sparse_decode_attention_basiskv_b200.layer import DecodeLayer

    world, rank, local, dist = _init_dist()
    K, W = args.steps, args.warmup
    wl = synth.with_sizes(WL, steps=K + W, B=args.batch or WL.B, T=args.context or WL.T)
    if (wl.B, wl.T) != (WL.B, WL.T):
        wl = synth.with_sizes(wl, name=f"{WL.name} at B={wl.B}, T={wl.T}")
    append = wl.append_tokens > 0
    flush = needs_flush(wl)
    pb = synth.make_problem(wl, device="cuda")
    layer = DecodeLayer.from_problem(pb)
    T0 = wl.T
    queries = [synth.make_query(wl, pb.cache["K"], T0, step=i)[0] for i in range(N_QUERIES)]
    if append:
        k_all, v_all = synth.make_tokens(wl, pb.factors, K + W, device="cuda")
        k_steps = [k_all[:, i].contiguous() for i in range(K + W)]
        v_steps = [v_all[:, i].contiguous() for i in range(K + W)]
    else:
        k_steps = v_steps = [None] * (K + W)
    del pb.cache
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream()

    def T_after(i):
        return T0 + i + 1 if append else T0

    def step(i):
        layer.decode(queries[i % N_QUERIES], k_steps[i], v_steps[i], max_seq_len=T_after(i))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # ------------------------------------------------ device-timed region
    warm = StepTimer(stream, flush)
    for i in range(W):
        warm.step(lambda i=i: step(i))
    barrier()
    assert bkv.read_device_status() == 0
    # Back to back, the steps are timed as one span (events only at its ends:
    # an event between two steps would keep the next step's first kernel from
    # starting while the previous one finishes); their spread comes from a
    # second pass with an event after every step.
    timer = StepTimer(stream, flush)
    launches0 = bkv.launch_count()
    with ClockSampler(local) as clocks:
        barrier()
        if flush:
            for i in range(W, W + K):
                timer.step(lambda i=i: step(i))
        else:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(W, W + K):
                step(i)
            e1.record(stream)
        barrier()
    launches = bkv.launch_count() - launches0
    ms = timer.total_ms() if flush else e0.elapsed_time(e1)
    assert bkv.read_device_status() == 0
    if flush:
        per_step = timer.per_step_ms()
    else:
        layer.seq_lens.fill_(T_after(W - 1))
        dist_timer = StepTimer(stream, False)
        for i in range(W, W + K):
            dist_timer.step(lambda i=i: step(i))
        barrier()
        per_step = dist_timer.per_step_ms()
        assert bkv.read_device_status() == 0
    bytes_steps = [algorithmic_bytes(wl, T_after(i), append) for i in range(W, W + K)]
    total_bytes = sum(b["total"] for b in bytes_steps)
    ms_max, value = replica_throughput(ms, total_bytes, dist, "cuda")
    ms_per_step = ms_max / K

    # ------------------------------ roofline: the routing stage, timed alone
    # The scoring kernel (with the query fold it needs) through the C-ABI's
    # scores-only call: two launches, the scoring kernel is ~98% of them.
    T_r = T_after(W + K - 1)
    layer.seq_lens.fill_(T_r)
    scores = torch.empty(wl.B, wl.Hkv,
                         layer.dims.max_pages_per_seq * (wl.page_size // wl.sel_page),
                         device="cuda")
    reps = max(20, min(200, K))

    def route():
        bkv.basiskv_route(layer.dims, queries[0], layer.seq_lens, T_r, layer.block_table,
                          layer.P_K, layer.U_K, layer.Z, layer.E, wl.top_k, scores, None,
                          layer.workspace)
    for _ in range(3):
        route()
    torch.cuda.synchronize()
    rt = StepTimer(stream, flush)
    for _ in range(reps):
        rt.step(route)
    torch.cuda.synchronize()
    route_ms = rt.total_ms() / reps
    route_bytes = (wl.B * wl.Hkv * T_r * (wl.router["r_b"] + wl.router["r_q"])
                   * (1 if wl.cache_fp8 else 2))
    peak, peak_kind = measured_peak()
    achieved = route_bytes / (route_ms / 1e3) / 1e9
    traffic = None
    tr_path = os.path.join(ROOT, "profiles", "route_traffic.json")
    if os.path.exists(tr_path):
        with open(tr_path) as f:
            tr = json.load(f)
        # DRAM traffic of one launch, captured with ncu on a smaller batch of the
        # same kernel (B = 4) and scaled by the units processed: traffic grows in
        # proportion to the pages streamed.
        if tr.get("kernel_source_sha") == _route_source_sha() and wl.name == synth.LLAMA8B_T32K_B16.name:
            traffic = tr["traffic_over_algorithmic"] * route_bytes

    # ------------------------------------ end to end through the public API
    # Each step's q (and k, v) come from pinned host memory as one packed
    # copy and y goes back to pinned host memory.  Back to back: on a copy
    # stream, the inputs of step i + 1 copied while step i computes (two
    # device slots) and y of step i read back while step i + 1 computes (two
    # y buffers).  Flushed: each step's copies and compute timed on their own.
    layer.seq_lens.fill_(T0)
    nq = queries[0].numel()
    nk = k_steps[0].numel() if append else 0
    n_in = nq + 2 * nk

    def packed(i):
        parts = [queries[i % N_QUERIES].reshape(-1)]
        if append:
            parts += [k_steps[i].reshape(-1), v_steps[i].reshape(-1)]
        return torch.cat(parts).cpu().pin_memory()
    packed_h = [packed(i) for i in range(K + W)]
    slots = [torch.empty(n_in, dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    def views(sl):
        q = sl[:nq].view_as(queries[0])
        if not append:
            return q, None, None
        return (q, sl[nq:nq + nk].view_as(k_steps[0]), sl[nq + nk:].view_as(v_steps[0]))
    vws = [views(sl) for sl in slots]
    ys = [torch.empty(wl.B, wl.hidden, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    y_h = [torch.empty(wl.B, wl.hidden, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    cs = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(first, last, start_ev=None):
        if start_ev is not None:
            cs.wait_event(start_ev)
        with torch.cuda.stream(cs):
            slots[first % 2].copy_(packed_h[first], non_blocking=True)
            ev_in[first % 2].record(cs)
        for i in range(first, last):
            s_ = i % 2
            if i + 1 < last:  # next inputs while this step computes
                with torch.cuda.stream(cs):
                    if i >= first + 1:
                        cs.wait_event(ev_out[(i + 1) % 2])  # step i - 1 has read its slot
                    slots[(i + 1) % 2].copy_(packed_h[i + 1], non_blocking=True)
                    ev_in[(i + 1) % 2].record(cs)
            stream.wait_event(ev_in[s_])
            q_d, k_d, v_d = vws[s_]
            layer.decode(q_d, k_d, v_d, max_seq_len=T_after(i), y=ys[s_])
            ev_out[s_].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(ev_out[s_])
                y_h[s_].copy_(ys[s_], non_blocking=True)
        stream.wait_stream(cs)

    def e2e_one(i):  # copies and compute of one step on the launching stream
        slots[0].copy_(packed_h[i], non_blocking=True)
        q_d, k_d, v_d = vws[0]
        layer.decode(q_d, k_d, v_d, max_seq_len=T_after(i), y=ys[0])
        y_h[0].copy_(ys[0], non_blocking=True)

    if flush:
        for i in range(W):
            e2e_one(i)
        barrier()
        et = StepTimer(stream, True)
        for i in range(W, W + K):
            et.step(lambda i=i: e2e_one(i))
        barrier()
        e2e_ms = et.total_ms()
    else:
        e2e_run(0, W)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(W, W + K, e0)
        e1.record(stream)
        barrier()
        e2e_ms = e0.elapsed_time(e1)
    e2e_ms_max, e2e_value = replica_throughput(e2e_ms, total_bytes, dist, "cuda")
    h2d = n_in * 2
    d2h = wl.B * wl.hidden * 2

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = cpu_baseline(wl) if world == 1 and not args.no_cpu_baseline else None
    avg = {k: sum(b[k] for b in bytes_steps) / K for k in bytes_steps[0]}
    line = {
        "metric": METRIC, "value": value, "unit": "TB/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
        "step_times": {**step_stats(per_step),
                       "how": ("each step between its own events, the L2 flushed before it"
                               if flush else "a second pass of the same steps with an event "
                               "after every step")},
        "tokens_per_s": world * wl.B / (ms_per_step / 1e3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 caches, f16 x f16 -> f32" if wl.cache_fp8 else "bf16",
        "data": "synthetic (seeded generators; planted-page queries)",
        "config": bench_config(wl, world, K, W),
        "bytes_per_step": avg,
        "frac_of_peak": value / world / (peak / 1e3),
        "roofline": {"bound": "hbm",
                     "kernel": ("route_f8_kernel" if wl.cache_fp8 else "route_mma_kernel")
                     + " (+ its query fold)",
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "ms_per_launch": route_ms, "algorithmic_bytes": route_bytes},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TB/s", "us_per_step": e2e_ms_max / K * 1e3,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def run_stack(args) -> None:
    """The 32 attention layers of the Llama-8B shape, each with its own Value
    width (Table 12's per-layer V ranks with the given average): one fused
    decode step per layer per model step, the layers in order on one stream."""
    import sparse_decode_attention_basiskv_b200 as bkv
    from sparse_decode_attention_basiskv_b200.layer import DecodeLayer, DecodeStack

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    K, W = args.steps, args.warmup
    avg = int(args.stack[3:])
    base = synth.with_sizes(synth.LLAMA8B_32L_T32K_B16_AVG64, steps=K + W,
                            B=args.batch or synth.LLAMA8B_32L_T32K_B16_AVG64.B,
                            T=args.context or synth.LLAMA8B_32L_T32K_B16_AVG64.T)
    if avg != 64:
        base = synth.with_sizes(base, name=base.name.replace("avg_v64", f"avg_v{avg}"))
    widths = synth.v_rank_schedule(avg, base.layers)
    wls = synth.stack_layers(base, widths)
    layers, qs, ks, vs = [], [], [], []
    for l, wl in enumerate(wls):  # one layer at a time bounds the temporaries
        pb = synth.make_problem(wl, device="cuda", layer=l)
        layers.append(DecodeLayer.from_problem(pb))
        qs.append([pb.q, synth.make_query(wl, pb.cache["K"], wl.T, step=1)[0]])
        # eight distinct tokens per layer, cycled over the steps (bounded memory)
        k_all, v_all = synth.make_tokens(wl, pb.factors, N_TOKENS, device="cuda", stream_id=l)
        ks.append([k_all[:, i].contiguous() for i in range(N_TOKENS)])
        vs.append([v_all[:, i].contiguous() for i in range(N_TOKENS)])
        del pb, k_all, v_all
        torch.cuda.empty_cache()
    stack = DecodeStack(layers)
    T0 = base.T
    stream = torch.cuda.current_stream()

    def step(i, T_after):
        stack.decode([q[i % 2] for q in qs], [k[i % N_TOKENS] for k in ks],
                     [v[i % N_TOKENS] for v in vs], max_seq_len=T_after)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(W):
        step(i, T0 + i + 1)
    barrier()
    assert bkv.read_device_status() == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = bkv.launch_count()
    with ClockSampler(local) as clocks:
        barrier()
        ev0.record(stream)
        for i in range(W, W + K):
            step(i, T0 + i + 1)
        ev1.record(stream)
        barrier()
    launches = bkv.launch_count() - launches0
    assert bkv.read_device_status() == 0
    per_layer = [sum(algorithmic_bytes(wl, T0 + i + 1)["total"] for i in range(W, W + K))
                 for wl in wls]
    total_bytes = sum(per_layer)
    ms_max, value = replica_throughput(ev0.elapsed_time(ev1), total_bytes, dist, "cuda")

    # roofline: the scoring kernel (+ its fold) of every layer, back to back
    T_r = T0 + W + K
    for L in layers:
        L.seq_lens.fill_(T_r)
    scores = [torch.empty(base.B, base.Hkv, L.dims.max_pages_per_seq, device="cuda")
              for L in layers]

    def route_all():
        for L, sc, q in zip(layers, scores, qs):
            bkv.basiskv_route(L.dims, q[0], L.seq_lens, T_r, L.block_table, L.P_K, L.U_K, L.Z,
                              L.E, base.top_k, sc, None, L.workspace)
    for _ in range(3):
        route_all()
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    r0.record(stream)
    for _ in range(reps):
        route_all()
    r1.record(stream)
    torch.cuda.synchronize()
    route_ms = r0.elapsed_time(r1) / reps
    route_bytes = sum(base.B * base.Hkv * T_r * (wl.r_v + wl.r_k) * 2 for wl in wls)
    peak, peak_kind = measured_peak()
    achieved = route_bytes / (route_ms / 1e3) / 1e9

    # end to end through the public API: every layer's q, k, v of a step as
    # one packed copy from pinned host memory into one of two device slots,
    # and every layer's y back as one copy, on a copy stream that overlaps
    # the neighbouring steps' compute (as in the single-layer bench)
    for L in layers:
        L.seq_lens.fill_(T0)
    nL = len(layers)
    nq, nk = qs[0][0].numel(), ks[0][0].numel()
    per = nq + 2 * nk
    packed_h = []
    for i in range(N_TOKENS):  # step i uses packed_h[i % N_TOKENS]
        parts = []
        for l in range(nL):
            parts += [qs[l][i % 2].reshape(-1), ks[l][i].reshape(-1), vs[l][i].reshape(-1)]
        packed_h.append(torch.cat(parts).cpu().pin_memory())
    slots = [torch.empty(nL * per, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    views = [[(sl[l * per:l * per + nq].view_as(qs[l][0]),
               sl[l * per + nq:l * per + nq + nk].view_as(ks[l][0]),
               sl[l * per + nq + nk:(l + 1) * per].view_as(vs[l][0])) for l in range(nL)]
             for sl in slots]
    ybuf = [torch.empty(nL, base.B, base.hidden, dtype=torch.bfloat16, device="cuda")
            for _ in range(2)]
    y_h = [torch.empty(nL, base.B, base.hidden, dtype=torch.bfloat16).pin_memory()
           for _ in range(2)]
    cs = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(first, last, start_ev=None):
        if start_ev is not None:
            cs.wait_event(start_ev)
        with torch.cuda.stream(cs):
            slots[first % 2].copy_(packed_h[first % N_TOKENS], non_blocking=True)
            ev_in[first % 2].record(cs)
        for i in range(first, last):
            s_ = i % 2
            if i + 1 < last:  # next inputs while this step computes
                with torch.cuda.stream(cs):
                    if i >= first + 1:
                        cs.wait_event(ev_out[(i + 1) % 2])  # step i - 1 has read its slot
                    slots[(i + 1) % 2].copy_(packed_h[(i + 1) % N_TOKENS], non_blocking=True)
                    ev_in[(i + 1) % 2].record(cs)
            stream.wait_event(ev_in[s_])
            v_ = views[s_]
            stack.decode([x[0] for x in v_], [x[1] for x in v_], [x[2] for x in v_],
                         max_seq_len=T0 + i + 1, ys=list(ybuf[s_].unbind(0)))
            ev_out[s_].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(ev_out[s_])
                y_h[s_].copy_(ybuf[s_], non_blocking=True)
        stream.wait_stream(cs)

    e2e_run(0, W)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(W, W + K, e0)
    e1.record(stream)
    barrier()
    e2e_ms, e2e_value = replica_throughput(e0.elapsed_time(e1), total_bytes, dist, "cuda")
    h2d = nL * per * 2
    d2h = nL * base.B * base.hidden * 2

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = cpu_baseline(wls[0]) if world == 1 and not args.no_cpu_baseline else None
    line = {
        "metric": METRIC + f" — {base.layers}-layer stack, per-layer Value widths",
        "value": value, "unit": "TB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_max / K, "us_per_layer_step": ms_max / K * 1e3 / len(layers),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generators; planted-page queries)",
        "config": {"workload": base.name, "layers": len(layers), "v_widths": widths,
                   "avg_v_width": sum(widths) / len(widths), "global_batch": base.B * world,
                   "seq_len": T0, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs far larger than L2; no flush"},
        "bytes_per_step": total_bytes / K,
        "frac_of_peak": value / world / (peak / 1e3),
        "roofline": {"bound": "hbm", "kernel": "route_mma_kernel (+ its query fold), all layers",
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "ms_per_launch": route_ms / len(layers),
                     "algorithmic_bytes": route_bytes / len(layers)},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TB/s", "ms_per_step": e2e_ms / K,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


SWEEP_CAPACITY_BYTES = 150e9  # device memory given to the sweep's caches


def cache_bytes_per_layer(wl) -> int:
    """Bytes of one layer's paged K, Z and E caches (every physical page)."""
    cb = 1 if wl.cache_fp8 else 2
    return (wl.B * wl.pages_capacity() * wl.Hkv * wl.page_size * (wl.d + wl.r_v + wl.r_k) * cb)


def sweep_physical_layers(wl, layers: int = 32) -> int:
    """Distinct caches a sweep point holds: one per layer while the 32 fit
    under the capacity, else as many as fit (cycled by layer), 0 if none."""
    return min(layers, int(SWEEP_CAPACITY_BYTES // cache_bytes_per_layer(wl)))


def sweep_points(spec: str) -> list:
    pts = {f"b{w.B}_t{w.T // 1024}k_v{w.r_v}": w for w in synth.SWEEP}
    if spec == "all":
        return list(pts.values())
    out = []
    for name in spec.split(","):
        if name not in pts:
            raise SystemExit(f"unknown sweep point {name!r}; known: {', '.join(pts)}")
        out.append(pts[name])
    return out


def run_sweep(args) -> None:
    """The 32-layer decode sweep at the Llama-3.1-8B layer shape: per point,
    32 layers with their own factors (and their own caches while they fit
    under the capacity), K model steps of one fused decode per layer, one
    appended token per sequence per step; one JSON line per point."""
    import sparse_decode_attention_basiskv_b200 as bkv
    from sparse_decode_attention_basiskv_b200.layer import DecodeLayer

    world, rank, local, dist = _init_dist()
    K, W = args.steps, args.warmup
    peak, peak_kind = measured_peak()
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for base in sweep_points(args.sweep):
        wl = synth.with_sizes(base, steps=K + W)
        n_layers = base.layers
        L_phys = sweep_physical_layers(wl, n_layers)
        if L_phys == 0:
            if rank == 0:
                print(json.dumps({"metric": "sweep point skipped", "workload": wl.name,
                                  "reason": "one layer's cache exceeds the capacity"}), flush=True)
            continue
        table = synth.block_table(wl)
        caches, query_sets = [], []
        for p in range(L_phys):  # physical caches, drawn with layer p's factors
            paged = synth.make_paged_cache(wl, synth.make_factors(wl, p), table.cuda(), "cuda", p)
            keys = synth.PagedKeys(paged["K"], table, wl.page_size)
            query_sets.append([synth.make_query(wl, keys, wl.T, step=s)[0] for s in range(2)])
            caches.append(paged)
            del keys
        layers, toks = [], []
        for l in range(n_layers):
            f = synth.make_factors(wl, l)
            layers.append(DecodeLayer.from_parts(wl, f, caches[l % L_phys], table))
            k_all, v_all = synth.make_tokens(wl, f, N_TOKENS, device="cuda", stream_id=l)
            toks.append(([k_all[:, i].contiguous() for i in range(N_TOKENS)],
                         [v_all[:, i].contiguous() for i in range(N_TOKENS)]))
            del k_all, v_all
        torch.cuda.empty_cache()
        T0 = wl.T

        def model_step(i):
            for l, L in enumerate(layers):
                L.decode(query_sets[l % L_phys][i % 2], toks[l][0][i % N_TOKENS],
                         toks[l][1][i % N_TOKENS], max_seq_len=T0 + i + 1)

        for i in range(W):
            model_step(i)
        barrier()
        assert bkv.read_device_status() == 0
        timer = StepTimer(stream, False)
        launches0 = bkv.launch_count()
        with ClockSampler(local) as clocks:
            barrier()
            for i in range(W, W + K):
                timer.step(lambda i=i: model_step(i))
            barrier()
        launches = bkv.launch_count() - launches0
        assert bkv.read_device_status() == 0
        per_step = timer.per_step_ms()
        layer_bytes = [algorithmic_bytes(wl, T0 + i + 1)["total"] for i in range(W, W + K)]
        total_bytes = n_layers * sum(layer_bytes)
        ms_max, value = replica_throughput(timer.total_ms(), total_bytes, dist, "cuda")
        ms_step = ms_max / K
        if rank == 0:
            touched = n_layers * algorithmic_bytes(wl, T0 + W + 1)["total"]
            line = {
                "metric": f"BasisKV {n_layers}-layer decode sweep, achieved HBM TB/s",
                "value": value, "unit": "TB/s", "n_gpus": world, "steps": K, "warmup": W,
                "ms_per_model_step": ms_step, "us_per_layer_step": ms_step * 1e3 / n_layers,
                "step_times": step_stats(per_step),
                "tokens_per_s": world * wl.B / (ms_step / 1e3),
                "frac_of_peak": value / world / (peak / 1e3), "peak": peak,
                "peak_kind": peak_kind, "higher_is_better": True, "scaling": "weak",
                "dtype": "bf16", "data": "synthetic (seeded generators; planted-page queries)",
                "config": {**bench_config(wl, world, K, W), "layers": n_layers,
                           "physical_caches": L_phys,
                           "caches": (f"{n_layers} distinct" if L_phys == n_layers else
                                      f"{L_phys} physical caches cycled by layer mod {L_phys} "
                                      f"(each {cache_bytes_per_layer(wl) / 1e9:.1f} GB); every "
                                      "layer has its own factors"),
                           "l2": (f"{touched / 1e9:.2f} GB touched per model step, far above "
                                  "L2; no flush")},
                "bytes_per_layer_step": sum(layer_bytes) / K,
                "gpu_launches": launches, "clocks": clocks.summary()}
            print(json.dumps(line), flush=True)
        del layers, caches, toks, query_sets
        torch.cuda.empty_cache()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_prefill(args) -> None:
    """The prefill-chunk append on the tensor cores: a 4096-token chunk of
    the Qwen3-32B layer appended to every sequence of the batch in one call
    ([z | e] = [v | k] W_app^T per KV head, scattered into the pages)."""
    import sparse_decode_attention_basiskv_b200 as bkv
    from sparse_decode_attention_basiskv_b200.layer import DecodeLayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    K, W = args.steps, args.warmup
    base = synth.QWEN32B_T64K_B8
    wl = synth.with_sizes(base, B=args.batch or base.B, T=args.context or base.T, steps=1)
    if args.cache == "e4m3":
        wl = synth.with_sizes(wl, cache_fp8=1, name=wl.name + "_e4m3")
    n = wl.prefill_tokens
    pb = synth.make_problem(wl, device="cuda")
    layer = DecodeLayer.from_problem(pb)
    k, v = synth.make_tokens(wl, pb.factors, n, device="cuda", stream_id=1)
    del pb
    torch.cuda.empty_cache()
    lens = [torch.full((wl.B,), wl.T, dtype=torch.int32, device="cuda") for _ in range(K + W)]
    stream = torch.cuda.current_stream()

    def step(i, kk=k, vv=v):
        bkv.basiskv_append(layer.dims, kk, vv, n, lens[i], layer.block_table, layer.A_V,
                           layer.P_K, layer.U_K, layer.K, layer.Z, layer.E, layer.workspace,
                           W_app=layer.W_app)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(W):
        step(i)
    barrier()
    assert bkv.read_device_status() == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = bkv.launch_count()
    with ClockSampler(local) as clocks:
        barrier()
        ev0.record(stream)
        for i in range(W, W + K):
            step(i)
        ev1.record(stream)
        barrier()
    launches = bkv.launch_count() - launches0
    assert bkv.read_device_status() == 0
    assert all(int(x) == wl.T + n for x in lens[W + K - 1].tolist())
    cb = 1 if wl.cache_fp8 else 2
    rows = wl.B * n
    per_step = (rows * wl.Hkv * (2 * wl.d * 2 + (wl.d + wl.r_v + wl.r_k) * cb)
                + wl.Hkv * (wl.r_v + wl.r_k) * 2 * wl.d * 2)
    ms_max, value = replica_throughput(ev0.elapsed_time(ev1), per_step * K, dist, "cuda")
    ms_step = ms_max / K
    flops = 2.0 * rows * wl.Hkv * (wl.r_v + wl.r_k) * 2 * wl.d
    peak, peak_kind = measured_peak()

    # end to end: the chunk's k and v from pinned host memory, one step after another
    k_h, v_h = k.cpu().pin_memory(), v.cpu().pin_memory()
    k_d, v_d = torch.empty_like(k), torch.empty_like(v)
    probe_h = torch.empty(wl.B, dtype=torch.int32).pin_memory()
    for t in lens:
        t.fill_(wl.T)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(W, W + K):
        k_d.copy_(k_h, non_blocking=True)
        v_d.copy_(v_h, non_blocking=True)
        step(i, k_d, v_d)
        probe_h.copy_(lens[i], non_blocking=True)
    e1.record(stream)
    barrier()
    e2e_ms, e2e_value = replica_throughput(e0.elapsed_time(e1), per_step * K, dist, "cuda")
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "BasisKV prefill-chunk append, achieved HBM TB/s (Qwen3-32B layer, 4096-token chunks)",
        "value": value, "unit": "TB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "us_per_chunk": ms_step * 1e3 / wl.B,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 operands, fp32 accumulate" + (", e4m3 caches" if wl.cache_fp8 else ""),
        "data": "synthetic (seeded generators)",
        "config": {"workload": wl.name, "chunks_per_step": wl.B, "chunk_tokens": n,
                   "rows_per_step": rows, "global_batch": wl.B * world, "seq_len": wl.T,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"{per_step / 1e6:.0f} MB streamed per step; no flush"},
        "bytes_per_step": per_step,
        "roofline": {"bound": "hbm", "kernel": "append_tc_kernel (+ the length update)",
                     "achieved": per_step / (ms_step / 1e3) / 1e9, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": per_step / (ms_step / 1e3) / 1e9 / peak, "traffic": None,
                     "tensor_tflops": flops / (ms_step / 1e3) / 1e12},
        "cpu_baseline": None,
        "e2e": {"value": e2e_value, "unit": "TB/s", "ms_per_step": e2e_ms / K,
                "h2d_bytes_per_step": 2 * k.numel() * 2, "d2h_bytes_per_step": wl.B * 4},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def _route_source_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for n in ("route.cu", "route_mma.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "sparse_decode_attention_basiskv_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


DECODE_WORKLOADS = {w.name: w for w in (
    synth.LLAMA8B_T32K_B16, synth.LLAMA8B_T4K,
    synth.with_sizes(synth.QWEN32B_T64K_B8, name="qwen32b_layer_b8_t64k_v96", prefill_tokens=0))}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 1000; 128 model steps with --sweep)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=synth.LLAMA8B_T32K_B16.name,
                    choices=list(DECODE_WORKLOADS),
                    help="the single-layer decode workload of the default mode")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the batch (smaller cases for profiling)")
    ap.add_argument("--context", type=int, default=0,
                    help="override the context length (smaller cases for profiling)")
    ap.add_argument("--router", default="full", choices=["full", "b16r16", "b16r16_page4"],
                    help="full: the default router (all latent and residual dims, sink + "
                         "newest page); b16r16: the pages' narrow router and budget at the "
                         "cache's 16-token pages; b16r16_page4: the same at 4-token routing "
                         "pages (2048 routed + 64 recent tokens)")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "e4m3"],
                    help="element type of the K, Z and E caches")
    ap.add_argument("--prefill", action="store_true",
                    help="time the prefill-chunk append (Qwen3-32B layer, 4096-token chunks) "
                         "instead of the decode step")
    ap.add_argument("--stack", default="", choices=["", "avg64", "avg96"],
                    help="time the 32-layer stack with per-layer Value widths of this average "
                         "instead of one layer")
    ap.add_argument("--sweep", default="",
                    help="time the 32-layer decode sweep: 'all' or comma-separated points "
                         "such as b8_t32k_v64")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 128 if args.sweep else 1000
    global WL
    WL = DECODE_WORKLOADS[args.workload]
    if args.router == "b16r16":
        WL = synth.LLAMA8B_T32K_B16_B16R16
    elif args.router == "b16r16_page4":
        WL = synth.LLAMA8B_T32K_B16_B16R16_PAGE4
    if args.cache == "e4m3":
        WL = synth.with_sizes(WL, cache_fp8=1, name=WL.name + "_e4m3")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.stack:
        run_stack(args)
    elif args.prefill:
        run_prefill(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
