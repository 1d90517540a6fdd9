"""Benchmark of the Gated DeltaNet mixer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|long|varlen|decode] [--no-extras]

One step is one gdn_prefill call over the workload: the whole chunked-prefill
path (q/k normalisation, decay cumsum, UT transform, intra-chunk attention,
inter-chunk state passing) for a Qwen3.5-0.8B-like mixer layer, 1 x 4096
tokens, 16 q/k and 16 v heads, d = 128, bf16, chunk 64. The JSON line also
carries the 1000-step decode workload (64 sequences x 32 v heads) and the
32768-token long prefill as sub-objects, each with its own roofline.

Multi-GPU: one process per GPU (torchrun); every rank runs its own copy of
the workload (independent sequences, no data exchange), so scaling is weak
and the value is the sum over ranks divided by the slowest rank's time.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
import workloads  # noqa: E402

METRIC = "prefill tokens/s & decode steps/s per mixer layer; % tensor/HBM roofline"
DATA = ("synthetic: seeded q, k, v ~ N(0,1) (bf16), alpha = sigmoid(N(3,1)) passed as "
        "g = log(alpha), beta = sigmoid(N(0,1)), fp32 gates")
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- helpers ---
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def prefill_flops_per_token_head(C=64, d=128):
    """Algorithmic flops of the chunked method per token per value head,
    triangle-aware: KK^T and QK^T strictly/inclusive lower (C^2 d each per
    chunk), T [beta V | beta gamma K] (2 C^2 d), (M o QK^T) U (C^2 d) and the
    three d x d x C state products (6 C d^2), i.e. 5 C d + 6 d^2 per token."""
    return 5 * C * d + 6 * d * d


def prefill_bytes(T, Hqk, Hv, d, N, state_in):
    """Algorithmic HBM bytes of one prefill: every input read once, every output written once."""
    b = T * Hqk * d * 2 * 2 + T * Hv * d * 2 + T * Hv * d * 2 + T * Hv * 4 * 2
    b += N * Hv * d * d * 4 * (2 if state_in else 1) + (N + 1) * 4
    return b


def decode_bytes(B, Hqk, Hv, d, state_bytes=4):
    """Algorithmic HBM bytes of one decode step: state read + written, q, k, v, o, gates."""
    return B * Hv * d * d * state_bytes * 2 + B * Hqk * d * 2 * 2 + B * Hv * d * 2 * 2 + B * Hv * 4 * 2


# the source files each kernel is built from (its traffic record is void once one changes)
KERNEL_SOURCES = {
    "prefill_pc": ("common.cuh", "sm100.cuh", "prefill_pc.cuh"),        # 32-row slices, 4096 tokens
    "prefill_pc_long": ("common.cuh", "sm100.cuh", "prefill_pc.cuh"),   # 128-row slices, 32768 tokens
    "decode": ("common.cuh", "decode.cuh"),
}


def _code_only(src):
    """Source text without comments and with whitespace collapsed, so that an
    edit of comments alone keeps a kernel's traffic record (the kernel
    sources hold no string literal that contains a comment marker)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_deltanet_linear_21_b200", "csrc")
    for fn in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(fn.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_record(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    if kernel not in KERNEL_SOURCES:
        return None
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML
    about every 0.5 ms while a timed region runs (reading only; nothing is
    changed)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index):
        self.device_index = device_index
        self.samples = []
        self.max_mhz = None
        self._stop = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device_index)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def __enter__(self):
        import threading
        try:
            self.nvml, self.handle = self._handle()
            self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
        except Exception:
            self.handle = None
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    mhz = self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
                    rs = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                self._stop.wait(0.0005)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        reasons = set()
        for _, rs in self.samples:
            for name, const in self.REASONS:
                if rs & getattr(self.nvml, const, 0):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


def reduce_max(x, world, device=None):
    """Max over ranks of a host number; every rank calls it at the same point."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank, ms_max, world):
    """Whole-job rate: every rank processes units_per_rank per step; the job's
    step time is the slowest rank's."""
    return world * units_per_rank / (ms_max * 1e-3)


def timed(fn, stream):
    """Device time (ms) of fn() on `stream`, bracketed by synchronisation."""
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


MIN_SAMPLED_MS = 300.0


def timed_replays(graph, stream, steps, sampler=None, min_ms=MIN_SAMPLED_MS):
    """Per-step device time of a graph holding `steps` steps: each replay is timed
    on its own with CUDA events (exactly `steps` steps between the events), and
    the replays are repeated until about `min_ms` of device time has passed (at
    least 5), so that the clock sampler sees the whole region many times; the
    median replay is returned with the number of replays."""
    first = timed(graph.replay, stream)
    reps = max(5, min(2000, int(min_ms / max(first, 1e-3)) + 1))
    times = []
    if sampler is not None:
        with sampler:
            for _ in range(reps):
                times.append(timed(graph.replay, stream))
    else:
        for _ in range(reps):
            times.append(timed(graph.replay, stream))
    return statistics.median(times) / steps, reps


# ------------------------------------------------------------ our workload ---
def device_prefill_inputs(lengths, Hqk, Hv, d, seed, device, state_std=0.0, dtype=torch.bfloat16):
    """Seeded inputs generated on the device (same distributions as workloads.py)."""
    gen = torch.Generator(device=device).manual_seed(seed)
    T = sum(lengths)
    q = torch.randn(T, Hqk, d, generator=gen, device=device).to(dtype)
    k = torch.randn(T, Hqk, d, generator=gen, device=device).to(dtype)
    v = torch.randn(T, Hv, d, generator=gen, device=device).to(dtype)
    x = torch.randn(T, Hv, generator=gen, device=device, dtype=torch.float64) + 3.0
    y = torch.randn(T, Hv, generator=gen, device=device, dtype=torch.float64)
    g = torch.nn.functional.logsigmoid(x).float()
    beta = torch.sigmoid(y).float()
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths), 0)
    s0 = None
    if state_std > 0:
        s0 = torch.randn(len(lengths), Hv, d, d, generator=gen, device=device) * state_std
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu.to(device), state_in=s0)


def run_prefill_bench(gdn, w, steps, warmup, device, rank, sampler=None, min_ms=MIN_SAMPLED_MS):
    stream = torch.cuda.current_stream()
    T = w.total_tokens
    one = prefill_bytes(T, w.Hqk, w.Hv, w.d, len(w.lengths), w.state_std > 0)
    copies = l2_copies(w)   # rotate inputs over > 3x L2
    bufs = [device_prefill_inputs(w.lengths, w.Hqk, w.Hv, w.d, 7919 * rank + 31 * i + w.index,
                                  device, w.state_std, w.torch_dtype) for i in range(copies)]
    outs = [(torch.empty(T, w.Hv, w.d, dtype=w.torch_dtype, device=device),
             torch.empty(len(w.lengths), w.Hv, w.d, w.d, device=device)) for _ in range(copies)]

    def step(i):
        x = bufs[i % copies]
        o, s = outs[i % copies]
        gdn.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"],
                    o=o, state_out=s)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    # capture the K steps once, replay on the device without host gaps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(steps):
            step(i)
    torch.cuda.synchronize()
    graph.replay()   # untimed replay: first-replay costs
    torch.cuda.synchronize()
    ms, reps = timed_replays(graph, stream, steps, sampler, min_ms=min_ms)
    return dict(ms=ms, tokens=T, bytes=one, copies=copies, graph=graph, replays=reps)


def run_decode_bench(gdn, w, steps_timed, warmup, device, rank, sampler=None, state_dtype=torch.float32,
                     min_ms=MIN_SAMPLED_MS):
    stream = torch.cuda.current_stream()
    B, Hqk, Hv, d = w.batch, w.Hqk, w.Hv, w.d
    gen = torch.Generator(device=device).manual_seed(workloads.SEED_DECODE_STEP + 7919 * rank)
    n = steps_timed
    qs = torch.randn(n, B, Hqk, d, generator=gen, device=device).to(torch.bfloat16)
    ks = torch.randn(n, B, Hqk, d, generator=gen, device=device).to(torch.bfloat16)
    vs = torch.randn(n, B, Hv, d, generator=gen, device=device).to(torch.bfloat16)
    gs = torch.nn.functional.logsigmoid(torch.randn(n, B, Hv, generator=gen, device=device) + 3.0)
    bs = torch.sigmoid(torch.randn(n, B, Hv, generator=gen, device=device))
    state = (torch.randn(B, Hv, d, d, generator=gen, device=device) * w.state_std).to(state_dtype)
    o = torch.empty(B, Hv, d, dtype=torch.bfloat16, device=device)

    def run(a, b):
        for t in range(a, b):
            gdn.decode(qs[t], ks[t], vs[t], gs[t], bs[t], state, o=o)

    run(0, min(warmup, n))
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(0, n)
    graph.replay()
    torch.cuda.synchronize()
    ms, reps = timed_replays(graph, stream, n, sampler, min_ms=min_ms)
    return dict(ms=ms, bytes=decode_bytes(B, Hqk, Hv, d, state.element_size()), steps=n, replays=reps)


def run_e2e(gdn, w, steps, device):
    """Same prefill through the public API with inputs in pinned host memory: every
    step copies q, k, v, g, beta (and the states) up, calls gdn.prefill and copies o
    and the final states down. Steps are pipelined the way a serving loop runs them:
    step i+1's inputs go up on one copy stream while step i computes and step i-1's
    results come down on another (PCIe carries both directions at once), over two
    sets of device buffers ordered by events. The timed region, on the launching
    stream, holds every step's copies and calls."""
    main = torch.cuda.current_stream()
    x = workloads.inputs_for(w) if w.total_tokens <= 8192 else None
    if x is None:
        x = {kk: (vv.cpu() if isinstance(vv, torch.Tensor) else vv)
             for kk, vv in device_prefill_inputs(w.lengths, w.Hqk, w.Hv, w.d, 11, device).items()}
    host = {kk: vv.pin_memory() for kk, vv in x.items() if isinstance(vv, torch.Tensor)}
    T, N = w.total_tokens, len(w.lengths)
    o_h = torch.empty(T, w.Hv, w.d, dtype=torch.bfloat16).pin_memory()
    s_h = torch.empty(N, w.Hv, w.d, w.d).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = o_h.numel() * o_h.element_size() + s_h.numel() * s_h.element_size()
    sets = [({kk: torch.empty_like(vv, device=device) for kk, vv in host.items()},
             torch.empty(T, w.Hv, w.d, dtype=torch.bfloat16, device=device),
             torch.empty(N, w.Hv, w.d, w.d, dtype=torch.float32, device=device)) for _ in range(2)]
    ws = torch.empty(max(1, gdn.prefill_workspace_bytes(N, w.Hv, w.d, w.d)), dtype=torch.uint8, device=device)
    up, cmp, down = (torch.cuda.Stream(device=device) for _ in range(3))
    ev_up, ev_cmp, ev_down = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def step(i):
        b = i & 1
        dev, o_d, s_d = sets[b]
        up.wait_event(ev_cmp[b])     # the call two steps back has read these inputs
        with torch.cuda.stream(up):
            for kk in host:
                dev[kk].copy_(host[kk], non_blocking=True)
        ev_up[b].record(up)
        cmp.wait_event(ev_up[b])
        cmp.wait_event(ev_down[b])   # the results two steps back have left these outputs
        gdn.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev.get("state_in"),
                    dev["cu_seqlens"], o=o_d, state_out=s_d, workspace=ws, stream=cmp)
        ev_cmp[b].record(cmp)
        down.wait_event(ev_cmp[b])
        with torch.cuda.stream(down):
            o_h.copy_(o_d, non_blocking=True)
            s_h.copy_(s_d, non_blocking=True)
        ev_down[b].record(down)

    def run(n):
        start = torch.cuda.Event()
        start.record(main)
        for st in (up, cmp, down):
            st.wait_event(start)
        for i in range(n):
            step(i)
        for st in (up, cmp, down):
            e = torch.cuda.Event()
            e.record(st)
            main.wait_event(e)

    run(2)
    ms = timed(lambda: run(steps), main) / steps
    return dict(ms=ms, h2d=h2d, d2h=d2h, tokens=T)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_read_gbs(nbytes=1 << 30, passes=5):
    """Host sequential-read bandwidth: every core sums its own slice of a 1 GiB
    fp64 array (numpy releases the GIL inside the reduction); best of several
    passes, after a pass that touches every page."""
    import threading

    import numpy as np
    a = np.ones(nbytes // 8)
    cores = os.cpu_count() or 1
    parts = np.array_split(a, cores)
    best = 0.0
    for _ in range(passes + 1):
        ts = [threading.Thread(target=np.add.reduce, args=(p,)) for p in parts]
        t0 = time.perf_counter()
        for t in ts:
            t.start()
        for t in ts:
            t.join()
        best = max(best, a.nbytes / (time.perf_counter() - t0) / 1e9)
    return round(best, 1), cores


def cpu_baseline(w, reps=3):
    """The fp64 oracle as it stands, on the host cores: median of `reps` whole
    passes of the workload with every core (OpenMP over (sequence, head)) and
    with one core, next to the host CPU model and its read bandwidth."""
    import oracle
    x = workloads.inputs_for(w)
    cores = os.cpu_count() or 1

    def median_pass(threads):
        times = []
        for _ in range(reps):
            t0 = time.perf_counter()
            oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"],
                           n_threads=threads)
            times.append(time.perf_counter() - t0)
        return statistics.median(times)

    t_all = median_pass(cores)
    t_one = median_pass(1)
    gbs, bw_threads = host_read_gbs()
    return dict(value=w.total_tokens / t_all, unit="tokens/s", cores=cores, kind="oracle",
                sample=f"median of {reps} full passes of the workload ({w.total_tokens} tokens x {w.Hv} heads) "
                       f"with {cores} threads: {t_all:.3f} s each",
                single_core={"value": w.total_tokens / t_one, "unit": "tokens/s", "cores": 1,
                             "sample": f"median of {reps} full passes with 1 thread: {t_one:.2f} s each"},
                cpu_model=cpu_model(),
                host_read_gbs={"value": gbs, "threads": bw_threads,
                               "method": "every core sums its slice of a 1 GiB fp64 array, best of 5 passes"})


def l2_copies(w):
    """Copies of a prefill workload's inputs the GPU arm rotates over between
    timed calls, so that they span more than 3x the 126 MB L2."""
    one = prefill_bytes(w.total_tokens, w.Hqk, w.Hv, w.d, len(w.lengths), w.state_std > 0)
    return max(2, -(-3 * L2_BYTES // one))


def workload_config(w, copies=None, n=1):
    if w.kind == "decode":
        return {"workload": f"{w.name}: {w.batch} sequences x 1 token, {w.steps} consecutive steps, "
                            f"Hqk={w.Hqk} Hv={w.Hv} d_k=d_v={w.d} {w.dtype}, fp32 state in place",
                "global_batch": w.batch * n, "seq_len": 1,
                "parallelism": f"dp{n} (independent sequences per rank, no exchange)"}
    cfg = {"workload": f"{w.name}: {w.kind} "
                       + (f"T={w.lengths[0]}" if len(w.lengths) == 1 else f"{len(w.lengths)} seqs "
                          f"(total {w.total_tokens} tokens)")
                       + f" Hqk={w.Hqk} Hv={w.Hv} d_k=d_v={w.d} {w.dtype} chunk={w.chunk}",
           "global_batch": len(w.lengths) * n, "seq_len": w.total_tokens,
           "parallelism": f"dp{n} (independent sequences per rank, no exchange)"}
    if copies:
        cfg["l2"] = f"GPU arm: inputs rotated over {copies} copies (> 3x the 126 MB L2)"
    return cfg


def prefill_subline(r, w, steps, ms_max, world, pk, pk_kind, traffic=None):
    """A prefill workload's sub-object of the JSON line (traffic: DRAM bytes per
    launch from an ncu capture, or None)."""
    fl = prefill_flops_per_token_head(w.chunk, w.d) * r["tokens"] * w.Hv
    return {"value": aggregate_rate(r["tokens"], ms_max, world), "unit": "tokens/s", "ms_per_step": ms_max,
            "steps": steps, "timed_replays": r["replays"], "gpu_launches": steps,
            "config": workload_config(w, r["copies"], world),
            "roofline": roofline_tensor(fl, r["ms"], pk, pk_kind, traffic=traffic),
            "roofline_hbm_view": roofline_hbm(r["bytes"], r["ms"], pk, pk_kind),
            "binding_frac": binding_frac(fl, r["bytes"], r["ms"], pk)}


def roofline_tensor(flops, ms, pk, kind, key="bf16_tflops", traffic=None):
    achieved = flops / (ms * 1e-3) / 1e12
    peak = pk[key]
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": f"{key} ({kind})"}


def roofline_hbm(nbytes, ms, pk, kind, traffic=None):
    achieved = nbytes / (ms * 1e-3) / 1e9
    peak = pk["hbm_gbs"]
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": f"hbm_gbs ({kind})"}


def binding_frac(flops, nbytes, ms, pk):
    """Fraction of the binding roofline: the larger of the tensor time and the
    HBM time at the measured peaks, over the measured time."""
    t_tc = flops / (pk["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    return round(max(t_tc, t_hbm) / (ms * 1e-3), 4)


# -------------------------------------------------------------------- main ---
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill", choices=["prefill", "long", "varlen", "decode"])
    ap.add_argument("--no-extras", action="store_true", help="main workload only (for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = workloads.workload(args.workload)

    if args.impl == "reference":
        if rank != 0:
            return
        times = []
        cores = os.cpu_count() or 1
        import oracle
        x = workloads.inputs_for(w) if w.kind == "prefill" else None
        if w.kind == "decode":
            state = workloads.decode_state(w.batch, w.Hv, w.d).double().numpy()
            xs = [workloads.decode_step_inputs(s, w.batch, w.Hqk, w.Hv, w.d) for s in range(4)]

        def ref_step(i):
            if w.kind == "prefill":
                oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], x["cu_seqlens"],
                               n_threads=cores)
            else:
                xi = xs[i % 4]
                oracle.decode(xi["q"], xi["k"], xi["v"], xi["g"], xi["beta"], state, n_threads=cores)

        for i in range(args.warmup):
            ref_step(i)
        t0 = time.perf_counter()
        for i in range(args.steps):
            ref_step(i)
        el = time.perf_counter() - t0
        ms = el * 1e3 / args.steps
        if w.kind == "prefill":
            value, unit = w.total_tokens / (ms * 1e-3), "tokens/s"
        else:
            value, unit = 1.0 / (ms * 1e-3), "steps/s"
        sample = (f"{args.steps} step(s) of the whole workload, fp64 C oracle, OpenMP over "
                  f"(sequence, head), {cores} threads")
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
                "config": workload_config(w, l2_copies(w) if w.kind == "prefill" else None),
                "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    # ------------------------------------------------------------ our arm ---
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=120))
    import gated_deltanet_linear_21_b200 as gdn

    pk, pk_kind = peaks()

    def max_over_ranks(x):
        return reduce_max(x, world, device)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize()

    if w.kind == "prefill":
        clk = ClockSampler(local)
        barrier()
        r = run_prefill_bench(gdn, w, args.steps, args.warmup, device, rank, clk)
        barrier()
        ms = max_over_ranks(r["ms"])
        value = aggregate_rate(r["tokens"], ms, world)
        flops = prefill_flops_per_token_head(w.chunk, w.d) * r["tokens"] * w.Hv
        # the ncu captures were taken on the 4096-token layer and on the 32768-token prompt
        tr = traffic_record({"prefill": "prefill_pc", "long": "prefill_pc_long"}.get(w.name, "")) \
            if w.total_tokens in (4096, 32768) else None
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
                "config": workload_config(w, r["copies"], world),
                "roofline": roofline_tensor(flops, r["ms"], pk, pk_kind,
                                            traffic=tr["bytes_per_launch"] if tr else None),
                "roofline_hbm_view": roofline_hbm(r["bytes"], r["ms"], pk, pk_kind),
                "binding_frac": binding_frac(flops, r["bytes"], r["ms"], pk),
                "timed_replays": r["replays"],
                "gpu_launches": args.steps, "clocks": clk.summary()}
        del r["graph"]
    else:
        clk = ClockSampler(local)
        barrier()
        r = run_decode_bench(gdn, w, w.steps, args.warmup, device, rank, clk)
        barrier()
        ms = max_over_ranks(r["ms"])
        tr = traffic_record("decode")
        line = {"metric": METRIC, "value": aggregate_rate(1, ms, world), "unit": "steps/s", "n_gpus": world,
                "steps": r["steps"], "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
                "config": dict(workload_config(w, None, world),
                               l2="state 134 MB > 126 MB L2; fresh q/k/v buffers every step"),
                "roofline": roofline_hbm(r["bytes"], r["ms"], pk, pk_kind,
                                         traffic=tr["bytes_per_launch"] if tr else None),
                "gpu_launches": r["steps"], "clocks": clk.summary()}

    if not args.no_extras and w.kind == "prefill":
        # decode workload: 1000 consecutive steps, fresh tokens each step
        wd = workloads.workload("decode")
        rd = run_decode_bench(gdn, wd, wd.steps, args.warmup, device, rank)
        msd = max_over_ranks(rd["ms"])
        trd = traffic_record("decode")
        line["decode"] = {"value": aggregate_rate(1, msd, world), "unit": "steps/s", "ms_per_step": msd,
                          "steps": rd["steps"], "gpu_launches": rd["steps"],
                          "config": workload_config(wd, None, world),
                          "roofline": roofline_hbm(rd["bytes"], rd["ms"], pk, pk_kind,
                                                   traffic=trd["bytes_per_launch"] if trd else None)}
        # the same decode with the state stored in bf16 (gdn_decode_bf16_state)
        rh = run_decode_bench(gdn, wd, wd.steps, args.warmup, device, rank, state_dtype=torch.bfloat16)
        msh = max_over_ranks(rh["ms"])
        line["decode_bf16_state"] = {"value": aggregate_rate(1, msh, world), "unit": "steps/s", "ms_per_step": msh,
                                     "steps": rh["steps"], "gpu_launches": rh["steps"],
                                     "config": dict(workload_config(wd, None, world), state="bf16 (fp32 arithmetic)"),
                                     "roofline": roofline_hbm(rh["bytes"], rh["ms"], pk, pk_kind)}
        # one request at a time: B=1 decode, 1000 steps in one CUDA graph
        wb = workloads.Workload("decode_b1", 2, "decode", batch=1, steps=1000, Hqk=16, Hv=32,
                                state_std=wd.state_std)
        rb = run_decode_bench(gdn, wb, wb.steps, args.warmup, device, rank)
        msb = max_over_ranks(rb["ms"])
        line["decode_b1"] = {"value": aggregate_rate(1, msb, world), "unit": "steps/s", "ms_per_step": msb,
                             "steps": rb["steps"], "gpu_launches": rb["steps"],
                             "config": workload_config(wb, None, world),
                             "roofline": roofline_hbm(rb["bytes"], rb["ms"], pk, pk_kind)}
        # long prompt: 32768 tokens, 16 q/k and 32 v heads
        wl = workloads.workload("long")
        nl = max(2, args.steps // 4)
        rl = run_prefill_bench(gdn, wl, nl, args.warmup, device, rank)
        del rl["graph"]
        msl = max_over_ranks(rl["ms"])
        fl = prefill_flops_per_token_head(wl.chunk, wl.d) * rl["tokens"] * wl.Hv
        trl = traffic_record("prefill_pc_long")   # captured on this workload itself
        line["long_prefill"] = prefill_subline(rl, wl, nl, msl, world, pk, pk_kind,
                                               traffic=trl["bytes_per_launch"] if trl else None)
        # the longest prompt: 81920 tokens, 16 q/k and 32 v heads
        wx = workloads.workload("long", T=81920)
        nx = max(2, args.steps // 10)
        rx = run_prefill_bench(gdn, wx, nx, args.warmup, device, rank)
        del rx["graph"]
        # (the 32768-token capture scaled by the tokens: every (head, chunk) moves the same bytes)
        line["long_prefill_81920"] = prefill_subline(
            rx, wx, nx, max_over_ranks(rx["ms"]), world, pk, pk_kind,
            traffic=round(trl["bytes_per_launch"] * wx.total_tokens / wl.total_tokens) if trl else None)
        if trl:
            line["long_prefill_81920"]["roofline"]["traffic_scaled_from"] = "the 32768-token capture, by tokens"
        # packed varlen: 8 sequences of 128..8192 tokens with their own states
        wv = workloads.workload("varlen")
        nv = max(2, args.steps // 4)
        rv = run_prefill_bench(gdn, wv, nv, args.warmup, device, rank)
        del rv["graph"]
        line["varlen_prefill"] = prefill_subline(rv, wv, nv, max_over_ranks(rv["ms"]), world, pk, pk_kind)
        # the 4096-token layer with f16 inputs and output
        wf = workloads.workload("prefill", dtype="f16")
        rf = run_prefill_bench(gdn, wf, args.steps, args.warmup, device, rank)
        del rf["graph"]
        line["prefill_f16"] = prefill_subline(rf, wf, args.steps, max_over_ranks(rf["ms"]), world, pk, pk_kind)

    if w.kind == "prefill":
        e = run_e2e(gdn, w, max(3, args.steps // 2), device)
        ems = max_over_ranks(e["ms"])
        line["e2e"] = {"value": aggregate_rate(e["tokens"], ems, world), "unit": "tokens/s",
                       "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"]}
    if rank == 0 and world == 1 and not args.no_extras and w.kind == "prefill":
        line["cpu_baseline"] = cpu_baseline(w)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
