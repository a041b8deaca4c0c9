"""Benchmark of the hybrid-block decode step (full layer + selection + sparse layers).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2] [--impl hs2|reference]

One step = hs2_full_attn (split-K flash-decode) + hs2_select (importance, exact
top-k, window merge) + one hs2_sparse_attn per reusing layer, for every sequence
of the batch, on device-resident synthetic inputs.  L2 is flushed before every
timed step, outside the timed interval: a 256 MiB buffer is written, then another
256 MiB buffer is read, so that the write-back of the flush's own dirty lines does
not land in the timed step either.  Rank 0 prints one JSON line.

With N > 1 (torchrun), every rank runs an independent replica of the workload on
its own GPU (the step has no exchange between sequences): weak scaling.
``--impl reference`` times the float64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from long_context_token_b200 import workloads  # noqa: E402

METRIC = "hybrid-block decode steps/s & HBM GB/s (full+select+sparse) at 128K-1M ctx"
UNIT = "steps/s"
FLUSH_BYTES = 256 << 20
LAUNCHES_PER_STEP_FUSED = 1     # full layer with the split merge and selection in its tail
LAUNCHES_PER_STEP_FULL = 2      # split-K flash-decode, split merge (other shapes)
LAUNCHES_PER_STEP_SELECT = 3    # importance+histogram, compaction, exact finish
LAUNCHES_PER_STEP_BLOCKS = 2    # importance, exact block selection
LAUNCHES_PER_FULL_FUSED = 1     # full layer merging its own split partials (block mode)
LAUNCHES_PER_SPARSE = 1         # gather attention with the split merge on chip (cluster)


# DRAM bytes (read + write) of one full-layer launch, from an ncu capture of the same
# kernel (dram__bytes_read.sum + dram__bytes_write.sum): the one-launch full layer (stream,
# split merge and token selection) where "fused"; the captures are summarised in profiles/.
NCU_TRAFFIC = {
    2: {"bytes": 4 * (134_890_752 + 659_328), "kernel": "full_attn_tc_kernel<16, 0>",
        "capture": "2 x 131072 keys (two launches averaged), scaled x4", "fused": True},
    3: {"bytes": 246_885_888 + 3_051_008, "kernel": "full_attn_fp8_kernel<16, 0>",
        "capture": "the whole launch", "fused": True},
    4: {"bytes": 277_461_760 + 4_877_824, "kernel": "full_attn_fp8_kernel<64, 0>",
        "capture": "the whole launch", "fused": True},
    5: {"bytes": 67_430_656 + 3_554_816, "kernel": "full_attn_mq_kernel<16>",
        "capture": "the whole launch", "fused": False},
}


def roofline_of(w, ab, full_s, peaks, peak_kind) -> dict:
    """Roofline of the dominant kernel (the full layer, measured with its split merge):
    HBM-bound for one query token per sequence (16-64 flop per byte), tensor-bound for
    several tokens per sequence (each K/V tile serves 128/h tokens)."""
    if w.n_q > 1:
        achieved = ab["full_flops"] / full_s / 1e12
        peak = float(peaks["bf16_tflops"])
        return {"bound": "tensor", "kernel": "full_attn_mq (several-token flash attention)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_kind": peak_kind + " bf16 burst", "alg_flops_per_launch": ab["full_flops"]}
    achieved = ab["full"] / full_s / 1e9
    peak = float(peaks["hbm_gbs"])
    return {"bound": "hbm", "kernel": "full_attn (split-K flash-decode)", "achieved": achieved,
            "peak": peak, "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time: every rank contributes its device-timed total and gets
    the max back (a no-op without a process group).  The replicas share nothing else."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, total_ms: float) -> float:
    """Steps/s of the whole job: each of the `world` replicas ran `steps` steps, and the
    job took as long as its slowest rank (weak scaling: per-GPU work is fixed)."""
    return world * steps / (total_ms / 1e3)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def alg_bytes(w: workloads.Workload, lens) -> dict:
    """Bytes the method must move per step (see the design notes): K and V of every
    visible row once, each sparse layer's gathered rows, indices, queries, outputs."""
    d = 128
    elem = 1 if w.kv == "fp8" else 2
    row = d * elem + (4 if w.kv == "fp8" else 0)      # one K (or V) row incl. its scale
    ctx_rows = int(sum(int(L) for L in lens))
    width = w.window + w.k_sel
    sel_rows = sum(min(int(L) - w.n_q + i + 1, width) for L in lens for i in range(w.n_q))
    q_bytes = w.batch * w.n_q * w.h_q * d * 2
    out_bytes = w.batch * w.n_q * w.h_q * d * 4
    full = 2 * ctx_rows * row + q_bytes + out_bytes
    idx_bytes = w.batch * w.n_q * width * 4
    sparse = 2 * sel_rows * row + idx_bytes + q_bytes + out_bytes
    # Dense work of the full layer: Q.K^T and P.V over every visible (row, key) pair,
    # 2 * 128 flops each (the several-token case is bound by these, not by bytes).
    vis = sum(int(L) - w.n_q + i + 1 for L in lens for i in range(w.n_q))
    full_flops = 2 * 2 * d * w.h_q * vis
    return dict(full=full, step=full + idx_bytes + w.n_sparse * sparse, sparse=sparse,
                kv_once=2 * ctx_rows * row, full_flops=full_flops)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed loop runs."""

    def __init__(self, device: torch.device):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no clocks rather than guess
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
            "sw_power_cap": getattr(nv, "nvmlClocksThrottleReasonSwPowerCap", 0x4),
            "hw_power_brake": getattr(nv, "nvmlClocksThrottleReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            self._stop.wait(0.001)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def oracle_sample(inp: workloads.Inputs, w: workloads.Workload, budget_s: float,
                  block: int = 1):
    """Time the float64 oracle on whole sequences of the workload until `budget_s`
    has passed (at least one).  Returns (seconds, sequences done)."""
    import oracle
    bits = workloads.numpy_bits(inp)
    t0 = time.perf_counter()
    done = 0
    while True:
        b = done % w.batch
        sub = dict(bits)
        for key in ("q", "k", "v", "k_scale", "v_scale", "lens"):
            if sub[key] is not None:
                sub[key] = bits[key][b:b + 1]
        sub["q_layers"] = [ql[b:b + 1] for ql in bits["q_layers"]]
        oracle.hybrid_block_step(sub, block)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return time.perf_counter() - t0, done


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, w):
    """The reference arm: the float64 CPU oracle.  Each of its steps is a bounded sample
    of the workload, one sequence of the batch (1/B of a whole step); `value` is in
    whole-workload steps/s (sequences/s divided by B) and `ms_per_step` is the measured
    time of one such sample, so that steps x ms_per_step is the time spent."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    inp = workloads.generate(w)
    for _ in range(args.warmup):
        oracle_sample(inp, w, 0.0, args.block)
    secs, seqs = 0.0, 0
    for _ in range(args.steps):
        s, n = oracle_sample(inp, w, 0.0, args.block)
        secs += s
        seqs += n
    value = seqs / (secs * w.batch)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "step": f"one sequence of the batch of {w.batch} (1/{w.batch} of a whole step); "
                "value = sequences/s / batch",
        "sequences_timed": seqs, "seconds_timed": secs,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args.block, args.deterministic),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                         "sample": f"{seqs} whole sequences of the batch, one per step, "
                                   "full layer + selection + every sparse layer in float64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_prefill(args, w):
    """Chunked prefill of the full layer (no selection): args.prefill new tokens per
    sequence of the workload's cache, timed like the decode step (CUDA graph replays,
    L2 flushed before each, CUDA events on the launching stream).  One GPU."""
    from long_context_token_b200 import hs2
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--prefill runs on one GPU")
    if w.kv != "bf16":
        raise SystemExit("--prefill needs a bf16 workload")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    n = args.prefill
    inp = workloads.make_inputs(w.batch, w.max_len, n_q=n, h_q=w.h_q, kv="bf16", seed=w.seed,
                                n_sparse=0)
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev))
    q = inp.q.to(dev)
    ws = hs2.prefill_workspace(cache, n, w.h_q)
    out = torch.empty(w.batch, n, w.h_q, 128, dtype=torch.float32, device=dev)
    lse = torch.empty(w.batch, n, w.h_q, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(k):
        flush.fill_(float(k))
        torch.sum(drain, dim=0, out=drain_out)

    def step():
        hs2.prefill_attn(q, cache, inp.sm_scale, ws, out=out, lse=lse)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush_l2(1)
        graph.replay()
    torch.cuda.synchronize()
    if hs2.check_device_status(ws) != 0:
        raise RuntimeError("device-side error during warm-up")
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    replay_ms = []
    wall0 = time.perf_counter()
    with ClockSampler(dev) as clk:
        for k in range(args.steps):
            flush_l2(k)
            torch.cuda.nvtx.range_push("hs2 step")
            start.record(stream)
            graph.replay()
            end.record(stream)
            torch.cuda.nvtx.range_pop()
            end.synchronize()
            replay_ms.append(start.elapsed_time(end))
    wall = time.perf_counter() - wall0
    status = hs2.check_device_status(ws)
    total_ms = sum(replay_ms)
    tokens = w.batch * n
    # Q.K^T and P.V over every visible (row, key) pair: 2 * 2 * 128 flops each.
    vis = sum(int(L) - n + i + 1 for L in inp.lens.tolist() for i in range(n))
    flops = 4 * 128 * w.h_q * vis
    peaks, peak_kind = measured_peaks()
    avg_s = total_ms / args.steps / 1e3
    line = {
        "metric": "chunked-prefill full layer tokens/s", "value": tokens * args.steps / (total_ms / 1e3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w) | {"workload": f"prefill chunk {n} x h{w.h_q} vs "
                                              f"{w.batch} x {w.max_len} bf16", "n_q": n,
                                  "selection": "none (full layer only)"},
        "roofline": {"bound": "tensor", "kernel": "full_attn_mq + split merge",
                     "achieved": flops / avg_s / 1e12, "peak": float(peaks["bf16_tflops"]),
                     "unit": "TFLOP/s", "frac": flops / avg_s / 1e12 / float(peaks["bf16_tflops"]),
                     "peak_kind": peak_kind + " bf16 burst", "alg_flops_per_launch": flops,
                     "traffic": None},
        "gpu_launches": args.steps * 2,
        "clocks": clk.summary(),
        "device_status": status,
        "wall_s_timed_region": wall,
    }
    if not args.no_e2e:
        hq = inp.q.clone().pin_memory()
        hout = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        hlse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            hs2.prefill_attn(q, cache, inp.sm_scale, ws, out=out, lse=lse)
            hout.copy_(out, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            e2e_step()
        e_ms = 0.0
        for k in range(args.steps):
            flush_l2(k)
            torch.cuda.nvtx.range_push("hs2 step end to end")
            start.record(stream)
            g2.replay()
            end.record(stream)
            torch.cuda.nvtx.range_pop()
            end.synchronize()
            e_ms += start.elapsed_time(end)
        line["e2e"] = {"value": tokens * args.steps / (e_ms / 1e3), "unit": "tokens/s",
                       "h2d_bytes_per_step": hq.numel() * 2,
                       "d2h_bytes_per_step": hout.numel() * 4 + hlse.numel() * 4,
                       "path": "hs2 C ABI via the Python binding, step replayed from a CUDA graph"}
        del g2
    del graph
    if not args.no_cpu_baseline:
        import oracle
        bits = workloads.numpy_bits(inp)
        k = 8  # the chunk's first tokens of the first sequence
        sub = dict(bits, q=bits["q"][:1, :k], k=bits["k"][:1], v=bits["v"][:1],
                   lens=(bits["lens"][:1] - (n - k)).astype(bits["lens"].dtype))
        t0 = time.perf_counter()
        done = 0
        while True:
            oracle.prefill_attn(sub)
            done += k
            if time.perf_counter() - t0 >= args.cpu_budget:
                break
        secs = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": done / secs, "unit": "tokens/s", "cores": host_cores(),
                                "kind": "oracle",
                                "sample": f"{done} tokens ({k} per call: the chunk's first {k} "
                                          f"tokens of sequence 0, same positions) in {secs:.1f} s, "
                                          "float64 numpy oracle"}
    print(json.dumps(line), flush=True)


def config_of(w, block: int = 1, deterministic: bool = False):
    # The one-launch full layer (one token per row, up to 64 heads; any FP8 shape up to 64
    # heads) shares each row's key tiles out at run time unless asked for fixed chunks.
    one_launch = w.h_q <= 64 and (w.kv == "fp8" or w.n_q == 1)
    shared = one_launch and not deterministic
    return {"workload": w.name, "batch": w.batch, "context": w.max_len,
            "selection": "token" if block == 1 else f"blocks of {block} positions",
            "ragged_from": w.len_lo, "n_q": w.n_q, "h_q": w.h_q, "h_kv": 1, "head_dim": 128,
            "kv_cache": w.kv, "window": w.window, "k_sel": w.k_sel, "sparse_layers": w.n_sparse,
            "key_tiles": ("shared out among a row's CTAs at run time" if shared
                          else "fixed chunks per CTA (bitwise-reproducible runs)"),
            "l2": "flushed before every timed step (256 MiB write, then 256 MiB read of "
                  "another buffer)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", type=int, default=2, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="hs2", choices=["hs2", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle time for the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="fixed key chunks per CTA in the full layer (hs2_set_deterministic)")
    ap.add_argument("--block", type=int, default=1,
                    help="1: token-level selection (the method); N > 1: whole blocks of N "
                         "positions (the first-generation comparator)")
    ap.add_argument("--prefill", type=int, default=0,
                    help="N > 0: time the chunked-prefill full layer for N new tokens per "
                         "sequence of the workload's bf16 cache instead of the decode step")
    ap.add_argument("--batch", type=int, default=None,
                    help="run fewer sequences of the workload (profiling captures only)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = workloads.WORKLOADS[args.workload]
    if args.batch is not None:
        import dataclasses
        w = dataclasses.replace(w, batch=args.batch, name=f"{w.name} (first {args.batch} seqs)")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.prefill > 0:
        return run_prefill(args, w)

    from long_context_token_b200 import hs2
    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    inp = workloads.generate(w)
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev),
                      None if inp.k_scale is None else inp.k_scale.to(dev),
                      None if inp.v_scale is None else inp.v_scale.to(dev))
    B, n_q, h = w.batch, w.n_q, w.h_q
    width = w.window + w.k_sel
    n_layers = len(inp.q_layers)
    ws = hs2.alloc_workspace(cache, n_q, h, w.window, w.k_sel)
    fused = args.block == 1 and hs2.select_fused(cache, n_q, h)
    hs2.set_deterministic(args.deterministic)
    # Every input of a step (the full layer's queries, then each sparse layer's) sits in
    # one device buffer, and every result (the full layer's output, each sparse layer's
    # output, then the index set) in another, so that the end-to-end leg moves each with
    # a single copy.  Offsets are multiples of 16 bytes.
    q_elems = B * n_q * h * 128
    din = torch.empty((1 + n_layers) * q_elems, dtype=torch.bfloat16, device=dev)
    q = din[:q_elems].view(B, n_q, h, 128)
    qls = [din[(1 + i) * q_elems:(2 + i) * q_elems].view(B, n_q, h, 128) for i in range(n_layers)]
    q.copy_(inp.q)
    for d_, h_ in zip(qls, inp.q_layers):
        d_.copy_(h_)
    o_bytes = q_elems * 4
    idx_bytes = B * n_q * width * 4
    dout = torch.empty((1 + n_layers) * o_bytes + idx_bytes, dtype=torch.uint8, device=dev)
    out = dout[:o_bytes].view(torch.float32).view(B, n_q, h, 128)
    outs = [dout[(1 + i) * o_bytes:(2 + i) * o_bytes].view(torch.float32).view(B, n_q, h, 128)
            for i in range(n_layers)]
    idx = dout[(1 + n_layers) * o_bytes:].view(torch.int32).view(B, n_q, width)
    lse = torch.empty(B, n_q, h, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    drain_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(k):
        flush.fill_(float(k))
        torch.sum(drain, dim=0, out=drain_out)
    stream = torch.cuda.current_stream(dev)

    from cuda.bindings import runtime as cudart

    def cuda_ok(res):
        err = res[0] if isinstance(res, tuple) else res
        if int(err) != 0:
            raise RuntimeError(f"CUDA runtime call failed: {err}")
        return res[1] if isinstance(res, tuple) and len(res) > 1 else None

    # Phase marks recorded from inside the captured graph (external event-record nodes),
    # so the per-phase durations come from replays of the same step.
    marks = [cuda_ok(cudart.cudaEventCreate()) for _ in range(4)]

    def mark(k):
        cuda_ok(cudart.cudaEventRecordWithFlags(marks[k], stream.cuda_stream,
                                                cudart.cudaEventRecordExternal))

    def first_layer(with_marks=False):
        """The full layer and the selection: one call (hs2_full_attn_select) for the token
        selection, as a user makes it; the full layer and the block selection for the
        comparator.  The marked capture splits the token path into its two calls where
        they are separate kernels anyway, to time the full layer alone."""
        if args.block > 1:
            hs2.full_attn(q, cache, w.window, w.k_sel, inp.sm_scale, ws, out=out, lse=lse)
            if with_marks:
                mark(1)
            hs2.select_blocks(q, cache, ws, w.window, w.k_sel, args.block, inp.sm_scale, idx=idx)
        elif fused or not with_marks:
            hs2.full_attn_select(q, cache, w.window, w.k_sel, inp.sm_scale, ws, out=out, idx=idx,
                                 lse=lse)
            if with_marks:
                mark(1)
        else:
            hs2.full_attn(q, cache, w.window, w.k_sel, inp.sm_scale, ws, out=out, lse=lse)
            if with_marks:
                mark(1)
            hs2.select(q, cache, ws, w.window, w.k_sel, inp.sm_scale, idx=idx)

    def step(with_marks=False):
        if with_marks:
            mark(0)
        first_layer(with_marks)
        if with_marks:
            mark(2)
        for ql, o in zip(qls, outs):
            hs2.sparse_attn(ql, cache, idx, ws, inp.sm_scale, out=o)
        if with_marks:
            mark(3)

    # Eager warm-up (first launches set kernel attributes), then one step is captured in
    # a CUDA graph and replayed: no host launch overhead inside the timed intervals.
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    # Two captures of the same step: the timed one has nothing between the kernels (a
    # kernel may start while its predecessor drains, as in a real decode loop); the other
    # carries event-record nodes between the phases and gives the per-phase durations
    # (the record nodes serialise the phases, so its total is a little longer).
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph_marked = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_marked):
        stream = torch.cuda.current_stream(dev)
        step(with_marks=True)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush_l2(1)
        graph.replay()
        flush_l2(1)
        graph_marked.replay()
    torch.cuda.synchronize()
    if hs2.check_device_status(ws) != 0:
        raise RuntimeError("device-side error during warm-up")

    def elapsed(a, b):
        return float(cuda_ok(cudart.cudaEventElapsedTime(marks[a], marks[b])))

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    step_ms, first_ms, full_ms, sel_ms, sp_ms, replay_ms = [], [], [], [], [], []
    with ClockSampler(dev) as clk:
        for k in range(args.steps):
            flush_l2(k)
            torch.cuda.nvtx.range_push("hs2 step")
            start.record(stream)
            graph.replay()
            end.record(stream)
            torch.cuda.nvtx.range_pop()
            end.synchronize()
            replay_ms.append(start.elapsed_time(end))
        if world > 1:
            torch.distributed.barrier()
        wall = time.perf_counter() - wall0
        for k in range(args.steps):
            flush_l2(k)
            torch.cuda.nvtx.range_push("hs2 step with phase marks")
            graph_marked.replay()
            torch.cuda.nvtx.range_pop()
            end.record(stream)
            end.synchronize()
            step_ms.append(elapsed(0, 3))
            first_ms.append(elapsed(0, 2))
            full_ms.append(elapsed(0, 1))
            sel_ms.append(elapsed(1, 2))
            sp_ms.append(elapsed(2, 3))
    if world > 1:
        torch.distributed.barrier()
    total_ms = max_over_ranks(sum(replay_ms), dev)
    status = hs2.check_device_status(ws)

    # End to end through the public API: each step copies its queries from pinned host
    # memory in one copy, runs the full layer + selection + sparse layers and copies every
    # result (the outputs and the index set) back in one copy; the step is replayed from
    # a CUDA graph, as a serving loop would.  The KV cache is device-resident model state.
    e2e = None
    if not args.no_e2e:
        hin = torch.empty(din.shape, dtype=din.dtype).pin_memory()
        hin.copy_(din.cpu())
        hout = torch.empty(dout.shape, dtype=dout.dtype).pin_memory()

        def e2e_step():
            din.copy_(hin, non_blocking=True)
            if args.block > 1:
                hs2.full_attn_select_blocks(q, cache, w.window, w.k_sel, args.block,
                                            inp.sm_scale, ws, out=out, idx=idx, lse=lse)
            else:
                hs2.full_attn_select(q, cache, w.window, w.k_sel, inp.sm_scale, ws, out=out,
                                     idx=idx, lse=lse)
            for ql, o in zip(qls, outs):
                hs2.sparse_attn(ql, cache, idx, ws, inp.sm_scale, out=o)
            hout.copy_(dout, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            e2e_step()
        for _ in range(3):
            g2.replay()
        torch.cuda.synchronize()
        e_ms = 0.0
        for k in range(args.steps):
            flush_l2(k)
            torch.cuda.nvtx.range_push("hs2 step end to end")
            start.record(stream)
            g2.replay()
            end.record(stream)
            torch.cuda.nvtx.range_pop()
            end.synchronize()
            e_ms += start.elapsed_time(end)
        e_ms = max_over_ranks(e_ms, dev)
        e2e = {"value": whole_job_rate(world, args.steps, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(hin.numel() * hin.element_size()),
               "d2h_bytes_per_step": int(hout.numel()),
               "copies_per_step": {"h2d": 1, "d2h": 1},
               "path": "hs2 C ABI via the Python binding, step replayed from a CUDA graph"}
        del g2
    del graph, graph_marked

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    lens = inp.lens.tolist()
    ab = alg_bytes(w, lens)
    peaks, peak_kind = measured_peaks()
    first_avg = statistics.mean(first_ms if fused else full_ms) / 1e3
    value = whole_job_rate(world, args.steps, total_ms)
    if args.block > 1:
        phases = {"full_attn": statistics.mean(full_ms), "select": statistics.mean(sel_ms)}
        launches = LAUNCHES_PER_FULL_FUSED + LAUNCHES_PER_STEP_BLOCKS
    elif fused:
        phases = {"full_attn_select": statistics.mean(first_ms)}
        launches = LAUNCHES_PER_STEP_FUSED
    else:
        phases = {"full_attn": statistics.mean(full_ms), "select": statistics.mean(sel_ms)}
        launches = LAUNCHES_PER_STEP_FULL + LAUNCHES_PER_STEP_SELECT
    roof = roofline_of(w, ab, first_avg, peaks, peak_kind)
    if fused:
        roof["kernel"] = ("full layer with the split merge and the token selection in its "
                          "tail (one launch)")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.kv == "bf16" else "fp8-e4m3",
        "data": "synthetic", "config": config_of(w, args.block, args.deterministic),
        "hbm_gbs": ab["step"] / (total_ms / args.steps / 1e3) / 1e9,
        "alg_bytes_per_step": ab["step"],
        "phase_ms": phases | {"sparse_layers": statistics.mean(sp_ms),
                              "step_with_phase_marks": statistics.mean(step_ms),
                              "step_p10": float(np.percentile(replay_ms, 10)),
                              "step_p50": float(np.percentile(replay_ms, 50)),
                              "step_p90": float(np.percentile(replay_ms, 90))},
        "roofline": roof | {
                     "alg_bytes_per_launch": ab["full"],
                     "traffic": (NCU_TRAFFIC[args.workload]["bytes"]
                                 if args.workload in NCU_TRAFFIC and args.batch is None
                                 and NCU_TRAFFIC[args.workload]["fused"] == fused else None),
                     "traffic_source": (NCU_TRAFFIC[args.workload]
                                        if args.workload in NCU_TRAFFIC and args.batch is None
                                        and NCU_TRAFFIC[args.workload]["fused"] == fused
                                        else None)},
        "gpu_launches": args.steps * (launches + w.n_sparse * LAUNCHES_PER_SPARSE),
        "clocks": clk.summary(),
        "device_status": status,
        "wall_s_timed_region": wall,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline:
        secs, seqs = oracle_sample(inp, w, args.cpu_budget, args.block)
        cv = seqs / (secs * w.batch)
        line["cpu_baseline"] = {"value": cv, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                                "sample": f"{seqs} one-sequence hybrid-block steps (sequences "
                                          f"taken in turn from the {w.batch} of the batch) in "
                                          f"{secs:.1f} s, float64 numpy oracle; steps/s = "
                                          f"sequences/s / {w.batch}"}
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
