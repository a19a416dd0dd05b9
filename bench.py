"""Throughput of the quantised top-k MoE FFN layer forward on B200.

One step = one qmoe_forward (router, schedule, gate/up GEMM, down GEMM,
combine) over one batch of seeded synthetic tokens already resident in HBM.
Headline workload: the decode-shaped layer (d=2048, E=128, top-8, I=768, INT4
group-128 weights) at T=256 tokens, the largest of its token sweep; the
other sweep points are reported under "sweep".  On one GPU the same run then
measures the prefill (T=8192, FP8), fine-grained + shared (T=4096, INT4,
Zipf 1.2) and mixed-precision (T=16384, INT8/INT4, Zipf 1.0) layers, each
under "configs" with its own roofline, warm-L2 companion, host-buffer e2e,
realised expert load and CPU-oracle baseline.  L2 (126 MB) is flushed by
writing a 256 MB buffer between timed steps, outside each step's events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--T T] [--also NAME ...]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the same workload

Multi-GPU (torchrun, one rank per GPU): the layer does not shard; every rank
runs an independent replica on its own batch (weak scaling, no collective on
the data path).  Timing is the max over ranks; value counts all ranks' tokens.
Under torchrun only the headline workload runs (unless --also-multi).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s on 1xB200; % of HBM / tensor-core roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
ROOF_TIMING = ("CUDA events around every gate/up launch on its stream, in a second pass of the same steps "
               "(L2 flushed between steps); avg_launch_ms is the gate/up time per step, summed over its "
               "launches_per_step launches (one per weight format); peak = the measured burst figure")


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(backend: str):
    import torch.distributed as dist
    world, rank, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float across the job (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, tokens_per_rank: int, local_ms: float, device=None):
    """(step ms, whole-job tokens/s): the slowest rank's step time, and every
    rank's tokens over that time."""
    ms = max_over_ranks(local_ms, device)
    return ms, world * tokens_per_rank / (ms / 1e3)


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# workload bookkeeping
# ---------------------------------------------------------------------------
def workload_desc(L) -> str:
    from quantized_top_routed_b200 import synth
    fmts = sorted({synth.FMT_NAMES[ex.fmt] for ex in L.experts})
    return (f"{L.name} T={L.T} d={L.d} E={L.E} k={L.k} I={L.I} shared={L.S} "
            f"weights={'+'.join(fmts)}" + (" zipf-bias" if L.router_b is not None else ""))


def compute_dtype(L) -> str:
    """MMA input type: a layer whose experts are all FP8 computes in fp16
    (exact e4m3 -> fp16 conversion), any other layer in bf16."""
    from quantized_top_routed_b200 import synth
    return "f16" if all(ex.fmt == synth.FMT_FP8 for ex in L.experts) else "bf16"


def gate_up_bytes(L, touched) -> int:
    """Algorithmic HBM bytes of one gate/up GEMM launch: the codes and scales of
    every touched expert's W13 (and always-on shared experts), the token rows
    read once and the H rows written once."""
    wb = sum(L.experts[e].w13.nbytes + L.experts[e].s13.nbytes for e in touched)
    wb += sum(L.experts[L.E + s].w13.nbytes + L.experts[L.E + s].s13.nbytes for s in range(L.S))
    return int(wb + L.T * L.d * 2 + L.T * (L.k + L.S) * L.I * 2)


def down_bytes(L, touched) -> int:
    """Algorithmic HBM bytes of one down GEMM launch: W2 codes and scales of every
    touched (and shared) expert, H read once and Y written once."""
    wb = sum(L.experts[e].w2.nbytes + L.experts[e].s2.nbytes for e in list(touched) + list(range(L.E, L.E + L.S)))
    return int(wb + L.T * (L.k + L.S) * L.I * 2 + L.T * (L.k + L.S) * L.d * 2)


def layer_bytes(L, touched) -> int:
    """Algorithmic HBM bytes of one forward: touched experts' weights and scales,
    router weights, x read once and out written once."""
    wb = sum(L.experts[e].w13.nbytes + L.experts[e].s13.nbytes + L.experts[e].w2.nbytes + L.experts[e].s2.nbytes
             for e in list(touched) + list(range(L.E, L.E + L.S)))
    return int(wb + L.router_w.nbytes + 4 * L.T * L.d)


def gate_up_flops(L) -> float:
    return 4.0 * L.T * (L.k + L.S) * L.d * L.I


def layer_flops(L) -> float:
    return 2.0 * L.T * L.d * L.E + 6.0 * L.T * (L.k + L.S) * L.d * L.I


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# clocks sampled during the timed region (NVML, read-only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def time_steps(fn, steps, warmup, flush, stream):
    """Per-step CUDA-event times (ms) on `stream`; L2 flushed between steps
    when `flush` is a buffer (None: warm L2, steps back to back)."""
    import torch
    for _ in range(warmup):
        if flush is not None:
            flush.zero_()
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        if flush is not None:
            flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def route_counts(qmoe, dl, x, T, stream):
    """Per-expert routed-row counts of this batch, from the library's router."""
    import torch
    L = dl.layer
    dev = dl.x.device
    counts = torch.empty(L.E, dtype=torch.int32, device=dev)
    scratch = [torch.empty((T, L.k), dtype=torch.int32, device=dev),
               torch.empty((T, L.k), dtype=torch.float32, device=dev), counts,
               torch.empty(L.E + 1, dtype=torch.int32, device=dev),
               torch.empty(T * L.k, dtype=torch.int32, device=dev),
               torch.empty((T, L.k), dtype=torch.int32, device=dev)]
    qmoe.qmoe_route(dl.handle, x, None, T, *scratch, stream)
    torch.cuda.synchronize()
    return counts.cpu().numpy().astype(np.int64)


def load_report(L, counts):
    """Realised per-expert load of the batch: the routed-row histogram, and for
    a Zipf-biased router the exponent s of a least-squares fit
    log(count) = a - s * log(rank) over the experts that received rows."""
    from quantized_top_routed_b200 import synth
    rep = {"counts": [int(c) for c in counts], "touched_experts": int((counts > 0).sum()),
           "max_over_mean": round(float(counts.max() / max(counts.mean(), 1e-9)), 3)}
    target = synth.CONFIGS.get(L.name, {}).get("zipf")
    if target:
        c = np.sort(counts[counts > 0])[::-1].astype(np.float64)
        r = np.arange(1, len(c) + 1, dtype=np.float64)
        slope = np.polyfit(np.log(r), np.log(c), 1)[0] if len(c) > 1 else float("nan")
        rep.update({"zipf_s_target": target, "zipf_s_fit": round(float(-slope), 3),
                    "fit": "least squares of log(count) on log(rank), experts with rows"})
    return rep


def compute_dtype_note(L) -> str:
    if compute_dtype(L) == "f16":
        return ("f16: every expert is FP8 e4m3, so the grouped GEMMs take fp16 inputs (codes, x rows and H "
                "convert exactly or with >= bf16 precision); x and H must stay inside |v| < 65504; fp32 accumulation")
    return "bf16 MMA inputs (dequantised weights, x rows, H), fp32 accumulation"


def measure_layer(args, name, T, rank, world, dev, peaks, flush, headline):
    """Time one workload through qmoe_forward (device buffers, L2 flushed and
    warm), per-kernel events, the host-buffer entry point, and the roofline of
    the dominant kernel.  Returns the record (without the CPU baseline)."""
    import torch
    from quantized_top_routed_b200 import qmoe, synth

    L = synth.make_layer(name, T=T, seed=args.seed + rank)
    dl = qmoe.DeviceLayer(L, max_tokens=L.T, device=str(dev))
    T = L.T
    stream = torch.cuda.current_stream()
    out = torch.empty((T, L.d), dtype=torch.int16, device=dev)
    counts = route_counts(qmoe, dl, dl.x, T, stream)
    touched = [int(e) for e in np.nonzero(counts)[0]]   # bytes never count untouched experts
    steps = args.steps if headline else min(args.steps, args.other_steps)

    def step():
        qmoe.qmoe_forward(dl.handle, dl.x, T, out, stream)

    # ---- timed region ------------------------------------------------------
    # No per-kernel events here, only the step's own pair.
    barrier(dev)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        times = time_steps(step, steps, args.warmup, flush, stream)
    torch.cuda.synchronize()
    barrier(dev)
    qmoe.qmoe_check_error(dl.handle, stream)
    ms, value = job_rate(world, T, sum(times) / len(times), dev)

    # warm L2: the same steps back to back without the flush
    warm = time_steps(step, steps, args.warmup, None, stream)
    warm_ms, warm_value = job_rate(world, T, sum(warm) / len(warm), dev)

    # ---- per-kernel times: the same steps again with an event pair around
    # every launch (L2 flushed between steps as above) ---------------------------
    qmoe.qmoe_profile(dl.handle, True)
    time_steps(step, min(steps, 100), 0, flush, stream)
    stage_ms, calls = qmoe.qmoe_profile_read(dl.handle)
    qmoe.qmoe_profile(dl.handle, False)

    # ---- end to end through the host-buffer entry point ----------------------
    x_host = torch.from_numpy(L.x.view(np.int16).copy()).pin_memory()
    out_host = torch.empty((T, L.d), dtype=torch.int16).pin_memory()

    def e2e_step():
        qmoe.qmoe_forward_host(dl.handle, x_host, T, out_host, stream)

    barrier(dev)
    e2e_times = time_steps(e2e_step, steps, args.warmup, flush, stream)
    barrier(dev)
    qmoe.qmoe_check_error(dl.handle, stream)
    e2e_ms, e2e_value = job_rate(world, T, sum(e2e_times) / len(e2e_times), dev)

    # ---- roofline of the dominant kernel -----------------------------------
    # gate/up time per step: the sum over its launches (one per weight format
    # present, two in the mixed layer), against the whole gate/up work
    gu_ms = stage_ms["gate_up"] / max(calls, 1)
    gu_launches = len({e.fmt for e in L.experts})
    if L.name in ("decode", "tiny"):
        algo = gate_up_bytes(L, touched)
        achieved = algo / (gu_ms / 1e3) / 1e9
        roof = {"kernel": "grouped_gemm gate/up (SwiGLU)", "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic_from_profiles(L, "gate_up"), "peak_source": peaks["source"],
                "algorithmic_bytes": algo, "avg_launch_ms": round(gu_ms, 5),
                "launches_per_step": gu_launches, "timing": ROOF_TIMING}
    else:
        fl = gate_up_flops(L)
        achieved = fl / (gu_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"kernel": "grouped_gemm gate/up (SwiGLU)", "bound": "tensor", "achieved": round(achieved, 1),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "frac_of_sustained_peak": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "traffic": traffic_from_profiles(L, "gate_up"), "peak_source": peaks["source"],
                "algorithmic_flops": fl, "avg_launch_ms": round(gu_ms, 5),
                "launches_per_step": gu_launches, "timing": ROOF_TIMING}

    rec = {
        "value": round(value, 1), "unit": UNIT, "ms_per_step": round(ms, 5), "steps": steps,
        "dtype": compute_dtype(L), "dtype_note": compute_dtype_note(L),
        "config": {"workload": workload_desc(L), "T": T, "global_batch": world * T,
                   "parallelism": f"replicas x{world}", "l2": "flushed between timed steps (256 MB write)",
                   "touched_experts": len(touched)},
        "warm_l2": {"value": round(warm_value, 1), "ms_per_step": round(warm_ms, 5),
                    "note": "the same steps back to back, L2 not flushed"},
        "layer": {"bytes": layer_bytes(L, touched), "flops": layer_flops(L),
                  "hbm_frac": round(layer_bytes(L, touched) / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                  "tensor_frac": round(layer_flops(L) / (ms / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
                  "stage_ms": {k_: round(v / max(calls, 1), 5) for k_, v in stage_ms.items()}},
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "ms_per_step": round(e2e_ms, 5),
                "h2d_bytes_per_step": int(T * L.d * 2), "d2h_bytes_per_step": int(T * L.d * 2)},
        "gpu_launches": qmoe.qmoe_launches_per_forward(dl.handle, T) * steps,
        "load": load_report(L, counts),
        "clocks": clk.summary(),
    }
    if headline and args.sweep and L.name == "decode" and rank == 0:
        rec["sweep"] = sweep_decode(L, dl, flush, stream, peaks)
    dl.close()
    return L, rec


def run_ours(args):
    import torch
    import oracle.qmoe_oracle as O  # cpu_baseline leg only

    world, rank = init_dist("nccl")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    # The headline workload, then (one GPU, default run) the other workloads,
    # each measured in the same process with its own roofline and baseline.
    names = [args.config] + [n for n in args.also if n != args.config]
    if world > 1 and not args.also_multi:
        names = names[:1]
    result = None
    for i, name in enumerate(names):
        L, rec = measure_layer(args, name, args.T if i == 0 else None, rank, world, dev, peaks, flush, i == 0)
        if rank == 0 and not args.no_cpu_baseline:
            rec["cpu_baseline"] = cpu_baseline(L, O, args)
        del L
        if i == 0:
            result = {"metric": METRIC, "value": rec.pop("value"), "unit": UNIT, "n_gpus": world,
                      "steps": rec.pop("steps"), "warmup": args.warmup, "ms_per_step": rec.pop("ms_per_step"),
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                      "dtype": rec.pop("dtype"), "data": "synthetic (seeded, shapes of the workload)"}
            result.update(rec)
            if len(names) > 1:
                result["configs"] = {}
        else:
            result["configs"][name] = rec
    if rank == 0:
        print(json.dumps(result), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def sweep_decode(L, dl, flush, stream, peaks):
    import dataclasses
    import torch
    from quantized_top_routed_b200 import qmoe
    rows = []
    for T in (1, 8, 32, 128, 256):
        if T > L.T:
            continue
        sub = dataclasses.replace(L, T=T, x=L.x[:T])
        out = torch.empty((T, L.d), dtype=torch.int16, device=dl.x.device)
        xs = dl.x[:T]
        counts = route_counts(qmoe, dl, xs, T, stream)
        touched = [int(e) for e in np.nonzero(counts)[0]]
        fwd = lambda: qmoe.qmoe_forward(dl.handle, xs, T, out, stream)  # noqa: E731
        times = time_steps(fwd, 200, 5, flush, stream)
        qmoe.qmoe_profile(dl.handle, True)
        time_steps(fwd, 100, 0, flush, stream)
        stage_ms, calls = qmoe.qmoe_profile_read(dl.handle)
        qmoe.qmoe_profile(dl.handle, False)
        ms = sum(times) / len(times)
        lb = layer_bytes(sub, touched)
        gu = stage_ms["gate_up"] / max(calls, 1)
        dn = stage_ms["down"] / max(calls, 1)
        rows.append({"T": T, "tokens_per_s": round(T / (ms / 1e3), 1), "ms": round(ms, 5),
                     "touched_experts": len(touched), "layer_hbm_frac": round(lb / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                     "gate_up_hbm_frac": round(gate_up_bytes(sub, touched) / (gu / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                     "down_hbm_frac": round(down_bytes(sub, touched) / (dn / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                     "stage_ms": {k_: round(v / max(calls, 1), 5) for k_, v in stage_ms.items()}})
    return rows


def traffic_from_profiles(L, kernel):
    """DRAM bytes per launch from a committed ncu summary, if one matches this
    workload and kernel (profiles/traffic.json), else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    # counters taken on another version of the kernel say nothing about this one
    import hashlib
    h = hashlib.sha256()
    for name in ("gemm.cu", "qmoe_internal.cuh"):
        with open(os.path.join(ROOT, "quantized_top_routed_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if d.get("kernel_source_sha256") != h.hexdigest():
        return None
    key = f"{L.name}:T={L.T}:{kernel}"
    v = d.get(key)
    return None if v is None else v.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# the fp64 oracle, timed on the host cores
# ---------------------------------------------------------------------------
def oracle_sample_tokens(L, n, step):
    return np.array([(step * n + i) % L.T for i in range(n)])


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(L, O, args):
    """The fp64 oracle as it stands, single-threaded, on a bounded sample of the
    same batch: whole tokens (routing, dequantisation of their experts, the
    expert FFNs and the combine), one oracle call per token, until about
    --cpu-seconds have passed (at least one token)."""
    from threadpoolctl import threadpool_limits
    n, dt = 0, 0.0
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        while n < args.cpu_tokens and (n == 0 or dt < args.cpu_seconds):
            O.forward(L, tokens=oracle_sample_tokens(L, 1, n))
            n += 1
            dt = time.perf_counter() - t0
    return {"value": round(n / dt, 4), "unit": UNIT, "cores": 1, "host_cores": host_cores(), "nproc": os.cpu_count(),
            "omp_num_threads": os.environ.get("OMP_NUM_THREADS"), "kind": "oracle",
            "sample": f"{n} tokens of the same batch, one oracle call each (routing, dequantisation of the "
                      f"token's experts, the expert FFNs and the combine in float64), one thread, {dt:.1f} s"}


def oracle_task(O, L, step):
    """One sampled task of the workload through the oracle: route token t and run
    the FFN of its slot j (expert-centric task list order), weighted by its gate."""
    t = step % L.T
    j = (step // L.T) % L.k
    r = O.route(L, tokens=[t])
    e = int(r["idx"][0, j])
    w13, w2 = O.dequantize_expert(L.experts[e], L.d, L.I)
    y = O.expert_ffn(O.bf16_to_f64(L.x[t:t + 1]), w13, w2, L.I)
    return r["gates"][0, j] * y


def run_reference(args):
    """--impl reference: the fp64 CPU oracle, as it stands, on the same workload.

    Each step is one sampled task (a token's routing plus one of its k expert
    FFNs), so K steps stay within minutes; throughput is scaled to tokens
    (one task = 1/k token)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle.qmoe_oracle as O
    from threadpoolctl import threadpool_limits
    from quantized_top_routed_b200 import synth
    L = synth.make_layer(args.config, T=args.T, seed=args.seed)
    with threadpool_limits(limits=1):
        for w in range(args.warmup):
            oracle_task(O, L, w)
        times = []
        for s in range(args.steps):
            t0 = time.perf_counter()
            oracle_task(O, L, args.warmup + s)
            times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = (1.0 / L.k) / (ms / 1e3)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, shapes of the workload)",
        "config": {"workload": workload_desc(L), "T": L.T, "sample": "one routed task (1/k token) per step"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": "per step one token's routing and one of its k expert FFNs in float64, "
                                   "single thread; tokens/s = (1/k) / step time"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", default="decode", choices=("tiny", "decode", "prefill", "fine", "mixed"),
                    help="the headline workload (default: decode, T=256)")
    ap.add_argument("--also", nargs="*", default=["prefill", "fine", "mixed"],
                    choices=("tiny", "decode", "prefill", "fine", "mixed"),
                    help="further workloads measured in the same run (one GPU) under 'configs'")
    ap.add_argument("--also-multi", action="store_true", help="measure --also workloads under torchrun too")
    ap.add_argument("--other-steps", type=int, default=30, help="timed steps of each --also workload (at most --steps)")
    ap.add_argument("--T", type=int, default=None, help="tokens per step (default: the workload's)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-sweep", dest="sweep", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=48, help="at most this many tokens in the timed oracle sample")
    ap.add_argument("--cpu-seconds", type=float, default=8.0, help="time budget of the oracle sample per workload")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
