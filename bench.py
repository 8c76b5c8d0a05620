"""Benchmark of the paged-attention hot path on B200.

One step = one pass of the whole path over one synthetic continuous batch:
slot mapping, scatter of the new K/V into the paged cache, attention
(split-KV decode + combine, and the tcgen05 prefill kernel when the batch has
longer queries).  Default workload: the decode-heavy GQA batch (64 sequences,
q_len 1, past U[512, 4096], 32/8 heads, head size 128, block size 16,
20000-block pool); metric: algorithmic HBM bytes of the step per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Multi-GPU (torchrun, one rank per GPU): the path does not shard inside one
batch, so every rank runs its own replica of the workload; times are the max
over ranks and ``value`` counts the bytes of all ranks (weak scaling).

``--impl reference`` times the fp64 CPU oracle on this host's cores over a
bounded sample of the same workload (there is no other implementation of
this path to run).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged attn: decode KV GB/s & prefill TFLOP/s, % of B200 roofline"
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------- work counts

def decode_cutoff(spec: workloads.Spec) -> int:
    """q_len up to which the library takes the split-KV decode path (its rule:
    at most 4 query tokens and at most 32 query rows per KV head)."""
    g = spec.q_heads // spec.kv_heads
    return max(1, min(4, 32 // g))


def algorithmic_counts(spec: workloads.Spec) -> dict:
    """Bytes and FLOPs the method must move / compute for one step.

    attention bytes: every K/V row of a sequence read once per KV head, plus
    Q read and O written; FLOPs: 4 * q_heads * d per visible (query, key)
    pair, causal; scatter bytes: new K/V read and written, slots read.  The
    decode_* and prefill_* entries split the same counts between the
    sequences each kernel serves."""
    T = spec.seqlens_kv.astype(np.int64)
    ql = spec.q_lens.astype(np.int64)
    past = spec.past.astype(np.int64)
    d, kvh, qh = spec.head_size, spec.kv_heads, spec.q_heads
    kv_seq = T * kvh * d * 2 * 2
    q_seq = ql * qh * d * 2
    # sum over i < q_len of (past + i + 1) visible keys
    flops_seq = 4 * qh * d * (ql * past + ql * (ql + 1) // 2)
    dec = (ql > 0) & (ql <= decode_cutoff(spec))
    pre = ql > decode_cutoff(spec)
    scatter_bytes = 4 * spec.token_count * kvh * d * 2 + 4 * spec.token_count
    kv_bytes, q_bytes = int(kv_seq.sum()), int(q_seq.sum())
    return dict(kv_bytes=kv_bytes, q_bytes=q_bytes, o_bytes=q_bytes, flops=int(flops_seq.sum()),
                scatter_bytes=scatter_bytes,
                step_bytes=kv_bytes + 2 * q_bytes + scatter_bytes,
                decode_bytes=int(kv_seq[dec].sum() + q_seq[dec].sum()),
                prefill_flops=int(flops_seq[pre].sum()),
                prefill_bytes=int(kv_seq[pre].sum() + 2 * q_seq[pre].sum()),
                decode=bool(spec.q_lens.max() <= decode_cutoff(spec)))


# Datasheet figures, reported beside the measured ones: HBM3e bandwidth of an
# HGX B200 and its dense 16-bit tensor-core rate.
NOMINAL_HBM_GBS = 7700.0
NOMINAL_TFLOPS = 2250.0


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), tflops=float(p["bf16_tflops"]),
                    tflops_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    return dict(hbm_gbs=6650.0, tflops=1590.0, tflops_sustained=1400.0, source="fallback")


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and throttle reasons sampled through NVML (every ~1 ms) on
    this rank's GPU while the timed region runs (read only: nothing is set)."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, torch_device: int):
        self.dev = torch_device
        self.samples = []
        self.max_mhz = None
        self.stop_flag = threading.Event()
        self.thread = None
        self.err = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            busid = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), bus,
                                          getattr(props, "pci_device_id", 0))
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId(busid.encode())
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        idx = self.dev
        if vis and all(v.strip().isdigit() for v in vis.split(",")):
            idx = int(vis.split(",")[self.dev])
        return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            bits = {k: getattr(pynvml, v, 0) for k, v in self.REASONS.items()}
        except Exception as e:  # NVML unavailable: report it, do not guess
            self.err = f"nvml unavailable: {e}"
            return

        def run():
            while not self.stop_flag.is_set():
                try:
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(mhz), [k for k, b in bits.items() if b and (r & b)]))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.001)
        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self) -> dict:
        self.stop_flag.set()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "samples": 0,
                    "reasons": [self.err or "no samples"]}
        mhz = [m for m, _ in self.samples]
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": self.max_mhz,
                "samples": len(mhz), "reasons": reasons}


# ----------------------------------------------------------------- distributed

def dist_setup(n_gpus: int):
    """(rank, world, local_rank); initialises torch.distributed for N > 1."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = os.environ.get("PA_BENCH_BACKEND", "nccl")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


# ----------------------------------------------------------------- oracle timing

def time_oracle(spec: workloads.Spec, x: dict, target_s: float, seed: int = 0):
    """Run the fp64 oracle over a sample of (sequence, KV head) units of the
    workload for about target_s seconds.  Returns (GB/s, seconds, sample text,
    threads).  Bytes counted are the same algorithmic bytes as the GPU's."""
    import oracle
    rng = np.random.default_rng(seed)
    units = [(b, h) for b in range(spec.batch) for h in range(spec.kv_heads) if spec.q_lens[b] > 0]
    order = rng.permutation(len(units))
    cu = np.concatenate([[0], np.cumsum(spec.q_lens)])
    g = spec.q_heads // spec.kv_heads
    scale = 1.0 / math.sqrt(spec.head_size)
    done_bytes, done_flops, done_units, rows_done = 0, 0, 0, 0
    t0 = time.perf_counter()
    i = 0
    while i < len(order) and time.perf_counter() - t0 < target_s:
        b, h = units[order[i]]
        i += 1
        rows = np.array([(t, h * g + j) for t in range(cu[b], cu[b + 1]) for j in range(g)],
                        dtype=np.int64)
        oracle.attention(x["query"], x["key_cache"], x["value_cache"], x["block_table"],
                         x["cu_seqlens_q"], x["seqlens_kv"], scale, rows=rows)
        T = int(spec.seqlens_kv[b])
        done_bytes += T * spec.head_size * 2 * 2 + 2 * rows.shape[0] * spec.head_size * 2
        q, p = int(spec.q_lens[b]), int(spec.past[b])
        done_flops += 4 * g * spec.head_size * (q * p + q * (q + 1) // 2)
        done_units += 1
        rows_done += rows.shape[0]
    dt = time.perf_counter() - t0
    sample = (f"{done_units} of {len(units)} (sequence, KV head) units, {rows_done} output rows, "
              f"fp64 oracle attention, {dt:.1f} s")
    return dict(gbs=done_bytes / dt / 1e9, tflops=done_flops / dt / 1e12, seconds=dt,
                sample=sample, cores=oracle.max_threads())


# ----------------------------------------------------------------- profiles

_CODE_TOKENS = re.compile(r'"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'|//[^\n]*|/\*.*?\*/', re.S)


def _strip_comments(src: str) -> str:
    """C/C++/CUDA source without its comments (string and character literals
    kept), with blank-line runs and trailing blanks removed."""
    code = _CODE_TOKENS.sub(lambda m: "" if m.group(0).startswith("/") else m.group(0), src)
    lines = [ln.rstrip() for ln in code.splitlines()]
    return "\n".join(ln for ln in lines if ln)


# Sources each profiled kernel is built from: a profile stays tied to them.
KERNEL_SOURCES = {
    "decode_split_kv": ("pa_decode.cu", "pa_common.cuh", "pa_internal.h"),
    "decode_combine": ("pa_decode.cu", "pa_common.cuh", "pa_internal.h"),
    "prefill_tcgen05": ("pa_prefill.cu", "pa_common.cuh", "pa_internal.h"),
    "scatter_kv": ("pa_scatter.cu", "pa_common.cuh", "pa_internal.h"),
    "slot_mapping": ("pa_scatter.cu", "pa_common.cuh", "pa_internal.h"),
    "qkv_rotary_scatter": ("pa_qkv.cu", "pa_common.cuh", "pa_internal.h"),
    "sparse_local_selected": ("pa_sparse.cu", "pa_common.cuh", "pa_internal.h"),
    # head sizes 136 .. 256: the one-tile-per-CTA prefill kernel
    "prefill_tcgen05@d256": ("pa_prefill256.cu", "pa_common.cuh", "pa_internal.h"),
}


def kernel_source_hash(files=None) -> str:
    """Hash of the code of the given kernel sources (default: all of them): a
    profile taken on them stays valid through comment-only edits, and any
    code change invalidates it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "scatter_kv_b200", "csrc")
    for name in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if it was taken
    on the kernel's current sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    key = kernel + "@d256" if workload.endswith("_d256") else kernel
    if not m or not h or h.group(1) != kernel_source_hash(KERNEL_SOURCES.get(key)):
        return None
    return float(m.group(1))


# ----------------------------------------------------------------- main arms

def unit_of(spec: workloads.Spec) -> str:
    """Decode-only batches are judged on bytes moved, the others on FLOPs."""
    return "GB/s" if algorithmic_counts(spec)["decode"] else "TFLOP/s"


def config_of(spec: workloads.Spec, world: int = 1) -> dict:
    return {"workload": spec.name, "batch": spec.batch, "tokens": spec.token_count,
            "q_heads": spec.q_heads, "kv_heads": spec.kv_heads, "head_size": spec.head_size,
            "block_size": spec.block_size, "num_blocks": spec.num_blocks, "seed": spec.seed,
            "l2": "flushed between steps, outside the timed events: 252 MB written, then "
                  "252 MB read so no dirty line is left to write back",
            "parallelism": f"replicas x{world}"}


def run_reference(args, spec, rank, world):
    if rank != 0:
        return
    x = workloads.generate(spec)
    import oracle
    # The new tokens must be in the cache before attention reads them.
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                                spec.block_size)
    oracle.scatter_kv(x["key"], x["value"], slots, x["key_cache"], x["value_cache"])
    unit = unit_of(spec)
    key = "gbs" if unit == "GB/s" else "tflops"
    # Each step is a bounded sample sized so the whole run takes about two minutes.
    per_step = max(0.5, min(15.0, 120.0 / max(1, args.steps + args.warmup)))
    for w in range(args.warmup):
        time_oracle(spec, x, per_step, seed=1000 + w)
    runs = [time_oracle(spec, x, per_step, seed=k) for k in range(args.steps)]
    value = float(np.median([r[key] for r in runs]))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": float(np.mean([r["seconds"] for r in runs])) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(spec, world),
        "cpu_baseline": {"value": value, "unit": unit, "cores": runs[-1]["cores"],
                         "kind": "oracle", "sample": runs[-1]["sample"]},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def kernel_roofline(name: str, avg_ms: float, counts: dict, peaks: dict, workload: str) -> dict:
    """Roofline record of one kernel: algorithmic work of one launch over its
    average launch time, against the measured peak (and the nominal one)."""
    if name == "prefill_tcgen05":
        achieved = counts["prefill_flops"] / (avg_ms * 1e-3) / 1e12
        rec = {"bound": "tensor", "achieved": achieved, "peak": peaks["tflops"], "unit": "TFLOP/s",
               "frac": achieved / peaks["tflops"], "frac_nominal": achieved / NOMINAL_TFLOPS,
               "peak_source": f"{peaks['source']} bf16 burst (fp16 same rate)",
               "work": f"{counts['prefill_flops']} FLOP per launch (causal, prefill sequences)"}
    else:
        alg = counts["scatter_bytes"] if name == "scatter_kv" else counts["decode_bytes"]
        achieved = alg / (avg_ms * 1e-3) / 1e9
        rec = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
               "frac": achieved / peaks["hbm_gbs"], "frac_nominal": achieved / NOMINAL_HBM_GBS,
               "peak_source": f"{peaks['source']} copy bandwidth",
               "work": f"{alg} bytes per launch"}
    rec["traffic"] = profiled_traffic(name, workload)
    rec["kernel"] = name
    rec["kernel_ms"] = avg_ms
    return rec


def measure_workload(args, spec, wl_key, world, dev, steps, e2e=True, cpu=True, int4=False):
    """Time one workload: CUDA-graph replays of the whole step (value),
    traced eager steps (per-kernel times), and optionally the end-to-end step
    through the public API with host buffers.  int4: the same batch over INT4
    caches (random codes, per-channel scales), scatter and attention through
    the INT4 entry points."""
    import torch
    import scatter_kv_b200 as pa

    counts = algorithmic_counts(spec)
    peaks = load_peaks()
    x = workloads.generate(spec)
    if int4:
        rng = np.random.default_rng(spec.seed)
        shape = (spec.num_blocks, spec.block_size, spec.kv_heads, spec.head_size // 2)
        x["key_cache"] = rng.integers(0, 256, size=shape, dtype=np.uint8)
        x["value_cache"] = rng.integers(0, 256, size=shape, dtype=np.uint8)
        x["k_scale"] = rng.uniform(0.1, 0.3, size=(spec.kv_heads, spec.head_size)).astype(np.float32)
        x["v_scale"] = rng.uniform(0.1, 0.3, size=(spec.kv_heads, spec.head_size)).astype(np.float32)
        # A quarter of the K/V bytes, plus every (sequence, KV head)'s scales.
        scale_bytes = 2 * spec.batch * spec.kv_heads * spec.head_size * 4
        counts["kv_bytes"] //= 4
        counts["decode_bytes"] = counts["kv_bytes"] + counts["q_bytes"] + scale_bytes
        counts["scatter_bytes"] = (2 * spec.token_count * spec.kv_heads * spec.head_size * 2
                                   + 2 * spec.token_count * spec.kv_heads * spec.head_size // 2
                                   + 4 * spec.token_count)
        counts["step_bytes"] = (counts["kv_bytes"] + 2 * counts["q_bytes"] + scale_bytes
                                + counts["scatter_bytes"])
    d = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in x.items()}
    dims = pa.make_dims(batch=spec.batch, token_count=spec.token_count, q_heads=spec.q_heads,
                        kv_heads=spec.kv_heads, head_size=spec.head_size,
                        num_blocks=spec.num_blocks, block_size=spec.block_size,
                        max_blocks_per_seq=x["block_table"].shape[1],
                        max_seqlen_q=int(spec.q_lens.max()), max_seqlen_kv=int(spec.seqlens_kv.max()),
                        min_seqlen_q=int(spec.q_lens[spec.q_lens > 0].min()))
    bufs = pa.allocate(dims, device=dev)
    scale = 0.0                     # the library's default, 1 / sqrt(head_size)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    scrub = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    scrub_out = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2(k):
        # Write a buffer twice the L2 size, then read another one of that size:
        # the read evicts the dirty lines the write left, so their write-back
        # to HBM happens here and not inside the next timed step.
        flush.fill_(k)
        torch.sum(scrub, 0, dtype=torch.int64, out=scrub_out)

    def step():
        if int4:
            pa.pa_compute_slot_mapping(d["block_table"], d["cu_seqlens_q"], d["seqlens_kv"],
                                       bufs.slot_mapping, dims, bufs.status, stream)
            pa.pa_scatter_kv_int4(d["key"], d["value"], bufs.slot_mapping, d["k_scale"],
                                  d["v_scale"], d["key_cache"], d["value_cache"], dims, bufs.status,
                                  stream)
            pa.pa_attention_int4(d["query"], d["key_cache"], d["value_cache"], d["k_scale"],
                                 d["v_scale"], d["block_table"], d["cu_seqlens_q"], d["seqlens_kv"],
                                 scale, bufs.out, dims, bufs.workspace, None, bufs.status, stream)
            return
        pa.step(d["query"], d["key"], d["value"], d["key_cache"], d["value_cache"],
                d["block_table"], d["cu_seqlens_q"], d["seqlens_kv"], scale, dims, bufs, stream)

    rec = {}
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
        stream.synchronize()
        status = int(bufs.status[0].item())
        if status != 0:
            raise RuntimeError(f"device status {status:#x} on the {spec.name} inputs")

        # ---- the step as a CUDA graph (launch-bound small kernels replay
        # without host gaps); tracing stays off during capture.
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        graph.replay()
        stream.synchronize()

        # ---- device-timed region: K graph replays, L2 flushed between steps
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        clocks = ClockSampler(dev.index)
        clocks.start()
        barrier(world, dev)
        torch.cuda.synchronize()
        for k in range(steps):
            flush_l2(k)
            ev[k][0].record(stream)
            graph.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        barrier(world, dev)
        rec["clocks"] = clocks.stop()
        ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev)

        # ---- per-kernel durations: K eager steps with the library's event
        # tracing (one event pair around every launch), same flushes.
        pa.pa_trace_read()
        pa.pa_trace_enable(True)
        barrier(world, dev)
        torch.cuda.synchronize()
        for k in range(steps):
            flush_l2(k)
            step()
        torch.cuda.synchronize()
        pa.pa_trace_enable(False)
        trace = pa.pa_trace_read()

        # ---- end-to-end through the public API with host buffers
        ms_e2e, h2d, d2h = None, 0, 0
        if e2e:
            host = {k: torch.from_numpy(np.ascontiguousarray(x[k])).pin_memory()
                    for k in ("query", "key", "value", "block_table", "cu_seqlens_q", "seqlens_kv")}
            out_host = torch.empty(bufs.out.shape, dtype=bufs.out.dtype).pin_memory()
            h2d = sum(t.numel() * t.element_size() for t in host.values())
            d2h = out_host.numel() * out_host.element_size()
            ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
            barrier(world, dev)
            torch.cuda.synchronize()
            for k in range(steps):
                flush_l2(k)
                ev2[k][0].record(stream)
                for name, t in host.items():
                    d[name].copy_(t, non_blocking=True)
                step()
                out_host.copy_(bufs.out, non_blocking=True)
                ev2[k][1].record(stream)
            torch.cuda.synchronize()
            barrier(world, dev)
            ms_e2e = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2), world, dev)

    per_kernel = {}
    for name, t in trace:
        per_kernel.setdefault(name, []).append(t)
    total_k = sum(sum(v) for v in per_kernel.values())
    # The dominant kernel: the prefill kernel whenever the batch has prefill
    # sequences (the library then runs the decode part on a side stream, so
    # the decode launches' traced spans overlap the prefill's and are not
    # their own time), else the kernel with the most traced time.
    if "prefill_tcgen05" in per_kernel and counts["prefill_flops"] > 0:
        dominant = "prefill_tcgen05"
    else:
        dominant = max(per_kernel, key=lambda n: sum(per_kernel[n]))
    roof = kernel_roofline(dominant, float(np.mean(per_kernel[dominant])), counts, peaks, wl_key)
    roof["share_of_kernel_time"] = sum(per_kernel[dominant]) / total_k if total_k else None

    step_s = ms / steps * 1e-3
    unit = unit_of(spec)
    per_sec = (lambda sec: counts["step_bytes"] * world / sec / 1e9) if unit == "GB/s" else \
        (lambda sec: counts["flops"] * world / sec / 1e12)
    # The step's own roofline: the slower of its FLOPs at the tensor peak and
    # its bytes (attention K/V + Q + O, and the scatter's) at HBM bandwidth.
    flop_us = counts["flops"] / (peaks["tflops"] * 1e12) * 1e6
    byte_us = counts["step_bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6
    rec.update({
        "value": per_sec(step_s), "unit": unit, "ms_per_step": ms / steps,
        "tokens_per_s": spec.token_count * world / step_s,
        "roofline": roof,
        "step_roofline": {"flop_us": flop_us, "byte_us": byte_us,
                          "bound": "tensor" if flop_us > byte_us else "hbm",
                          "frac": max(flop_us, byte_us) / (step_s * 1e6),
                          "frac_nominal": max(counts["flops"] / (NOMINAL_TFLOPS * 1e12),
                                              counts["step_bytes"] / (NOMINAL_HBM_GBS * 1e9))
                          / step_s},
        "gpu_launches": sum(len(v) for v in per_kernel.values()),
        "kernels": {n: {"launches": len(v), "avg_ms": float(np.mean(v))}
                    for n, v in per_kernel.items()},
        "algorithmic": {k: v for k, v in counts.items() if k != "decode"},
        "config": config_of(spec, world),
    })
    if e2e:
        rec["e2e"] = {"value": per_sec(ms_e2e / steps * 1e-3), "unit": unit,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if int4:
        rec["config"]["kv_cache"] = "INT4, two codes per byte, fp32 per-channel scales"
        e2e = False
    if cpu and world == 1 and not args.no_cpu_baseline and not int4:
        r = time_oracle(spec, x_with_scatter(x, spec), args.cpu_seconds)
        rec["cpu_baseline"] = {"value": r["gbs"] if unit == "GB/s" else r["tflops"], "unit": unit,
                               "cores": r["cores"], "kind": "oracle", "sample": r["sample"]}
    del d, bufs, flush, scrub, graph
    torch.cuda.empty_cache()
    return rec


def measure_qkv_rotary(args, spec, world, dev, steps):
    """The fused split-QKV + rotary + scatter pass over one batch of new
    tokens (packed QKV of the workload's shape, rotary on all head_size
    dimensions, split pairing), timed alone: CUDA-graph replays, L2 flushed
    between them.  HBM-bound: its algorithmic bytes are the packed QKV read,
    Q written, K and V written into the cache, the cos/sin rows read and the
    slots written."""
    import torch
    import scatter_kv_b200 as pa

    x = workloads.generate(spec)
    T, qh, kvh, d = spec.token_count, spec.q_heads, spec.kv_heads, spec.head_size
    rng = np.random.default_rng(spec.seed)
    qkv = torch.from_numpy(rng.standard_normal((T, qh + 2 * kvh, d), dtype=np.float32)
                           .astype(np.float16)).to(dev)
    maxpos = int(spec.seqlens_kv.max())
    ang = np.arange(maxpos)[:, None] * (10000.0 ** (-2.0 * np.arange(d // 2) / d))[None, :]
    cos = torch.from_numpy(np.cos(ang).astype(np.float16)).to(dev)
    sin = torch.from_numpy(np.sin(ang).astype(np.float16)).to(dev)
    meta = {k: torch.from_numpy(np.ascontiguousarray(x[k])).to(dev)
            for k in ("block_table", "cu_seqlens_q", "seqlens_kv", "key_cache", "value_cache")}
    dims = pa.make_dims(batch=spec.batch, token_count=T, q_heads=qh, kv_heads=kvh, head_size=d,
                        num_blocks=spec.num_blocks, block_size=spec.block_size,
                        max_blocks_per_seq=x["block_table"].shape[1])
    rot = pa.pa_rotary()
    rot.rotary_dim, rot.interleaved, rot.max_position = d, 0, maxpos
    q_out = torch.empty((T, qh, d), dtype=torch.float16, device=dev)
    slots = torch.empty(T, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    qp, kp, vp, stride = pa.packed_qkv_views(qkv, dims)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    scrub = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    scrub_out = torch.empty((), dtype=torch.int64, device=dev)

    def call():
        pa.pa_split_qkv_rotary_scatter(qp, kp, vp, stride, stride, cos, sin, rot,
                                       meta["block_table"], meta["cu_seqlens_q"],
                                       meta["seqlens_kv"], q_out, meta["key_cache"],
                                       meta["value_cache"], slots, dims, status, stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
        stream.synchronize()
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item()):#x} in the fused QKV pass")
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            call()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        barrier(world, dev)
        torch.cuda.synchronize()
        for k in range(steps):
            flush.fill_(k)
            torch.sum(scrub, 0, dtype=torch.int64, out=scrub_out)
            ev[k][0].record(stream)
            graph.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        barrier(world, dev)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev) / steps
    nbytes = (T * (qh + 2 * kvh) * d * 2 + T * qh * d * 2 + 2 * T * kvh * d * 2 + T * d * 2
              + 4 * T)
    gbs = nbytes / (ms * 1e-3) / 1e9
    peaks = load_peaks()
    return {"workload": spec.name + ", packed QKV, rotary_dim = head_size, split pairing",
            "us": ms * 1e3, "bytes": nbytes, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"],
            "frac_nominal": gbs / NOMINAL_HBM_GBS, "peak_source": f"{peaks['source']} copy bandwidth",
            "traffic": profiled_traffic("qkv_rotary_scatter", "prefill"),
            "timing": "CUDA-graph replays of the one call, L2 flushed between them"}


def measure_sparse(args, spec, world, dev, steps, num_selected=1024, window=128):
    """Sparse paged attention (local window + selected positions) on the
    decode-heavy batch: every (token, KV head) selects num_selected sorted
    positions below its window.  HBM-bound: its algorithmic bytes are the
    K/V rows of every selected and window key, read once per KV head, plus
    Q read and O written.  Timed alone: CUDA-graph replays, L2 flushed."""
    import torch
    import scatter_kv_b200 as pa

    x = workloads.generate(spec)
    rng = np.random.default_rng(spec.seed)
    T, kvh, d = spec.token_count, spec.kv_heads, spec.head_size
    cu = x["cu_seqlens_q"]
    sel = np.full((T, kvh, num_selected), -1, np.int32)
    nkeys = 0
    for b in range(spec.batch):
        for t in range(int(cu[b]), int(cu[b + 1])):
            P = int(spec.past[b]) + t - int(cu[b])
            lo = max(0, P - window)
            for h in range(kvh):
                k = min(num_selected, lo)
                sel[t, h, :k] = np.sort(rng.choice(lo, size=k, replace=False)) if k else []
                nkeys += k + (P - lo + 1)
    dd = {k: torch.from_numpy(np.ascontiguousarray(x[k])).to(dev)
          for k in ("query", "key_cache", "value_cache", "block_table", "cu_seqlens_q", "seqlens_kv")}
    seld = torch.from_numpy(sel).to(dev)
    dims = pa.make_dims(batch=spec.batch, token_count=T, q_heads=spec.q_heads, kv_heads=kvh,
                        head_size=d, num_blocks=spec.num_blocks, block_size=spec.block_size,
                        max_blocks_per_seq=x["block_table"].shape[1])
    out = torch.empty((T, spec.q_heads, d), dtype=torch.float16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    scrub = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    scrub_out = torch.empty((), dtype=torch.int64, device=dev)

    def call():
        pa.pa_sparse_attention(dd["query"], dd["key_cache"], dd["value_cache"], dd["block_table"],
                               dd["cu_seqlens_q"], dd["seqlens_kv"], seld, num_selected, window,
                               0.0, out, dims, status, stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
        stream.synchronize()
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item()):#x} in sparse attention")
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            call()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        barrier(world, dev)
        torch.cuda.synchronize()
        for k in range(steps):
            flush.fill_(k)
            torch.sum(scrub, 0, dtype=torch.int64, out=scrub_out)
            ev[k][0].record(stream)
            graph.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        barrier(world, dev)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev) / steps
    nbytes = nkeys * d * 2 * 2 + 2 * T * spec.q_heads * d * 2
    gbs = nbytes / (ms * 1e-3) / 1e9
    peaks = load_peaks()
    return {"workload": f"{spec.name}, {num_selected} selected positions + window {window} "
                        "per (token, KV head)",
            "us": ms * 1e3, "bytes": nbytes, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"],
            "frac_nominal": gbs / NOMINAL_HBM_GBS, "peak_source": f"{peaks['source']} copy bandwidth",
            "traffic": profiled_traffic("sparse_local_selected", "decode"),
            "timing": "CUDA-graph replays of the one call, L2 flushed between them"}


def run_gpu(args, spec, rank, world, local):
    import torch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.only and args.part != "step":
        # One other part alone (for profiling): its record as the line.
        if args.part == "int4":
            rec = measure_workload(args, spec, args.workload + "_int4", world, dev, args.steps,
                                   e2e=False, int4=True)
        elif args.part == "sparse":
            rec = measure_sparse(args, spec, world, dev, args.steps)
        elif args.part == "d256":
            rec = measure_workload(args, workloads.spec_prefill_mha_d256(), "prefill_d256", world,
                                   dev, args.steps, e2e=False, cpu=False)
        else:
            rec = measure_qkv_rotary(args, spec, world, dev, args.steps)
        if rank == 0:
            print(json.dumps({"part": args.part, **rec}), flush=True)
        return rec
    main = measure_workload(args, spec, args.workload, world, dev, args.steps)
    # The other full-size workloads, measured in the same process and reported
    # in the same line (each with its own clocks, roofline and CPU baseline).
    others = {}
    if not args.only:
        for key in ("prefill", "mixed", "long_decode", "decode"):
            if key == args.workload:
                continue
            o = workloads.CONFIGS[workloads.CONFIG_KEYS[key]]()
            others[key] = measure_workload(args, o, key, world, dev, max(10, args.steps // 2),
                                           e2e=True)
        others["long_decode_int4"] = measure_workload(
            args, workloads.CONFIGS[workloads.CONFIG_KEYS["long_decode"]](), "long_decode_int4",
            world, dev, max(10, args.steps // 2), e2e=False, int4=True)
        others["sparse_local_selected"] = measure_sparse(
            args, workloads.CONFIGS[workloads.CONFIG_KEYS["decode"]](), world, dev,
            max(10, args.steps // 2))
        others["prefill_d256"] = measure_workload(args, workloads.spec_prefill_mha_d256(),
                                                  "prefill_d256", world, dev,
                                                  max(10, args.steps // 2), e2e=True)
        others["fused_split_qkv_rotary_scatter"] = measure_qkv_rotary(
            args, workloads.CONFIGS[workloads.CONFIG_KEYS["prefill"]](), world, dev,
            max(10, args.steps // 2))
    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": main["value"], "unit": main["unit"], "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic", "config": main["config"], "roofline": main["roofline"],
        "step_roofline": main["step_roofline"], "cpu_baseline": main.get("cpu_baseline"),
        "e2e": main["e2e"], "gpu_launches": main["gpu_launches"],
        "timing": "value: CUDA-graph replays of the step; kernels: eager traced steps",
        "kernels": main["kernels"], "algorithmic": main["algorithmic"],
        "tokens_per_s": main["tokens_per_s"], "clocks": main["clocks"],
        "workloads": others,
    }
    print(json.dumps(line), flush=True)
    return line


def x_with_scatter(x, spec):
    """The workload as the oracle sees it after the step's scatter."""
    import oracle
    y = dict(x)
    y["key_cache"] = x["key_cache"].copy()
    y["value_cache"] = x["value_cache"].copy()
    slots = oracle.slot_mapping(x["block_table"], x["cu_seqlens_q"], x["seqlens_kv"],
                                spec.block_size)
    oracle.scatter_kv(x["key"], x["value"], slots, y["key_cache"], y["value_cache"])
    return y


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=sorted(workloads.CONFIG_KEYS))
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true",
                    help="measure only --workload (default: every full-size workload)")
    ap.add_argument("--part", default="step", choices=["step", "int4", "sparse", "qkv_rotary", "d256"],
                    help="with --only: the part to measure on --workload's batch (step: the "
                         "whole step; int4: INT4-cache scatter + decode; sparse: sparse "
                         "attention; qkv_rotary: the fused split-QKV pass; d256: causal "
                         "prefill at head size 256)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    spec = workloads.CONFIGS[workloads.CONFIG_KEYS[args.workload]]()
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, spec, rank, world)
        else:
            run_gpu(args, spec, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
