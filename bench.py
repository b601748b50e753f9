"""Benchmark of the paged decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the paged cache write
of this step's new K/V (one token per sequence) followed by decode attention of
every sequence over its paged cache.  The default workload is the LLaMA-2-7B
layer shape (64 sequences x 2048 tokens, 32 heads MHA, head_dim 128, fp16,
blocks shuffled across a 12288-block pool).  The KV read of one step (2 GiB) is
larger than the 126 MB L2, so no flush is needed between steps.

Prints ONE JSON line (rank 0).  `value` is whole-job achieved HBM GB/s: decode
bytes (sum_s len_s * Hkv * D * 2 * kv_bytes + q + out) of every rank's step
divided by the max-over-ranks device time of a step.  Multi-GPU runs are
independent replicas (the path has no exchange step).  `--impl reference`
times the fp64 CPU oracle on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_463_b200 import binding as pab  # noqa: E402
from paged_kv_cache_463_b200 import workloads as wl  # noqa: E402

METRIC = "paged decode: achieved HBM GB/s (% of B200 peak) and seq-steps/sec"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
DEFAULT_WORKLOAD = "llama2-7b-mha"


# ---------------------------------------------------------------- helpers
def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_peak():
    """Dense bf16 tensor peak in TFLOP/s: the driver's cuBLAS burst
    measurement, else the profiling recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured cuBLAS bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback 1590 TFLOP/s (no MEASURED_PEAKS.json)"


def traffic_record(kernel_name: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for f in ("decode.cuh", "ptx.cuh", "paged_attn.cu"):
        with open(os.path.join(ROOT, "paged_kv_cache_463_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    for line in open(path, encoding="utf-8"):
        parts = line.split()
        if len(parts) >= 4 and parts[0] == kernel_name and parts[1] == workload and parts[2] == digest:
            return float(parts[3])
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML (the library behind
    nvidia-smi) every ~2 ms on a background thread while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self.error = None

    def _run(self):
        import pynvml
        h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        while not self._stop.is_set():
            try:
                mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                reasons = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((mhz, reasons))
            except Exception as e:  # keep timing even if a query fails
                self.error = str(e)
            self._stop.wait(0.002)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                ids = [x for x in vis.split(",") if x.strip()]
                if self.gpu < len(ids) and ids[self.gpu].strip().isdigit():
                    self.gpu = int(ids[self.gpu])
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:
            self.error = str(e)
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples: " + str(self.error)]}
        active = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": active, "samples": len(self.samples), "source": "NVML, 2 ms period"}


def dist_setup():
    """One process per GPU (torchrun env); NCCL when there are GPUs, gloo on a
    host without one (the multi-process plumbing is tested that way)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device(f"cuda:{local}"))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (device time is taken as the max over ranks)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- CPU oracle leg
def oracle_sample(spec: wl.WorkloadSpec, budget_s: float, max_seqs: int | None = None):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload:
    the first k sequences of a seeded copy of the workload restricted to them.
    Returns (GB/s under the decode byte formula, seq-steps/s, description, threads)."""
    import numpy as np
    from oracle import attention, cache_write  # the oracle: test infrastructure, CPU baseline only
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    k_total, t_total, bytes_total, seqs_done = 0, 0.0, 0, 0
    k = 1
    while True:
        sub = wl.scaled(spec, num_seqs=k, pool_blocks=None,
                        prefix_groups=min(spec.prefix_groups, 1) if spec.prefix_groups else 0)
        w = wl.make_workload(sub, "cpu")
        raw = _raw_numpy(w)
        t0 = time.perf_counter()
        kc, vc = raw["kc"].copy(), raw["vc"].copy()
        cache_write.reshape_and_cache(raw["nk"], raw["nv"], kc, vc, raw["slots"], src_dtype=sub.q_dtype,
                                      cache_dtype=sub.kv_dtype, k_scale=w.k_scale, v_scale=w.v_scale)
        attention.decode_attention(raw["q"], kc, vc, raw["bt"], raw["lens"], w.scale, q_dtype=sub.q_dtype,
                                   kv_dtype=sub.kv_dtype, k_scale=w.k_scale, v_scale=w.v_scale)
        dt = time.perf_counter() - t0
        t_total += dt
        bytes_total += wl.decode_bytes(w)
        seqs_done += k
        k_total += 1
        if t_total >= budget_s or (max_seqs is not None and seqs_done >= max_seqs):
            break
        k = min(2 * k, spec.num_seqs)
    desc = (f"{seqs_done} sequences of {spec.name} ({k_total} oracle call(s); per sequence all "
            f"{spec.num_heads} heads over its full length), cache write + fp64 decode attention")
    return bytes_total / t_total / 1e9, seqs_done / t_total, desc, threads, t_total


def _raw_numpy(w):
    import numpy as np
    def r(t):
        t = t.cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.float8_e4m3fn:
            return t.view(torch.uint8).numpy()
        return t.numpy()
    d = {"q": r(w.query), "nk": r(w.new_key), "nv": r(w.new_value), "slots": r(w.slot_mapping),
         "bt": r(w.block_tables), "lens": r(w.seq_lens)}
    if w.spec.kv_dtype == "fp8_e4m3":
        from oracle import cache_write
        d["kc"] = cache_write.quantize(r(w.key_src), w.spec.q_dtype, w.k_scale)
        d["vc"] = cache_write.quantize(r(w.value_src), w.spec.q_dtype, w.v_scale)
    else:
        d["kc"], d["vc"] = r(w.key_cache), r(w.value_cache)
    return d


# ---------------------------------------------------------------- arms
def run_reference(args, world, rank):
    if rank != 0:
        return 0
    spec = wl.SPEC_BY_NAME[args.workload]
    per_step_budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals, rates = [], []
    desc, threads, elapsed = "", 1, 0.0
    for i in range(args.warmup + args.steps):
        gbs, sps, desc, threads, el = oracle_sample(spec, per_step_budget, max_seqs=2)
        if i >= args.warmup:
            vals.append(gbs)
            rates.append(sps)
            elapsed += el
    value = statistics.median(vals)
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": spec.name, "description": spec.description},
            "seq_steps_per_s": statistics.median(rates),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


class DecodeBench:
    """One workload on one GPU: its seeded inputs in HBM, a library context,
    and CUDA graphs of one whole step (cache write + decode call) and of the
    decode call alone."""

    def __init__(self, spec: wl.WorkloadSpec, args, local: int, shared_opt: str = "auto"):
        self.spec, self.args, self.local = spec, args, local
        self.dev = dev = f"cuda:{local}"
        self.w = w = wl.make_workload(spec, dev)
        part = {"auto": pab.PA_PARTITION_AUTO, "none": pab.PA_PARTITION_NONE}.get(args.partition)
        part = int(args.partition) if part is None else part
        self.shared = shared = w.group_start is not None and shared_opt != "off"
        if shared_opt == "on" and not shared:
            raise SystemExit(f"workload {spec.name} has no shared-prefix groups")
        self.pa = pa = pab.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks,
                                          block_size=spec.block_size, q_dtype=spec.q_dtype, kv_dtype=spec.kv_dtype,
                                          max_num_seqs=spec.num_seqs, max_blocks_per_seq=w.block_tables.shape[1],
                                          partition_tokens=part, device=local, shared_prefix=shared)
        if spec.kv_dtype == "fp8_e4m3":  # the pool quantised once by the library's own cache write
            NB, bs, Hkv, D = w.key_src.shape
            self.kc = torch.empty((NB, bs, Hkv, D), dtype=torch.float8_e4m3fn, device=dev)
            self.vc = torch.empty_like(self.kc)
            pa.reshape_and_cache(w.key_src.view(-1, Hkv, D), w.value_src.view(-1, Hkv, D), self.kc, self.vc,
                                 torch.arange(NB * bs, dtype=torch.int64, device=dev), w.k_scale, w.v_scale)
            w.key_src = w.value_src = None
        else:
            self.kc, self.vc = w.key_cache, w.value_cache
        self.out = torch.empty_like(w.query)
        self.stream = torch.cuda.current_stream()
        self.max_len = w.max_seq_len
        self.chosen_part = pa.get_partition_tokens()
        # cache write + decode, + the merge kernel (auto partitioning or a split),
        # + the prefix pass (shared-prefix decode)
        self.launches_per_step = 2 + (1 if (self.chosen_part < 0 or shared or 0 < self.chosen_part < self.max_len)
                                      else 0) + (1 if shared else 0)
        if shared:
            gsizes = (w.group_start[1:] - w.group_start[:-1]).cpu()
            self.max_group = int(gsizes.max().item())
            self.max_prefix = int(w.group_prefix_len.max().item())
        self.dec_bytes = wl.decode_bytes(w)
        # bytes the call must move: with shared prefixes, each group's prefix once
        self.alg_bytes = wl.shared_decode_bytes(w) if shared else self.dec_bytes
        self.g_step = self.g_dec = None

    def attend(self, q, bt, lens, o=None, st=None):
        w, pa = self.w, self.pa
        o = self.out if o is None else o
        st = self.stream if st is None else st
        if self.shared:
            pa.paged_attention_decode_shared_prefix(o, q, self.kc, self.vc, bt, lens, self.max_len, w.group_start,
                                                    w.group_prefix_len, self.max_group, self.max_prefix, w.scale,
                                                    w.k_scale, w.v_scale, st)
        else:
            pa.paged_attention_decode(o, q, self.kc, self.vc, bt, lens, self.max_len, w.scale, w.k_scale,
                                      w.v_scale, st)

    def write(self, k, v, slots, st=None):
        w = self.w
        self.pa.reshape_and_cache(k, v, self.kc, self.vc, slots, w.k_scale, w.v_scale,
                                  self.stream if st is None else st)

    def step(self):
        w = self.w
        self.write(w.new_key, w.new_value, w.slot_mapping)
        self.attend(w.query, w.block_tables, w.seq_lens)

    def warm_and_capture(self, warmup: int, graph: bool):
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        if self.pa.get_error() != 0:
            raise SystemExit("device check fired during warm-up")
        if graph:
            w = self.w
            side = torch.cuda.Stream(device=self.dev)
            side.wait_stream(self.stream)
            self.g_step, self.g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_step, stream=side):
                self.write(w.new_key, w.new_value, w.slot_mapping, side)
                self.attend(w.query, w.block_tables, w.seq_lens, self.out, side)
            with torch.cuda.graph(self.g_dec, stream=side):
                self.attend(w.query, w.block_tables, w.seq_lens, self.out, side)
            self.stream.wait_stream(side)
            for _ in range(warmup):
                self.g_step.replay()
            torch.cuda.synchronize()

    def timed_steps(self, steps: int, world: int):
        """K whole steps between a barrier + synchronize on each side; returns
        (total ms max over ranks, per-step cache-write ms list or None, decode ms list or None, clocks)."""
        w, st = self.w, self.stream
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(self.local) as clk:
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(st)
            for i in range(steps):
                if self.g_step is not None:
                    self.g_step.replay()
                    continue
                a, m, e = ev[i]
                a.record(st)
                self.write(w.new_key, w.new_value, w.slot_mapping)
                m.record(st)
                self.attend(w.query, w.block_tables, w.seq_lens)
                e.record(st)
            t1.record(st)
            torch.cuda.synchronize()
        barrier(world)
        total = max_over_ranks(t0.elapsed_time(t1), world)
        if self.pa.get_error() != 0:
            raise SystemExit("device check fired during the timed region")
        if self.g_step is None:
            return total, [a.elapsed_time(m) for a, m, _ in ev], [m.elapsed_time(e) for _, m, e in ev], clk.summary()
        return total, None, None, clk.summary()

    def decode_loop(self, min_seconds: float):
        """The decode call alone (its graph, or direct launches), replayed back
        to back for at least ``min_seconds``; CUDA events on the launching
        stream around the whole loop, NVML clocks sampled during it.
        Returns (ms per call, calls, clocks)."""
        st = self.stream
        w = self.w

        def once():
            if self.g_dec is not None:
                self.g_dec.replay()
            else:
                self.attend(w.query, w.block_tables, w.seq_lens)

        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(10):
            once()
        e1.record(st)
        torch.cuda.synchronize()
        est = max(1e-3, e0.elapsed_time(e1) / 10)
        n = int(min(200000, max(50, math.ceil(min_seconds * 1e3 / est))))
        with ClockSampler(self.local) as clk:
            e0.record(st)
            for _ in range(n):
                once()
            e1.record(st)
            torch.cuda.synchronize()
        if self.pa.get_error() != 0:
            raise SystemExit("device check fired during the decode loop")
        return e0.elapsed_time(e1) / n, n, clk.summary()

    def end_to_end(self, steps: int, warmup: int, world: int):
        """The same step through the public API from pinned host buffers:
        every step uploads its inputs (new K/V, query, slot mapping, block
        tables, lengths) and reads its output back.  Uploads run on one copy
        stream and read-backs on another (the two directions of the host link
        in parallel), into double-buffered device tensors, so step i+1's
        upload and step i-1's read-back overlap step i's kernels, as in a
        serving loop.  Returns (ms per step max over ranks, h2d bytes, d2h bytes)."""
        w, st, dev = self.w, self.stream, self.dev
        names = ("new_key", "new_value", "query", "slot_mapping", "block_tables", "seq_lens")
        host = {k: getattr(w, k).cpu().pin_memory() for k in names}
        dev_in = [{k: torch.empty_like(getattr(w, k)) for k in host} for _ in range(2)]
        outs = [torch.empty_like(self.out) for _ in range(2)]
        out_host = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = out_host[0].numel() * out_host[0].element_size()
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_read = [torch.cuda.Event() for _ in range(2)]
        for e in ev_done + ev_read:
            e.record(st)

        def upload(i):
            b = i % 2
            up.wait_event(ev_done[b])  # step i - 2's kernels are done with these inputs
            with torch.cuda.stream(up):
                for k, t in host.items():
                    dev_in[b][k].copy_(t, non_blocking=True)
            ev_in[b].record(up)

        def compute_and_read_back(i):
            b = i % 2
            st.wait_event(ev_in[b])
            st.wait_event(ev_read[b])  # step i - 2's output has been read back
            d = dev_in[b]
            self.write(d["new_key"], d["new_value"], d["slot_mapping"])
            self.attend(d["query"], d["block_tables"], d["seq_lens"], outs[b])
            ev_done[b].record(st)
            down.wait_event(ev_done[b])
            with torch.cuda.stream(down):
                out_host[b].copy_(outs[b], non_blocking=True)
            ev_read[b].record(down)

        def run(n):
            upload(0)
            for i in range(n):
                if i + 1 < n:
                    upload(i + 1)
                compute_and_read_back(i)
            tail = torch.cuda.Event()
            tail.record(down)
            st.wait_event(tail)  # the last read-back is inside the timed region

        run(warmup)
        barrier(world)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(st)
        run(steps)
        s1.record(st)
        torch.cuda.synchronize()
        ms = max_over_ranks(s0.elapsed_time(s1), world)
        if self.pa.get_error() != 0:
            raise SystemExit("device check fired during the end-to-end steps")
        return ms / steps, h2d, d2h

    def close(self):
        self.g_step = self.g_dec = None
        self.pa.close()


def _workload_config(b: DecodeBench, graph: bool, world: int) -> dict:
    spec, w = b.spec, b.w
    return {"workload": spec.name, "description": spec.description, "num_seqs": spec.num_seqs,
            "num_heads": spec.num_heads, "num_kv_heads": spec.num_kv_heads, "head_dim": spec.head_dim,
            "block_size": spec.block_size, "kv_dtype": spec.kv_dtype, "q_dtype": spec.q_dtype,
            "sum_seq_len": int(w.seq_lens.sum().item()),
            "partition_tokens": "auto (chosen by the decode kernel from the lengths)" if b.chosen_part < 0
            else b.chosen_part,
            "l2": "inputs larger than L2 (KV read per step >> 126 MB), no flush",
            "shared_prefix": bool(b.shared),
            "launch": "one CUDA graph replay per step" if graph else "eager launches",
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}


def _roofline(b: DecodeBench, dec_ms: float, peak: float, peak_kind: str, traffic):
    achieved = b.alg_bytes / (dec_ms * 1e-3) / 1e9
    r = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
         "traffic": traffic,
         "kernel": ("paged_prefix_kernel + paged_decode_kernel + merge (the whole call)" if b.shared
                    else "paged_decode_kernel"),
         "algorithmic_bytes": b.alg_bytes,
         "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
         if peak_kind == "measured" else "fallback 6.65 TB/s"}
    if traffic is not None:
        r["traffic_note"] = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of the decode kernel on the "
                             "16-sequence case of this workload, scaled x4 to the 64-sequence launch")
    return r


def workload_entry(spec: wl.WorkloadSpec, args, local: int, shared_opt: str, peak: float, peak_kind: str) -> dict:
    """Device-timed decode call (>= 1 s of back-to-back graph replays), the
    whole step and the end-to-end step of one more workload (1 GPU)."""
    b = DecodeBench(spec, args, local, shared_opt)
    try:
        b.warm_and_capture(args.warmup, args.graph)
        total_ms, _, _, _ = b.timed_steps(args.steps, 1)
        dec_ms, calls, clocks = b.decode_loop(args.decode_seconds)
        e2e_ms, h2d, d2h = b.end_to_end(args.steps, args.warmup, 1)
        S = spec.num_seqs
        gbs = b.dec_bytes / (dec_ms * 1e-3) / 1e9
        e = {"workload": spec.name, "config": _workload_config(b, args.graph, 1),
             "decode_ms": dec_ms, "decode_calls_timed": calls,
             "gbs": gbs, "unit": "GB/s (the metric's byte formula: every sequence's whole length)",
             "pct_of_nominal_8tbs": 100.0 * gbs / NOMINAL_HBM_GBS, "pct_of_measured_copy": 100.0 * gbs / peak,
             "seq_steps_per_s": S / (dec_ms * 1e-3), "bytes_per_call": b.dec_bytes,
             "step_ms": total_ms / args.steps, "step_gbs": b.dec_bytes / (total_ms / args.steps * 1e-3) / 1e9,
             "roofline": _roofline(b, dec_ms, peak, peak_kind, None),
             "e2e": {"gbs": b.dec_bytes / (e2e_ms * 1e-3) / 1e9, "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h},
             "gpu_launches_per_step": b.launches_per_step, "clocks": clocks}
        if spec.prefix_groups:
            e["unique_bytes_per_call"] = b.alg_bytes
            e["unique_gbs"] = b.alg_bytes / (dec_ms * 1e-3) / 1e9
            e["unique_note"] = ("bytes the call must read: each group's shared prefix once plus every private "
                                "suffix, q and out")
        return e
    finally:
        b.close()


# The bench line's extra workloads: the other full-size configurations of the
# hot path, each timed on the same GPU after the headline one.
EXTRA_WORKLOADS = [("gqa-70b-like", "auto"), ("long-context-split-kv", "auto"), ("shared-prefix-fp8", "off"),
                   ("shared-prefix-fp8", "on")]


def run_ours(args, world, rank, local):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the product path has no CPU fallback)")
    from paged_kv_cache_463_b200 import build
    build.build()
    spec = wl.SPEC_BY_NAME[args.workload]
    if args.num_seqs:
        spec = wl.scaled(spec, num_seqs=args.num_seqs, pool_blocks=None,
                         prefix_groups=min(spec.prefix_groups, args.num_seqs) if spec.prefix_groups else 0)
    peak, peak_kind = measured_hbm_peak()
    b = DecodeBench(spec, args, local, args.shared_prefix)
    b.warm_and_capture(args.warmup, args.graph)
    # ---- device-timed region: K whole steps (each one graph replay of the
    # cache write + decode call, or direct launches with --eager)
    total_ms, write_ms, decode_ms, clocks = b.timed_steps(args.steps, world)
    # ---- the decode call alone, >= decode_seconds of back-to-back replays
    dec_ms, calls, dec_clocks = b.decode_loop(args.decode_seconds)
    dec_ms = max_over_ranks(dec_ms, world)
    if decode_ms is not None:  # eager: the calls inside the timed steps are timed one by one too
        write_ms = sum(write_ms) / len(write_ms)
    else:
        write_ms = max(0.0, total_ms / args.steps - dec_ms)
    # ---- end to end through the public API, host buffers every step
    e2e_step_ms, h2d, d2h = b.end_to_end(args.steps, args.warmup, world)

    S = spec.num_seqs
    ms_per_step = total_ms / args.steps
    value = world * b.dec_bytes * args.steps / (total_ms * 1e-3) / 1e9
    seq_steps = world * S * args.steps / (total_ms * 1e-3)
    e2e_value = world * b.dec_bytes / (e2e_step_ms * 1e-3) / 1e9
    traffic = None if b.shared else traffic_record("paged_decode_kernel", spec.name)
    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"f16": "f16", "bf16": "bf16", "fp8_e4m3": "fp8_e4m3"}[spec.kv_dtype],
        "data": "synthetic",
        "config": _workload_config(b, args.graph, world),
        "seq_steps_per_s": seq_steps,
        "pct_of_nominal_8tbs": 100.0 * value / world / NOMINAL_HBM_GBS,
        "pct_of_measured_copy": 100.0 * value / world / peak,
        "bytes_per_step": b.dec_bytes,
        "bytes_note": ("value counts every sequence's prefix (the metric's byte formula); the roofline counts "
                       "each group's shared prefix once (the bytes the call must read)") if b.shared else None,
        "decode_ms": dec_ms, "decode_calls_timed": calls,
        "decode_timing": (f"{calls} back-to-back replays of the decode call's CUDA graph" if args.graph
                          else f"{calls} back-to-back direct decode calls") +
                         ", CUDA events on the launching stream around the loop; NVML clocks in decode_clocks",
        "decode_clocks": dec_clocks,
        "cache_write_ms": write_ms,
        "roofline": _roofline(b, dec_ms, peak, peak_kind, traffic),
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_step_ms,
                "how": "pinned host inputs -> device (upload stream, double-buffered) -> cache write + decode -> "
                       "output -> pinned host (read-back stream), every step; uploads and read-backs overlap "
                       "the neighbouring steps' kernels"},
        "gpu_launches": b.launches_per_step * args.steps,
        "clocks": clocks,
    }
    b.close()
    del b
    torch.cuda.empty_cache()
    if world == 1 and args.workload == DEFAULT_WORKLOAD and not args.num_seqs and not args.no_extra:
        per = []
        for name, sp_opt in EXTRA_WORKLOADS:
            per.append(workload_entry(wl.SPEC_BY_NAME[name], args, local, sp_opt, peak, peak_kind))
            torch.cuda.empty_cache()
        result["per_workload"] = per
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, sps, desc, threads, el = oracle_sample(spec, args.cpu_budget)
        result["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                  "sample": desc, "seq_steps_per_s": sps, "seconds": el}
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                g1, s1, d1, _, e1 = oracle_sample(spec, args.cpu_budget / 2)
            result["cpu_baseline"]["one_core"] = {"value": g1, "unit": "GB/s", "cores": 1, "sample": d1,
                                                  "seq_steps_per_s": s1, "seconds": e1}
            result["cpu_baseline"]["cores_note"] = (
                f"cores = the BLAS thread pool the oracle ran with; its per-(sequence, head) matrix-vector "
                f"products are too small to spread over it, so the pool run is {gbs / g1:.2f}x the one-thread "
                f"run (effective parallelism about 1)")
        except ImportError:
            pass
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def run_copy_blocks(args, world, rank, local):
    """Block copies (copy-on-write / swap) on the 7B layer's block shape
    (16 tokens x 32 heads x 128 dims fp16 = 128 KiB per tensor): device ->
    device pairs, then a swap out to pinned host memory and back in.  GB/s
    count bytes read + written on the device side (2 x K and V per block)."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    from paged_kv_cache_463_b200 import build
    build.build()
    spec = wl.SPEC_BY_NAME["llama2-7b-mha"]
    nb = 12288
    pa = pab.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, nb, max_num_seqs=1,
                            max_blocks_per_seq=128, device=local)
    dev = f"cuda:{local}"
    kc = torch.randn((nb, 16, spec.num_kv_heads, spec.head_dim), device=dev).half()
    vc = torch.randn_like(kc)
    block_bytes = kc[0].numel() * kc.element_size()
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(0))
    n = 4096
    pairs = torch.stack([perm[:n], perm[n:2 * n]], 1).to(torch.int64).to(dev)
    hn = 1024
    hk = torch.empty((hn, 16, spec.num_kv_heads, spec.head_dim), dtype=torch.float16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.stack([perm[:hn], torch.arange(hn)], 1).to(torch.int64).to(dev)
    in_pairs = torch.stack([torch.arange(hn), perm[2 * n:2 * n + hn]], 1).to(torch.int64).to(dev)
    stream = torch.cuda.current_stream()

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    d2d_ms = timed(lambda: pa.paged_copy_blocks(kc, vc, kc, vc, pairs, stream=stream), args.steps)
    out_ms = timed(lambda: pa.paged_copy_blocks(hk, hv, kc, vc, out_pairs, stream=stream), max(3, args.steps // 10))
    in_ms = timed(lambda: pa.paged_copy_blocks(kc, vc, hk, hv, in_pairs, stream=stream), max(3, args.steps // 10))
    if pa.get_error() != 0:
        raise SystemExit("device check fired")
    d2d = 2 * 2 * n * block_bytes / (d2d_ms * 1e-3) / 1e9
    line = {"metric": "paged block copy (copy-on-write, swap): GB/s read+written", "value": d2d, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": d2d_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": "block copy, 7B layer block shape (128 KiB per tensor per block)",
                       "pairs": n, "swap_blocks": hn},
            "swap_out_to_pinned_host_gbs": 2 * hn * block_bytes / (out_ms * 1e-3) / 1e9,
            "swap_in_from_pinned_host_gbs": 2 * hn * block_bytes / (in_ms * 1e-3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": d2d, "peak": measured_hbm_peak()[0], "unit": "GB/s",
                         "frac": d2d / measured_hbm_peak()[0]}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    pa.close()
    return 0


def run_block_manager(args, world, rank, local):
    """Host bookkeeping of a decode step with the native block manager, on the
    256-sequence shared-prefix workload's shape: 8 prompts of 1024 tokens are
    admitted through the prefix cache (the first one per group allocates, the
    other 31 share its 64 blocks), every sequence gets its private suffix, and
    then each step appends one token to all 256 sequences (slots and any
    copy-on-write pairs) and exports the batch's block tables and lengths.
    Host wall time (this is CPU code); the oracle's manager is timed on a
    bounded number of steps beside it."""
    import time
    from oracle.block_manager import BlockManager as OracleBM  # CPU-baseline leg only
    spec = wl.SPEC_BY_NAME["shared-prefix-fp8"]
    lay = wl.build_layout(spec)
    S, bs = spec.num_seqs, spec.block_size
    nb = lay.num_blocks + S * (args.steps + args.warmup) // bs + 2 * S
    bt_stride = lay.block_tables.shape[1] + (args.steps + args.warmup) // bs + 2

    def admit(bm, alloc, append):
        for g in range(spec.prefix_groups):
            prompt = [g * 100000 + t for t in range(spec.prefix_tokens)]
            for s in range(lay.group_start[g], lay.group_start[g + 1]):
                alloc(bm, s, prompt)
                append(bm, s, lay.seq_lens[s] - spec.prefix_tokens)

    sids = list(range(S))

    def run(step, steps):
        t0 = time.perf_counter()
        for _ in range(steps):
            step()
        return (time.perf_counter() - t0) / steps

    nat = pab.BlockManager(nb, bs)
    admit(nat, lambda bm, s, p: bm.allocate_with_prefix(s, p), lambda bm, s, n: bm.append_tokens(s, n))

    def nat_step():  # one batched append call + the batch's tables
        nat.append_batch(sids)
        nat.build_batch(sids, bt_stride)

    run(nat_step, args.warmup)
    sec = run(nat_step, args.steps)
    ora = OracleBM(nb, bs)
    admit(ora, lambda bm, s, p: bm.allocate_with_prefix(s, p), lambda bm, s, n: bm.append_tokens(s, n))

    def ora_step():
        for s in sids:
            ora.append_tokens(s, 1)
        ora.build_batch(sids, bt_stride)

    osteps = max(3, min(args.steps, 50))
    osec = run(ora_step, osteps)
    line = {"metric": "block-manager decode-step bookkeeping (append 1 token x 256 sequences + batch tables): "
                      "steps/s", "value": 1.0 / sec, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sec, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "config": {"workload": "shared-prefix-fp8 layout: 256 sequences, 8 prompts of 1024 tokens through the "
                                   "prefix cache, private suffixes U[16,1024]", "blocks": nb, "bt_stride": bt_stride,
                       "timing": "host wall clock (CPU code), through the ctypes binding"},
            "cached_blocks": nat.cached_blocks(),
            "cpu_baseline": {"value": 1.0 / osec, "unit": "steps/s", "cores": 1, "kind": "oracle",
                             "sample": f"{osteps} steps of the same loop with the Python oracle manager"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    nat.close()
    return 0


def run_prefill(args, world, rank, local):
    """Prefill step: write the prompts' K/V into the paged cache
    (reshape_and_cache) and run causal multi-query paged attention over them
    (paged_attention_prefill).  Workload: 16 prompts x 2048 tokens of the GQA
    70B-like layer (64 query / 8 KV heads, head_dim 128, bf16), blocks
    shuffled across the pool.  Metric: attention TFLOP/s counting the causal
    half only, 4 * Hq * D * L(L+1)/2 per sequence."""
    import numpy as np
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    from paged_kv_cache_463_b200 import build
    build.build()
    S, L = (args.num_seqs or 16), 2048
    spec = wl.WorkloadSpec("prefill-gqa-70b-like", S, 64, 8, 128, 16, "bf16", "bf16", L, L, seed=1010,
                           description=f"{S} prompts x {L} tokens, 64 q / 8 kv heads, head_dim 128, bf16")
    dev = f"cuda:{local}"
    w = wl.make_workload(spec, dev)
    T = S * L
    gen = torch.Generator(device=dev).manual_seed(1010)
    q = torch.randn((T, spec.num_heads, spec.head_dim), generator=gen, device=dev).bfloat16()
    k_new = torch.randn((T, spec.num_kv_heads, spec.head_dim), generator=gen, device=dev).bfloat16()
    v_new = torch.randn_like(k_new)
    # every prompt position's slot, from the block tables
    bt = w.block_tables.long()
    pos = torch.arange(L, device=dev)
    slots = (bt[:, pos // 16] * 16 + pos % 16).reshape(-1)
    qstart = torch.arange(0, T + 1, L, dtype=torch.int32, device=dev)
    pa = pab.PagedAttention(spec.num_heads, spec.num_kv_heads, spec.head_dim, w.num_blocks, q_dtype="bf16",
                            kv_dtype="bf16", max_num_seqs=S, max_blocks_per_seq=w.block_tables.shape[1], device=local)
    kc, vc = w.key_cache, w.value_cache
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    flops = 4.0 * spec.num_heads * spec.head_dim * S * L * (L + 1) / 2

    def step():
        pa.reshape_and_cache(k_new, v_new, kc, vc, slots, stream=stream)
        pa.paged_attention_prefill(out, q, kc, vc, w.block_tables, w.seq_lens, qstart, L, L, w.scale, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pa.get_error() != 0:
        raise SystemExit("device check fired during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for a, m, e in ev:
            a.record(stream)
            pa.reshape_and_cache(k_new, v_new, kc, vc, slots, stream=stream)
            m.record(stream)
            pa.paged_attention_prefill(out, q, kc, vc, w.block_tables, w.seq_lens, qstart, L, L, w.scale,
                                       stream=stream)
            e.record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    if pa.get_error() != 0:
        raise SystemExit("device check fired during the timed region")
    attn_ms = sum(m.elapsed_time(e) for _, m, e in ev) / args.steps
    value = world * flops * args.steps / (total_ms * 1e-3) / 1e12
    achieved = flops / (attn_ms * 1e-3) / 1e12
    peak, peak_kind = measured_bf16_peak()
    line = {"metric": "paged prefill attention: TFLOP/s (causal half) and tokens/s", "value": value,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": spec.name, "description": spec.description, "num_seqs": S, "prompt_tokens": L,
                       "step": "reshape_and_cache of every prompt token + paged_attention_prefill",
                       "l2": "K/V and queries (1.1 GB) larger than L2, no flush"},
            "tokens_per_s": world * T * args.steps / (total_ms * 1e-3),
            "attention_ms": attn_ms,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None, "kernel": "paged_prefill_kernel",
                         "peak_kind": peak_kind},
            "gpu_launches": 2 * args.steps, "clocks": clk.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import time
        from oracle import attention  # CPU-baseline leg only
        rows = [(t, h) for t in range(L - 4, L) for h in range(spec.num_heads)]
        hq = q.cpu().view(torch.int16).numpy().view(np.uint16)
        t_a = time.perf_counter()
        attention.prefill_attention(hq[:L], raw_np(kc), raw_np(vc), w.block_tables.cpu().numpy()[:1],
                                    w.seq_lens.cpu().numpy()[:1], np.array([0, L]), w.scale, q_dtype="bf16",
                                    kv_dtype="bf16", rows=rows)
        el = time.perf_counter() - t_a
        f = 4.0 * spec.num_heads * spec.head_dim * sum(t + 1 for t in range(L - 4, L))
        line["cpu_baseline"] = {"value": f / el / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                                "sample": f"the last 4 positions x {spec.num_heads} heads of one 2048-token prompt"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    pa.close()
    return 0


def raw_np(t):
    import numpy as np
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["decode-step", "copy-blocks", "block-manager", "prefill"], default="decode-step",
                    help="decode-step: the hot path (default); copy-blocks: block copies for COW / swap; "
                         "block-manager: host bookkeeping of a decode step; prefill: causal multi-query attention")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(wl.SPEC_BY_NAME))
    ap.add_argument("--partition", default="auto", help="auto | none | tokens per partition")
    ap.add_argument("--eager", dest="graph", action="store_false",
                    help="launch each step's kernels directly instead of replaying a captured CUDA graph")
    ap.add_argument("--num-seqs", type=int, default=0, help="smaller batch of the same workload (profiling)")
    ap.add_argument("--shared-prefix", choices=["auto", "on", "off"], default="auto",
                    help="shared-prefix decode for workloads with prefix groups (auto: when the workload has them)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--decode-seconds", type=float, default=1.0,
                    help="minimum length of the back-to-back decode-call loop behind decode_ms and the roofline")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other full-size workloads (per_workload) of the default run")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        if args.op == "copy-blocks":
            return run_copy_blocks(args, world, rank, local)
        if args.op == "block-manager":
            return run_block_manager(args, world, rank, local)
        if args.op == "prefill":
            return run_prefill(args, world, rank, local)
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
