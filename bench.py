"""Benchmark of the SAW-INT4 paged INT4 KV-cache hot path on B200.

One step = one serving step of the decode workload (Llama-3-8B layer shape: 64 sequences with
lengths uniform on {512..8192}, 32 query / 8 kv heads, head_dim 128, 16-token pages): the new
token of every sequence is rotated, INT4-quantized and scattered into the paged cache, then
decode attention runs over the whole INT4 cache (saw_decode_step through the C ABI).  The
headline value is decode tokens/s (sequences served per second, summed over ranks).  The same
line also reports the rotate+quantize kernel's GB/s on the prefill workload (32 x 2048 tokens,
8 kv heads), both kernels' fractions of the HBM roofline, an end-to-end number through host
buffers (pinned inputs copied in and the output copied back every step, in a double-buffered
loop whose copies overlap the neighbouring steps' kernels; the serialised loop is reported
beside it), and the CPU oracle as a baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With --impl reference the script times the CPU oracle (the plain C reference in oracle/) on a
bounded sample of the same workload and prints its line; under torchrun only rank 0 does so.

Profiling aids (their numbers are not bench values): --loop-launches L --loop-seconds 0 cuts every
per-kernel timing loop to L launches, so that a one-pass ncu launch list covers the whole bench;
--profile rot_quant|decode builds one kernel's workload and launches that kernel six times, for a
full ncu capture of a single launch; --profile window runs the windowed serving step six times.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "INT4 paged decode tokens/s"
UNIT = "tokens/s"
HBM_TARGET_GBS = 8000.0            # the 8 TB/s roofline the targets are stated against
CODE_ROW_BYTES = 64
BYTES_PER_TOKEN_HEAD_APPEND = 2 * 128 * 2 + 2 * CODE_ROW_BYTES + 2 * 4   # bf16 in, codes+scales out
WORKLOAD_TEXT = ("decode step, Llama-3-8B layer shape: batch 64, seq_lens uniform 512-8192, "
                 "32 q / 8 kv heads, head_dim 128, page 16, one new token per seq appended "
                 "(rotate + INT4 quantize + scatter) then INT4 paged decode attention; bf16 "
                 "N(0,1) with 4 key outlier channels x U[10,30]")
CPU_SAMPLE_SEQS = 8
WORKLOADS = {
    "long": "long-context decode: batch 8 x 32768 tokens, 64 q / 8 kv heads, head_dim 128, page 16, "
            "block table a shuffled permutation of 16384 pages, decode only; bf16 N(0,1) with 4 "
            "key outlier channels x20",
    "serving": "high-concurrency serving step: batch 256, seq_lens round(lognormal(ln 1024, 1.0)) "
               "clipped to [64, 16384], 32 q / 8 kv heads, head_dim 128, page 16, one new token per "
               "seq appended then decoded (fused step); bf16 N(0,1) with 4 key outlier channels "
               "x U[10,30]",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", default="saw", choices=["saw", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # profiling aids: shorter per-kernel loops (for a launch list under ncu), or one kernel's
    # workload alone, launched a few times (for a full ncu capture of one launch)
    ap.add_argument("--loop-launches", type=int, default=200,
                    help="per-kernel timing loops run at least this many launches")
    ap.add_argument("--loop-seconds", type=float, default=0.5,
                    help="... and at least this long (0: exactly --loop-launches)")
    ap.add_argument("--profile", choices=["rot_quant", "decode", "window"],
                    help="run only this kernel (window: the windowed step) on its workload, 6 times")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


# ---- ranks (weak scaling: each rank serves its own batch; no exchange on the data path) ------

def rank_workload(rank: int):
    """The decode workload rank `rank` serves: the same shapes on every rank, its own seed."""
    from bit_paged_kv_block_b200 import synth
    return synth.make_workload("decode", seed=rank)


def max_over_ranks(value: float, pg=None, device="cpu") -> float:
    """The maximum of `value` over all ranks of the process group (the value itself alone)."""
    if pg is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's step time."""
    return world * units_per_rank / (ms_per_step_max / 1e3)


# ---- byte accounting (algorithmic bytes, not measured traffic) ----------------------------

def decode_bytes(wl) -> int:
    """Algorithmic bytes of one INT4 decode: per cached token and kv head D / 2 bytes of codes
    for K and for V plus 8 B of fp16 (scale, zero) pairs (136 B at D = 128); per sequence the
    bf16 queries, fp32 outputs, its length and its block-table entries."""
    D = wl.head_dim
    lens = wl.seq_lens.astype(np.int64)
    pages = (lens + 15) // 16
    per_seq = wl.num_q_heads * D * (2 + 4) + 4 + 4 * pages
    return int((wl.num_kv_heads * lens * (D + 8)).sum() + per_seq.sum())


def decode_bytes_bf16(wl) -> int:
    """Algorithmic bytes of one decode over the uncompressed bf16 cache: 512 B per cached
    token and kv head (K and V, 128 bf16 each) plus the same per-sequence terms."""
    lens = wl.seq_lens.astype(np.int64)
    pages = (lens + 15) // 16
    per_seq = wl.num_q_heads * 128 * (2 + 4) + 4 + 4 * pages
    return int((wl.num_kv_heads * lens * 512).sum() + per_seq.sum())


def append_bytes(num_tokens: int, hkv: int) -> int:
    return num_tokens * (hkv * BYTES_PER_TOKEN_HEAD_APPEND + 8)


# ---- clocks ----------------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while a timed loop runs.

    The sampling thread lives for the whole benchmark but records only inside `with
    sampler.timed():` blocks, so the record covers every timed region (the headline steps and
    the per-kernel and per-line loops) and none of the set-up work between them."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.ok = [], set(), False
        self.headline_samples = 0
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()
        self._active = threading.Event()
        self._t = None

    def _sample(self):
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, b in self.REASONS.items():
                if bits & b and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            if self._active.wait(0.05):
                self._sample()
                time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def stop(self):
        self._stop.set()
        self._active.set()
        if self._t is not None:
            self._t.join()

    class _Timed:
        def __init__(self, owner):
            self.owner = owner

        def __enter__(self):
            if self.owner.ok:
                self.owner._sample()          # at least one sample per region
            self.owner._active.set()

        def __exit__(self, *exc):
            self.owner._active.clear()

    def timed(self):
        return ClockSampler._Timed(self)

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "headline_region_samples": self.headline_samples,
                "source": "NVML every 5 ms inside every timed region of this run (the headline "
                          "steps and each per-kernel / per-line timing loop)"}


# ---- roofline denominators -----------------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor-core TFLOP/s measured on this machine (the burst figure: the prefill kernel
    is timed alone); fp16 runs at the same nominal rate.  Fallback: 1590."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def sources_digest(sources) -> str:
    """sha256 over the named csrc files, in order (the kernel's whole source)."""
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "bit_paged_kv_block_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def kernel_traffic(kernel: str, units: float):
    """dram bytes per launch from the committed ncu summary, if it was taken on the current
    kernel sources (scaled by `units` / the captured units); else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        if sources_digest(rec["sources"]) != rec["sources_sha256"]:
            return None
        return rec["dram_bytes_per_launch"] * units / rec["units"]
    except Exception:
        return None



# ---- timing helpers ----------------------------------------------------------------------------

MIN_LAUNCHES = 200        # per-launch loops: at least this many launches ...
MIN_LOOP_SECONDS = 0.5    # ... and at least this long, whatever --steps is


def loop_count(fn, stream, min_launches=None, min_seconds=None, cap=20000):
    """Launches a timing loop needs to reach both bounds (estimated from 10 back-to-back runs)."""
    import torch
    min_launches = MIN_LAUNCHES if min_launches is None else min_launches
    min_seconds = MIN_LOOP_SECONDS if min_seconds is None else min_seconds
    if min_seconds <= 0:
        return min_launches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(10):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    est = max(e0.elapsed_time(e1) / 10 / 1e3, 1e-6)
    return int(min(cap, max(min_launches, math.ceil(min_seconds / est))))


def per_launch_ms(fn, stream, clocks, n=None):
    """Mean CUDA-event duration of one call of fn (events around each call, on its stream)."""
    import torch
    for _ in range(3):
        fn()
    if n is None:
        n = loop_count(fn, stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    torch.cuda.synchronize()
    with clocks.timed():
        for e in evs:
            e[0].record(stream)
            fn()
            e[1].record(stream)
        torch.cuda.synchronize()
    return statistics.mean(e[0].elapsed_time(e[1]) for e in evs), n


def back_to_back_ms(fn, stream, clocks, n=None, pg=None, dev="cpu"):
    """Mean time of one call of fn in a loop of n back-to-back calls (one event pair), max over
    ranks."""
    import torch
    for _ in range(3):
        fn()
    if n is None:
        n = loop_count(fn, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with clocks.timed():
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1) / n, pg, dev), n


def host_cpu():
    """The host's CPU model (from /proc/cpuinfo) and its logical CPU count."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, os.cpu_count() or 1

# ---- the CPU oracle baseline ------------------------------------------------------------

def oracle_sample(wl, seed_seqs: int = CPU_SAMPLE_SEQS, nthreads=None):
    """Oracle-built history cache for the first `seed_seqs` sequences (CPU only)."""
    import oracle
    from bit_paged_kv_block_b200 import synth
    sub = synth.Workload(**{**wl.__dict__})
    sel = np.arange(seed_seqs)
    sub.num_seqs = seed_seqs
    sub.seq_lens = wl.seq_lens[sel].copy()
    sub.new_tokens = wl.new_tokens[sel].copy()
    sub.block_table = np.ascontiguousarray(wl.block_table[sel])
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    bits = lambda t: t.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    pages, scales = oracle.empty_cache(wl.num_pages, wl.num_kv_heads)
    seq, pos = synth.token_index(sub, "history")
    oracle.rotate_quantize_paged(bits(synth.kv_values(sub, "K", tokens="history")),
                                 bits(synth.kv_values(sub, "V", tokens="history")),
                                 synth.slot_mapping(sub, seq, pos), pages, scales,
                                 nthreads=os.cpu_count() or 1)
    seq, pos = synth.token_index(sub, "new")
    new = (bits(synth.kv_values(sub, "K", tokens="new")),
           bits(synth.kv_values(sub, "V", tokens="new")), synth.slot_mapping(sub, seq, pos))
    q = bits(synth.q_values(wl))[sel].copy()
    return sub, pages, scales, new, q, nthreads


def oracle_step(sub, pages, scales, new, q, nthreads):
    import oracle
    oracle.rotate_quantize_paged(new[0], new[1], new[2], pages, scales, nthreads=nthreads)
    return oracle.decode_fp64(q, pages, scales, sub.block_table, sub.seq_lens,
                              nthreads=nthreads)


def _timed_reps(fn, min_seconds):
    fn()                                               # warm
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            return reps, el


def cpu_baseline(wl, seconds_each: float = 6.0):
    """The oracle as it stands on the host cores: the decode step on a sample of the decode
    workload (all host threads, then one thread) and the rotate + quantize + scatter on a sample
    of the prefill workload (same two thread counts)."""
    import oracle
    from bit_paged_kv_block_b200 import synth
    model, ncpu = host_cpu()
    out = {"unit": UNIT, "kind": "oracle", "cpu_model": model, "nproc": ncpu}
    # decode step, all threads (8 sequences) and one thread (2 sequences)
    for key, nseq, nth in (("all_cores", CPU_SAMPLE_SEQS, ncpu), ("single_thread", 2, 1)):
        sub, pages, scales, new, q, nthreads = oracle_sample(wl, nseq, nthreads=nth)
        reps, el = _timed_reps(lambda: oracle_step(sub, pages, scales, new, q, nthreads), seconds_each)
        out[key] = {"value": sub.num_seqs * reps / el, "unit": UNIT, "cores": nthreads,
                    "sample": f"first {sub.num_seqs} of the 64 sequences ({int(sub.seq_lens.sum())} "
                              f"cached tokens): oracle append of their new tokens + fp64 decode, "
                              f"{reps} repetitions in {el:.1f} s on {nthreads} thread(s)"}
    out["value"] = out["all_cores"]["value"]
    out["cores"] = out["all_cores"]["cores"]
    out["sample"] = out["all_cores"]["sample"]
    # rotate + quantize + scatter on the prefill workload's first 2 sequences (4096 tokens)
    pre = synth.make_workload("prefill", seed=0)
    sub = synth.Workload(**{**pre.__dict__})
    sub.num_seqs = 2
    sub.seq_lens = pre.seq_lens[:2].copy()
    sub.new_tokens = pre.new_tokens[:2].copy()
    sub.block_table = np.ascontiguousarray(pre.block_table[:2])
    bits = lambda t: t.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    seq, pos = synth.token_index(sub, "all")
    kb, vb = bits(synth.kv_values(sub, "K")), bits(synth.kv_values(sub, "V"))
    slots = synth.slot_mapping(sub, seq, pos)
    pages, scales = oracle.empty_cache(pre.num_pages, pre.num_kv_heads)
    nbytes = append_bytes(len(seq), pre.num_kv_heads)
    quant = {"workload": "prefill rotate + INT4 quantize + scatter (32 x 2048 tokens, 8 kv heads), "
                         f"sample: its first 2 sequences ({len(seq)} tokens), same byte accounting "
                         "as the GPU line", "unit": "GB/s"}
    for key, nth in (("all_cores", ncpu), ("single_thread", 1)):
        reps, el = _timed_reps(lambda: oracle.rotate_quantize_paged(kb, vb, slots, pages, scales,
                                                                     nthreads=nth), seconds_each / 2)
        quant[key] = {"GBps": nbytes * reps / el / 1e9, "cores": nth, "repetitions": reps,
                      "seconds": el}
    out["rot_quant"] = quant
    return out


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from bit_paged_kv_block_b200 import synth
    wl = synth.make_workload("decode", seed=0)
    # size each step's sample so that warmup + K steps stay within about two minutes
    sub, pages, scales, new, q, nthreads = oracle_sample(wl, 1)
    t0 = time.perf_counter()
    oracle_step(sub, pages, scales, new, q, nthreads)
    per_seq = max(time.perf_counter() - t0, 1e-4)
    n = int(max(1, min(CPU_SAMPLE_SEQS, 120.0 / (per_seq * (args.steps + args.warmup)))))
    if n > 1:
        sub, pages, scales, new, q, nthreads = oracle_sample(wl, n)
    for _ in range(max(args.warmup, 0)):
        oracle_step(sub, pages, scales, new, q, nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(sub, pages, scales, new, q, nthreads)
    el = time.perf_counter() - t0
    value = sub.num_seqs * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT, "sample_seqs": sub.num_seqs},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": f"each step: first {sub.num_seqs} of the 64 sequences, "
                                   f"oracle append + fp64 decode"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- the CUDA path --------------------------------------------------------------------------

def run_saw(args):
    import torch
    from bit_paged_kv_block_b200 import saw, synth

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    # ---- inputs: each rank serves its own batch (weak scaling, no exchange on the path) ----
    wl = rank_workload(rank)
    kv, sc = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, dev)
    seq, pos = synth.token_index(wl, "history")
    saw.saw_rotate_quantize_paged(synth.kv_values(wl, "K", tokens="history", device=dev),
                                  synth.kv_values(wl, "V", tokens="history", device=dev),
                                  torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(dev),
                                  kv, sc)
    seq, pos = synth.token_index(wl, "new")
    k_new = synth.kv_values(wl, "K", tokens="new", device=dev)
    v_new = synth.kv_values(wl, "V", tokens="new", device=dev)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(dev)
    q = synth.q_values(wl, device=dev)
    table = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    out = torch.empty((wl.num_seqs, wl.num_q_heads, 128), dtype=torch.float32, device=dev)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        saw.saw_decode_step(q, k_new, v_new, slots, kv, sc, table, lens, out, ws,
                            dev_status=status, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps, device events, max over ranks ----------------------
    clocks = ClockSampler(local_rank).start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with clocks.timed():
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    clocks.headline_samples = len(clocks.samples)
    ms = e0.elapsed_time(e1)
    if pg:
        pg.barrier()
    ms = max_over_ranks(ms, pg, dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item()):#x}")
    ms_per_step = ms / args.steps
    value = job_throughput(wl.num_seqs, world, ms_per_step)

    # ---- per-kernel durations (same inputs, events around each launch, >= 200 launches and
    # >= 0.5 s per loop whatever --steps is) ---------------------------------------------------
    t_append, n_app = per_launch_ms(lambda: saw.saw_rotate_quantize_paged(
        k_new, v_new, slots, kv, sc, dev_status=status, stream=stream), stream, clocks)
    decode_call = lambda: saw.saw_paged_decode_attn(q, kv, sc, table, lens, out, ws,
                                                    dev_status=status, stream=stream)
    t_decode, n_kt = per_launch_ms(decode_call, stream, clocks)
    dec_bytes = decode_bytes(wl)
    peak_gbs, peak_kind = measured_peaks()
    dec_gbs = dec_bytes / (t_decode * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": dec_gbs, "peak": peak_gbs, "unit": "GB/s",
                "frac": dec_gbs / peak_gbs, "peak_kind": peak_kind,
                "kernel": "paged_decode_kernel", "algorithmic_bytes_per_launch": dec_bytes,
                "launch_ms": t_decode, "launches_timed": n_kt,
                "frac_of_8TBps": dec_gbs / HBM_TARGET_GBS,
                "traffic": kernel_traffic("paged_decode_kernel", int(wl.seq_lens.sum()))}

    # ---- the long-context and high-concurrency workloads: one line each ------------------------
    def workload_line(name, fused):
        """Decode-only (long context) or fused append + decode (serving) on another workload."""
        w2 = synth.make_workload(name, seed=rank)
        kv2, sc2 = saw.allocate_cache(w2.num_pages, w2.num_kv_heads, dev)
        sq, sp = synth.token_index(w2, "history")
        saw.saw_rotate_quantize_paged(synth.kv_values(w2, "K", tokens="history", device=dev),
                                      synth.kv_values(w2, "V", tokens="history", device=dev),
                                      torch.from_numpy(synth.slot_mapping(w2, sq, sp)).to(dev),
                                      kv2, sc2)
        sq, sp = synth.token_index(w2, "new")
        kn2 = synth.kv_values(w2, "K", tokens="new", device=dev)
        vn2 = synth.kv_values(w2, "V", tokens="new", device=dev)
        sl2 = torch.from_numpy(synth.slot_mapping(w2, sq, sp)).to(dev)
        q2 = synth.q_values(w2, device=dev)
        tab2 = torch.from_numpy(w2.block_table).to(dev)
        len2 = torch.from_numpy(w2.seq_lens).to(dev)
        out2 = torch.empty((w2.num_seqs, w2.num_q_heads, 128), dtype=torch.float32, device=dev)
        ws2 = saw.allocate_workspace(w2.num_kv_heads, w2.num_q_heads, w2.num_seqs, dev)
        dec2 = lambda: saw.saw_paged_decode_attn(q2, kv2, sc2, tab2, len2, out2, ws2,
                                                 dev_status=status, stream=stream)
        if fused:
            step2 = lambda: saw.saw_decode_step(q2, kn2, vn2, sl2, kv2, sc2, tab2, len2, out2, ws2,
                                                dev_status=status, stream=stream)
        else:
            step2 = dec2
        st_ms, st_n = back_to_back_ms(step2, stream, clocks, pg=pg, dev=dev)
        d_ms, d_n = per_launch_ms(dec2, stream, clocks)
        torch.cuda.synchronize()
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item()):#x} on {name}")
        b2 = decode_bytes(w2)
        g2 = b2 / (d_ms * 1e-3) / 1e9
        step_bytes = b2 + (append_bytes(int(w2.new_tokens.sum()), w2.num_kv_heads) if fused else 0)
        line2 = {"workload": WORKLOADS[name], "batch": w2.num_seqs,
                 "kv_tokens": int(w2.seq_lens.sum()),
                 "step": "append one new token per sequence + decode" if fused else "decode only",
                 "step_ms": st_ms, "steps_timed": st_n,
                 "tokens_per_s": job_throughput(w2.num_seqs, world, st_ms),
                 "kv_tokens_per_s": world * int(w2.seq_lens.sum()) / (st_ms * 1e-3),
                 "step_GBps": step_bytes / (st_ms * 1e-3) / 1e9,
                 "launch_ms": d_ms, "launches_timed": d_n,
                 "algorithmic_bytes_per_launch": b2, "decode_GBps": g2,
                 "frac_of_measured_peak": g2 / peak_gbs, "frac_of_8TBps": g2 / HBM_TARGET_GBS}
        del kv2, sc2, kn2, vn2, q2, out2, ws2
        return line2

    long_ctx = workload_line("long", fused=False)
    serving = workload_line("serving", fused=True)

    # ---- prefill rotate+quantize throughput (the write side at full bandwidth) -------------
    pre = synth.make_workload("prefill", seed=rank)
    pkv, psc = saw.allocate_cache(pre.num_pages, pre.num_kv_heads, dev)
    pseq, ppos = synth.token_index(pre, "all")
    pk = synth.kv_values(pre, "K", device=dev)
    pv = synth.kv_values(pre, "V", device=dev)
    pslots = torch.from_numpy(synth.slot_mapping(pre, pseq, ppos)).to(dev)
    t_rq, n_rq = per_launch_ms(lambda: saw.saw_rotate_quantize_paged(pk, pv, pslots, pkv, psc,
                                                                     stream=stream), stream, clocks)
    rq_bytes = append_bytes(pre.total_tokens, pre.num_kv_heads)
    rq_gbs = rq_bytes / (t_rq * 1e-3) / 1e9
    rot_quant = {"workload": "prefill: 32 seqs x 2048 tokens, 8 kv heads, head_dim 128, page 16, "
                             "pages by seeded permutation",
                 "GBps": rq_gbs, "frac_of_8TBps": rq_gbs / HBM_TARGET_GBS,
                 "frac_of_measured_peak": rq_gbs / peak_gbs, "launch_ms": t_rq,
                 "launches_timed": n_rq, "algorithmic_bytes_per_launch": rq_bytes,
                 "traffic": kernel_traffic("rotate_quantize_kernel", pre.total_tokens)}

    # ---- the plain INT4 baseline (no rotation) on the same workloads: rotation overhead -------
    def mean_event_ms(fn, n=None):
        return per_launch_ms(fn, stream, clocks, n)[0]

    t_rq_plain = mean_event_ms(lambda: saw.saw_quantize_paged_plain(pk, pv, pslots, pkv, psc,
                                                                    stream=stream))
    del pk, pv, pkv, psc
    pkv2, psc2 = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, dev)
    seq, pos = synth.token_index(wl, "history")
    saw.saw_quantize_paged_plain(synth.kv_values(wl, "K", tokens="history", device=dev),
                                 synth.kv_values(wl, "V", tokens="history", device=dev),
                                 torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(dev),
                                 pkv2, psc2)
    plain_step = lambda: saw.saw_decode_step_plain(q, k_new, v_new, slots, pkv2, psc2, table, lens,
                                                   out, ws, dev_status=status, stream=stream)
    pl_ms, _ = back_to_back_ms(plain_step, stream, clocks, pg=pg, dev=dev)
    plain_int4 = {"what": "the same step and prefill quantize on a plain INT4 cache (H = I)",
                  "step_ms": pl_ms, "tokens_per_s": job_throughput(wl.num_seqs, world, pl_ms),
                  "step_rotation_overhead": ms_per_step / pl_ms - 1.0,
                  "prefill_quant_launch_ms": t_rq_plain,
                  "prefill_quant_rotation_overhead": t_rq / t_rq_plain - 1.0}
    del pkv2, psc2

    # ---- the uncompressed BF16 cache on the same step: what the INT4 compression buys -------
    kvb = saw.allocate_cache_bf16(wl.num_pages, wl.num_kv_heads, dev)
    seq, pos = synth.token_index(wl, "history")
    saw.saw_append_bf16_paged(synth.kv_values(wl, "K", tokens="history", device=dev),
                              synth.kv_values(wl, "V", tokens="history", device=dev),
                              torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(dev), kvb)
    wsb = saw.allocate_workspace_bf16(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    bf16_step = lambda: saw.saw_decode_step_bf16(q, k_new, v_new, slots, kvb, table, lens, out, wsb,
                                                 dev_status=status, stream=stream)
    bf_ms, _ = back_to_back_ms(bf16_step, stream, clocks, pg=pg, dev=dev)
    t_dec_bf16 = mean_event_ms(lambda: saw.saw_paged_decode_attn_bf16(
        q, kvb, table, lens, out, wsb, dev_status=status, stream=stream))
    bf_gbs = decode_bytes_bf16(wl) / (t_dec_bf16 * 1e-3) / 1e9
    bf16_baseline = {"what": "the same step on an uncompressed bf16 paged cache (4x the KV bytes)",
                     "step_ms": bf_ms, "tokens_per_s": job_throughput(wl.num_seqs, world, bf_ms),
                     "int4_step_speedup": bf_ms / ms_per_step,
                     "decode_launch_ms": t_dec_bf16, "decode_GBps": bf_gbs,
                     "decode_frac_of_measured_peak": bf_gbs / peak_gbs,
                     "int4_decode_speedup": t_dec_bf16 / t_decode}
    del kvb, wsb

    # ---- chunked prefill over the INT4 cache: a 512-token chunk per sequence -----------------
    pfl = synth.custom("chunked_prefill", [4096] * 8, num_q_heads=32, num_kv_heads=8,
                       seed=40 + rank, outlier_range=(10.0, 30.0))
    pkv3, psc3 = saw.allocate_cache(pfl.num_pages, pfl.num_kv_heads, dev)
    seq, pos = synth.token_index(pfl)
    saw.saw_rotate_quantize_paged(synth.kv_values(pfl, "K", device=dev),
                                  synth.kv_values(pfl, "V", device=dev),
                                  torch.from_numpy(synth.slot_mapping(pfl, seq, pos)).to(dev),
                                  pkv3, psc3)
    chunk = 512
    q_start = torch.arange(0, (pfl.num_seqs + 1) * chunk, chunk, dtype=torch.int32, device=dev)
    qpf = torch.randn(pfl.num_seqs * chunk, pfl.num_q_heads, 128, generator=torch.Generator(
        device="cpu").manual_seed(41), ).to(torch.bfloat16).to(dev)
    opf = torch.empty(qpf.shape, dtype=torch.float32, device=dev)
    wpf = saw.allocate_prefill_workspace(pfl.num_kv_heads, pfl.num_q_heads, pfl.num_seqs,
                                         int(qpf.shape[0]), dev)
    tab3, len3 = torch.from_numpy(pfl.block_table).to(dev), torch.from_numpy(pfl.seq_lens).to(dev)
    run_pf = lambda: saw.saw_paged_prefill_attn(qpf, q_start, pkv3, psc3, tab3, len3, opf, wpf,
                                                dev_status=status, stream=stream)
    for _ in range(3):
        run_pf()
    t_pf = mean_event_ms(run_pf)
    g = pfl.num_q_heads // pfl.num_kv_heads
    # the tensor-core kernel's tiles: 128 / G query tokens each, reading their causal range
    tile_tok = 128 // g
    page_reads = pfl.num_seqs * pfl.num_kv_heads * sum(
        (4096 - chunk + t0 + min(tile_tok, chunk - t0) + 15) // 16 for t0 in range(0, chunk, tile_tok))
    # causal attention: query i of a chunk at the end of L tokens sees L - chunk + i + 1 tokens
    visible = sum(4096 - chunk + i + 1 for i in range(chunk)) * pfl.num_seqs * pfl.num_q_heads
    tc_peak, tc_peak_kind = measured_tensor_peak()
    prefill_attn = {"workload": "8 seqs x 4096 cached tokens, last 512 of each as queries, 32 q / 8 kv heads",
                    "launch_ms": t_pf,
                    "query_tokens_per_s": world * pfl.num_seqs * chunk / (t_pf * 1e-3),
                    "attention_TFLOPs": 4 * 128 * visible / (t_pf * 1e-3) / 1e12,
                    "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel",
                                 "achieved": 4 * 128 * visible / (t_pf * 1e-3) / 1e12,
                                 "peak": tc_peak, "unit": "TFLOP/s",
                                 "frac": 4 * 128 * visible / (t_pf * 1e-3) / 1e12 / tc_peak,
                                 "peak_kind": tc_peak_kind,
                                 "note": "fp16 operands at the dense bf16 rate; flops = 4 D per "
                                         "visible (query, head, cache token)"},
                    "page_reads_per_launch": page_reads,
                    "note": "each 128-row tile (32 query tokens x 4 heads) reads its causal range of "
                            "the sequence's pages once; the repeats across tiles come from L2"}
    del pkv3, psc3, qpf, opf, wpf

    # ---- head dimensions 64 and 256: the decode workload's shape with other head vectors -------
    head_dims = {}
    for hd in (64, 256):
        whd = synth.custom(f"decode_d{hd}", wl.seq_lens, num_q_heads=wl.num_q_heads,
                           num_kv_heads=wl.num_kv_heads, seed=50 + rank, head_dim=hd)
        kv4, sc4 = saw.allocate_cache(whd.num_pages, whd.num_kv_heads, dev, head_dim=hd)
        seq, pos = synth.token_index(whd)
        saw.saw_rotate_quantize_paged(synth.kv_values(whd, "K", device=dev),
                                      synth.kv_values(whd, "V", device=dev),
                                      torch.from_numpy(synth.slot_mapping(whd, seq, pos)).to(dev),
                                      kv4, sc4)
        q4 = synth.q_values(whd, device=dev)
        o4 = torch.empty(q4.shape, dtype=torch.float32, device=dev)
        ws4 = saw.allocate_workspace(whd.num_kv_heads, whd.num_q_heads, whd.num_seqs, dev,
                                     head_dim=hd)
        tab4 = torch.from_numpy(whd.block_table).to(dev)
        run_d4 = lambda: saw.saw_paged_decode_attn(q4, kv4, sc4, tab4, lens, o4, ws4,
                                                   dev_status=status, stream=stream)
        for _ in range(3):
            run_d4()
        t_d4 = mean_event_ms(run_d4)
        d4_gbs = decode_bytes(whd) / (t_d4 * 1e-3) / 1e9
        head_dims[f"head_dim_{hd}"] = {
            "workload": f"the decode batch (same lengths and heads) at head_dim {hd}",
            "decode_launch_ms": t_d4, "algorithmic_bytes_per_launch": decode_bytes(whd),
            "decode_GBps": d4_gbs, "decode_frac_of_measured_peak": d4_gbs / peak_gbs}
        del kv4, sc4, q4, o4, ws4

    # ---- full-precision sink / recent window ("InnerQ", Figure 2): W = 16 + 112 bf16 tokens ----
    sink, recent = 16, 112
    W = sink + recent
    wkv, wtab = saw.allocate_window(wl.num_seqs, wl.num_kv_heads, sink, recent, dev)
    wkv5, wsc5 = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, dev)
    kh = synth.kv_values(wl, "K", tokens="history", device=dev)
    vh = synth.kv_values(wl, "V", tokens="history", device=dev)
    seqh, posh = synth.token_index(wl, "history")
    Lh = wl.seq_lens[seqh] - 1                      # history length of each token's sequence
    in_win = (posh < sink) | (posh >= np.maximum(sink, Lh - recent))
    j = posh - sink
    qslot = np.where(in_win, -1, wl.block_table[seqh, np.maximum(j, 0) // 16] * 16 + j % 16)
    wslot = np.where(posh < sink, posh, sink + (posh - sink) % max(recent, 1))
    wtab_np = wtab.cpu().numpy()
    wslot = np.where(in_win, wtab_np[seqh, wslot // 16] * 16 + wslot % 16, -1)
    saw.saw_rotate_quantize_paged(kh, vh, torch.from_numpy(qslot.astype(np.int64)).to(dev), wkv5, wsc5)
    saw.saw_append_bf16_paged(kh, vh, torch.from_numpy(wslot.astype(np.int64)).to(dev), wkv)
    del kh, vh
    win = (sink, recent, wkv, wtab)
    wsw = saw.allocate_window_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    win_step = lambda: saw.saw_decode_step_window(q, k_new, v_new, win, wkv5, wsc5, table, lens,
                                                  out, wsw, dev_status=status, stream=stream)
    win_decode = lambda: saw.saw_paged_decode_attn_window(q, win, wkv5, wsc5, table, lens, out, wsw,
                                                          dev_status=status, stream=stream)
    win_ms, _ = back_to_back_ms(win_step, stream, clocks, pg=pg, dev=dev)
    t_wdec = mean_event_ms(win_decode)
    win_tokens = int(np.minimum(wl.seq_lens, W).sum())
    win_bytes = (decode_bytes(wl) - wl.num_kv_heads * win_tokens * 136
                 + wl.num_kv_heads * win_tokens * 512)
    window = {"what": f"the same step with a bf16 window of {sink} sink + {recent} recent tokens "
                      "per sequence beside the INT4 cache (append with eviction, then the window "
                      "part and the quantized part merged)",
              "step_ms": win_ms, "tokens_per_s": job_throughput(wl.num_seqs, world, win_ms),
              "step_vs_int4": win_ms / ms_per_step,
              "decode_launch_ms": t_wdec,
              "decode_algorithmic_bytes": win_bytes,
              "decode_GBps": win_bytes / (t_wdec * 1e-3) / 1e9}
    del wkv, wtab, wkv5, wsc5, wsw

    # ---- end to end through the public API with host buffers ------------------------------
    # A double-buffered serving loop: each step's inputs (q, new k / v, slot mapping, block
    # table, lengths) travel in one pinned host block by one host-to-device copy on a copy
    # stream, the step runs on the compute stream, and its output comes back by one
    # device-to-host copy on a second copy stream.  Two slots of device inputs and outputs let
    # step i's output copy and step i + 1's input copy run on the copy engines while the compute
    # stream works; every byte still crosses the bus inside the timed region.
    parts = [q, k_new, v_new, slots, table, lens]
    nbytes = [t_.numel() * t_.element_size() for t_ in parts]
    offs = [0]
    for nb in nbytes[:-1]:
        offs.append(offs[-1] + (nb + 255) // 256 * 256)
    total = offs[-1] + (nbytes[-1] + 255) // 256 * 256
    h_in, d_in, d_views = [], [], []
    for _ in range(2):
        hb = torch.empty(total, dtype=torch.uint8).pin_memory()
        for t_, o, nb in zip(parts, offs, nbytes):
            hb[o:o + nb].copy_(t_.reshape(-1).view(torch.uint8).cpu())
        db = torch.empty(total, dtype=torch.uint8, device=dev)
        h_in.append(hb)
        d_in.append(db)
        d_views.append([db[o:o + nb].view(t_.dtype).view(t_.shape) for t_, o, nb in zip(parts, offs, nbytes)])
    d_out = [torch.empty_like(out) for _ in range(2)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(nbytes)
    d2h = out.numel() * out.element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]   # the slot's kernels have run
    ev_back = [torch.cuda.Event() for _ in range(2)]   # the slot's output is on the host

    def e2e_step(i):
        b_ = i & 1
        s_in.wait_event(ev_done[b_])        # step i - 2's kernels are done with the input slot
        with torch.cuda.stream(s_in):
            d_in[b_].copy_(h_in[b_], non_blocking=True)
        ev_in[b_].record(s_in)
        stream.wait_event(ev_in[b_])
        stream.wait_event(ev_back[b_])      # step i - 2's output has left the output slot
        qv, kv_new, vv_new, sl, tbv, lnv = d_views[b_]
        saw.saw_decode_step(qv, kv_new, vv_new, sl, kv, sc, tbv, lnv, d_out[b_], ws,
                            dev_status=status, stream=stream)
        ev_done[b_].record(stream)
        s_out.wait_event(ev_done[b_])
        with torch.cuda.stream(s_out):
            h_out[b_].copy_(d_out[b_], non_blocking=True)
        ev_back[b_].record(s_out)

    for i in range(4):
        e2e_step(i)
    n_e2e = loop_count(step, stream)
    n_e2e += n_e2e & 1
    torch.cuda.synchronize()
    with clocks.timed():
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(n_e2e):
            e2e_step(i)
        stream.wait_stream(s_out)
        e1.record(stream)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, pg, dev)
    # the same copies and step without overlap (one stream: copy in, step, copy out), for context
    def e2e_serial():
        d_in[0].copy_(h_in[0], non_blocking=True)
        qv, kv_new, vv_new, sl, tbv, lnv = d_views[0]
        saw.saw_decode_step(qv, kv_new, vv_new, sl, kv, sc, tbv, lnv, d_out[0], ws,
                            dev_status=status, stream=stream)
        h_out[0].copy_(d_out[0], non_blocking=True)

    serial_ms, _ = back_to_back_ms(e2e_serial, stream, clocks, n=n_e2e, pg=pg, dev=dev)
    step()   # the device-only step on the same inputs, for the check below
    torch.cuda.synchronize()
    e2e_matches = bool(torch.equal(h_out[(n_e2e - 1) & 1], out.cpu()))
    e2e = {"value": job_throughput(wl.num_seqs, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
           "ms_per_step": e2e_ms,
           "how": "public API (saw_decode_step), one pinned host-to-device copy of the step's inputs "
                  "and one device-to-host copy of its output per step, on copy streams overlapping "
                  "the neighbouring steps' kernels (two buffer slots)",
           "output_equals_device_step": e2e_matches,
           "serial": {"value": job_throughput(wl.num_seqs, world, serial_ms), "ms_per_step": serial_ms,
                      "how": "the same two copies and step on one stream, no overlap"}}

    clocks.stop()
    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(wl)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int4 codes; f32 quantizer; f16 mma, f32 accumulate",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT, "batch": wl.num_seqs,
                   "kv_tokens_per_step": int(wl.seq_lens.sum()), "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2 (the decode reads "
                         f"{dec_bytes / 1e6:.0f} MB of INT4 cache per step > 126 MB)"},
        "kv_tokens_per_s": world * int(wl.seq_lens.sum()) / (ms_per_step / 1e3),
        "step_GBps": (dec_bytes + append_bytes(wl.num_seqs, wl.num_kv_heads)) / (ms_per_step * 1e-3) / 1e9,
        "roofline": roofline,
        "rot_quant_GBps": rq_gbs,
        "rot_quant_frac": rq_gbs / peak_gbs,
        "rot_quant_frac_of_8TBps": rq_gbs / HBM_TARGET_GBS,
        "rot_quant": rot_quant,
        "long_context": long_ctx,
        "serving": serving,
        "plain_int4": plain_int4,
        "bf16_baseline": bf16_baseline,
        "prefill_attn": prefill_attn,
        **head_dims,
        "window": window,
        "append_launch_ms": t_append,
        "e2e": e2e,
        "gpu_launches": 3 * args.steps,
        "clocks": clocks.summary(),
        "cpu_baseline": base,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def window_profile_step(wl, q, tab, lens, out, dev):
    """The windowed serving step of the bench's window line (16 sink + 112 recent bf16 tokens) on
    the decode workload: the cache and window filled from the history tokens, the step appends the
    new tokens (window append with eviction) and decodes (window part + quantized part + merge)."""
    import torch
    from bit_paged_kv_block_b200 import saw, synth
    sink, recent = 16, 112
    wkv, wtab = saw.allocate_window(wl.num_seqs, wl.num_kv_heads, sink, recent, dev)
    kv, sc = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, dev)
    kh = synth.kv_values(wl, "K", tokens="history", device=dev)
    vh = synth.kv_values(wl, "V", tokens="history", device=dev)
    seqh, posh = synth.token_index(wl, "history")
    lh = wl.seq_lens[seqh] - 1
    in_win = (posh < sink) | (posh >= np.maximum(sink, lh - recent))
    j = posh - sink
    qslot = np.where(in_win, -1, wl.block_table[seqh, np.maximum(j, 0) // 16] * 16 + j % 16)
    wslot = np.where(posh < sink, posh, sink + (posh - sink) % max(recent, 1))
    wtab_np = wtab.cpu().numpy()
    wslot = np.where(in_win, wtab_np[seqh, wslot // 16] * 16 + wslot % 16, -1)
    saw.saw_rotate_quantize_paged(kh, vh, torch.from_numpy(qslot.astype(np.int64)).to(dev), kv, sc)
    saw.saw_append_bf16_paged(kh, vh, torch.from_numpy(wslot.astype(np.int64)).to(dev), wkv)
    win = (sink, recent, wkv, wtab)
    ws = saw.allocate_window_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    k_new = synth.kv_values(wl, "K", tokens="new", device=dev)
    v_new = synth.kv_values(wl, "V", tokens="new", device=dev)
    return lambda: saw.saw_decode_step_window(q, k_new, v_new, win, kv, sc, tab, lens, out, ws)


def run_profile(args):
    """One kernel on its workload, 3 warm-up launches then 3 more, nothing else (for ncu)."""
    import torch
    from bit_paged_kv_block_b200 import saw, synth
    dev = torch.device("cuda", 0)
    if args.profile == "rot_quant":
        pre = synth.make_workload("prefill")
        kv, sc = saw.allocate_cache(pre.num_pages, pre.num_kv_heads, dev)
        seq, pos = synth.token_index(pre, "all")
        k = synth.kv_values(pre, "K", device=dev)
        v = synth.kv_values(pre, "V", device=dev)
        slots = torch.from_numpy(synth.slot_mapping(pre, seq, pos)).to(dev)
        fn = lambda: saw.saw_rotate_quantize_paged(k, v, slots, kv, sc)
    else:
        wl = synth.make_workload("decode")
        kv, sc = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, dev)
        seq, pos = synth.token_index(wl, "all")
        saw.saw_rotate_quantize_paged(synth.kv_values(wl, "K", device=dev),
                                      synth.kv_values(wl, "V", device=dev),
                                      torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(dev), kv, sc)
        q = synth.q_values(wl, device=dev)
        tab = torch.from_numpy(wl.block_table).to(dev)
        lens = torch.from_numpy(wl.seq_lens).to(dev)
        out = torch.empty((wl.num_seqs, wl.num_q_heads, 128), dtype=torch.float32, device=dev)
        ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
        fn = lambda: saw.saw_paged_decode_attn(q, kv, sc, tab, lens, out, ws)
        if args.profile == "window":
            fn = window_profile_step(wl, q, tab, lens, out, dev)
    for _ in range(6):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "launches": 6}), flush=True)
    return 0


def main():
    args = parse()
    global MIN_LAUNCHES, MIN_LOOP_SECONDS
    MIN_LAUNCHES, MIN_LOOP_SECONDS = args.loop_launches, args.loop_seconds
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return run_profile(args)
    return run_saw(args)


if __name__ == "__main__":
    sys.exit(main())
