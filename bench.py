"""Benchmark of the fused RoPE + paged-KV + ragged-attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rpk|reference]
                    [--workload NAME] [--no-workloads] [--no-backward] [--no-cpu-baseline]

One step is one pass of the whole path over one batch: rope_qk_paged_ragged
for the batch's new tokens (RoPE on Q and K, K/V written into the paged
cache) followed by ragged_paged_attention over the cache. The default
workload is the Llama-3-8B-shaped decode batch (64 sequences, 1 new token
each, cached contexts U[512, 8192], 32 q / 8 kv heads, d 128, page 64); its
metric is the K/V bytes attention reads per second.

Every run also measures the four other workloads, each on its own timed loop
of at least 200 ms of device time, reported under "workloads" with its own
roofline, RoPE + scatter bandwidth, clocks and oracle baseline: the fp32 tiny
prefill (launch-bound), the Gemma-like sliding-window decode (K/V bytes of the
window per second), the ragged causal prefill (16 sequences of U[128, 4096]
tokens) and the mixed chunked M-RoPE prefill (TFLOP/s of visible (query, key)
pairs). The attention backward on the ragged prefill workload (query, key and
value gradients from the forward's output and log-sum-exp) is reported under
"backward".

Under torchrun each rank runs its own batch (a different seed): sequences are
independent, so the path shards with no exchange (weak scaling); the time is
the max over ranks.

Prints exactly one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ragged_paged_kv_rope_b200 as R  # noqa: E402
from ragged_paged_kv_rope_b200 import metrics as M  # noqa: E402
from ragged_paged_kv_rope_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="rpk", choices=["rpk", "reference"])
    ap.add_argument("--workload", default="llama3_8b_decode", choices=sorted(W.SPECS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--no-workloads", "--no-prefill", dest="no_workloads", action="store_true",
                    help="time only the chosen workload (not the other four)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip timing the attention backward on the ragged prefill workload")
    ap.add_argument("--cache-dtype", default=None, choices=["e4m3"],
                    help="hold the KV cache as e4m3 codes with per-head scales")
    return ap.parse_args()


# ----------------------------------------------------------------- plumbing

def dist_setup(backend: str | None = None):
    """(world, rank, local_rank) from the torchrun environment; joins the
    process group when world > 1 (NCCL on GPUs, gloo where there is none)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def _reduce_device():
    if torch.distributed.is_initialized() and torch.distributed.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest value over all ranks (device times are max-reduced)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    """The sum over all ranks (units every rank processed)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch: sequences are independent, so the path
    shards across ranks with no exchange (weak scaling)."""
    return seed + 1000 * rank


def whole_job_throughput(units_this_rank: float, seconds_this_rank: float, world: int) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return sum_over_ranks(units_this_rank, world) / max_over_ranks(seconds_this_rank, world)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def strip_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines (string and character
    literals kept), so that an edit to comments alone leaves the digest as is."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def sources_digest(names) -> str:
    """SHA-256 over the given csrc files (a kernel's .cu and the headers it
    includes), comments and blank lines left out."""
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "ragged_paged_kv_rope_b200", "csrc", n)) as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()


def load_traffic(key: str):
    """Per-launch DRAM bytes of a kernel on a workload ("kernel@workload") from
    the committed ncu summary, if the kernel's sources are unchanged since the
    capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
        ent = table[key]
        if sources_digest(ent["sources"]) != ent["sha256"]:
            return None
        return ent
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs.

    The sampler is started (and seen to produce samples) before the warm-up;
    samples carry nvidia-smi's timestamp and those inside the timed window
    (widened by one sampling period on each side) are summarised. When the
    timed region is shorter than the sampling period, the nearest samples are
    used and the summary says so.
    """

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.window = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            self.out = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=self.out, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 5.0 and os.path.getsize(self.path) == 0:
                time.sleep(0.05)
        except OSError:
            self.proc = None
        return self

    def mark(self, t_begin: float, t_end: float):
        self.window = (t_begin, t_end)

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(2 * self.PERIOD_MS / 1000.0)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()

    def _rows(self):
        import datetime
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        return rows

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = self._rows()
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        note = "samples inside the timed region"
        sel = rows
        if self.window is not None:
            pad = self.PERIOD_MS / 1000.0
            a, b = self.window
            sel = [r for r in rows if a - pad <= r[0] <= b + pad]
            if not sel:
                mid = 0.5 * (a + b)
                sel = sorted(rows, key=lambda r: abs(r[0] - mid))[:3]
                note = (f"timed region ({1e3 * (b - a):.1f} ms) shorter than the sampling "
                        f"period; nearest {len(sel)} samples")
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in sel for n, v in zip(names, r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in sel),
                "sm_max_mhz": max(r[2] for r in sel), "reasons": reasons,
                "samples": len(sel), "note": note}


# ------------------------------------------------------------- the GPU path

class Step:
    """Device-resident inputs of one workload and the two C-ABI calls of a step."""

    def __init__(self, wl: W.Workload, device):
        sp = wl.spec
        self.wl, self.sp = wl, sp
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
        self.q = wl.q.to(device)
        self.k_new = wl.k_new.to(device)
        self.v_new = wl.v_new.to(device)
        self.offsets = i32(wl.q_offsets)
        self.kv_lens = i32(wl.kv_lens)
        self.position_ids = None if wl.position_ids is None else i32(wl.position_ids)
        self.error_word = torch.zeros(1, dtype=torch.int32, device=device)
        f32 = lambda a: None if a is None else torch.from_numpy(
            np.ascontiguousarray(a, dtype=np.float32)).to(device)
        self.cache = R.PagedKVCache(wl.k_pages.to(device), wl.v_pages.to(device),
                                    i32(wl.block_table), i32(wl.cache_lens), self.error_word,
                                    k_scale=f32(wl.k_scale), v_scale=f32(wl.v_scale))
        self.table = R.freqs_cis(wl.max_position, sp.rotary_dim, sp.theta, device=device)
        self.q_rot = torch.empty_like(self.q)
        self.out = torch.empty_like(self.q)
        n = R.ragged_paged_attention_workspace_size(wl.total_tokens, sp.n_heads, sp.head_dim,
                                                    sp.batch, wl.max_kv_len, sp.page_size)
        self.workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=device)

    def rope(self, stream=None):
        sp = self.sp
        R.rope_qk_paged_ragged(self.q, self.offsets, self.k_new, self.v_new, self.cache,
                               self.table, self.position_ids, sp.interleaved, sp.rotary_dim,
                               self.q_rot, mrope_section=sp.mrope_section, stream=stream)

    def attention(self, stream=None):
        sp, wl = self.sp, self.wl
        R.ragged_paged_attention(self.q_rot, self.offsets, self.kv_lens, self.cache, sp.n_heads,
                                 sp.n_kv_heads, sp.head_dim, sp.softmax_scale, sp.window,
                                 self.out, max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len,
                                 workspace=self.workspace, stream=stream)

    def launches_per_step(self) -> int:
        """Kernels of this library launched per step: RoPE, then attention
        (the decode path adds a combine kernel when a sequence can span
        several 512-key splits)."""
        sp, wl = self.sp, self.wl
        decode = wl.max_q_len * (sp.n_heads // sp.n_kv_heads) <= 16 and sp.dtype == "bf16"
        if decode:
            # the library's launch plan: one wave when the units fit, else about two
            # waves of CTAs with 8..24 tiles per split
            most = max(8, ((wl.max_kv_len + 63) // 64 + 1 + 63) // 64)
            band = wl.max_kv_len
            if sp.window > 0:
                band = min(band, sp.window + wl.max_q_len - 1)
            max_tiles = (band + 63) // 64 + 1
            units = max(1, sp.batch * sp.n_kv_heads)
            sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
            wave = sms * (2 if sp.head_dim <= 128 else 1)
            if units <= wave:
                tps = max(-(-max_tiles // (wave // units)), most)
            else:
                per_unit = max(1, -(-2 * wave // units))
                tps = -(-max_tiles // per_unit)
                tps = min(max(tps, most), max(24 if sp.head_dim <= 128 else 16, most))
            splits = -(-max_tiles // tps)
            return 2 + (1 if splits > 1 else 0)
        return 2


def time_steps(step: Step, steps: int, warmup: int, world: int, clocks=None):
    """Per-step device times of the rope call and the attention call (ms)."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        step.rope()
        step.attention()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t_begin = time.time()
    start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        step.rope()
        ev[i][1].record(stream)
        step.attention()
        ev[i][2].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.mark(t_begin, time.time())
    barrier(world)
    total_ms = start.elapsed_time(end)
    rope_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    return total_ms, rope_ms, attn_ms


def time_e2e(step: Step, steps: int, warmup: int, world: int):
    """Same step through the public API with host inputs: pinned host -> device
    copies of the step's inputs, the two calls, device -> host copy of the
    output, all inside the timed region."""
    wl = step.wl
    host = {
        "q": wl.q.pin_memory(), "k_new": wl.k_new.pin_memory(), "v_new": wl.v_new.pin_memory(),
        "offsets": torch.from_numpy(wl.q_offsets).pin_memory(),
        "kv_lens": torch.from_numpy(wl.kv_lens).pin_memory(),
        "cache_lens": torch.from_numpy(wl.cache_lens).pin_memory(),
        "block_table": torch.from_numpy(wl.block_table).pin_memory(),
    }
    if wl.position_ids is not None:
        host["position_ids"] = torch.from_numpy(wl.position_ids).pin_memory()
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    dst = {"q": step.q, "k_new": step.k_new, "v_new": step.v_new, "offsets": step.offsets,
           "kv_lens": step.kv_lens, "cache_lens": step.cache.cache_lens,
           "block_table": step.cache.block_table}
    if step.position_ids is not None:
        dst["position_ids"] = step.position_ids
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()
    stream = torch.cuda.current_stream()

    def one():
        for k, t in host.items():
            dst[k].copy_(t, non_blocking=True)
        step.rope()
        step.attention()
        out_host.copy_(step.out, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return a.elapsed_time(b) / steps, h2d, d2h


def steps_for(ms_one: float, min_ms: float = 200.0, lo: int = 5, hi: int = 20000) -> int:
    """Loop count whose timed region lasts at least min_ms of device time."""
    return int(min(hi, max(lo, math.ceil(min_ms / max(ms_one, 1e-3)))))


def one_step_ms(step: "Step") -> float:
    """Device time of one warm step (RoPE + attention), to size a timed loop."""
    stream = torch.cuda.current_stream()
    for _ in range(2):
        step.rope()
        step.attention()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    step.rope()
    step.attention()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def kernel_of(wl: W.Workload) -> tuple[str, str]:
    """(traffic key prefix, description) of the kernel the attention call runs."""
    sp = wl.spec
    if sp.dtype != "bf16":
        return "attn_simt", "ragged_paged_attention (CUDA-core fp32 kernel)"
    if is_decode(wl):
        return "attn_decode", "ragged_paged_attention (split-KV decode + combine)"
    if sp.n_heads // sp.n_kv_heads <= 128:
        if sp.cache_dtype is None and sp.head_dim in (64, 128, 256):
            return "attn_prefill", "ragged_paged_attention (tcgen05 prefill)"
        if sp.cache_dtype == "e4m3" and sp.head_dim in (64, 128):
            return ("attn_prefill_e4m3",
                    "ragged_paged_attention (tcgen05 prefill, e4m3 codes widened to f16 on chip)")
    return "attn_simt", "ragged_paged_attention (CUDA-core kernel)"


def measure_workload(name: str, device, world: int, local: int, rank: int, seed: int,
                     cpu_s: float | None):
    """One workload measured on its own: a timed loop of at least 200 ms of
    device time (RoPE + attention per step, CUDA events on the launching
    stream), its attention roofline, its RoPE + scatter bandwidth, the clocks
    sampled during its timed loop and the oracle on a bounded sample."""
    wl = W.make(name, seed=rank_seed(seed, rank))
    sp = wl.spec
    step = Step(wl, device)
    metric, unit, amount, scale = metric_of(wl)
    n = steps_for(one_step_ms(step))
    with ClockSampler(local) as clocks:
        total_ms, rope_ms, attn_ms = time_steps(step, n, 3, world, clocks)
    clk = clocks.summary()
    step_ms = max_over_ranks(total_ms / n, world)
    attn = max_over_ranks(statistics.mean(attn_ms), world)
    rope = max_over_ranks(statistics.mean(rope_ms), world)
    peaks = load_peaks()
    key, kdesc = kernel_of(wl)
    achieved = amount / (attn * 1e-3) / scale
    traffic = load_traffic(f"{key}@{name}")
    if sp.dtype != "bf16":
        roofline = {"bound": "launch", "kernel": kdesc, "achieved": achieved, "unit": unit,
                    "note": "fp32 correctness workload of a few hundred kFLOP: the step is "
                            "launch latency, no roofline applies"}
    elif is_decode(wl):
        roofline = {"bound": "hbm", "kernel": kdesc, "achieved": achieved,
                    "peak": peaks["hbm_gbs"], "unit": unit, "frac": achieved / peaks["hbm_gbs"],
                    "traffic": None if traffic is None else traffic["bytes_per_launch"],
                    "algorithmic_bytes_per_launch": amount,
                    "peak_source": f"{peaks['source']} hbm_gbs"}
    else:
        roofline = {"bound": "tensor", "kernel": kdesc, "achieved": achieved,
                    "peak": peaks["bf16_tflops"], "unit": unit,
                    "frac": achieved / peaks["bf16_tflops"],
                    "traffic": None if traffic is None else traffic["bytes_per_launch"],
                    "algorithmic_flops_per_launch": amount,
                    "peak_source": f"{peaks['source']} bf16_tflops (burst: kernel timed alone)"}
    elt = 4 if sp.dtype == "f32" else 2
    rope_b = M.rope_bytes(wl.total_tokens, sp.n_heads, sp.n_kv_heads, sp.head_dim,
                          sp.rotary_dim, elt)
    rope_traffic = load_traffic(f"rope@{name}")
    rope_gbs = rope_b / (rope * 1e-3) / 1e9
    entry = {
        "metric": metric, "value": sum_over_ranks(amount, world) / (step_ms * 1e-3) / scale,
        "unit": unit, "steps": n, "warmup": 3, "ms_per_step": step_ms,
        "description": sp.description, "new_tokens_per_step": wl.total_tokens,
        "tokens_per_s": sum_over_ranks(wl.total_tokens, world) / (step_ms * 1e-3),
        "breakdown_ms": {"rope_qk_paged_ragged": rope, "ragged_paged_attention": attn},
        "roofline": roofline,
        "rope_roofline": {"bound": "hbm", "kernel": "rope_scatter_kernel", "achieved": rope_gbs,
                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": rope_gbs / peaks["hbm_gbs"],
                          "traffic": None if rope_traffic is None
                          else rope_traffic["bytes_per_launch"],
                          "algorithmic_bytes_per_launch": rope_b},
        "clocks": clk,
        "gpu_launches": step.launches_per_step() * n,
        "error_word": int(step.error_word.item()),
        "l2": "inputs larger than L2" if (wl.k_pages.numel() * wl.k_pages.element_size() * 2
                                          + wl.q.numel() * wl.q.element_size() * 3
                                          > L2_BYTES) else "inputs fit in L2 (launch-bound case)",
    }
    if cpu_s is not None and rank == 0 and world == 1:
        entry["cpu_baseline"] = cpu_baseline(wl, unit, scale, budget_s=cpu_s,
                                             per_pass_s=cpu_s / 2)
    del step
    torch.cuda.empty_cache()
    return entry


def backward_measure(device, world, warmup=3, batch=None):
    """The attention backward (its two kernels) on the ragged prefill workload:
    the forward runs once for the output and log-sum-exp, then the backward is
    timed with a seeded N(0, 1) output gradient. Algorithmic FLOPs are 2.5x the
    forward's visible-pair FLOPs: five products of 2 d FLOP per visible (row,
    key) pair and head (S, dP, dQ, dK, dV); the kernels recompute S and dP in
    each of their two passes, which is not counted."""
    wl = W.make("ragged_prefill", seed=0, **({} if batch is None else {"batch": batch}))
    sp = wl.spec
    step = Step(wl, device)
    step.rope()
    T, H, d = wl.q.shape
    lse = torch.empty((T, H), dtype=torch.float32, device=device)
    R.ragged_paged_attention(step.q_rot, step.offsets, step.kv_lens, step.cache, sp.n_heads,
                             sp.n_kv_heads, sp.head_dim, sp.softmax_scale, sp.window, step.out,
                             max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len,
                             workspace=step.workspace, log_sum_exp=lse)
    gen = torch.Generator().manual_seed(1)
    d_out = torch.randn((T, H, d), generator=gen).to(step.q.dtype).to(device)
    d_q = torch.empty((T, H, d), dtype=torch.float32, device=device)
    d_k = torch.zeros(tuple(step.cache.k_pages.shape), dtype=torch.float32, device=device)
    d_v = torch.zeros_like(d_k)

    def run():
        R.ragged_paged_attention_backward(step.q_rot, step.offsets, step.kv_lens, step.cache,
                                          sp.n_heads, sp.n_kv_heads, sp.head_dim,
                                          sp.softmax_scale, sp.window, step.out, d_out, lse,
                                          d_q, d_k, d_v, max_q_len=wl.max_q_len,
                                          max_kv_len=wl.max_kv_len)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    run()
    b.record()
    torch.cuda.synchronize()
    steps = steps_for(a.elapsed_time(b))
    barrier(world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        a.record()
        run()
        b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    flops = 2.5 * M.attention_flops(wl.q_lens, wl.kv_lens, sp.window, sp.n_heads, sp.head_dim)
    peaks = load_peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    G = sp.n_heads // sp.n_kv_heads
    if sp.dtype == "bf16" and sp.cache_dtype is None and sp.head_dim in (64, 128) and G <= 128:
        kernel = "tcgen05 dK/dV and dQ kernels (attn_bwd_dkv_tc_kernel, attn_bwd_dq_tc_kernel)"
    elif sp.dtype == "bf16" and sp.cache_dtype is None and G <= 16:
        kernel = "warp-level tensor-core (mma.sync) dQ and dK/dV kernels"
    else:
        kernel = "CUDA-core dQ and dK/dV kernels"
    # DRAM bytes per launch of the two tcgen05 kernels (committed small-case
    # captures scaled to this workload) beside the bytes of their inputs.
    kv_tokens = int(np.sum(wl.kv_lens))
    inputs = {"q_and_d_out": 2 * T * H * d * 2,
              "k_and_v": 2 * kv_tokens * sp.n_kv_heads * d * 2,
              "lse_and_delta": 2 * T * H * 4}
    traffic = {}
    for key in ("attn_bwd_dkv", "attn_bwd_dq"):
        ent = load_traffic(f"{key}@ragged_prefill") if batch is None else None
        traffic[key] = None if ent is None else ent["bytes_per_launch"]
    return {"workload": "ragged_prefill", "kernel": kernel, "backward_ms": ms, "steps": steps,
            "algorithmic_flops": flops, "tflops": tflops,
            "tensor_peak_tflops": peaks["bf16_tflops"], "frac": tflops / peaks["bf16_tflops"],
            "traffic": traffic, "input_bytes": inputs,
            "error_word": int(step.error_word.item())}


# ------------------------------------------------------------ the metric

def is_decode(wl: W.Workload) -> bool:
    """True when the attention call takes the split-KV decode path (bf16, at
    most 16 (token, query head) rows per KV head and sequence)."""
    sp = wl.spec
    return sp.dtype == "bf16" and int(wl.q_lens.max()) * (sp.n_heads // sp.n_kv_heads) <= 16


def cache_elt(wl: W.Workload) -> int:
    """Bytes per cached K or V element: 1 for an e4m3 cache, else q's element size."""
    if wl.spec.cache_dtype == "e4m3":
        return 1
    return 2 if wl.spec.dtype == "bf16" else 4


def metric_of(wl: W.Workload):
    """(metric, unit, amount per step, scale to the unit) of a workload: K/V
    bytes read for decode (GB/s, HBM-bound), visible-pair FLOPs for prefill
    (TFLOP/s, tensor-bound)."""
    sp = wl.spec
    if is_decode(wl):
        elt = cache_elt(wl)
        return ("decode_attention_kv_GBps", "GB/s",
                M.attention_kv_bytes(wl.q_lens, wl.kv_lens, sp.window, sp.n_kv_heads,
                                     sp.head_dim, elt), 1e9)
    return ("prefill_attention_TFLOPs", "TFLOP/s",
            M.attention_flops(wl.q_lens, wl.kv_lens, sp.window, sp.n_heads, sp.head_dim), 1e12)


# -------------------------------------------------------- the oracle on CPU

def _row_visible(wl: W.Workload, b: int) -> np.ndarray:
    """Visible keys of each row (token) of sequence b under the workload's band."""
    sp = wl.spec
    lo, hi = M._bands(int(wl.q_lens[b]), int(wl.kv_lens[b]), sp.window)
    return np.maximum(hi - lo + 1, 0)


def oracle_sample_time(wl: W.Workload, max_seconds: float = 20.0, chunk_tokens: int = 128):
    """Time the fp64 oracle (RoPE, cache image, attention) on a bounded sample
    of the workload; returns (seconds, amount, tokens, sample, threads), amount
    in the workload's unit (K/V bytes or visible-pair FLOPs).

    RoPE and the cache image run over the whole batch and are charged in
    proportion to the rows sampled. Attention runs sequence by sequence, all
    query heads of `chunk_tokens` tokens at a time, until the time budget is
    used: a decode sequence counts its K/V bytes once all its rows are done,
    a prefill chunk counts 4 d FLOPs per visible (row, key) pair."""
    import oracle as O
    sp = wl.spec
    table = O.freqs_cis(wl.max_position, sp.rotary_dim, sp.theta)
    kp, code = O.oracle._raw(wl.k_pages)
    vp, _ = O.oracle._raw(wl.v_pages)
    kp, vp = kp.copy(), vp.copy()
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    args = (wl.q_offsets, wl.cache_lens, wl.position_ids, sp.mrope_section, table,
            sp.interleaved, sp.rotary_dim)
    q_rot = O.rope(wl.q, *args)
    k_rot = O.rope(wl.k_new, *args)
    O.cache_image(k_rot, wl.v_new, wl.q_offsets, wl.cache_lens, wl.block_table, kp, vp,
                  inplace=True)
    qr = O.round_to(q_rot, code)
    t_rope = time.perf_counter() - t0
    decode = is_decode(wl)
    elt = cache_elt(wl)
    H = sp.n_heads
    done_seq, done_tok, amount = 0, 0, 0
    t1 = time.perf_counter()
    out_of_time = False
    for b in range(sp.batch):
        lo, hi = int(wl.q_offsets[b]), int(wl.q_offsets[b + 1])
        vis = _row_visible(wl, b)
        step = (hi - lo) if decode else chunk_tokens
        for t0_ in range(lo, hi, max(1, step)):
            t1_ = min(hi, t0_ + max(1, step))
            rows = np.array([[t, h] for t in range(t0_, t1_) for h in range(H)], np.int32)
            O.attention(qr, wl.q_offsets, wl.kv_lens, kp, vp, wl.block_table, sp.n_kv_heads,
                        sp.softmax_scale, sp.window, rows=rows, n_threads=threads)
            done_tok += t1_ - t0_
            if not decode:
                amount += 4 * H * sp.head_dim * int(vis[t0_ - lo:t1_ - lo].sum())
            if time.perf_counter() - t1 > max_seconds:
                out_of_time = True
                break
        if decode and not out_of_time:
            amount += M.attention_kv_bytes(wl.q_lens[b:b + 1], wl.kv_lens[b:b + 1], sp.window,
                                           sp.n_kv_heads, sp.head_dim, elt)
            done_seq += 1
        if out_of_time:
            break
    t_attn = time.perf_counter() - t1
    share = done_tok / max(1, wl.total_tokens)
    seconds = t_attn + t_rope * share
    if decode:
        sample = f"{done_seq} of {sp.batch} sequences (all rows), RoPE + cache image + attention"
    else:
        sample = (f"{done_tok} of {wl.total_tokens} query tokens (all heads, the first "
                  f"sequences in order), RoPE + cache image + attention")
    return seconds, amount, done_tok, sample, threads


def cpu_baseline(wl: W.Workload, unit: str, scale: float, budget_s: float, per_pass_s: float):
    """Whole passes of the oracle over a bounded sample, about budget_s seconds."""
    total_s, total_amount, passes, t_all = 0.0, 0, 0, time.perf_counter()
    while passes < 1 or (time.perf_counter() - t_all < budget_s and passes < 50):
        secs, amount, toks, sample, threads = oracle_sample_time(wl, max_seconds=per_pass_s)
        total_s += secs
        total_amount += amount
        passes += 1
    return {"value": total_amount / total_s / scale, "unit": unit, "cores": threads,
            "kind": "oracle", "sample": f"{sample}; {passes} passes", "seconds": total_s}


# --------------------------------------------------------------------- main

def main():
    args = parse()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return reference_arm(args, world, rank)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    over = {} if args.batch is None else {"batch": args.batch}
    if args.cache_dtype:
        over["cache_dtype"] = args.cache_dtype
    wl = W.make(args.workload, seed=rank_seed(args.seed, rank), **over)
    sp = wl.spec
    step = Step(wl, device)
    elt = cache_elt(wl)
    kv_bytes = M.attention_kv_bytes(wl.q_lens, wl.kv_lens, sp.window, sp.n_kv_heads,
                                    sp.head_dim, elt)
    metric, unit, amount, scale = metric_of(wl)
    decode = is_decode(wl)
    with ClockSampler(local) as clocks:
        total_ms, rope_ms, attn_ms = time_steps(step, args.steps, args.warmup, world, clocks)
    clk = clocks.summary()
    step_ms = max_over_ranks(total_ms / args.steps, world)
    job_amount = sum_over_ranks(amount, world)
    job_tokens = sum_over_ranks(wl.total_tokens, world)
    attn_ms_mean = max_over_ranks(statistics.mean(attn_ms), world)
    rope_ms_mean = max_over_ranks(statistics.mean(rope_ms), world)
    err = int(step.error_word.item())
    peaks = load_peaks()
    value = job_amount / (step_ms * 1e-3) / scale
    achieved = amount / (attn_ms_mean * 1e-3) / scale
    key, kdesc = kernel_of(wl)
    if decode and sp.cache_dtype is not None:
        key = f"{key}_{sp.cache_dtype}"
    traffic = load_traffic(f"{key}@{sp.name}")
    if decode:
        roofline = {"bound": "hbm", "kernel": kdesc,
                    "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": unit,
                    "frac": achieved / peaks["hbm_gbs"],
                    "traffic": None if traffic is None else traffic["bytes_per_launch"],
                    "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)"
                    if peaks["source"] == "measured" else "fallback 6.65 TB/s",
                    "algorithmic_bytes_per_launch": kv_bytes}
    else:
        roofline = {"bound": "tensor", "kernel": kdesc, "achieved": achieved,
                    "peak": peaks["bf16_tflops"], "unit": unit,
                    "frac": achieved / peaks["bf16_tflops"],
                    "traffic": None if traffic is None else traffic["bytes_per_launch"],
                    "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops)"
                    if peaks["source"] == "measured" else "fallback 1.59 PFLOP/s",
                    "algorithmic_flops_per_launch": amount}

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = time_e2e(step, max(3, args.steps // 2), 2, world)
        e2e_ms = max_over_ranks(e2e_ms, world)
        e2e = {"value": job_amount / (e2e_ms * 1e-3) / scale, "unit": unit,
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": "pinned host inputs copied in, output copied out, inside the timed region"}

    launches = step.launches_per_step() * args.steps
    del step
    torch.cuda.empty_cache()
    workloads = {}
    if not args.no_workloads:
        # every other workload, each measured on its own timed loop
        for name in ("tiny_prefill_f32", "gemma_swa_decode", "ragged_prefill",
                     "mixed_chunked_mrope"):
            if name == args.workload:
                continue
            workloads[name] = measure_workload(
                name, device, world, local, rank, args.seed,
                None if args.no_cpu_baseline else 4.0)
    backward = None if args.no_backward else backward_measure(
        device, world, batch=args.batch if args.workload == "ragged_prefill" else None)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # whole passes of the oracle over (a bounded sample of) the batch, ~10-30 s in all
        cpu = cpu_baseline(wl, unit, scale, budget_s=10.0, per_pass_s=20.0)

    line = {
        "metric": metric, "value": value, "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": sp.dtype,
        "data": "synthetic (seeded N(0,1) values, shuffled page tables)",
        "config": {"workload": sp.name, "description": sp.description,
                   "cache_dtype": sp.cache_dtype or sp.dtype,
                   "batch_per_gpu": sp.batch, "new_tokens_per_step": wl.total_tokens,
                   "kv_bytes_per_step": kv_bytes,
                   "l2": f"inputs larger than L2: {kv_bytes / 1e9:.2f} GB of K/V per step "
                         f"vs {L2_BYTES / 2**20:.0f} MiB L2",
                   "parallelism": f"replicas x{world} (independent sequences, no exchange)"},
        "tokens_per_s": job_tokens / (step_ms * 1e-3),
        "breakdown_ms": {"rope_qk_paged_ragged": rope_ms_mean,
                         "ragged_paged_attention": attn_ms_mean},
        "roofline": roofline,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches,
        "error_word": err,
        "workloads": workloads,
        "backward": backward,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


def reference_arm(args, world, rank):
    """The fp64 oracle timed on the host cores, as the reference arm."""
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    over = {} if args.batch is None else {"batch": args.batch}
    if args.cache_dtype:
        over["cache_dtype"] = args.cache_dtype
    wl = W.make(args.workload, seed=args.seed, **over)
    sp = wl.spec
    metric, unit, _, scale = metric_of(wl)
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_sample_time(wl, max_seconds=2.0)
    times, vals = [], []
    budget = max(2.0, 120.0 / max(1, args.steps))
    for _ in range(args.steps):
        secs, kvb, toks, sample, threads = oracle_sample_time(wl, max_seconds=budget)
        times.append(secs)
        vals.append(kvb / secs / scale)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) values, shuffled page tables)",
        "config": {"workload": sp.name, "description": sp.description},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
