#!/usr/bin/env python
"""Throughput of one MLA absorbed decode step on B200, as one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dsv2] [--impl ours|reference]

A step is the whole hot path over one batch: mla_absorb_query, mla_append_latent, mla_decode
(plan, attention, combine) and mla_output, on synthetic inputs of the DeepSeek-V2 attention
shape (H=128, d_h=128, r=512, d_r=64, B=64 sequences of S=8192 cached rows, paged 64-row
blocks with a permuted table). Every rank owns its own batch (weak scaling, no collective on
the data path); ``value`` is the tokens decoded by all ranks divided by the slowest rank's
device time. ``--impl reference`` times the CPU float64 oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA absorbed decode: cache TB/s (frac of HBM/MMA roofline), tokens/s, B=64 S=8k"
REF_BUDGET_S = 150.0  # whole --impl reference run
DATASHEET_HBM_GBS = 8000.0
DATASHEET_BF16_TFLOPS = 2250.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="dsv2")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-kernel", default="auto", choices=["auto", "simt", "tensor"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill", type=int, nargs=2, default=None, metavar=("B", "S"),
                    help="time mla_prefill on B prompts of S tokens at the workload's head shape")
    ap.add_argument("--fp8", action="store_true",
                    help="time a decode step over an fp8 (e4m3) latent cache of the workload")
    ap.add_argument("--front", action="store_true",
                    help="time the decode front end (mla_project) at the workload's shape")
    ap.add_argument("--context-parallel", type=int, default=0, metavar="G",
                    help="time the context-parallel split of a long-context batch into G "
                         "slices (emulated one after another on this process's GPU)")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, world: int, device="cpu"):
    """Element-wise max of a list of floats over all ranks (the slowest rank's times)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_rate(units_per_rank_step: float, world: int, steps: int, elapsed_ms: float):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank_step * world * steps / (elapsed_ms * 1e-3)


# DRAM bytes (read + write) of one attention launch, from an ncu capture of that kernel source
# on that workload, keyed by the workload and a hash of the kernel's code: when the kernel
# changes (or another workload runs), the figure does not apply and the bench reports null.
ATTEND_SOURCES = ("decode_tc.cu", "tc_ptx.cuh", "tma_map.h", "common.cuh")
ATTEND_TRAFFIC = {("dsv2", "e0cbfa00550c8757"): 644_814_080 + 8_152_832}


def attend_traffic(args):
    """The captured DRAM bytes of the tensor-core attention launch for this run, or None."""
    if args.decode_kernel == "simt":
        return None
    return ATTEND_TRAFFIC.get((args.workload, attend_source_hash()))


def attend_source_hash() -> str:
    """Hash of the attention kernel's code: comments and whitespace do not count."""
    import hashlib
    import re

    h = hashlib.sha256()
    for f in ATTEND_SOURCES:
        with open(os.path.join(ROOT, "mla_latent_kv_44_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def rank_seed(rank: int) -> int:
    """Seed of a rank's own batch: every replica decodes different sequences."""
    return rank


def workload_desc(w):
    return (f"{w.name}: H={w.num_heads} d_h={w.head_dim} r={w.kv_rank} d_r={w.rope_dim} "
            f"B={w.batch} S={w.cached if not w.ragged_max else 'U[1,%d]' % w.ragged_max} "
            f"T={w.new_tokens} {w.dtype} paged {w.block_size}-row blocks")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------------------
# SM clocks and clock-event reasons, read through NVML every 2 ms by a host thread over the
# warm-up and the timed region (read-only queries; nothing is set). nvidia-smi is the fallback.
# ---------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str, index: int, period_s: float = 0.002):
        self.uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        self.index = index
        self.period = period_s
        self.samples = []          # (time, sm_mhz, max_mhz, [reasons])
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            except pynvml.NVMLError:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            masks = [(n, getattr(pynvml, a)) for n, a in self.REASONS if hasattr(pynvml, a)]
            self.source = "nvml"
            self._thread = threading.Thread(target=self._nvml_loop, args=(pynvml, h, masks),
                                            daemon=True)
            self._thread.start()
        except Exception:  # no NVML binding or library: nvidia-smi at its fastest period
            self._start_smi()
        t_end = time.time() + 5.0
        while not self.samples and time.time() < t_end:
            time.sleep(0.01)

    def _nvml_loop(self, pynvml, h, masks):
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.time(), float(sm), float(mx),
                                     [n for n, m in masks if bits & m]))
            except Exception:
                pass
            self._stop.wait(self.period)

    def _start_smi(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.SMI_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.source = "nvidia-smi"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

        def read():
            for line in self._proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                try:
                    self.samples.append((time.time(), float(parts[0]), float(parts[1]),
                                         [n for n, v in zip(names, parts[4:8])
                                          if v.lower() == "active"]))
                except (ValueError, IndexError):
                    continue
        threading.Thread(target=read, daemon=True).start()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)
        if self._proc:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()

    def summary(self, t0, t1, label="timed region"):
        rows = [s for s in self.samples if t0 <= s[0] <= t1]
        window = label
        if not rows and self.samples:
            mid = 0.5 * (t0 + t1)
            rows = sorted(self.samples, key=lambda s: abs(s[0] - mid))[:3]
            window = "nearest samples to the timed region"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        reasons = sorted({n for s in rows for n in s[3]})
        return {"sm_mhz": statistics.median(s[1] for s in rows),
                "sm_max_mhz": max(s[2] for s in rows), "reasons": reasons,
                "samples": len(rows), "window": window, "source": self.source}


# ---------------------------------------------------------------------------------------
# the CPU oracle on a bounded sample (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------------------
def oracle_sample(w, heads: int, seed: int = 0, seq: int = 0):
    """Inputs of sequence ``seq`` restricted to the first ``heads`` heads, as the GPU stores them."""
    import numpy as np

    import mla_inputs as mi

    rows = int(mi.total_rows(w, seed)[seq])
    d = mi.sequence_draw(w, seq, rows, seed)
    wuk, wuv = mi.up_projection_weights(w, seed)
    st = lambda x: mi.storage_round(w, x)  # noqa: E731
    return (st(d.ckv_raw), st(d.krope_raw), st(d.q_nope)[:, :heads], st(d.q_rope_raw)[:, :heads],
            st(wuk)[:heads], st(wuv)[:heads], np.ones(w.kv_rank, np.float32))


def oracle_run(w, inputs):
    from oracle import mla_ref

    ckv, kr, qn, qr, wuk, wuv, gamma = inputs
    return mla_ref.decode_sequence_from_raw(ckv, kr, qn, qr, wuk, wuv, gamma, w.softmax_scale,
                                            w.rms_eps, w.rope_base, store_bf16=(w.dtype == "bf16"),
                                            form="naive")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def _absorbed_run(w, inputs):
    from oracle import mla_ref

    ckv, kr, qn, qr, wuk, wuv, gamma = inputs
    return mla_ref.decode_sequence_from_raw(ckv, kr, qn, qr, wuk, wuv, gamma, w.softmax_scale,
                                            w.rms_eps, w.rope_base, store_bf16=(w.dtype == "bf16"),
                                            form="absorbed")


def cpu_baseline(w, budget_s: float = 15.0):
    """The float64 oracle on the host's cores, three ways (input generation is not timed):

    * the naive form (K and V rebuilt per head), all heads, whole sequences one after another
      until about ``budget_s`` seconds -- the line's value;
    * the same form on one BLAS thread, on a subset of the heads of sequence 0 (scaled to all
      heads);
    * the absorbed float64 form over the whole batch (every sequence, all heads), or as many
      sequences as fit in 3 * budget_s seconds, scaled to the batch and marked extrapolated.
    """
    n, spent, rows = 0, 0.0, 0
    while n < w.batch and spent < budget_s:
        inp = oracle_sample(w, w.num_heads, seq=n)
        t0 = time.perf_counter()
        oracle_run(w, inp)
        spent += time.perf_counter() - t0
        rows += int(inp[0].shape[0])
        n += 1
    line = {"value": n * w.new_tokens / spent, "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": (f"naive float64 oracle (K and V rebuilt per head, all {w.num_heads} heads): "
                       f"sequences 0-{n - 1} of {w.name} ({rows} cached rows in all), "
                       f"{spent:.1f} s of oracle time on the host's cores; value = query tokens "
                       f"per second")}
    try:
        from threadpoolctl import threadpool_limits

        heads = max(1, w.num_heads // 16)
        inp = oracle_sample(w, heads, seq=0)
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            oracle_run(w, inp)
            dt1 = time.perf_counter() - t0
        line["naive_one_thread"] = {
            "value": w.new_tokens / (dt1 * w.num_heads / heads), "unit": "tokens/s", "cores": 1,
            "sample": f"naive float64 oracle on one BLAS thread, {heads} of {w.num_heads} heads of "
                      f"sequence 0 ({dt1:.1f} s), scaled to all heads"}
    except ImportError:
        line["naive_one_thread"] = None
    n2, spent2 = 0, 0.0
    while n2 < w.batch and spent2 < 3 * budget_s:
        inp = oracle_sample(w, w.num_heads, seq=n2)
        t0 = time.perf_counter()
        _absorbed_run(w, inp)
        spent2 += time.perf_counter() - t0
        n2 += 1
    line["absorbed_f64_batch"] = {
        "value": n2 * w.new_tokens / spent2, "unit": "tokens/s", "cores": blas_threads(),
        "sequences": n2, "of": w.batch, "extrapolated": n2 < w.batch,
        "seconds_per_batch": spent2 * w.batch / n2,
        "sample": f"absorbed float64 oracle (W_UK folded into the query), {n2} of {w.batch} "
                  f"sequences, all heads, {spent2:.1f} s on the host's cores"}
    return line


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    per_step = REF_BUDGET_S / max(1, args.steps + args.warmup)
    one = oracle_sample(w, 1)
    t0 = time.perf_counter()
    oracle_run(w, one)
    t_head = time.perf_counter() - t0
    heads = int(max(1, min(w.num_heads, per_step / max(t_head, 1e-6))))
    inp = oracle_sample(w, heads)
    for _ in range(args.warmup):
        oracle_run(w, inp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_run(w, inp)
    dt = time.perf_counter() - t0
    tokens = args.steps * w.new_tokens * heads / w.num_heads
    value = tokens / dt
    sample = (f"naive float64 oracle on {heads} of {w.num_heads} heads of one "
              f"{int(inp[0].shape[0])}-row sequence per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w), "sample": sample},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------
def attention_roofline(w, rows, attend_ms: float, peaks, traffic):
    """Roofline object of the attention kernel for one launch over ``rows`` cached rows.

    Algorithmic work per attended row and query token, all heads: the 576-value row read once
    (1152 B in bf16) and 2 * H * (576 + 512) FLOP. ``peaks`` is load_peaks()'s tuple; ``traffic``
    the captured DRAM bytes of this kernel source or None. Returns (roofline dict, algorithmic
    bytes, achieved GB/s, achieved TFLOP/s).
    """
    T = w.new_tokens
    attended = int(sum(int(n) - T + 1 + t_ for n in rows for t_ in range(T)))
    row_bytes = w.row_width * 2
    flops_row = w.num_heads * 2 * (w.row_width + w.kv_rank)
    attend_bytes = attended * row_bytes
    attend_flops = attended * flops_row
    hbm, tc_burst, _tc_sust, peak_src = peaks
    attend_s = attend_ms * 1e-3
    gbs = attend_bytes / attend_s / 1e9
    tflops = attend_flops / attend_s / 1e12
    bound = "hbm" if attend_bytes / (hbm * 1e9) >= attend_flops / (tc_burst * 1e12) else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}
    else:
        roof = {"bound": "tensor", "achieved": tflops, "peak": tc_burst, "unit": "TFLOP/s",
                "frac": tflops / tc_burst}
    roof.update({"traffic": traffic, "kernel": "mla attention (split-KV main)",
                 "traffic_note": ("DRAM read+write bytes per launch from one ncu capture of this "
                                  "kernel source (cold L2); algorithmic bytes are %d" % attend_bytes)
                 if traffic else "no ncu capture of this kernel source",
                 "algorithmic_bytes_per_launch": attend_bytes,
                 "algorithmic_flops_per_launch": attend_flops,
                 "avg_launch_us": attend_ms * 1e3, "peak_source": f"{peak_src} (MEASURED_PEAKS.json)"
                 if peak_src == "measured" else "fallback",
                 "tensor_view": {"achieved_tflops": tflops, "peak": tc_burst,
                                 "frac": tflops / tc_burst},
                 # the same achieved rates against the datasheet figures (about 8 TB/s HBM3e,
                 # 2.25 PFLOP/s dense bf16), for context
                 "frac_datasheet": {"hbm": gbs / DATASHEET_HBM_GBS,
                                    "tensor": tflops / DATASHEET_BF16_TFLOPS}})
    return roof, attend_bytes, gbs, tflops


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import mla_latent_kv_44_b200 as mla
    from mla_latent_kv_44_b200.step import DecodeState

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    kernel = {"auto": mla.DECODE_AUTO, "simt": mla.DECODE_SIMT,
              "tensor": mla.DECODE_TENSOR}[args.decode_kernel]
    st = DecodeState(w, seed=rank_seed(rank), device=str(dev), decode_kernel=kernel)
    stream = torch.cuda.Stream(device=dev)
    B, T = w.batch, w.new_tokens
    tokens_per_step = B * T

    def barrier():
        if world > 1:
            dist.barrier()

    props = torch.cuda.get_device_properties(dev)
    clock = ClockSampler(str(getattr(props, "uuid", "")), local)
    if rank == 0:
        clock.start()
    barrier()
    t_warm0 = time.time()

    # ---- warm-up ----
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            st.step_fused(stream)
    stream.synchronize()
    if int(st.dev_err.item()) != 0:
        raise RuntimeError(f"device error bits {int(st.dev_err.item())}")

    # ---- timed region: K steps of mla_decode_step, one event before and one after. Inside, the
    # kernels follow one another with programmatic dependent launch (each starts its set-up while
    # the previous one drains), which an event between them would break.
    ev_start = torch.cuda.Event(enable_timing=True)
    ev_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        ev_start.record(stream)
        for _ in range(args.steps):
            st.step_fused(stream)
        ev_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier()
    elapsed_ms = ev_start.elapsed_time(ev_end)
    if int(st.dev_err.item()) != 0:
        raise RuntimeError(f"device error bits {int(st.dev_err.item())}")

    # ---- per-kernel breakdown: a separate, shorter run of the four calls (six kernels) with an
    # event between every kernel ----
    names = ["absorb", "append", "plan", "attend", "combine", "output"]
    calls = [st.absorb, st.append, lambda s_: st.attend(s_, mla.STAGE_PLAN),
             lambda s_: st.attend(s_, mla.STAGE_ATTEND), lambda s_: st.attend(s_, mla.STAGE_COMBINE),
             st.project]
    n_detail = min(args.steps, 50)
    evd = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
           for _ in range(n_detail)]
    with torch.cuda.stream(stream):
        for k in range(n_detail):
            evd[k][0].record(stream)
            for i, fn in enumerate(calls):
                fn(stream)
                evd[k][i + 1].record(stream)
    stream.synchronize()
    stage_ms = {n: sum(evd[k][i].elapsed_time(evd[k][i + 1]) for k in range(n_detail)) / n_detail
                for i, n in enumerate(names)}
    # the attention kernel's own duration (the roofline's denominator): from this run, where an
    # event on its stream brackets every launch
    attend_only_ms = stage_ms["attend"]

    # ---- e2e through host buffers: every step uploads its inputs from pinned host memory (one
    # packed copy) and reads its output o back. Steps are pipelined over two input and two
    # output buffer sets: step k+1's upload and step k-1's download run on copy streams while
    # step k computes.
    fields = ["q_nope", "q_rope", "ckv_new", "krope_new", "seq_new", "pos_new", "seq_lens"]
    layout, total = [], 0
    for f in fields:
        t_ = getattr(st, f)
        nbytes = t_.numel() * t_.element_size()
        layout.append((f, total, nbytes, t_.dtype, tuple(t_.shape)))
        total = (total + nbytes + 255) // 256 * 256
    host_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    for f, off, nbytes, _, _ in layout:
        host_in[off:off + nbytes].copy_(getattr(st, f).contiguous().view(-1).view(torch.uint8).cpu())
    dev_sets = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    views = [{f: dev_sets[i][off:off + nbytes].view(dt).view(shape)
              for f, off, nbytes, dt, shape in layout} for i in range(2)]
    outs = [torch.empty_like(st.o) for _ in range(2)]
    host_out = [torch.empty(st.o.shape, dtype=st.o.dtype).pin_memory() for _ in range(2)]
    h2d = total
    d2h = host_out[0].numel() * host_out[0].element_size()
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    mk = lambda: [torch.cuda.Event() for _ in range(2)]
    ev_in, ev_used, ev_done, ev_read = mk(), mk(), mk(), mk()

    def upload(k):
        i = k % 2
        with torch.cuda.stream(up):
            if k >= 2:
                up.wait_event(ev_used[i])         # step k-2 finished reading this set
            dev_sets[i].copy_(host_in, non_blocking=True)
            ev_in[i].record(up)

    def run_e2e(n):
        upload(0)
        for k in range(n):
            i = k % 2
            if k + 1 < n:
                upload(k + 1)
            stream.wait_event(ev_in[i])
            if k >= 2:
                stream.wait_event(ev_read[i])     # step k-2's output has been read back
            for f in fields:
                setattr(st, f, views[i][f])
            st.o = outs[i]
            st.step_fused(stream)
            ev_used[i].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_used[i])
                host_out[i].copy_(outs[i], non_blocking=True)
                ev_read[i].record(down)
        last = [ev_read[(n - 1) % 2]] + ([ev_read[n % 2]] if n > 1 else [])
        for e_ in last:
            stream.wait_event(e_)

    e2e_steps = min(args.steps, 200)
    with torch.cuda.stream(stream):
        run_e2e(3)
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        up.wait_event(e0)
        run_e2e(e2e_steps)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    barrier()

    # ---- max over ranks ----
    elapsed_ms, e2e_ms, attend_ms = max_over_ranks([elapsed_ms, e2e_ms, attend_only_ms],
                                                   world, dev)
    if rank == 0:
        clock.stop()
    clocks = clock.summary(t_warm0, t_wall1, "warm-up and timed steps") if rank == 0 else None
    launches_per_step = st.fused_launches()
    del st
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    import mla_inputs as mi

    rows = mi.total_rows(w, 0)
    roof, attend_bytes, gbs, tflops = attention_roofline(w, rows, attend_ms, load_peaks(),
                                                         attend_traffic(args))
    # per-stage rates of the projections and the append (algorithmic bytes and FLOPs over the
    # per-kernel times of the breakdown run)
    N, H = tokens_per_step, w.num_heads
    stage_work = {
        "absorb": (H * w.head_dim * w.kv_rank * 2 + N * H * (w.head_dim + w.rope_dim) * 2 +
                   N * H * w.row_width * 2, 2 * N * H * w.head_dim * w.kv_rank),
        "append": (N * (w.row_width * 2 + w.kv_rank * 4) + N * w.row_width * 2, 0),
        "output": (H * w.head_dim_v * w.kv_rank * 2 + N * H * w.kv_rank * 4 +
                   N * H * w.head_dim_v * 2, 2 * N * H * w.head_dim_v * w.kv_rank),
    }
    stages_rate = {k: {"GB/s": b / (stage_ms[k] * 1e-3) / 1e9,
                       "GFLOP/s": f / (stage_ms[k] * 1e-3) / 1e9}
                   for k, (b, f) in stage_work.items()}
    ms_per_step = elapsed_ms / args.steps
    value = aggregate_rate(tokens_per_step, world, args.steps, elapsed_ms)
    e2e_value = aggregate_rate(tokens_per_step, world, e2e_steps, e2e_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) projections, N(0,1/r) weights; per-rank seed)",
        "config": {"workload": workload_desc(w), "batch_per_gpu": B, "global_batch": B * world,
                   "seq_len": int(rows.max()) - T, "new_tokens": T,
                   "parallelism": f"dp{world} (sequence-sharded replicas, no collective)",
                   "l2": f"inputs larger than L2: {attend_bytes / 1e9:.2f} GB of cache per step",
                   "decode_kernel": args.decode_kernel},
        "roofline": roof,
        "cache_tbs": gbs / 1e3,
        "attend_tflops": tflops,
        "stages_us": {k: v * 1e3 for k, v in stage_ms.items()},
        "stages_note": ("per-kernel times of the four separate calls, from a run with an event "
                        "after every kernel (the timed steps use mla_decode_step); "
                        "the timed steps chain the kernels with programmatic dependent launch"),
        "stages_rate": stages_rate,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
# Context-parallel split (each sequence's rows cut into G block-aligned slices, one per GPU of
# a group; every slice decoded by mla_decode, the partials all-gathered and merged by
# mla_combine_partials). With one GPU the G ranks run one after another on it: each slice's
# decode and the merge are timed with CUDA events; the exchange between GPUs is not.
# ---------------------------------------------------------------------------------------
def run_context_parallel(args):
    import numpy as np
    import torch

    import mla_inputs as mi
    import mla_latent_kv_44_b200 as mla
    from mla_latent_kv_44_b200 import context_parallel as cp
    from mla_latent_kv_44_b200.step import DecodeState

    rank, world, local = dist_env()
    if world > 1:
        if rank == 0:
            print(json.dumps({"metric": "context-parallel decode", "unavailable":
                              "the G ranks are emulated on one GPU; run without torchrun"}))
        return 0
    G = args.context_parallel
    w = mi.scaled(mi.WORKLOADS["dsv2"], batch=8, cached=32767)
    dev = torch.device("cuda", 0)
    st = DecodeState(w, device=str(dev), sequences=[])
    stream = torch.cuda.Stream(device=dev)
    B, T, H, r = w.batch, w.new_tokens, w.num_heads, w.kv_rank
    n = B * T
    with torch.cuda.stream(stream):
        st.absorb(stream)
        st.append(stream)
    plans = [cp.rank_plan(st.layout.table, st.rows, T, G, k, st.layout.block_size)
             for k in range(G)]
    tables = [torch.from_numpy(p.table).to(dev) for p in plans]
    lens = [torch.from_numpy(p.lens).to(dev) for p in plans]
    wss = [torch.empty(mla.decode_workspace_size(st.cfg, len(p.lens), p.q_per_seq),
                       dtype=torch.uint8, device=dev) for p in plans]
    parts_o = torch.empty((G, n, H, r), device=dev)
    parts_l = torch.empty((G, n, H), device=dev)

    def one_step(ev=None):
        for k, p in enumerate(plans):
            if ev is not None:
                ev[k][0].record(stream)
            mla.decode(st.cfg, st.q, st.pool, tables[k], lens[k], p.q_per_seq, wss[k],
                       parts_o[k], parts_l[k], st.dev_err, stream)
            if ev is not None:
                ev[k][1].record(stream)
        if ev is not None:
            ev[G][0].record(stream)
        mla.combine_partials(st.cfg, parts_o, parts_l, st.out_latent, st.lse, stream)
        if ev is not None:
            ev[G][1].record(stream)

    props = torch.cuda.get_device_properties(dev)
    clock = ClockSampler(str(getattr(props, "uuid", "")), 0)
    clock.start()
    t0 = time.time()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            one_step()
    stream.synchronize()
    evs = []
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(G + 1)]
            one_step(ev)
            evs.append(ev)
    stream.synchronize()
    clock.stop()
    if int(st.dev_err.item()) != 0:
        raise RuntimeError(f"device error bits {int(st.dev_err.item())}")
    per = np.array([[e[k][0].elapsed_time(e[k][1]) * 1e3 for k in range(G + 1)] for e in evs])
    slice_us = per[:, :G].mean(axis=0)
    merge_us = float(per[:, G].mean())
    step_us = float(slice_us.max()) + merge_us
    rows_total = int(np.sum(st.rows))
    print(json.dumps({
        "metric": "context-parallel decode tokens/s (slowest slice + merge; exchange excluded)",
        "value": n / (step_us * 1e-6), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"dsv2-long: H=128 r=512 d_r=64 B={B} S={int(st.rows[0])} T={T} "
                               f"bf16 paged 64-row blocks", "slices": G,
                   "emulated": "G slices one after another on one GPU"},
        "slice_us": [round(float(x), 2) for x in slice_us],
        "slice_rows": [int(np.sum(p.lens) // (1 if p.q_per_seq == T else T)) for p in plans],
        "merge_us": merge_us,
        "exchange_bytes_per_rank": n * H * (r + 1) * 4,
        "single_gpu_rows_per_step": rows_total,
        "clocks": clock.summary(t0, time.time(), "warm-up and timed steps"),
    }), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
# Decode front end (mla_project): the projections of one step's hidden states, which stream
# every front-end weight once (W_DQ, W_QR, W_DKV, W_KR from x; W_UQ from c_q).
# ---------------------------------------------------------------------------------------
def run_front(args, w):
    import numpy as np
    import torch

    import mla_inputs as mi
    import mla_latent_kv_44_b200 as mla

    rank, world, local = dist_env()
    if world > 1:
        if rank == 0:
            print(json.dumps({"metric": "decode front end", "unavailable":
                              "measured on one GPU; run without torchrun"}))
        return 0
    dev = torch.device("cuda", 0)
    n = w.batch * w.new_tokens
    d = mi.layer_draw(w, 0, x_rows=n)
    cfg = mla.Config(num_heads=w.num_heads, head_dim=w.head_dim, kv_rank=w.kv_rank,
                     rope_dim=w.rope_dim, block_size=64, dtype=w.dtype)
    tdt = cfg.torch_dtype

    def up(a):
        return None if a is None else torch.from_numpy(
            np.ascontiguousarray(mi.storage_round(w, a), dtype=np.float32)).to(dev, tdt)

    wq = d.w_dq if w.q_rank else d.w_q
    x, w_dq, w_uq, w_qr, w_dkv, w_kr = map(up, (d.x, wq, d.w_uq, d.w_qr, d.w_dkv, d.w_kr))
    gq = None if d.gamma_q is None else torch.from_numpy(d.gamma_q.astype(np.float32)).to(dev)
    H, dh, dr, r = w.num_heads, w.head_dim, w.rope_dim, w.kv_rank
    q_nope = torch.empty((n, H, dh), dtype=tdt, device=dev)
    q_rope = torch.empty((n, H, dr), dtype=tdt, device=dev)
    ckv = torch.empty((n, r), dtype=tdt, device=dev)
    kr = torch.empty((n, dr), dtype=tdt, device=dev)
    front = mla.front_config(w.d_model, w.q_rank or 0, w.rms_eps)
    ws = torch.empty(mla.project_workspace_size(cfg, front, n), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        mla.project(cfg, front, x, w_dq, gq, w_uq, w_qr, w_dkv, w_kr, q_nope, q_rope, ckv, kr,
                    ws, err, stream)

    props = torch.cuda.get_device_properties(dev)
    clock = ClockSampler(str(getattr(props, "uuid", "")), 0)
    clock.start()
    t0 = time.time()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
    stream.synchronize()
    clock.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())}")
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    esz = 2 if w.dtype == "bf16" else 4
    weights = sum(int(t.numel()) for t in (w_dq, w_uq, w_qr, w_dkv, w_kr) if t is not None)
    moved = (weights + x.numel() + q_nope.numel() + q_rope.numel() + ckv.numel() +
             kr.numel()) * esz
    flops = 2 * n * weights
    hbm, _, _, src = load_peaks()
    gbs = moved / (us * 1e-6) / 1e9
    print(json.dumps({
        "metric": "decode front end (mla_project): weight stream GB/s",
        "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": f"{args.workload} front end: d_model={w.d_model} "
                               f"q_rank={w.q_rank} H={H} d_h={dh} d_r={dr} r={r} tokens={n}",
                   "l2": "weights larger than L2 (streamed every step)"},
        "us_per_step": us, "algorithmic_bytes": moved, "algorithmic_flops": flops,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "peak_source": src},
        "gpu_launches": (4 if w.q_rank else 2) * args.steps,
        "clocks": clock.summary(t0, time.time(), "warm-up and timed steps"),
    }), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
# Prefill (mla_prefill): B prompts of S tokens, causal, in the expanded form. FLOPs counted:
# the K and V expansion (2 n r H (d_h + d_v)) and the attention over the causal half
# (2 H (d_h + d_r + d_v) per visible (query, key) pair).
# ---------------------------------------------------------------------------------------
def run_prefill(args, w):
    import torch

    import mla_latent_kv_44_b200 as mla

    rank, world, local = dist_env()
    if world > 1:
        if rank == 0:
            print(json.dumps({"metric": "prefill", "unavailable":
                              "measured on one GPU; run without torchrun"}))
        return 0
    B, S = args.prefill
    dev = torch.device("cuda", 0)
    H, dh, dr, dv, r = w.num_heads, w.head_dim, w.rope_dim, w.head_dim_v, w.kv_rank
    cfg = mla.Config(num_heads=H, head_dim=dh, kv_rank=r, rope_dim=dr, block_size=64,
                     dtype=w.dtype)
    tdt = cfg.torch_dtype
    n = B * S
    gen = torch.Generator(device=dev).manual_seed(1234)

    def draw(*shape, std=1.0):
        return (torch.randn(*shape, generator=gen, device=dev) * std).to(tdt)

    q_nope, q_rope = draw(n, H, dh), draw(n, H, dr)
    rows = draw(n, r + dr)
    w_uk, w_uv = draw(H, dh, r, std=r ** -0.5), draw(H, dv, r, std=r ** -0.5)
    pos = torch.arange(S, dtype=torch.int32, device=dev).repeat(B)
    cu = torch.arange(0, n + 1, S, dtype=torch.int32, device=dev)
    o = torch.empty((n, H, dv), dtype=tdt, device=dev)
    ws = torch.empty(mla.prefill_workspace_size(cfg, n), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        mla.prefill(cfg, q_nope, q_rope, pos, rows, w_uk, w_uv, cu, S, o, ws, err, stream)

    props = torch.cuda.get_device_properties(dev)
    clock = ClockSampler(str(getattr(props, "uuid", "")), 0)
    clock.start()
    t0 = time.time()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
    stream.synchronize()
    clock.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())}")
    ms = e0.elapsed_time(e1) / args.steps
    pairs = B * S * (S + 1) // 2
    flops = 2 * n * r * H * (dh + dv) + 2 * H * (dh + dr + dv) * pairs
    tflops = flops / (ms * 1e-3) / 1e12
    _, peak, _, src = load_peaks()
    print(json.dumps({
        "metric": "MLA prefill TFLOP/s (causal, expanded form)", "value": tflops,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "dtype": w.dtype, "data": "synthetic (seeded N(0,1))",
        "config": {"workload": f"{args.workload} heads: H={H} d_h={dh} d_r={dr} d_v={dv} "
                               f"r={r}, {B} prompts x {S} tokens"},
        "ms_per_step": ms, "tokens_per_s": n / (ms * 1e-3), "algorithmic_flops": flops,
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "peak_source": src},
        "gpu_launches": 3 * args.steps,
        "clocks": clock.summary(t0, time.time(), "warm-up and timed steps"),
    }), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
# FP8 latent cache: the workload's cache as e4m3 codes with per-row scales. A step appends the
# new rows (mla_append_latent_fp8) and decodes over the fp8 pool (mla_decode_fp8).
# ---------------------------------------------------------------------------------------
def run_fp8(args, w):
    import numpy as np
    import torch

    import mla_inputs as mi
    import mla_latent_kv_44_b200 as mla

    rank, world, local = dist_env()
    if world > 1:
        if rank == 0:
            print(json.dumps({"metric": "fp8 decode", "unavailable":
                              "measured on one GPU; run without torchrun"}))
        return 0
    dev = torch.device("cuda", 0)
    B, T, H, r, dr = w.batch, w.new_tokens, w.num_heads, w.kv_rank, w.rope_dim
    D, bs = r + dr, 64
    rows = mi.total_rows(w, 0).astype(np.int64)
    cfg = mla.Config(num_heads=H, head_dim=w.head_dim, kv_rank=r, rope_dim=dr, block_size=bs,
                     dtype=w.dtype)
    tdt = cfg.torch_dtype
    nblk = [-(-int(L) // bs) for L in rows]
    first = np.concatenate([[0], np.cumsum(nblk)])
    table = np.zeros((B, max(nblk)), dtype=np.int32)
    for b in range(B):
        table[b, :nblk[b]] = first[b] + np.arange(nblk[b])
    tab = torch.from_numpy(table).to(dev)
    pool = torch.zeros((int(first[-1]), bs, D), dtype=torch.uint8, device=dev)
    scale = torch.zeros((int(first[-1]), bs), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    gamma = torch.ones(r, device=dev)
    gen = torch.Generator(device=dev).manual_seed(99)
    # the cache: every sequence's rows appended (seeded N(0, 1) raw rows, like the bf16 bench)
    for b in range(B):
        L = int(rows[b])
        ckv = torch.randn(L, r, generator=gen, device=dev).to(tdt)
        kr = torch.randn(L, dr, generator=gen, device=dev).to(tdt)
        seq = torch.full((L,), b, dtype=torch.int32, device=dev)
        pos = torch.arange(L, dtype=torch.int32, device=dev)
        mla.append_latent_fp8(cfg, ckv, kr, gamma, seq, pos, tab, pool, scale, err)
    n = B * T
    ckv_new = torch.randn(n, r, generator=gen, device=dev).to(tdt)
    kr_new = torch.randn(n, dr, generator=gen, device=dev).to(tdt)
    seq_new = torch.arange(B, dtype=torch.int32, device=dev).repeat_interleave(T)
    pos_new = torch.from_numpy(np.concatenate([np.arange(L - T, L) for L in rows]).astype(
        np.int32)).to(dev)
    q = torch.randn(n, H, D, generator=gen, device=dev).to(tdt)
    lens = torch.from_numpy(rows.astype(np.int32)).to(dev)
    ws = torch.empty(mla.decode_fp8_workspace_size(cfg, B, T, table.shape[1]),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((n, H, r), device=dev)
    lse = torch.empty((n, H), device=dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def step():
        mla.append_latent_fp8(cfg, ckv_new, kr_new, gamma, seq_new, pos_new, tab, pool, scale,
                              err, stream)
        mla.decode_fp8(cfg, q, pool, scale, tab, lens, T, ws, out, lse, err, stream)

    props = torch.cuda.get_device_properties(dev)
    clock = ClockSampler(str(getattr(props, "uuid", "")), 0)
    clock.start()
    t0 = time.time()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
    stream.synchronize()
    clock.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())}")
    ms = e0.elapsed_time(e1) / args.steps
    cache_bytes = int(np.sum(rows)) * T * (D + 4)
    gbs = cache_bytes / (ms * 1e-3) / 1e9
    hbm, _, _, src = load_peaks()
    print(json.dumps({
        "metric": "MLA absorbed decode over an fp8 cache: tokens/s", "value": n / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "dtype": "fp8 e4m3 cache (per-row scale)",
        "data": "synthetic (seeded N(0,1) raw rows)",
        "config": {"workload": f"{args.workload}: H={H} r={r} d_r={dr} B={B} "
                               f"S={int(rows[0])} T={T}, fp8 pool of 64-row blocks"},
        "ms_per_step": ms, "cache_bytes_per_step": cache_bytes,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "peak_source": src},
        "gpu_launches": 5 * args.steps,
        "clocks": clock.summary(t0, time.time(), "warm-up and timed steps"),
    }), flush=True)
    return 0


def main():
    args = parse()
    import mla_inputs as mi

    if args.fp8:
        return run_fp8(args, mi.WORKLOADS[args.workload])
    if args.prefill:
        return run_prefill(args, mi.WORKLOADS[args.workload])
    if args.front:
        return run_front(args, mi.WORKLOADS[args.workload])
    if args.context_parallel:
        return run_context_parallel(args)
    w = mi.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
