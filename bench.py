#!/usr/bin/env python
"""Bench: MLA paged decode on B200 -- µs per decode step and effective KV GB/s.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                [--op decode|prefill|kv_pack] [--batch B]

One step = one decode call (split-KV partial kernel + combine kernel) over a
resident synthetic workload (default: FP8 E4M3 cache, q_len 4, 32 heads,
81,920 keys, batch 16). After W warm-up steps, exactly K steps are timed, each
bracketed by CUDA events on the launching stream, with the SM clock read
through NVML during them. The same K steps are then timed again after a
loaded window (--clock-window-s seconds of back-to-back steps, which bring the
clocks to those of continuous decoding under the power cap) and reported
beside them as "sustained". The roofline is the partial kernel's: the same
protocol on partial-only calls (no combine) gives its average launch duration.
When the cache pool is smaller than twice the L2,
a 256 MiB buffer is rewritten between steps; otherwise the inputs are larger
than L2 and nothing is flushed. With N > 1 (torchrun) every rank runs an
independent replica on its own GPU ("replicas only": the decode has no
exchange step); the time is the max over ranks and the value the KV bytes of
all ranks over that time.

--op prefill times a ragged prefill step (TFLOP/s) and --op kv_pack the fused
K/V pack + FP8 quantise (GB/s), with the same JSON keys. --batch draws a
smaller case of a workload (for profiler captures).

--impl reference times the fp64 CPU oracle (no other implementation of this
path is available to run) on the host cores, one bounded sample of the
workload per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = (1590.0, 1400.0)  # burst, sustained under the power cap
PUBLISHED_US = {"fp8_long_b4": 49.5, "fp8_long_b16": 148.1}  # TokenSpeed, article section 二


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="fp8_long_b16")
    ap.add_argument("--op", default="decode", choices=["decode", "kv_pack", "prefill"],
                    help="decode (the headline) or the fused K/V pack + FP8 quantise kernel")
    ap.add_argument("--kernel", default="auto", choices=["auto", "tcgen05", "simt", "tcgen05_solo"])
    ap.add_argument("--batch", type=int, default=0,
                    help="draw the workload with this many entries instead (small cases for ncu captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--warm-l2", action="store_true",
                    help="never flush L2 between steps (a warm-L2 line for the workloads whose pool fits in L2)")
    ap.add_argument("--clock-window-s", type=float, default=1.5,
                    help="seconds of back-to-back steps before the sustained timing (0: no sustained timing)")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world, dev, backend="nccl", timeout_s=180):
    """One process per GPU (replicas): a process group only for the barrier and the timing
    reduction; nothing on the data path crosses ranks."""
    if world > 1:
        import torch.distributed as dist
        kw = {"device_id": dev} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def max_over_ranks(x, world, dev):
    """The largest of the ranks' values (every rank gets it); x itself on one rank."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- helpers

def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak(dtype, sustained=True):
    """Dense tensor peak in TFLOP/s for the MMA input type: the measured cuBLAS BF16 figure
    (sustained: the seconds-long loop under the power cap), x 2 for FP8 (nominal 4.5 / 2.25)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        bf16, kind = float(d["bf16_tflops_sustained" if sustained else "bf16_tflops"]), "measured"
    except Exception:
        bf16, kind = FALLBACK_BF16_TFLOPS[1 if sustained else 0], "fallback"
    ratio = 2.0 if dtype == "fp8" else 1.0
    src = f"{kind} bf16 {'sustained' if sustained else 'burst'}" + (" x 2 (fp8/bf16 nominal)" if ratio != 1 else "")
    return bf16 * ratio, src


def algorithmic_flops(seq_lens, q_len, heads):
    """2 * (576 + 512) flops per (query row, visible key): S = q.K^T over 576 dims and O += p.V
    over 512; row t of an entry with n keys sees n - q_len + t + 1 of them."""
    from mla_paged_decode_04_b200.inputs import D_QK, D_V
    total = 0
    for n in seq_lens:
        for t in range(q_len):
            total += max(0, int(n) - q_len + t + 1)
    return total * heads * 2 * (D_QK + D_V)


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_paged_decode_04_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h", ".cpp")):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload, kernel_name):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(workload, {}).get(kernel_name)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed work runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        self.device_index = device_index

    def start(self):
        try:
            import torch
            sel = []
            try:
                uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
                sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
            except Exception:
                sel = []
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        try:
            rows = [l.strip().split(", ") for l in open(self.path) if l.strip()]
            os.unlink(self.path)
        except Exception:
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


class NvmlClockPoller:
    """SM clock and clock-event reasons read through NVML about every 0.5 ms from a host thread,
    so that a timed region of a few milliseconds still gets samples (nvidia-smi's loop samples
    every 100 ms at best). Read-only: nothing is set. window(t0, t1) summarises the samples
    taken between two host perf_counter() times."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index):
        import threading
        self.samples = []  # (perf_counter, sm_mhz, reason bits)
        self.ok = False
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.nv = pynvml
            self.bits = {name: getattr(pynvml, attr, 0) for name, attr in self.REASONS}
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.perf_counter(), float(mhz), int(rs)))
            except Exception:
                pass
            time.sleep(0.0005)

    def start(self):
        if self.ok:
            import threading
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def window(self, t0, t1):
        sel = [s for s in self.samples if t0 <= s[0] <= t1]
        if not sel:
            return None
        reasons = sorted({name for _, _, rs in sel for name, bit in self.bits.items() if bit and rs & bit})
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sel), "source": "nvml, ~0.5 ms polling during the timed steps",
                "caveat": "NVML's SM clock lags power capping over regions of a few ms; inside the kernels "
                          "(clock64 against globaltimer) back-to-back calls run below it"}


def roofline_fields(alg_bytes, flops, seconds, hbm_peak, hbm_kind, dtype, sustained):
    """Roofline of one partial-kernel launch of `seconds`: the HBM side (algorithmic bytes at the
    measured copy bandwidth) and the tensor side (algorithmic flops at the measured cuBLAS peak,
    burst or sustained), `bound` being the side with the higher floor. hbm_frac is always given:
    decode reads the KV cache once, so HBM is the yardstick of the workloads the cache dominates."""
    tpeak, tkind = measured_tensor_peak(dtype, sustained=sustained)
    t_hbm = alg_bytes / (hbm_peak * 1e9)
    t_tensor = flops / (tpeak * 1e12)
    hbm_ach = alg_bytes / seconds / 1e9
    ten_ach = flops / seconds / 1e12
    hbm = {"bound": "hbm", "achieved": round(hbm_ach, 1), "peak": hbm_peak, "unit": "GB/s",
           "frac": round(hbm_ach / hbm_peak, 4), "peak_source": f"{hbm_kind} (of measured copy bandwidth)"
           if hbm_kind == "measured" else hbm_kind, "floor_us": round(t_hbm * 1e6, 2)}
    ten = {"bound": "tensor", "achieved": round(ten_ach, 1), "peak": round(tpeak, 1), "unit": "TFLOP/s",
           "frac": round(ten_ach / tpeak, 4), "peak_source": tkind, "floor_us": round(t_tensor * 1e6, 2)}
    bind, other = (ten, hbm) if t_tensor > t_hbm else (hbm, ten)
    out = dict(bind)
    out.update({"hbm_frac": hbm["frac"], "tensor_frac": ten["frac"], "tensor_peak": ten["peak"], "other": other})
    return out


# ---------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    import mla_paged_decode_04_b200 as mla
    from mla_paged_decode_04_b200.inputs import D_QK, D_V, WORKLOADS, make_inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, dev)

    w = WORKLOADS[args.workload]
    inp = make_inputs(args.workload, device=dev, batch=args.batch or None)
    g = inp.to(dev)
    B, T, H = g.batch, g.q_len, g.heads
    dec = mla.MlaDecoder(B, T, H, g.max_seq_len, g.dtype, dev, kernel=args.kernel)
    plan = dec.plan
    out = torch.empty((B, T, H, D_V), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    # L2 between steps: a cache pool at least twice the 126 MB L2 already
    # streams the previous step's pages out, so it is not flushed (a written
    # flush buffer would leave ~126 MB of dirty lines for the kernel to write
    # back); a smaller pool is flushed by rewriting a 256 MB buffer.
    L2_BYTES = 126 << 20
    pool_bytes = g.kv_cache.numel() * g.kv_cache.element_size()
    flush_l2 = pool_bytes < 2 * L2_BYTES and not args.warm_l2
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush_l2 else None

    class _Flush:
        def zero_(self):
            if flush_buf is not None:
                flush_buf.zero_()

    flush = _Flush()
    esize = 1 if g.dtype == "fp8" else 2
    kv_tokens = int(inp.seq_lens.clamp(min=0).sum())
    kv_bytes = kv_tokens * D_QK * esize
    q_bytes = g.q.numel() * esize
    table_bytes = sum((int(n) + 63) // 64 for n in inp.seq_lens.tolist()) * 4 + B * 4
    out_bytes = out.numel() * 2 + lse.numel() * 4
    alg_bytes_step = kv_bytes + q_bytes + table_bytes + out_bytes
    alg_bytes_partial = kv_bytes + q_bytes + table_bytes + (out_bytes if plan.split_kv == 1 else 0)
    call = (g.q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale, out, lse, dec.workspace,
            g.q_scale, g.kv_scale)
    # balanced schedule (plan.schedule == MLA_SCHEDULE_BALANCED = 1): the workspace-clear kernel, the
    # partial kernel and the combine; otherwise a memset (not one of ours), the partial kernel and,
    # with splits, the combine
    kernels_per_step = 3 if plan.schedule == 1 else 1 + (1 if plan.split_kv > 1 else 0)

    def step():
        # one call: the combine is launched as the partial kernel's dependent
        mla.mla_decode(plan, *call)

    poller = NvmlClockPoller(local)
    poller.start()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if dec.status() != 0:
        raise RuntimeError("device status word set during warm-up")

    def timed(fn, n, per_step=False):
        """n steps back to back, timed by CUDA events on the launching stream: one pair around
        all n steps (an event recorded between two steps widens the gap between them; used when
        nothing runs between steps), or, with per_step, a pair around each step (the L2 flush,
        when there is one, runs between the pairs). Returns the per-step times in ms (the mean
        n times without per_step) and the host time window the steps ran in."""
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        if per_step:
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
            for k in range(n):
                flush.zero_()
                evs[k][0].record()
                fn()
                evs[k][1].record()
        else:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for k in range(n):
                fn()
            e1.record()
        torch.cuda.synchronize()
        h1 = time.perf_counter()
        if world > 1:
            dist.barrier()
        if per_step:
            return [a.elapsed_time(b) for a, b in evs], h0, h1
        return [e0.elapsed_time(e1) / n] * n, h0, h1

    def partial_only():
        # the partial kernel alone (after its workspace clear), without the combine
        mla.mla_decode_partial(plan, *call)

    def partial_ms():
        """Average launch duration of the partial kernel: the timed steps' protocol applied to
        partial-only calls (K back to back under one event pair, or with the L2 flushed between
        calls an event pair around each)."""
        ms, _, _ = timed(partial_only, args.steps, per_step=flush_l2)
        return ms

    # (1) the timed steps: W warm-up steps above, then exactly K steps (an event pair around each
    # when the L2 is flushed between steps, so that the flush stays outside the timed region)
    step_ms, wall0, wall1 = timed(step, args.steps, per_step=flush_l2)
    clocks = poller.window(wall0, wall1)
    # the same K steps with an event pair around each, for the spread only
    each_ms, _, _ = timed(step, args.steps, per_step=True)
    part_ms = partial_ms()
    if dec.status() != 0:
        raise RuntimeError("device status word set during the timed steps")

    # (2) the same K steps after a loaded window (continuous decoding: the clocks settle under
    # the power cap), reported beside the timed steps
    sustained = None
    if args.clock_window_s > 0:
        sampler = ClockSampler(local)
        sampler.start()
        t_end = time.perf_counter() + args.clock_window_s
        while time.perf_counter() < t_end:
            for _ in range(20):
                flush.zero_()
                step()
            torch.cuda.synchronize()
        sus_ms, s0, s1 = timed(step, args.steps, per_step=flush_l2)
        sus_part_ms = partial_ms()
        smi = sampler.stop()
        sus_clocks = poller.window(s0, s1) or smi
        if sus_clocks is not None and smi is not None:
            sus_clocks = dict(sus_clocks, loaded_window_nvidia_smi=smi)
        if dec.status() != 0:
            raise RuntimeError("device status word set during the sustained steps")
        sustained = {"us_per_step": round(statistics.mean(sus_ms) * 1e3, 2),
                     "value": round(world * kv_bytes / (max_over_ranks(statistics.mean(sus_ms), world, dev) / 1e3)
                                    / 1e9, 2),
                     "partial_us": round(statistics.mean(sus_part_ms) * 1e3, 2),
                     "clocks": sus_clocks,
                     "how": f"the same {args.steps} steps after {args.clock_window_s} s of back-to-back steps"}
    poller.stop()
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    value = world * kv_bytes * args.steps / (total_ms / 1e3) / 1e9

    # end to end through the public API: inputs from pinned host memory each step,
    # result read back to pinned host memory, all inside the timed region
    e2e = None
    if not args.no_e2e:
        hq = inp.q.cpu().pin_memory() if not inp.q.is_cuda else inp.q.cpu().pin_memory()
        hbt = inp.block_tables.cpu().pin_memory()
        hsl = inp.seq_lens.cpu().pin_memory()
        h2d = hq.numel() * hq.element_size() + hbt.numel() * 4 + hsl.numel() * 4
        d2h = out.numel() * 2 + lse.numel() * 4
        # two sets of device inputs and outputs and of pinned read-back buffers
        dev_sets = [(torch.empty_like(g.q), torch.empty_like(g.block_tables), torch.empty_like(g.seq_lens),
                     torch.empty_like(out), torch.empty_like(lse)) for _ in range(2)]
        host_sets = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                      torch.empty(lse.shape, dtype=lse.dtype).pin_memory()) for _ in range(2)]

        def e2e_step(k):
            dq, dbt, dsl, dout, dlse = dev_sets[k % 2]
            hout, hlse = host_sets[k % 2]
            dq.copy_(hq, non_blocking=True)
            dbt.copy_(hbt, non_blocking=True)
            dsl.copy_(hsl, non_blocking=True)
            dec(dq, g.kv_cache, dbt, dsl, g.softmax_scale, g.q_scale, g.kv_scale, out=dout, lse=dlse)
            hout.copy_(dout, non_blocking=True)
            hlse.copy_(dlse, non_blocking=True)

        def serial(n):
            """Each step's copies and decode one after another on one stream, an event pair around
            each step (the L2 flush, when there is one, between the pairs)."""
            ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
            for k in range(n):
                flush.zero_()
                ev2[k][0].record()
                e2e_step(k)
                ev2[k][1].record()
            torch.cuda.synchronize()
            return sum(a.elapsed_time(b) for a, b in ev2)

        def pipelined(n):
            """Two steps in flight, as with two independent micro-batches: step k's inputs go up on
            one copy stream while step k - 1 computes, and its result comes back on another while
            step k + 1 computes; each set of buffers is reused only after its previous step's
            read-back. One event pair from the first upload to the last read-back."""
            comp = torch.cuda.current_stream()
            s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            done_comp, done_out = [None, None], [None, None]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s_in.wait_stream(comp)
            s_out.wait_stream(comp)
            e0.record(s_in)
            for k in range(n):
                b = k % 2
                dq, dbt, dsl, dout, dlse = dev_sets[b]
                hout, hlse = host_sets[b]
                with torch.cuda.stream(s_in):
                    if done_comp[b] is not None:
                        s_in.wait_event(done_comp[b])
                    dq.copy_(hq, non_blocking=True)
                    dbt.copy_(hbt, non_blocking=True)
                    dsl.copy_(hsl, non_blocking=True)
                    ev_in = torch.cuda.Event()
                    ev_in.record(s_in)
                comp.wait_event(ev_in)
                if done_out[b] is not None:
                    comp.wait_event(done_out[b])
                dec(dq, g.kv_cache, dbt, dsl, g.softmax_scale, g.q_scale, g.kv_scale, out=dout, lse=dlse)
                done_comp[b] = torch.cuda.Event()
                done_comp[b].record(comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done_comp[b])
                    hout.copy_(dout, non_blocking=True)
                    hlse.copy_(dlse, non_blocking=True)
                    done_out[b] = torch.cuda.Event()
                    done_out[b].record(s_out)
            e1.record(s_out)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1)

        for k in range(3):
            e2e_step(k)
        torch.cuda.synchronize()
        ser_ms = max_over_ranks(serial(args.steps), world, dev)
        ser = {"value": round(world * kv_bytes * args.steps / (ser_ms / 1e3) / 1e9, 2), "unit": "GB/s",
               "us_per_step": round(ser_ms / args.steps * 1e3, 2),
               "how": "each step's uploads, decode and read-back one after another on one stream"}
        if flush_l2:
            # the pipeline cannot flush the L2 between steps: the serial timing is the line
            e2e = dict(ser, h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h))
        else:
            pipelined(3)
            pip_ms = max_over_ranks(pipelined(args.steps), world, dev)
            e2e = {"value": round(world * kv_bytes * args.steps / (pip_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                   "us_per_step": round(pip_ms / args.steps * 1e3, 2),
                   "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                   "how": "two steps in flight (uploads and read-backs on two copy streams, overlapping the "
                          "neighbouring steps' decode), one event pair from the first upload to the last "
                          "read-back", "serial": ser}
        last = (args.steps - 1) % 2
        if not (torch.equal(host_sets[last][0], dev_sets[last][3].cpu()) and torch.equal(host_sets[last][0], out.cpu())):
            raise RuntimeError("e2e read-back differs from the device result")

    peak, peak_kind = measured_peak()
    flops = algorithmic_flops(inp.seq_lens.tolist(), T, H)
    # the partial kernel's function name, as ncu lists it
    if plan.kernel == 2:
        kname = "simt_partial_kernel"
    elif g.dtype == "fp8":
        kname = "tc_fp8_pair_kernel" if plan.kernel == 1 else "tc_fp8_partial_kernel"
    else:
        kname = "tc16_pair_kernel" if plan.schedule == 1 else "tc_partial_kernel"
    # The timed steps are a few milliseconds of work after a short warm-up: the tensor side is
    # taken against the measured burst peak. The sustained block (after the loaded window, under
    # the power cap) is taken against the measured sustained peak.
    roofline = roofline_fields(alg_bytes_partial, flops, statistics.mean(part_ms) / 1e3, peak, peak_kind,
                               g.dtype, sustained=False)
    roofline.update({"traffic": traffic_from_profile(args.workload, kname), "kernel": kname,
                     "alg_bytes_per_launch": int(alg_bytes_partial), "alg_flops_per_launch": int(flops),
                     "partial_us": round(statistics.mean(part_ms) * 1e3, 2),
                     "partial_how": ("the workspace clear and the partial kernel, " + ("an event pair around each call, the L2 flushed between calls" if flush_l2 else f"{args.steps} partial-only calls back to back under one event pair"))})
    if sustained is not None:
        r2 = roofline_fields(alg_bytes_partial, flops, sustained["partial_us"] / 1e6, peak, peak_kind, g.dtype,
                             sustained=True)
        sustained["roofline"] = {"bound": r2["bound"], "frac": r2["frac"], "hbm_frac": r2["hbm_frac"],
                                 "tensor_frac": r2["tensor_frac"], "tensor_peak": r2["tensor_peak"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    us = ms_per_step * 1e3
    vs = None
    if args.workload in PUBLISHED_US:
        vs = round(PUBLISHED_US[args.workload] / us, 3)  # >1: faster than the published figure
    line = {
        "metric": "MLA decode effective KV GB/s (us/step in ms_per_step) on 1 B200",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "us_per_step": round(us, 2),
        "per_step_events": {"us_mean": round(statistics.mean(each_ms) * 1e3, 2),
                            "us_p10": round(sorted(each_ms)[len(each_ms) // 10] * 1e3, 2),
                            "us_p90": round(sorted(each_ms)[(9 * len(each_ms)) // 10] * 1e3, 2),
                            "how": "the same K steps again, an event pair around each"},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": vs,
        "dtype": {"fp8": "fp8_e4m3", "bf16": "bf16", "fp16": "fp16"}[g.dtype],
        "data": "synthetic (seeded, generated on device)",
        "config": {"workload": args.workload, "batch": B, "q_len": T, "heads": H,
                   "seq_len_max": g.max_seq_len, "kv_tokens": kv_tokens, "page_size": 64,
                   "split_kv": plan.split_kv, "fold": plan.fold, "kernel": kname,
                   "kv_bytes_per_step": kv_bytes,
                   "l2": (f"256 MiB buffer rewritten between steps (cache pool {pool_bytes >> 20} MiB)" if flush_l2
                          else f"warm L2: no flush between steps (cache pool {pool_bytes >> 20} MiB)" if args.warm_l2
                          else f"inputs larger than L2: cache pool {pool_bytes >> 20} MiB >= 2 x 126 MB L2, "
                               "no flush"),
                   "parallelism": f"replicas x{world}"},
        "gpu_launches": kernels_per_step * args.steps,
        "wall_s_timed": round(wall1 - wall0, 4),
        "roofline": roofline, "e2e": e2e, "clocks": clocks, "sustained": sustained, "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- oracle timing

def _oracle_sample_inputs(workload, index=0):
    """One batch entry of the workload, same shape and distributions, drawn on the CPU."""
    from mla_paged_decode_04_b200.inputs import WORKLOADS, make_inputs_custom
    w = WORKLOADS[workload]
    n = w.max_seq_len if w.seq[0] == "fixed" else int(w.seq[1]) if w.seq[0] == "lognormal" else (w.seq[1] + w.seq[2]) // 2
    return make_inputs_custom(1, w.q_len, w.heads, w.dtype, [n], seed=2000 + 97 * index + w.config,
                              pool="exact", q_std=w.q_std, kv_std=w.kv_std), n


def cpu_baseline(workload, target_s=10.0, max_entries=16):
    """The oracle on the host cores over a bounded sample: whole batch entries of the workload (all
    their query rows), drawn one at a time until about target_s seconds of oracle time."""
    import oracle
    t_total, work_bytes, entries, rows_total, n = 0.0, 0, 0, 0, 0
    while entries < max_entries and (entries == 0 or t_total < target_s):
        inp, n = _oracle_sample_inputs(workload, entries)
        rows_total = inp.q_len * inp.heads
        t0 = time.perf_counter()
        oracle.mla_decode(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens, inp.softmax_scale,
                          dtype=inp.dtype, q_scale=inp.q_scale, kv_scale=inp.kv_scale)
        t_total += time.perf_counter() - t0
        work_bytes += n * 576 * (1 if inp.dtype == "fp8" else 2)
        entries += 1
    cores = oracle.num_threads()
    one = cpu_baseline_one_core(workload)
    return {"value": round(work_bytes / t_total / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle", "seconds": round(t_total, 3),
            "sample": f"{entries} batch entries of the workload ({n} keys, all {rows_total} query rows each); "
                      f"KV bytes of those entries over the oracle's time",
            "one_core": one}


def cpu_baseline_one_core(workload, target_s=5.0):
    """The oracle on one host core: query rows of the workload's first entry, 32 at a time, until
    about target_s seconds; KV bytes counted per row (the fraction of the entry's rows done)."""
    import oracle
    inp, n = _oracle_sample_inputs(workload, 0)
    rows_total = inp.q_len * inp.heads
    esize = 1 if inp.dtype == "fp8" else 2
    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        t_total, done = 0.0, 0
        while done < rows_total and (done == 0 or t_total < target_s):
            rows = list(range(done, min(rows_total, done + 32)))
            t0 = time.perf_counter()
            oracle.mla_decode(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens, inp.softmax_scale,
                              dtype=inp.dtype, q_scale=inp.q_scale, kv_scale=inp.kv_scale, rows=rows)
            t_total += time.perf_counter() - t0
            done += len(rows)
    finally:
        oracle.set_num_threads(cores)
    work_bytes = n * 576 * esize * done / rows_total
    return {"value": round(work_bytes / t_total / 1e9, 5), "unit": "GB/s", "cores": 1, "seconds": round(t_total, 3),
            "sample": f"{done} of the {rows_total} query rows of one batch entry ({n} keys); "
                      f"KV bytes scaled by the row fraction"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from mla_paged_decode_04_b200.inputs import WORKLOADS
    inp, n = _oracle_sample_inputs(args.workload)
    rows_total = inp.q_len * inp.heads
    rows = list(range(0, rows_total, rows_total // 8))[:8]
    esize = 1 if inp.dtype == "fp8" else 2

    def one():
        oracle.mla_decode(inp.q, inp.kv_cache, inp.block_tables, inp.seq_lens, inp.softmax_scale,
                          dtype=inp.dtype, q_scale=inp.q_scale, kv_scale=inp.kv_scale, rows=rows)

    for _ in range(args.warmup):
        one()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        one()
        times.append(time.perf_counter() - t0)
    dt = sum(times)
    work_bytes = n * 576 * esize * len(rows) / rows_total
    value = work_bytes * args.steps / dt / 1e9
    w = WORKLOADS[args.workload]
    sample = (f"{len(rows)} of the {rows_total} query rows of one batch entry ({n} keys, "
              f"{inp.dtype}) per step; KV bytes scaled by the row fraction")
    line = {"impl": "reference", "metric": "MLA decode effective KV GB/s (us/step in ms_per_step) on 1 B200",
            "value": round(value, 5), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {"fp8": "fp8_e4m3", "bf16": "bf16", "fp16": "fp16"}[w.dtype],
            "data": "synthetic (seeded)",
            "config": {"workload": args.workload, "batch": w.batch, "q_len": w.q_len,
                       "heads": w.heads, "seq_len_max": w.max_seq_len, "page_size": 64},
            "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_prefill(args):
    """--op prefill --impl reference: the oracle's ragged prefill on the host cores, each step a
    bounded sample (the last 8 tokens of entry 0 of the workload, all heads), flops of those rows."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from mla_paged_decode_04_b200.inputs import PREFILL_WORKLOADS, make_prefill_workload
    name = args.workload if args.workload in PREFILL_WORKLOADS else "prefill_fp8"
    inp = make_prefill_workload(name)
    cu, H = inp.cu_seqlens_q.tolist(), inp.heads
    toks = list(range(max(cu[0], cu[1] - 8), cu[1]))
    rows = [t * H + h for t in toks for h in range(H)]
    n0, q0 = int(inp.seq_lens[0]), cu[1] - cu[0]
    flops = sum(n0 - q0 + (t - cu[0]) + 1 for t in toks) * H * 2 * (576 + 512)

    def one():
        oracle.mla_prefill(inp.q, inp.cu_seqlens_q, inp.kv_cache, inp.block_tables, inp.seq_lens,
                           inp.softmax_scale, dtype=inp.dtype, q_scale=inp.q_scale, kv_scale=inp.kv_scale, rows=rows)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = f"{len(rows)} query rows per step (the last {len(toks)} tokens of entry 0, all heads); flops of those rows"
    line = {"impl": "reference", "metric": "MLA ragged prefill TFLOP/s (algorithmic flops per step / step time) on 1 B200",
            "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": {"fp8": "fp8_e4m3", "bf16": "bf16", "fp16": "fp16"}[inp.dtype], "data": "synthetic (seeded)",
            "config": {"workload": name, "batch": inp.batch, "heads": H, "total_q": inp.total_q},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_kv_pack(args):
    """Fused K/V pack + FP8 quantise on a prefill-sized write: 16 x 81,920 BF16 tokens into an
    FP8 cache of twice the pages (permuted slots). One JSON line; HBM roofline."""
    import torch
    import mla_paged_decode_04_b200 as mla

    import torch.distributed as dist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, dev)
    n = 16 * 81920
    num_pages = 2 * n // 64
    g = torch.Generator(device=dev).manual_seed(4242)
    latent = torch.randn(n, 512, generator=g, device=dev).to(torch.bfloat16)
    rope = torch.randn(n, 64, generator=g, device=dev).to(torch.bfloat16)
    slots = torch.randperm(num_pages * 64, generator=g, device=dev)[:n].to(torch.int64)
    cache = torch.empty(num_pages, 64, 576, dtype=torch.float8_e4m3fn, device=dev)
    scale = float(mla.kv_amax(latent, rope).item()) / 448.0
    alg = n * (512 + 64) * 2 + n * 576 + n * 8  # inputs, FP8 rows, slots
    for _ in range(max(args.warmup, 3)):
        mla.kv_pack(latent, rope, slots, cache, kv_scale=scale)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    t_end = time.perf_counter() + args.clock_window_s
    while time.perf_counter() < t_end:
        for _ in range(20):
            mla.kv_pack(latent, rope, slots, cache, kv_scale=scale)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for k in range(args.steps):
        evs[k][0].record()
        mla.kv_pack(latent, rope, slots, cache, kv_scale=scale)
        evs[k][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = [a.elapsed_time(b) for a, b in evs]
    mean_s = max_over_ranks(statistics.mean(ms), world, dev) / 1e3
    peak, peak_kind = measured_peak()
    achieved = alg / mean_s / 1e9
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "fused K/V pack + FP8 quantise GB/s (inputs + FP8 rows + slots per call)",
        "value": round(world * achieved, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(mean_s * 1e3, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16->fp8_e4m3", "data": "synthetic (seeded, generated on device)",
        "config": {"workload": "kv_pack_bf16_fp8", "tokens": n, "num_pages": num_pages,
                   "l2": "inputs larger than L2 (1.5 GB read, 755 MB written per call), no flush"},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_kind, "traffic": None,
                     "kernel": "kv_pack_fp8_kernel", "alg_bytes_per_launch": int(alg)},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def prefill_flops(cu, seq_lens, heads):
    """Algorithmic flops of a ragged prefill step: 2 * (576 + 512) per (query row, visible key);
    token t of an entry with qlen new tokens and n keys sees n - qlen + t + 1 keys."""
    from mla_paged_decode_04_b200.inputs import D_QK, D_V
    total = 0
    for b in range(len(seq_lens)):
        qlen, n = cu[b + 1] - cu[b], int(seq_lens[b])
        # sum over t of max(0, n - qlen + t + 1)
        for t in range(qlen):
            total += max(0, n - qlen + t + 1)
    return total * heads * 2 * (D_QK + D_V)


def run_prefill(args):
    """Ragged prefill over the paged cache (tokenspeed-mla package card: variable-length
    sequences without padding): one mla_prefill call per step on a named workload. Compute-bound:
    the roofline is the tensor peak of the input type, HBM beside it."""
    import torch
    import mla_paged_decode_04_b200 as mla
    from mla_paged_decode_04_b200.inputs import PREFILL_WORKLOADS, make_prefill_workload

    import torch.distributed as dist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, dev)
    name = args.workload if args.workload in PREFILL_WORKLOADS else "prefill_fp8"
    w = PREFILL_WORKLOADS[name]
    inp = make_prefill_workload(name, device=dev, batch=args.batch or None)
    g = inp.to(dev)
    pre = mla.MlaPrefill(g.batch, g.max_q_len, g.heads, g.max_seq_len, g.dtype, dev)
    out = torch.empty((g.total_q, g.heads, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((g.total_q, g.heads), dtype=torch.float32, device=dev)
    cu = inp.cu_seqlens_q.tolist()
    flops = prefill_flops(cu, inp.seq_lens.tolist(), g.heads)
    esize = 1 if g.dtype == "fp8" else 2
    kv_bytes = int(inp.seq_lens.sum()) * 576 * esize
    alg_bytes = kv_bytes + g.q.numel() * esize + out.numel() * 2 + lse.numel() * 4
    pool_bytes = g.kv_cache.numel() * esize
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # the cache pool fits in L2
    call = (g.q, g.cu_seqlens_q, g.kv_cache, g.block_tables, g.seq_lens, g.softmax_scale)

    def step():
        mla.mla_prefill(pre.plan, *call, out, lse, pre.workspace, g.q_scale, g.kv_scale)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if pre.status() != 0:
        raise RuntimeError("device status word set during warm-up")
    sampler = ClockSampler(local)
    sampler.start()
    t_end = time.perf_counter() + args.clock_window_s
    while time.perf_counter() < t_end:
        flush.zero_()
        step()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record()
        step()
        evs[k][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    if pre.status() != 0:
        raise RuntimeError("device status word set during the timed steps")
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)
    total_ms = max_over_ranks(total_ms, world, dev)
    mean_s = total_ms / args.steps / 1e3
    value = world * flops / mean_s / 1e12

    # end to end through MlaPrefill: packed q, offsets and tables from pinned host memory,
    # out/lse back, inside the timed region
    hq = inp.q.cpu().pin_memory()
    hcu, hbt, hsl = (inp.cu_seqlens_q.pin_memory(), inp.block_tables.pin_memory(), inp.seq_lens.pin_memory())
    dq, dcu, dbt, dsl = (torch.empty_like(g.q), torch.empty_like(g.cu_seqlens_q), torch.empty_like(g.block_tables),
                         torch.empty_like(g.seq_lens))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = hq.numel() * esize + (hcu.numel() + hbt.numel() + hsl.numel()) * 4
    d2h = hout.numel() * 2 + hlse.numel() * 4

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dcu.copy_(hcu, non_blocking=True)
        dbt.copy_(hbt, non_blocking=True)
        dsl.copy_(hsl, non_blocking=True)
        pre(dq, dcu, g.kv_cache, dbt, dsl, g.softmax_scale, g.q_scale, g.kv_scale, out=out, lse=lse)
        hout.copy_(out, non_blocking=True)
        hlse.copy_(lse, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush.zero_()
        ev2[k][0].record()
        e2e_step()
        ev2[k][1].record()
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in ev2)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    e2e = {"value": round(world * flops / (e2e_ms / args.steps / 1e3) / 1e12, 2), "unit": "TFLOP/s",
           "ms_per_step": round(e2e_ms / args.steps, 4), "h2d_bytes_per_step": int(h2d),
           "d2h_bytes_per_step": int(d2h)}

    tpeak, tpeak_kind = measured_tensor_peak(g.dtype, sustained=True)
    hpeak, hpeak_kind = measured_peak()
    kname = "tc_fp8_pair_kernel" if g.dtype == "fp8" else "tc16_pair_kernel"
    achieved_t = flops / mean_s / 1e12
    achieved_h = alg_bytes / mean_s / 1e9
    roofline = {"bound": "tensor", "achieved": round(achieved_t, 1), "peak": round(tpeak, 1), "unit": "TFLOP/s",
                "frac": round(achieved_t / tpeak, 4), "peak_source": tpeak_kind, "traffic": None,
                "kernel": kname, "scope": "whole step (partial + combine)", "alg_flops_per_step": int(flops),
                "floor_ms": round(flops / (tpeak * 1e12) * 1e3, 4),
                "other": {"bound": "hbm", "achieved": round(achieved_h, 1), "peak": hpeak, "unit": "GB/s",
                          "frac": round(achieved_h / hpeak, 4), "peak_source": hpeak_kind,
                          "floor_ms": round(alg_bytes / (hpeak * 1e9) * 1e3, 4)}}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        H = g.heads
        hcache = inp.kv_cache.cpu()
        n0, q0 = int(inp.seq_lens[0]), cu[1] - cu[0]
        dt, sample_flops, ntok, end = 0.0, 0, 0, cu[1]
        while end > cu[0] and (ntok == 0 or dt < 10.0):  # the last tokens of entry 0 (its longest rows), 8 at a time
            toks = list(range(max(cu[0], end - 8), end))
            rows = [t * H + h for t in toks for h in range(H)]
            t0 = time.perf_counter()
            oracle.mla_prefill(hq, inp.cu_seqlens_q, hcache, inp.block_tables, inp.seq_lens, g.softmax_scale,
                               dtype=g.dtype, q_scale=g.q_scale, kv_scale=g.kv_scale, rows=rows)
            dt += time.perf_counter() - t0
            sample_flops += sum(n0 - q0 + (t - cu[0]) + 1 for t in toks) * H * 2 * (576 + 512)
            ntok += len(toks)
            end -= 8
        cpu = {"value": round(sample_flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
               "kind": "oracle", "seconds": round(dt, 3),
               "sample": f"{ntok * H} query rows (the last {ntok} tokens of entry 0, all heads); flops of those rows"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "MLA ragged prefill TFLOP/s (algorithmic flops per step / step time) on 1 B200",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"fp8": "fp8_e4m3", "bf16": "bf16", "fp16": "fp16"}[g.dtype],
        "data": "synthetic (seeded, generated on device)",
        "config": {"workload": name, "batch": g.batch, "heads": g.heads, "total_q": g.total_q,
                   "max_q_len": g.max_q_len, "kv_tokens": int(inp.seq_lens.sum()), "fold": pre.plan.fold,
                   "units": pre.plan.batch * pre.plan.q_groups, "desc": w.desc,
                   "l2": f"256 MiB buffer rewritten between steps (cache pool {pool_bytes >> 20} MiB)",
                   "parallelism": f"replicas x{world}"},
        "gpu_launches": (3 if pre.plan.schedule == 1 else 2) * args.steps,  # clear, partial, combine
        "roofline": roofline, "e2e": e2e, "clocks": clocks, "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.op == "kv_pack":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the K/V pack reference arm is not timed; "
                              "its oracle is checked byte for byte in tests/test_kv_pack.py"}), flush=True)
        else:
            run_kv_pack(args)
        return
    if args.op == "prefill":
        if args.impl == "reference":
            run_reference_prefill(args)
        else:
            run_prefill(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
