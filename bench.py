"""Benchmark of the masked attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 1..6]

Default (headline) workload: the long block-dense custom mask -- one sequence of 29576
queries / keys, rows < 24576 see keys [0, 24576), the last 5000 rows add causal attention
inside their own 100-row block; Hq=32, Hkv=8, d=128, bf16 N(0,1) inputs -- given once as
packed CUSTOM bits and once as typed ranges. One step = both forwards. It is the largest
of the five benchmark workloads that fit one GPU.

Metric: effective TFLOP/s = 4 * d * (unmasked pairs) * Hq / time, summed over the masks of
the step (masked pairs are not counted). Prints ONE JSON line on rank 0. After the
headline, the other four benchmark workloads are timed one by one and reported in the same
line under "per_config", and the backward of the chunk-causal (d=128) and Gemma2 (d=256)
workloads under "backward" (--no-per-config skips both).

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent batch of the
same workload (seed offset by rank); there is no collective on the data path. Timing is
the max over ranks of CUDA-event time; the value is the work of all ranks / that time.

--impl reference times the fp64 CPU oracle on a bounded row sample of the same workload
(rank 0 only): the CPU baseline arm.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective masked-attn TFLOP/s (unmasked pairs) and % of B200 bf16 tensor peak"
# --pass bwd: the backward pass, counted as the usual 10 d FLOPs per unmasked pair and head
# (S, dP, dV, dK, dQ: five 2 d products; the kernels recompute S and dP once more for dQ)
METRIC_BWD = "effective masked-attn backward TFLOP/s (10 d FLOPs per unmasked pair) and % of B200 bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


def workload(cfg: int, rank: int):
    import workloads as W
    seed = cfg + 7919 * rank
    return W.config(cfg, seed=seed)


def flops_of(stats, wl):
    return 4.0 * wl.d * stats["unmasked_pairs"] * wl.hq


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("attn_fwd.cu", "device_common.cuh", "mma_groups.inc", "tmem_ldst.inc", "attn_internal.h"):
        with open(os.path.join(ROOT, "masked_flash_attention_attn_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(workload_name):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", "fwd_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload_name)
    if not e or e.get("kernel_source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of one GPU, sampled through NVML every
    `period_s` seconds on a background thread while the timed region runs; falls back to an
    `nvidia-smi -lms` subprocess when NVML cannot be used. `stop()` returns the summary of
    the samples taken inside [mark_start(), mark_end()] -- or, when NVML and nvidia-smi both
    fail, {"error": why} instead of a silent null."""
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, log_dir=None, period_s=0.01):
        import threading
        self.samples = []          # (host time, sm MHz, max sm MHz, reason names)
        self.errors = []
        self.t0 = self.t1 = None
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        self.log_path = os.path.join(log_dir or tempfile.gettempdir(), f"clocks_dev{device_index}.csv")
        try:
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception as e:          # pragma: no cover - needs a GPU
            self.errors.append(f"device uuid: {type(e).__name__}: {e}")
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def sample():
                sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                bits = int(get_reasons(h))
                return (time.perf_counter(), sm, smax, [n for n, b in self.REASON_BITS.items() if bits & b])

            self.samples.append(sample())    # fails here, not on the thread, if NVML is unusable

            def loop():
                while not self._stop.wait(period_s):
                    try:
                        self.samples.append(sample())
                    except Exception as e:   # pragma: no cover
                        self.errors.append(f"nvml sample: {type(e).__name__}: {e}")
                        return

            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            self.source = f"nvml every {period_s * 1e3:.0f} ms"
            return
        except Exception as e:
            self.errors.append(f"nvml: {type(e).__name__}: {e}")
        try:
            os.makedirs(os.path.dirname(self.log_path), exist_ok=True)
            self._fh = open(self.log_path, "w")
            self._proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.SMI_FIELDS}",
                                           "--format=csv,noheader,nounits", "-lms", "50"],
                                          stdout=self._fh, stderr=subprocess.PIPE)
            self.source = "nvidia-smi -lms 50"
            # wait (up to 3 s) for its first sample so the timed region is covered
            t_wait = time.perf_counter()
            while time.perf_counter() - t_wait < 3.0 and os.path.getsize(self.log_path) == 0:
                if self._proc.poll() is not None:
                    break
                time.sleep(0.02)
        except Exception as e:
            self.errors.append(f"nvidia-smi: {type(e).__name__}: {e}")
            self._proc = None

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def _smi_rows(self):
        self._proc.terminate()
        try:
            _, err = self._proc.communicate(timeout=5)
        except Exception:
            self._proc.kill()
            err = b""
        self._fh.close()
        rows = []
        with open(self.log_path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    rows.append((None, float(p[1]), float(p[2]),
                                 [n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                                     "sw_power_cap"), p[5:9]) if v.lower().startswith("active")]))
                except ValueError:
                    continue
        if not rows and err:
            self.errors.append("nvidia-smi: " + err.decode(errors="replace").strip()[:200])
        return rows

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
            rows = self.samples
            inside = [r for r in rows if self.t0 is not None and self.t1 is not None and self.t0 <= r[0] <= self.t1]
            # a timed region shorter than the sampling period still gets its nearest samples
            if not inside and rows and self.t0 is not None:
                inside = sorted(rows, key=lambda r: abs(r[0] - self.t0))[:2]
        elif self._proc is not None:
            inside = self._smi_rows()      # nvidia-smi rows carry no host time: all of them
        else:
            inside = []
        if not inside:
            return {"error": "; ".join(self.errors) or "no clock samples"}
        reasons = sorted({n for r in inside for n in r[3]})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_min_mhz": min(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons, "samples": len(inside),
                "source": self.source}


def oracle_sample(wl, specs, budget_s, rows_per_block=128):
    """Time the fp64 oracle on row blocks (one query head each, cycling through sequences,
    heads and the masks of the step) until budget_s has passed. Returns (pairs*heads, seconds, desc)."""
    import oracle
    from oracle import masks as OM
    from oracle import attention as OA
    import torch
    g = wl.hq // wl.hkv
    pairs, t_used, blocks = 0, 0.0, 0
    b_order = sorted(range(wl.batch), key=lambda b: -wl.lq(b))
    kv = {}
    while t_used < budget_s:
        b = b_order[blocks % len(b_order)]
        spec = specs[blocks % len(specs)]
        h = (blocks // len(b_order)) % wl.hq
        lq, lk = wl.lq(b), wl.lk(b)
        r1 = lq - (blocks * 977) % max(1, lq - rows_per_block)
        r0 = max(0, r1 - rows_per_block)
        if b not in kv:
            kk, vv = wl.kv_of_seq(b)
            kv[b] = (kk.to(torch.float64).numpy(), vv.to(torch.float64).numpy())
        kk, vv = kv[b]
        q0 = int(wl.cu_seqlens_q[b])
        t0 = time.perf_counter()
        m = OM.dense_mask_rows(spec, b, lq, lk, r0, r1)
        qq = wl.q[q0 + r0:q0 + r1, h].to(torch.float64).numpy()
        OA.attention_one_head(qq, kk[:, h // g], vv[:, h // g], m, wl.scale)
        t_used += time.perf_counter() - t0
        pairs += int(m.sum())
        blocks += 1
    desc = (f"{blocks} blocks of <= {rows_per_block} query rows x 1 head over all keys, cycling the "
            f"{len(specs)} masks of the step; fp64 NumPy")
    return pairs, t_used, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = workload(args.config, 0)
    specs = wl.masks
    per_step = max(0.25, min(4.0, 150.0 / max(1, args.steps)))  # whole run within a few minutes
    for _ in range(args.warmup):
        oracle_sample(wl, specs, 0.2)
    pairs, secs = 0, 0.0
    desc = None
    for _ in range(args.steps):
        p, s, desc = oracle_sample(wl, specs, per_step)
        pairs, secs = pairs + p, secs + s
    flops = 4.0 * wl.d * pairs
    val = flops / secs / 1e12
    cores = blas_threads()
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, args, world),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} steps x ~{per_step:.0f} s: {desc}"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def custom_bytes(spec):
    """Bytes of a CUSTOM mask's packed bits (what attn_plan scans on the device)."""
    return int(np.asarray(spec.bits).nbytes) if getattr(spec, "bits", None) is not None else 0


def config_of(wl, args, world):
    tq = int(wl.cu_seqlens_q[-1])
    tk = int(wl.cu_seqlens_k[-1]) if not wl.paged else int(wl.k_cache.shape[0] * wl.page_size)
    in_bytes = 2 * (tq * wl.hq * wl.d + 2 * tk * wl.hkv * wl.d)
    return {"workload": wl.name, "batch": wl.batch,
            "lengths_q": [wl.lq(b) for b in range(wl.batch)][:64],
            "hq": wl.hq, "hkv": wl.hkv, "head_dim": wl.d,
            "masks": [m.kind + (f"({m.window})" if m.kind == "SLIDING_WINDOW" else "") for m in wl.masks],
            "seed": wl.seed, "kv_splits": getattr(args, "kv_splits", 0), "pass": getattr(args, "pass_", "fwd"),
            "parallelism": f"dp{world} (independent batches, no collective)",
            "l2": f"inputs {in_bytes / 2**20:.0f} MiB vs 126 MiB L2; no flush" if in_bytes > L2_BYTES
            else "inputs fit L2; L2 flushed between steps"}


def reduce_over_ranks(times_ms, work, device):
    """Max over ranks of each timing and sum over ranks of the work (for the JSON line only;
    nothing on the data path is exchanged)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    w = torch.tensor([float(work)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return [float(x) for x in t], float(w[0])


def device_inputs(wl, dev):
    q = wl.q.to(dev)
    if wl.paged:
        return q, wl.k_cache.to(dev), wl.v_cache.to(dev)
    return q, wl.k.to(dev), wl.v.to(dev)


def make_plan(M, wl, spec, dev, kv_splits=0, backward=False, q_rows=None):
    import torch
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, mask=spec, scale=wl.scale,
              kv_splits=kv_splits, backward=backward, q_rows=q_rows)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_table=torch.from_numpy(wl.page_table).to(dev),
                  page_size=wl.page_size, num_pages=wl.k_cache.shape[0])
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    return M.attn_plan(**kw)


def kernel_name(wl, fp8=False, bwd=False):
    """The kernel a forward (or backward) of this workload launches."""
    if bwd:
        pre = "masked_attn_bwd256" if wl.d == 256 else "masked_attn_bwd"
        return f"{pre}_dq_kernel + {pre}_dkv_kernel d={wl.d}{' paged' if wl.paged else ''}"
    base = "masked_attn_fwd_pair_kernel (2-SM)" if wl.d == 256 else "masked_attn_fwd_kernel"
    return f"{base}{' e4m3' if fp8 else ''} d={wl.d}{' paged' if wl.paged else ''}"


def stage_mask(spec, dev):
    """attn_mask_desc_t.mask_bits is a device pointer: CUSTOM bits are staged in HBM before
    planning, so a timed attn_plan covers the device scan, not a host upload."""
    import torch
    if spec.kind == "CUSTOM" and isinstance(spec.bits, np.ndarray):
        spec = dataclasses.replace(spec, bits=torch.from_numpy(
            np.ascontiguousarray(spec.bits.astype(np.uint32).view(np.int32))).to(dev))
        torch.cuda.synchronize()
    return spec


def build_plans(M, wl, dev, kv_splits=0, backward=False):
    """One plan per mask of the workload; attn_plan is timed on its own (host wall clock; it
    synchronises its stream). The first plan of a kind also pays one-off costs (context
    set-up, module loading): each mask is planned once untimed, then the kept plan is timed."""
    plans, plan_ms = [], []
    for spec in wl.masks:
        spec = stage_mask(spec, dev)
        make_plan(M, wl, spec, dev, kv_splits, backward=backward)
        t0 = time.perf_counter()
        plans.append(make_plan(M, wl, spec, dev, kv_splits, backward=backward))
        plan_ms.append((time.perf_counter() - t0) * 1e3)
    return plans, plan_ms


def kv_bytes_read(wl):
    """K and V bytes one forward must read at least once (bf16): the keys of every sequence."""
    return sum(wl.lk(b) for b in range(wl.batch)) * wl.hkv * wl.d * 2 * 2


def measure_e4m3_gemm_tflops(dev, n=8192, iters=20):
    """Dense e4m3 tensor rate of this GPU, measured: cuBLASLt's fp8 GEMM (torch._scaled_mm,
    n x n x n, e4m3 inputs, bf16 out) timed with CUDA events after warm-up -- the e4m3
    counterpart of the driver's cuBLAS bf16 figure. None when the call is not available."""
    import torch
    try:
        gen = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn(n, n, generator=gen, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, generator=gen, device=dev).to(torch.float8_e4m3fn).t()   # column-major operand
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record()
        for _ in range(iters):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        t1.record()
        torch.cuda.synchronize()
        return 2.0 * n ** 3 * iters / (t0.elapsed_time(t1) * 1e-3) / 1e12
    except Exception:   # noqa: BLE001 -- no fp8 GEMM here: the caller falls back to the ratio rule
        return None


def choose_peak(clocks, fp8=False, e4m3_tflops=None):
    """Tensor peak for the roofline: the measured burst cuBLAS bf16 figure, or the sustained
    one when the sampled SM clock fell below 90 % of its maximum (a long run at the power cap).
    e4m3: the fp8 GEMM rate measured in this run when given, else bf16 x 2 (the nominal ratio)."""
    pk, pk_src = peaks()
    burst = float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(pk.get("bf16_tflops_sustained", burst))
    use_sustained = isinstance(clocks, dict) and "sm_mhz" in clocks and \
        clocks["sm_mhz"] < 0.9 * clocks["sm_max_mhz"]
    peak = sustained if use_sustained else burst
    pk_src += " bf16_tflops_sustained" if use_sustained else " bf16_tflops (burst)"
    if fp8 and e4m3_tflops:
        peak, pk_src = e4m3_tflops, "measured in this run: cuBLASLt e4m3 GEMM (torch._scaled_mm, 8192^3, bf16 out)"
    elif fp8:   # e4m3 tensor rate: the measured bf16 figure x the nominal fp8 / bf16 ratio (4.5 / 2.25)
        peak *= 2.0
        pk_src += " x 2 (nominal e4m3 / bf16 ratio)"
    hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return peak, pk_src, hbm


def time_config(M, cfg, dev, stream, steps, warmup, peak, hbm_peak, bwd=False):
    """Forward (or, with `bwd`, backward) of one benchmark workload (every mask of it) on this
    GPU: CUDA-event time of each launch over `steps` steps after `warmup`, L2 flushed between
    launches when the inputs fit in it. Returns the per-config entry of the bench line."""
    import torch
    wl = workload(cfg, 0)
    q, k, v = device_inputs(wl, dev)
    plans, plan_ms = build_plans(M, wl, dev, backward=bwd)
    stats = [M.attn_plan_get_stats(p) for p in plans]
    flops = [flops_of(s, wl) * (2.5 if bwd else 1.0) for s in stats]
    tq = q.shape[0]
    outs = [torch.empty(tq, wl.hq, wl.d, dtype=torch.bfloat16, device=dev) for _ in plans]
    lses = [torch.empty(tq, wl.hq, dtype=torch.float32, device=dev) for _ in plans]
    in_bytes = (q.numel() + k.numel() + v.numel()) * 2
    if bwd:
        for i, p in enumerate(plans):
            M.attn_masked_fwd(p, q, k, v, outs[i], lses[i], stream)
        gen = torch.Generator(device=dev).manual_seed(wl.seed + 101)
        dout = torch.randn(tq, wl.hq, wl.d, generator=gen, device=dev).to(torch.bfloat16)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        in_bytes += sum(o.numel() * 2 + l.numel() * 4 for o, l in zip(outs, lses)) + dout.numel() * 2
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev) if in_bytes <= L2_BYTES else None
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in plans] for _ in range(steps)]
    for s in range(warmup + steps):
        for i, p in enumerate(plans):
            if flush is not None:
                flush.fill_(s & 255)
            if s >= warmup:
                ev[s - warmup][i][0].record(stream)
            if bwd:
                M.attn_masked_bwd(p, q, k, v, outs[i], lses[i], dout, dq, dk, dv, stream)
            else:
                M.attn_masked_fwd(p, q, k, v, outs[i], lses[i], stream)
            if s >= warmup:
                ev[s - warmup][i][1].record(stream)
    torch.cuda.synchronize()
    for p in plans:
        st = M.attn_plan_check_status(p)
        if st != 0:
            raise RuntimeError(f"workload {cfg}: {'backward' if bwd else 'forward'} reported {M.STATUS.get(st, st)}")
    launch_ms = [[ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(steps)] for i in range(len(plans))]
    mean_ms = [statistics.mean(x) for x in launch_ms]
    step_ms = sum(mean_ms)
    tflops = sum(flops) / (step_ms * 1e-3) / 1e12
    entry = {"config": cfg, "workload": wl.name, "pass": "bwd" if bwd else "fwd",
             "kernel": kernel_name(wl, bwd=bwd), "steps": steps,
             "ms_per_step": step_ms, "tflops_per_s": tflops, "frac": tflops / peak,
             "per_mask": [{"mask": m.kind, "ms": mm, "ms_median": statistics.median(x),
                           "tflops_per_s": f / (mm * 1e-3) / 1e12, "frac": f / (mm * 1e-3) / 1e12 / peak,
                           "unmasked_pairs_per_head": s["unmasked_pairs"],
                           "tiles_e_f_p": [s["tiles_empty"], s["tiles_full"], s["tiles_partial"]],
                           "kv_splits_max": s["kv_splits_max"], "plan_ms": pm}
                          for m, s, f, x, mm, pm in zip(wl.masks, stats, flops, launch_ms, mean_ms, plan_ms)],
             "l2": "L2 flushed between launches" if flush is not None else
                   f"inputs {in_bytes / 2**20:.0f} MiB vs 126 MiB L2; no flush"}
    if wl.paged and not bwd:
        # the K/V stream: bytes of the keys every request holds, read once per launch at least
        kvb = kv_bytes_read(wl)
        gbs = kvb / (step_ms / len(plans) * 1e-3) / 1e9
        entry["kv_stream"] = {"bytes_per_launch": kvb, "gbs": gbs, "hbm_peak_gbs": hbm_peak,
                              "frac_of_hbm": gbs / hbm_peak}
    mask_bytes = sum(s["mask_tile_reads"] for s in stats) * 2048.0
    entry["mask_gbs"] = mask_bytes / (step_ms * 1e-3) / 1e9
    if bwd:
        entry["flops_note"] = "10 d FLOPs per unmasked pair and head (2.5 x the forward's 4 d)"
        del dout, dq, dk, dv
    del q, k, v, outs, lses, flush, plans
    torch.cuda.empty_cache()
    return entry


def shard_rows_plan(M, wl, world):
    """Query-row shards of one problem for `world` ranks: work-balanced by the host tile
    classes of the workload's analytic mask form (a CUSTOM-only workload gets equal row
    blocks). Returns [(begin, end)] sequence-local rows per rank."""
    from masked_flash_attention_attn_b200 import sharding as S
    lengths = [(wl.lq(b), wl.lk(b)) for b in range(wl.batch)]
    analytic = next((m for m in wl.masks if m.kind != "CUSTOM"), None)
    if analytic is None:
        lq_max = max(lq for lq, _ in lengths)
        return [S.query_shard(lq_max, r, world) for r in range(world)]
    cls, _ = M.attn_classify_host(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q,
                                  cu_seqlens_k=wl.cu_seqlens_k, mask=analytic)
    return S.balanced_query_shards(cls, lengths, world)


def run_shard_rows(args, rank, world, local_rank):
    """One problem split over the ranks by query rows (--shard-rows): every rank plans its
    own rows of every sequence against all keys; K and V start sharded by rows across the
    ranks and each step first all-gathers them (NCCL all_gather_into_tensor into every GPU's
    own memory), then runs the forward of every mask of the workload on this rank's rows.
    The timed step is gather + forward; the value is the whole problem's work over the
    slowest rank's time (strong scaling: the total work is fixed)."""
    import torch
    import torch.distributed as dist
    import masked_flash_attention_attn_b200 as M
    from masked_flash_attention_attn_b200 import sharding as S

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workload(args.config, 0)            # the same problem on every rank
    if wl.paged:
        raise SystemExit("--shard-rows: a workload with contiguous K/V (1, 2, 4 or 5)")
    stream = torch.cuda.current_stream()
    shards = shard_rows_plan(M, wl, world)
    q_rows = shards[rank]
    total_k = int(wl.cu_seqlens_k[-1])
    a, b = S.row_shard(total_k, rank, world)
    k_local, v_local = wl.k[a:b].to(dev), wl.v[a:b].to(dev)
    q = wl.q.to(dev)
    gk = S.RowGather(total_k, (wl.hkv, wl.d), torch.bfloat16, dev)
    gv = S.RowGather(total_k, (wl.hkv, wl.d), torch.bfloat16, dev)
    plans = [make_plan(M, wl, stage_mask(spec, dev), dev, q_rows=q_rows) for spec in wl.masks]
    stats = [M.attn_plan_get_stats(p) for p in plans]
    full_flops = 0.0
    for spec in wl.masks:   # the whole problem's work (every rank's shard together)
        full_flops += flops_of(M.attn_plan_get_stats(make_plan(M, wl, stage_mask(spec, dev), dev)), wl)
    tq = q.shape[0]
    outs = [torch.empty(tq, wl.hq, wl.d, dtype=torch.bfloat16, device=dev) for _ in plans]
    lses = [torch.empty(tq, wl.hq, dtype=torch.float32, device=dev) for _ in plans]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        k, v = gk.gather(k_local), gv.gather(v_local)
        if ev is not None:
            ev[1].record(stream)
        for i, p in enumerate(plans):
            M.attn_masked_fwd(p, q, k, v, outs[i], lses[i], stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank, args.clock_log)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark_start()
    t0.record(stream)
    for s_ in range(args.steps):
        step(ev[s_])
    t1.record(stream)
    while not t1.query():
        time.sleep(2e-4)
    sampler.mark_end()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    for p in plans:
        st = M.attn_plan_check_status(p)
        if st != 0:
            raise RuntimeError(f"forward reported {M.STATUS.get(st, st)}")
    ms = t0.elapsed_time(t1)
    gather_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    fwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    jobs = sum(s["jobs"] for s in stats)
    (ms, gather_ms, fwd_ms), _ = reduce_over_ranks([ms, gather_ms, fwd_ms], 0.0, dev)
    if rank != 0:
        return
    value = full_flops * args.steps / (ms * 1e-3) / 1e12
    kv_bytes = 2 * total_k * wl.hkv * wl.d * 2
    peak, pk_src, _ = choose_peak(clocks)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16, lengths from seed)",
        "config": dict(config_of(wl, args, world),
                       parallelism=f"query-row shards x{world} + NCCL K/V all-gather (one problem, no batch split)",
                       shards=shards),
        "pct_of_peak": 100.0 * value / world / peak, "peak_source": pk_src,
        "gather": {"kv_bytes": kv_bytes, "bytes_received_per_rank": gk.bytes_received + gv.bytes_received,
                   "ms": gather_ms,
                   "gbs_per_rank": (gk.bytes_received + gv.bytes_received) / (gather_ms * 1e-3) / 1e9
                   if world > 1 and gather_ms > 0 else None},
        "forward_ms": fwd_ms, "jobs_rank0": jobs,
        "gpu_launches": len(plans) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import masked_flash_attention_attn_b200 as M

    if not os.path.exists(M._LIB_PATH):
        raise RuntimeError("libattn_b200.so is not built: run `python -m masked_flash_attention_attn_b200.build`")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workload(args.config, rank)
    stream = torch.cuda.current_stream()
    q, k, v = device_inputs(wl, dev)
    bwd = args.pass_ == "bwd"
    fp8 = args.dtype == "e4m3"
    if bwd and wl.paged:
        raise SystemExit("--pass bwd: contiguous K/V only (workloads 1, 2, 4, 5)")
    if fp8 and (bwd or wl.paged or wl.d not in (128, 256)):
        raise SystemExit("--dtype e4m3: the forward with contiguous K/V, head_dim 128 or 256 (workloads 2, 4, 5)")
    plans, plan_ms = build_plans(M, wl, dev, args.kv_splits, backward=bwd)
    stats = [M.attn_plan_get_stats(p) for p in plans]
    flops = [flops_of(s, wl) * (2.5 if bwd else 1.0) for s in stats]
    tq = q.shape[0]
    outs = [torch.empty(tq, wl.hq, wl.d, dtype=torch.bfloat16, device=dev) for _ in plans]
    lses = [torch.empty(tq, wl.hq, dtype=torch.float32, device=dev) for _ in plans]
    in_bytes = q.numel() * 2 + k.numel() * 2 + v.numel() * 2
    if bwd:
        # the forward's out / lse are inputs of the backward; dout is seeded N(0,1)
        for i, p in enumerate(plans):
            M.attn_masked_fwd(p, q, k, v, outs[i], lses[i], stream)
        gen = torch.Generator(device=dev).manual_seed(wl.seed + 101)
        dout = torch.randn(tq, wl.hq, wl.d, generator=gen, device=dev).to(torch.bfloat16)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        in_bytes += sum(o.numel() * 2 + l.numel() * 4 for o, l in zip(outs, lses)) + dout.numel() * 2
    if fp8:
        # per-tensor e4m3 inputs; V transposed once per plan (a cache would keep it in that layout)
        import workloads as W
        (q8, qs), (k8, ks), (v8, vs) = (W.quantize_e4m3(t) for t in (wl.q, wl.k, wl.v))
        q8, k8, v8 = q8.to(dev), k8.to(dev), v8.to(dev)
        ldvs = [(st["vt_keys"] + 15) // 16 * 16 for st in stats]
        vts = [torch.empty(wl.hkv, wl.d, ld, dtype=torch.uint8, device=dev) for ld in ldvs]
        for p, vt, ld in zip(plans, vts, ldvs):
            M.attn_fp8_transpose_v(p, v8, vt, ld, stream)
        in_bytes = q8.numel() + k8.numel() + v8.numel()
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev) if in_bytes <= L2_BYTES else None

    def run_one(i, p):
        if bwd:
            M.attn_masked_bwd(p, q, k, v, outs[i], lses[i], dout, dq, dk, dv, stream)
        elif fp8:
            M.attn_masked_fwd_fp8(p, q8, k8, vts[i], ldvs[i], qs, ks, vs, outs[i], lses[i], stream)
        else:
            M.attn_masked_fwd(p, q, k, v, outs[i], lses[i], stream)

    def step(events=None):
        for i, p in enumerate(plans):
            if flush is not None:
                flush.fill_(i)
            if events is not None:
                events[i][0].record(stream)
            run_one(i, p)
            if events is not None:
                events[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    for p in plans:
        st = M.attn_plan_check_status(p)
        if st != 0:
            raise RuntimeError(f"forward reported {M.STATUS.get(st, st)}")
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in plans] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank, args.clock_log)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark_start()
    t_start.record(stream)
    for s in range(args.steps):
        step(ev[s])
    t_end.record(stream)
    while not t_end.query():     # poll (GIL released) so the sampler thread runs meanwhile
        time.sleep(2e-4)
    sampler.mark_end()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    launch_ms = [[ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(args.steps)] for i in range(len(plans))]
    for p in plans:
        st = M.attn_plan_check_status(p)
        if st != 0:
            raise RuntimeError(f"forward reported {M.STATUS.get(st, st)}")

    # ---- end to end through the public API: pinned host inputs in, results out, every step ----
    hq_, hk_, hv_ = (t.cpu().pin_memory() for t in (q, k, v))
    ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    hl = [torch.empty(l.shape, dtype=l.dtype).pin_memory() for l in lses]
    e2e_steps = max(3, min(args.steps, 20))

    if bwd:
        hdo = dout.cpu().pin_memory()
        hg = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]

    if fp8:
        hq_, hk_, hv_ = (t.cpu().pin_memory() for t in (q8, k8, vts[0]))

    def e2e_step():
        if fp8:   # host e4m3 q, k and transposed v in; out / lse back
            q8.copy_(hq_, non_blocking=True)
            k8.copy_(hk_, non_blocking=True)
            vts[0].copy_(hv_, non_blocking=True)
            for i, p in enumerate(plans):
                run_one(i, p)
                ho[i].copy_(outs[i], non_blocking=True)
                hl[i].copy_(lses[i], non_blocking=True)
            return
        q.copy_(hq_, non_blocking=True)
        k.copy_(hk_, non_blocking=True)
        v.copy_(hv_, non_blocking=True)
        if bwd:
            dout.copy_(hdo, non_blocking=True)
        for i, p in enumerate(plans):
            if bwd:
                outs[i].copy_(ho[i], non_blocking=True)
                lses[i].copy_(hl[i], non_blocking=True)
                M.attn_masked_bwd(p, q, k, v, outs[i], lses[i], dout, dq, dk, dv, stream)
                for h, t in zip(hg, (dq, dk, dv)):
                    h.copy_(t, non_blocking=True)
            else:
                M.attn_masked_fwd(p, q, k, v, outs[i], lses[i], stream)
                ho[i].copy_(outs[i], non_blocking=True)
                hl[i].copy_(lses[i], non_blocking=True)

    if bwd:   # the host copies of out / lse hold the forward's results
        for i in range(len(plans)):
            ho[i].copy_(outs[i])
            hl[i].copy_(lses[i])

    pipelined = not bwd and not fp8
    if pipelined:
        # Forward end to end with the transfers overlapped: step s's inputs go up on one stream
        # while step s-1 computes and step s-2's results come back on another (two device
        # buffer sets, two pinned result sets). Every step still moves its own inputs in and
        # its own results out inside the timed region.
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        sets = [(q, k, v, outs, lses),
                (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 [torch.empty_like(o) for o in outs], [torch.empty_like(l) for l in lses])]
        host_res = [(ho, hl), ([torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs],
                               [torch.empty(l.shape, dtype=l.dtype).pin_memory() for l in lses])]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(nsteps, e_start=None, e_end=None):
            if e_start is not None:
                e_start.record(s_in)
            for st_ in range(nsteps):
                b = st_ & 1
                qb, kb, vb, ob, lb = sets[b]
                if st_ >= 2:
                    s_in.wait_event(ev_comp[b])      # step st_-2 has read this buffer set
                with torch.cuda.stream(s_in):
                    qb.copy_(hq_, non_blocking=True)
                    kb.copy_(hk_, non_blocking=True)
                    vb.copy_(hv_, non_blocking=True)
                ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if st_ >= 2:
                    stream.wait_event(ev_out[b])      # step st_-2's results have left the outputs
                for i, p in enumerate(plans):
                    M.attn_masked_fwd(p, qb, kb, vb, ob[i], lb[i], stream)
                ev_comp[b].record(stream)
                s_out.wait_event(ev_comp[b])
                with torch.cuda.stream(s_out):
                    for i in range(len(plans)):
                        host_res[b][0][i].copy_(ob[i], non_blocking=True)
                        host_res[b][1][i].copy_(lb[i], non_blocking=True)
                ev_out[b].record(s_out)
            if e_end is not None:
                e_end.record(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(e2e_steps, e0, e1)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
    else:
        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
    h2d = in_bytes if not fp8 else q8.numel() + k8.numel() + vts[0].numel()
    d2h = sum(o.numel() * 2 + l.numel() * 4 for o, l in zip(outs, lses))
    if bwd:
        d2h = len(plans) * sum(t.numel() * 2 for t in (dq, dk, dv))

    # ---- reduce over ranks (reporting only) ----
    (ms, e2e_ms), total_flops = reduce_over_ranks([ms, e2e_ms], sum(flops), dev)
    if rank != 0:
        return
    value = total_flops * args.steps / (ms * 1e-3) / 1e12
    e2e_val = total_flops * e2e_steps / (e2e_ms * 1e-3) / 1e12
    # The timed regions here are short (well under the seconds a GEMM needs to settle at the
    # power cap) and the SM clock stays near its maximum (see "clocks"), so the burst cuBLAS
    # figure is the denominator; the sustained one is used only when the sampled clock fell
    # below 90 % of the maximum.
    peak, pk_src, hbm_peak = choose_peak(clocks, fp8, measure_e4m3_gemm_tflops(dev) if fp8 else None)
    avg_launch_ms = sum(sum(x) for x in launch_ms) / sum(len(x) for x in launch_ms)
    achieved = (sum(flops) / len(flops)) / (avg_launch_ms * 1e-3) / 1e12
    tr = None if (bwd or fp8) else traffic_for(wl.name)
    mask_bytes = sum(s["mask_tile_reads"] for s in stats) * 2048.0
    line = {
        "metric": METRIC_BWD if bwd else METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16",
        "data": "synthetic (seeded N(0,1) bf16, lengths from seed" + ("; per-tensor e4m3)" if fp8 else ")"),
        "config": config_of(wl, args, world),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": tr,
                     "peak_source": pk_src,
                     "kernel": kernel_name(wl, fp8, bwd),
                     "algorithmic_flops_per_launch": sum(flops) / len(flops),
                     "avg_launch_ms": avg_launch_ms,
                     # DRAM GB/s of the captured launch (ncu bytes over this run's mean launch time)
                     "dram_gbs": (tr / (avg_launch_ms * 1e-3) / 1e9) if tr else None},
        "per_mask": [{"mask": m.kind, "unmasked_pairs_per_head": s["unmasked_pairs"], "tflops_per_s":
                      f / (statistics.mean(x) * 1e-3) / 1e12, "ms": statistics.mean(x),
                      "ms_median": statistics.median(x),
                      "tiles_e_f_p": [s["tiles_empty"], s["tiles_full"], s["tiles_partial"]],
                      "kv_splits_max": s["kv_splits_max"], "merge_tiles": s["merge_tiles"],
                      "workspace_bytes": s["workspace_bytes"],
                      "plan_ms": pm,
                      # CUSTOM: the device scan of the packed bits happens inside attn_plan
                      "custom_scan_gbs": (custom_bytes(m) / (pm * 1e-3) / 1e9) if m.kind == "CUSTOM" else None}
                     for m, s, f, x, pm in zip(wl.masks, stats, flops, launch_ms, plan_ms)],
        "mask_gbs": mask_bytes / (sum(statistics.mean(x) for x in launch_ms) * 1e-3) / 1e9,
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "steps": e2e_steps, "transfers_overlapped": pipelined},
        # the forward kernel per plan and step, plus the split-KV merge kernel where a plan split
        # backward: delta, dQ and dK/dV kernels per plan and step
        "gpu_launches": (3 * len(plans) if bwd else sum(1 + (s["merge_tiles"] > 0) for s in stats)) * args.steps,
        "clocks": clocks,
    }
    if wl.paged and not bwd:
        kvb = kv_bytes_read(wl)
        gbs = kvb / (avg_launch_ms * 1e-3) / 1e9
        line["kv_stream"] = {"bytes_per_launch": kvb, "gbs": gbs, "hbm_peak_gbs": hbm_peak,
                             "frac_of_hbm": gbs / hbm_peak}
    if world == 1 and not args.no_per_config and not bwd and not fp8:
        # the other benchmark workloads, each timed on its own after the headline (outside
        # its timed region): every configuration's throughput in the same line
        del q, k, v, outs, lses
        torch.cuda.empty_cache()
        def section(cfg, **kw):
            # a failure here is reported in the entry; the headline above stands on its own
            try:
                return time_config(M, cfg, dev, stream, peak=peak, hbm_peak=hbm_peak, **kw)
            except Exception as e:   # noqa: BLE001 -- recorded in the line, not swallowed
                torch.cuda.synchronize()
                return {"config": cfg, "pass": "bwd" if kw.get("bwd") else "fwd", "error": f"{type(e).__name__}: {e}"}

        line["per_config"] = [section(c, steps=max(3, min(args.steps, 30)), warmup=3)
                              for c in (1, 2, 3, 4, 5) if c != args.config]
        # the backward of the chunk-causal (d = 128) and Gemma2 (d = 256) workloads
        line["backward"] = [section(c, steps=max(3, min(args.steps, 20)), warmup=3, bwd=True) for c in (4, 2)]
    if world == 1 and not args.no_cpu_baseline and not bwd and not fp8:
        pairs, secs, desc = oracle_sample(wl, wl.masks, args.cpu_seconds)
        line["cpu_baseline"] = {"value": 4.0 * wl.d * pairs / secs / 1e12, "unit": "TFLOP/s",
                                "cores": blas_threads(), "kind": "oracle", "sample": desc,
                                "seconds": secs}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=5, choices=[1, 2, 3, 4, 5, 6],
                    help="1-5: the benchmark workloads (5, the long block-dense CUSTOM mask, is the "
                         "headline: the largest single-GPU one); 6: long-context tree verify (split-KV case)")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd"], default="fwd",
                    help="fwd: the forward (the benchmark metric); bwd: the backward pass (workloads 1, 2, 4, 5)")
    ap.add_argument("--dtype", choices=["bf16", "e4m3"], default="bf16",
                    help="e4m3: the fp8 forward (contiguous K/V, head_dim 128 or 256: workloads 2, 4, 5)")
    ap.add_argument("--kv-splits", type=int, default=0,
                    help="split-KV: 0 automatic, 1 never, N >= 2 at most N key ranges per query tile")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--clock-log", default=None,
                    help="folder for the raw nvidia-smi clock samples (default: the temp folder)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other benchmark workloads after the headline")
    ap.add_argument("--shard-rows", action="store_true",
                    help="split ONE problem over the ranks by query rows, with a K/V all-gather per step "
                         "(strong scaling; contiguous K/V workloads)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.shard_rows:
            run_shard_rows(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
