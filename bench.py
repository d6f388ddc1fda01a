"""Benchmark of the LiftQuant decode operator (lq_gemm) on B200.

One step = one lq_gemm call (whiten + lift + +-1 contraction + row scale) over one batch of
synthetic inputs already resident in HBM. The default workload is the Llama-3-70B MLP
gate/up shape (K = 8192 -> N = 28672, d = 10, D = 24: 2.4 bit, batch 1, block-256 Hadamard
whitening), the batch-1 GEMV whose packed-weight bandwidth is the headline; the same run then
times the 2048-token prefill GEMM of that layer (TFLOP/s, nested as "prefill"). Inputs rotate
over enough copies of the packed weights that no timed step finds its codes in L2. Prints one
JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl lq|reference]

Multi-GPU: independent replicas (one process per GPU, launched by torchrun); the path has
no exchange step, so the ranks only meet for the barrier and the max-over-ranks timing.
"""
import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import fractional_bit_weight_b200 as lq  # noqa: E402
from fractional_bit_weight_b200 import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# name -> (workload spec index into synth.workload_specs(cfg), cfg, metric kind)
WORKLOADS = {
    "llama2_7b_qproj_b1": (2, 0, "gemv"),
    "llama3_70b_gateup_b1": (3, 0, "gemv"),
    "llama3_70b_gateup_b4": (3, 1, "gemv"),
    "llama3_70b_gateup_b16": (3, 2, "gemv"),
    "llama3_70b_down_b4": (3, 4, "gemv"),
    "llama3_70b_down_b16": (3, 5, "gemv"),
    "llama3_70b_down_b1": (3, 3, "gemv"),
    "sweep_d10D24_b1": (4, 8, "gemv"),
    "prefill_b2048": (5, 0, "gemm"),
    # encoder: 512 rows of the q_proj shape, seeded 2^(D-d) search per block
    "encode_seeded_512x4096_d10D24": (None, None, "encode"),
}
PREFILL = "prefill_b2048"
# --route: lq_gemm's own choice, or one kernel family through lq_gemm_on_route
ROUTES = {"auto": None, "gemv_i8": lq.ROUTE_GEMV_I8, "gemm_tc": lq.ROUTE_GEMM_TC,
          "gemv_groups": lq.ROUTE_GEMV_GROUPS, "gemv_bulk": lq.ROUTE_GEMV_BULK,
          "gemm_dq": lq.ROUTE_GEMM_DQ}

# the encoder workload: (N, K, d, D, mode, seed); w ~ N(0, 1) stands for whitened weights,
# M ~ N(0, 1/D)
ENCODE = {"encode_seeded_512x4096_d10D24": (512, 4096, 10, 24, lq.LQ_ENCODE_SEEDED, 5)}
# fp32 FMA rate of B200 from its unit counts and clock: 148 SMs x 128 lanes x 2 flop x 1.965 GHz
FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="lq", choices=["lq", "reference"])
    p.add_argument("--workload", default="llama3_70b_gateup_b1", choices=sorted(WORKLOADS))
    p.add_argument("--prefill-steps", type=int, default=10,
                   help="steps of the 2048-token prefill GEMM timed after a GEMV workload "
                        "(reported as the nested 'prefill' object; 0 skips it)")
    p.add_argument("--route", default="auto", choices=sorted(ROUTES),
                   help="kernel family for the lq_gemm call (auto: the library's choice)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout,
                                                 device_id=torch.device("cuda", local))
        else:
            # a host without GPUs runs only the reference arm (the oracle); its ranks meet over gloo
            torch.distributed.init_process_group("gloo", timeout=timeout)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(v, ws):
    if ws == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def source_digest(name):
    """Digest of one kernel source file under fractional_bit_weight_b200/csrc."""
    with open(os.path.join(ROOT, "fractional_bit_weight_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(workload, field):
    """A figure of the workload's dominant kernel from profiles/traffic.json (an ncu capture:
    DRAM bytes per launch, tensor-pipe activity), if the file defining that kernel is
    unchanged since (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(workload)
    try:
        if not ent or ent.get("source_digest") != source_digest(ent["source"]):
            return None
    except (OSError, KeyError):
        return None
    return ent.get(field)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    def __init__(self, index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        names = {
            "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap,
            "hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
            "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
            "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
            "hw_power_brake_slowdown": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown,
        }
        for k, bit in names.items():
            if r & bit:
                self.reasons.add(k)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(0.002)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- workload on the device

class DeviceWorkload:
    def __init__(self, spec, dev, min_copies=1, route=None):
        name, seed, li, K, N, d, D, batch, kw = spec
        self.name, self.K, self.N, self.d, self.D, self.batch = name, K, N, d, D, batch
        layer = synth.build(spec, with_bits=False)     # sign, M, s, x from the seeded recipe
        self.layer = layer
        self.block = layer.block
        self.L = lq.lifted_bits(K, d, D)
        self.packed_bytes = N * self.L // 8 if self.L % 8 == 0 else N * self.L / 8
        self.row_words = lq.row_stride_bytes(K, d, D) // 4
        g = torch.Generator(device=dev)
        g.manual_seed(seed * 1000 + li)
        # rotate over copies so that the bytes streamed between reuses exceed 3x L2
        stored = N * self.row_words * 4
        self.ncopies = max(min_copies, min(64, math.ceil(3 * L2_BYTES / stored)))
        self.packed = []
        for _ in range(self.ncopies):
            b = (torch.randint(0, 2, (N, self.L), generator=g, device=dev, dtype=torch.int8)
                 * 2 - 1).to(torch.int8)
            self.packed.append(lq.pack(b, K, d, D))
            del b
        self.x = _x_tensor(layer).to(dev)
        self.s = torch.from_numpy(np.ascontiguousarray(layer.s_raw)).to(dev)
        self.M = torch.from_numpy(layer.M).to(dev)
        self.sign = torch.from_numpy(layer.sign).to(dev)
        self.y = torch.empty((batch, N), dtype=torch.float32, device=dev)
        self.route = route
        self.ws = lq.new_workspace(batch, K, N, d, D, device=dev, block=self.block, route=route)
        self.stored_bytes = stored

    def step(self, i, x=None, y=None):
        lq.gemm(self.x if x is None else x, self.packed[i % self.ncopies], self.M, self.s,
                self.d, self.D, sign=self.sign, block=self.block,
                y=self.y if y is None else y, workspace=self.ws, route=self.route)

    def algorithmic_bytes(self):
        """Bytes one call must move at minimum: packed codes, s, x, y, M, sign."""
        return (self.packed_bytes + self.s.numel() * self.s.element_size()
                + self.x.numel() * self.x.element_size() + self.y.numel() * 4
                + self.M.numel() * 4 + self.sign.numel())

    def flops(self):
        """The method's algorithmic flops of one call: the lifted contraction (2 B N L) plus the
        lift and the FWHT."""
        G = -(-self.K // self.d)
        fwht = self.batch * self.K * int(math.log2(self.block)) if self.block else 0
        return 2.0 * self.batch * self.N * self.L + 2.0 * self.batch * G * self.d * self.D + fwht

    def actual_route(self):
        if self.route is not None:
            return self.route
        return lq.gemm_route(self.batch, self.K, self.N, self.d, self.D, self.block)

    def tensor_flops(self):
        """Tensor-core flops the route's contraction kernel executes per call: the lifted GEMM
        2 B N Lp (L padded to its 64-coordinate stage); the dequantise-once GEMM 2 B N Kw (the
        G*d inputs padded to 64), which is D/d times fewer than the lifted count."""
        if self.actual_route() == lq.ROUTE_GEMM_DQ:
            G = -(-self.K // self.d)
            Kw = -(-(G * self.d) // 64) * 64
            return 2.0 * self.batch * self.N * Kw
        Lp = -(-self.L // 64) * 64
        return 2.0 * self.batch * self.N * Lp


def _x_tensor(layer):
    if layer.x_dtype == synth.BF16:
        return torch.from_numpy(layer.x_raw.view(np.int16).copy()).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(layer.x_raw))


def kernels_per_step(wl):
    """Kernels one lq_gemm call launches for this workload: as the library reports it, or on a
    forced route its fixed count (staged GEMV, int8 GEMV and lifted GEMM 2; W, xt, GEMM 3)."""
    fixed = {lq.ROUTE_GEMV_BULK: 2, lq.ROUTE_GEMV_I8: 2, lq.ROUTE_GEMM_TC: 2, lq.ROUTE_GEMM_DQ: 3}
    if wl.route in fixed:
        return fixed[wl.route]
    return lq.gemm_launches(wl.batch, wl.K, wl.N, wl.d, wl.D, wl.block)


def time_steps(fn, steps, warmup, ws, ncopies=None):
    """Device time of exactly `steps` calls of fn(i), after `warmup` untimed calls.

    With ncopies (the number of rotating input copies, fn(i) reading copy i % ncopies), the
    calls are captured into CUDA graphs and replayed, so host launch overhead stays out of the
    timing: one graph over all copies in order (0 .. ncopies-1) and, when steps is not a
    multiple of ncopies, one over copies 0 .. (steps % ncopies)-1. The warm replay ends with
    the full graph, so the first timed step reads copy 0, which was last read ncopies - 1 steps
    earlier; every timed step reads a copy that ncopies - 1 other copies were streamed after.
    Returns (seconds, the smallest number of other copies read between two reads of a copy)."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    plan = []
    reuse = None
    if ncopies:
        full, rem = divmod(steps, ncopies)
        g_full = g_rem = None
        if full:
            g_full = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_full):
                for i in range(ncopies):
                    fn(i)
        if rem:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem):
                for i in range(rem):
                    fn(i)
        if g_rem is not None:
            g_rem.replay()
        # the warm-up ends with a pass over every copy in order (eager if no full graph)
        if g_full is not None:
            g_full.replay()
        else:
            for i in range(ncopies):
                fn(i)
        torch.cuda.synchronize()
        plan = [g_full] * full + ([g_rem] if g_rem is not None else [])
        reuse = ncopies - 1
    barrier(ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if plan:
        for g in plan:
            g.replay()
    else:
        for i in range(steps):
            fn(warmup + i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    del plan
    return e0.elapsed_time(e1) / 1e3, reuse   # seconds


# ---------------------------------------------------------------- CPU oracle baseline

def cpu_oracle_run(wl, budget_s=10.0, max_rows=None):
    """Times the fp64 oracle on the host cores over a bounded sample of rows of the same
    workload; returns (value in the workload's unit, sample description, threads)."""
    import oracle
    threads = len(os.sched_getaffinity(0))
    layer = wl.layer
    rng = np.random.Generator(np.random.PCG64(0))
    # measure one small batch of rows to size the sample, then run the sample
    probe = min(wl.N, 64)
    rows = np.arange(probe)
    b = synth.random_signs(rng, (probe, wl.L))
    p = oracle.pack(b, wl.K, wl.d, wl.D)
    t0 = time.perf_counter()
    oracle.forward(layer.x, p, layer.M, layer.s[rows], wl.d, wl.D, sign=layer.sign,
                   block=layer.block, nthreads=threads)
    dt = max(time.perf_counter() - t0, 1e-6)
    n = int(min(wl.N if max_rows is None else max_rows, max(probe, probe * budget_s / dt)))
    b = synth.random_signs(rng, (n, wl.L))
    p = oracle.pack(b, wl.K, wl.d, wl.D)
    s = np.resize(layer.s, n)
    t0 = time.perf_counter()
    oracle.forward(layer.x, p, layer.M, s, wl.d, wl.D, sign=layer.sign, block=layer.block,
                   nthreads=threads)
    dt = time.perf_counter() - t0
    frac = n / wl.N
    sample = (f"{n} of {wl.N} rows x batch {wl.batch} ({frac:.3f} of one call), fp64 oracle, "
              f"{threads} OpenMP threads")
    return frac, dt, sample, threads


# ---------------------------------------------------------------- main

def measure(wl, name, kind, steps, warmup, ws, local, peaks, peak_src):
    """Times `steps` calls of the workload (inputs resident in HBM) and returns the headline
    fields of its JSON line."""
    with ClockSampler(local) as clk:
        secs, reuse = time_steps(wl.step, steps, warmup, ws, ncopies=wl.ncopies)
    secs = max_over_ranks(secs, ws)
    per_step = secs / steps
    gbs = wl.packed_bytes * steps * ws / secs / 1e9
    tflops = wl.flops() * steps * ws / secs / 1e12
    if kind == "gemv":
        metric, value, unit = "lq_gemv_packed_weight_GBps", gbs, "GB/s"
        achieved = wl.algorithmic_bytes() / per_step / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": recorded_traffic(name, "dram_bytes_per_launch"),
                "peak_source": f"{peak_src} hbm_gbs (copy, read+write)",
                "packed_frac": wl.packed_bytes / per_step / 1e9 / peak}
    else:
        # value: the method's algorithmic (lifted) flops per second, comparable across routes;
        # roofline: the flops the tensor cores actually execute on this route, per second of
        # the whole call (all its kernels), against the measured dense peak
        metric, value, unit = "lq_prefill_gemm_TFLOPs", tflops, "TFLOP/s"
        achieved = wl.tensor_flops() / per_step / 1e12
        # the burst figure: the timed region is short and the clocks stay at their maximum
        # (the sampled clocks are in the same line); fp16 dense rate = bf16 dense rate
        peak = float(peaks.get("bf16_tflops", peaks.get("bf16_tflops_sustained")))
        route = wl.actual_route()
        rname = {lq.ROUTE_GEMM_TC: "lifted tcgen05 GEMM", lq.ROUTE_GEMM_DQ:
                 "dequantise-once: fp16 W = M b, then a dense tcgen05 GEMM"}.get(route, str(route))
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": recorded_traffic(name, "dram_bytes_per_launch"),
                "tensor_pipe_active": recorded_traffic(name, "tensor_pipe_active"),
                "route": rname, "executed_tensor_flops": wl.tensor_flops(),
                "algorithmic_flops": wl.flops(),
                "peak_source": f"{peak_src} bf16_tflops (burst; fp16 dense = bf16 dense)"}
    streamed = reuse * wl.stored_bytes
    l2 = (f"{wl.ncopies} copies of the packed weights ({wl.ncopies * wl.stored_bytes / 1e6:.0f} "
          f"MB) read in rotation, warm-up included: between two reads of a copy "
          f"{reuse} other copies ({streamed / 1e6:.0f} MB"
          f"{' > L2' if streamed > L2_BYTES else ' <= L2'}) are streamed")
    if kind == "gemm":
        l2 += f"; y alone is {wl.y.numel() * 4 / 1e6:.0f} MB per step"
    return {
        "metric": metric, "value": value, "unit": unit, "ms_per_step": per_step * 1e3,
        "config": {"workload": wl.name, "K": wl.K, "N": wl.N, "d": wl.d, "D": wl.D,
                   "batch": wl.batch, "bits_per_weight": wl.D / wl.d, "hadamard_block": wl.block,
                   "packed_bytes": wl.packed_bytes, "parallelism": f"replicas x{ws}",
                   "l2": l2},
        "roofline": roof,
        "gpu_launches": kernels_per_step(wl) * steps,
        "clocks": clk.summary(),
        "tflops": tflops,
    }


def main():
    args = parse()
    ws, rank, local = dist_setup()
    cfg, idx, kind = WORKLOADS[args.workload]
    if kind == "encode":
        return encode_main(args, ws, rank, local)
    spec = synth.workload_specs(cfg)[idx]
    if args.impl == "reference":
        return reference_arm(args, spec, kind, ws, rank)

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = DeviceWorkload(spec, dev, route=ROUTES[args.route])
    peaks, peak_src = measured_peaks()
    m = measure(wl, args.workload, kind, args.steps, args.warmup, ws, local, peaks, peak_src)

    out = {
        "metric": m["metric"], "value": m["value"], "unit": m["unit"], "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": m["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded: random sign codes, N(0,1/D) M, N(0,1) bf16 x)",
        "config": m["config"],
        "roofline": m["roofline"],
        "gpu_launches": m["gpu_launches"],
        "timing": "CUDA graphs of the steps, replayed; CUDA events on the launching stream",
        "clocks": m["clocks"],
    }
    if kind == "gemv":
        out["tflops"] = m["tflops"]
    if not args.no_e2e:
        out["e2e"] = e2e_run(wl, args, ws)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        frac, dt, sample, threads = cpu_oracle_run(wl)
        cpu_val = (wl.packed_bytes * frac / dt / 1e9) if kind == "gemv" else \
            (wl.flops() * frac / dt / 1e12)
        out["cpu_baseline"] = {"value": cpu_val, "unit": m["unit"], "cores": threads,
                               "kind": "oracle", "sample": sample}
    del wl
    if args.prefill_steps > 0 and kind == "gemv":
        # the second half of the metric: the 2048-token prefill GEMM, timed in the same run
        pcfg, pidx, _ = WORKLOADS[PREFILL]
        pwl = DeviceWorkload(synth.workload_specs(pcfg)[pidx], dev, min_copies=2)
        p = measure(pwl, PREFILL, "gemm", args.prefill_steps, max(3, args.warmup // 4), ws,
                    local, peaks, peak_src)
        out["prefill"] = {"metric": p["metric"], "value": p["value"], "unit": p["unit"],
                          "steps": args.prefill_steps, "ms_per_step": p["ms_per_step"],
                          "config": p["config"], "roofline": p["roofline"],
                          "gpu_launches": p["gpu_launches"], "clocks": p["clocks"]}
        out["gpu_launches"] += p["gpu_launches"]
        del pwl
    if rank == 0:
        print(json.dumps(out))
    if ws > 1:
        torch.distributed.destroy_process_group()


def encode_inputs(name):
    N, K, d, D, mode, seed = ENCODE[name]
    rng = np.random.Generator(np.random.PCG64([seed, N, K]))
    M = (rng.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)
    w = rng.standard_normal((N, K)).astype(np.float32)
    return N, K, d, D, mode, M, w


def encode_oracle_sample(name, budget_s=10.0):
    """The oracle's seeded search on the host cores over the first rows of the workload, sized
    to about budget_s; returns (weights per second, sample description, threads)."""
    import oracle
    N, K, d, D, mode, M, w = encode_inputs(name)
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    oracle.encode_rows(w[:1, :d * 64], M, d, D, mode, nthreads=threads)     # 64 blocks
    per_block = max(time.perf_counter() - t0, 1e-6) / 64
    G = -(-K // d)
    nblk = int(max(threads, min(N * G, budget_s / per_block)))
    rows, cols = max(1, nblk // G), min(K, nblk * d)
    t0 = time.perf_counter()
    oracle.encode_rows(w[:rows, :cols], M, d, D, mode, nthreads=threads)
    dt = time.perf_counter() - t0
    done = rows * cols
    return done / dt, f"{rows} rows x {cols} inputs of {N} x {K}, fp64 oracle", threads


def encode_main(args, ws, rank, local):
    """One step = one lq_encode call over the whole matrix (weights resident in HBM)."""
    name = args.workload
    N, K, d, D, mode, M, w = encode_inputs(name)
    G = -(-K // d)
    cand = N * G * (1 << (D - d)) if mode == lq.LQ_ENCODE_SEEDED else N * G * (1 << D)
    if args.impl == "reference":
        if rank == 0:
            v, sample, threads = encode_oracle_sample(name)
            print(json.dumps({
                "impl": "reference", "metric": "lq_encode_weights_per_s", "value": v,
                "unit": "weights/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": N * K / v * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": name, "N": N, "K": K, "d": d, "D": D, "mode": "seeded"},
                "cpu_baseline": {"value": v, "unit": "weights/s", "cores": threads,
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": v, "unit": "weights/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}))
        if ws > 1:
            torch.distributed.destroy_process_group()
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wd, Md = torch.from_numpy(w).to(dev), torch.from_numpy(M).to(dev)
    b = torch.empty((N, G, D), dtype=torch.int8, device=dev)
    lib = lq.lib()

    def step(i, wsrc=None):
        rc = lib.lq_encode(wd.data_ptr() if wsrc is None else wsrc.data_ptr(), N, K,
                           Md.data_ptr(), d, D, mode, b.data_ptr(), None,
                           torch.cuda.current_stream().cuda_stream)
        if rc != lq.LQ_OK:
            raise RuntimeError(lib.lq_last_error().decode())

    with ClockSampler(local) as clk:
        secs, _ = time_steps(step, args.steps, args.warmup, ws)
    secs = max_over_ranks(secs, ws)
    per_step = secs / args.steps
    value = N * K * args.steps * ws / secs
    # algorithmic work of the incremental walk: per candidate 2d flops for u, d for r_F, d for
    # e and 2d for the distance (6d), against the fp32 FMA rate
    achieved = cand * 6 * d / per_step / 1e12
    out = {
        "metric": "lq_encode_weights_per_s", "value": value, "unit": "weights/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded: w N(0,1), M N(0,1/D))",
        "config": {"workload": name, "N": N, "K": K, "d": d, "D": D, "mode": "seeded",
                   "candidates_per_step": cand, "parallelism": f"replicas x{ws}",
                   "l2": f"w is {N * K * 4 / 1e6:.1f} MB; the search is ALU-bound"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": FP32_TFLOPS,
                     "unit": "TFLOP/s", "frac": achieved / FP32_TFLOPS, "traffic": None,
                     "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz"},
        "gpu_launches": args.steps,
        "timing": "CUDA events on the launching stream",
        "clocks": clk.summary(),
    }
    if not args.no_e2e:
        w_host = torch.from_numpy(w).pin_memory()
        b_host = torch.empty((N, G, D), dtype=torch.int8).pin_memory()
        w_dev = torch.empty_like(wd)

        def e2e_step(i):
            w_dev.copy_(w_host, non_blocking=True)
            step(i, w_dev)
            b_host.copy_(b, non_blocking=True)

        e2e_secs = max_over_ranks(time_steps(e2e_step, args.steps, args.warmup, ws)[0], ws)
        out["e2e"] = {"value": N * K * args.steps * ws / e2e_secs, "unit": "weights/s",
                      "h2d_bytes_per_step": N * K * 4, "d2h_bytes_per_step": N * G * D}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, sample, threads = encode_oracle_sample(name)
        out["cpu_baseline"] = {"value": v, "unit": "weights/s", "cores": threads,
                               "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(out))
    if ws > 1:
        torch.distributed.destroy_process_group()


def e2e_run(wl, args, ws):
    """Same metric through the public call with host buffers: every step copies x from pinned
    host memory to the device and y back, inside the timed region."""
    x_host = wl.x.cpu().pin_memory()
    y_host = torch.empty(wl.y.shape, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(wl.x)

    def step(i):
        x_dev.copy_(x_host, non_blocking=True)
        wl.step(i, x=x_dev)
        y_host.copy_(wl.y, non_blocking=True)

    secs = max_over_ranks(time_steps(step, args.steps, args.warmup, ws)[0], ws)
    if wl.flops() and WORKLOADS[args.workload][2] == "gemm":
        v, u = wl.flops() * args.steps * ws / secs / 1e12, "TFLOP/s"
    else:
        v, u = wl.packed_bytes * args.steps * ws / secs / 1e9, "GB/s"
    return {"value": v, "unit": u, "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": y_host.numel() * 4}


def reference_arm(args, spec, kind, ws, rank):
    """The oracle, as it stands, on the host cores: each step is a bounded sample of the
    workload. Under torchrun only rank 0 runs it."""
    if rank != 0:
        if ws > 1:
            torch.distributed.destroy_process_group()
        return
    import oracle
    name, seed, li, K, N, d, D, batch, kw = spec
    layer = synth.build(spec, with_bits=False)
    L = lq_free_lifted_bits(K, d, D)
    threads = len(os.sched_getaffinity(0))
    rng = np.random.Generator(np.random.PCG64(1))
    rows = min(N, 256 if kind == "gemv" else 16)
    toks = min(batch, 64)
    b = synth.random_signs(rng, (rows, L))
    p = oracle.pack(b, K, d, D)
    x = layer.x[:toks]

    def step():
        oracle.forward(x, p, layer.M, layer.s[:rows], d, D, sign=layer.sign, block=layer.block,
                       nthreads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    secs = time.perf_counter() - t0
    frac = rows / N * toks / batch
    packed = N * L / 8
    G = -(-K // d)
    flops = 2.0 * batch * N * L + 2.0 * batch * G * d * D
    if kind == "gemv":
        metric, unit = "lq_gemv_packed_weight_GBps", "GB/s"
        value = packed * frac * args.steps / secs / 1e9
    else:
        metric, unit = "lq_prefill_gemm_TFLOPs", "TFLOP/s"
        value = flops * frac * args.steps / secs / 1e12
    sample = f"{rows} of {N} rows x {toks} of {batch} tokens per step, fp64 oracle"
    out = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": name, "K": K, "N": N, "d": d, "D": D, "batch": batch},
           "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))
    if ws > 1:
        torch.distributed.destroy_process_group()


def lq_free_lifted_bits(K, d, D):
    return (K + d - 1) // d * D


if __name__ == "__main__":
    main()
