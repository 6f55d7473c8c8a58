#!/usr/bin/env python
"""Benchmark of the fused per-chunk inverse + WY hot path on B200.

Workload (one "step"): the fused chunk pipeline (A from K K^T, Neumann order
N=3 with the band mask and S=8 residual steps, then W = T diag(beta) K and
U = T diag(beta) V) over B=4, H=16, T=4096, k=64, d=128, bf16 — 4096 chunks.
Inputs are seeded synthetic tensors with the recipe of
``gated_deltanet_chunk_02_b200.inputs``; three input/output copies rotate so
each step's 270 MB working set is cold in the 126 MB L2.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded sample of the same workload instead.

Multi-GPU (torchrun): every rank runs its own independent batch (weak scaling,
no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(B=4, H=16, T=4096, k=64, d=128, dtype="bf16", N=3, mask=1, S=8, gated=0)
METRIC = "GDN chunk inverse+WY: chunks/s and % of roofline (k=64, d=128, bf16)"
ROTATE = 3


def algorithmic_bytes_per_chunk(k: int, d: int, elem: int) -> int:
    """K, V in + beta, g in + W, U out (the fused kernel reads and writes nothing else)."""
    return 2 * k * d * elem + 2 * k * 4 + 2 * k * d * elem


def algorithmic_flops_per_chunk(k: int, d: int, N: int, S: int) -> int:
    """Dense product flops the method issues per chunk: K K^T, (N-1) chain
    products, the residual (A T0, S-1 Horner products, T0 Q) and the two WY
    products."""
    kk = 2 * k * k * d
    chain = (N - 1) * 2 * k ** 3
    resid = (S + 1) * 2 * k ** 3 if S > 0 else 0
    wy = 2 * 2 * k * k * d
    return kk + chain + resid + wy


def load_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


KERNEL_SOURCES = {
    "fused": ["tc.cu", "tc.h", "common.cuh"],
    "neumann": ["tc.cu", "tc.h", "common.cuh"],
    "int8": ["tc.cu", "tc.h", "common.cuh"],
    "build_A": ["tc.cu", "tc.h", "common.cuh"],
    "wy": ["tc.cu", "tc.h", "common.cuh"],
    "fwdsub": ["simt.cu", "kernels.h", "common.cuh"],
    "forward": ["tc.cu", "scan.cu", "simt.cu", "common.cuh"],
}


def kernel_source_hash(kernel: str = "fused") -> str:
    """Hash of the CUDA sources the kernel is built from (ties a recorded ncu
    traffic figure to the code it was measured on)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_deltanet_chunk_02_b200", "csrc")
    for name in KERNEL_SOURCES.get(kernel, sorted(os.listdir(csrc))):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str) -> float | None:
    """DRAM bytes per launch from the committed ncu summary, or None when the
    summary is missing or was taken on different kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                key, v = line.split(":", 1)
                vals[key.strip()] = v.strip()
    if vals.get(f"{kernel}.source_hash") != kernel_source_hash(kernel):
        return None
    v = vals.get(f"{kernel}.dram_bytes_per_launch")
    return float(v) if v else None


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML
    every ~2 ms while the timed region runs (reading only; no setting is
    touched)."""

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu = gpu_index
        self.period = period_s
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            h = pynvml.nvmlDeviceGetHandleByIndex(self._physical_index())
            self._h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:            # NVML missing: report no samples
            self._nvml = None
        return self

    def _physical_index(self) -> int:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[self.gpu])
            except (ValueError, IndexError):
                pass
        return self.gpu

    def _sample(self):
        n = self._nvml
        mhz = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
        rs = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        self.samples.append((mhz, rs))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                break
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)
        if self._nvml is not None:
            try:
                self._sample()
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = sorted(m for m, _ in self.samples)
        reasons = set()
        for _, rs in self.samples:
            for name, const in self.REASONS:
                bit = getattr(self._nvml, const, 0) if self._nvml else 0
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def shard_seed(rank: int, copy: int) -> int:
    """Seed of input copy `copy` on rank `rank`: every rank draws its own batch
    (weak scaling: the units of work are independent chunks, no exchange)."""
    return 1000 * rank + copy


def aggregate_throughput(units_per_rank: int, world: int, ms_total: float, steps: int) -> float:
    """Whole-job units/s: the units all ranks processed over the max-over-ranks time."""
    return units_per_rank * world / (ms_total * 1e-3 / steps)


class OracleInputs:
    """The workload's inputs drawn once, chunked and upcast to float64 for the
    oracle; ``window(i, n)`` gives n consecutive chunks starting at chunk i
    (wrapping), so consecutive timed steps see different chunks."""

    def __init__(self, w: dict, seed: int = 0):
        import oracle as O
        from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs, as_f64_numpy
        wl = Workload(B=w["B"], H=w["H"], T=w["T"], k=w["k"], d=w["d"], dtype=w["dtype"])
        inp = make_inputs(wl, seed=seed)
        k = w["k"]
        self.K = O.to_chunks(as_f64_numpy(inp["K"]), k)
        self.V = O.to_chunks(as_f64_numpy(inp["V"]), k)
        self.b = O.to_chunks(as_f64_numpy(inp["beta"]), k)
        self.g = O.to_chunks(as_f64_numpy(inp["g"]), k)
        self.nc = self.K.shape[0]

    def window(self, i: int, n: int):
        import numpy as np
        idx = (i + np.arange(n)) % self.nc
        return self.K[idx], self.V[idx], self.b[idx], self.g[idx]


def cpu_oracle_step(w: dict, data: OracleInputs, first: int, n: int) -> tuple[float, int]:
    """Time the oracle (as it stands) on n chunks of the workload starting at
    chunk ``first``: A, the inverse, W and U.  Returns (seconds, BLAS threads)."""
    import oracle as O
    from threadpoolctl import threadpool_info
    K, V, b, g = data.window(first, n)
    t0 = time.perf_counter()
    A = O.build_A(K, b, g)
    T = O.invert_neumann(A, w["N"], bool(w["mask"]), w["S"])
    O.wy(T, K, V, b, g if w["gated"] else None)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()
                   if i.get("user_api") == "blas"] or [1])
    return dt, threads


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_oracle_parallel(w: dict, data: OracleInputs, first: int, n: int,
                        threads: int | None = None) -> tuple[float, int]:
    """Time the oracle (as it stands) on n chunks starting at chunk ``first``,
    split into one window per host core and run on a thread pool with BLAS
    held to one thread per call (numpy releases the GIL inside its products
    and array loops, so the windows run in parallel).  Returns (seconds,
    threads used)."""
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor

    import oracle as O
    from threadpoolctl import threadpool_limits
    threads = max(1, min(threads or host_cores(), n))
    cuts = np.linspace(0, n, threads + 1).astype(int)
    wins = [data.window(first + a, b - a) for a, b in zip(cuts, cuts[1:]) if b > a]

    def one(win):
        K, V, b, g = win
        A = O.build_A(K, b, g)
        T = O.invert_neumann(A, w["N"], bool(w["mask"]), w["S"])
        O.wy(T, K, V, b, g if w["gated"] else None)

    with threadpool_limits(limits=1), ThreadPoolExecutor(max_workers=len(wins)) as ex:
        t0 = time.perf_counter()
        list(ex.map(one, wins))
        dt = time.perf_counter() - t0
    return dt, len(wins)


def cpu_forward_baseline(wl, seed: int, N: int, mask: int, S: int) -> dict:
    """The oracle's chunk-wise forward (A, the inverse, the chunk scan) on every
    head of the workload, one head per host core at a time, and its token-by-
    token recurrence on the first 4096 tokens of one head on one core."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle as O
    from gated_deltanet_chunk_02_b200.inputs import make_inputs, as_f64_numpy
    from threadpoolctl import threadpool_limits
    inp = make_inputs(wl, seed=seed, with_q=True)
    k, BH = wl.k, wl.B * wl.H
    ch = {key: O.to_chunks(as_f64_numpy(inp[key]), k).reshape(BH, wl.T // k, k, -1)
          for key in ("Q", "K", "V")}
    ch.update({key: O.to_chunks(as_f64_numpy(inp[key]), k).reshape(BH, wl.T // k, k)
               for key in ("beta", "g")})

    def head(h):
        A = O.build_A(ch["K"][h], ch["beta"][h], ch["g"][h])
        T = O.invert_neumann(A, N, bool(mask), S)
        O.chunk_forward(*(ch[key][h:h + 1] for key in ("Q", "K", "V", "beta", "g")), T[None])

    threads = max(1, min(host_cores(), BH))
    with threadpool_limits(limits=1), ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        list(ex.map(head, range(BH)))
        dt = time.perf_counter() - t0
    n_tok = min(4096, wl.T)
    f = lambda key: as_f64_numpy(inp[key]).reshape(BH, wl.T, -1)[:1, :n_tok]
    g = lambda key: as_f64_numpy(inp[key]).reshape(BH, wl.T)[:1, :n_tok]
    with threadpool_limits(limits=1):
        t1 = time.perf_counter()
        O.token_recurrence(f("Q"), f("K"), f("V"), g("beta"), g("loggate"))
        dt1 = time.perf_counter() - t1
    nc = BH * (wl.T // k)
    return {"value": nc / dt, "unit": "chunks/s", "cores": threads, "kind": "oracle",
            "sample": f"all {BH} heads x {wl.T // k} chunks (the whole forward): A, the inverse "
                      f"(N={N}, mask={mask}, S={S}) and the chunk scan, fp64, one head per thread",
            "token_recurrence": {"value": (n_tok // k) / dt1, "unit": "chunks/s", "cores": 1,
                                 "sample": f"first {n_tok} tokens of one head, token by token"}}


# chunks the reference arm processes over a whole run (warm-up and timed steps
# together), so that any --steps / --warmup ends in a few minutes of host time
REFERENCE_CHUNK_BUDGET = 32768


def reference_window(steps: int, warmup: int, sample_chunks: int) -> int:
    """Chunks per step of the reference arm: at most ``sample_chunks``, and
    few enough that all steps together stay within the budget (at least 1)."""
    return max(1, min(sample_chunks, REFERENCE_CHUNK_BUDGET // max(1, steps + warmup)))


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, each step a bounded window of the workload
    (rank 0 only)."""
    if rank != 0:
        return 0
    w = dict(WORKLOAD)
    data = OracleInputs(w)
    nc = data.nc
    n_sample = reference_window(args.steps, args.warmup, args.sample_chunks)
    pos = 0
    for _ in range(args.warmup):
        cpu_oracle_parallel(w, data, pos, n_sample)
        pos += n_sample
    total, threads = 0.0, 1
    for _ in range(args.steps):
        dt, threads = cpu_oracle_parallel(w, data, pos, n_sample)
        pos += n_sample
        total += dt
    value = n_sample * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "chunks/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, nc),
        "ms_per_step_scaled_to_workload": 1e3 * total / args.steps * nc / n_sample,
        "cpu_baseline": {"value": value, "unit": "chunks/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n_sample} consecutive of {nc} chunks per step (a new window "
                                   f"each step, split over {threads} host threads); ms_per_step is "
                                   f"the measured time of one such step"},
        "e2e": {"value": value, "unit": "chunks/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: dict, nc: int, rotate: int = ROTATE) -> dict:
    mask = "band mask" if w["mask"] else "no mask"
    return {"workload": f"fused chunk inverse+WY (A=KK^T gated, Neumann N={w['N']} + {mask}, "
                        f"S={w['S']} residual, W/U), B=4 H=16 T=4096 k=64 d=128 bf16",
            "B": w["B"], "H": w["H"], "T": w["T"], "k": w["k"], "d": w["d"], "N": w["N"],
            "mask": w["mask"], "S": w["S"], "chunks": nc,
            "l2": f"inputs larger than L2: {rotate} rotating input/output sets of 270 MB"}



# component kernels that take the series order / mask, and the residual order
SERIES_KERNELS = ("neumann", "newton", "fused_raw", "int8", "int8_residual", "int16",
                  "int16_residual", "forward")
RESIDUAL_KERNELS = ("neumann", "fused_raw", "int8_residual", "int16_residual", "forward")


def run_component(args, world, rank, local, dev) -> int:
    """Device-timed run of one component kernel (A, Neumann, fwdsub, INT8, WY
    or the full forward) on its own workload; same JSON keys as the headline."""
    import torch
    from gated_deltanet_chunk_02_b200 import gdn
    from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs
    kern = args.kernel
    if kern == "forward":
        wl = Workload(B=1, H=16, T=65536, k=64, dtype="bf16")
    elif kern == "fused_raw":                       # the headline step plus its prologue
        wl = Workload(B=4, H=16, T=4096, k=args.k or 64, dtype="bf16")
    else:
        k = args.k or 64
        wl = Workload(B=1, H=32, T=16384, k=k, dtype="bf16")
    k, d, nc = wl.k, wl.d, wl.n_chunks
    stream = torch.cuda.current_stream(dev)
    sets = []
    for r in range(args.rotate):
        inp = make_inputs(wl, seed=shard_seed(rank, r), with_q=(kern == "forward"),
                          raw_keys=(kern == "fused_raw"))
        st = {key: v.to(dev) for key, v in inp.items()}
        st["A"] = torch.empty(wl.B, wl.H, wl.T // k, k, k, device=dev)
        st["T"] = torch.empty_like(st["A"])
        if kern in ("neumann", "newton", "blocked", "fwdsub", "int8", "int8_residual", "int16",
                    "int16_residual", "wy"):
            gdn.gdn_build_A(st["K"], st["beta"], st["g"], st["A"], k, stream=stream)
        if kern == "wy":
            gdn.gdn_invert_fwdsub(st["A"], st["T"], stream=stream)
        if kern in ("wy", "forward", "fused_raw"):
            st["W"] = torch.empty_like(st["K"])
            st["U"] = torch.empty_like(st["V"])
        if kern == "forward":
            st["O"] = torch.empty_like(st["Q"])
            st["Sf"] = torch.empty(wl.B, wl.H, d, d, device=dev)
            st["ws"] = torch.empty(gdn.gdn_forward_workspace_bytes(st["K"], k), dtype=torch.uint8,
                                   device=dev)
        sets.append(st)

    def step(i):
        st = sets[i % len(sets)]
        if kern == "neumann":
            gdn.gdn_invert_neumann(st["A"], st["T"], args.N, args.mask, args.S, gdn.GDN_PREC_F16,
                                   stream=stream)
        elif kern == "fused_raw":
            gdn.gdn_chunk_wy_fused_raw(st["K"], st["V"], st["beta"], st["loggate"], args.N,
                                       args.mask, args.S, 0, st["W"], st["U"], k=k, stream=stream)
        elif kern == "newton":
            gdn.gdn_invert_newton(st["A"], st["T"], args.N, args.mask, args.M, stream=stream)
        elif kern == "fwdsub":
            gdn.gdn_invert_fwdsub(st["A"], st["T"], stream=stream)
        elif kern == "blocked":
            gdn.gdn_invert_blocked(st["A"], st["T"], stream=stream)
        elif kern == "int8":
            gdn.gdn_invert_neumann_i8(st["A"], st["T"], args.N, args.mask, stream=stream)
        elif kern == "int8_residual":
            gdn.gdn_invert_neumann_i8_residual(st["A"], st["T"], args.N, args.mask, args.S,
                                               stream=stream)
        elif kern == "int16":
            gdn.gdn_invert_neumann_i16(st["A"], st["T"], args.N, args.mask, stream=stream)
        elif kern == "int16_residual":
            gdn.gdn_invert_neumann_i16_residual(st["A"], st["T"], args.N, args.mask, args.S,
                                                stream=stream)
        elif kern == "build_A":
            gdn.gdn_build_A(st["K"], st["beta"], st["g"], st["A"], k, stream=stream)
        elif kern == "wy":
            gdn.gdn_wy(st["T"], st["K"], st["V"], st["beta"], None, st["W"], st["U"], stream=stream)
        else:
            gdn.gdn_forward(st["Q"], st["K"], st["V"], st["beta"], st["g"], None, args.N,
                            args.mask, args.S, 0, st["O"], st["Sf"], st["ws"], k=k, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    assert gdn.gdn_get_status(stream) == gdn.GDN_OK
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launches0 = gdn.gdn_launch_count()
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    launches = gdn.gdn_launch_count() - launches0
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    assert gdn.gdn_get_status(stream) == gdn.GDN_OK
    ms_step = ms / args.steps
    # algorithmic bytes and dense-product flops per chunk
    kk2 = k * k * 4
    kd = k * d * 2
    chain = (args.N - 1 + (args.S + 1 if args.S > 0 else 0)) * 2 * k ** 3
    per = {
        "neumann": (2 * kk2, chain),
        "newton": (2 * kk2, (args.N - 1 + 2 * args.M) * 2 * k ** 3),
        "fused_raw": (algorithmic_bytes_per_chunk(k, d, 2),
                      algorithmic_flops_per_chunk(k, d, args.N, args.S)),
        "fwdsub": (2 * kk2, 2 * k ** 3 // 6),
        "blocked": (2 * kk2, 4 * 2 * k ** 3),
        "int8": (2 * kk2, (args.N - 1) * 2 * k ** 3),
        "int16": (2 * kk2, (args.N - 1) * 2 * k ** 3),
        "int8_residual": (2 * kk2, (args.N - 1 + args.S + 1) * 2 * k ** 3),
        "int16_residual": (2 * kk2, (args.N - 1 + args.S + 1) * 2 * k ** 3),
        "build_A": (kd + 8 * k + kk2, 2 * k * k * d),
        "wy": (kk2 + 2 * kd + 4 * k + 2 * kd, 4 * k * k * d),
        "forward": (4 * kd + 8 * k, algorithmic_flops_per_chunk(k, d, args.N, args.S)
                    + 2 * (4 * k * d * d + k * k * d + k * k * d)),
    }[kern]
    bytes_l, flops_l = per[0] * nc, per[1] * nc
    peaks, peak_kind = load_peaks()
    # the integer kernels' products are int8 MMAs: their tensor peak is the
    # measured bf16 peak times the nominal int8 : bf16 ratio (4.5 : 2.25)
    integer = kern in ("int8", "int8_residual", "int16", "int16_residual")
    tc_peak = float(peaks["bf16_tflops"]) * (2.0 if integer else 1.0)
    tc_kind = peak_kind + (" x 2 (nominal int8:bf16 ratio)" if integer else "")
    gbs = bytes_l / (ms_step * 1e-3) / 1e9
    tfl = flops_l / (ms_step * 1e-3) / 1e12
    t_hbm = bytes_l / (float(peaks["hbm_gbs"]) * 1e9)
    t_tc = flops_l / (tc_peak * 1e12)
    bound = "hbm" if (t_hbm >= t_tc or kern == "fwdsub") else "tensor"
    line = {
        "metric": f"{kern} kernel: chunks/s (k={k}, d={d}, bf16 data)",
        "value": aggregate_throughput(nc, world, ms, args.steps), "unit": "chunks/s",
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{kern}, B={wl.B} H={wl.H} T={wl.T} k={k} d={d}"
                               + (f" N={args.N} mask={args.mask}" if kern in SERIES_KERNELS else "")
                               + (f" S={args.S}" if kern in RESIDUAL_KERNELS else "")
                               + (f" M={args.M}" if kern == "newton" else ""),
                   "chunks": nc},
        "roofline": {"bound": bound, "achieved": gbs if bound == "hbm" else tfl,
                     "peak": float(peaks["hbm_gbs"]) if bound == "hbm" else tc_peak,
                     "unit": "GB/s" if bound == "hbm" else ("TOP/s" if integer else "TFLOP/s"),
                     "frac": gbs / float(peaks["hbm_gbs"]) if bound == "hbm" else tfl / tc_peak,
                     "traffic": recorded_traffic(kern),
                     "peak_source": peak_kind if bound == "hbm" else tc_kind,
                     "tensor_peak": tc_peak, "tensor_peak_source": tc_kind,
                     "roofline_frac": max(t_hbm, t_tc) / (ms_step * 1e-3), "tflops": tfl,
                     "bytes_per_launch": bytes_l, "flops_per_launch": flops_l},
        "clocks": clocks.summary(), "e2e": None, "gpu_launches": launches,
    }
    if kern == "forward" and rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_forward_baseline(wl, shard_seed(rank, 0), args.N, args.mask,
                                                    args.S)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0

def run_decode(args, world, rank, local, dev) -> int:
    """Device-timed decode steps: every sequence of the batch advances by
    ``--tokens`` tokens through ``gdn_decode`` (16 query/key heads, 32 value
    heads, d = 128, fp32 state).  State sets rotate so that the timed steps
    touch more than L2 holds."""
    import torch
    from gated_deltanet_chunk_02_b200 import gdn
    from gated_deltanet_chunk_02_b200.inputs import make_decode_inputs
    B, Hk, Hv, n, d = args.batch, 16, 32, args.tokens, 128
    elem = 2
    per_set = B * Hv * d * d * 4
    sets_n = max(args.rotate, -(-3 * 64 * 2 ** 20 // per_set))      # >= 192 MB in total
    stream = torch.cuda.current_stream(dev)
    base = make_decode_inputs(B, Hk, Hv, n, d=d, dtype="bf16", seed=shard_seed(rank, 0))
    sets = []
    for r in range(sets_n):
        st = {key: v.to(dev) for key, v in base.items()}
        st["O"] = torch.empty_like(st["V"])
        sets.append(st)

    def steps_all(st_):
        for st in sets:
            gdn.gdn_decode(st["Q"], st["K"], st["V"], st["beta"], st["loggate"], st["S0"],
                           st["O"], stream=st_)

    # one CUDA graph replays a decode step on every state set (a serving loop
    # replays its captured step; at batch 1 host launch costs would otherwise
    # be timed instead of the kernel)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        steps_all(side)
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    assert gdn.gdn_get_status(stream) == gdn.GDN_OK
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        steps_all(torch.cuda.current_stream(dev))
    replays = max(1, args.steps // sets_n)
    for _ in range(max(1, args.warmup // sets_n + 1)):
        graph.replay()
    torch.cuda.synchronize(dev)
    assert gdn.gdn_get_status(stream) == gdn.GDN_OK
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for _ in range(replays):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    steps = replays * sets_n
    launches = steps                              # one kernel per decode step
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    assert gdn.gdn_get_status(stream) == gdn.GDN_OK
    del graph
    ms_step = ms / steps
    # state read + written once per call; per token q, k (per key head), v, o
    # (per value head), beta and the log-gate
    bytes_l = B * Hv * 2 * d * d * 4 + B * n * (Hk * 2 * d * elem + Hv * (2 * d * elem + 8))
    flops_l = B * Hv * n * 8 * d * d
    peaks, peak_kind = load_peaks()
    gbs = bytes_l / (ms_step * 1e-3) / 1e9
    line = {
        "metric": f"decode step: tokens/s (batch {B}, {n} token(s), 32 value heads, d=128)",
        "value": world * B * n / (ms_step * 1e-3), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "us_per_step": ms_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"decode, B={B} Hk={Hk} Hv={Hv} n={n} d={d}, bf16 q/k/v, "
                               "fp32 state in place",
                   "l2": f"{sets_n} rotating state sets, {sets_n * per_set / 2**20:.0f} MB",
                   "launch": "CUDA graph of one step per state set"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]),
                     "unit": "GB/s", "frac": gbs / float(peaks["hbm_gbs"]), "traffic": None,
                     "peak_source": peak_kind, "bytes_per_launch": bytes_l,
                     "flops_per_launch": flops_l},
        "clocks": clocks.summary(), "e2e": None, "gpu_launches": launches,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_error(args, world, rank, local, dev) -> int:
    """Approximation error of the fused step against the exact inverse on the
    whole B=4, H=16, T=4096, k=64 bf16 workload, per Neumann order N, band mask
    and residual order S: T from the fused kernel against forward substitution
    (fp32), W and U against the WY factors of that exact T.  Not timed; one
    JSON line with the table."""
    import torch
    from gated_deltanet_chunk_02_b200 import gdn
    from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs

    w = Workload(B=4, H=16, T=4096, k=64, d=128, dtype="bf16")
    inp = make_inputs(w, seed=shard_seed(rank, 0), gate_scale=args.gate_scale)
    s = {key: inp[key].to(dev) for key in ("K", "V", "beta", "g")}
    k = w.k
    stream = torch.cuda.current_stream(dev)
    A = torch.empty(w.B, w.H, w.T // k, k, k, device=dev)
    T_ex = torch.empty_like(A)
    gdn.gdn_build_A(s["K"], s["beta"], s["g"], A, k, stream=stream)
    gdn.gdn_invert_fwdsub(A, T_ex, stream=stream)
    W_ex, U_ex = torch.empty_like(s["K"]), torch.empty_like(s["V"])
    gdn.gdn_wy(T_ex, s["K"], s["V"], s["beta"], None, W_ex, U_ex, stream=stream)
    T = torch.empty_like(A)
    W, U = torch.empty_like(W_ex), torch.empty_like(U_ex)

    def rel(x, ref):
        x, ref = x.double(), ref.double()
        return float((x - ref).norm() / ref.norm())

    def snr(e):
        return None if e == 0.0 else -20.0 * math.log10(e)

    rows = []
    for N in (1, 2, 3, 4):
        for mask in (1, 0):
            for S in (0, 8):
                gdn.gdn_chunk_wy_fused(s["K"], s["V"], s["beta"], s["g"], N, mask, S, 0, W, U, T,
                                       k=k, stream=stream)
                torch.cuda.synchronize(dev)
                et, ew, eu = rel(T, T_ex), rel(W, W_ex), rel(U, U_ex)
                worst = float(((T - T_ex).double().flatten(3).norm(dim=-1)
                               / T_ex.double().flatten(3).norm(dim=-1)).max())
                rows.append({"N": N, "mask": mask, "S": S, "T_rel_fro": et, "T_snr_db": snr(et),
                             "T_worst_chunk": worst, "W_rel_fro": ew, "U_rel_fro": eu})
    assert gdn.gdn_get_status(stream) == gdn.GDN_OK
    if rank == 0:
        print(json.dumps({"metric": "fused step: error against the exact inverse",
                          "config": {"workload": f"B={w.B} H={w.H} T={w.T} k={k} d={w.d} bf16, "
                                                 f"log-gate scale {args.gate_scale}",
                                     "chunks": w.n_chunks},
                          "reference": "forward substitution (fp32) and its WY factors",
                          "table": rows}), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-chunks", type=int, default=4096,
                    help="chunks of the cpu_baseline leg (4096 = the whole step)")
    ap.add_argument("--sample-chunks", type=int, default=512,
                    help="chunks per step of the reference arm (capped so the run stays bounded)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=12)
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (profiling)")
    ap.add_argument("--N", type=int, default=WORKLOAD["N"], help="Neumann order")
    ap.add_argument("--S", type=int, default=WORKLOAD["S"], help="residual steps")
    ap.add_argument("--mask", type=int, default=WORKLOAD["mask"], help="band mask on/off")
    ap.add_argument("--kernel", default="fused",
                    choices=["fused", "fused_raw", "neumann", "newton", "blocked", "fwdsub", "int8",
                             "int8_residual", "int16", "int16_residual",
                             "build_A", "wy", "forward", "decode", "error"],
                    help="time one component instead of the fused step (not the headline)")
    ap.add_argument("--k", type=int, default=None, help="chunk size for --kernel runs")
    ap.add_argument("--batch", type=int, default=64, help="sequences per --kernel decode step")
    ap.add_argument("--M", type=int, default=3, help="sequential correction steps (--kernel newton)")
    ap.add_argument("--tokens", type=int, default=1, help="tokens per --kernel decode call")
    ap.add_argument("--gate-scale", type=float, default=1.0,
                    help="log-gate scale of the --kernel error inputs (0.05: slow decay)")
    ap.add_argument("--rotate", type=int, default=ROTATE,
                    help="input/output sets cycled through the timed steps")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_setup()
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import torch
    from gated_deltanet_chunk_02_b200 import gdn
    from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.kernel == "decode":
        return run_decode(args, world, rank, local, dev)
    if args.kernel == "error":
        return run_error(args, world, rank, local, dev)
    if args.kernel != "fused":
        return run_component(args, world, rank, local, dev)
    w = dict(WORKLOAD, N=args.N, S=args.S, mask=args.mask)
    wl = Workload(B=w["B"], H=w["H"], T=w["T"], k=w["k"], d=w["d"], dtype=w["dtype"])
    nc = wl.n_chunks
    k, d = w["k"], w["d"]
    elem = 2
    sets = []
    for r in range(args.rotate):
        inp = make_inputs(wl, seed=shard_seed(rank, r))
        s = {key: inp[key].to(dev) for key in ("K", "V", "beta", "g")}
        s["W"] = torch.empty_like(s["K"])
        s["U"] = torch.empty_like(s["V"])
        sets.append(s)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        s = sets[i % len(sets)]
        gdn.gdn_chunk_wy_fused(s["K"], s["V"], s["beta"], s["g"], w["N"], w["mask"], w["S"],
                               w["gated"], s["W"], s["U"], None, k=k, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    assert gdn.gdn_get_status(stream) == gdn.GDN_OK

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launches0 = gdn.gdn_launch_count()
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    launches = gdn.gdn_launch_count() - launches0
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world, dev)
    status = gdn.gdn_get_status(stream)
    assert status == gdn.GDN_OK, status

    # The same step without the residual (S = 0), timed the same way after the
    # headline, reported beside it: the series + mask + WY alone.
    s0 = None
    if w["S"] != 0 and args.steps > 0:
        def step0(i):
            s = sets[i % len(sets)]
            gdn.gdn_chunk_wy_fused(s["K"], s["V"], s["beta"], s["g"], w["N"], w["mask"], 0,
                                   w["gated"], s["W"], s["U"], None, k=k, stream=stream)
        for i in range(args.warmup):
            step0(i)
        barrier(world)
        torch.cuda.synchronize(dev)
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(args.steps):
            step0(i)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        s0 = max_over_ranks(f0.elapsed_time(f1), world, dev) / args.steps
        assert gdn.gdn_get_status(stream) == gdn.GDN_OK

    # End to end through the public API: every step copies its inputs from
    # pinned host memory, runs the fused step and copies W and U back to pinned
    # host memory.  Consecutive steps overlap as a serving pipeline would: step
    # i's inputs travel host->device while step i-1 computes and step i-2's
    # results travel back (copy-in, compute and copy-out streams, two device
    # buffer sets); the time is first copy-in to last copy-out.
    if args.no_e2e:
        args.e2e_steps = 0
    host = {key: sets[0][key].cpu().pin_memory() for key in ("K", "V", "beta", "g")}
    hostW = [torch.empty(sets[0]["W"].shape, dtype=sets[0]["W"].dtype).pin_memory() for _ in range(2)]
    hostU = [torch.empty_like(hostW[0]).pin_memory() for _ in range(2)]
    dbufs = [{key: torch.empty_like(sets[0][key]) for key in ("K", "V", "beta", "g", "W", "U")}
             for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_comp = stream
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in", "comp", "out")}
    started = [False, False]

    def e2e_step(i):
        b = i % 2
        d = dbufs[b]
        if started[b]:
            s_in.wait_event(ev["comp"][b])            # step i-2 no longer reads these inputs
        for key in ("K", "V", "beta", "g"):
            with torch.cuda.stream(s_in):
                d[key].copy_(host[key], non_blocking=True)
        ev["in"][b].record(s_in)
        s_comp.wait_event(ev["in"][b])
        if started[b]:
            s_comp.wait_event(ev["out"][b])           # step i-2's W, U have left
        gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], w["N"], w["mask"], w["S"],
                               w["gated"], d["W"], d["U"], None, k=k, stream=s_comp)
        ev["comp"][b].record(s_comp)
        s_out.wait_event(ev["comp"][b])
        with torch.cuda.stream(s_out):
            hostW[b].copy_(d["W"], non_blocking=True)
            hostU[b].copy_(d["U"], non_blocking=True)
        ev["out"][b].record(s_out)
        started[b] = True

    for i in range(3 if args.e2e_steps else 0):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.e2e_steps):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / max(args.e2e_steps, 1), world, dev)
    h2d = sum(host[key].numel() * host[key].element_size() for key in host)
    d2h = 2 * hostW[0].numel() * hostW[0].element_size()

    peaks, peak_kind = load_peaks()
    ms_step = ms / args.steps
    bytes_per_launch = algorithmic_bytes_per_chunk(k, d, elem) * nc
    flops_per_launch = algorithmic_flops_per_chunk(k, d, w["N"], w["S"]) * nc
    achieved_gbs = bytes_per_launch / (ms_step * 1e-3) / 1e9
    tflops = flops_per_launch / (ms_step * 1e-3) / 1e12
    peak_gbs = float(peaks["hbm_gbs"])
    t_hbm = bytes_per_launch / (peak_gbs * 1e9)
    t_tc = flops_per_launch / (float(peaks["bf16_tflops"]) * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    traffic = recorded_traffic("fused")

    line = {
        "metric": METRIC,
        "value": aggregate_throughput(nc, world, ms, args.steps),
        "unit": "chunks/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(w, nc, args.rotate),
        "roofline": {
            "bound": bound,
            "achieved": achieved_gbs if bound == "hbm" else tflops,
            "peak": peak_gbs if bound == "hbm" else float(peaks["bf16_tflops"]),
            "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": (achieved_gbs / peak_gbs) if bound == "hbm"
            else tflops / float(peaks["bf16_tflops"]),
            "traffic": traffic,
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback",
            "roofline_frac": max(t_hbm, t_tc) / (ms_step * 1e-3),
            "tflops": tflops,
            "bytes_per_launch": bytes_per_launch,
            "flops_per_launch": flops_per_launch,
        },
        "clocks": clocks.summary(),
        "e2e": ({"value": nc * world / (e2e_ms * 1e-3), "unit": "chunks/s",
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
                if args.e2e_steps else None),
        "gpu_launches": launches,
    }
    if s0 is not None:
        line["s0"] = {"ms_per_step": s0,
                      "value": nc * world / (s0 * 1e-3),
                      "frac": bytes_per_launch / (s0 * 1e-3) / 1e9 / peak_gbs,
                      "note": "same step with S=0 (no residual), timed after the headline"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_cpu = min(nc, args.cpu_chunks)
        data = OracleInputs(w)
        dt, threads = cpu_oracle_parallel(w, data, 0, n_cpu)
        # the same oracle held to one thread, on the first 256 chunks
        from threadpoolctl import threadpool_limits
        n_one = min(nc, 256)
        with threadpool_limits(limits=1):
            dt1, _ = cpu_oracle_step(w, data, 0, n_one)
        line["cpu_baseline"] = {"value": n_cpu / dt, "unit": "chunks/s",
                                "cores": threads, "kind": "oracle",
                                "sample": f"first {n_cpu} of {nc} chunks "
                                          f"({'one whole step' if n_cpu == nc else 'part of a step'}), fp64, "
                                          f"one window per host thread",
                                "one_core": {"value": n_one / dt1, "unit": "chunks/s", "cores": 1,
                                             "sample": f"first {n_one} of {nc} chunks"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
