"""Benchmark of the NVFP4 training hot path on B200.

One step = the three training GEMMs (fprop, dgrad, wgrad) of both linears of a 12B-class
MLP (tokens 8192, d_model 5120, up 5120 -> 20480, down 20480 -> 5120), each with the
quantization of its two operands: 2D-scaled weights, 1x16 activations, stochastically
rounded gradients, random-Hadamard-transformed wgrad inputs.  Every kernel is the library's
(libnvfp4.so through its C ABI); the timed region queues the same calls the nvfp4_linear_*
entry points make, with CUDA events around each GEMM and each quantizer launch.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle instead, on a bounded
sample of the same workload.  Under torchrun (N > 1) every rank runs an independent replica
on its own GPU (the path has no exchange step); the time is the max over ranks.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS & quantize GB/s on 1 B200, % of FP4/HBM roofline"
FP4_OVER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of the bf16-output GEMM at the
# MLP's shapes (8192 x 20480 x 5120), from an ncu capture of the current kernel
# (95.4 MB read + 298.8 MB written); None whenever the kernel changes until it is re-captured.
GEMM_BF16_DRAM_BYTES = 394.2e6


def _peaks(path=None):
    """The roofline denominators: the measured copy bandwidth and bf16 GEMM rates of this
    machine's GPUs when MEASURED_PEAKS.json holds them as numbers, else the fallback figures."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        out = {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
               "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
               "source": "measured"}
        if all(v > 0 for k, v in out.items() if k != "source"):
            return out
    except (OSError, KeyError, ValueError, TypeError, AttributeError):
        pass
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---- multi-rank plumbing (also exercised by the CPU gloo tests) --------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ---- clocks ------------------------------------------------------------------------------

class ClockSampler:
    """Samples the SM clock, power and the clock-event (throttle) reasons of one GPU while
    running: through NVML every 2 ms (read-only queries), else with nvidia-smi every 50 ms.
    `mark()` opens and closes the window whose samples `summary()` reports."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int, uuid: str = None, period_s: float = 0.002):
        self.device_index = device_index
        self.uuid = uuid
        self.period_s = period_s
        self.proc = None
        self.nvml = None
        self.samples = []  # (host time, sm MHz, max MHz, watts, set of active reasons)
        self.thread = None
        self.stop = threading.Event()
        self.window = [None, None]
        self.source = None

    def __enter__(self):
        if not self._start_nvml():
            self._start_smi()
        return self

    def _start_nvml(self):
        try:
            import pynvml as N
            N.nvmlInit()
            h = None
            if self.uuid:
                try:
                    h = N.nvmlDeviceGetHandleByUUID(self.uuid)
                except N.NVMLError:
                    h = None
            if h is None:
                h = N.nvmlDeviceGetHandleByIndex(self.device_index)
            bits = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap}
            smax = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
        except Exception:
            return False
        self.nvml = N
        self.source = "nvml"

        def poll():
            while not self.stop.is_set():
                try:
                    sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                    watts = N.nvmlDeviceGetPowerUsage(h) / 1000.0
                    active = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                    reasons = {k for k, b in bits.items() if active & b}
                    self.samples.append((time.time(), float(sm), float(smax), watts, reasons))
                except Exception:
                    pass
                self.stop.wait(self.period_s)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        return True

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 10 and self.proc.poll() is None:
                time.sleep(0.05)  # the first sample marks nvidia-smi as running
        except OSError:
            self.proc = None

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm, smax, watts = float(parts[0]), float(parts[1]), float(parts[2])
            except ValueError:
                continue
            reasons = {n for n, v in zip(self.REASONS, parts[3:7])
                       if v.lower().startswith("active")}
            self.samples.append((time.time(), sm, smax, watts, reasons))

    def mark(self, which):
        self.window[0 if which == "start" else 1] = time.time()

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        t0, t1 = self.window
        rows = [r for r in list(self.samples)
                if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1 + 0.002)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        reasons = set().union(*[r[4] for r in rows])
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_max_mhz": max(r[2] for r in rows),
                "power_w_max": max(r[3] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "source": self.source}


# ---- the workload ------------------------------------------------------------------------

OPS = ("fprop", "dgrad", "wgrad")


class Step:
    """Device buffers and the call sequence of one step of the MLP workload."""

    def __init__(self, workload, device, seed_offset=0):
        import torch
        from nvfp4_bit_quantized_03_b200 import binding as B
        self.B = B
        self.torch = torch
        self.wl = workload
        self.device = device
        self.seed = workload.seed
        self.mask = B.sign_mask_from_seed(workload.seed)
        self.host = []     # pinned host copies of the inputs (for the end-to-end timing)
        self.layers = []
        for li, lin in enumerate(workload.linears):
            X, W, dY = synth.linear_inputs(lin, workload.seed, layer_index=li)
            tens = {}
            for name, arr in (("X", X), ("W", W), ("dY", dY)):
                h = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).pin_memory()
                self.host.append(h)
                tens[name] = h.to(device)
            T, I, O = lin.T, lin.I, lin.O
            Q = B.QuantizedTensor
            layer = {
                "lin": lin, **tens,
                "fprop": (Q(T, I, device), Q(O, I, device)),
                "dgrad": (Q(T, O, device), Q(I, O, device)),
                "wgrad": (Q(O, T, device), Q(I, T, device)),
                "out": {"fprop": torch.empty((T, O), dtype=torch.bfloat16, device=device),
                        "dgrad": torch.empty((T, I), dtype=torch.bfloat16, device=device),
                        "wgrad": torch.empty((O, I), dtype=torch.float32, device=device)},
            }
            self.layers.append(layer)
        self.workspace = torch.empty((B.workspace_bytes(1 << 14, 1 << 14),), dtype=torch.uint8,
                                     device=device)
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=device)
        self.flops_per_gemm = [2 * L["lin"].T * L["lin"].I * L["lin"].O for L in self.layers]

    @property
    def gemm_flops(self):
        return sum(3 * f for f in self.flops_per_gemm)

    def quant_bytes(self):
        """Algorithmic quantizer bytes of one step: each of X, W and dY is read twice (the amax
        pass and the quantize pass, 2 B/elem each) and written in its two GEMM orientations
        (0.5 + 1/16 B/elem each): 5.125 B/elem."""
        total = 0
        for L in self.layers:
            lin = L["lin"]
            for n in (lin.T * lin.I, lin.O * lin.I, lin.T * lin.O):
                total += n * (2 + 2 + 2 * (0.5 + 1 / 16))
        return total

    def n_quant_launches(self):
        return 2 * 3 * len(self.layers)   # (amax + quantize) x (X, W, dY)

    def n_gemm_launches(self):
        return 3 * len(self.layers)

    def run(self, events=None, inputs=None, outputs=None, per_layer=None):
        """Queue one step on the current stream.  With `events`, record CUDA events around
        every GEMM (events['gemm']) and every operand quantization (events['quant']).
        `inputs` / `outputs` (one dict per layer) replace the step's own device buffers;
        `per_layer(li, stage)` is called before a layer's quantizations ('in'), after them
        ('quantized') and after its GEMMs ('out')."""
        B = self.B
        ws, st = self.workspace, self.dev_status

        def timed(kind, fn):
            if events is None:
                fn()
                return
            e0 = self.torch.cuda.Event(enable_timing=True)
            e1 = self.torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            events[kind].append((e0, e1))

        for li, L in enumerate(self.layers):
            src = inputs[li] if inputs is not None else L
            X, W, dY = src["X"], src["W"], src["dY"]
            out = outputs[li] if outputs is not None else L["out"]
            if per_layer is not None:
                per_layer(li, "in")
            # Each operand is quantized once into both orientations its two GEMMs read:
            # W with 16x16 scales (row-wise for fprop, column-wise for dgrad); X row-wise
            # (fprop) and RHT'd column-wise (wgrad); dY row-wise with SR stream 0 (dgrad) and
            # RHT'd column-wise with SR stream 1 (wgrad).
            xa, wb = L["fprop"]
            dya, wcb = L["dgrad"]
            dyc, xcb = L["wgrad"]
            timed("quant", lambda: B.quantize(W, B.ROWWISE | B.COLWISE | B.BLOCK2D, out_row=wb,
                                              out_col=wcb, workspace=ws, dev_status=st))
            timed("quant", lambda: B.quantize_row_rht(X, self.mask, 0, out_row=xa, out_col=xcb,
                                                      workspace=ws, dev_status=st))
            timed("quant", lambda: B.quantize_row_rht(dY, self.mask, B.SR, seed=self.seed,
                                                      offset=0, out_row=dya, out_col=dyc,
                                                      workspace=ws, dev_status=st))
            if per_layer is not None:
                per_layer(li, "quantized")
            timed("gemm", lambda: B.gemm(xa, wb, out=out["fprop"], dev_status=st))
            timed("gemm", lambda: B.gemm(dya, wcb, out=out["dgrad"], dev_status=st))
            timed("gemm", lambda: B.gemm(dyc, xcb, out=out["wgrad"], dev_status=st))
            if per_layer is not None:
                per_layer(li, "out")

    def run_end_to_end(self, steps, outs_host):
        """Queue `steps` steps that take their inputs from pinned host memory and return their
        results to it, pipelined: host -> device copies on one stream, device -> host copies on
        another, the library calls on the current stream.  Two sets of device inputs and
        outputs alternate between steps; events order each copy after what it depends on
        (a layer's GEMMs wait for its inputs; its results leave once its GEMMs are done; an
        input set is overwritten only after the step two before has quantized it, an output
        set only after the step two before has copied it out), so every step still moves all
        of its bytes both ways."""
        torch = self.torch
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        if not hasattr(self, "_e2e_sets"):
            self._e2e_sets = []
            for k in range(2):
                ins = [L if k == 0 else {n: torch.empty_like(L[n]) for n in ("X", "W", "dY")}
                       for L in self.layers]
                outs = [L["out"] if k == 0 else {op: torch.empty_like(L["out"][op]) for op in OPS}
                        for L in self.layers]
                self._e2e_sets.append((ins, outs))
        nl = len(self.layers)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready = [[ev() for _ in range(nl)] for _ in range(steps)]
        in_free = [[ev() for _ in range(nl)] for _ in range(steps)]
        out_ready = [[ev() for _ in range(nl)] for _ in range(steps)]
        out_free = [[ev() for _ in range(nl)] for _ in range(steps)]
        start = ev()
        start.record(comp)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(steps):
            ins, outs = self._e2e_sets[i % 2]
            with torch.cuda.stream(s_in):
                for li in range(nl):
                    if i >= 2:
                        s_in.wait_event(in_free[i - 2][li])
                    k = 3 * li
                    for n in ("X", "W", "dY"):
                        ins[li][n].copy_(self.host[k], non_blocking=True)
                        k += 1
                    in_ready[i][li].record(s_in)

            def per_layer(li, stage, i=i):
                if stage == "in":
                    comp.wait_event(in_ready[i][li])
                    if i >= 2:
                        comp.wait_event(out_free[i - 2][li])
                elif stage == "quantized":
                    in_free[i][li].record(comp)
                else:
                    out_ready[i][li].record(comp)

            self.run(inputs=ins, outputs=outs, per_layer=per_layer)
            with torch.cuda.stream(s_out):
                for li in range(nl):
                    s_out.wait_event(out_ready[i][li])
                    for j, op in enumerate(OPS):
                        outs_host[3 * li + j].copy_(outs[li][op], non_blocking=True)
                    out_free[i][li].record(s_out)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)

    def h2d_bytes(self):
        return sum(h.numel() * h.element_size() for h in self.host)

    def output_host_buffers(self):
        bufs = []
        for L in self.layers:
            for op in OPS:
                o = L["out"][op]
                bufs.append(self.torch.empty(o.shape, dtype=o.dtype).pin_memory())
        return bufs


# ---- CPU oracle leg ----------------------------------------------------------------------

def host_threads(cap=64):
    """Host cores this process may run on."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(cap, n))


def blas_threads():
    """Threads numpy's BLAS uses for the FP64 reference products (1 if it cannot be told)."""
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        return 1


def oracle_sample(workload, tokens=128, max_out=512, max_in=4096, threads=1):
    """Time the CPU oracle on a bounded sample of the workload: for every linear, a
    `tokens` x min(I, max_in) activation, a min(O, max_out) x min(I, max_in) weight and a
    `tokens` x min(O, max_out) gradient drawn with the workload's generators and seed; the
    timed part is the three GEMMs' operand quantizations (the C oracle on `threads` threads)
    and their FP64 reference products (numpy matmul).
    Returns (seconds, GEMM flops of the sample)."""
    import oracle
    inputs = []
    for li, lin in enumerate(workload.linears):
        small = synth.Linear(lin.name, tokens, min(lin.I, max_in), min(lin.O, max_out))
        inputs.append(synth.linear_inputs(small, workload.seed, layer_index=li))
    mask = oracle.sign_mask_from_seed(workload.seed)
    s = workload.seed
    flops = 0
    t0 = time.perf_counter()
    for X, W, dY in inputs:
        q = dict(threads=threads)
        for qa, qb in ((oracle.quantize(X, **q), oracle.quantize(W, block2d=True, **q)),
                       (oracle.quantize(dY, sr=True, seed=s, offset=0, **q),
                        oracle.quantize(W, transpose=True, block2d=True, **q)),
                       (oracle.quantize(dY, transpose=True, rht=True, sign_mask=mask, sr=True,
                                        seed=s, offset=1, **q),
                        oracle.quantize(X, transpose=True, rht=True, sign_mask=mask, **q))):
            oracle.gemm_ref(qa, qb)
            flops += 2 * qa.rows * qb.rows * qa.cols
    return time.perf_counter() - t0, flops


# The quantizer sweep's modes for the CPU baseline: (name, oracle calls, outputs).  Bytes are
# counted as for the GPU: two 2-byte reads of every element (amax pass, quantize pass) plus
# 0.5 B of codes and 1/16 B of scales per element per output.
CPU_QUANT_MODES = (
    ("1x16_rtn_row", ({},), 1),
    ("16x16_2d_rowcol", ({"block2d": True}, {"block2d": True, "transpose": True}), 2),
    ("1x16_sr_row", ({"sr": True, "seed": 1},), 1),
    ("rht_1x16_sr_col", ({"transpose": True, "rht": True, "sign_mask": 0x5A3C, "sr": True,
                          "seed": 1},), 1),
)


def cpu_quantize_baseline(threads, log2n_1t=(20, 22, 24), log2n_all=(20, 22, 24, 26)):
    """The oracle's quantizer in GB/s of algorithmic bytes on tensors of the quantizer sweep
    (2^n bf16 elements in rows of 4096, N(0,1) with 1 % x50 outliers), single-threaded and on
    `threads` threads.  Per mode the rate at the largest size is reported; sizes above those
    timed are not run (the CPU rate does not depend on the size once the tensor is out of
    cache)."""
    import oracle
    out = {}
    for label, sizes, th in (("1t", log2n_1t, 1), ("all", log2n_all, threads)):
        per_mode = {}
        for log2n in sizes:
            rows, cols = synth.quant_sweep_shape(log2n)
            x = synth.activations((rows, cols), seed=synth.QUANT_SWEEP_SEED)
            n = rows * cols
            for name, calls, outs in CPU_QUANT_MODES:
                t0 = time.perf_counter()
                for kw in calls:
                    oracle.quantize(x, threads=th, **kw)
                secs = time.perf_counter() - t0
                per_mode[name] = n * (4 + outs * (0.5 + 1 / 16)) / secs / 1e9
            del x
        total_bytes = sum(4 + outs * (0.5 + 1 / 16) for _, _, outs in CPU_QUANT_MODES)
        # the modes' aggregate: all four modes' bytes over their summed time, per element
        agg = total_bytes / sum((4 + outs * (0.5 + 1 / 16)) / per_mode[name]
                                for name, _, outs in CPU_QUANT_MODES)
        out[label] = {"gbps": agg, "threads": th, "log2n": max(sizes), "modes": per_mode}
    return {"value": out["all"]["gbps"], "unit": "GB/s", "cores": threads,
            "value_single_thread": out["1t"]["gbps"],
            "kind": "oracle",
            "sample": "quantizer sweep tensors 2^n bf16 elements in rows of 4096 (N(0,1), 1% x50): "
                      f"single thread up to 2^{max(log2n_1t)}, {threads} threads up to "
                      f"2^{max(log2n_all)}; modes 1x16 RTN row, 16x16 2D row+col, 1x16 SR row, "
                      "RHT+1x16 SR col; 4.5625 B/elem per one-output call, 5.125 for row+col; "
                      "larger sweep sizes not run",
            "single_thread": out["1t"], "all_cores": out["all"]}


def cpu_gemm_baseline():
    """The oracle's GEMM step timed alone: its plain FP64 triple loop (one thread) on the
    fprop operands of the single-fprop workload (256 x 512 x 512) and of a 512-row slice of the
    4096^3 layer, in GFLOP/s; numpy's FP64 BLAS on the same dequantized operands is timed too
    and labelled "library"."""
    import oracle
    out = {"unit": "GFLOP/s", "kind": "oracle", "threads": 1, "blas_threads": blas_threads()}
    for name, wl, rows in (("fprop_t256_i512_o512", synth.fprop_small(), None),
                           ("linear_4096_first_512_rows", synth.layer_4096(), 512)):
        lin = wl.linears[0]
        X, W, _ = synth.linear_inputs(lin, wl.seed)
        if rows is not None:
            X = X[:rows]
        qa, qb = oracle.fprop_operands(X, W)
        A, B = qa.dequantize(), qb.dequantize()
        flop = 2.0 * A.shape[0] * B.shape[0] * A.shape[1]
        t0 = time.perf_counter()
        oracle.gemm_ref_loop(A, B)
        t_loop = time.perf_counter() - t0
        t0 = time.perf_counter()
        for _ in range(5):
            A @ B.T
        t_blas = (time.perf_counter() - t0) / 5
        out[name] = {"shape": f"{A.shape[0]} x {B.shape[0]} x {A.shape[1]}",
                     "oracle_loop_gflops": flop / t_loop / 1e9,
                     "library_numpy_fp64_gflops": flop / t_blas / 1e9}
    return out


def cpu_baseline(workload):
    threads = host_threads()
    secs, flops = oracle_sample(workload, tokens=1024, max_out=2048, max_in=5120,
                                threads=threads)
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "oracle_threads": threads, "blas_threads": blas_threads(),
            "sample": "per linear: 1024 tokens x min(O,2048) out- x min(I,5120) in-features drawn "
                      "with the workload's generators; fprop/dgrad/wgrad operand quantization "
                      f"(C oracle, {threads} threads) + FP64 reference GEMMs (numpy matmul of "
                      "the dequantized operands)",
            "seconds": secs,
            "quantize": cpu_quantize_baseline(threads),
            "gemm": cpu_gemm_baseline()}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    wl = synth.mlp_12b()
    threads = host_threads()
    for _ in range(args.warmup):
        oracle_sample(wl, tokens=128, max_out=512, max_in=4096, threads=threads)
    times, flops = [], 0
    for _ in range(args.steps):
        secs, flops = oracle_sample(wl, tokens=128, max_out=512, max_in=4096, threads=threads)
        times.append(secs)
    total = sum(times)
    value = flops * len(times) / total / 1e12
    sample = ("per linear: 128 tokens x min(O,512) out- x min(I,4096) in-features drawn with "
              f"the workload's generators; operand quantization (C oracle, {threads} threads) + "
              "FP64 reference GEMMs (numpy matmul)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---- GPU leg -----------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    peaks = _peaks()
    wl = synth.mlp_12b()
    step = Step(wl, device)

    def barrier():
        if world > 1:
            dist.barrier()

    events = {"gemm": [], "quant": []}
    props = torch.cuda.get_device_properties(device)
    uuid = getattr(props, "uuid", None)
    uuid = f"GPU-{uuid}" if uuid is not None and not str(uuid).startswith("GPU-") else uuid
    with ClockSampler(device.index if device.index is not None else 0, uuid=uuid) as clocks:
        for _ in range(args.warmup):
            step.run()
        torch.cuda.synchronize()
        st = int(step.dev_status.item())
        if st != 0:
            raise RuntimeError(f"device status {st} after warm-up")
        barrier()
        torch.cuda.synchronize()
        clocks.mark("start")
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(args.steps):
            step.run(events)
        t1.record()
        torch.cuda.synchronize()
        clocks.mark("end")
        barrier()
    ms_local = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms_local, device)
    value = whole_job_rate(step.gemm_flops / 1e12, world, ms / 1e3)

    gemm_ms = [a.elapsed_time(b) for a, b in events["gemm"]]
    quant_ms = [a.elapsed_time(b) for a, b in events["quant"]]
    gemm_avg_ms = sum(gemm_ms) / len(gemm_ms)
    # the step's GEMMs come as (fprop, dgrad, wgrad) per linear: bf16, bf16, FP32 outputs.
    # The roofline object describes the dominant kernel, the bf16-output instantiation.
    bf16_ms = [t for i, t in enumerate(gemm_ms) if i % 3 != 2]
    f32_ms = [t for i, t in enumerate(gemm_ms) if i % 3 == 2]
    bf16_avg_ms = sum(bf16_ms) / len(bf16_ms)
    f32_avg_ms = sum(f32_ms) / len(f32_ms)
    flops_per_launch = step.flops_per_gemm[0]  # every GEMM of this workload: 2*8192*5120*20480
    achieved = flops_per_launch / (bf16_avg_ms / 1e3) / 1e12
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    quant_gbs = step.quant_bytes() * args.steps / (sum(quant_ms) / 1e3) / 1e9

    # end-to-end: inputs from pinned host memory, outputs back to pinned host memory
    e2e = None
    if not args.no_e2e:
        outs = step.output_host_buffers()
        e2e_steps = max(1, min(args.steps, 10))
        barrier()
        torch.cuda.synchronize()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record()
        step.run_end_to_end(e2e_steps, outs)
        s1.record()
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(s0.elapsed_time(s1) / e2e_steps, device)
        d2h = sum(o.numel() * o.element_size() for o in outs)
        e2e = {"value": whole_job_rate(step.gemm_flops / 1e12, world, e2e_ms / 1e3),
               "unit": "TFLOP/s", "h2d_bytes_per_step": step.h2d_bytes(),
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
               "method": f"{e2e_steps} steps timed with CUDA events; each step copies X, W and "
                         "dY of both linears from pinned host memory, queues the step's library "
                         "calls through the C ABI (the three one-pass quantizations and three "
                         "GEMMs per linear that the nvfp4_linear_* entry points make) and copies "
                         "Y, dX and dW back to pinned host memory; host-to-device and "
                         "device-to-host copies run on their own streams, overlapping each other "
                         "and the compute, with two alternating sets of device buffers"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    st = int(step.dev_status.item())
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e2m1",
            "data": "synthetic: seeded N(0,1) activations with 1% x50 outliers, N(0,0.02) "
                    "random-init weights, N(0,1e-3) gradients with 0.5% x100 spikes",
            "config": {"workload": wl.name, "tokens": 8192, "d_model": 5120, "d_ff": 20480,
                       "gemms_per_step": 6, "gemm_tflop_per_step": step.gemm_flops / 1e12,
                       "outputs": "Y and dX bf16, dW fp32",
                       "recipe": "W 16x16 RTN (row+col, one pass), X 1x16 RTN + RHT16 col (one pass), dY 1x16 SR + RHT16 SR col (one pass)",
                       "l2": "inputs larger than L2: 1.26 GB of bf16 inputs read per step",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                         "traffic": GEMM_BF16_DRAM_BYTES,
                         "kernel": "gemm_nvf4_kernel<bf16 out> (fprop and dgrad, 4 of 6 GEMMs)",
                         "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} "
                                        f"TFLOP/s x {FP4_OVER_BF16:g} (nominal FP4:BF16)",
                         "avg_launch_ms": bf16_avg_ms,
                         "all_gemms_avg_launch_ms": gemm_avg_ms,
                         "fp32_out_gemm_avg_launch_ms": f32_avg_ms,
                         "fp32_out_gemm_tflops": flops_per_launch / (f32_avg_ms / 1e3) / 1e12},
            "quantize": {"gbps": quant_gbs, "peak_gbs": peaks["hbm_gbs"],
                         "frac": quant_gbs / peaks["hbm_gbs"],
                         "bytes_per_step": step.quant_bytes(),
                         "ms_per_step": sum(quant_ms) / args.steps},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": (step.n_gemm_launches() + step.n_quant_launches()) * args.steps,
            "clocks": clocks.summary(),
            "dev_status": st,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0 if st == 0 else 1


def run_kernel_case(args):
    """One kernel family alone, at the MLP workload's shapes, for profiling: warm-up launches,
    then `steps` launches bracketed by CUDA events.  Prints a JSON line (not a bench value)."""
    import torch
    from nvfp4_bit_quantized_03_b200 import binding as B
    peaks = _peaks()
    T, D, F = 8192, 5120, 20480
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = torch.empty((B.workspace_bytes(1 << 14, 1 << 14),), dtype=torch.uint8, device=dev)
    if args.kernel == "gemm_f32":
        # the wgrad GEMM of the MLP's up-projection: dW [20480 x 5120] = dY^T . X over K = 8192
        # tokens, FP32 out, both operands RHT'd column-wise quantizations
        dY = torch.from_numpy(synth.gradients((T, F), seed=2).view(np.int16)).view(torch.bfloat16).to(dev)
        X = torch.from_numpy(synth.activations((T, D), seed=2).view(np.int16)).view(torch.bfloat16).to(dev)
        qa = B.rht_quantize(dY, 0x5A3C, B.SR, seed=1, offset=1, workspace=ws)
        qb = B.rht_quantize(X, 0x5A3C, 0, workspace=ws)
        out = torch.empty((F, D), dtype=torch.float32, device=dev)
        fn = lambda: B.gemm(qa, qb, out=out)  # noqa: E731
        work, unit, peak = 2 * T * D * F / 1e12, "TFLOP/s", peaks["bf16_tflops"] * FP4_OVER_BF16
        shape = f"M={F} N={D} K={T}, FP32 out"
    elif args.kernel in ("gemm", "gemm_amax", "chain", "chain_amax", "gemm_mx"):
        X = torch.from_numpy(synth.activations((T, D), seed=2).view(np.int16)).view(torch.bfloat16).to(dev)
        W = torch.from_numpy(synth.weights((F, D), seed=2).view(np.int16)).view(torch.bfloat16).to(dev)
        mx = B.MX if args.kernel == "gemm_mx" else 0
        qa, _ = B.quantize(X, B.ROWWISE | mx, workspace=ws)
        qb, _ = B.quantize(W, B.ROWWISE | (mx or B.BLOCK2D), workspace=ws)
        out = torch.empty((T, F), dtype=torch.bfloat16, device=dev)
        amax = torch.empty(2, dtype=torch.float32, device=dev)
        qr, qc = B.QuantizedTensor(T, F, dev), B.QuantizedTensor(F, T, dev)

        def chain():
            # the GEMM output quantized for the next layer: row-wise and RHT'd column-wise, SR
            B.gemm(qa, qb, out=out)
            B.quantize_row_rht(out, 0x5A3C, B.SR, seed=1, out_row=qr, out_col=qc, workspace=ws)

        def chain_amax():
            # the same, with both maxima taken in the GEMM's epilogue instead of an amax pass;
            # the two quantized outputs read them in place
            qr.amax, qc.amax = amax[0:1], amax[1:2]
            B.gemm_amax(qa, qb, 0x5A3C, out=out, amax_out=amax)
            B.quantize_row_rht(out, 0x5A3C, B.SR | B.AMAX_GIVEN, seed=1, out_row=qr,
                               out_col=qc)

        fn = {"gemm": lambda: B.gemm(qa, qb, out=out),
              "gemm_amax": lambda: B.gemm_amax(qa, qb, 0x5A3C, out=out, amax_out=amax),
              "chain": chain, "chain_amax": chain_amax,
              "gemm_mx": lambda: B.gemm(qa, qb, out=out, mx=True)}[args.kernel]
        work, unit, peak = 2 * T * D * F / 1e12, "TFLOP/s", peaks["bf16_tflops"] * FP4_OVER_BF16
        shape = f"M={T} N={F} K={D}, bf16 out" + (
            ", then SR dual quantization of D" if args.kernel.startswith("chain") else "") + (
            ", MXFP4 operands" if mx else "")
    else:
        x = torch.from_numpy(synth.gradients((T, F), seed=2).view(np.int16)).view(torch.bfloat16).to(dev)
        n = T * F
        if args.kernel == "rowwise":
            q = B.QuantizedTensor(T, F, dev)
            fn = lambda: B.quantize(x, B.ROWWISE | B.SR, seed=1, out_row=q, workspace=ws)  # noqa: E731
        elif args.kernel == "rowwise_rtn":
            q = B.QuantizedTensor(T, F, dev)
            fn = lambda: B.quantize(x, B.ROWWISE, out_row=q, workspace=ws)  # noqa: E731
        elif args.kernel == "tile2d":
            # as the step quantizes W: 16x16 scales, row-wise and column-wise outputs
            q = B.QuantizedTensor(T, F, dev)
            q2 = B.QuantizedTensor(F, T, dev)
            fn = lambda: B.quantize(x, B.ROWWISE | B.COLWISE | B.BLOCK2D, out_row=q,  # noqa: E731
                                    out_col=q2, workspace=ws)
        elif args.kernel == "dual_rtn":
            q = B.QuantizedTensor(T, F, dev)
            q2 = B.QuantizedTensor(F, T, dev)
            fn = lambda: B.quantize_row_rht(x, 0x5A3C, 0, out_row=q, out_col=q2,  # noqa: E731
                                            workspace=ws)
        elif args.kernel == "rht":
            q = B.QuantizedTensor(F, T, dev)
            fn = lambda: B.rht_quantize(x, 0x5A3C, B.SR, seed=1, out_col=q, workspace=ws)  # noqa: E731
        elif args.kernel == "rowwise_mx":
            q = B.QuantizedTensor(T, F, dev)
            fn = lambda: B.quantize(x, B.ROWWISE | B.MX, out_row=q, workspace=ws)  # noqa: E731
        elif args.kernel == "rht_mx":
            q = B.QuantizedTensor(F, T, dev)
            fn = lambda: B.rht_quantize(x, 0x5A3C, B.SR | B.MX, seed=1, out_col=q,  # noqa: E731
                                        workspace=ws)
        else:
            q = B.QuantizedTensor(T, F, dev)
            q2 = B.QuantizedTensor(F, T, dev)
            fn = lambda: B.quantize_row_rht(x, 0x5A3C, B.SR, seed=1, out_row=q, out_col=q2,  # noqa: E731
                                            workspace=ws)
        outs = 2 if args.kernel in ("dual", "dual_rtn", "tile2d") else 1
        work, unit, peak = n * (4 + outs * (0.5 + 1 / 16)) / 1e9, "GB/s", peaks["hbm_gbs"]
        shape = f"{T} x {F} bf16, amax pass + quantize pass"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    rate = work / (ms / 1e3)
    print(json.dumps({"kernel_case": args.kernel, "shape": shape, "ms_per_launch": ms,
                      "achieved": rate, "unit": unit, "peak": peak, "frac": rate / peak}),
          flush=True)
    return 0


SWEEP_MODES = {
    # name: (flags, rht, outputs)
    "1x16_rtn_row": (1, False, 1),
    "1x16_rtn_col": (2, False, 1),
    "1x16_rtn_rowcol": (3, False, 2),
    "16x16_2d_rowcol": (1 | 2 | 4, False, 2),
    "1x16_sr_row": (1 | 8, False, 1),
    "1x16_sr_col": (2 | 8, False, 1),
    "rht_1x16_sr_col": (8, True, 1),
    "rht_1x16_rtn_col": (0, True, 1),
    "dual_rtn_row_rhtcol": (0, "dual", 2),
    "dual_sr_row_rhtcol": (8, "dual", 2),
}


def run_sweep(args):
    """Quantizer bandwidth sweep: bf16 tensors of 2^n elements in rows of 4096 (N(0,1) with 1 %
    x50 outliers), each mode timed over `steps` calls after `warmup`; one JSON line per point.
    GB/s counts the algorithmic bytes of a call: two 2-byte reads of every element (the amax
    pass and the quantize pass) plus 0.5625 bytes of codes and scales per element per output."""
    import torch
    from nvfp4_bit_quantized_03_b200 import binding as B
    peaks = _peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    lo, hi = args.sweep_min, args.sweep_max
    for log2n in range(lo, hi + 1):
        rows, cols = synth.quant_sweep_shape(log2n)
        ws = torch.empty((max(B.workspace_bytes(rows, cols, 1 | 2 | 8), 16),), dtype=torch.uint8,
                         device=dev)
        x = torch.from_numpy(synth.activations((rows, cols), seed=synth.QUANT_SWEEP_SEED)
                             .view(np.int16)).view(torch.bfloat16).to(dev)
        n = rows * cols
        for name, (flags, rht, outs) in SWEEP_MODES.items():
            dual = rht == "dual"
            qr = B.QuantizedTensor(rows, cols, dev) if (flags & 1 or dual) else None
            qc = B.QuantizedTensor(cols, rows, dev) if (flags & 2 or rht) else None
            if dual:
                fn = lambda: B.quantize_row_rht(x, 0x5A3C, flags, seed=1, out_row=qr,  # noqa: E731
                                                out_col=qc, workspace=ws)
            elif rht:
                fn = lambda: B.rht_quantize(x, 0x5A3C, flags, seed=1, out_col=qc, workspace=ws)  # noqa: E731
            else:
                fn = lambda: B.quantize(x, flags, seed=1, out_row=qr, out_col=qc, workspace=ws)  # noqa: E731
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            # the calls are replayed from a CUDA graph so that small sizes time the GPU, not
            # the Python dispatch; a graph that cannot be captured falls back to plain calls
            graph = None
            try:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for _ in range(args.steps):
                        fn()
                graph = g
            except RuntimeError:
                torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            if graph is not None:
                graph.replay()
            torch.cuda.synchronize()
            e0.record()
            if graph is not None:
                graph.replay()
            else:
                for _ in range(args.steps):
                    fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
            graph_used = graph is not None
            del graph
            gbs = n * (4 + outs * (0.5 + 1 / 16)) / (ms / 1e3) / 1e9
            print(json.dumps({"sweep": "quantize", "log2n": log2n, "mode": name, "ms": ms,
                              "graph": graph_used,
                              "input_fits_in_l2": 2 * n < 126 * 2**20,
                              "gbps": gbs, "frac_of_measured_hbm": gbs / peaks["hbm_gbs"]}),
                  flush=True)
            del qr, qc
        del x
        torch.cuda.empty_cache()
    return 0


def run_dense8b(args):
    """8B-class dense transformer layer stack at tokens 16384, d 4096: four layers whose five
    linears (QKV 4096->6144, O 4096->4096, gate and up 4096->14336, down 14336->4096) run
    fprop + dgrad + wgrad with the full NVFP4 recipe, and a final layer whose linears stay bf16
    (the pages' selective-precision policy), run as torch bf16 matmuls (cuBLAS) and timed apart.
    The four NVFP4 layers share one set of synthetic inputs: their work is identical.  Prints
    one JSON line (not the benchmark's headline line)."""
    import torch
    wl = synth.dense_8b_layer()
    dev = torch.device("cuda", torch.cuda.current_device())
    step = Step(wl, dev)
    layers = 4

    def bf16_layer():
        for L in step.layers:
            X, W, dY = L["X"], L["W"], L["dY"]
            torch.matmul(X, W.t(), out=L["bf16_out"][0])
            torch.matmul(dY, W, out=L["bf16_out"][1])
            torch.matmul(dY.t(), X, out=L["bf16_out"][2])

    for L in step.layers:
        T, I, O = L["lin"].T, L["lin"].I, L["lin"].O
        L["bf16_out"] = (torch.empty((T, O), dtype=torch.bfloat16, device=dev),
                         torch.empty((T, I), dtype=torch.bfloat16, device=dev),
                         torch.empty((O, I), dtype=torch.bfloat16, device=dev))
    for _ in range(args.warmup):
        for _ in range(layers):
            step.run()
        bf16_layer()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    nv_ms = bf_ms = 0.0
    for _ in range(args.steps):
        ev[0].record()
        for _ in range(layers):
            step.run()
        ev[1].record()
        bf16_layer()
        ev[2].record()
        torch.cuda.synchronize()
        nv_ms += ev[0].elapsed_time(ev[1])
        bf_ms += ev[1].elapsed_time(ev[2])
    nv_ms /= args.steps
    bf_ms /= args.steps
    flops_layer = step.gemm_flops
    st = int(step.dev_status.item())
    print(json.dumps({
        "workload": wl.name, "steps": args.steps, "warmup": args.warmup,
        "nvfp4_layers": layers, "nvfp4_ms_per_step": nv_ms,
        "nvfp4_tflops": layers * flops_layer / (nv_ms / 1e3) / 1e12,
        "nvfp4_tflop_per_step": layers * flops_layer / 1e12,
        "bf16_layer_ms": bf_ms, "bf16_tflops": flops_layer / (bf_ms / 1e3) / 1e12,
        "bf16_share_of_step": bf_ms / (nv_ms + bf_ms),
        "recipe": "NVFP4 layers: W 16x16 RTN, X 1x16 RTN + RHT16 col, dY 1x16 SR + RHT16 SR col; "
                  "bf16 layer: torch.matmul (cuBLAS), no quantization",
        "data": "synthetic, seed 4: activations N(0,1) with 1% x50, weights N(0,0.02), "
                "gradients N(0,1e-3) with 0.5% x100; one input set shared by the 4 NVFP4 layers",
        "dev_status": st}), flush=True)
    return 0 if st == 0 else 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["gemm", "gemm_f32", "gemm_amax", "chain", "chain_amax",
                                         "gemm_mx", "rowwise", "rowwise_rtn", "tile2d", "rht",
                                         "dual", "dual_rtn", "rowwise_mx", "rht_mx"], default=None,
                    help="time one kernel family alone at the workload's shapes (profiling)")
    ap.add_argument("--sweep", action="store_true",
                    help="quantizer bandwidth sweep over 2^n-element tensors (one line per point)")
    ap.add_argument("--sweep-min", type=int, default=20)
    ap.add_argument("--sweep-max", type=int, default=30)
    ap.add_argument("--workload", choices=["mlp12b", "dense8b"], default="mlp12b",
                    help="dense8b: the 8B-class layer stack (4 NVFP4 layers + 1 bf16 layer), "
                         "reported on its own JSON line")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.kernel:
        return run_kernel_case(args)
    if args.sweep:
        return run_sweep(args)
    if args.workload == "dense8b":
        return run_dense8b(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
