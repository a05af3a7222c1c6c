"""Benchmark of the NVFP4 W4A4 linear hot path on B200.

One step = the weight-gradient GEMM of the DiT FFN up projection, the largest
of the workloads on one GPU, through the whole path: dY bf16 [32768, 3072]
and X bf16 [32768, 14336] each get the global amax of their 16-point
random-Hadamard-transformed values and the RHT-fused, transposing 1D NVFP4
quantization (16-blocks along the 32768 tokens, 4-vs-6 on), then the tcgen05
block-scaled FP4 GEMM dW = dY^T X [3072, 14336] with an fp32 output.  `value`
is whole-step throughput in TFLOP/s of the GEMM's 2*M*N*K (quantization time
included), inputs resident in HBM, L2 flushed between steps, device-timed
with CUDA events, max over ranks.  Each rank runs its own independent step
(weak scaling, no data-path collective).  The other workloads (QKV
projection, FFN pair, KV cache, data gradient, window gather) are timed as
rows.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NVFP4 GEMM TFLOPS (%FP4 peak) and quantize/dequant GB/s (%HBM) on 1 B200"
T_TOK, D_OUT, D_IN = 32768, 3072, 14336   # dW = dY^T X: M = D_OUT, N = D_IN, K = T_TOK
WORKLOAD = ("DiT weight gradient of the FFN up projection, W4A4: dY bf16 [32768x3072] "
            "N(0,1e-3), X bf16 [32768x14336] N(0,1) with 1% Student-t(3)x8 channels; "
            "RHT16 along tokens (shared random signs) + transposing 1D NVFP4 quantization "
            "(4-vs-6 on) of both; dW = dY^T X [3072x14336] fp32")
FLUSH_BYTES = 256 << 20
# our kernels per step: amax + encode for dY, amax + encode for X, the GEMM
# library launches per headline step: amax and encode for dY and X, the GEMM,
# and the GEMM's split-tail reduction when its workspace enables the split
LAUNCHES_PER_STEP_UNSPLIT = 5
QOUT = 0.5 + 1.0 / 16  # bytes written per quantized element (codes + scale bytes)


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of
# the step's kernels from ncu captures, valid only for the sources they were
# taken on (hash of the kernel's source files).
TRAFFIC = {
    # one ncu capture of the full-size step: python bench.py --profile
    # wgrad_step, the first rep's six launches (after the four setup ones);
    # "gemm" is the GEMM with its split last round plus the reduction of the
    # split tiles' partial sums (gemm_kernel<true> + split_reduce_kernel)
    "gemm": {"bytes_per_launch": 978168832 + 162859776 + 18881280 + 0,
             "source_sha256": "a98bdb93b5a01ecee19b2418a8fcee018491071c9762879bac0daebc5c0ccf57"},
    "encode_x": {"bytes_per_launch": 954204160 + 251442176,
                 "source_sha256": "d443ba1bae7321cd2d15be6d2775c8c68c4ae04fb60685defd54ee1f4596e1ec"},
    "amax_x": {"bytes_per_launch": 939580928 + 470272,
               "source_sha256": "d443ba1bae7321cd2d15be6d2775c8c68c4ae04fb60685defd54ee1f4596e1ec"},
}


def _sources_digest(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        try:
            h.update(open(os.path.join(ROOT, "nvfp4_block_scaled_20_b200", "csrc", f), "rb").read())
        except OSError:
            return None
    return h.hexdigest()


KERNEL_SOURCES = {"gemm": ["gemm.cu", "device_common.cuh"],
                  "encode_x": ["quantize.cu", "device_common.cuh"],
                  "amax_x": ["quantize.cu", "device_common.cuh"]}


def kernel_traffic(kernel):
    rec = TRAFFIC.get(kernel)
    if not rec or rec["source_sha256"] != _sources_digest(KERNEL_SOURCES[kernel]):
        return None
    return rec["bytes_per_launch"]


def launches_per_step(nv, ws_g):
    """Library launches of one headline step: the GEMM adds its split-tail
    reduction kernel when ws_g is large enough for the split."""
    from nvfp4_block_scaled_20_b200 import capi
    split = ws_g.numel() > capi.nvfp4_workspace_bytes(0)
    return LAUNCHES_PER_STEP_UNSPLIT + (1 if split else 0)


def peaks():
    """Roofline denominators from MEASURED_PEAKS.json (driver-written), else
    the pool's fallback measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)
        return self.summary()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ dist
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle
# Bounded sample of the step for the oracle: every token (the GEMM's K), the
# first CPU_A columns of dY (rows of dW) and CPU_B columns of X per host
# thread (columns of dW): RHT16 + transposing quantization of those columns,
# then the fp64 GEMM of their CPU_A x (CPU_B * threads) outputs.
CPU_A, CPU_B = 64, 64


def host_threads():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


class CpuWgradSample:
    """The oracle's share of the step on `threads` host threads (the C
    oracle releases the interpreter lock, so its calls run in parallel).
    Inputs: the sample's columns, generated on the host."""

    def __init__(self, threads):
        from nvfp4_block_scaled_20_b200 import synth
        self.threads = threads
        self.mask = synth.rht_sign_mask(0)
        self.dy = synth.activation_cols(4, 1, T_TOK, D_OUT, 0, CPU_A, n_out=0,
                                        std=1e-3).float().numpy()
        self.x = synth.activation_cols(4, 2, T_TOK, D_IN, 0, CPU_B * threads).float().numpy()
        self.flops = 2.0 * CPU_A * CPU_B * threads * T_TOK

    def step(self, pool):
        import numpy as np
        import oracle
        mask = self.mask
        qa = oracle.quantize_1d(self.dy, rht=True, mask=mask, block_axis=1, sf_layout=1)

        def part(t):
            xb = np.ascontiguousarray(self.x[:, t * CPU_B:(t + 1) * CPU_B])
            qb = oracle.quantize_1d(xb, rht=True, mask=mask, block_axis=1, sf_layout=1)
            oracle.gemm((qa[0], qa[1], qa[2], 1), (qb[0], qb[1], qb[2], 1), CPU_A, CPU_B, T_TOK)

        list(pool.map(part, range(self.threads)))
        return self.flops

    def describe(self):
        return ("RHT16 + transposing quantization of dY[:, :%d] and X[:, :%d] over all %d "
                "tokens, fp64 GEMM of the %dx%d outputs (C oracle, %d host threads over "
                "column blocks of X)" % (CPU_A, CPU_B * self.threads, T_TOK, CPU_A,
                                         CPU_B * self.threads, self.threads))


def cpu_single_thread_quantizers():
    """Single-threaded oracle quantizers (GB/s at the algorithmic 4.5625 B per
    bf16 element): the QKV projection's X [2640, 3072] (1D) and the first
    2304 rows of its W [9216, 3072] (2D), and the first 65520 rows (two heads)
    of one KV tensor [24 * 32760, 128] (1D, row-major scales)."""
    import oracle
    from nvfp4_block_scaled_20_b200 import synth
    x = synth.activation(1, 1, 2640, 3072).float().numpy()
    w = synth.weight(1, 2, 9216, 3072)[:2304].float().numpy().copy()
    kv = synth.kv_tensor(3, 0, 0, heads=2).float().numpy()
    out = {}
    for name, fn, a in (("qkv_X_2640x3072_1d", oracle.quantize_1d, x),
                        ("qkv_W_2304x3072_2d", oracle.quantize_2d, w),
                        ("kv_65520x128_1d", oracle.quantize_1d, kv)):
        t0 = time.perf_counter()
        fn(a)
        el = time.perf_counter() - t0
        out[name] = {"GB/s": round((4 + QOUT) * a.size / el / 1e9, 4), "s": round(el, 3)}
    return out


def cpu_baseline(min_seconds=10.0):
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    oracle.build()
    threads = host_threads()
    smp = CpuWgradSample(threads)
    with ThreadPoolExecutor(max_workers=threads) as pool:
        smp.step(pool)  # warm-up
        flops, t0 = 0.0, time.perf_counter()
        while True:
            flops += smp.step(pool)
            el = time.perf_counter() - t0
            if el >= min_seconds:
                break
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "nproc": os.cpu_count(), "sample": smp.describe(),
            "single_thread_quantizers": cpu_single_thread_quantizers()}


def run_reference(args, world, rank):
    """The oracle as the reference arm: each step the bounded sample above,
    on the host's cores; rank 0 only."""
    if rank != 0:
        return 0
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    oracle.build()
    threads = host_threads()
    smp = CpuWgradSample(threads)
    with ThreadPoolExecutor(max_workers=threads) as pool:
        for _ in range(args.warmup):
            smp.step(pool)
        t0 = time.perf_counter()
        flops = 0.0
        for _ in range(args.steps):
            flops += smp.step(pool)
        el = time.perf_counter() - t0
    v = flops / el / 1e12
    sample = "each step: " + smp.describe()
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 encode / f64 accumulate", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ncu cases
PROFILE_CASES = {
    "wgrad_step": "the benchmark's step at full size: RHT16 + transposing quantize of dY "
                  "[32768, 3072] and X [32768, 14336], GEMM dW [3072, 14336] fp32 (1.6 GB on "
                  "the device)",
    "qkv_step": "DiT QKV step: quantize X [2640, 3072] (1D) and W [9216, 3072] (2D) in one "
                "mixed call, GEMM",
    "h_quantize": "1D quantize of an FFN-hidden-sized bf16 [8192, 14336]: amax + encode, "
                  "then encode alone (global scale given)",
    "w_quantize_2d": "2D quantize of W_up [14336, 3072]",
    "wgrad_x_quantize": "RHT16 + transposing quantize of X [8192, 14336] (a quarter of the "
                        "weight-gradient tokens)",
    "kv_quantize": "batched quantize + batched dequant of 4 KV tensors [24 * 32760, 128]",
    "ffn_gemm": "FFN up GEMM + GELU 8192x14336x3072 and down GEMM 8192x3072x14336",
    "wgrad_gemm": "weight-gradient GEMM 3072x14336x8192, fp32 out (a quarter of the tokens)",
    "transpose_2d": "transpose of W_dn's [3072, 14336] 2D encoding (the data-gradient operand)",
}


def run_profile_case(name, reps=3):
    """The case's kernels launched `reps` times on inputs generated once (a few
    GB on the device at most)."""
    import torch
    import nvfp4_block_scaled_20_b200 as nv
    from nvfp4_block_scaled_20_b200 import build, synth
    build.build()
    dev = torch.device("cuda", 0)
    ws = nv.workspace(8, dev)

    ws_g = ws
    if name == "wgrad_step":
        dy, xw, mask = synth.wgrad(dev)
        qdy = nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1, ws=ws)
        qxw = nv.quantize_1d(xw, rht=True, mask=mask, block_axis=1, ws=ws)
        dw = torch.empty((dy.shape[1], xw.shape[1]), dtype=torch.float32, device=dev)
        ws_g = nv.gemm_workspace(dy.shape[1], xw.shape[1], dy.shape[0], device=dev)

        def run():
            nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1, out=qdy, ws=ws)
            nv.quantize_1d(xw, rht=True, mask=mask, block_axis=1, out=qxw, ws=ws)
            nv.gemm(qdy, qxw, out=dw, ws=ws_g)
    elif name == "qkv_step":
        x, w = synth.qkv_linear(dev)

        def run():
            qx, qw = nv.quantize_mixed([x, w], [False, True], ws=ws)
            nv.gemm(qx, qw, ws=ws)
    elif name == "h_quantize":
        h = synth.activation(2, 9, 8192, 14336, device=dev)
        qh = nv.quantize_1d(h, ws=ws)

        def run():
            nv.quantize_1d(h, out=qh, ws=ws)
            nv.quantize_1d(h, alpha_in=qh.alpha, out=qh, ws=ws)
    elif name == "w_quantize_2d":
        w = synth.weight(2, 2, 14336, 3072, device=dev)

        def run():
            nv.quantize_2d(w, ws=ws)
    elif name == "wgrad_x_quantize":
        x = synth.activation(4, 2, 8192, 14336, device=dev)

        def run():
            nv.quantize_1d(x, rht=True, mask=synth.rht_sign_mask(0), block_axis=1, ws=ws)
    elif name == "kv_quantize":
        kv = [synth.kv_tensor(3, l, wh, device=dev) for l in range(2) for wh in range(2)]

        def run():
            nv.dequantize(nv.quantize_1d_batched(kv, ws=ws))
    elif name == "ffn_gemm":
        x, wu, wd = synth.ffn_pair(dev)
        qx, qu, qd = nv.quantize_1d(x, ws=ws), nv.quantize_2d(wu, ws=ws), nv.quantize_2d(wd, ws=ws)
        h = torch.empty((x.shape[0], wu.shape[0]), dtype=torch.bfloat16, device=dev)
        qh = nv.quantize_1d(h.zero_(), ws=ws)

        def run():
            nv.gemm(qx, qu, out=h, epilogue=nv.NVFP4_EPI_GELU_TANH, ws=ws)
            nv.gemm(nv.quantize_1d(h, out=qh, ws=ws), qd, ws=ws)
    elif name == "transpose_2d":
        wd = synth.weight(2, 3, 3072, 14336, device=dev)
        qd = nv.quantize_2d(wd, ws=ws)
        qt = nv.transpose_2d(qd)

        def run():
            nv.transpose_2d(qd, out=qt)
    else:  # wgrad_gemm
        dy, xw, mask = synth.wgrad(dev, t=8192)
        qdy = nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1, ws=ws)
        qxw = nv.quantize_1d(xw, rht=True, mask=mask, block_axis=1, ws=ws)
        ws_g = nv.gemm_workspace(dy.shape[1], xw.shape[1], dy.shape[0], device=dev)

        def run():
            nv.gemm(qdy, qxw, out_dtype=torch.float32, ws=ws_g)

    for _ in range(reps):
        run()
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0 and nv.device_error(ws_g) == 0
    print("profile case %s: %s, %d reps" % (name, PROFILE_CASES[name], reps))
    return 0


# ------------------------------------------------------------------ GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--rows", default="auto", choices=["auto", "on", "off"],
                    help="also time every hot-path row at its full workload size "
                         "(auto: on a single GPU only)")
    ap.add_argument("--profiler-range", action="store_true",
                    help="bracket the timed step replays with cudaProfilerStart/Stop (for a "
                         "launch list taken with ncu --profile-from-start off)")
    ap.add_argument("--profile", default=None, choices=sorted(PROFILE_CASES),
                    help="run one case a few times (untimed, no JSON line): the program "
                         "the ncu captures under profiles/ are taken on")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.profile:
        return run_profile_case(args.profile)

    import torch
    import nvfp4_block_scaled_20_b200 as nv
    from nvfp4_block_scaled_20_b200 import build, synth
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    pk = peaks()

    # inputs: each rank its own batch (seeded by rank), resident in HBM
    if rank == 0:
        dy, xw, mask = synth.wgrad(dev)
    else:
        dy = synth.activation(4 + 1000 * rank, 1, T_TOK, D_OUT, n_out=0, std=1e-3, device=dev)
        xw = synth.activation(4 + 1000 * rank, 2, T_TOK, D_IN, device=dev)
        mask = synth.rht_sign_mask(0)
    # the generator runs on torch's current stream, the path on `stream`
    torch.cuda.synchronize(dev)
    T = nv.NVFP4_SF_TCGEN05
    qdy = nv.QTensor(*nv._alloc_q(D_OUT, T_TOK, T, dev), D_OUT, T_TOK, T)
    qxw = nv.QTensor(*nv._alloc_q(D_IN, T_TOK, T, dev), D_IN, T_TOK, T)
    dw = torch.empty((D_OUT, D_IN), dtype=torch.float32, device=dev)
    ws_dy, ws_x = nv.workspace(1, dev), nv.workspace(1, dev)
    # the GEMM's workspace with room for its split last round
    ws_g = nv.gemm_workspace(D_OUT, D_IN, T_TOK, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer larger than L2 (evicts every input), then read another
        # one so the next kernel does not pay for writing back dirty lines
        flush.zero_()
        torch.sum(flush_rd, dim=0, out=flush_sink)

    def quant(x, q, ws, alpha_in=None):
        nv.quantize_1d(x, rht=True, mask=mask, block_axis=1, out=q, ws=ws, alpha_in=alpha_in,
                       stream=stream)

    def amax(x, q, ws):
        nv.global_scale(x, rht=True, mask=mask, block_axis=1, out=q.alpha, ws=ws, stream=stream)

    def gemm():
        nv.gemm(qdy, qxw, out=dw, ws=ws_g, stream=stream)

    def step():
        quant(dy, qdy, ws_dy)
        quant(xw, qxw, ws_x)
        gemm()

    # warm-up (also sets kernel attributes before graph capture)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    assert nv.device_error(ws_g, stream) == 0

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    graphs = {"step": capture(step),
              "quant_dy": capture(lambda: quant(dy, qdy, ws_dy)),
              "amax_dy": capture(lambda: amax(dy, qdy, ws_dy)),
              "encode_dy": capture(lambda: quant(dy, qdy, ws_dy, qdy.alpha)),
              "quant_x": capture(lambda: quant(xw, qxw, ws_x)),
              "amax_x": capture(lambda: amax(xw, qxw, ws_x)),
              "encode_x": capture(lambda: quant(xw, qxw, ws_x, qxw.alpha)),
              "gemm": capture(gemm)}

    def timed(g, reps):
        """Mean device time (ms) of one graph replay, L2 flushed before each."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        with torch.cuda.stream(stream):
            torch.cuda._sleep(2_000_000)  # let the host run ahead of the device
            for s0, e0 in evs:
                flush_l2()
                s0.record(stream)
                g.replay()
                e0.record(stream)
        stream.synchronize()
        return sum(s0.elapsed_time(e0) for s0, e0 in evs) / reps

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graphs["step"].replay()
    stream.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)
    barrier(world)
    torch.cuda.synchronize(dev)
    if args.profiler_range:
        torch.cuda.profiler.start()
    step_ms = timed(graphs["step"], args.steps)
    torch.cuda.synchronize(dev)
    if args.profiler_range:
        torch.cuda.profiler.stop()
    barrier(world)
    # per-kernel breakdown (same protocol)
    reps = max(10, min(args.steps, 100))
    part = {k: timed(graphs[k], reps) for k in graphs if k != "step"}
    assert nv.device_error(ws_g, stream) == 0

    step_ms_max = reduce_max(step_ms, world, dev)
    flops = 2.0 * D_OUT * D_IN * T_TOK
    value = world * flops / (step_ms_max * 1e-3) / 1e12

    fp4_peak = 4.0 * pk["bf16_tflops"]  # nominal FP4:BF16 dense ratio 9 : 2.25
    hbm = pk["hbm_gbs"]

    def gbs(nbytes, ms):
        v = nbytes / (ms * 1e-3) / 1e9
        return {"ms": round(ms, 5), "GB/s": round(v, 1), "frac_hbm": round(v / hbm, 3)}

    n_dy, n_x = T_TOK * D_OUT, T_TOK * D_IN
    gemm_tflops = flops / (part["gemm"] * 1e-3) / 1e12
    breakdown = {
        "gemm": {"ms": round(part["gemm"], 5), "TFLOP/s": round(gemm_tflops, 1),
                 "frac_fp4_peak": round(gemm_tflops / fp4_peak, 3)},
        "quantize_dy": gbs((4 + QOUT) * n_dy, part["quant_dy"]),
        "amax_only_dy": gbs(2 * n_dy, part["amax_dy"]),
        "encode_only_dy": gbs((2 + QOUT) * n_dy, part["encode_dy"]),
        "quantize_x": gbs((4 + QOUT) * n_x, part["quant_x"]),
        "amax_only_x": gbs(2 * n_x, part["amax_x"]),
        "encode_only_x": gbs((2 + QOUT) * n_x, part["encode_x"]),
        "traffic_bytes": {"gemm": kernel_traffic("gemm"), "encode_x": kernel_traffic("encode_x"),
                          "amax_x": kernel_traffic("amax_x")},
        "note": "quantize_* = the step's two launches (amax pass, then the encode pass that "
                "reduces the amax partials into the global scale) counted at the algorithmic "
                "two-read bytes (4 + 0.5625 B/element); encode_only_* = the encode pass alone "
                "with the global scale given (2 + 0.5625 B/element); amax_only_* = the amax "
                "pass and the global-scale reduction (2 B/element).  Each timed after an L2 "
                "flush.",
    }
    # roofline of the step's dominant kernel (largest share of the step)
    cands = {"gemm": part["gemm"], "encode_x": part["encode_x"], "amax_x": part["amax_x"]}
    top = max(cands, key=cands.get)
    if top == "gemm":
        roof = {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1),
                "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4),
                "traffic": kernel_traffic("gemm"),
                "kernel": ("gemm_kernel (CTA-pair tcgen05.mma kind::mxf4nvf4), 3072x14336x32768"
                           + (", last round split along K + split_reduce_kernel"
                              if launches_per_step(nv, ws_g) > LAUNCHES_PER_STEP_UNSPLIT else "")),
                "peak_source": "%s bf16 burst %.1f TFLOP/s x 4 (nominal dense FP4:BF16 "
                               "ratio)" % (pk["source"], pk["bf16_tflops"])}
    else:
        nb = (2 + QOUT) * n_x if top == "encode_x" else 2 * n_x
        ach = nb / (part[top] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 4), "traffic": kernel_traffic(top),
                "kernel": ("encode_cols_tma_kernel<rht> (transposing RHT16 encode of X)"
                           if top == "encode_x" else "amax_cols_tma_kernel<rht> of X"),
                "peak_source": "%s HBM copy bandwidth" % pk["source"]}
    roof["algorithmic"] = ("GEMM: 2*M*N*K FLOP per launch; encode: 2 B read + 0.5625 B "
                           "written per element; amax: 2 B read per element")
    roof["shares_ms"] = {k: round(v, 5) for k, v in cands.items()}

    rows = None
    if args.rows == "on" or (args.rows == "auto" and world == 1):
        del graphs
        graphs = None
        torch.cuda.empty_cache()
        rows = measure_rows(nv, synth, torch, dev, stream, timed, pk, reps)
        rows["a2_rht16_transposed_quantize"] = {
            "X_32768x14336": dict(breakdown["quantize_x"], bytes=int((4 + QOUT) * n_x)),
            "dY_32768x3072": dict(breakdown["quantize_dy"], bytes=int((4 + QOUT) * n_dy)),
            "note": "from the headline step's breakdown"}
        rows["a5_gemm"]["wgrad_3072x14336x32768_fp32"] = dict(breakdown["gemm"], flops=flops)
        rows["steps"]["wgrad"] = {"ms": round(step_ms, 5),
                                  "TFLOP/s": round(flops / (step_ms * 1e-3) / 1e12, 1),
                                  "frac_fp4_peak": round(flops / (step_ms * 1e-3) / 1e12
                                                         / fp4_peak, 3),
                                  "flops": flops, "note": "the headline step"}
    # clocks sampled over every timed region (step, breakdown, rows)
    clk = clocks.stop()

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(nv, torch, dev, stream, dy, xw, mask, qdy, qxw, ws_dy, ws_x, ws_g,
                          args, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 scales, fp32 accumulate; fp32 encode)",
            "data": "synthetic (seeded splitmix64 generator, DiT weight-gradient shapes)",
            "config": {"workload": WORKLOAD, "M": D_OUT, "N": D_IN, "K": T_TOK,
                       "parallelism": "replica per GPU (weak scaling)" if world > 1 else "single GPU",
                       "l2": "flushed before every timed step: 256 MiB write, then 256 MiB read "
                             "(the step's inputs, 1.14 GB, are larger than L2 too)",
                       "timing": "CUDA events around a CUDA-graph replay of the step, max over ranks"},
            "roofline": roof,
            "breakdown": breakdown,
            "gpu_launches": launches_per_step(nv, ws_g) * args.steps,
            "clocks": clk,
        }
        if rows:
            line["rows"] = rows
        if e2e:
            line["e2e"] = e2e
        if cpu:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del graphs
        dist.destroy_process_group()
    return 0


def measure_rows(nv, synth, torch, dev, stream, timed, pk, reps):
    """Every other hot-path row at its full workload size, same protocol as the
    step (graph replay between CUDA events, L2 flushed before each replay):

    the DiT QKV step (mixed quantize of X [2640, 3072] 1D and W [9216, 3072]
    2D, GEMM); a1 global amax, a3 1D quantize and a5 GEMMs on the DiT FFN
    pair (X [8192, 3072], W_up [14336, 3072], W_dn [3072, 14336], H [8192,
    14336]); a4 2D quantize on both FFN weights; the data-gradient GEMM on
    transposed weight codes; a6 batched quantize and a7 batched dequant of
    the 60-tensor KV cache (30 layers x {K, V} x [24 * 32760, 128]) and the
    window gather; and, as context only (not on the product path), the same
    GEMM shapes through cuBLAS's NVFP4 GEMM (torch._scaled_mm) where this torch
    exposes it.  Bytes are the algorithmic ones: an input read by both passes
    counts twice.  The weight-gradient rows come from the headline step."""
    hbm = pk["hbm_gbs"]
    fp4 = 4.0 * pk["bf16_tflops"]
    T = nv.NVFP4_SF_TCGEN05
    qout = 0.5 + 1.0 / 16

    def graph(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    def bw(fn, nbytes, note=None):
        ms = timed(graph(fn), reps)
        v = nbytes / (ms * 1e-3) / 1e9
        r = {"ms": round(ms, 5), "GB/s": round(v, 1), "frac_hbm": round(v / hbm, 3),
             "bytes": int(nbytes)}
        if note:
            r["note"] = note
        return r

    def tc(fn, flops):
        ms = timed(graph(fn), reps)
        v = flops / (ms * 1e-3) / 1e12
        return {"ms": round(ms, 5), "TFLOP/s": round(v, 1), "frac_fp4_peak": round(v / fp4, 3),
                "flops": flops}

    def q(rows, cols, layout=T):
        return nv.QTensor(*nv._alloc_q(rows, cols, layout, dev), rows, cols, layout)

    out = {}
    ws = nv.workspace(1, dev)
    # ---------------- FFN pair
    x, wu, wd = synth.ffn_pair(dev)
    torch.cuda.synchronize(dev)  # generated on torch's current stream
    Mf, D = x.shape
    Hd = wu.shape[0]
    qx, qu, qd, qh = q(Mf, D), q(Hd, D), q(D, Hd), q(Mf, Hd)
    h = torch.empty((Mf, Hd), dtype=torch.bfloat16, device=dev)
    y = torch.empty((Mf, D), dtype=torch.bfloat16, device=dev)
    nv.quantize_1d(x, out=qx, ws=ws, stream=stream)
    nv.quantize_2d(wu, out=qu, ws=ws, stream=stream)
    nv.quantize_2d(wd, out=qd, ws=ws, stream=stream)
    nv.gemm(qx, qu, out=h, epilogue=nv.NVFP4_EPI_GELU_TANH, ws=ws, stream=stream)
    ne_h = Mf * Hd
    out["a1_global_amax"] = {
        "H_8192x14336": bw(lambda: nv.global_scale(h, out=qh.alpha, ws=ws, stream=stream),
                           2 * ne_h)}
    out["a3_quantize_1d"] = {
        "H_8192x14336": bw(lambda: nv.quantize_1d(h, out=qh, ws=ws, stream=stream),
                           (4 + qout) * ne_h),
        "H_8192x14336_encode_only": bw(
            lambda: nv.quantize_1d(h, out=qh, ws=ws, alpha_in=qh.alpha, stream=stream),
            (2 + qout) * ne_h),
        "X_8192x3072": bw(lambda: nv.quantize_1d(x, out=qx, ws=ws, stream=stream),
                          (4 + qout) * Mf * D, "50 MB input: its second read hits L2"),
    }
    out["a4_quantize_2d"] = {
        "W_up_14336x3072": bw(lambda: nv.quantize_2d(wu, out=qu, ws=ws, stream=stream),
                              (4 + qout) * Hd * D, "88 MB input: its second read hits L2"),
        "W_dn_3072x14336": bw(lambda: nv.quantize_2d(wd, out=qd, ws=ws, stream=stream),
                              (4 + qout) * Hd * D, "88 MB input: its second read hits L2"),
    }
    nv.quantize_1d(h, out=qh, ws=ws, stream=stream)
    g_up = tc(lambda: nv.gemm(qx, qu, out=h, epilogue=nv.NVFP4_EPI_GELU_TANH, ws=ws,
                              stream=stream), 2.0 * Mf * Hd * D)
    ws_dn = nv.gemm_workspace(Mf, D, Hd, device=dev)  # the down GEMM splits its last round
    g_dn = tc(lambda: nv.gemm(qh, qd, out=y, ws=ws_dn, stream=stream), 2.0 * Mf * D * Hd)

    ws_h = nv.workspace(1, dev)

    def ffn_step():
        nv.quantize_1d(x, out=qx, ws=ws, stream=stream)
        # the up GEMM leaves H's amax in ws_h: H's quantization is one encode pass
        nv.gemm(qx, qu, out=h, epilogue=nv.NVFP4_EPI_GELU_TANH, amax_ws=ws_h, stream=stream)
        nv.quantize_1d(h, out=qh, ws=ws_h, amax_ready=True, stream=stream)
        nv.gemm(qh, qd, out=y, ws=ws_dn, stream=stream)

    ffn = tc(ffn_step, 4.0 * Mf * Hd * D)
    ffn["note"] = ("quantize X, up GEMM + GELU recording H's amax, encode H (no amax pass), "
                   "down GEMM (weights pre-quantized)")

    # data gradient of the down projection: dX [8192, 14336] = dY [8192, 3072] . W_dn,
    # W_dn's 2D encoding transposed (no re-quantization)
    dyf = synth.activation(2, 7, Mf, D, n_out=0, std=1e-3, device=dev)
    torch.cuda.synchronize(dev)
    qdy, qdt = q(Mf, D), q(Hd, D)
    qdt.alpha = qd.alpha
    dx = torch.empty((Mf, Hd), dtype=torch.bfloat16, device=dev)
    nv.quantize_1d(dyf, out=qdy, ws=ws, stream=stream)
    out["next1_dgrad"] = {
        "transpose_2d_W_dn_3072x14336": bw(
            lambda: nv.transpose_2d(qd, out=qdt, stream=stream), 2 * (0.5 + 1.0 / 16) * Hd * D,
            "codes and tile scales read once and written once"),
        "dgrad_gemm_8192x14336x3072": tc(lambda: nv.gemm(qdy, qdt, out=dx, ws=ws, stream=stream),
                                         2.0 * Mf * Hd * D),
    }
    del x, wu, wd, qx, qu, qd, qh, h, y, dyf, qdy, qdt, dx

    out["a5_gemm"] = {"ffn_up_gelu_8192x14336x3072": g_up, "ffn_down_8192x3072x14336": g_dn}
    out["steps"] = {"ffn_pair": ffn}

    # ---------------- QKV projection (the mixed quantize call and the GEMM)
    xq, wq = synth.qkv_linear(dev)
    torch.cuda.synchronize(dev)
    Mq, Kq = xq.shape
    Nq = wq.shape[0]
    qa, qb = q(Mq, Kq), q(Nq, Kq)
    yq = torch.empty((Mq, Nq), dtype=torch.bfloat16, device=dev)
    ws_xw = nv.workspace(2, dev)

    def qkv_quant():
        nv.quantize_mixed([xq, wq], [False, True], outs=[qa, qb], ws=ws_xw, stream=stream)

    def qkv_step():
        qkv_quant()
        nv.gemm(qa, qb, out=yq, ws=ws, stream=stream)

    out["a3_a4_quantize_mixed"] = {"qkv_X_2640x3072_W_9216x3072": bw(
        qkv_quant, (4 + qout) * (Mq + Nq) * Kq,
        "one amax and one encode launch for X (1D) and W (2D); 73 MB of inputs: the second "
        "read hits L2")}
    out["a5_gemm"]["qkv_2640x9216x3072"] = tc(lambda: nv.gemm(qa, qb, out=yq, ws=ws,
                                                              stream=stream), 2.0 * Mq * Nq * Kq)
    out["steps"]["qkv"] = tc(qkv_step, 2.0 * Mq * Nq * Kq)
    out["steps"]["qkv"]["note"] = "mixed quantize of X and W, GEMM, bf16 Y"
    # the same projection with a rank-128, scale-1 adapter fused in (W4A4 + LoRA)
    rl = 128
    lu = synth.activation(22, 101, Mq, rl, n_out=0, std=0.5, device=dev)
    lb = synth.weight(22, 102, Nq, rl, device=dev)
    lscr = torch.empty(nv.capi.nvfp4_lora_scratch_bytes(Mq, rl), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    lora = tc(lambda: nv.gemm_lora(qa, qb, lu, lb, 1.0, out=yq, ws=ws, scratch=lscr,
                                   stream=stream), 2.0 * Mq * Nq * (Kq + rl))
    lora["note"] = ("FP4 GEMM plus the rank-128 bf16 adapter product in the same launch "
                    "(and the adapter input's scaling kernel); flops 2 M N (K + r)")
    out["next4_gemm_lora"] = {"qkv_2640x9216x3072_rank128": lora}
    del xq, wq, qa, qb, yq, lu, lb, lscr

    # ---------------- 4-bit Ulysses payload (one rank's side; the exchange itself
    # needs several GPUs and is not timed here)
    from nvfp4_block_scaled_20_b200 import ulysses
    s_loc, heads, hd, world_sp = 8190, 24, 128, 4  # 32760 tokens over SP = 4
    lay = ulysses.PayloadLayout(s_loc, heads, hd, world_sp)
    qsh = synth.kv_tensor(5, 0, 0, heads=s_loc, tokens=heads, head_dim=hd, device=dev)
    torch.cuda.synchronize(dev)
    sbuf = torch.empty(lay.buffer_bytes, dtype=torch.uint8, device=dev)
    uout = torch.empty((world_sp * s_loc * lay.heads_per_rank, hd), dtype=torch.bfloat16,
                       device=dev)
    ne_q = s_loc * heads * hd
    out["next3_ulysses_payload"] = {
        "pack_Q_8190x24x128": bw(lambda: ulysses.pack(qsh, lay, sbuf, stream=stream),
                                 (4 + qout) * ne_q,
                                 "quantize into the 4 destination segments (two passes)"),
        "unpack_to_bf16": bw(lambda: ulysses.unpack(sbuf, lay, uout, stream=stream),
                             (qout + 2) * ne_q, "dequantize the 4 received segments"),
        "payload_bytes": lay.buffer_bytes, "bf16_bytes": 2 * ne_q,
        "compression": round(2 * ne_q / lay.buffer_bytes, 3),
        "note": "the NCCL all-to-all between the two is not measured: one GPU per run here",
    }
    del qsh, sbuf, uout

    # ---------------- context: the library's NVFP4 GEMM on the same shapes
    out["context_cublas_nvfp4_scaled_mm"] = library_ceiling(torch, dev, tc)

    # ---------------- KV cache
    kv = [synth.kv_tensor(3, l, wh, device=dev) for l in range(30) for wh in range(2)]
    torch.cuda.synchronize(dev)
    R, C = kv[0].shape
    kq = [q(R, C, nv.NVFP4_SF_ROWMAJOR) for _ in kv]
    kout = [torch.empty((R, C), dtype=torch.bfloat16, device=dev) for _ in kv]
    ws_kv = nv.workspace(len(kv), dev)
    ne_kv = len(kv) * R * C
    out["a6_kv_quantize_batched"] = bw(
        lambda: nv.quantize_1d_batched(kv, outs=kq, ws=ws_kv, stream=stream),
        (4 + qout) * ne_kv, "60 tensors, one amax launch + one encode launch")
    out["a7_kv_dequant_batched"] = bw(
        lambda: nv.dequantize(kq, outs=kout, stream=stream), (qout + 2) * ne_kv,
        "60 tensors, one launch")
    # sliding window with sinks: frames of 1560 tokens (32760 = 21 frames);
    # global sink frames [0, 3), shot sink frames [6, 9), window frames [12, 21)
    fr = 1560
    token_ranges = [(0, 3 * fr), (6 * fr, 9 * fr), (12 * fr, 21 * fr)]
    ranges = nv.window_row_ranges(24, R // 24, token_ranges)
    rows_w = nv.merged_rows(ranges)
    wout = [o[:rows_w] for o in kout]
    out["next2_window_gather_dequant"] = bw(
        lambda: nv.dequantize_rows(kq, ranges, outs=wout, stream=stream),
        (qout + 2) * len(kv) * rows_w * C,
        "60 tensors, 24 heads x (3 + 3 + 9 of 21 frames), one launch")
    del kv, kq, kout
    assert (nv.device_error(ws, stream) == 0 and nv.device_error(ws_h, stream) == 0
            and nv.device_error(ws_kv, stream) == 0 and nv.device_error(ws_dn, stream) == 0)
    torch.cuda.empty_cache()
    return out


def library_ceiling(torch, dev, tc):
    """cuBLAS's NVFP4 GEMM (torch._scaled_mm with float4 operands and e4m3
    block scales) on the workloads' GEMM shapes, same timing protocol, bf16
    output: an empirical ceiling reported for context.  Not on the product
    path; operands are random codes with unit scales."""
    if not (hasattr(torch, "float4_e2m1fn_x2") and hasattr(torch, "_scaled_mm")):
        return {"unavailable": "this torch exposes no float4 _scaled_mm"}
    out = {"note": "context only: cuBLAS NVFP4 GEMM via torch._scaled_mm, not the product path"}

    def rup(v, m):
        return (v + m - 1) // m * m

    for name, (M, N, K) in (("qkv_2640x9216x3072", (2640, 9216, 3072)),
                            ("ffn_up_8192x14336x3072", (8192, 14336, 3072)),
                            ("ffn_down_8192x3072x14336", (8192, 3072, 14336)),
                            ("wgrad_3072x14336x32768", (3072, 14336, 32768))):
        try:
            g = torch.Generator(device=dev).manual_seed(M + N + K)
            a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev,
                              generator=g).view(torch.float4_e2m1fn_x2)
            b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev,
                              generator=g).view(torch.float4_e2m1fn_x2)
            sa = torch.full((rup(M, 128), rup(K // 16, 4)), 0x38, dtype=torch.uint8,
                            device=dev).view(torch.float8_e4m3fn)
            sb = torch.full((rup(N, 128), rup(K // 16, 4)), 0x38, dtype=torch.uint8,
                            device=dev).view(torch.float8_e4m3fn)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            out[name] = tc(lambda: torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16,
                                                    out=y), 2.0 * M * N * K)
            del a, b, sa, sb, y
        except Exception as e:  # noqa: BLE001 -- context row only
            out[name] = {"unavailable": str(e).split("\n")[0][:160]}
    return out


def measure_e2e(nv, torch, dev, stream, dy, xw, mask, qdy, qxw, ws_dy, ws_x, ws_g, args, world):
    """The same step through the public API with the inputs copied from pinned
    host memory and the fp32 dW copied back, every step.  Steps are pipelined
    over three streams (inputs in, compute, result out; device buffers double
    buffered), so step i's host-to-device copies overlap step i-1's compute
    and step i-2's device-to-host copy; every step still moves all its bytes
    inside the timed region."""
    hdy = dy.cpu().pin_memory()
    hxw = xw.cpu().pin_memory()
    hdw = [torch.empty((D_OUT, D_IN), dtype=torch.float32).pin_memory() for _ in range(2)]
    ddy = [torch.empty_like(dy) for _ in range(2)]
    dxw = [torch.empty_like(xw) for _ in range(2)]
    dw = [torch.empty((D_OUT, D_IN), dtype=torch.float32, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
    ev_in, ev_used, ev_done, ev_out = ev(), ev(), ev(), ev()
    steps = max(3, min(args.steps, 20))

    def one(i):
        b = i % 2
        # inputs: wait until step i-2's compute has read buffer b
        if i >= 2:
            s_in.wait_event(ev_used[b])
        with torch.cuda.stream(s_in):
            ddy[b].copy_(hdy, non_blocking=True)
            dxw[b].copy_(hxw, non_blocking=True)
        ev_in[b].record(s_in)
        # compute: inputs landed, and step i-2's result has left dw[b]
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])
        nv.quantize_1d(ddy[b], rht=True, mask=mask, block_axis=1, out=qdy, ws=ws_dy, stream=stream)
        nv.quantize_1d(dxw[b], rht=True, mask=mask, block_axis=1, out=qxw, ws=ws_x, stream=stream)
        ev_used[b].record(stream)
        nv.gemm(qdy, qxw, out=dw[b], ws=ws_g, stream=stream)
        ev_done[b].record(stream)
        # result out
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            hdw[b].copy_(dw[b], non_blocking=True)
        ev_out[b].record(s_out)

    def run(n):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(n):
            one(i)
        stream.wait_event(ev_out[(n - 1) % 2])
        stream.wait_event(ev_out[n % 2])
        end.record(stream)
        return start, end

    run(3)
    torch.cuda.synchronize(dev)
    barrier(world)
    s0, e0 = run(steps)
    torch.cuda.synchronize(dev)
    ms = reduce_max(s0.elapsed_time(e0) / steps, world, dev)
    assert nv.device_error(ws_g, stream) == 0
    return {"value": world * 2.0 * D_OUT * D_IN * T_TOK / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": (dy.numel() + xw.numel()) * 2,
            "d2h_bytes_per_step": D_OUT * D_IN * 4,
            "pipelined": "h2d / compute / d2h on three streams, device buffers double buffered"}


if __name__ == "__main__":
    sys.exit(main())
