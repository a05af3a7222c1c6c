"""Benchmark of the NVFP4 W4A4 linear hot path on B200.

One step = the DiT QKV projection (X bf16 [2640, 3072], W bf16 [9216, 3072])
through the whole path: global amax + 1D quantization of X (4-vs-6 on),
global amax + 2D 16x16 quantization of W (4-vs-6 on), tcgen05 block-scaled
FP4 GEMM Y = X W^T with a bf16 output.  `value` is whole-step throughput in
TFLOP/s of the GEMM's 2*M*N*K (quantization time included), inputs resident
in HBM, L2 flushed between steps, device-timed with CUDA events, max over
ranks.  Each rank runs its own independent step (weak scaling, no data-path
collective).

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
M, N, K = 2640, 9216, 3072
WORKLOAD = "DiT QKV projection W4A4: X bf16 [2640x3072] (1% Student-t(3)x8 channels), " \
           "W bf16 [9216x3072] N(0,0.02); 1D act + 2D weight NVFP4, 4-vs-6 on; Y bf16 [2640x9216]"
FLUSH_BYTES = 256 << 20
# our kernels per step: one amax and one encode launch for X and W together
# (nvfp4_quantize_mixed), the GEMM
LAUNCHES_PER_STEP = 3
# CPU-oracle sample: the first rows of the same workload
CPU_MS, CPU_NS = 64, 128


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one QKV-shape
# GEMM launch from an ncu capture (profiles/gemm_kernel_2sm_qkv_and_ffn.md),
# valid only for the kernel source it was taken on.
GEMM_TRAFFIC = {"source_sha256": "168fb4235c29b87813e02abca004d94d89bdaa83efa2e3d15356fca6914bc170",
                "bytes_per_launch": 20541440 + 4496896}


def gemm_traffic():
    import hashlib
    src = os.path.join(ROOT, "nvfp4_block_scaled_20_b200", "csrc", "gemm.cu")
    try:
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    if GEMM_TRAFFIC["source_sha256"] != digest:
        return None
    return GEMM_TRAFFIC["bytes_per_launch"]


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
def cpu_sample_step(x_rows, w_rows):
    """The oracle on a bounded sample of the workload: quantize the first
    CPU_MS activation rows and CPU_NS weight rows, then the fp64 GEMM of the
    CPU_MS x CPU_NS outputs.  Returns the sample's 2*m*n*K."""
    import oracle
    a = oracle.quantize_1d(x_rows, sf_layout=oracle.SF_TCGEN05)
    b = oracle.quantize_2d(w_rows, sf_layout=oracle.SF_TCGEN05)
    oracle.gemm((a[0], a[1], a[2], 1), (b[0], b[1], b[2], 1), x_rows.shape[0], w_rows.shape[0], K)
    return 2.0 * x_rows.shape[0] * w_rows.shape[0] * K


def cpu_inputs():
    from nvfp4_block_scaled_20_b200 import synth
    x, w = synth.qkv_linear("cpu")
    return (x[:CPU_MS].float().numpy().copy(), w[:CPU_NS].float().numpy().copy())


def cpu_baseline(min_seconds=10.0):
    import oracle
    oracle.build()
    xr, wr = cpu_inputs()
    flops, t0, reps = 0.0, time.perf_counter(), 0
    while True:
        flops += cpu_sample_step(xr, wr)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": "%d reps of: 1D-quantize X[:%d], 2D-quantize W[:%d], fp64 GEMM %dx%dx%d "
                      "(single-threaded C oracle)" % (reps, CPU_MS, CPU_NS, CPU_MS, CPU_NS, K)}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    xr, wr = cpu_inputs()
    for _ in range(args.warmup):
        cpu_sample_step(xr, wr)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += cpu_sample_step(xr, wr)
    el = time.perf_counter() - t0
    v = flops / el / 1e12
    sample = ("each step: 1D-quantize X[:%d], 2D-quantize W[:%d], fp64 GEMM %dx%dx%d "
              "(single-threaded C oracle)" % (CPU_MS, CPU_NS, CPU_MS, CPU_NS, K))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 encode / f64 accumulate", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ncu cases
PROFILE_CASES = {
    "qkv_step": "DiT QKV step: quantize X [2640, 3072] (1D) and W [9216, 3072] (2D) in one mixed call, GEMM",
    "h_quantize": "1D quantize of an FFN-hidden-sized bf16 [8192, 14336]: amax + encode, "
                  "then encode alone (global scale given)",
    "w_quantize_2d": "2D quantize of W_up [14336, 3072]",
    "wgrad_x_quantize": "RHT16 + transposing quantize of X [8192, 14336] (a quarter of the "
                        "weight-gradient tokens)",
    "kv_quantize": "batched quantize + batched dequant of 4 KV tensors [24 * 32760, 128]",
    "ffn_gemm": "FFN up GEMM + GELU 8192x14336x3072 and down GEMM 8192x3072x14336",
    "wgrad_gemm": "weight-gradient GEMM 3072x14336x8192, fp32 out (a quarter of the tokens)",
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

    if name == "qkv_step":
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
    else:  # wgrad_gemm
        dy, xw, mask = synth.wgrad(dev, t=8192)
        qdy = nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1, ws=ws)
        qxw = nv.quantize_1d(xw, rht=True, mask=mask, block_axis=1, ws=ws)

        def run():
            nv.gemm(qdy, qxw, out_dtype=torch.float32, ws=ws)

    for _ in range(reps):
        run()
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0
    print("profile case %s: %s, %d reps" % (name, PROFILE_CASES[name], reps))
    return 0


# ------------------------------------------------------------------ GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--rows", default="auto", choices=["auto", "on", "off"],
                    help="also time every hot-path row at its full workload size "
                         "(auto: on a single GPU only)")
    ap.add_argument("--profile", default=None, choices=sorted(PROFILE_CASES),
                    help="run one small case a few times (untimed, no JSON line): the "
                         "program the ncu captures under profiles/ are taken on")
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
    x, w = synth.qkv_linear(dev)
    if rank:
        x = synth.activation(1 + 1000 * rank, 1, M, K, device=dev)
        w = synth.weight(1 + 1000 * rank, 2, N, K, device=dev)
    # the generator runs on torch's current stream, the path on `stream`
    torch.cuda.synchronize(dev)
    qa = nv.QTensor(*nv._alloc_q(M, K, nv.NVFP4_SF_TCGEN05, dev), M, K, nv.NVFP4_SF_TCGEN05)
    qb = nv.QTensor(*nv._alloc_q(N, K, nv.NVFP4_SF_TCGEN05, dev), N, K, nv.NVFP4_SF_TCGEN05)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws_a, ws_b, ws_g = nv.workspace(1, dev), nv.workspace(1, dev), nv.workspace(0, dev)
    ws_xw = nv.workspace(2, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer larger than L2 (evicts every input), then read another
        # one so the next kernel does not pay for writing back dirty lines
        flush.zero_()
        torch.sum(flush_rd, dim=0, out=flush_sink)

    def quant_xw():
        nv.quantize_mixed([x, w], [False, True], outs=[qa, qb], ws=ws_xw, stream=stream)

    def quant_x():
        nv.quantize_1d(x, out=qa, ws=ws_a, stream=stream)

    def quant_w():
        nv.quantize_2d(w, out=qb, ws=ws_b, stream=stream)

    def amax_x():
        nv.global_scale(x, out=qa.alpha, ws=ws_a, stream=stream)

    def pass2_x():
        nv.quantize_1d(x, out=qa, ws=ws_a, alpha_in=qa.alpha, stream=stream)

    def amax_w():
        nv.global_scale(w, out=qb.alpha, ws=ws_b, stream=stream)

    def pass2_w():
        nv.quantize_2d(w, out=qb, ws=ws_b, alpha_in=qb.alpha, stream=stream)

    def gemm():
        nv.gemm(qa, qb, out=y, ws=ws_g, stream=stream)

    def step():
        quant_xw()
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

    graphs = {"step": capture(step), "amax_x": capture(amax_x), "pass2_x": capture(pass2_x),
              "amax_w": capture(amax_w), "pass2_w": capture(pass2_w), "gemm": capture(gemm),
              "quant_x": capture(quant_x), "quant_w": capture(quant_w),
              "quant_xw": capture(quant_xw)}

    def timed(g, reps):
        """Mean device time (ms) of one graph replay, L2 flushed before each."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        with torch.cuda.stream(stream):
            torch.cuda._sleep(2_000_000)  # let the host run ahead of the device
            for s, e in evs:
                flush_l2()
                s.record(stream)
                g.replay()
                e.record(stream)
        stream.synchronize()
        return sum(s.elapsed_time(e) for s, e in evs) / reps

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graphs["step"].replay()
    stream.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)
    barrier(world)
    torch.cuda.synchronize(dev)
    step_ms = timed(graphs["step"], args.steps)
    torch.cuda.synchronize(dev)
    barrier(world)
    # per-kernel breakdown (same protocol)
    reps = max(20, min(args.steps, 200))
    part = {k: timed(graphs[k], reps)
            for k in ("amax_x", "pass2_x", "quant_x", "amax_w", "pass2_w", "quant_w", "quant_xw",
                      "gemm")}
    assert nv.device_error(ws_g, stream) == 0

    step_ms_max = reduce_max(step_ms, world, dev)
    flops = 2.0 * M * N * K
    value = world * flops / (step_ms_max * 1e-3) / 1e12

    fp4_peak = 4.0 * pk["bf16_tflops"]  # nominal FP4:BF16 dense ratio 9 : 2.25
    gemm_tflops = flops / (part["gemm"] * 1e-3) / 1e12
    hbm = pk["hbm_gbs"]

    def gbs(nbytes, ms):
        v = nbytes / (ms * 1e-3) / 1e9
        return {"ms": round(ms, 5), "GB/s": round(v, 1), "frac_hbm": round(v / hbm, 3)}

    q_out = 0.5 + 1.0 / 16  # bytes written per element (codes + scale bytes)
    breakdown = {
        "gemm": {"ms": round(part["gemm"], 5), "TFLOP/s": round(gemm_tflops, 1),
                 "frac_fp4_peak": round(gemm_tflops / fp4_peak, 3)},
        "quantize_xw_mixed": gbs((4 + q_out) * (M + N) * K, part["quant_xw"]),
        "quantize_x": gbs((4 + q_out) * M * K, part["quant_x"]),
        "quantize_w": gbs((4 + q_out) * N * K, part["quant_w"]),
        "amax_only_x": gbs(2 * M * K, part["amax_x"]),
        "encode_only_x": gbs((2 + q_out) * M * K, part["pass2_x"]),
        "amax_only_w": gbs(2 * N * K, part["amax_w"]),
        "encode_only_w": gbs((2 + q_out) * N * K, part["pass2_w"]),
        "note": "quantize_xw_mixed is the step's quantization: one amax and one encode launch "
                "for X (1D) and W (2D); quantize_x / quantize_w are the single-tensor calls "
                "(amax + encode each).  All counted at the algorithmic two-read bytes "
                "(4 + 0.5625 B/element); X (16 MB) and W (57 MB) fit in L2, so the second read is "
                "served from L2.  Each line is timed after an L2 flush.",
    }

    rows = None
    if args.rows == "on" or (args.rows == "auto" and world == 1):
        del graphs
        rows = measure_rows(nv, synth, torch, dev, stream, timed, pk, reps)
        graphs = None
    # clocks sampled over every timed region (step, breakdown, rows)
    clk = clocks.stop()

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(nv, torch, dev, stream, x, w, qa, qb, ws_xw, ws_g, args, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 scales, fp32 accumulate; fp32 encode)",
            "data": "synthetic (seeded splitmix64 generator, DiT QKV shapes)",
            "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K,
                       "parallelism": "replica per GPU (weak scaling)" if world > 1 else "single GPU",
                       "l2": "flushed before every timed step: 256 MiB write, then 256 MiB read",
                       "timing": "CUDA events around a CUDA-graph replay of the step, max over ranks"},
            "roofline": {"bound": "tensor", "achieved": round(gemm_tflops, 1),
                         "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                         "frac": round(gemm_tflops / fp4_peak, 4), "traffic": gemm_traffic(),
                         "kernel": "gemm_kernel (CTA-pair tcgen05.mma kind::mxf4nvf4)",
                         "peak_source": "%s bf16 burst %.1f TFLOP/s x 4 (nominal dense FP4:BF16 "
                                        "ratio)" % (pk["source"], pk["bf16_tflops"])},
            "breakdown": breakdown,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
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
    """Every hot-path row at its full workload size, same protocol as the step
    (graph replay between CUDA events, L2 flushed before each replay):

    a1 global amax, a3 1D quantize and a5 GEMMs on the DiT FFN pair (X
    [8192, 3072], W_up [14336, 3072], W_dn [3072, 14336], H [8192, 14336]);
    a4 2D quantize on both FFN weights; a2 RHT16 + transposing quantize and
    the fp32 GEMM of the weight-gradient path (dY [32768, 3072], X [32768,
    14336]); a6 batched quantize and a7 batched dequant of the 60-tensor KV
    cache (30 layers x {K, V} x [24 * 32760, 128]).  Bytes are the
    algorithmic ones: an input read by both passes counts twice."""
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
    g_dn = tc(lambda: nv.gemm(qh, qd, out=y, ws=ws, stream=stream), 2.0 * Mf * D * Hd)

    ws_h = nv.workspace(1, dev)

    def ffn_step():
        nv.quantize_1d(x, out=qx, ws=ws, stream=stream)
        # the up GEMM leaves H's amax in ws_h: H's quantization is one encode pass
        nv.gemm(qx, qu, out=h, epilogue=nv.NVFP4_EPI_GELU_TANH, amax_ws=ws_h, stream=stream)
        nv.quantize_1d(h, out=qh, ws=ws_h, amax_ready=True, stream=stream)
        nv.gemm(qh, qd, out=y, ws=ws, stream=stream)

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

    # ---------------- weight gradient
    dy, xw, mask = synth.wgrad(dev)
    torch.cuda.synchronize(dev)
    Tk, Do = dy.shape
    Di = xw.shape[1]
    qdy, qxw = q(Do, Tk), q(Di, Tk)
    dw = torch.empty((Do, Di), dtype=torch.float32, device=dev)
    out["a2_rht16_transposed_quantize"] = {
        "X_32768x14336": bw(lambda: nv.quantize_1d(xw, rht=True, mask=mask, block_axis=1,
                                                   out=qxw, ws=ws, stream=stream),
                            (4 + qout) * Tk * Di),
        "dY_32768x3072": bw(lambda: nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1,
                                                   out=qdy, ws=ws, stream=stream),
                            (4 + qout) * Tk * Do),
    }
    g_wg = tc(lambda: nv.gemm(qdy, qxw, out=dw, ws=ws, stream=stream), 2.0 * Do * Di * Tk)

    def wgrad_step():
        nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1, out=qdy, ws=ws, stream=stream)
        nv.quantize_1d(xw, rht=True, mask=mask, block_axis=1, out=qxw, ws=ws, stream=stream)
        nv.gemm(qdy, qxw, out=dw, ws=ws, stream=stream)

    wg = tc(wgrad_step, 2.0 * Do * Di * Tk)
    wg["note"] = "RHT16 + transposing quantize of dY and X, fp32 GEMM"
    out["a5_gemm"] = {"ffn_up_gelu_8192x14336x3072": g_up, "ffn_down_8192x3072x14336": g_dn,
                      "wgrad_3072x14336x32768_fp32": g_wg}
    out["steps"] = {"ffn_pair": ffn, "wgrad": wg}
    del dy, xw, qdy, qxw, dw

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
            and nv.device_error(ws_kv, stream) == 0)
    torch.cuda.empty_cache()
    return out


def measure_e2e(nv, torch, dev, stream, x, w, qa, qb, ws_xw, ws_g, args, world):
    """Same step through the public API with the inputs copied from pinned host
    memory and the bf16 result copied back, every step.  Steps are pipelined
    over three streams (inputs in, compute, result out; device buffers double
    buffered), so step i's host-to-device copies overlap step i-1's compute
    and step i-2's device-to-host copy; every step still moves all its bytes
    inside the timed region."""
    hx = x.cpu().pin_memory()
    hw = w.cpu().pin_memory()
    hy = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dx = [torch.empty_like(x) for _ in range(2)]
    dw = [torch.empty_like(w) for _ in range(2)]
    y = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
    ev_in, ev_used, ev_done, ev_out = ev(), ev(), ev(), ev()
    steps = max(3, min(args.steps, 50))

    def one(i):
        b = i % 2
        # inputs: wait until step i-2's compute has read buffer b
        if i >= 2:
            s_in.wait_event(ev_used[b])
        with torch.cuda.stream(s_in):
            dx[b].copy_(hx, non_blocking=True)
            dw[b].copy_(hw, non_blocking=True)
        ev_in[b].record(s_in)
        # compute: inputs landed, and step i-2's result has left y[b]
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])
        nv.quantize_mixed([dx[b], dw[b]], [False, True], outs=[qa, qb], ws=ws_xw, stream=stream)
        ev_used[b].record(stream)
        nv.gemm(qa, qb, out=y[b], ws=ws_g, stream=stream)
        ev_done[b].record(stream)
        # result out
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            hy[b].copy_(y[b], non_blocking=True)
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
    s, e = run(steps)
    torch.cuda.synchronize(dev)
    ms = reduce_max(s.elapsed_time(e) / steps, world, dev)
    return {"value": world * 2.0 * M * N * K / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": x.numel() * 2 + w.numel() * 2,
            "d2h_bytes_per_step": M * N * 2,
            "pipelined": "h2d / compute / d2h on three streams, device buffers double buffered"}


if __name__ == "__main__":
    sys.exit(main())
