"""Benchmark of the quantized attention hot path on B200.

One step = the whole path on one batch of the L=8704 FLUX.1 Kontext editing workload (512 text +
4096 target + 4096 context tokens, H=24, D=128, FP8 mode, outlier channels in Q and K):
calibrate+quantize of Q, K, V (one launch) -> fused attention, inputs resident in HBM.  Metric: algorithmic
FLOPs of BMM1 + BMM2 (4 * H * D * L^2) per second.  The L2 is flushed between steps (a
256 MiB write, then a 256 MiB read of another buffer, outside the timed events).  ``e2e`` repeats the measurement through the same C ABI
with the bf16 inputs in pinned host memory: every step copies Q, K, V to the device and the
output back.  ``--impl reference`` times the CPU oracle instead (rank 0 only) on a bounded row
sample of the same workload.  Extras in the same line (skipped by ``--no-extras``): the static
-scale quantize, FP4 mode on the same shape, the varlen FP4 batch, and the measured FP8 GEMM
rate next to the derived peak.  ``--gemm`` prints the line of the block's linear layers instead
(FP8 and FP4 GEMMs, the V projection with its fused E4M3 epilogue).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--mode fp8|fp4]
                    [--workload NAME] [--static-scales] [--no-extras] [--pair-kernel] [--gemm]
Multi-GPU (launched with torchrun): every rank runs its own replica of the workload (weak
scaling, no data-path collective); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0
FP8_PER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor throughput ratio on B200
FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 ratio (9 vs 2.25 PFLOP/s)
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes (read + write) of one launch of the attention kernel at L=8704 (B=1, H=24, D=128),
# from ncu on the current kernel:
#   ncu --set full --clock-control none -k regex:k_attn_fp8_fwd -s 3 -c 1 -o attn_fwd128 \
#       python bench.py --steps 1 --warmup 3 --no-cpu-baseline --no-e2e --no-extras
# (80.53 MB read + 26.77 MB written).  Set to None whenever the kernel changes, until captured
# again.  Other shapes of the same kernel: scaled by their algorithmic bytes (Q8 + K8 + V8 +
# bf16 output), and so marked.
ATTN_TRAFFIC_L8704 = 107305728
# the same for the pair-of-SMs variant (--pair-kernel): 80.30 MB read + 22.40 MB written
ATTN_TRAFFIC_L8704_PAIR = 102706432
ATTN_TRAFFIC_SOURCE = "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch, L=8704"
# DRAM bytes (read + write) of one Q, K, V quantize launch at L=8704 (B=1, H=24, D=128), from
#   ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum,lts__t_sector_hit_rate.pct \
#       --clock-control none -k regex:"k_quant_qkv|k_calib_quant_qkv" -s 3 -c 1 --csv --log-file q.csv \
#       python bench.py --steps 1 --warmup 3 --no-cpu-baseline --no-e2e --no-extras [--mode fp4] [--static-scales]
# keyed by (mode, static scales); None again whenever those kernels change.
QUANT_TRAFFIC_L8704 = {("fp8", False): 207469312, ("fp8", True): 202917120,
                       ("fp4", False): 262223104, ("fp4", True): 235917824}
ATTN_KERNEL = {128: "k_attn_fp8_fwd<128> (one SM per pair of Q tiles, persistent)",
               64: "k_attn_fp8_fwd<64>"}
ATTN_KERNEL_PAIR = "k_attn_fp8_pair (cluster of two CTAs per pair of Q tiles; opt-in variant)"


def attn_traffic(w, pair=False):
    """(bytes per launch, how it was obtained) for the attention kernel on workload w."""
    ref = ATTN_TRAFFIC_L8704_PAIR if pair else ATTN_TRAFFIC_L8704
    if ref is None or w.D != 128:
        return None, "not captured for this kernel"
    tokens = sum(w.seqlens) if w.varlen else w.B * w.L
    algo = tokens * w.H * w.D * (3 + 2)            # Q8, K8, V8 read; bf16 output written
    algo_ref = 8704 * 24 * 128 * (3 + 2)
    if not w.varlen and (w.L, w.H, w.B) == (8704, 24, 1):
        return ref, ATTN_TRAFFIC_SOURCE
    return ref * algo / algo_ref, (ATTN_TRAFFIC_SOURCE + ", scaled by this workload's algorithmic bytes")


def quant_traffic(w, static):
    """DRAM bytes of the quantize launch per the ncu capture, for the L=8704 shape only."""
    if w.varlen or (w.L, w.H, w.B, w.D) != (8704, 24, 1, 128):
        return None
    return QUANT_TRAFFIC_L8704.get((w.mode, bool(static)))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, BF16_FALLBACK_TFLOPS, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled through NVML every 5 ms
    by a background thread while the timed region runs (reading only; no setting is changed).
    The GPU is matched by PCI address, so CUDA_VISIBLE_DEVICES renumbering does not matter."""

    PERIOD_S = 0.005

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._thread = None

    def _handle(self, nv):
        props = torch.cuda.get_device_properties(self.cuda_index)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        try:
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:          # no NVML: the line says so
            self.error = f"nvml unavailable: {type(e).__name__}"
            return self
        self._stop = threading.Event()

        def run():
            while True:
                try:
                    self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                         nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception as e:
                    self.error = f"nvml query failed: {type(e).__name__}"
                    return
                if self._stop.wait(self.PERIOD_S):
                    return

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": [self.error or "no samples"]}
        import pynvml as nv
        names = {nv.nvmlClocksEventReasonHwSlowdown: "hw_slowdown",
                 nv.nvmlClocksEventReasonHwThermalSlowdown: "hw_thermal_slowdown",
                 nv.nvmlClocksEventReasonSwThermalSlowdown: "sw_thermal_slowdown",
                 nv.nvmlClocksEventReasonSwPowerCap: "sw_power_cap",
                 nv.nvmlClocksEventReasonHwPowerBrakeSlowdown: "hw_power_brake_slowdown"}
        reasons = sorted({nm for _, bits in self.samples for bit, nm in names.items() if bits & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "nvml every 5 ms during the timed steps"}


class L2Flush:
    """Leaves a cold, clean L2: writing a buffer larger than the L2 evicts every line; reading a
    second one then evicts those dirty lines, so their write-back does not land in the next
    timed step."""

    def __init__(self):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.max()


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value over the ranks (time is reported as the slowest rank's)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_workload(w, rank: int, world: int):
    """Weak scaling: every rank runs its own seeded problem of the same shape."""
    if world == 1:
        return w
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 100 * rank)


def run_gpu(args):
    import precision_quantized_attention_b200 as qa
    rank, world, local = dist_setup(args.gpus)
    if args.pair_kernel:
        qa._lib.debug_use_pair_kernel(True)
    w = workloads.WORKLOADS[args.workload or ("edit_fp8" if args.mode == "fp8" else "edit_fp4")]
    w = replica_workload(w, rank, world)
    q, k, v = workloads.make_qkv(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    static_amax = None
    if args.static_scales:                       # calibrate once, outside the timed region
        cal = qa.QuantizedAttention(w.shape, w.mode, cu_seqlens=w.cu_seqlens, sm_scale=w.sm_scale)
        cal.quantize(qd, kd, vd)
        static_amax = cal.amax.tolist()
        del cal
    path = qa.QuantizedAttention(w.shape, w.mode, cu_seqlens=w.cu_seqlens, sm_scale=w.sm_scale,
                                 static_amax=static_amax)
    flush = L2Flush()
    stream = torch.cuda.current_stream()

    def step():
        path.quantize(qd, kd, vd)
        return path.attend()

    for _ in range(args.warmup):
        step()
    status = qa.get_error()
    if status != 0:
        raise RuntimeError(f"device error {status} during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush()
            ev[i][0].record(stream)
            path.quantize(qd, kd, vd)
            ev[i][1].record(stream)
            path.attend()
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    quant_ms = [e[0].elapsed_time(e[1]) for e in ev]
    status = qa.get_error()
    if status != 0:
        raise RuntimeError(f"device error {status} during timing")
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world)
    attn = max_over_ranks(sum(attn_ms) / len(attn_ms), world)
    quant = max_over_ranks(sum(quant_ms) / len(quant_ms), world)

    if args.no_e2e:
        e2e_ms = float("nan")
    else:
        e2e_ms = e2e_time(args, w, q, k, v, qd, kd, vd, step, flush, stream, world)
    # our kernels per step: the Q, K, V calibrate+quantize launch, the attention launch, and the
    # combine launch when tail pairs are cut
    launches = 2 + (1 if path.attn_workspace is not None else 0)
    extra = {}
    if not args.no_extras:
        # the quantize launch with static scales (the amax just calibrated, as post-training
        # calibration would give): one streaming pass, no grid barrier
        if not args.static_scales:
            extra["quant_static_ms"] = time_quantize(w, qd, kd, vd, path.amax.tolist(), flush,
                                                     min(args.steps, 100))
        # FP4 mode on the same L=8704 shape, timed the same way in the same run
        if w.name == "edit_fp8" and world == 1:
            extra["fp4"] = run_mode_extra(workloads.WORKLOADS["edit_fp4"], flush, min(args.steps, 100),
                                          args.warmup)
            # the varlen batch of four packed sequences (FP4), the same way
            extra["varlen_fp4"] = run_mode_extra(workloads.WORKLOADS["varlen_fp4"], flush,
                                                 min(args.steps, 50), args.warmup)
        extra["fp8_measured"] = measured_fp8_rates(flush)
    report(args, w, (q, k, v), rank, world, ms, attn, quant, e2e_ms, clocks, launches, extra)
    barrier(world)
    del path
    if world > 1:
        torch.distributed.destroy_process_group()


def time_quantize(w, qd, kd, vd, amax, flush, steps):
    """Mean ms of the Q, K, V quantize launch with the given (static) amax values."""
    import precision_quantized_attention_b200 as qa
    sp = qa.QuantizedAttention(w.shape, w.mode, cu_seqlens=w.cu_seqlens, sm_scale=w.sm_scale,
                               static_amax=amax)
    for _ in range(3):
        sp.quantize(qd, kd, vd)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for e0, e1 in ev:
        flush()
        e0.record()
        sp.quantize(qd, kd, vd)
        e1.record()
    torch.cuda.synchronize()
    if qa.get_error() != 0:
        raise RuntimeError("device error in the static-scale quantize timing")
    return sum(e0.elapsed_time(e1) for e0, e1 in ev) / len(ev)


def run_mode_extra(w, flush, steps, warmup):
    """Step, attention and quantize (calibrated and static) times of workload w, timed like the
    main line (inputs resident, L2 flushed between steps, CUDA events)."""
    import precision_quantized_attention_b200 as qa
    q, k, v = workloads.make_qkv(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    path = qa.QuantizedAttention(w.shape, w.mode, cu_seqlens=w.cu_seqlens, sm_scale=w.sm_scale)
    for _ in range(warmup):
        path.quantize(qd, kd, vd)
        path.attend()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize()
    for e in ev:
        flush()
        e[0].record()
        path.quantize(qd, kd, vd)
        e[1].record()
        path.attend()
        e[2].record()
    torch.cuda.synchronize()
    if qa.get_error() != 0:
        raise RuntimeError(f"device error in the {w.name} timing")
    step = sum(e[0].elapsed_time(e[2]) for e in ev) / steps
    attn = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    quant = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    quant_static = time_quantize(w, qd, kd, vd, path.amax.tolist(), flush, steps)
    out = {"workload": w.name, "steps": steps, "step_ms": step, "attn_ms": attn,
           "quant_ms": quant, "quant_static_ms": quant_static, "flops": w.flops,
           "numel": q.numel(), "w": w}
    if w.mode == "fp4":
        out["fp4_direct"] = fp4_direct_estimate(qd, kd, vd, path.amax, flush, steps)
    return out


def fp4_direct_estimate(qd, kd, vd, amax, flush, steps):
    """What attention reading the packed E2M1 codes directly (instead of the FP8 requant codes)
    would save: the requant output's write in the quantize pass; the attention kernel itself is
    bound by its softmax, not by its 80 MB of code reads.  Times the per-tensor static FP4
    quantize of Q, K, V with and without the FP8 requant output."""
    import precision_quantized_attention_b200 as qa
    n = qd.numel()
    u8 = dict(dtype=torch.uint8, device="cuda")
    e2m1 = [torch.empty(n // 2, **u8) for _ in range(3)]
    bs = [torch.empty(n // 16, **u8) for _ in range(3)]
    c8 = [torch.empty(n, **u8) for _ in range(3)]
    gs = [torch.zeros(1, device="cuda") for _ in range(3)]
    s8 = [torch.zeros(1, device="cuda") for _ in range(3)]
    am = [amax[i:i + 1] for i in range(3)]

    def run(requant):
        for i, x in enumerate((qd, kd, vd)):
            qa.quantize_fp4_block(x, am[i], e2m1[i], bs[i], gs[i], c8[i] if requant else None,
                                  s8[i] if requant else None)

    times = {}
    for requant in (True, False):
        for _ in range(3):
            run(requant)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for e0, e1 in ev:
            flush()
            e0.record()
            run(requant)
            e1.record()
        torch.cuda.synchronize()
        times[requant] = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    if qa.get_error() != 0:
        raise RuntimeError("device error in the FP4-direct estimate")
    return {"quant_with_fp8_requant_ms": times[True], "quant_without_ms": times[False],
            "saving_ms": times[True] - times[False],
            "how": "per-tensor static FP4 quantize of Q, K, V with and without the FP8 requant "
                   "output (qattn_quantize_fp4_block); the attention kernel would read E2M1 + "
                   "block scales instead of E4M3 codes"}


def measured_fp8_rates(flush, reps=5):
    """Measured dense FP8 rates on this GPU beside the derived peak: this library's FP8 GEMM
    and torch._scaled_mm (cuBLASLt) on the block's QKV projection shape, L2 flushed."""
    import precision_quantized_attention_b200 as qa
    M, N, K = GEMM_SHAPES["qkv_proj"]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(3)
    a8 = torch.randint(0, 256, (M, K), dtype=torch.uint8, device="cuda", generator=gen)
    b8 = torch.randint(0, 256, (N, K), dtype=torch.uint8, device="cuda", generator=gen)
    a8 = torch.where((a8 & 0x7F) == 0x7F, a8 ^ 1, a8)
    b8 = torch.where((b8 & 0x7F) == 0x7F, b8 ^ 1, b8)
    sa, sb = torch.tensor([0.01], device="cuda"), torch.tensor([0.002], device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    out = {"shape": f"{M}x{N}x{K}"}

    def rate(fn):
        for _ in range(2):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for e0, e1 in ev:
            flush()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        ms = min(e0.elapsed_time(e1) for e0, e1 in ev)
        return 2.0 * M * N * K / (ms * 1e-3) / 1e12

    out["k_gemm_fp8_pair_tflops"] = rate(lambda: qa.gemm_fp8(a8, b8, y, sa, sb))
    if qa.get_error() != 0:
        raise RuntimeError("device error in the FP8 GEMM rate")
    try:
        af, bf = a8.view(torch.float8_e4m3fn), b8.view(torch.float8_e4m3fn)
        out["torch_scaled_mm_tflops"] = rate(
            lambda: torch._scaled_mm(af, bf.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16))
    except Exception as e:                       # not every torch build has it
        out["torch_scaled_mm_tflops"] = None
        out["torch_scaled_mm_error"] = type(e).__name__
    return out


def e2e_time(args, w, q, k, v, qd, kd, vd, step, flush, stream, world):
    """The whole path through the public API with the bf16 inputs in pinned host memory: every
    step copies its Q, K, V host->device, runs calibrate+quantize and attention, and copies the
    output back.  Steps are pipelined as a serving loop would run them: the host->device copies,
    the compute and the device->host copy of consecutive steps run on three streams over two
    sets of device buffers, so step i's upload overlaps step i-1's compute and download.  Timed
    with events from the first upload to the last download; no L2 flush is needed since every
    step writes 160 MB of fresh input (more than the L2) into HBM."""
    import precision_quantized_attention_b200 as qa
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    ohs = [torch.empty(w.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    paths = [qa.QuantizedAttention(w.shape, w.mode, cu_seqlens=w.cu_seqlens, sm_scale=w.sm_scale)
             for _ in range(2)]
    ins = [(qd, kd, vd), tuple(torch.empty_like(t) for t in (qd, kd, vd))]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n):
        ev = lambda: torch.cuda.Event(enable_timing=True)
        start, end = ev(), ev()
        quant_done, comp_done, down_done = [None] * n, [None] * n, [None] * n
        start.record(h2d)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(h2d):
                if i >= 2:
                    h2d.wait_event(quant_done[i - 2])      # slot b's inputs are consumed
                for dst, src in zip(ins[b], (qh, kh, vh)):
                    dst.copy_(src, non_blocking=True)
                up = ev()
                up.record(h2d)
            stream.wait_event(up)
            if i >= 2:
                stream.wait_event(down_done[i - 2])       # slot b's output was downloaded
            paths[b].quantize(*ins[b], stream)
            quant_done[i] = ev()
            quant_done[i].record(stream)
            paths[b].attend(stream)
            comp_done[i] = ev()
            comp_done[i].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(comp_done[i])
                ohs[b].copy_(paths[b].out, non_blocking=True)
                down_done[i] = ev()
                down_done[i].record(d2h)
        end.record(d2h)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n

    run(max(2, args.warmup))
    barrier(world)
    ms = run(args.steps)
    status = qa.get_error()
    if status != 0:
        raise RuntimeError(f"device error {status} in the end-to-end run")
    barrier(world)
    return max_over_ranks(ms, world)


def workload_data(w) -> str:
    """How the synthetic inputs were made (same recipe as the tests)."""
    parts = ["synthetic: seeded N(0,1) bf16 Q/K/V"]
    if w.text_scale != 1.0:
        parts.append(f"text rows x{w.text_scale:g}")
    if w.outliers:
        parts.append(f"{w.outliers} of {w.D} Q/K channels per head x{w.outlier_scale:g}")
    if w.varlen:
        parts.append("packed sequences " + "+".join(str(x) for x in w.seqlens))
    return ", ".join(parts)


def bench_config(w, world, static_scales=False):
    """The workload description both arms print."""
    return {"workload": f"{w.name}: B={w.B} H={w.H} L={w.L} D={w.D} {w.mode.upper()} full attention"
                        + (" (512 text + 4096 target + 4096 context tokens)"
                           if w.L == workloads.L_EDIT else ""),
            "mode": w.mode, "B": w.B, "H": w.H, "L": w.L, "D": w.D,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "scales": ("static: Q, K, V amax calibrated once before the timed steps"
                       if static_scales else "calibrated every step (amax of Q, K and V)"),
            "l2": "flushed between steps outside the timed events: a 256 MiB write, then a "
                  "256 MiB read of another buffer so the write's dirty lines are written back "
                  "before the step starts"}


def quantize_bytes(w, numel):
    """Algorithmic bytes of the Q, K, V quantize launch: bf16 read once (2 B), E4M3 codes
    written (1 B); FP4 mode also writes the packed E2M1 codes (0.5 B) and one block-scale byte
    per 16 elements."""
    per_elem = 3.0 if w.mode == "fp8" else 3.0 + 0.5 + 1.0 / 16
    return 3 * numel * per_elem


def report(args, w, qkv, rank, world, ms, attn, quant, e2e_ms, clocks, launches, extra=None):
    q = qkv[0]
    hbm_gbs, bf16_tf, peak_kind = load_peaks()
    fp8_peak = bf16_tf * FP8_PER_BF16
    flops = w.flops
    achieved_tf = flops / (attn * 1e-3) / 1e12
    extra = extra or {}
    in_bytes = 3 * q.numel() * 2
    quant_bytes = quantize_bytes(w, q.numel())
    pair = bool(getattr(args, "pair_kernel", False)) and w.D == 128
    kname = ATTN_KERNEL_PAIR if pair else ATTN_KERNEL[w.D]
    traffic, traffic_src = attn_traffic(w, pair)
    clock = clocks.summary()
    quantize = {"ms": quant, "algorithmic_bytes": quant_bytes,
                "gbs": quant_bytes / (quant * 1e-3) / 1e9,
                "frac_hbm": quant_bytes / (quant * 1e-3) / 1e9 / hbm_gbs,
                "hbm_peak_gbs": hbm_gbs, "launches": 1,
                "traffic": quant_traffic(w, args.static_scales),
                "path": ("static scales (qattn_quantize_qkv, one pass)" if args.static_scales
                         else "calibrated every step (qattn_calibrate_quantize_qkv: amax, grid "
                              "barrier, quantize)")}
    if "quant_static_ms" in extra:
        qs = extra["quant_static_ms"]
        quantize["static"] = {"ms": qs, "gbs": quant_bytes / (qs * 1e-3) / 1e9,
                              "frac_hbm": quant_bytes / (qs * 1e-3) / 1e9 / hbm_gbs,
                              "traffic": quant_traffic(w, True),
                              "path": "static scales (qattn_quantize_qkv, one pass), the amax "
                                      "calibrated in the timed steps"}
    def mode_block(x):
        """The JSON block of a workload timed by run_mode_extra."""
        w4 = x.pop("w")
        qb4 = quantize_bytes(w4, x["numel"])
        t4, t4_src = attn_traffic(w4, pair)
        a_tf = x["flops"] / (x["attn_ms"] * 1e-3) / 1e12
        return {"workload": bench_config(w4, world)["workload"], "steps": x["steps"],
                "ms_per_step": x["step_ms"], "value": x["flops"] / (x["step_ms"] * 1e-3) / 1e12,
                "roofline": {"bound": "tensor", "achieved": a_tf, "peak": fp8_peak,
                             "unit": "TFLOP/s", "frac": a_tf / fp8_peak, "traffic": t4,
                             "traffic_source": t4_src, "kernel_ms": x["attn_ms"],
                             "kernel": kname},
                "quantize": {"ms": x["quant_ms"], "algorithmic_bytes": qb4,
                             "frac_hbm": qb4 / (x["quant_ms"] * 1e-3) / 1e9 / hbm_gbs,
                             "traffic": quant_traffic(w4, False),
                             "static": {"ms": x["quant_static_ms"],
                                        "frac_hbm": qb4 / (x["quant_static_ms"] * 1e-3) / 1e9 / hbm_gbs,
                                        "traffic": quant_traffic(w4, True)}},
                "fp4_direct_estimate": x.get("fp4_direct")}

    fp4 = mode_block(extra["fp4"]) if "fp4" in extra else None
    varlen = mode_block(extra["varlen_fp4"]) if "varlen_fp4" in extra else None
    result = {
        "metric": "quantized attention TFLOP/s @L=8704,H=24,D=128 and % of B200 FP8 peak",
        "value": world * flops / (ms * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": workload_data(w),
        "config": bench_config(w, world, args.static_scales),
        "roofline": {"bound": "tensor", "achieved": achieved_tf, "peak": fp8_peak,
                     "unit": "TFLOP/s", "frac": achieved_tf / fp8_peak,
                     "traffic": traffic, "traffic_source": traffic_src,
                     "kernel": kname,
                     "peak_source": f"{peak_kind} bf16 burst {bf16_tf} TFLOP/s x {FP8_PER_BF16} "
                                    "(nominal FP8/BF16 ratio)",
                     "fp8_measured_tflops": extra.get("fp8_measured"),
                     "kernel_ms": attn},
        "quantize": quantize,
        "fp4": fp4,
        "varlen_fp4": varlen,
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": q.numel() * 2,
                "schedule": "pinned host bf16 Q/K/V -> device, "
                            + ("quantize with the static scales" if args.static_scales
                               else "fused calibrate+quantize")
                            + ", attention, bf16 output -> host every step; uploads, compute and "
                            "downloads on three streams over two buffer sets, so consecutive "
                            "steps overlap"},
        "gpu_launches": world * launches * args.steps,   # all ranks' launches in the timed steps
        "clocks": clock,
    }
    if rank == 0:
        # the oracle is timed on the host cores at N=1 only
        run_cpu = world == 1 and not args.no_cpu_baseline
        result["cpu_baseline"] = cpu_baseline(w, qkv=qkv) if run_cpu else None
        print(json.dumps(result), flush=True)


def cpu_baseline(w, rows_per_head: int = 1024, seed: int = 0, qkv=None):
    """The oracle as it stands, on the host cores: quantize all of Q, K, V, then attention for
    a seeded sample of `rows_per_head` query rows of every head; throughput counts the sampled
    rows' BMM1 + BMM2 FLOPs only (the full-tensor quantization is charged to the sample).
    Input generation is outside the timed region."""
    import oracle
    q, k, v = qkv if qkv is not None else workloads.make_qkv(w)
    g = torch.Generator().manual_seed(seed)
    rows = []
    for h in range(w.H):
        pick = torch.randperm(w.L, generator=g)[:rows_per_head]
        rows.extend((h * w.L + pick).tolist())
    rows = sorted(rows)
    t0 = time.perf_counter()
    oracle.method_forward(q, k, v, w.mode, sm_scale=w.sm_scale, rows=rows)
    dt = time.perf_counter() - t0
    flops = 4.0 * w.D * w.L * len(rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": dt,
            "sample": f"{rows_per_head} of {w.L} query rows per head x {w.H} heads "
                      f"({len(rows)} rows, {flops:.3e} FLOP) of {w.name}, plus amax+quantize "
                      "of the full Q, K, V"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = workloads.WORKLOADS[args.workload or ("edit_fp8" if args.mode == "fp8" else "edit_fp4")]
    qkv = workloads.make_qkv(w)
    for _ in range(args.warmup):
        cpu_baseline(w, rows_per_head=8, qkv=qkv)
    times, flops = [], 0.0
    for i in range(args.steps):
        r = cpu_baseline(w, rows_per_head=256, seed=i + 1, qkv=qkv)
        times.append(r["seconds"])
        flops = r["value"] * r["seconds"] * 1e12
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    cores = r["cores"]
    print(json.dumps({
        "impl": "reference",
        "metric": "quantized attention TFLOP/s @L=8704,H=24,D=128 and % of B200 FP8 peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": workload_data(w),
        "config": bench_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


# The transformer block's FP8 linear layers on the joint sequence (M = 512 + 4096 + 4096 tokens,
# hidden 3072): the QKV and output projections and the two MLP GEMMs.
GEMM_SHAPES = {"qkv_proj": (8704, 9216, 3072), "out_proj": (8704, 3072, 3072),
               "mlp_up": (8704, 12288, 3072), "mlp_down": (8704, 3072, 12288)}


def run_gemm(args):
    """FP8 GEMM (qattn_gemm_fp8) on the block's linear-layer shapes: seeded random E4M3 codes
    (every finite code, both signs), each launch after an L2 flush, CUDA events around each
    launch; value = all shapes' FLOPs over their summed time."""
    import oracle
    import precision_quantized_attention_b200 as qa
    torch.cuda.set_device(0)
    _, bf16_tf, peak_kind = load_peaks()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    flush = L2Flush()
    per_shape, total_flops, total_ms, cpu = {}, 0.0, 0.0, None

    def codes(rows, cols):
        c = torch.randint(0, 256, (rows, cols), dtype=torch.uint8, device="cuda", generator=gen)
        return torch.where((c & 0x7F) == 0x7F, c ^ 1, c)      # no NaN codes

    with ClockSampler(0) as clocks:
        for name, (M, N, K) in GEMM_SHAPES.items():
            a8, b8 = codes(M, K), codes(N, K)
            sa = torch.tensor([0.01], device="cuda")
            sb = torch.tensor([0.002], device="cuda")
            y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            for _ in range(args.warmup):
                qa.gemm_fp8(a8, b8, y, sa, sb)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            torch.cuda.synchronize()
            for e0, e1 in ev:
                flush()
                e0.record()
                qa.gemm_fp8(a8, b8, y, sa, sb)
                e1.record()
            torch.cuda.synchronize()
            if qa.get_error() != 0:
                raise RuntimeError("device error during the GEMM timing")
            ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / len(ev)
            flops = 2.0 * M * N * K
            per_shape[name] = {"M": M, "N": N, "K": K, "ms": ms,
                               "tflops": flops / (ms * 1e-3) / 1e12}
            total_flops += flops
            total_ms += ms
            if cpu is None and not args.no_cpu_baseline:
                rows = list(range(0, M, M // 16))[:16]       # the oracle on 16 rows
                a_rows, b_all = a8[rows].cpu().numpy(), b8.cpu().numpy()
                t0 = time.perf_counter()
                oracle.gemm_e4m3(a_rows, b_all, 0.01, 0.002)
                dt = time.perf_counter() - t0
                cpu = {"value": 2.0 * len(rows) * N * K / dt / 1e12, "unit": "TFLOP/s",
                       "cores": os.cpu_count(), "kind": "oracle", "seconds": dt,
                       "sample": f"16 of {M} rows of {name} (numpy FP64 matmul)"}
    value = total_flops / (total_ms * 1e-3) / 1e12
    fused = v_projection_fused(flush, args.steps)
    fp4 = fp4_gemm_rates(flush, args.steps, args.warmup)
    # the burst GEMM figure, unless the power cap held the clock down during the timed launches:
    # then the figure measured over a seconds-long loop under the cap (when the peaks file has it)
    clk = clocks.summary()
    if "sw_power_cap" in (clk or {}).get("reasons", []):
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                bf16_tf = float(json.load(f)["bf16_tflops_sustained"])
                peak_kind = "measured sustained (sw_power_cap seen while timing)"
        except Exception:
            pass
    fp8_peak = bf16_tf * FP8_PER_BF16
    for rec in per_shape.values():
        rec["frac"] = rec["tflops"] / fp8_peak
    fp4_peak = bf16_tf * FP4_PER_BF16
    for rec in fp4["per_shape"].values():
        rec["frac"] = rec["tflops"] / fp4_peak
    fp4["peak"] = fp4_peak
    fp4["peak_source"] = f"{peak_kind} bf16 {bf16_tf} TFLOP/s x {FP4_PER_BF16} (nominal FP4/BF16 ratio)"
    fp4["frac"] = fp4["value"] / fp4_peak
    print(json.dumps({
        "metric": "FP8 GEMM TFLOP/s on the FLUX.1 Kontext block's linear layers "
                  "(QKV and output projections, MLP; 8704 tokens, hidden 3072)",
        "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic: seeded random E4M3 codes, per-tensor multipliers 0.01 and 0.002",
        "config": {"workload": "qkv_proj 8704x9216x3072, out_proj 8704x3072x3072, "
                               "mlp_up 8704x12288x3072, mlp_down 8704x3072x12288 (M x N x K)",
                   "l2": "flushed before every launch, outside the timed events"},
        "roofline": {"bound": "tensor", "achieved": value, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": value / fp8_peak, "traffic": None, "kernel": "k_gemm_fp8_pair",
                     "peak_source": f"{peak_kind} bf16 {bf16_tf} TFLOP/s x {FP8_PER_BF16} "
                                    "(nominal FP8/BF16 ratio)", "per_shape": per_shape},
        "v_projection_fused_quantize": fused,
        "fp4": fp4,
        "gpu_launches": len(GEMM_SHAPES) * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu,
    }), flush=True)


def fp4_gemm_rates(flush, steps, warmup):
    """The per-block FP4 GEMM (qattn_gemm_fp4) on the same shapes: seeded random packed E2M1
    codes and E4M3 block scales, timed like the FP8 launches."""
    import precision_quantized_attention_b200 as qa
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9)
    per_shape, flops_sum, ms_sum = {}, 0.0, 0.0
    for name, (M, N, K) in GEMM_SHAPES.items():
        xp = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device="cuda", generator=gen)
        wp = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device="cuda", generator=gen)
        xb = torch.randint(0, 0x7F, (M, K // 16), dtype=torch.uint8, device="cuda", generator=gen)
        wb = torch.randint(0, 0x7F, (N, K // 16), dtype=torch.uint8, device="cuda", generator=gen)
        sx, sw = torch.tensor([0.01], device="cuda"), torch.tensor([0.002], device="cuda")
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        for _ in range(warmup):
            qa.gemm_fp4(xp, xb, sx, wp, wb, sw, y)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        torch.cuda.synchronize()
        for e0, e1 in ev:
            flush()
            e0.record()
            qa.gemm_fp4(xp, xb, sx, wp, wb, sw, y)
            e1.record()
        torch.cuda.synchronize()
        if qa.get_error() != 0:
            raise RuntimeError("device error during the FP4 GEMM timing")
        ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / len(ev)
        flops = 2.0 * M * N * K
        per_shape[name] = {"M": M, "N": N, "K": K, "ms": ms, "tflops": flops / (ms * 1e-3) / 1e12}
        flops_sum += flops
        ms_sum += ms
    return {"kernel": "k_gemm_fp4_pair (kind::mxf4nvf4, 256 x 192 tiles on pairs of SMs; "
                      "k_gemm_fp4 for M <= 128)",
            "value": flops_sum / (ms_sum * 1e-3) / 1e12, "unit": "TFLOP/s", "ms": ms_sum,
            "per_shape": per_shape, "gpu_launches": len(GEMM_SHAPES) * steps}


def v_projection_fused(flush, steps):
    """The value projection (8704 tokens, 3072 -> 3072) feeding the attention's V codes, with
    static scales: the GEMM's bf16 output then a separate quantize launch, against the GEMM with
    the quantize fused into its epilogue (qattn_gemm_fp8_e4m3, codes only)."""
    import precision_quantized_attention_b200 as qa
    M, N, K = GEMM_SHAPES["out_proj"]               # same shape as the value projection
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    a8 = torch.randint(0, 256, (M, K), dtype=torch.uint8, device="cuda", generator=gen)
    b8 = torch.randint(0, 256, (N, K), dtype=torch.uint8, device="cuda", generator=gen)
    a8 = torch.where((a8 & 0x7F) == 0x7F, a8 ^ 1, a8)
    b8 = torch.where((b8 & 0x7F) == 0x7F, b8 ^ 1, b8)
    sa, sb = torch.tensor([0.01], device="cuda"), torch.tensor([0.002], device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    codes = torch.empty(M, N, dtype=torch.uint8, device="cuda")
    scale = torch.zeros(1, device="cuda")
    qa.gemm_fp8(a8, b8, y, sa, sb)
    amax = y.float().abs().max().reshape(1)          # the static calibration

    def separate():
        qa.gemm_fp8(a8, b8, y, sa, sb)
        qa.quantize_fp8(y.reshape(-1), amax, codes.reshape(-1), scale)

    def fused_call():
        qa.gemm_fp8_e4m3(a8, b8, codes, sa, sb, amax, scale)

    def ms(fn):
        for _ in range(3):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for e0, e1 in ev:
            flush()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps

    t_sep, t_fused = ms(separate), ms(fused_call)
    if qa.get_error() != 0:
        raise RuntimeError("device error in the fused value-projection timing")
    return {"shape": f"{M}x{N}x{K}", "gemm_then_quantize_ms": t_sep, "fused_ms": t_fused,
            "saved_ms": t_sep - t_fused,
            "how": "static amax; separate = qattn_gemm_fp8 (bf16 out) + qattn_quantize_fp8; fused = "
                   "qattn_gemm_fp8_e4m3 (codes only)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--mode", default="fp8", choices=["fp8", "fp4"])
    ap.add_argument("--workload", default=None, choices=sorted(workloads.WORKLOADS),
                    help="time another dense workload (default: the L=8704 editing workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--static-scales", action="store_true",
                    help="quantize with amax values calibrated once before timing (one pass)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the static-scale quantize, FP4-mode and measured FP8 rate timings")
    ap.add_argument("--pair-kernel", action="store_true",
                    help="D = 128 attention on the pair-of-SMs variant (k_attn_fp8_pair)")
    ap.add_argument("--gemm", action="store_true",
                    help="time the FP8 GEMM of the transformer block's linear layers instead")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.gemm:
        run_gemm(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
