"""Benchmark of the RFQ MXFP4 W4A4 linear layer on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path on the video-DiT FFN workload, the
largest of the benchmark's workloads (X bf16 32768 x 5120, Laplace body with 8
outlier channels; W bf16 13824 x 5120; Y bf16):
  1. rfq_quantize_weight   W -> Q(W)                       (kernel 1, no residual)
  2. rfq_quantize_mxfp4    X -> Q(X), Q(R), R = X - DQ(Q(X)) (kernel 1, fused)
  3. rfq_gemm              Y = DQ(QX) DQ(QW)^T + DQ(QR) DQ(QW)^T (kernel 2, tcgen05)
Inputs are resident in HBM; L2 is flushed between timed steps (a 256 MiB buffer
is written, then read back so L2 is left clean), outside the per-step CUDA events.
``value`` is executed MMA TFLOP/s over the whole step (4*M*N*K per step: the
residual doubles K on the tensor pipe).  The same line carries, as extra keys, the
LLM FFN up-projection step (4096 x 4096 -> 12288), the quantize-only bandwidth
workload (8192 x 4096), the GEMM with the residual off (plain MXFP4), the
rfq_linear M sweep (M = 16 .. 16384, K = N = 4096), the activation and output
fidelity of RFQ against plain MXFP4 and MXFP8, the training-side GEMMs and the
MXFP8 comparator on the FFN shape, the tensor-core rate of the GEMM's own MMA
shapes measured by the library's probe, and a library comparator: cuBLASLt's MXFP4
GEMM (through torch) on the DiT step's own quantized operands, plain and with RFQ
written as one GEMM over the operands concatenated along K.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs under torchrun: every rank runs its own replica of the step (the
layer has no exchange step; weak scaling), time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
FP4_OVER_BF16 = 9.0 / 2.25          # nominal dense MXFP4 : bf16 tensor throughput on B200
# DRAM bytes (read + write) per launch from ncu captures of the current kernels (the
# GEMM on the FFN and DiT workloads; the quantizer on 16384 x 4096, twice the
# bench workload's units, scaled by 1/2; summaries under profiles/).  None until
# captured, and again once a kernel changes.
NCU_TRAFFIC_BYTES = {"gemm_ffn_rfq_bf16": 46.665472e6 + 53.230336e6, "gemm_dit_rfq_bf16": 470.674176e6 + 872.390656e6,
                     "quantize_8192x4096_rfq": (134.430976e6 + 39.872512e6) / 2}
L2_FLUSH_BYTES = 256 << 20
REFERENCE_RUN_SECONDS = 150.0   # host time of a whole --impl reference run


def make_l2_flush(torch):
    """Flush L2 between timed launches: write a 256 MiB buffer (twice L2), then read it
    back so that L2 holds clean lines and the next timed kernel pays no write-back of
    the flush itself."""
    buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    words = buf.view(torch.int64)

    def flush():
        buf.zero_()
        words.sum()
    return flush


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz, self.power_w = [], set(), None, []
        self.handle_by = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = self._handle(pynvml, device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _handle(self, pynvml, device_index):
        # NVML enumerates every GPU of the machine; find the one torch uses by UUID
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.handle_by = "uuid"
            return h
        except Exception:
            self.handle_by = "index"
            return pynvml.nvmlDeviceGetHandleByIndex(device_index)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM))
                self.power_w.append(self._nvml.nvmlDeviceGetPowerUsage(self._h) / 1000.0)
                r = self._nvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nvml:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nvml:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "power_w_median": statistics.median(self.power_w) if self.power_w else None,
                "power_w_max": max(self.power_w) if self.power_w else None, "nvml_device_by": self.handle_by}


# ----------------------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        return dist.get_rank(), world, local
    return 0, 1, 0


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    from block_scaled_gemm_rfq_b200.sharding import max_over_ranks as _max
    return _max(v) if world > 1 else v


# ----------------------------------------------------------------------------- the CUDA path
def to_device_bf16(bits):
    import numpy as np
    import torch
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


class RfqStep:
    """Buffers and launches of one step (all through the C ABI binding)."""

    def __init__(self, rfq, x, w, residual=True, out_dtype=None):
        import torch
        self.rfq, self.x, self.w, self.residual = rfq, x, w, residual
        self.M, self.K = x.shape
        self.N = w.shape[0]
        dev = x.device
        u8 = lambda n: torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
        self.qw_c, self.qw_s = u8(rfq.codes_bytes(self.N, self.K)), u8(rfq.scales_bytes(self.N, self.K))
        self.qx_c, self.qx_s = u8(rfq.codes_bytes(self.M, self.K)), u8(rfq.scales_bytes(self.M, self.K))
        self.qr_c = u8(rfq.codes_bytes(self.M, self.K)) if residual else None
        self.qr_s = u8(rfq.scales_bytes(self.M, self.K)) if residual else None
        self.y = torch.empty((self.M, self.N), dtype=out_dtype or torch.bfloat16, device=dev)

    def quantize_w(self):
        self.rfq.quantize_weight(self.w, self.qw_c, self.qw_s)

    def quantize_x(self):
        self.rfq.quantize_mxfp4(self.x, self.qx_c, self.qx_s, self.qr_c, self.qr_s)

    def gemm(self):
        self.rfq.gemm(self.qx_c, self.qx_s, self.qr_c, self.qr_s, self.qw_c, self.qw_s, self.M, self.N, self.K,
                      self.y)

    def run(self):
        self.quantize_w()
        self.quantize_x()
        self.gemm()


def time_phases(step: RfqStep, steps: int, warmup: int, flush, world: int):
    """Per-step CUDA events around each kernel; L2 flushed between steps."""
    import torch
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        flush()
        e = ev[i]
        e[0].record()
        step.quantize_w()
        e[1].record()
        step.quantize_x()
        e[2].record()
        step.gemm()
        e[3].record()
    torch.cuda.synchronize()
    barrier(world)
    qw = [e[0].elapsed_time(e[1]) for e in ev]
    qx = [e[1].elapsed_time(e[2]) for e in ev]
    gm = [e[2].elapsed_time(e[3]) for e in ev]
    tot = [e[0].elapsed_time(e[3]) for e in ev]
    return {"quantize_w_ms": qw, "quantize_x_ms": qx, "gemm_ms": gm, "step_ms": tot}


def time_kernel(fn, iters, flush):
    import torch
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    out = []
    for _ in range(iters):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        out.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in out]


def time_stream(fns, reps):
    """Per-call ms of back-to-back calls, replayed from a CUDA graph so that host
    launch overhead is out of the figure: fns[i] use distinct buffers whose total
    is larger than L2, so every call reads its operands from HBM.  One pass over
    all fns is captured; the graph is replayed 3 times untimed, then reps times
    between one event pair."""
    import torch
    for f in fns:   # eager warm-up (first-call setup happens outside the capture)
        f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / (reps * len(fns))


def time_training(rfq, wk, flush, fp4_peak, hbm_peak):
    """Backward pass of the FFN layer (straight-through): the transposed quantizer on
    X and dY, dgrad (dX = dY . W, contraction over N) and wgrad (dW = dY^T . X,
    contraction over the M tokens), each GEMM timed alone after an L2 flush."""
    import numpy as np
    import torch
    M, K, N = wk.M, wk.K, wk.N
    x = to_device_bf16(wk.x_bits)
    w = to_device_bf16(wk.w_bits)
    dy = torch.randn((M, N), device="cuda", generator=torch.Generator("cuda").manual_seed(5)).mul_(1e-3)
    dy = dy.to(torch.bfloat16)
    out = {}
    # transposed quantizers
    qxt = rfq.quantize_mxfp4_t_alloc(x, residual=True)
    t = time_kernel(lambda: rfq.quantize_mxfp4_t(x, qxt.codes, qxt.scales, qxt.r_codes, qxt.r_scales), 20, flush)
    out["quantize_t_x"] = {"shape": [M, K], "us": 1e3 * statistics.mean(t),
                           "gbs": quantize_bytes(M, K, True) / (statistics.mean(t) * 1e-3) / 1e9}
    out["quantize_t_x"]["frac_hbm"] = out["quantize_t_x"]["gbs"] / hbm_peak
    qdyt = rfq.quantize_mxfp4_t_alloc(dy, residual=False)
    t = time_kernel(lambda: rfq.quantize_mxfp4_t(dy, qdyt.codes, qdyt.scales), 20, flush)
    out["quantize_t_dy"] = {"shape": [M, N], "us": 1e3 * statistics.mean(t),
                            "gbs": quantize_bytes(M, N, False) / (statistics.mean(t) * 1e-3) / 1e9}
    # dgrad: A = Q(dY) [M][N] (+ residual), B = Q(W^T) [K][N] -> dX [M][K]
    qdy = rfq.quantize_mxfp4_alloc(dy, residual=True)
    qwt = rfq.quantize_mxfp4_t_alloc(w, residual=False)
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    t = time_kernel(lambda: rfq.gemm(qdy.codes, qdy.scales, qdy.r_codes, qdy.r_scales, qwt.codes, qwt.scales,
                                     M, K, N, dx), 10, flush)
    f = 4.0 * M * N * K
    out["dgrad_gemm"] = {"us": 1e3 * statistics.mean(t), "tflops_executed": f / (statistics.mean(t) * 1e-3) / 1e12}
    out["dgrad_gemm"]["frac_fp4_peak"] = out["dgrad_gemm"]["tflops_executed"] / fp4_peak
    # wgrad: A = Q(X^T) [K][M] (+ residual), B = Q(dY^T) [N][M] -> dW [N][K] (transposed store)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    t = time_kernel(lambda: rfq.gemm_yt(qxt.codes, qxt.scales, qxt.r_codes, qxt.r_scales, qdyt.codes, qdyt.scales,
                                        K, N, M, dw), 10, flush)
    out["wgrad_gemm"] = {"us": 1e3 * statistics.mean(t), "tflops_executed": f / (statistics.mean(t) * 1e-3) / 1e12}
    out["wgrad_gemm"]["frac_fp4_peak"] = out["wgrad_gemm"]["tflops_executed"] / fp4_peak
    rfq.check_device_error()
    return out


def time_mxfp8(rfq, wk, flush, fp8_peak, hbm_peak, step):
    """The MXFP8 comparator on the FFN workload: quantizer (X, 2 B in + 1 + 1/32 B out
    per element) and GEMM (2 M N K flops at the FP8 rate, half the FP4 rate), beside
    the RFQ GEMM (4 M N K at the FP4 rate: the same tensor-pipe time in theory)."""
    import torch
    M, K, N = wk.M, wk.K, wk.N
    x, w = step.x, step.w
    qa = rfq.quantize_mxfp8_alloc(x)
    qw = rfq.quantize_mxfp8_alloc(w)
    t = time_kernel(lambda: rfq.quantize_mxfp8(x, qa.codes, qa.scales), 20, flush)
    qbytes = M * K * 2 + M * K + M * K // 32
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    tg = time_kernel(lambda: rfq.gemm_mxfp8(qa.codes, qa.scales, qw.codes, qw.scales, M, N, K, y), 20, flush)
    rfq.check_device_error()
    f = 2.0 * M * N * K
    g_ms = statistics.mean(tg)
    return {"quantize_x": {"us": 1e3 * statistics.mean(t), "gbs": qbytes / (statistics.mean(t) * 1e-3) / 1e9},
            "gemm": {"us": 1e3 * g_ms, "tflops": f / (g_ms * 1e-3) / 1e12,
                     "frac_fp8_peak": f / (g_ms * 1e-3) / 1e12 / fp8_peak,
                     "peak_basis": "half the MXFP4 peak (the probe's kind::mxf8f6f4 rate per clock is half "
                                   "of kind::mxf4's)"}}


def quantize_bytes(M, K, residual):
    """Algorithmic HBM bytes of the fused quantizer: read X once (2 B/elem), write codes
    (0.5 B/elem) and scales (1 B per 32 elements) per output."""
    outs = 2 if residual else 1
    return M * K * 2 + outs * (M * K // 2 + M * K // 32)


def measure_mma_peak(rfq, local, iters=50000, launches=5):
    """The tensor-core rate of the GEMM's own MMA shapes, operands resident in shared
    memory (rfq_mma_rate_probe): CUDA events around each launch, the SM clock sampled
    meanwhile, and the rate per SM clock from the kernel's clock64 span."""
    import torch
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
    out = {}
    for variant, name, pair in ((0, "mxf4_pair", 2), (1, "mxf4_single", 1), (2, "mxf8_pair", 2)):
        rfq.mma_rate_probe(variant, 1000, cycles)
        torch.cuda.synchronize()
        used = 0
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
        with ClockSampler(local, period_s=0.005) as clk:
            for a, b in ev:
                a.record()
                flops, used = rfq.mma_rate_probe(variant, iters, cycles)
                b.record()
            torch.cuda.synchronize()
        rfq.check_device_error()
        ms = [a.elapsed_time(b) for a, b in ev]
        clusters = used // pair
        span = int(cycles[:clusters].max().item())
        per_clk = flops / used / span          # flops per SM per SM-clock cycle
        c = clk.summary()
        out[name] = {"tflops": flops / (min(ms) * 1e-3) / 1e12,
                     "tflops_median": flops / (statistics.median(ms) * 1e-3) / 1e12,
                     "flops_per_sm_per_clock": per_clk, "sm_mhz": c["sm_mhz"], "reasons": c["reasons"],
                     "iterations": iters, "ms": statistics.median(ms), "sms_used": used,
                     "tflops_all_sms_at_probe_clock": per_clk * sms * (c["sm_mhz"] or 0) * 1e6 / 1e12}
    return out


def gemm_peak(peaks, probe, step_mhz, sms):
    """Denominator of the GEMM roofline: the largest of the derived MXFP4 peak
    (measured cuBLAS bf16 x the nominal 4x ratio), the probe's event-timed rate and the
    probe's per-clock rate at the clock the timed GEMM ran at -- so the fraction is
    never flattered by a low denominator."""
    derived = peaks["bf16_tflops"] * FP4_OVER_BF16
    cands = {"derived_bf16x4": derived}
    if probe:
        p = probe["mxf4_pair"]
        cands["probe_event_timed"] = p["tflops"]
        if step_mhz:
            cands["probe_per_clock_at_step_clock"] = p["flops_per_sm_per_clock"] * sms * step_mhz * 1e6 / 1e12
    basis = max(cands, key=cands.get)
    return cands[basis], basis, cands


def time_gemm_pair(rfq, x, w, flush, iters):
    """RFQ GEMM and the same GEMM with the residual off (plain MXFP4), each alone after
    an L2 flush: the overhead the pages call negligible."""
    on = RfqStep(rfq, x, w, residual=True)
    off = RfqStep(rfq, x, w, residual=False)
    for st in (on, off):
        st.quantize_w()
        st.quantize_x()
    t_off = time_kernel(off.gemm, iters, flush)
    t_on = time_kernel(on.gemm, iters, flush)
    M, K, N = on.M, on.K, on.N
    rfq.check_device_error()
    return {"gemm_ms": statistics.mean(t_off), "gemm_ms_rfq": statistics.mean(t_on),
            "gemm_overhead": statistics.mean(t_on) / statistics.mean(t_off),
            "tflops_executed": 2.0 * M * N * K / (statistics.mean(t_off) * 1e-3) / 1e12,
            "tflops_executed_rfq": 4.0 * M * N * K / (statistics.mean(t_on) * 1e-3) / 1e12}


def concat_scales_along_k(s1, s2, rows: int, K: int):
    """The E8M0 scale arrays of two [rows][K] MX operands, in the block-scaled MMA layout
    (atoms of 128 rows x 4 blocks, 512 bytes, the block index fastest: the layout the
    quantizer writes and cuBLASLt's 32x4x4 swizzle), joined into the scales of the
    [rows][2K] operand [A1 | A2]: per 128-row tile, A1's K/128 atoms then A2's.  K must be
    a multiple of 128 (whole atoms).  Works on torch tensors and numpy arrays alike."""
    if K % 128:
        raise ValueError("K must be a multiple of 128")
    rt, kb4 = (rows + 127) // 128, K // 128
    a, b = s1.reshape(rt, kb4, 512), s2.reshape(rt, kb4, 512)
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return torch.cat([a, b], dim=1).reshape(-1)
    except ImportError:
        pass
    import numpy as np
    return np.concatenate([a, b], axis=1).reshape(-1)


def time_library_gemm(rfq, step, flush, iters):
    """A library comparator on the step's own quantized operands: cuBLASLt's MXFP4 GEMM
    (torch's scaled_mm, 1x32 E8M0 block scales in the 32x4x4 swizzled layout, which is
    the layout the quantizer writes) for the plain product QX.QW^T, and for RFQ as one
    GEMM over the operands concatenated along K ([QX | QR] . [QW | QW]^T, K' = 2K),
    beside rfq_gemm on the same buffers; and how many bf16 outputs agree bit for bit."""
    import torch
    try:
        import torch.nn.functional as F
        BW, SW = F.ScalingType.BlockWise1x32, F.SwizzleType.SWIZZLE_32_4_4
        fp4, e8 = torch.float4_e2m1fn_x2, torch.float8_e8m0fnu
    except AttributeError as e:
        return {"unavailable": f"torch has no MX scaled_mm: {e}"}
    M, N, K = step.M, step.N, step.K
    if K % 128:
        return {"unavailable": "K is not a multiple of 128"}
    Kb = K // 2

    def lib(a, b, sa, sb, kb):
        return F.scaled_mm(a.view(M, kb).view(fp4), b.view(N, kb).view(fp4).t(), sa.view(e8), BW, sb.view(e8), BW,
                           swizzle_a=SW, swizzle_b=SW, output_dtype=torch.bfloat16)

    a2 = torch.cat([step.qx_c.view(M, Kb), step.qr_c.view(M, Kb)], dim=1)
    b2 = torch.cat([step.qw_c.view(N, Kb), step.qw_c.view(N, Kb)], dim=1)
    sa2, sb2 = concat_scales_along_k(step.qx_s, step.qr_s, M, K), concat_scales_along_k(step.qw_s, step.qw_s, N, K)
    try:
        y_lib = lib(a2, b2, sa2, sb2, 2 * Kb)
    except Exception as e:   # no MXFP4 kernel for this device or build
        return {"unavailable": f"scaled_mm MXFP4 failed: {repr(e)[:160]}"}
    y_off = torch.empty_like(step.y)
    off = lambda: step.rfq.gemm(step.qx_c, step.qx_s, None, None, step.qw_c, step.qw_s, M, N, K, y_off)
    legs = {"rfq": step.gemm, "lib_rfq": lambda: lib(a2, b2, sa2, sb2, 2 * Kb),
            "off": off, "lib_off": lambda: lib(step.qx_c, step.qw_c, step.qx_s, step.qw_s, Kb)}
    for fn in legs.values():
        fn()
    torch.cuda.synchronize()
    # the four legs interleaved launch by launch (an L2 flush before each), so that a
    # change of clock or power state during the comparison affects all of them alike
    ev = {k: [] for k in legs}
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(iters):
            for k, fn in legs.items():
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                ev[k].append((a, b))
        torch.cuda.synchronize()
    t = {k: statistics.mean(a.elapsed_time(b) for a, b in v) for k, v in ev.items()}
    t_rfq, t_lib_rfq, t_off, t_lib_off = t["rfq"], t["lib_rfq"], t["off"], t["lib_off"]
    step.gemm()
    y_lib = lib(a2, b2, sa2, sb2, 2 * Kb)
    torch.cuda.synchronize()
    rfq.check_device_error()
    same = float((step.y.view(torch.int16) == y_lib.view(torch.int16)).float().mean())
    S = float(step.y.float().abs().max())
    diff = float((step.y.float() - y_lib.float()).abs().max()) / S
    del a2, b2, sa2, sb2, y_lib, y_off
    f = 2.0 * M * N * K
    return {"library": "cuBLASLt MXFP4 through torch.nn.functional.scaled_mm", "workload": f"M{M}_K{K}_N{N}",
            "rfq_gemm_ms": t_rfq, "library_rfq_as_2k_ms": t_lib_rfq,
            "rfq_gemm_off_ms": t_off, "library_plain_ms": t_lib_off,
            "rfq_speedup_vs_library": t_lib_rfq / t_rfq, "plain_speedup_vs_library": t_lib_off / t_off,
            "rfq_tflops_executed": 2 * f / (t_rfq * 1e-3) / 1e12,
            "library_rfq_tflops_executed": 2 * f / (t_lib_rfq * 1e-3) / 1e12,
            "bf16_outputs_identical": same, "max_abs_diff_over_S": diff,
            "timing": "the four legs interleaved, each launch after an L2 flush", "clocks": clk.summary()}


def time_ffn_step(rfq, wk, flush, world, fp4_peak, steps):
    """The LLM FFN up-projection step (4096 x 4096 -> 12288): the same three phases."""
    x, w = to_device_bf16(wk.x_bits), to_device_bf16(wk.w_bits)
    st = RfqStep(rfq, x, w, residual=True)
    ph = time_phases(st, steps, 3, flush, world)
    rfq.check_device_error()
    M, K, N = wk.M, wk.K, wk.N
    f = 4.0 * M * N * K
    g = statistics.mean(ph["gemm_ms"])
    out = {"workload": wk.name, "ms_per_step": statistics.mean(ph["step_ms"]),
           "tflops_step": f / (statistics.mean(ph["step_ms"]) * 1e-3) / 1e12,
           "gemm": {"ms": g, "tflops_executed": f / (g * 1e-3) / 1e12, "frac_fp4_peak": f / (g * 1e-3) / 1e12 / fp4_peak},
           "quantize_x_ms": statistics.mean(ph["quantize_x_ms"]), "quantize_w_ms": statistics.mean(ph["quantize_w_ms"])}
    out["rfq_off"] = time_gemm_pair(rfq, x, w, flush, 10)
    out["rfq_off"]["frac_fp4_peak"] = out["rfq_off"]["tflops_executed"] / fp4_peak
    return out, st


def time_quantize_bandwidth(rfq, rank, w, flush, hbm_peak, steps):
    """Quantize-only bandwidth workload (8192 x 4096, heavy-tailed).  Four input/output
    sets (X alone is 4 x 67 MB > L2) are rotated and launched back to back inside one
    event pair: the average launch duration.  The single launch after an L2 flush is
    reported beside it (it carries the fixed launch and ramp cost of an isolated kernel)."""
    import torch
    from block_scaled_gemm_rfq_b200 import workloads as wl
    qb = wl.quantize_bandwidth(seed=rank)
    xq0 = to_device_bf16(qb.x_bits)
    qsets = [RfqStep(rfq, xq0 if i == 0 else xq0.clone(), w[:8], residual=True) for i in range(4)]
    n_rot = max(40, steps)
    for st in qsets:
        st.quantize_x()
    flush()
    torch.cuda.synchronize()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_ev.record()
    for it in range(n_rot):
        qsets[it % 4].quantize_x()
    b_ev.record()
    torch.cuda.synchronize()
    q_ms = a_ev.elapsed_time(b_ev) / n_rot
    tq = time_kernel(qsets[0].quantize_x, max(20, steps // 2), flush)
    # the same measurement on a one-block launch of the same kernel (X 1 x 32): the fixed
    # cost that an event pair around a single launch after the flush carries for any kernel
    tiny = RfqStep(rfq, torch.zeros((1, 32), dtype=torch.bfloat16, device="cuda"),
                   torch.zeros((8, 32), dtype=torch.bfloat16, device="cuda"), residual=True)
    t_tiny = time_kernel(tiny.quantize_x, max(20, steps // 2), flush)
    rfq.check_device_error()
    qbytes = quantize_bytes(qb.M, qb.K, True)
    q_gbs = qbytes / (q_ms * 1e-3) / 1e9
    iso, fixed = statistics.mean(tq), statistics.mean(t_tiny)
    return {"workload": qb.name, "ms": q_ms, "bytes": qbytes, "gbs": q_gbs,
            "frac_hbm": q_gbs / hbm_peak, "launches": n_rot,
            "timing": "4 rotated input/output sets (268 MB of X) back to back, one event pair",
            "isolated_launch_ms": iso, "isolated_launch_gbs": qbytes / (iso * 1e-3) / 1e9,
            "isolated_launch_frac_hbm": qbytes / (iso * 1e-3) / 1e9 / hbm_peak,
            "one_block_launch_ms": fixed,
            "isolated_launch_beyond_one_block_frac_hbm": qbytes / ((iso - fixed) * 1e-3) / 1e9 / hbm_peak
            if iso > fixed else None}


def time_m_sweep(rfq, rank, flush, fp4_peak, hbm_peak):
    """rfq_linear at M in {16, ..., 16384}, K = N = 4096, RFQ and plain MXFP4: one call
    between events after an L2 flush ("isolated"), and calls replayed back to back from a
    CUDA graph over distinct weight/activation sets whose total exceeds L2 ("stream":
    layer after layer, every call reads its weight from HBM).  For M <= 64 the other
    path (quantize + GEMM, or the single-kernel layer) is timed beside it."""
    import torch
    from block_scaled_gemm_rfq_b200 import workloads as wl
    sweep = {}
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    for Ms in wl.SWEEP_M:
        sk = wl.m_sweep(Ms, seed=rank)
        xs, ws = to_device_bf16(sk.x_bits), to_device_bf16(sk.w_bits)
        row = {}
        n_sets = max(2, int(2 * 126e6 // (sk.N * sk.K * 0.53 + Ms * sk.K * 2)) + 1)
        for res in (True, False):
            qws = rfq.quantize_weight_alloc(ws)
            y = torch.empty((Ms, sk.N), dtype=torch.bfloat16, device="cuda")
            wsb = torch.empty(rfq.linear_workspace_bytes(Ms, sk.K, res), dtype=torch.uint8, device="cuda")
            t = time_kernel(lambda: rfq.linear(xs, qws.codes, qws.scales, sk.N, y, wsb, res), 20, flush)
            sets = [(xs.clone(), rfq.quantize_weight_alloc(ws),
                     torch.empty((Ms, sk.N), dtype=torch.bfloat16, device="cuda"),
                     torch.empty(rfq.linear_workspace_bytes(Ms, sk.K, res), dtype=torch.uint8, device="cuda"))
                    for _ in range(n_sets)]
            calls = [lambda a=a: rfq.linear(a[0], a[1].codes, a[1].scales, sk.N, a[2], a[3], res) for a in sets]
            t_stream = time_stream(calls, max(2, 400 // n_sets))
            f = (4.0 if res else 2.0) * Ms * sk.N * sk.K
            w_bytes = sk.N * sk.K // 2 + rfq.scales_bytes(sk.N, sk.K)
            io_bytes = Ms * sk.K * 2 + Ms * sk.N * 2
            # roofline time of the layer: the slower of the MMA work at the MXFP4 peak and
            # the weight + activation + output bytes at the HBM peak
            t_roof = max(f / (fp4_peak * 1e12), (w_bytes + io_bytes) / (hbm_peak * 1e9))
            cell = {"us": 1e3 * statistics.mean(t), "us_stream": 1e3 * t_stream, "stream_sets": n_sets,
                    "tflops_useful_stream": 2.0 * Ms * sk.N * sk.K / (t_stream * 1e-3) / 1e12,
                    "roofline_us": 1e6 * t_roof, "frac_roofline_stream": 1e6 * t_roof / (1e3 * t_stream),
                    "path": "fused" if Ms <= 32 else
                            ("quantize+split-K gemm" if Ms <= 256 and (1 if Ms <= 128 else 2) * ((sk.N + 255) // 256)
                             < sms // 2 else "quantize+gemm")}
            if Ms <= rfq.FUSED_MAX_M:
                s2 = RfqStep(rfq, xs, ws, residual=res)
                s2.quantize_w()
                y2 = torch.empty((Ms, sk.N), dtype=torch.bfloat16, device="cuda")
                if Ms <= 32:
                    # the two-kernel path (quantize, then GEMM) on the same problem
                    def other(a):
                        rfq.quantize_mxfp4(a[0], s2.qx_c, s2.qx_s, s2.qr_c, s2.qr_s)
                        rfq.gemm(s2.qx_c, s2.qx_s, s2.qr_c, s2.qr_s, a[1].codes, a[1].scales, Ms, sk.N, sk.K, y2)
                    name = "two_kernel_us_stream"
                else:
                    def other(a):   # the single-kernel layer, which rfq_linear leaves aside above 32 rows
                        rfq.linear_fused(a[0], a[1].codes, a[1].scales, sk.N, y2, res)
                    name = "fused_us_stream"
                cell[name] = 1e3 * time_stream([lambda a=a: other(a) for a in sets], max(2, 400 // n_sets))
                del s2
            del sets
            row["rfq" if res else "off"] = cell
        row["rfq_overhead_stream"] = row["rfq"]["us_stream"] / row["off"]["us_stream"]
        sweep[str(Ms)] = row
        rfq.check_device_error()
    return sweep


def run_cuda(args, rank, world, local):
    import numpy as np
    import torch

    import block_scaled_gemm_rfq_b200 as rfq
    from block_scaled_gemm_rfq_b200 import workloads as wl

    rfq.load_library()
    peaks = load_peaks()
    hbm_peak = peaks["hbm_gbs"]
    derived_fp4 = peaks["bf16_tflops"] * FP4_OVER_BF16
    flush = make_l2_flush(torch)
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count

    # ---- the headline step: the video-DiT FFN layer (the largest workload)
    wk = wl.dit_ffn(seed=rank)
    M, K, N = wk.M, wk.K, wk.N
    x, w = to_device_bf16(wk.x_bits), to_device_bf16(wk.w_bits)
    step = RfqStep(rfq, x, w, residual=True)
    flops = 4.0 * M * N * K

    with ClockSampler(local) as clk:
        ph = time_phases(step, args.steps, args.warmup, flush, world)
    rfq.check_device_error()
    clocks = clk.summary()
    step_ms_total = sum(ph["step_ms"])
    step_ms_max = max_over_ranks(step_ms_total, world)
    ms_per_step = step_ms_max / args.steps
    value = world * flops * args.steps / (step_ms_max * 1e-3) / 1e12

    gemm_ms = statistics.mean(ph["gemm_ms"])
    qx_ms = statistics.mean(ph["quantize_x_ms"])
    qw_ms = statistics.mean(ph["quantize_w_ms"])
    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12

    extra = {}
    # the tensor-core ceiling of the GEMM's own instruction shapes, measured here
    probe = measure_mma_peak(rfq, local) if not args.no_probe else None
    fp4_peak, peak_basis, peak_cands = gemm_peak(peaks, probe, clocks.get("sm_mhz"), sms)
    if probe:
        extra["mma_peak"] = probe
    extra["gemm_peak_candidates_tflops"] = peak_cands
    extra["rfq_off"] = time_gemm_pair(rfq, x, w, flush, max(5, min(10, args.steps)))
    extra["rfq_off"]["frac_fp4_peak"] = extra["rfq_off"]["tflops_executed"] / fp4_peak

    # ---- the other workloads of the benchmark, as extra keys
    ffn, _ = time_ffn_step(rfq, wl.ffn_up(seed=rank), flush, world, fp4_peak, max(10, min(20, args.steps)))
    extra["ffn_up"] = ffn
    extra["quantize_bandwidth"] = time_quantize_bandwidth(rfq, rank, w, flush, hbm_peak, args.steps)
    if not args.no_sweep:
        extra["m_sweep_rfq_linear"] = time_m_sweep(rfq, rank, flush, fp4_peak, hbm_peak)
    if not args.no_fidelity:
        # activation and output error of RFQ, plain MXFP4 and MXFP8 on 1024 rows of each workload
        extra["fidelity"] = run_fidelity(args)["fidelity"]
    if not args.no_training:
        # the backward-pass GEMMs and the MXFP8 comparator on the FFN workload
        fk = wl.ffn_up(seed=rank)
        fstep = RfqStep(rfq, to_device_bf16(fk.x_bits), to_device_bf16(fk.w_bits), residual=True)
        extra["training_ffn"] = time_training(rfq, fk, flush, fp4_peak, hbm_peak)
        extra["mxfp8_ffn"] = time_mxfp8(rfq, fk, flush, fp4_peak / 2.0, hbm_peak, fstep)
        del fstep

    # ---- end to end through the public API with host buffers: pinned X, W in; Y out.
    # Steps stream through two device buffer sets on three streams (host->device
    # copies, compute, device->host copies), so one step's copies overlap the
    # neighbouring steps' compute and opposite-direction copies; every step still
    # moves its own inputs in and its own result out inside the timed region.
    xh = torch.from_numpy(wk.x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    wh = torch.from_numpy(wk.w_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    e2e_steps = max(6, min(12, args.steps // 4))
    bufs = [step, RfqStep(rfq, torch.empty_like(x), torch.empty_like(w), residual=True)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()

    def e2e_run(n):
        done_cmp = [None, None]   # compute of the step that last used each buffer set
        done_out = [None, None]   # its device->host copy
        last = None
        for i in range(n):
            b = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if done_cmp[i % 2] is not None:
                    s_in.wait_event(done_cmp[i % 2])
                b.x.copy_(xh, non_blocking=True)
                b.w.copy_(wh, non_blocking=True)
                e_in = ev(); e_in.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(e_in)
                if done_out[i % 2] is not None:
                    s_cmp.wait_event(done_out[i % 2])
                b.run()
                e_c = ev(); e_c.record(s_cmp)
                done_cmp[i % 2] = e_c
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_c)
                yh[i % 2].copy_(b.y, non_blocking=True)
                e_o = ev(); e_o.record(s_out)
                done_out[i % 2] = e_o
                last = e_o
        return last

    torch.cuda.synchronize()
    e2e_run(2)
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b_end = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    last = e2e_run(e2e_steps)
    s_in.wait_event(last)
    b_end.record(s_in)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b_end), world) / e2e_steps

    def e2e_serial():   # the same, one step at a time on one stream (no overlap), for reference
        x.copy_(xh, non_blocking=True)
        w.copy_(wh, non_blocking=True)
        step.run()
        yh[0].copy_(step.y, non_blocking=True)
    a2, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a2.record()
    for _ in range(3):
        e2e_serial()
    b2.record()
    torch.cuda.synchronize()
    e2e_serial_ms = max_over_ranks(a2.elapsed_time(b2), world) / 3
    if not np.array_equal(yh[0].view(torch.int16).numpy()[:4], yh[1].view(torch.int16).numpy()[:4]):
        raise RuntimeError("pipelined and serial end-to-end steps disagree")
    rfq.check_device_error()
    if not args.no_library:
        # last: nothing of this run is timed after the library's kernels have run
        extra["library_gemm"] = time_library_gemm(rfq, step, flush, max(5, min(10, args.steps)))

    result = {
        "metric": "RFQ W4A4 GEMM TFLOPS (% MXFP4 peak); fused RFQ quantize GB/s (% HBM)",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "mxfp4 (e2m1 x e2m1, e8m0 scales), fp32 accumulate, bf16 out",
        "data": "synthetic (seeded numpy: X Laplace(0,1) + 8 outlier channels x80; W N(0,0.015))",
        "config": {"workload": wk.name, "M": M, "K": K, "N": N, "rfq": True, "y": "bf16",
                   "step": "rfq_quantize_weight + rfq_quantize_mxfp4 (X, residual) + rfq_gemm",
                   "l2": "flushed between steps (256 MiB written then read back, outside the step events); "
                         "the step's operands (1.5 GB) exceed L2 anyway",
                   "parallelism": f"replicas x{world}"},
        "gemm": {"ms": gemm_ms, "tflops_executed": gemm_tflops, "tflops_useful": gemm_tflops / 2,
                 "frac_fp4_peak": gemm_tflops / fp4_peak, "frac_derived_peak": gemm_tflops / derived_fp4},
        "quantize_x": {"ms": qx_ms, "gbs": quantize_bytes(M, K, True) / (qx_ms * 1e-3) / 1e9,
                       "frac_hbm": quantize_bytes(M, K, True) / (qx_ms * 1e-3) / 1e9 / hbm_peak},
        "quantize_w": {"ms": qw_ms, "gbs": quantize_bytes(N, K, False) / (qw_ms * 1e-3) / 1e9,
                       "frac_hbm": quantize_bytes(N, K, False) / (qw_ms * 1e-3) / 1e9 / hbm_peak},
        "roofline": {"bound": "tensor", "kernel": "rfq_gemm_kernel<pair, residual, bf16>", "achieved": gemm_tflops,
                     "peak": fp4_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                     "peak_basis": {"derived_bf16x4": f"{peaks['source']} bf16_tflops {peaks['bf16_tflops']} x "
                                                      f"{FP4_OVER_BF16} (nominal MXFP4:bf16 ratio), burst",
                                    "probe_event_timed": "rfq_mma_rate_probe kind::mxf4 CTA pairs, events, this run",
                                    "probe_per_clock_at_step_clock": "probe flops per SM clock x SMs x the step's "
                                                                     "median SM clock"}[peak_basis],
                     "traffic": NCU_TRAFFIC_BYTES.get("gemm_dit_rfq_bf16"), "traffic_unit": "bytes"},
        "roofline_quantize": {"bound": "hbm", "kernel": "rfq_quantize_kernel<residual>",
                              "achieved": extra["quantize_bandwidth"]["gbs"], "peak": hbm_peak, "unit": "GB/s",
                              "frac": extra["quantize_bandwidth"]["gbs"] / hbm_peak,
                              "peak_basis": f"{peaks['source']} hbm_gbs",
                              "traffic": NCU_TRAFFIC_BYTES.get("quantize_8192x4096_rfq"), "traffic_unit": "bytes"},
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": int(xh.numel() * 2 + wh.numel() * 2),
                "d2h_bytes_per_step": int(yh[0].numel() * 2),
                "timing": "steps streamed: H2D, compute and D2H on three streams over two buffer sets",
                "serial_ms_per_step": e2e_serial_ms,
                "serial_value": world * flops / (e2e_serial_ms * 1e-3) / 1e12},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
        "gpu": torch.cuda.get_device_name(),
    }
    result.update(extra)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:   # the CPU baseline is a 1-GPU figure
        result["cpu_baseline"] = cpu_baseline(wk, args.cpu_seconds)
    return result


# ----------------------------------------------------------------------------- the oracle on the host cores
def cpu_baseline(wk, budget_s: float):
    """The CPU oracle, as it stands, on a bounded sample of the same step, scaled to the
    whole step: quantize n_w rows of W and m rows of X (with residual) in the C oracle
    (rows spread over the host cores), and the float64 reference GEMM of those m rows
    against the n_w weight rows (numpy BLAS); each part is extrapolated by the rows (and,
    for the GEMM, columns) it covers."""
    import numpy as np

    import oracle
    oracle.build()
    M, K, N = wk.M, wk.K, wk.N
    m = min(M, 256)
    nw = min(N, 1024)
    t_start = time.perf_counter()
    t0 = time.perf_counter()
    qw = oracle.quantize_bf16(wk.w_bits[:nw], residual=False)
    t_qw_s = time.perf_counter() - t0
    t0 = time.perf_counter()
    qa = oracle.quantize_bf16(wk.x_bits[:m], residual=True)
    t_qx_s = time.perf_counter() - t0
    A, B = oracle.rfq_operands(qa, qw, True)
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.gemm_blas(A, B)
        reps += 1
        if time.perf_counter() - t0 > min(5.0, budget_s / 3):
            break
    t_gemm_s = (time.perf_counter() - t0) / reps
    sample_s = time.perf_counter() - t_start
    t_qw, t_qx = t_qw_s * (N / nw), t_qx_s * (M / m)
    t_gemm = t_gemm_s * (M / m) * (N / nw)
    total = t_qw + t_qx + t_gemm
    cores = len(os.sched_getaffinity(0))
    threads = oracle.threads()
    return {"value": 4.0 * M * N * K / total / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "threads": {"quantize_c_openmp": threads, "gemm_f64_blas": cores},
            "sample_seconds_measured": sample_s,
            "seconds_per_step_extrapolated": total,
            "parts_s_extrapolated": {"quantize_w": t_qw, "quantize_x": t_qx, "gemm_f64": t_gemm},
            "parts_s_measured": {"quantize_w": t_qw_s, "quantize_x": t_qx_s, "gemm_f64_one_rep": t_gemm_s,
                                 "gemm_reps": reps},
            "sample": f"oracle quantize of W rows [0,{nw}) and X rows [0,{m}) (C, OpenMP over rows, {threads} "
                      f"threads), float64 numpy matmul of those X rows x W rows (BLAS, up to {cores} threads), "
                      f"each part scaled by rows to the full {M}x{K}x{N} step"}


def run_reference(args):
    """--impl reference: the oracle, timed on the host cores on this workload's bounded
    samples, reported in the same metric/unit.  ``ms_per_step`` is the host time one
    step's sample actually took; the full-step time it extrapolates to is reported
    beside it as ``extrapolated_ms_per_full_step``."""
    from block_scaled_gemm_rfq_b200 import workloads as wl
    wk = wl.dit_ffn(seed=0)
    # Each step's sample shrinks with the number of steps so that the whole run stays
    # near REFERENCE_RUN_SECONDS of host time (the GEMM part of a sample is timed over
    # a third of its budget; the quantizer rows are fixed, well under a second).
    budget = max(0.3, min(args.cpu_seconds, REFERENCE_RUN_SECONDS / max(1, args.steps + args.warmup)))
    samples = []
    for _ in range(args.warmup):
        cpu_baseline(wk, budget)
    for _ in range(args.steps):
        samples.append(cpu_baseline(wk, budget))
    v = statistics.mean(s["value"] for s in samples)
    cb = dict(samples[-1])
    cb["value"] = v
    return {
        "impl": "reference",
        "metric": "RFQ W4A4 GEMM TFLOPS (% MXFP4 peak); fused RFQ quantize GB/s (% HBM)",
        "value": v, "unit": "TFLOP/s", "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(s["sample_seconds_measured"] for s in samples),
        "ms_per_step_is": "host time of one step's bounded sample (measured)",
        "extrapolated_ms_per_full_step": 1e3 * statistics.mean(s["seconds_per_step_extrapolated"] for s in samples),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (same seeded generator as the CUDA arm)",
        "config": {"workload": wk.name, "M": wk.M, "K": wk.K, "N": wk.N, "rfq": True, "y": "f64"},
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_fidelity(args):
    """--fidelity: the paper's central claim measured on the synthetic workloads with
    this library's kernels (RFQ paper, abstract and section 1: activation
    quantization dominates the FP4 error and the residual path recovers it).

    Activation fidelity: a GEMM against the K x K identity (which MXFP4 represents
    exactly) returns the dequantized activation DQ(QX) [+ DQ(QR)] in fp32, so
    ||X - X_hat|| / ||X|| is measured with RFQ on and off.  Output fidelity:
    ||Y - X W^T|| / ||X W^T|| against an fp32 product of the bf16 inputs."""
    import numpy as np
    import torch

    import block_scaled_gemm_rfq_b200 as rfq
    from block_scaled_gemm_rfq_b200 import workloads as wl
    rfq.load_library()
    report = {}
    cases = [("tiny", wl.tiny(0)), ("quantize_bandwidth", wl.quantize_bandwidth(0, M=1024)),
             ("ffn_up", wl.ffn_up(0, M=1024)), ("dit_ffn", wl.dit_ffn(0, M=1024))]
    for name, wk in cases:
        x = to_device_bf16(wk.x_bits)
        M, K = x.shape
        eye = torch.eye(K, dtype=torch.bfloat16, device="cuda")
        qe = rfq.quantize_weight_alloc(eye)
        xf = x.float()
        row = {"workload": wk.name, "M": M, "K": K}
        for res in (True, False):
            qa = rfq.quantize_mxfp4_alloc(x, residual=res)
            xhat = rfq.gemm_alloc(qa, qe, out_dtype=torch.float32, use_residual=res)
            row[f"x_rel_err_{'rfq' if res else 'mxfp4'}"] = float(torch.linalg.norm(xhat - xf) / torch.linalg.norm(xf))
        # MXFP8 comparator (identity exact in MXFP8 too)
        qe8 = rfq.quantize_mxfp8_alloc(eye)
        xhat8 = rfq.gemm_mxfp8_alloc(rfq.quantize_mxfp8_alloc(x), qe8, out_dtype=torch.float32)
        row["x_rel_err_mxfp8"] = float(torch.linalg.norm(xhat8 - xf) / torch.linalg.norm(xf))
        if wk.w_bits is not None:
            w = to_device_bf16(wk.w_bits)
            yref = xf @ w.float().t()
            qw = rfq.quantize_weight_alloc(w)
            for res in (True, False):
                qa = rfq.quantize_mxfp4_alloc(x, residual=res)
                y = rfq.gemm_alloc(qa, qw, out_dtype=torch.float32, use_residual=res)
                row[f"y_rel_err_{'rfq' if res else 'mxfp4'}"] = float(torch.linalg.norm(y - yref) / torch.linalg.norm(yref))
            y8 = rfq.gemm_mxfp8_alloc(rfq.quantize_mxfp8_alloc(x), rfq.quantize_mxfp8_alloc(w), out_dtype=torch.float32)
            row["y_rel_err_mxfp8"] = float(torch.linalg.norm(y8 - yref) / torch.linalg.norm(yref))
        rfq.check_device_error()
        report[name] = row
    return {"fidelity": report}


def run_single_kernel(args):
    """--kernel quantize|gemm|linear: time one kernel on a chosen shape (for sweeps and
    profiles); prints one JSON line with per-launch times."""
    import numpy as np
    import torch

    import block_scaled_gemm_rfq_b200 as rfq
    from block_scaled_gemm_rfq_b200 import workloads as wl
    rfq.load_library()
    if args.kernel == "probe":
        # the tensor-core rate of the GEMM's MMA shapes (rfq_mma_rate_probe), --steps launches each
        dev = torch.cuda.current_device()
        print(json.dumps({"kernel": "probe", "mma_peak": measure_mma_peak(rfq, dev, launches=max(1, args.steps))}))
        return
    M, K, N = args.M, args.K, args.N
    x = to_device_bf16(wl.random_matrix(M, K, seed=1, scale=2.0))
    w = to_device_bf16(wl.random_matrix(N, K, seed=2, scale=0.05)) if not args.kernel.startswith("quantize") \
        else x[:8]
    step = RfqStep(rfq, x, w, residual=not args.no_rfq)
    step.quantize_w()
    step.quantize_x()
    fused = lambda: rfq.linear_fused(x, step.qw_c, step.qw_s, N, step.y, not args.no_rfq)
    fn = {"quantize": step.quantize_x, "gemm": step.gemm, "linear": step.run,
          "two-kernel": lambda: (step.quantize_x(), step.gemm()), "fused": fused}.get(args.kernel)
    if args.kernel == "quantize-t":
        # the operand of X^T (blocks along M), as for the weight-gradient GEMM
        qt = rfq.quantize_mxfp4_t_alloc(x, residual=not args.no_rfq)
        fn = lambda: rfq.quantize_mxfp4_t(x, qt.codes, qt.scales, qt.r_codes, qt.r_scales)
    elif args.kernel == "gemm-yt":
        yt = torch.empty((N, M), dtype=torch.bfloat16, device="cuda")
        fn = lambda: rfq.gemm_yt(step.qx_c, step.qx_s, step.qr_c, step.qr_s, step.qw_c, step.qw_s, M, N, K, yt)
    elif args.kernel in ("quantize-mxfp8", "gemm-mxfp8"):
        q8a, q8w = rfq.quantize_mxfp8_alloc(x), rfq.quantize_mxfp8_alloc(w)
        fn = (lambda: rfq.quantize_mxfp8(x, q8a.codes, q8a.scales)) if args.kernel == "quantize-mxfp8" else \
            (lambda: rfq.gemm_mxfp8(q8a.codes, q8a.scales, q8w.codes, q8w.scales, M, N, K, step.y))
    rfq.debug_fused_split(args.split)
    t = time_kernel(fn, args.steps, make_l2_flush(torch))
    rfq.debug_fused_split(0)
    rfq.check_device_error()
    ms = statistics.mean(t)
    out = {"kernel": args.kernel, "M": M, "K": K, "N": N, "rfq": not args.no_rfq, "iters": args.steps,
           "split": args.split,
           "ms_mean": ms, "ms_min": min(t)}
    if args.kernel in ("quantize", "quantize-t"):
        out["gbs"] = quantize_bytes(M, K, not args.no_rfq) / (ms * 1e-3) / 1e9
    elif args.kernel == "quantize-mxfp8":
        out["gbs"] = (M * K * 3 + M * K // 32) / (ms * 1e-3) / 1e9
    elif args.kernel == "gemm-mxfp8":
        out["tflops"] = 2.0 * M * N * K / (ms * 1e-3) / 1e12
    else:
        out["tflops_executed"] = (2.0 if args.no_rfq else 4.0) * M * N * K / (ms * 1e-3) / 1e12
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--all-configs", action="store_true",
                    help="accepted for compatibility: every workload is timed by default")
    ap.add_argument("--no-training", action="store_true",
                    help="skip the training-side GEMMs and the MXFP8 comparator on the FFN workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-probe", action="store_true", help="skip the tensor-core rate probe")
    ap.add_argument("--no-sweep", action="store_true", help="skip the rfq_linear M sweep")
    ap.add_argument("--no-fidelity", action="store_true", help="skip the activation/output fidelity report")
    ap.add_argument("--no-library", action="store_true",
                    help="skip the library comparator (cuBLASLt MXFP4 on the step's own operands)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--kernel", choices=["quantize", "gemm", "linear", "two-kernel", "fused", "quantize-t", "gemm-yt",
                                         "quantize-mxfp8", "gemm-mxfp8", "probe"], default=None,
                    help="time one kernel on --M/--N/--K instead of the benchmark step (linear = quantize W "
                         "+ quantize X + GEMM; two-kernel = quantize X + GEMM; fused = rfq_linear_fused)")
    ap.add_argument("--split", type=int, default=0, help="with --kernel fused: K split (0 = automatic)")
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--N", type=int, default=12288)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--no-rfq", action="store_true", help="with --kernel: residual path off")
    ap.add_argument("--fidelity", action="store_true",
                    help="report activation and output error of RFQ vs plain MXFP4 on the workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.kernel:
        run_single_kernel(args)
        return
    if args.fidelity:
        print(json.dumps(run_fidelity(args)))
        return

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        print(json.dumps(run_reference(args)))
        return

    rank, world, local = dist_setup(args.gpus)
    try:
        res = run_cuda(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res))
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
